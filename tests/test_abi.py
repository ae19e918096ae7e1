"""The C-ABI library loads and exports every entry point include/smla.h declares;
host-side argument checks reject bad calls before anything is launched.
No kernel runs here (no GPU needed)."""
import ctypes
import os
import re

import pytest

import sparse_mla_decoding_b200 as smla

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    out = set()
    for name in os.listdir(os.path.join(ROOT, "include")):
        if not name.endswith(".h"):
            continue
        with open(os.path.join(ROOT, "include", name)) as f:
            text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
        out.update(re.findall(r"\b(smla_[a-z0-9_]+)\s*\(", text))
    return sorted(out)


def test_library_exports_every_declared_symbol():
    syms = declared_symbols()
    assert len(syms) >= 10
    L = smla.lib()
    for s in syms:
        assert hasattr(L, s), f"{s} declared in include/ but not exported"


def test_status_strings_and_version():
    L = smla.lib()
    assert L.smla_status_string(0) == b"SMLA_OK"
    assert L.smla_status_string(4) == b"SMLA_ERR_DEVICE_TIMEOUT"
    assert L.smla_status_string(99) == b"SMLA_UNKNOWN_STATUS"
    assert L.smla_version() == 102
    assert L.smla_last_cuda_error() == 0
    assert L.smla_last_cuda_error_string() == b"cudaSuccess"


def test_head_pair_form_setting_round_trips():
    # host-side only: the setting is read at the next decode launch
    prev = smla.set_head_pair_form(True)
    try:
        assert smla.set_head_pair_form(False) is True
        assert smla.set_head_pair_form(False) is False
    finally:
        smla.set_head_pair_form(prev)


def test_workspace_bytes_arithmetic():
    L = smla.lib()
    # header 256 + (R + P) * h * 512 * 4 (256-rounded) + (R + P) * h * 4 (256-rounded)
    R, P, h = 64, 74, 128
    o_bytes = (R + P) * h * 512 * 4
    l_bytes = (R + P) * h * 4
    rnd = lambda x: (x + 255) // 256 * 256
    assert L.smla_workspace_bytes(64, 1, 128, 2048, 74) == 256 + rnd(o_bytes) + rnd(l_bytes)
    assert L.smla_workspace_bytes(3, 2, 16, 64, 5) == 256 + rnd(11 * 16 * 2048) + rnd(11 * 16 * 4)
    assert L.smla_workspace_bytes(2, 1, 48, 64, 8) == 0       # unsupported h_q
    assert L.smla_workspace_bytes(2, 0, 16, 64, 8) == 0       # s_q < 1
    assert L.smla_workspace_bytes(2, 1, 16, 0, 8) == 0        # topk < 1


def test_argument_checks_return_before_launch():
    L = smla.lib()
    fake = ctypes.c_void_p(0x10000)          # never dereferenced: calls fail validation first
    # null outputs
    assert L.smla_get_mla_metadata(None, 2, 1, 64, 16, 8, None, None, None) == 1
    # unsupported head count
    assert L.smla_get_mla_metadata(None, 2, 1, 64, 48, 8, fake, fake, None) == 2
    # misaligned sched_meta
    assert L.smla_get_mla_metadata(None, 2, 1, 64, 16, 8, ctypes.c_void_p(0x10004), fake, None) == 1
    # bad sizes
    assert L.smla_get_mla_metadata(None, 2, 0, 64, 16, 8, fake, fake, None) == 1
    assert L.smla_get_mla_metadata(None, 2, 1, 0, 16, 8, fake, fake, None) == 1
    assert L.smla_get_mla_metadata(None, 2, 1, 64, 16, 0, fake, fake, None) == 1
    args = [fake, fake, 8, fake, 4, fake, fake, fake, fake, 8, -1.0, 2, 1, 16, 64, fake, fake, fake, 1 << 30, None]
    bad = list(args); bad[13] = 96                                   # h_q
    assert L.smla_flash_mla_with_kvcache(*bad) == 2
    bad = list(args); bad[0] = None                                  # q
    assert L.smla_flash_mla_with_kvcache(*bad) == 1
    bad = list(args); bad[17] = ctypes.c_void_p(0x10010)             # workspace not 256-aligned
    assert L.smla_flash_mla_with_kvcache(*bad) == 1
    bad = list(args); bad[18] = 16                                   # workspace too small
    assert L.smla_flash_mla_with_kvcache(*bad) == 1
    bad = list(args); bad[14] = 0                                    # topk
    assert L.smla_flash_mla_with_kvcache(*bad) == 1
    bad = list(args); bad[0] = ctypes.c_void_p(0x10002)              # q misaligned
    assert L.smla_flash_mla_with_kvcache(*bad) == 1
    ok_empty = list(args); ok_empty[11] = 0                          # batch 0: nothing to do
    assert L.smla_flash_mla_with_kvcache(*ok_empty) == 0
    assert L.smla_quantize_kv(None, None, 4, None, None, 4, None) == 1
    assert L.smla_quantize_kv(fake, fake, 8, None, fake, 4, None) == 1   # rows too few
    assert L.smla_quantize_kv(fake, fake, 0, None, fake, 0, None) == 0
    assert L.smla_get_device_status(None, None, None, None) == 1
    assert L.smla_reset_device_status(None, None) == 1
    assert L.smla_selftest_bounded_wait(fake, 0, None) == 1
    assert L.smla_selftest_bounded_wait(None, 1000, None) == 1


def test_sparse_fwd_workspace_and_argument_checks():
    L = smla.lib()
    fake = ctypes.c_void_p(0x10000)
    # workspace = decode workspace (batch 1) + scheduler tables + length + block table, each 256-rounded
    s_q, h_q, s_kv, topk, P = 130, 64, 1000, 200, 8
    dec = L.smla_workspace_bytes(1, s_q, h_q, topk, P)
    up = lambda x: (x + 255) // 256 * 256
    nb = (s_kv + 63) // 64
    expect = up(dec) + up(P * 8 * 4) + up((s_q + 1) * 4) + 256 + up(nb * 4)
    assert L.smla_sparse_fwd_workspace_bytes(s_q, h_q, s_kv, topk, P) == expect
    assert L.smla_sparse_fwd_workspace_bytes(s_q, 48, s_kv, topk, P) == 0
    assert L.smla_sparse_fwd_workspace_bytes(s_q, h_q, 0, topk, P) == 0
    assert L.smla_sparse_fwd_workspace_bytes(s_q, h_q, (2 ** 31 - 1) // 64 * 64 + 1, topk, P) == 0
    args = [fake, fake, s_kv, fake, s_q, h_q, topk, P, -1.0, fake, fake, fake, 1 << 30, None]
    bad = list(args); bad[5] = 96                                    # h_q
    assert L.smla_flash_mla_sparse_fwd(*bad) == 2
    bad = list(args); bad[0] = None                                  # q
    assert L.smla_flash_mla_sparse_fwd(*bad) == 1
    bad = list(args); bad[2] = 0                                     # s_kv
    assert L.smla_flash_mla_sparse_fwd(*bad) == 1
    bad = list(args); bad[11] = ctypes.c_void_p(0x10010)             # workspace not 256-aligned
    assert L.smla_flash_mla_sparse_fwd(*bad) == 1
    bad = list(args); bad[12] = expect - 1                           # workspace too small
    assert L.smla_flash_mla_sparse_fwd(*bad) == 1
    bad = list(args); bad[6] = 0                                     # topk
    assert L.smla_flash_mla_sparse_fwd(*bad) == 1


def test_python_binding_shape_checks():
    import torch
    with pytest.raises(ValueError):
        smla.get_mla_metadata(torch.zeros(3, dtype=torch.int32), 64, 16, 8)     # not on CUDA
    q = torch.zeros((4, 16, 576), dtype=torch.bfloat16)
    kv = torch.zeros((10, 656), dtype=torch.uint8)
    idx = torch.zeros((4, 1, 8), dtype=torch.int32)
    with pytest.raises(ValueError):
        smla.flash_mla_sparse_fwd(q, kv, idx)                                  # not on CUDA
    with pytest.raises(ValueError):
        smla.flash_mla_with_kvcache(q[None], kv.view(1, 10, 656), idx.view(1, 4, 8), torch.zeros(1, dtype=torch.int32),
                                    idx.view(1, 4, 8), torch.zeros((8, 8), dtype=torch.int32),
                                    torch.zeros(5, dtype=torch.int32))           # not on CUDA
