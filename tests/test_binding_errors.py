"""Host-side error reporting of the Python binding (no GPU needed).

The binding's status names must cover every code the C header declares, and
the device-status check that flash_mla_with_kvcache(check_device_status=True)
performs must turn set flags into an SmlaError that names them.
"""
import os
import re

import pytest

import sparse_mla_decoding_b200 as smla

HERE = os.path.dirname(os.path.abspath(__file__))


def _header_codes():
    text = open(os.path.join(HERE, "..", "include", "smla.h")).read()
    enum = text[text.index("typedef enum {"):text.index("} smla_status;")]
    return {int(v): k for k, v in re.findall(r"(SMLA_\w+)\s*=\s*(\d+)", enum)}


def test_status_names_cover_the_header():
    assert _header_codes() == smla.STATUS_NAMES


def test_status_flag_bits_match_the_kernels():
    text = open(os.path.join(HERE, "..", "sparse_mla_decoding_b200", "csrc", "sm100.cuh")).read()
    bits = {1 << int(b) for b in re.findall(r"kStatus\w+ = 1u << (\d+)", text)}
    assert bits == set(smla.STATUS_FLAGS)


def test_set_flags_raise(monkeypatch):
    monkeypatch.setattr(smla, "get_device_status", lambda ws: (1, 2))
    with pytest.raises(smla.SmlaError) as e:
        smla._raise_on_flags(object(), "smla_flash_mla_with_kvcache")
    assert e.value.status == 1
    assert "block table" in str(e.value)


def test_clear_flags_do_not_raise(monkeypatch):
    monkeypatch.setattr(smla, "get_device_status", lambda ws: (0, 0))
    smla._raise_on_flags(object(), "smla_flash_mla_with_kvcache")


def test_timeout_flag_maps_to_timeout_status(monkeypatch):
    monkeypatch.setattr(smla, "get_device_status", lambda ws: (4, 1))
    with pytest.raises(smla.SmlaError) as e:
        smla._raise_on_flags(object(), "x")
    assert e.value.status == 4 and "wait gave up" in str(e.value)
