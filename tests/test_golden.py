"""The code against numbers the pages print (tests/golden/pages_worked_values.txt).

Each value in the fixture cites its page and section; this test checks the
oracle's row layout and the metric's FLOP count against them.
"""
import os

import numpy as np
import torch

import bench
import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def _values():
    out = {}
    with open(os.path.join(HERE, "golden", "pages_worked_values.txt"), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = (x.strip() for x in line.split("="))
            out[k] = float(v) if "." in v else int(v)
    return out


def _bits(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_row_layout_matches_the_pages():
    g = _values()
    assert g["quantized_bytes"] + g["scale_bytes"] + g["rope_bytes"] == g["kv_row_bytes"]
    assert g["quant_dims"] + g["rope_dims"] == g["qk_dims"]
    rng = np.random.default_rng(3)
    lat = _bits(rng.standard_normal(g["quant_dims"]))
    rope = _bits(rng.standard_normal(g["rope_dims"]))
    row = oracle.quantize_token(lat, rope)
    assert row.shape == (g["kv_row_bytes"],)
    # one float32 scale per 1 x 128 tile, stored after the 512 quantised bytes
    n_tiles = g["quant_dims"] // g["quant_tile"]
    assert n_tiles * 4 == g["scale_bytes"]
    scales = row[g["quantized_bytes"]:g["quantized_bytes"] + g["scale_bytes"]].view("<f4")
    lat_f = oracle.bf16_bits_to_f64(lat).reshape(n_tiles, g["quant_tile"])
    assert np.array_equal(scales, (np.abs(lat_f).max(axis=1).astype(np.float32) / np.float32(448.0)))
    # the RoPE part is the input bf16 values, unquantised
    assert np.array_equal(row[g["quantized_bytes"] + g["scale_bytes"]:].view("<u2"), rope)
    # the dequantised key is 576 wide
    assert oracle.dequantize_row(row).shape == (g["qk_dims"],)


def test_bf16_cache_size_example():
    g = _values()
    bytes_ = g["qk_dims"] * 2 * g["bf16_kv_layers"] * g["bf16_kv_tokens"]
    assert round(bytes_ / 2 ** 30, 2) == g["bf16_kv_gib"]
    # the FP8 row is a little over half of the 1152-byte BF16 row
    assert 0.5 < g["kv_row_bytes"] / (g["qk_dims"] * 2) < 0.6


def test_metric_flop_count_matches_the_mma_budget_example():
    g = _values()
    flop = bench.step_flops(g["mma_heads"], np.array([[1]]))       # one valid slot of one query token
    assert flop == g["mma_heads"] * (g["qk_dims"] + g["quant_dims"]) * 2
    assert round(flop / g["mma_flop_per_clk"]) == g["mma_cycles"]
