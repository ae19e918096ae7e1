"""Pins for the float64 CPU oracle, checked against things other than itself.

Each check below is a closed form, a library special case, a brute force, or
an invariant that the definition of the method fixes:
  * e4m3 decode: the format's bit layout (closed forms) and torch.float8_e4m3fn
  * e4m3 encode: round trips over every finite code, ties-to-even midpoints,
    saturation, and torch's round-to-nearest-even cast
  * bf16 rounding: torch's float32 -> bfloat16 cast
  * quantiser: the e4m3 round-trip error bound; exactness on the e4m3 grid;
    the vectorised bulk quantiser bit-exact against the scalar one
  * attention: an independent numpy textbook softmax attention (quantisation
    disabled, and on the exact e4m3 grid through the full paged path),
    weights summing to 1, invariance under permuting the slots,
    split-then-combine equal to a single pass, the all-invalid case, and the
    closed forms for one valid slot and for n identical rows
  * paging: gathering through a permuted block table equals gathering from a
    logically ordered cache; poisoned rows past the length are never read
  * sparse prefill (flat cache): textbook attention over the rows each query
    token names, with out-of-range and negative indices skipped
  * scheduler: brute-force enumeration of the tile ranges
"""
import math

import numpy as np
import pytest
import torch

import oracle

DQK, DV = 576, 512


# --------------------------------------------------------------------------
# e4m3
# --------------------------------------------------------------------------

def test_e4m3_decode_closed_forms():
    assert oracle.e4m3_decode(0x00) == 0.0
    assert math.copysign(1.0, oracle.e4m3_decode(0x80)) == -1.0
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9            # smallest subnormal
    assert oracle.e4m3_decode(0x07) == 7 * 2.0 ** -9        # largest subnormal
    assert oracle.e4m3_decode(0x08) == 2.0 ** -6            # smallest normal
    assert oracle.e4m3_decode(0x38) == 1.0                  # exponent field 7 = bias
    assert oracle.e4m3_decode(0x3C) == 1.5
    assert oracle.e4m3_decode(0x7E) == 448.0                # largest finite
    assert oracle.e4m3_decode(0xFE) == -448.0
    assert math.isnan(oracle.e4m3_decode(0x7F))
    assert math.isnan(oracle.e4m3_decode(0xFF))
    assert oracle.e4m3_decode(0x77) == 240.0                # 1.875 * 2^7


def test_e4m3_decode_matches_torch_all_codes():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = np.array([oracle.e4m3_decode(c) for c in range(256)])
    nan = np.isnan(ref)
    assert (np.isnan(mine) == nan).all()
    assert np.array_equal(mine[~nan], ref[~nan])


def test_e4m3_encode_round_trip_every_finite_code():
    for c in range(256):
        v = oracle.e4m3_decode(c)
        if math.isnan(v):
            continue
        assert oracle.e4m3_encode(np.float32(v)) == c, hex(c)


def test_e4m3_encode_ties_to_even_and_saturation():
    # midpoint between 1.0 (0x38, even mantissa) and 1.125 (0x39) -> 1.0
    assert oracle.e4m3_encode(1.0625) == 0x38
    # midpoint between 1.125 (0x39) and 1.25 (0x3A, even) -> 1.25
    assert oracle.e4m3_encode(1.1875) == 0x3A
    # subnormal midpoint 1.5 * 2^-9 between codes 1 and 2 -> 2 (even)
    assert oracle.e4m3_encode(1.5 * 2.0 ** -9) == 0x02
    # 0.5 * 2^-9 is a tie between 0 and the smallest subnormal -> 0
    assert oracle.e4m3_encode(0.5 * 2.0 ** -9) == 0x00
    # tie across the subnormal/normal boundary: 7.5 * 2^-9 -> 8 * 2^-9 = 2^-6
    assert oracle.e4m3_encode(7.5 * 2.0 ** -9) == 0x08
    assert oracle.e4m3_encode(448.0) == 0x7E
    assert oracle.e4m3_encode(460.0) == 0x7E
    assert oracle.e4m3_encode(1e30) == 0x7E
    assert oracle.e4m3_encode(-1e30) == 0xFE
    assert oracle.e4m3_encode(float("nan")) & 0x7F == 0x7F
    assert oracle.e4m3_encode(-0.0) == 0x80


def test_e4m3_encode_matches_torch_cast():
    rng = np.random.default_rng(11)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(50.0),
        (rng.standard_normal(5000) * 2.0 ** -8).astype(np.float32),
        rng.uniform(-448, 448, 5000).astype(np.float32),
    ])
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = np.array([oracle.e4m3_encode(v) for v in x], dtype=np.uint8)
    assert np.array_equal(mine, ref)


# --------------------------------------------------------------------------
# bf16
# --------------------------------------------------------------------------

def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(12)
    x = rng.standard_normal(20000).astype(np.float32) * np.float32(3.0)
    # exact ties: low 16 bits = 0x8000 with even and odd kept parts
    # exact ties (low 16 bits = 0x8000) with both parities of the kept last bit, over many exponents
    expo = rng.integers(1, 254, 4000, dtype=np.uint32) << 23
    kept = rng.integers(0, 2 ** 7, 4000, dtype=np.uint32) << 16
    sign = rng.integers(0, 2, 4000, dtype=np.uint32) << 31
    ties = (sign | expo | kept | 0x8000).view(np.float32)
    x = np.concatenate([x, ties, np.array([0.0, -0.0, 1e-40, 3.0e38], np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    mine = np.array([oracle.bf16_from_float(v) for v in x], dtype=np.uint16)
    assert np.array_equal(mine, ref)
    assert oracle.bf16_to_float(0x3F80) == 1.0


# --------------------------------------------------------------------------
# quantiser / dequantiser
# --------------------------------------------------------------------------

def _bits(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_quantiser_round_trip_bound():
    rng = np.random.default_rng(13)
    for trial in range(40):
        lat = rng.standard_normal(DV).astype(np.float32) * np.float32(10.0 ** rng.uniform(-3, 3))
        if trial % 5 == 0:
            lat[rng.integers(0, DV, 4)] *= 30.0                  # outliers
        if trial % 7 == 0:
            lat[128:256] = 0.0                                   # an all-zero tile
        lb = _bits(lat)
        rope = _bits(rng.standard_normal(64))
        row = oracle.quantize_token(lb, rope)
        k = oracle.dequantize_row(row)
        x = oracle.bf16_bits_to_f64(lb)
        scales = row[512:528].view("<f4").astype(np.float64)
        for t in range(4):
            xs, ks, s = x[t * 128:(t + 1) * 128], k[t * 128:(t + 1) * 128], scales[t]
            assert s == np.float32(np.abs(xs).max()) / np.float32(448.0)
            # e4m3 relative 2^-4 (normal), absolute 2^-10*scale (subnormal), then bf16 2^-8
            bound = 2.0 ** -4 * np.abs(xs) + 2.0 ** -10 * s + 2.0 ** -8 * np.abs(ks) + 1e-30
            assert (np.abs(xs - ks) <= bound).all()
        assert np.array_equal(k[512:], oracle.bf16_bits_to_f64(rope))


def test_quantiser_exact_on_grid():
    """Latent values on the e4m3 grid with +-448 in every tile: scale = 1, dequant exact."""
    rng = np.random.default_rng(14)
    finite = np.array([oracle.e4m3_decode(c) for c in range(256) if not math.isnan(oracle.e4m3_decode(c))])
    lat = rng.choice(finite, DV)
    for t in range(4):
        lat[t * 128 + rng.integers(0, 128)] = 448.0 * (1 if t % 2 else -1)
    lb = _bits(lat)
    row = oracle.quantize_token(lb, _bits(np.zeros(64)))
    assert (row[512:528].view("<f4") == 1.0).all()
    assert np.array_equal(oracle.dequantize_row(row)[:512], lat)


def test_dequant_matches_library_definition():
    """k = bf16(float32(e4m3) * scale) computed with torch's own casts and float32 multiply."""
    rng = np.random.default_rng(16)
    for trial in range(20):
        lat = rng.standard_normal(DV).astype(np.float32) * np.float32(10.0 ** rng.uniform(-2, 2))
        row = oracle.quantize_token(_bits(lat), _bits(rng.standard_normal(64)))
        codes = torch.from_numpy(row[:512].copy()).view(torch.float8_e4m3fn).to(torch.float32).reshape(4, 128)
        scales = torch.from_numpy(row[512:528].copy().view("<f4").astype(np.float32)).reshape(4, 1)
        ref = (codes * scales).to(torch.bfloat16).to(torch.float64).reshape(-1).numpy()
        k = oracle.dequantize_row(row)
        assert np.array_equal(k[:512], ref)
        # every key value is a bf16 number (low 16 bits of its float32 encoding are zero)
        assert ((k.astype(np.float32).view(np.uint32) & 0xFFFF) == 0).all()


def test_bulk_quantiser_matches_scalar():
    rng = np.random.default_rng(15)
    n = 300
    lat = rng.standard_normal((n, DV)).astype(np.float32) * np.float32(3.0)
    lat[::7, 5] *= 8.0
    lat[3, 0:128] = 0.0
    lat[4, :] = 0.0
    lat[5, 128:256] = 2.0 ** -130                       # subnormal-scale tile
    lat[6, 256:384] = np.float32(1e30)                  # huge tile
    lb = _bits(lat)
    rope = _bits(rng.standard_normal((n, 64)))
    assert np.array_equal(oracle.quantize_tokens_bulk(lb, rope), oracle.quantize_tokens(lb, rope))


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------

def _textbook(q, K, scale):
    """Dense softmax attention written independently with numpy (float64)."""
    s = (q @ K.T) * scale
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    raw = (q @ K.T) * scale
    mx = raw.max(axis=1)
    lse = mx + np.log(np.exp(raw - mx[:, None]).sum(axis=1))
    return p @ K[:, :DV], lse


def _close(a, b, tol=1e-12):
    """Agreement to float64 summation-order noise, relative to the magnitude of b."""
    return np.allclose(a, b, rtol=0, atol=tol * max(1.0, float(np.abs(b).max())))


def test_attend_equals_textbook_dense_attention():
    rng = np.random.default_rng(21)
    for h, n in [(1, 1), (16, 37), (64, 200), (128, 64)]:
        q = rng.standard_normal((h, DQK))
        K = rng.standard_normal((n, DQK))
        o, lse = oracle.attend(q, K, np.ones(n, np.uint8))
        o_ref, lse_ref = _textbook(q, K, 1.0 / 24.0)
        assert np.allclose(o, o_ref, rtol=0, atol=1e-12)
        assert np.allclose(lse, lse_ref, rtol=0, atol=1e-12)


def test_weights_sum_to_one_and_match_softmax():
    rng = np.random.default_rng(22)
    q = rng.standard_normal((8, DQK))
    K = rng.standard_normal((50, DQK))
    valid = (rng.random(50) > 0.3).astype(np.uint8)
    o, lse, w = oracle.attend(q, K, valid, want_weights=True)
    assert np.allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert (w[:, valid == 0] == 0).all()
    assert np.allclose(o, w @ K[:, :DV], rtol=0, atol=1e-12)


def test_permutation_invariance():
    rng = np.random.default_rng(23)
    q = rng.standard_normal((4, DQK))
    K = rng.standard_normal((90, DQK))
    valid = (rng.random(90) > 0.2).astype(np.uint8)
    o1, l1 = oracle.attend(q, K, valid)
    perm = rng.permutation(90)
    o2, l2 = oracle.attend(q, K[perm], valid[perm])
    assert np.allclose(o1, o2, rtol=0, atol=1e-12) and np.allclose(l1, l2, rtol=0, atol=1e-12)


def test_split_then_combine_equals_single_pass():
    rng = np.random.default_rng(24)
    h, n = 6, 150
    q = rng.standard_normal((h, DQK))
    K = rng.standard_normal((n, DQK))
    valid = (rng.random(n) > 0.1).astype(np.uint8)
    o_ref, lse_ref = oracle.attend(q, K, valid)
    for trial in range(6):
        cuts = np.sort(rng.integers(0, n + 1, size=rng.integers(1, 6)))
        bounds = [0, *cuts.tolist(), n]                    # may contain empty parts
        parts = [(a, b) for a, b in zip(bounds[:-1], bounds[1:])]
        os_, ls_ = [], []
        for a, b in parts:
            o, l = oracle.attend(q, K[a:b], valid[a:b])
            os_.append(o)
            ls_.append(l)
        o, lse = oracle.combine(np.stack(os_), np.stack(ls_))
        assert np.allclose(o, o_ref, rtol=0, atol=1e-12)
        assert np.allclose(lse, lse_ref, rtol=0, atol=1e-12)


def test_all_invalid_gives_zero_and_minus_inf():
    rng = np.random.default_rng(25)
    q = rng.standard_normal((3, DQK))
    K = rng.standard_normal((10, DQK))
    o, lse = oracle.attend(q, K, np.zeros(10, np.uint8))
    assert (o == 0).all() and np.isneginf(lse).all()
    o, lse = oracle.attend(q, K[:0], np.zeros(0, np.uint8))
    assert (o == 0).all() and np.isneginf(lse).all()
    o, lse = oracle.combine(np.ones((3, 3, DV)), np.full((3, 3), -np.inf))
    assert (o == 0).all() and np.isneginf(lse).all()


def test_closed_forms_single_slot_and_identical_rows():
    rng = np.random.default_rng(26)
    q = rng.standard_normal((5, DQK))
    K = rng.standard_normal((20, DQK))
    valid = np.zeros(20, np.uint8)
    valid[7] = 1
    o, lse = oracle.attend(q, K, valid)
    assert np.array_equal(o, np.broadcast_to(K[7, :DV], o.shape))
    assert np.allclose(lse, (q @ K[7]) / 24.0, rtol=0, atol=1e-12)
    Kn = np.repeat(K[3:4], 9, axis=0)
    o, lse = oracle.attend(q, Kn, np.ones(9, np.uint8))
    assert np.allclose(o, np.broadcast_to(K[3, :DV], o.shape), rtol=0, atol=1e-12)
    assert np.allclose(lse, (q @ K[3]) / 24.0 + math.log(9), rtol=0, atol=1e-12)
    # adding invalid slots changes nothing
    o1, l1 = oracle.attend(q, K[:10], np.ones(10, np.uint8))
    K2 = np.concatenate([K[:10], np.full((5, DQK), np.nan)])
    o2, l2 = oracle.attend(q, K2, np.concatenate([np.ones(10, np.uint8), np.zeros(5, np.uint8)]))
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_softmax_scale_argument():
    rng = np.random.default_rng(27)
    q = rng.standard_normal((2, DQK))
    K = rng.standard_normal((30, DQK))
    o, lse = oracle.attend(q, K, np.ones(30, np.uint8), softmax_scale=0.3)
    o_ref, lse_ref = _textbook(q, K, 0.3)
    assert np.allclose(o, o_ref, atol=1e-12) and np.allclose(lse, lse_ref, atol=1e-12)


# --------------------------------------------------------------------------
# the paged path
# --------------------------------------------------------------------------

def _grid_cache(rng, seqlen, nblocks_total, perm):
    """A cache whose latent values lie on the e4m3 grid with scale 1, in a permuted block order."""
    finite = np.array([oracle.e4m3_decode(c) for c in range(256) if not math.isnan(oracle.e4m3_decode(c))])
    logical = np.zeros((nblocks_total * 64, 656), np.uint8)
    Kl = np.zeros((seqlen, DQK))
    for t in range(seqlen):
        lat = rng.choice(finite[np.abs(finite) <= 16], DV)
        for tt in range(4):
            lat[tt * 128 + (t % 128)] = 448.0
        rope = oracle.bf16_bits_to_f64(_bits(rng.standard_normal(64)))
        logical[t] = oracle.quantize_token(_bits(lat), _bits(rope))
        Kl[t, :DV] = lat
        Kl[t, DV:] = rope
    phys = np.zeros_like(logical)
    for lb in range(nblocks_total):
        phys[perm[lb] * 64:(perm[lb] + 1) * 64] = logical[lb * 64:(lb + 1) * 64]
    return phys.reshape(nblocks_total, 64, 656), Kl


def test_paged_grid_case_equals_textbook_over_all_tokens():
    rng = np.random.default_rng(31)
    seqlen = 200
    nb = 4
    perm = rng.permutation(nb)
    cache, Kl = _grid_cache(rng, seqlen, nb, perm)
    q_bits = _bits(rng.standard_normal((16, DQK)))
    q = oracle.bf16_bits_to_f64(q_bits)
    idx = rng.permutation(seqlen).astype(np.int32)
    o, lse = oracle.sparse_decode_token(q_bits, cache, perm.astype(np.int32), seqlen, idx)
    o_ref, lse_ref = _textbook(q, Kl, 1.0 / 24.0)
    assert _close(o, o_ref) and _close(lse, lse_ref)


def test_paged_validity_rules_and_poison():
    rng = np.random.default_rng(32)
    seqlen = 130                                      # 3 blocks; rows 130..191 unused
    nb = 4
    perm = rng.permutation(nb)
    cache, Kl = _grid_cache(rng, 192, nb, perm)
    flat = cache.reshape(-1, 656)
    for t in range(seqlen, 192):                       # poison rows past the length
        flat[perm[t // 64] * 64 + t % 64] = 0x7F
    q_bits = _bits(rng.standard_normal((4, DQK)))
    q = oracle.bf16_bits_to_f64(q_bits)
    idx = np.array([5, -1, 129, 130, 191, -7, 64, 1000, 0], np.int32)   # 130,191,1000 >= seqlen
    o, lse = oracle.sparse_decode_token(q_bits, cache, perm.astype(np.int32), seqlen, idx)
    keep = [5, 129, 64, 0]
    o_ref, lse_ref = _textbook(q, Kl[keep], 1.0 / 24.0)
    assert np.isfinite(o).all()
    assert _close(o, o_ref) and _close(lse, lse_ref)


def test_sparse_prefill_equals_textbook_over_its_rows():
    # flat cache of 150 rows (not a whole number of 64-row blocks), values on the e4m3 grid
    rng = np.random.default_rng(33)
    s_kv = 150
    cache, Kl = _grid_cache(rng, s_kv, 3, np.arange(3))
    kv_rows = cache.reshape(-1, 656)[:s_kv].copy()
    s_q, h = 5, 16
    q_bits = _bits(rng.standard_normal((s_q, h, DQK)))
    idx = rng.integers(-3, s_kv + 8, size=(s_q, 1, 40)).astype(np.int32)
    idx[2, 0, :] = -1                                    # a token with no valid slot
    ref = oracle.sparse_prefill(q_bits, kv_rows, idx)
    for t in range(s_q):
        keep = [int(i) for i in idx[t, 0] if 0 <= i < s_kv]
        o, lse = ref[t]
        if not keep:
            assert (o == 0).all() and np.isneginf(lse).all()
            continue
        o_ref, lse_ref = _textbook(oracle.bf16_bits_to_f64(q_bits[t]), Kl[keep], 1.0 / 24.0)
        assert _close(o, o_ref) and _close(lse, lse_ref)


def test_sparse_decode_batch_driver():
    rng = np.random.default_rng(33)
    seqlen = 128
    perm = rng.permutation(2)
    cache, Kl = _grid_cache(rng, seqlen, 2, perm)
    q_bits = _bits(rng.standard_normal((1, 2, 16, DQK)))
    idx = np.stack([rng.permutation(seqlen)[:40], rng.permutation(seqlen)[:40]]).astype(np.int32).reshape(1, 2, 40)
    res = oracle.sparse_decode(q_bits, cache, perm.astype(np.int32).reshape(1, 2), np.array([seqlen]), idx,
                               threads=2)
    for t in range(2):
        o_ref, l_ref = _textbook(oracle.bf16_bits_to_f64(q_bits[0, t]), Kl[idx[0, t]], 1.0 / 24.0)
        o, l = res[(0, t)]
        assert _close(o, o_ref) and _close(l, l_ref)


# --------------------------------------------------------------------------
# scheduler
# --------------------------------------------------------------------------

def _brute_sched(R, n, P):
    """Enumerate tiles one by one, filling parts of L tiles in order."""
    total = R * n
    L = -(-total // P) if total else 1
    owner = {}
    for r in range(R):
        for t in range(n):
            owner[(r, t)] = (r * n + t) // L
    parts = {p: [k for k, v in owner.items() if v == p] for p in range(P)}
    return L, owner, parts


@pytest.mark.parametrize("R,n,P", [(2, 1, 148), (64, 32, 148), (64, 32, 74), (7, 3, 5), (1, 1, 1),
                                   (0, 4, 8), (5, 7, 35), (5, 7, 36), (13, 2, 3), (256, 32, 148),
                                   (3, 100, 7), (4096, 32, 74)])
def test_sched_meta_brute_force(R, n, P):
    sm, ns = oracle.sched_meta(R, n, P)
    L, owner, parts = _brute_sched(R, n, P)
    # splits per request = number of distinct parts touching it
    S = [len({owner[(r, t)] for t in range(n)}) for r in range(R)]
    assert ns[0] == 0 and list(np.diff(ns)) == S
    covered = set()
    for p in range(P):
        tiles = parts[p]
        if not tiles:
            assert sm[p, 5] == 1 and (sm[p, :5] == 0).all()
            continue
        assert sm[p, 5] == 0
        tiles = sorted(tiles)
        assert (sm[p, 0], sm[p, 1]) == tiles[0]
        last = tiles[-1]
        end = (last[0], last[1] + 1) if last[1] + 1 < n else (last[0] + 1, 0)
        assert (sm[p, 2], sm[p, 3]) == end
        # slot of (p, first request) = this part's rank among the parts of that request
        r0 = tiles[0][0]
        parts_of_r0 = sorted({owner[(r0, t)] for t in range(n)})
        assert sm[p, 4] == ns[r0] + parts_of_r0.index(p)
        covered.update(tiles)
        assert len(tiles) <= L
    assert covered == set(owner)
    loads = [len(v) for v in parts.values() if v]
    assert all(x == L for x in loads[:-1])                 # all full except the last non-empty part


def test_sched_meta_rejects_bad_arguments():
    with pytest.raises(ValueError):
        oracle.sched_meta(4, 0, 8)
    with pytest.raises(ValueError):
        oracle.sched_meta(4, 2, 0)


# --------------------------------------------------------------------------
# dense decode: every visible token, FP8 or BF16 cache rows
# --------------------------------------------------------------------------

def test_bf16_row_matches_torch_cast():
    import torch
    rng = np.random.default_rng(51)
    vals = np.concatenate([rng.standard_normal(500) * 10.0 ** rng.integers(-30, 30, 500), [0.0, -0.0, 1e38, -3e-39],
                           rng.standard_normal(72)])[:576]
    bits = _bits(vals)
    row = bits.astype("<u2").tobytes()
    k = oracle.bf16_row(np.frombuffer(row, np.uint8))
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.array_equal(k, ref)


def test_dense_visible_len_closed_forms():
    for sl, s_q in [(100, 1), (100, 4), (3, 4), (0, 2), (64, 64)]:
        for t in range(s_q):
            assert oracle.dense_visible_len(sl, s_q, t, False) == sl
            assert oracle.dense_visible_len(sl, s_q, t, True) == max(0, min(sl, sl - s_q + 1 + t))
        # the last new token sees the whole cache; token t sees one more position than token t-1
        if sl >= s_q:
            assert oracle.dense_visible_len(sl, s_q, s_q - 1, True) == sl
            assert [oracle.dense_visible_len(sl, s_q, t, True) for t in range(s_q)] == list(range(sl - s_q + 1, sl + 1))


def test_dense_fp8_equals_sparse_decode_over_every_position():
    """Dense decode is the sparse decode whose index list is every visible position."""
    rng = np.random.default_rng(52)
    nb, seqlen = 5, 300
    lat = _bits(rng.standard_normal((nb * 64, DV)) * 3)
    rope = _bits(rng.standard_normal((nb * 64, 64)))
    cache = oracle.quantize_tokens(lat, rope).reshape(nb, 64, 656)
    bt = rng.permutation(nb).astype(np.int32)
    q_bits = _bits(rng.standard_normal((32, DQK)))
    for n in (1, 63, 64, 65, 300):
        o, lse = oracle.dense_decode_token(q_bits, cache, oracle.KV_FP8, bt, n)
        o2, lse2 = oracle.sparse_decode_token(q_bits, cache, bt, seqlen, np.arange(n, dtype=np.int32))
        assert np.array_equal(o, o2) and np.array_equal(lse, lse2)


def _bf16_cache(rng, nb, perm):
    """A paged BF16 cache (rows of 576 bf16 values) and its logical key matrix."""
    logical = _bits(rng.standard_normal((nb * 64, DQK)))
    Kl = oracle.bf16_bits_to_f64(logical)
    phys = np.zeros_like(logical)
    for lb in range(nb):
        phys[perm[lb] * 64:(perm[lb] + 1) * 64] = logical[lb * 64:(lb + 1) * 64]
    return np.frombuffer(phys.astype("<u2").tobytes(), np.uint8).reshape(nb, 64, 1152), Kl


def test_dense_bf16_equals_textbook_over_visible_tokens():
    rng = np.random.default_rng(53)
    nb = 4
    perm = rng.permutation(nb)
    cache, Kl = _bf16_cache(rng, nb, perm)
    q_bits = _bits(rng.standard_normal((16, DQK)))
    q = oracle.bf16_bits_to_f64(q_bits)
    for n in (1, 64, 130, 256):
        o, lse = oracle.dense_decode_token(q_bits, cache, oracle.KV_BF16, perm.astype(np.int32), n)
        o_ref, lse_ref = _textbook(q, Kl[:n], 1.0 / 24.0)
        assert _close(o, o_ref) and _close(lse, lse_ref)


def test_dense_batch_driver_applies_the_causal_mask():
    rng = np.random.default_rng(54)
    nb = 3
    perm = rng.permutation(nb)
    cache, Kl = _bf16_cache(rng, nb, perm)
    s_q, seqlen = 3, 150
    q_bits = _bits(rng.standard_normal((1, s_q, 8, DQK)))
    bt = perm.astype(np.int32).reshape(1, -1)
    for causal in (False, True):
        out = oracle.dense_decode(q_bits, cache, oracle.KV_BF16, bt, np.array([seqlen]), causal)
        for t in range(s_q):
            n = seqlen - (s_q - 1 - t) if causal else seqlen
            o_ref, lse_ref = _textbook(oracle.bf16_bits_to_f64(q_bits[0, t]), Kl[:n], 1.0 / 24.0)
            assert _close(out[(0, t)][0], o_ref) and _close(out[(0, t)][1], lse_ref)


def test_dense_zero_visible_tokens_gives_zero_and_minus_inf():
    rng = np.random.default_rng(55)
    cache, _ = _bf16_cache(rng, 1, np.array([0]))
    o, lse = oracle.dense_decode_token(_bits(rng.standard_normal((4, DQK))), cache, oracle.KV_BF16,
                                       np.array([0], np.int32), 0)
    assert (o == 0).all() and np.isneginf(lse).all()


def _brute_sched_varlen(n, P):
    """Enumerate tiles one by one, filling parts of L tiles in (request, tile) order."""
    total = int(np.sum(n))
    L = -(-total // P) if total else 1
    owner, g = {}, 0
    for r, nr in enumerate(n):
        for t in range(nr):
            owner[(r, t)] = g // L
            g += 1
    parts = {p: sorted(k for k, v in owner.items() if v == p) for p in range(P)}
    return L, owner, parts


@pytest.mark.parametrize("n,P", [([3, 1, 5, 2], 4), ([1], 148), ([128] * 64, 148), ([7, 1, 1, 1, 30, 2], 5),
                                 ([2048] * 2 + [64] * 30, 74), ([1] * 300, 148), ([4, 4, 4], 3), ([9, 9], 7)])
def test_sched_meta_varlen_brute_force(n, P):
    sm, ns, tp = oracle.sched_meta_varlen(np.array(n), P)
    assert list(tp) == [0] + list(np.cumsum(n))
    L, owner, parts = _brute_sched_varlen(n, P)
    S = [len({owner[(r, t)] for t in range(nr)}) for r, nr in enumerate(n)]
    assert ns[0] == 0 and list(np.diff(ns)) == S
    covered = set()
    for p in range(P):
        tiles = parts[p]
        if not tiles:
            assert sm[p, 5] == 1 and (sm[p, :5] == 0).all()
            continue
        assert sm[p, 5] == 0 and (sm[p, 0], sm[p, 1]) == tiles[0]
        last = tiles[-1]
        end = (last[0], last[1] + 1) if last[1] + 1 < n[last[0]] else (last[0] + 1, 0)
        assert (sm[p, 2], sm[p, 3]) == end
        r0 = tiles[0][0]
        parts_of_r0 = sorted({owner[(r0, t)] for t in range(n[r0])})
        assert sm[p, 4] == ns[r0] + parts_of_r0.index(p)
        covered.update(tiles)
        assert len(tiles) <= L
    assert covered == set(owner)


def test_sched_meta_varlen_equals_uniform_for_equal_counts():
    for R, k, P in [(64, 32, 148), (7, 3, 5), (256, 32, 148), (5, 7, 36)]:
        sm, ns, _ = oracle.sched_meta_varlen(np.full(R, k), P)
        sm_u, ns_u = oracle.sched_meta(R, k, P)
        assert np.array_equal(sm, sm_u) and np.array_equal(ns, ns_u)


def test_sched_meta_varlen_rejects_empty_requests():
    with pytest.raises(ValueError):
        oracle.sched_meta_varlen(np.array([2, 0, 1]), 4)


def test_dense_tile_counts():
    assert list(oracle.dense_tile_counts(np.array([1, 64, 65, 0]), 1, False)) == [1, 1, 2, 1]
    # causal: token t of 3 sees seqlen - 2 + t positions: 126..128 -> 2, 2, 2 tiles; 128..130 -> 2, 3, 3
    assert list(oracle.dense_tile_counts(np.array([128]), 3, True)) == [2, 2, 2]
    assert list(oracle.dense_tile_counts(np.array([130]), 3, True)) == [2, 3, 3]
