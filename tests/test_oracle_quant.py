"""Pins for the oracle's smooth-K and quantization steps.

Smooth K (「SageAttention：低比特量化Attention，实现推理加速」, section 技术方案, paragraph on smoothing K): the mean
is per channel over tokens. Per-block INT8 (same section, paragraph on per-block INT8 of
Q, K): one fp32 scale per block, Q blocks 128 tokens, K blocks 64 tokens, scale =
amax/127. V to E4M3 with a per-channel scale (「4比特量化三倍加速不掉点！清华即插即用的SageAttention迎来升级」, 技术方案 (4)).
The checks are closed forms, invariants and library routines; none re-types the
oracle's own formula.
"""
import numpy as np
import pytest

import oracle
from oracle import Layout


def _rand16(shape, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal(shape) * scale).astype(np.float16)


def test_k_mean_matches_numpy_mean():
    k = _rand16((2, 3, 200, 16), 1, 3.0)
    lay = Layout.dense(2, 3, 200, 16)
    mu = oracle.k_mean(k, lay)
    ref = k.astype(np.float64).mean(axis=2).astype(np.float32)   # library routine
    assert np.array_equal(mu, ref)


def test_k_mean_axis_is_tokens_not_channels():
    # a pure per-channel offset: the mean over tokens must return the offset exactly
    off = np.array([0.5, -2.0, 4.0, 0.0, 1.25, -0.75, 8.0, 3.0], np.float16)
    k = np.broadcast_to(off, (1, 1, 10, 8)).astype(np.float16).copy()
    mu = oracle.k_mean(k, Layout.dense(1, 1, 10, 8))
    assert np.array_equal(mu[0, 0], off.astype(np.float32))


def test_varlen_mean_is_per_sequence():
    H, d = 2, 8
    cu = [0, 5, 12]
    k = np.zeros((12, H, d), np.float16)
    k[:5] = 1.0
    k[5:] = -3.0
    mu = oracle.k_mean(k, Layout.packed(cu, H, d))
    assert np.all(mu[0] == 1.0) and np.all(mu[1] == -3.0)


def test_exact_multiples_give_exact_codes():
    # values u*c with integer c in [-127,127] and max |c| = 127, u a power of two:
    # scale = (127u)/127 = u exactly and every code is exactly c
    rng = np.random.default_rng(3)
    c = rng.integers(-127, 128, size=(1, 1, 128, 16))
    c[0, 0, 5, 3] = 127
    u = 0.125
    x = (c * u).astype(np.float16)
    codes, scales = oracle.quant_int8(x, Layout.dense(1, 1, 128, 16), 128)
    assert scales[0, 0, 0] == np.float32(u)
    assert np.array_equal(codes.astype(np.int64), c)


def _block_ids(n, blk):
    return np.arange(n) // blk


@pytest.mark.parametrize("blk", [128, 64])
def test_block_boundaries_and_ragged_tail(blk):
    n, d = 3 * blk + 17, 8
    # each block gets its own magnitude so a misplaced boundary changes the scales
    mags = np.array([1.0, 4.0, 0.25, 16.0])
    x = _rand16((1, 1, n, d), 7)
    x = (x.astype(np.float64) * mags[_block_ids(n, blk)][None, None, :, None]).astype(np.float16)
    codes, scales = oracle.quant_int8(x, Layout.dense(1, 1, n, d), blk)
    assert scales.shape[2] == -(-n // blk)
    xf = x.astype(np.float32)[0, 0]
    for b in range(scales.shape[2]):
        rows = slice(b * blk, min(n, (b + 1) * blk))
        amax = np.abs(xf[rows]).max()
        s = scales[0, 0, b]
        # closed form: 127 s reproduces the block's amax to within one fp32 rounding
        assert abs(127.0 * float(s) - float(amax)) <= 2 * np.spacing(np.float32(amax))
        cb = codes[0, 0, rows].astype(np.int64)
        assert np.abs(cb).max() == 127
        assert np.all(np.abs(xf[rows] - s * cb) <= s * (0.5 + 1e-5))


def test_ragged_tail_rows_do_not_enter_scale():
    # N = 130: block 1 holds two rows. In the varlen layout the rows right after the
    # sequence belong to the next sequence and carry a huge value that must not leak.
    H, d = 1, 8
    cu = [0, 130, 260]
    x = _rand16((260, H, d), 11)
    x[130:] = 1000.0
    codes, scales = oracle.quant_int8(x, Layout.packed(cu, H, d), 128)
    amax = np.abs(x[128:130].astype(np.float32)).max()
    assert abs(127.0 * float(scales[0, 0, 1]) - float(amax)) <= 2 * np.spacing(np.float32(amax))


def test_zero_block():
    x = np.zeros((1, 1, 64, 8), np.float16)
    codes, scales = oracle.quant_int8(x, Layout.dense(1, 1, 64, 8), 64)
    assert scales[0, 0, 0] == 0.0 and not codes.any()


def test_codes_round_half_to_even():
    # amax = 127 gives scale 1 exactly; x = k + 0.5 must round to the even neighbour
    x = np.zeros((1, 1, 4, 8), np.float16)
    x[0, 0, 0, 0] = 127.0
    x[0, 0, 1, :4] = [0.5, 1.5, 2.5, -3.5]
    codes, scales = oracle.quant_int8(x, Layout.dense(1, 1, 4, 8), 64)
    assert scales[0, 0, 0] == 1.0
    assert list(codes[0, 0, 1, :4]) == [0, 2, 2, -4]


def test_smoothed_k_reconstructs():
    lay = Layout.dense(1, 2, 300, 16)
    k = _rand16((1, 2, 300, 16), 5)
    k = (k.astype(np.float32) + np.linspace(-20, 20, 16)).astype(np.float16)
    z = oracle.quant_qk(k, k, lay, smooth_k=True)
    mu = z["k_mean"]
    kf = k.astype(np.float32)
    for h in range(2):
        for b in range(z["k_scale"].shape[2]):
            rows = slice(b * 64, min(300, (b + 1) * 64))
            s = z["k_scale"][0, h, b]
            rec = s * z["k_i8"][0, h, rows].astype(np.float32) + mu[0, h]
            assert np.all(np.abs(rec - kf[0, h, rows]) <= s * 0.5001 + 1e-5)
    # smoothing removes the offset: the smoothed scales are far below the raw ones
    raw = oracle.quant_qk(k, k, lay, smooth_k=False)
    assert z["k_scale"].max() < 0.25 * raw["k_scale"].max()


def test_v_fp8_per_channel():
    lay = Layout.dense(1, 1, 50, 8)
    v = _rand16((1, 1, 50, 8), 9)
    v[..., 3] *= 100
    v[..., 5] = 0
    codes, scales = oracle.quant_v_fp8(v, lay)
    vals = np.vectorize(oracle.e4m3_decode)(codes).astype(np.float64)
    assert scales[0, 0, 5] == 0 and not codes[..., 5].any()
    for c in range(8):
        if c == 5:
            continue
        assert np.abs(vals[0, 0, :, c]).max() == 448.0          # amax maps to 448
        rec = vals[0, 0, :, c] * scales[0, 0, c]
        ref = v[0, 0, :, c].astype(np.float64)
        # E4M3 keeps 3 mantissa bits: relative error <= 2^-4 above the subnormal range
        tol = np.maximum(np.abs(ref) * 2.0 ** -4, scales[0, 0, c] * 2.0 ** -10)
        assert np.all(np.abs(rec - ref) <= tol * 1.0001)


def test_v_fp8_smoothed_per_channel():
    # Smooth V (「4比特量化三倍加速不掉点！清华即插即用的SageAttention迎来升级」, 技术方案, the paragraph after (4)): codes encode
    # V - mean(V) per channel; the mean is the numpy token mean rounded to fp32
    lay = Layout.dense(1, 2, 70, 8)
    v = _rand16((1, 2, 70, 8), 19).astype(np.float64)
    v += np.array([50.0, -20.0, 0.0, 5.0, 100.0, -3.0, 7.0, 0.0])
    v[..., 7] = 2.5                                             # constant channel
    v = v.astype(np.float16)
    mu = oracle.v_mean(v, lay)
    assert np.array_equal(mu, v.astype(np.float64).mean(axis=2).astype(np.float32))
    codes, scales = oracle.quant_v_fp8(v, lay, mu=mu)
    vals = np.vectorize(oracle.e4m3_decode)(codes).astype(np.float64)
    assert np.all(scales[..., 7] == 0) and not codes[..., 7].any()   # V - mean = 0 exactly
    for h in range(2):
        for c in range(7):
            x = (v[0, h, :, c].astype(np.float32) - mu[0, h, c]).astype(np.float64)
            assert np.abs(vals[0, h, :, c]).max() == 448.0      # amax of |V - mean| maps to 448
            rec = vals[0, h, :, c] * scales[0, h, c]
            tol = np.maximum(np.abs(x) * 2.0 ** -4, scales[0, h, c] * 2.0 ** -10)
            assert np.all(np.abs(rec - x) <= tol * 1.0001)
    # the offsets are gone: smoothed scales are far below the raw ones on offset channels
    _, raw = oracle.quant_v_fp8(v, lay)
    assert np.all(scales[0, :, [0, 1, 4]] < 0.2 * raw[0, :, [0, 1, 4]])


def test_fine_groups_scales():
    # finer groups ([SA2] 技术方案 (2), restated for one scale per query row and per 32
    # keys): every Q token gets amax/127 of its own row, every 32 K tokens of their block
    N, d = 100, 16
    lay = Layout.dense(1, 2, N, d)
    q = _rand16((1, 2, N, d), 31) * (2.0 ** np.arange(N) % 7)[None, None, :, None].astype(np.float16)
    k = _rand16((1, 2, N, d), 32)
    z = oracle.quant_qk(q, k, lay, True, fine=True)
    qa = np.abs(q.astype(np.float32)).max(axis=3)
    assert z["q_scale"].shape == (1, 2, N)
    assert np.array_equal(z["q_scale"], (qa / np.float32(127)).astype(np.float32))
    kf = k.astype(np.float32) - z["k_mean"][:, :, None, :]
    assert z["k_scale"].shape == (1, 2, 4)
    for b in range(4):
        blk = np.abs(kf[:, :, 32 * b:min(N, 32 * b + 32)]).max(axis=(2, 3))
        assert np.array_equal(z["k_scale"][:, :, b], (blk / np.float32(127)).astype(np.float32))
    # every row of Q spends the full code range
    assert np.all(np.abs(z["q_i8"]).max(axis=3)[qa > 0] == 127)
