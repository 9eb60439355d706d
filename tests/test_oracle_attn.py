"""Pins for the oracle's attention: the fp64 reference and the quantized method.

* fp64 attention vs torch's scaled_dot_product_attention in float64 (library routine);
  N = 1 gives O = V; identical keys give O = mean(V).
* The smoothing invariant softmax(QK^T) = softmax(Q(K - mean K)^T) ("SageAttention"
  article, section 技术方案, paragraph on smoothing K), to ~1e-12 in fp64.
* The quantized method (same section; 「4比特量化三倍加速不掉点！清华即插即用的SageAttention迎来升级」, 技术方案 (3)-(4)):
  a single KV tile reduces the online softmax to a plain softmax over integer scores,
  recomputed here with a library integer matmul; many tiles agree with one tile up to
  the FP16 rounding of P; the result tracks fp64 attention on inputs built so that a
  dropped rescale, a wrong scale index or a transposed operand would fail.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import Layout, PV_FP16, PV_FP8


def _rand16(shape, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal(shape) * scale).astype(np.float16)


def _cos(a, b):
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))


def _rel_l1(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.abs(a - b).sum() / np.abs(b).sum())


@pytest.mark.parametrize("causal", [False, True])
def test_fp64_matches_torch_sdpa(causal):
    B, H, N, d = 2, 3, 70, 16
    q, k, v = (_rand16((B, H, N, d), s) for s in (1, 2, 3))
    sm = 1 / math.sqrt(d)
    got = oracle.attn_fp64(q, k, v, Layout.dense(B, H, N, d), causal, sm)
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(x.astype(np.float64)) for x in (q, k, v)), is_causal=causal, scale=sm)
    assert np.allclose(got, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_fp64_special_cases():
    d = 8
    v = _rand16((1, 1, 1, d), 4)
    q = _rand16((1, 1, 1, d), 5)
    o = oracle.attn_fp64(q, q, v, Layout.dense(1, 1, 1, d), False, 0.3)
    assert np.allclose(o, v.astype(np.float64), rtol=0, atol=1e-15)          # N = 1: O = V
    N = 20
    q = _rand16((1, 1, N, d), 6)
    k = np.broadcast_to(_rand16((d,), 7), (1, 1, N, d)).astype(np.float16)
    v = _rand16((1, 1, N, d), 8)
    o = oracle.attn_fp64(q, k, v, Layout.dense(1, 1, N, d), False, 0.3)
    assert np.allclose(o, v.astype(np.float64).mean(axis=2, keepdims=True), atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_smoothing_invariant_fp64(causal):
    B, H, N, d = 1, 2, 90, 16
    q, k, v = (_rand16((B, H, N, d), s) for s in (11, 12, 13))
    k = (k.astype(np.float64) + np.linspace(-30, 30, d)).astype(np.float16)
    lay = Layout.dense(B, H, N, d)
    k64 = k.astype(np.float64)
    ks = k64 - k64.mean(axis=2, keepdims=True)
    a = oracle.attn_fp64(q, k64, v, lay, causal, 0.25)
    b = oracle.attn_fp64(q, ks, v, lay, causal, 0.25)
    assert np.max(np.abs(a - b)) < 1e-12


def _single_tile_reference(z, v, causal, pv_mode, sm, vs=None):
    """Plain softmax over integer scores for one head (valid when one KV tile holds all
    keys): S by a library int64 matmul, t in base 2, P rounded once, O = P V / sum p."""
    qc = z["q_i8"][0, 0].astype(np.int64)
    kc = z["k_i8"][0, 0].astype(np.int64)
    N = qc.shape[0]
    S = qc @ kc.T
    sq = z["q_scale"][0, 0][np.arange(N) // 128].astype(np.float64)
    sk = z["k_scale"][0, 0][np.arange(N) // 64].astype(np.float64)
    t = S * sq[:, None] * sk[None, :] * sm / math.log(2)
    if causal:
        t[np.triu_indices(N, 1)] = -np.inf
    p = np.exp2(t - t.max(axis=1, keepdims=True))
    if pv_mode == PV_FP16:
        P = p.astype(np.float16).astype(np.float64)
        O = P @ v[0, 0].astype(np.float64) / p.sum(axis=1, keepdims=True)
    else:
        P = torch.from_numpy(448 * p).to(torch.float32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
        vv = torch.from_numpy(v[0, 0]).view(torch.float8_e4m3fn).to(torch.float64).numpy()
        O = P @ vv * vs[0, 0][None, :] / (448 * p.sum(axis=1, keepdims=True))
    return O.astype(np.float16)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("pv_mode", [PV_FP16, PV_FP8])
def test_single_tile_equals_plain_softmax(causal, pv_mode):
    N, d = 200, 32
    q, k, v = (_rand16((1, 1, N, d), s) for s in (21, 22, 23))
    k = (k.astype(np.float32) + 2.0).astype(np.float16)
    lay = Layout.dense(1, 1, N, d)
    sm = 1 / math.sqrt(d)
    z = oracle.quant_qk(q, k, lay, True)
    if pv_mode == PV_FP8:
        vq, vs = oracle.quant_v_fp8(v, lay)
    else:
        vq, vs = v, None
    got = oracle.attn_quant(z["q_i8"], z["q_scale"], z["k_i8"], z["k_scale"], vq, vs, lay,
                            causal, pv_mode, sm, tile_n=256)
    ref = _single_tile_reference(z, vq, causal, pv_mode, sm, vs)
    diff = np.abs(got.astype(np.float64) - ref.astype(np.float64))
    # identical up to fp64 summation order and fp16 output rounding (one fp16 ulp)
    assert diff.max() <= 2 * np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64).max()


def _increasing_scores(N, d, seed):
    """Scores that grow along the keys, so the running max changes from tile to tile."""
    q = _rand16((1, 1, N, d), seed)
    q = (np.abs(q.astype(np.float32)) + 0.5).astype(np.float16)
    k = _rand16((1, 1, N, d), seed + 1, 0.3).astype(np.float32)
    k += np.linspace(0, 0.6, N)[:, None]
    return q, k.astype(np.float16), _rand16((1, 1, N, d), seed + 2)


@pytest.mark.parametrize("pv_mode", [PV_FP16, PV_FP8])
def test_tiles_agree_and_rescale_matters(pv_mode):
    N, d = 640, 32
    q, k, v = _increasing_scores(N, d, 30)
    lay = Layout.dense(1, 1, N, d)
    sm = 1 / math.sqrt(d)
    one = oracle.sage_attention(q, k, v, lay, False, True, pv_mode, sm, tile_n=1024)
    many = oracle.sage_attention(q, k, v, lay, False, True, pv_mode, sm, tile_n=128)
    exact = oracle.attn_fp64(q, k, v, lay, False, sm)
    # E4M3 P keeps 3 mantissa bits, so the tile walk moves FP8 results more than FP16
    assert _cos(many, one) > (0.99999 if pv_mode == PV_FP16 else 0.9995)
    assert _cos(many, exact) > (0.9999 if pv_mode == PV_FP16 else 0.999)


@pytest.mark.parametrize("causal", [False, True])
def test_quantized_tracks_fp64(causal):
    B, H, N, d = 1, 2, 384, 64
    q, k, v = (_rand16((B, H, N, d), s) for s in (41, 42, 43))
    k = (k.astype(np.float32) + _rand16((d,), 44, 2.0)).astype(np.float16)
    lay = Layout.dense(B, H, N, d)
    sm = 1 / math.sqrt(d)
    exact = oracle.attn_fp64(q, k, v, lay, causal, sm)
    o16 = oracle.sage_attention(q, k, v, lay, causal, True, PV_FP16, sm)
    o8 = oracle.sage_attention(q, k, v, lay, causal, True, PV_FP8, sm)
    assert _cos(o16, exact) > 0.9999 and _rel_l1(o16, exact) < 0.02
    assert _cos(o8, exact) > 0.999


def test_block_scale_indexing():
    # K blocks of 64 tokens and Q blocks of 128 tokens with distinct magnitudes: the
    # oracle must track fp64 attention, while the same scores with K scales indexed per
    # 128 tokens instead of 64 (a plausible slip) must not
    N, d = 512, 32
    q, k, v = (_rand16((1, 1, N, d), s) for s in (51, 52, 53))
    mags = 2.0 ** np.array([-1, 1, 0, 1, -1, 0.5, -0.5, 1])
    k = (k.astype(np.float64) * mags[np.arange(N) // 64][None, None, :, None]).astype(np.float16)
    q = (q.astype(np.float64) * (2.0 ** np.array([1, -1, 0, 0.5]))[np.arange(N) // 128][None, None, :, None]).astype(np.float16)
    lay = Layout.dense(1, 1, N, d)
    sm = 1 / math.sqrt(d)
    exact = oracle.attn_fp64(q, k, v, lay, False, sm)
    o = oracle.sage_attention(q, k, v, lay, False, True, PV_FP16, sm)
    assert _cos(o, exact) > 0.9995
    z = oracle.quant_qk(q, k, lay, True)
    wrong = dict(z)
    wrong["k_scale"] = z["k_scale"][:, :, np.arange(z["k_scale"].shape[2]) // 2 * 2]
    slip = _single_tile_reference(wrong, v, False, PV_FP16, sm)
    assert _cos(slip, exact) < 0.99


def test_causal_first_row_and_constant_scores():
    N, d = 130, 16
    q, k, v = (_rand16((1, 1, N, d), s) for s in (61, 62, 63))
    lay = Layout.dense(1, 1, N, d)
    o = oracle.sage_attention(q, k, v, lay, True, True, PV_FP16, 0.25)
    assert np.array_equal(o[0, 0, 0], v[0, 0, 0])           # row 0 sees only key 0
    zq = np.zeros_like(q)                                   # all scores 0: O = mean V
    o = oracle.sage_attention(zq, k, v, lay, False, True, PV_FP16, 0.25)
    mean = v.astype(np.float64).mean(axis=2)[0, 0]
    assert np.max(np.abs(o[0, 0].astype(np.float64) - mean)) <= 1e-3


def test_fp8_single_token_is_exact():
    # N = 1: P = 448 exactly and V / s_v = +-448 exactly, so O = V up to fp32 scale rounding
    d = 16
    v = _rand16((1, 1, 1, d), 71)
    q = _rand16((1, 1, 1, d), 72)
    o = oracle.sage_attention(q, q, v, Layout.dense(1, 1, 1, d), False, True, PV_FP8, 0.25)
    assert np.array_equal(o, v)


def test_smoothing_helps_with_channel_outliers():
    # 「SageAttention：低比特量化Attention，实现推理加速」, 挑战: channel outliers in K ruin direct INT8 quantization;
    # smoothing K fixes it
    N, d = 512, 64
    q, k, v = (_rand16((1, 1, N, d), s) for s in (81, 82, 83))
    off = np.zeros(d)
    off[[3, 17, 40, 55]] = [30.0, -25.0, 40.0, 20.0]
    k = (k.astype(np.float64) + off).astype(np.float16)
    lay = Layout.dense(1, 1, N, d)
    sm = 1 / math.sqrt(d)
    exact = oracle.attn_fp64(q, k, v, lay, False, sm)
    smooth = oracle.sage_attention(q, k, v, lay, False, True, PV_FP16, sm)
    raw = oracle.sage_attention(q, k, v, lay, False, False, PV_FP16, sm)
    assert _rel_l1(smooth, exact) < 0.5 * _rel_l1(raw, exact)


def test_varlen_equals_per_sequence_dense():
    H, d = 2, 32
    lens = [70, 200, 129]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T = int(cu[-1])
    q, k, v = (_rand16((T, H, d), s) for s in (91, 92, 93))
    lay = Layout.packed(cu, H, d)
    o = oracle.sage_attention(q, k, v, lay, True, True, PV_FP16, 0.2)
    for s, n in enumerate(lens):
        sl = slice(cu[s], cu[s + 1])
        dq, dk, dv = (np.ascontiguousarray(x[sl].transpose(1, 0, 2))[None] for x in (q, k, v))
        od = oracle.sage_attention(dq, dk, dv, Layout.dense(1, H, n, d), True, True, PV_FP16, 0.2)
        assert np.array_equal(o[sl].transpose(1, 0, 2), od[0])


def test_sampled_rows_match_full():
    B, H, N, d = 1, 2, 300, 32
    q, k, v = (_rand16((B, H, N, d), s) for s in (101, 102, 103))
    lay = Layout.dense(B, H, N, d)
    full = oracle.sage_attention(q, k, v, lay, True, True, PV_FP16, 0.2)
    part = oracle.sage_attention(q, k, v, lay, True, True, PV_FP16, 0.2, heads=[(0, 1)], rows=(100, 180))
    assert np.array_equal(part[0, 1, 100:180], full[0, 1, 100:180])
    assert np.isnan(part[0, 0]).all() and np.isnan(part[0, 1, :100]).all()


# Smooth V (「4比特量化三倍加速不掉点！清华即插即用的SageAttention迎来升级」, 技术方案, the paragraph after (4)): the FP8 P.V runs on
# V - mean(V) and mean(V) is added to the output; softmax rows sum to 1, so in exact
# arithmetic the result is unchanged.

def test_smooth_v_single_token_and_constant_channels():
    d = 16
    v = _rand16((1, 1, 1, d), 111, 8.0)
    q = _rand16((1, 1, 1, d), 112)
    o = oracle.sage_attention(q, q, v, Layout.dense(1, 1, 1, d), False, True, PV_FP8, 0.25,
                              smooth_v=True)
    assert np.array_equal(o, v)                              # N = 1: V - mean = 0, O = mean
    N = 300
    q, k = _rand16((1, 1, N, d), 113), _rand16((1, 1, N, d), 114)
    row = _rand16((d,), 115, 10.0)
    v = np.broadcast_to(row, (1, 1, N, d)).astype(np.float16)  # every token the same V
    for causal in (False, True):
        o = oracle.sage_attention(q, k, v, Layout.dense(1, 1, N, d), causal, True, PV_FP8,
                                  0.25, smooth_v=True)
        assert np.array_equal(o, v)


def test_smooth_v_single_tile_closed_form():
    N, d = 200, 32
    q, k, v = (_rand16((1, 1, N, d), s) for s in (121, 122, 123))
    v = (v.astype(np.float64) + np.linspace(-20, 20, d)).astype(np.float16)
    lay = Layout.dense(1, 1, N, d)
    sm = 1 / math.sqrt(d)
    z = oracle.quant_qk(q, k, lay, True)
    vm = oracle.v_mean(v, lay)
    vq, vs = oracle.quant_v_fp8(v, lay, mu=vm)
    got = oracle.attn_quant(z["q_i8"], z["q_scale"], z["k_i8"], z["k_scale"], vq, vs, lay,
                            False, PV_FP8, sm, tile_n=256, v_mean=vm)
    ref = _single_tile_reference(z, vq, False, PV_FP8, sm, vs).astype(np.float64)
    # the unsmoothed closed form plus the channel mean, rounded once to fp16
    ref = ref + vm[0, 0][None, :]
    diff = np.abs(got[0, 0].astype(np.float64) - ref)
    assert diff.max() <= 3 * np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64).max()


@pytest.mark.parametrize("causal", [False, True])
def test_smooth_v_helps_with_channel_offsets(causal):
    # V channels with large offsets: without smoothing the E4M3 codes spend their range on
    # the offset; smoothing keeps the error at the level of offset-free V
    N, d = 512, 64
    q, k, v = (_rand16((1, 1, N, d), s) for s in (131, 132, 133))
    off = _rand16((d,), 134, 16.0).astype(np.float64)
    vo = (v.astype(np.float64) + off).astype(np.float16)
    lay = Layout.dense(1, 1, N, d)
    sm = 1 / math.sqrt(d)
    exact = oracle.attn_fp64(q, k, vo, lay, causal, sm)
    smooth = oracle.sage_attention(q, k, vo, lay, causal, True, PV_FP8, sm, smooth_v=True)
    raw = oracle.sage_attention(q, k, vo, lay, causal, True, PV_FP8, sm)
    err_s = np.abs(smooth.astype(np.float64) - exact).mean()
    err_r = np.abs(raw.astype(np.float64) - exact).mean()
    assert err_s < 0.25 * err_r
    # translation: O(V + off) - off tracks O(V) to the E4M3 error of offset-free V
    base = oracle.sage_attention(q, k, v, lay, causal, True, PV_FP8, sm, smooth_v=True)
    exact0 = oracle.attn_fp64(q, k, v, lay, causal, sm)
    err_0 = np.abs(base.astype(np.float64) - exact0).mean()
    assert err_s < 3 * err_0 + 1e-3


def test_smooth_v_rejected_in_fp16_mode():
    d = 16
    x = _rand16((1, 1, 4, d), 141)
    with pytest.raises(ValueError):
        oracle.sage_attention(x, x, x, Layout.dense(1, 1, 4, d), False, True, PV_FP16, 0.25,
                              smooth_v=True)


# Queries that are the last Nq positions of a longer sequence (Nq != Nk: prefill against
# cached keys, or decode with Nq = 1): the causal mask aligns at the bottom right, query i
# sees keys j <= i + Nk - Nq.

def _bottom_right_mask(nq, nk):
    i = np.arange(nq)[:, None]
    j = np.arange(nk)[None, :]
    return j <= i + (nk - nq)


@pytest.mark.parametrize("nq,nk", [(70, 200), (1, 130), (128, 128), (200, 70)])
@pytest.mark.parametrize("causal", [False, True])
def test_fp64_kv_matches_torch_sdpa_with_mask(nq, nk, causal):
    B, H, d = 1, 2, 16
    q = _rand16((B, H, nq, d), 151)
    k, v = _rand16((B, H, nk, d), 152), _rand16((B, H, nk, d), 153)
    sm = 1 / math.sqrt(d)
    got = oracle.attn_fp64(q, k, v, Layout.dense(B, H, nq, d), causal, sm,
                           kv_layout=Layout.dense(B, H, nk, d))
    mask = torch.from_numpy(_bottom_right_mask(nq, nk)) if causal else None
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(x.astype(np.float64)) for x in (q, k, v)), attn_mask=mask, scale=sm)
    ref = ref.numpy()
    if causal and nq > nk:        # rows without a visible key: zero here, NaN in torch
        dead = ~_bottom_right_mask(nq, nk).any(axis=1)
        assert dead.sum() == nq - nk
        assert np.all(got[:, :, dead] == 0)
        got, ref = got[:, :, ~dead], ref[:, :, ~dead]
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_kv_rows_are_the_tail_of_the_square_problem():
    # the last Nq queries of a causal square problem see exactly the keys the Nq x Nk
    # problem gives them: fp64 rows agree bit for bit
    N, nq, d = 300, 90, 32
    q, k, v = (_rand16((1, 1, N, d), s) for s in (161, 162, 163))
    sm = 1 / math.sqrt(d)
    full = oracle.attn_fp64(q, k, v, Layout.dense(1, 1, N, d), True, sm)
    tail = oracle.attn_fp64(np.ascontiguousarray(q[:, :, N - nq:]), k, v,
                            Layout.dense(1, 1, nq, d), True, sm,
                            kv_layout=Layout.dense(1, 1, N, d))
    assert np.array_equal(tail, full[:, :, N - nq:])


@pytest.mark.parametrize("pv_mode", [PV_FP16, PV_FP8])
def test_quantized_kv_decode_and_equal_lengths(pv_mode):
    d, nk = 64, 700
    k, v = _rand16((1, 2, nk, d), 171), _rand16((1, 2, nk, d), 172)
    kvl = Layout.dense(1, 2, nk, d)
    # decode: one query sees every key, so causal and non-causal agree exactly
    q1 = _rand16((1, 2, 1, d), 173)
    l1 = Layout.dense(1, 2, 1, d)
    a = oracle.sage_attention(q1, k, v, l1, True, True, pv_mode, kv_layout=kvl)
    b = oracle.sage_attention(q1, k, v, l1, False, True, pv_mode, kv_layout=kvl)
    assert np.array_equal(a, b)
    exact = oracle.attn_fp64(q1, k, v, l1, False, 1 / math.sqrt(d), kv_layout=kvl)
    assert _cos(a, exact) > (0.9999 if pv_mode == PV_FP16 else 0.999)
    # Nq = Nk through the separate layout is the self-attention path, bit for bit
    q = _rand16((1, 2, nk, d), 174)
    same = oracle.sage_attention(q, k, v, kvl, True, True, pv_mode, kv_layout=kvl)
    base = oracle.sage_attention(q, k, v, kvl, True, True, pv_mode)
    assert np.array_equal(same, base)


@pytest.mark.parametrize("causal", [False, True])
def test_quantized_kv_tracks_fp64(causal):
    nq, nk, d = 200, 900, 64
    q = _rand16((1, 2, nq, d), 181)
    k = (_rand16((1, 2, nk, d), 182).astype(np.float32) + _rand16((d,), 183, 2.0)).astype(np.float16)
    v = _rand16((1, 2, nk, d), 184)
    lq, lk = Layout.dense(1, 2, nq, d), Layout.dense(1, 2, nk, d)
    sm = 1 / math.sqrt(d)
    o = oracle.sage_attention(q, k, v, lq, causal, True, PV_FP16, sm, kv_layout=lk)
    exact = oracle.attn_fp64(q, k, v, lq, causal, sm, kv_layout=lk)
    assert _cos(o, exact) > 0.9999 and _rel_l1(o, exact) < 0.02
    # the K mean is taken over the keys, not the queries: using Q's length for it fails
    zq = oracle.quant_qk(q, k, lq, True, kv_layout=lk)
    mu = k.astype(np.float64).mean(axis=2).astype(np.float32)
    assert np.array_equal(zq["k_mean"], mu)


def test_quantized_kv_more_queries_than_keys():
    nq, nk, d = 300, 100, 32
    q = _rand16((1, 1, nq, d), 191)
    k, v = _rand16((1, 1, nk, d), 192), _rand16((1, 1, nk, d), 193)
    lq, lk = Layout.dense(1, 1, nq, d), Layout.dense(1, 1, nk, d)
    o = oracle.sage_attention(q, k, v, lq, True, True, PV_FP16, 0.2, kv_layout=lk)
    assert np.all(o[0, 0, :nq - nk] == 0)                 # no visible key
    exact = oracle.attn_fp64(q, k, v, lq, True, 0.2, kv_layout=lk)
    assert _cos(o[0, 0, nq - nk:], exact[0, 0, nq - nk:]) > 0.9999


def test_varlen_kv_equals_per_sequence_dense():
    H, d = 2, 32
    lq, lk = [70, 1, 129], [200, 333, 129]
    cq = np.concatenate([[0], np.cumsum(lq)])
    ck = np.concatenate([[0], np.cumsum(lk)])
    q = _rand16((int(cq[-1]), H, d), 201)
    k, v = _rand16((int(ck[-1]), H, d), 202), _rand16((int(ck[-1]), H, d), 203)
    o = oracle.sage_attention(q, k, v, Layout.packed(cq, H, d), True, True, PV_FP16, 0.2,
                              kv_layout=Layout.packed(ck, H, d))
    for s in range(3):
        sq, sk = slice(cq[s], cq[s + 1]), slice(ck[s], ck[s + 1])
        dq = np.ascontiguousarray(q[sq].transpose(1, 0, 2))[None]
        dk, dv = (np.ascontiguousarray(x[sk].transpose(1, 0, 2))[None] for x in (k, v))
        od = oracle.sage_attention(dq, dk, dv, Layout.dense(1, H, lq[s], d), True, True,
                                   PV_FP16, 0.2, kv_layout=Layout.dense(1, H, lk[s], d))
        assert np.array_equal(o[sq].transpose(1, 0, 2), od[0])


# Finer scale groups ([SA2] 技术方案 (2), restated for this tensor-core layout: one Q
# scale per query row and one K scale per 32 keys).

@pytest.mark.parametrize("pv_mode", [PV_FP16, PV_FP8])
def test_fine_single_tile_equals_plain_softmax(pv_mode):
    N, d = 200, 32
    q, k, v = (_rand16((1, 1, N, d), s) for s in (211, 212, 213))
    lay = Layout.dense(1, 1, N, d)
    sm = 1 / math.sqrt(d)
    z = oracle.quant_qk(q, k, lay, True, fine=True)
    if pv_mode == PV_FP8:
        vq, vs = oracle.quant_v_fp8(v, lay)
    else:
        vq, vs = v, None
    got = oracle.attn_quant(z["q_i8"], z["q_scale"], z["k_i8"], z["k_scale"], vq, vs, lay, False,
                            pv_mode, sm, tile_n=256, fine=True)
    # closed form with the scales expanded per row and per 32 keys
    qc = z["q_i8"][0, 0].astype(np.int64)
    kc = z["k_i8"][0, 0].astype(np.int64)
    S = qc @ kc.T
    t = (S * z["q_scale"][0, 0][:, None].astype(np.float64)
         * z["k_scale"][0, 0][np.arange(N) // 32][None, :].astype(np.float64) * sm / math.log(2))
    p = np.exp2(t - t.max(axis=1, keepdims=True))
    if pv_mode == PV_FP16:
        O = p.astype(np.float16).astype(np.float64) @ vq[0, 0].astype(np.float64) / p.sum(1, keepdims=True)
    else:
        P = torch.from_numpy(448 * p).to(torch.float32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
        vv = torch.from_numpy(vq[0, 0]).view(torch.float8_e4m3fn).to(torch.float64).numpy()
        O = P @ vv * vs[0, 0][None, :] / (448 * p.sum(1, keepdims=True))
    ref = O.astype(np.float16).astype(np.float64)
    diff = np.abs(got[0, 0].astype(np.float64) - ref)
    assert diff.max() <= 2 * np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64).max()


def _rounding_model(q, k, v, sm, q_rows, k_rows, draws, seed):
    """fp64 attention on Q and K moved by independent rounding errors, uniform within half
    a quantization step of the group each element belongs to (q_rows query rows or
    k_rows keys share one amax/127 scale; K is smoothed first, as it is quantized). It
    predicts the error a faithful per-group INT8 quantization leaves against fp64
    attention; returns (rel-L1, 1 - cos) per draw."""
    qf = q[0, 0].astype(np.float64)
    kf = k[0, 0].astype(np.float32) - k[0, 0].astype(np.float64).mean(axis=0).astype(np.float32)
    kf = kf.astype(np.float64)
    N = qf.shape[0]

    def steps(x, rows):
        assert N % rows == 0
        amax = np.abs(x).reshape(-1, rows, x.shape[1]).max(axis=(1, 2))
        return np.repeat(amax.astype(np.float32) / np.float32(127), rows)[:, None].astype(np.float64)

    sq, sk = steps(qf, q_rows), steps(kf, k_rows)
    exact = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(x.astype(np.float64)) for x in (q, k, v)), scale=sm).numpy()[0, 0]
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(draws):
        qe = qf + rng.uniform(-0.5, 0.5, qf.shape) * sq
        ke = kf + rng.uniform(-0.5, 0.5, kf.shape) * sk
        s = sm * qe @ ke.T
        p = np.exp(s - s.max(axis=1, keepdims=True))
        o = p @ v[0, 0].astype(np.float64) / p.sum(axis=1, keepdims=True)
        out.append((_rel_l1(o, exact), 1.0 - _cos(o, exact)))
    return np.array(out)


def test_fine_groups_error_matches_the_rounding_model_on_row_outliers():
    # Query rows of very different magnitude (1 in 16 is 96x louder) and K blocks with a
    # loud 32-key half. A code's error is at most half a step of its group's scale, so the
    # scores of a loud row carry errors ~96x larger than a quiet row's: the error of the
    # output concentrates in the loud rows whose two largest scores lie within that noise
    # of each other. The expected size of that error at a given scale granularity is what
    # fp64 attention on inputs moved by uniform half-step rounding errors gives; the
    # oracle's per-token / per-32-key groups must land within a factor 2 of that model's
    # mean relative L1 error (its draws spread over 0.7x-1.6x), and its cosine within the
    # model's worst draw (cosine is an L2 measure and heavy-tailed here: nearly all of the
    # squared error sits in the loud rows). One scale per 128 queries / 64 keys predicts
    # ~50x the error, so fine groups silently computed with block scales fail.
    N, d = 512, 64
    q, k, v = (_rand16((1, 1, N, d), s) for s in (221, 222, 223))
    rowmag = np.where(np.arange(N) % 16 == 0, 24.0, 0.25)
    q = (q.astype(np.float64) * rowmag[None, None, :, None]).astype(np.float16)
    kmag = np.where((np.arange(N) // 32) % 2 == 0, 6.0, 0.5)
    k = (k.astype(np.float64) * kmag[None, None, :, None]).astype(np.float16)
    lay = Layout.dense(1, 1, N, d)
    sm = 1 / math.sqrt(d)
    exact = oracle.attn_fp64(q, k, v, lay, False, sm)
    fine = oracle.sage_attention(q, k, v, lay, False, True, PV_FP16, sm, fine=True)
    block = oracle.sage_attention(q, k, v, lay, False, True, PV_FP16, sm)
    m_fine = _rounding_model(q, k, v, sm, 1, 32, 16, 7)
    m_block = _rounding_model(q, k, v, sm, 128, 64, 4, 8)
    assert m_block[:, 0].mean() > 10 * m_fine[:, 0].mean()      # the inputs separate the two
    r_fine, r_block = _rel_l1(fine, exact), _rel_l1(block, exact)
    assert 0.5 * m_fine[:, 0].mean() <= r_fine <= 2.0 * m_fine[:, 0].mean()
    assert 1.0 - _cos(fine, exact) <= m_fine[:, 1].max()
    assert 0.5 * m_block[:, 0].mean() <= r_block <= 2.0 * m_block[:, 0].mean()
    assert r_fine < 0.5 * r_block


# Smooth Q (「4比特量化三倍加速不掉点！清华即插即用的SageAttention迎来升级」, 技术方案 (1)): Q - mean(Q) is quantized and the
# vector-matrix product mean(Q) K^T is added back to the scores.

def _q_with_channel_offsets(N, d, seed, amp=8.0):
    q = _rand16((1, 2, N, d), seed).astype(np.float64)
    off = np.random.default_rng(seed + 1).uniform(-amp, amp, d)
    return (q + off).astype(np.float16)


def test_smooth_q_compensation_closed_form():
    N, d = 150, 32
    q = _q_with_channel_offsets(N, d, 231)
    k = (_rand16((1, 2, N, d), 232).astype(np.float64) + 3.0).astype(np.float16)
    lay = Layout.dense(1, 2, N, d)
    z = oracle.quant_qk(q, k, lay, True, smooth_q=True)
    muq = q.astype(np.float64).mean(axis=2).astype(np.float32)
    assert np.array_equal(z["q_mean"], muq)
    ks = k.astype(np.float32) - z["k_mean"][:, :, None, :]          # K as it is quantized
    ref = np.einsum("bhc,bhnc->bhn", muq.astype(np.float64), ks.astype(np.float64))
    assert np.allclose(z["q_comp"], ref, rtol=1e-6, atol=1e-6)
    # the Q codes reconstruct Q - mean(Q), not Q, within half a scale step
    qs = q.astype(np.float32) - muq[:, :, None, :]
    for blk in range(2):
        rows = slice(128 * blk, min(N, 128 * blk + 128))
        sc = z["q_scale"][:, :, blk][:, :, None, None]
        rec = sc * z["q_i8"][:, :, rows].astype(np.float32)
        assert np.all(np.abs(rec - qs[:, :, rows]) <= sc * 0.5001 + 1e-6)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("pv_mode", [PV_FP16, PV_FP8])
def test_smooth_q_single_tile_closed_form(causal, pv_mode):
    N, d = 200, 32
    q = _q_with_channel_offsets(N, d, 241)[:, :1]
    k, v = (_rand16((1, 1, N, d), s) for s in (242, 243))
    lay = Layout.dense(1, 1, N, d)
    sm = 1 / math.sqrt(d)
    z = oracle.quant_qk(q, k, lay, True, smooth_q=True)
    vq, vs = (oracle.quant_v_fp8(v, lay) if pv_mode == PV_FP8 else (v, None))
    got = oracle.attn_quant(z["q_i8"], z["q_scale"], z["k_i8"], z["k_scale"], vq, vs, lay,
                            causal, pv_mode, sm, tile_n=256, q_comp=z["q_comp"])
    qc = z["q_i8"][0, 0].astype(np.int64)
    kc = z["k_i8"][0, 0].astype(np.int64)
    sq = z["q_scale"][0, 0][np.arange(N) // 128].astype(np.float64)
    sk = z["k_scale"][0, 0][np.arange(N) // 64].astype(np.float64)
    t = ((qc @ kc.T) * sq[:, None] * sk[None, :] + z["q_comp"][0, 0][None, :]) * sm / math.log(2)
    if causal:
        t[np.triu_indices(N, 1)] = -np.inf
    p = np.exp2(t - t.max(axis=1, keepdims=True))
    if pv_mode == PV_FP16:
        O = p.astype(np.float16).astype(np.float64) @ v[0, 0].astype(np.float64) / p.sum(1, keepdims=True)
    else:
        P = torch.from_numpy(448 * p).to(torch.float32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
        vv = torch.from_numpy(vq[0, 0]).view(torch.float8_e4m3fn).to(torch.float64).numpy()
        O = P @ vv * vs[0, 0][None, :] / (448 * p.sum(1, keepdims=True))
    ref = O.astype(np.float16).astype(np.float64)
    diff = np.abs(got[0, 0].astype(np.float64) - ref)
    assert diff.max() <= 2 * np.spacing(np.abs(ref).astype(np.float16)).astype(np.float64).max()


@pytest.mark.parametrize("causal", [False, True])
def test_smooth_q_needs_its_compensation(causal):
    # with channel offsets in Q, smoothing Q keeps the scores' precision; dropping the
    # compensation (a plausible slip) changes the result completely
    N, d = 512, 64
    q = _q_with_channel_offsets(N, d, 251)
    k, v = (_rand16((1, 2, N, d), s) for s in (252, 253))
    lay = Layout.dense(1, 2, N, d)
    sm = 1 / math.sqrt(d)
    exact = oracle.attn_fp64(q, k, v, lay, causal, sm)
    sq = oracle.sage_attention(q, k, v, lay, causal, True, PV_FP16, sm, smooth_q=True)
    plain = oracle.sage_attention(q, k, v, lay, causal, True, PV_FP16, sm)
    assert _cos(sq, exact) > 0.9999 and _rel_l1(sq, exact) < 0.02
    assert _rel_l1(sq, exact) < 0.7 * _rel_l1(plain, exact)
    z = oracle.quant_qk(q, k, lay, True, smooth_q=True)
    dropped = oracle.attn_quant(z["q_i8"], z["q_scale"], z["k_i8"], z["k_scale"], v, None, lay,
                                causal, PV_FP16, sm)
    assert _rel_l1(dropped, exact) > 0.2


def test_smooth_q_is_a_no_op_for_zero_mean_q():
    # Q whose every channel sums to zero exactly: mean(Q) = 0, so the codes, the
    # compensation (all zero) and the output equal plain smooth-K attention bit for bit
    N, d = 256, 32
    h = _rand16((1, 1, N // 2, d), 261)
    q = np.concatenate([h, -h], axis=2)
    k, v = (_rand16((1, 1, N, d), s) for s in (262, 263))
    lay = Layout.dense(1, 1, N, d)
    z = oracle.quant_qk(q, k, lay, True, smooth_q=True)
    assert not z["q_mean"].any() and not z["q_comp"].any()
    a = oracle.sage_attention(q, k, v, lay, True, True, PV_FP16, smooth_q=True)
    b = oracle.sage_attention(q, k, v, lay, True, True, PV_FP16)
    assert np.array_equal(a, b)


def test_fp64_one_hot_dominant_score():
    # one key far ahead of the others: the output row is that key's V row
    N, d = 40, 16
    q = np.zeros((1, 1, 1, d), np.float16)
    q[..., 0] = 8
    k = _rand16((1, 1, N, d), 271, 0.01)
    k[0, 0, 17, 0] = 8                     # score 64 * sm above every other key
    v = _rand16((1, 1, N, d), 272)
    o = oracle.attn_fp64(q, k, v, Layout.dense(1, 1, 1, d), False, 1.0,
                         kv_layout=Layout.dense(1, 1, N, d))
    assert np.allclose(o[0, 0, 0], v[0, 0, 17].astype(np.float64), atol=1e-12)


def test_int8_scores_beat_e4m3_scores():
    # [SA1] 技术方案: INT8 per-block quantization of Q and K is more accurate for Q K^T than
    # E4M3 with the same blocks (amax mapped to 127 and to 448 respectively)
    N, d = 256, 64
    q, k = _rand16((1, 1, N, d), 281), _rand16((1, 1, N, d), 282)
    lay = Layout.dense(1, 1, N, d)
    exact = q[0, 0].astype(np.float64) @ k[0, 0].astype(np.float64).T
    z = oracle.quant_qk(q, k, lay, smooth_k=False)
    s_i8 = (z["q_i8"][0, 0].astype(np.int64) @ z["k_i8"][0, 0].astype(np.int64).T
            * z["q_scale"][0, 0][np.arange(N) // 128][:, None]
            * z["k_scale"][0, 0][np.arange(N) // 64][None, :])

    def e4m3_blocks(x, blk):
        out = np.empty(x.shape, np.float64)
        for b0 in range(0, x.shape[0], blk):
            xb = x[b0:b0 + blk].astype(np.float32)
            s = np.float32(np.abs(xb).max() / np.float32(448))
            codes = np.vectorize(lambda t: oracle.e4m3_encode(float(np.float32(t) / s)))(xb)
            out[b0:b0 + blk] = np.vectorize(oracle.e4m3_decode)(codes) * float(s)
        return out

    s_f8 = e4m3_blocks(q[0, 0], 128) @ e4m3_blocks(k[0, 0], 64).T
    err_i8 = np.abs(s_i8 - exact).mean()
    err_f8 = np.abs(s_f8 - exact).mean()
    assert err_i8 < 0.6 * err_f8


# ------------------------------------------------------------ split-K merge (R21, decode)


def _split_merge(z, v, nq, nk, d, causal, sm, split, round_p=True, weighted=True):
    """The decode path's arithmetic in fp64 from the oracle's codes (one head): keys in
    splits, P = f16(2^(t - m_split)), O_s = P V, l_s = sum p, merged with the weights
    2^(m_s - M). round_p=False keeps p unrounded; weighted=False drops the merge weights
    (a planted mistake)."""
    qi = z["q_i8"][0, 0].astype(np.int64)
    ki = z["k_i8"][0, 0].astype(np.int64)
    qs = np.float64(z["q_scale"][0, 0, 0])
    ks = z["k_scale"][0, 0].astype(np.float64)
    c = sm * math.log2(math.e)
    t = (qi @ ki.T).astype(np.float64) * qs * np.repeat(ks, 64)[:nk][None, :] * c
    if causal:
        vis = np.arange(nk)[None, :] <= np.arange(nq)[:, None] + nk - nq
        t = np.where(vis, t, -np.inf)
    vv = v[0, 0].astype(np.float64)
    out = np.zeros((nq, d))
    for i in range(nq):
        parts = []
        for k0 in range(0, nk, split):
            ts = t[i, k0:k0 + split]
            m = ts.max()
            if m == -np.inf:
                continue
            p = np.exp2(ts - m)
            pr = p.astype(np.float16).astype(np.float64) if round_p else p
            parts.append((m, p.sum(), pr @ vv[k0:k0 + split]))
        if not parts:
            continue
        M = max(m for m, _, _ in parts)
        w = [2.0 ** (m - M) if weighted else 1.0 for m, _, _ in parts]
        l = sum(wi * ls for wi, (_, ls, _) in zip(w, parts))
        out[i] = sum(wi * os_ for wi, (_, _, os_) in zip(w, parts)) / l
    return out


@pytest.mark.parametrize("nq,causal", [(1, True), (4, True), (3, False)])
def test_split_merge_matches_the_tile_walk(nq, causal):
    # R21: splitting the keys and merging (m_s, l_s, O_s) is the online softmax regrouped;
    # with p unrounded it equals one softmax exactly (fp64), and with P = f16(p) relative
    # to the split's maximum it stays within the bounds the GPU is held to against the
    # oracle's tile walk. Dropping the merge weights fails those bounds.
    nk, d = 1100, 64
    q = _rand16((1, 1, nq, d), 31 + nq)
    k = _rand16((1, 1, nk, d), 41 + nq)
    k = (k.astype(np.float32) + _rand16((1, 1, 1, d), 51, 2.0).astype(np.float32)).astype(np.float16)
    v = _rand16((1, 1, nk, d), 61 + nq)
    lq, lk = Layout.dense(1, 1, nq, d), Layout.dense(1, 1, nk, d)
    sm = 1.0 / math.sqrt(d)
    z = oracle.quant_qk(q, k, lq, True, kv_layout=lk)
    walk = oracle.attn_quant(z["q_i8"], z["q_scale"], z["k_i8"], z["k_scale"], v, None, lq,
                             causal, PV_FP16, sm, kv_layout=lk)[0, 0].astype(np.float64)
    one = _split_merge(z, v, nq, nk, d, causal, sm, split=nk, round_p=False)
    for split in (128, 256, 1024):
        exact = _split_merge(z, v, nq, nk, d, causal, sm, split, round_p=False)
        assert np.abs(exact - one).max() < 1e-12
        got = _split_merge(z, v, nq, nk, d, causal, sm, split)
        assert _cos(got, walk) >= 0.9999 and np.abs(got - walk).max() <= 1e-2, split
        bad = _split_merge(z, v, nq, nk, d, causal, sm, split, weighted=False)
        assert np.abs(bad - walk).max() > 1e-2, split
