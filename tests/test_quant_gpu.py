"""GPU K-QUANT vs the oracle, through the C ABI: INT8 codes, block scales, K means and
E4M3 V codes must match bit for bit (the K mean is an exact fp64 sum rounded once, so
smoothed-K codes need no +-1 allowance on these inputs)."""
import numpy as np
import pytest
import torch

import oracle
import quantized_attention_03_b200 as sage
from quantized_attention_03_b200 import inputs

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().cpu().numpy()


def _check_qk(z, ref, what):
    assert np.array_equal(_np(z["q_scale"]), ref["q_scale"]), f"{what}: q_scale"
    assert np.array_equal(_np(z["q_i8"]), ref["q_i8"]), f"{what}: q_i8"
    assert np.array_equal(_np(z["k_mean"]), ref["k_mean"]), f"{what}: k_mean"
    assert np.array_equal(_np(z["k_scale"]), ref["k_scale"]), f"{what}: k_scale"
    assert np.array_equal(_np(z["k_i8"]), ref["k_i8"]), f"{what}: k_i8"


DENSE_CASES = [
    (1, 2, 256, 64, True),
    (1, 2, 256, 64, False),
    (2, 3, 300, 128, True),      # ragged: 2 full Q blocks + 44 rows
    (1, 1, 1, 64, True),
    (1, 2, 17, 128, True),
    (1, 2, 129, 64, True),
]


@pytest.mark.parametrize("B,H,N,d,smooth", DENSE_CASES)
def test_quant_qk_bit_exact(B, H, N, d, smooth):
    w = inputs.Workload("t", 7 + N + d, B, H, N, d, False, 2.0)
    q, k, _ = inputs.make_dense(w)
    z = sage.quant_qk(q.cuda(), k.cuda(), smooth)
    assert sage.sage_get_device_status() == 0
    ref = oracle.quant_qk(q.numpy(), k.numpy(), oracle.Layout.dense(B, H, N, d), smooth)
    _check_qk(z, ref, f"{B}x{H}x{N}x{d}")


def test_quant_qk_edge_values():
    B, H, N, d = 1, 2, 384, 128
    g = torch.Generator().manual_seed(5)
    q = torch.randn((B, H, N, d), generator=g).half()
    k = torch.randn((B, H, N, d), generator=g).half()
    q[0, 0, 128:256] = 0                    # an all-zero Q block
    k[0, 1, 64:128] = 3.0                   # a constant K block
    q[0, 1, 5, 7] = 65504.0                 # extreme magnitudes
    q[0, 1, 6, 9] = -65504.0
    k[0, 0, 300, 3] = 60000.0
    z = sage.quant_qk(q.cuda(), k.cuda(), True)
    ref = oracle.quant_qk(q.numpy(), k.numpy(), oracle.Layout.dense(B, H, N, d), True)
    _check_qk(z, ref, "edge")
    assert float(z["q_scale"][0, 0, 1]) == 0.0


@pytest.mark.parametrize("d", [64, 128])
def test_quant_v_fp8_bit_exact(d):
    B, H, N = 2, 2, 300
    w = inputs.Workload("t", 11, B, H, N, d, False, 1.0)
    _, _, v = inputs.make_dense(w)
    v[0, 1, :, 5] = 0                       # an all-zero channel
    codes, scales = sage.quant_v_fp8(v.cuda())
    rc, rs = oracle.quant_v_fp8(v.numpy(), oracle.Layout.dense(B, H, N, d))
    assert np.array_equal(_np(scales), rs)
    assert np.array_equal(_np(codes), rc)


def test_quant_varlen_bit_exact():
    H, d = 4, 128
    lens = [1, 127, 128, 129, 700, 64]
    w = inputs.Workload("t", 21, 0, H, 0, d, True, 2.0, nseq=len(lens))
    q, k, v, cu = inputs.make_varlen(w, lens=lens)
    maxlen = max(lens)
    cu_d = cu.cuda()
    z = sage.quant_qk_varlen(q.cuda(), k.cuda(), cu_d, maxlen, True)
    lay = oracle.Layout.packed(cu.tolist(), H, d)
    ref = oracle.quant_qk(q.numpy(), k.numpy(), lay, True)
    _check_qk(z, ref, "varlen")
    codes, scales = sage.quant_v_fp8_varlen(v.cuda(), cu_d, maxlen)
    rc, rs = oracle.quant_v_fp8(v.numpy(), lay)
    assert np.array_equal(_np(scales), rs)
    assert np.array_equal(_np(codes), rc)
    assert sage.sage_get_device_status() == 0


@pytest.mark.parametrize("name", ["llm_prefill", "video_dit"])
def test_quant_full_size_configs(name):
    w = getattr(inputs, name)()
    q, k, v = inputs.make_dense(w)
    z = sage.quant_qk(q.cuda(), k.cuda(), True)
    ref = oracle.quant_qk(q.numpy(), k.numpy(), oracle.Layout.dense(w.B, w.H, w.N, w.d), True)
    _check_qk(z, ref, name)
    if "fp8" in w.pv_modes:
        codes, scales = sage.quant_v_fp8(v.cuda())
        rc, rs = oracle.quant_v_fp8(v.numpy(), oracle.Layout.dense(w.B, w.H, w.N, w.d))
        assert np.array_equal(_np(scales), rs) and np.array_equal(_np(codes), rc)


def test_bad_cu_seqlens_sets_device_status():
    H, d = 2, 64
    q = torch.zeros((100, H, d), dtype=torch.float16, device="cuda")
    cu = torch.tensor([0, 60, 40, 100], dtype=torch.int32, device="cuda")   # not monotonic
    sage.quant_qk_varlen(q, q, cu, 60, True)
    assert sage.sage_get_device_status() == sage.SAGE_ERR_BAD_SEQLENS
    assert sage.sage_get_device_status() == sage.SAGE_OK                   # cleared


def test_quant_qk_ws_matches_allocating_entry():
    B, H, N, d = 2, 4, 700, 128
    w = inputs.Workload("t", 77, B, H, N, d, False, 2.0)
    q, k, _ = (t.cuda() for t in inputs.make_dense(w))
    ref = sage.quant_qk(q, k, True)
    got = {name: torch.empty_like(t) for name, t in ref.items()}
    ws = torch.empty(B * H * d * 8, dtype=torch.uint8, device="cuda")
    sage.sage_quant_qk_ws(q, k, got["q_i8"], got["q_scale"], got["k_i8"], got["k_scale"],
                          got["k_mean"], B, H, N, d, True, ws, ws.numel())
    assert sage.sage_get_device_status() == 0
    for name in ref:
        assert torch.equal(got[name], ref[name]), name
    with pytest.raises(sage.SageError):
        sage.sage_quant_qk_ws(q, k, got["q_i8"], got["q_scale"], got["k_i8"], got["k_scale"],
                              got["k_mean"], B, H, N, d, True, ws, ws.numel() - 8)


def _v_with_offsets(B, H, N, d, seed):
    w = inputs.Workload("t", seed, B, H, N, d, False, 1.0)
    _, _, v = inputs.make_dense(w)
    g = torch.Generator().manual_seed(seed)
    v = (v.float() + torch.randn(d, generator=g) * 8.0).half()   # channel offsets
    v[0, 0, :, 1] = 2.5                     # a constant channel: V - mean = 0
    v[0, -1, :, 2] = 0                      # an all-zero channel
    v[-1, 0, :, 3] = -v[-1, 0, :, 3].abs() - 1.0   # an all-negative channel
    return v


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 300])
def test_quant_v_fp8_smooth_bit_exact(d, N):
    B, H = 2, 2
    v = _v_with_offsets(B, H, N, d, 31 + d + N)
    codes, scales, mean = sage.quant_v_fp8(v.cuda(), smooth_v=True)
    lay = oracle.Layout.dense(B, H, N, d)
    rm = oracle.v_mean(v.numpy(), lay)
    rc, rs = oracle.quant_v_fp8(v.numpy(), lay, mu=rm)
    assert np.array_equal(_np(mean), rm)
    assert np.array_equal(_np(scales), rs)
    assert np.array_equal(_np(codes), rc)
    assert sage.sage_get_device_status() == 0


def test_quant_v_fp8_smooth_varlen_bit_exact():
    H, d = 3, 128
    lens = [1, 129, 640, 0, 64]
    w = inputs.Workload("t", 41, 0, H, 0, d, True, 2.0, nseq=len(lens))
    _, _, v, cu = inputs.make_varlen(w, lens=lens)
    v = (v.float() + torch.linspace(-30, 30, d)).half()
    codes, scales, mean = sage.quant_v_fp8_varlen(v.cuda(), cu.cuda(), max(lens), smooth_v=True)
    lay = oracle.Layout.packed(cu.tolist(), H, d)
    rm = oracle.v_mean(v.numpy(), lay)
    rc, rs = oracle.quant_v_fp8(v.numpy(), lay, mu=rm)
    assert np.array_equal(_np(mean), rm)
    assert np.array_equal(_np(scales), rs)
    assert np.array_equal(_np(codes), rc)
    assert sage.sage_get_device_status() == 0


@pytest.mark.parametrize("Nq,Nk,d", [(1, 300, 128), (130, 1000, 64), (300, 100, 128)])
def test_quant_qk_kv_bit_exact(Nq, Nk, d):
    B, H = 2, 3
    w = inputs.Workload("t", 51 + Nq, B, H, Nk, d, True, 2.0, nq=Nq)
    q, k, _ = inputs.make_dense(w)
    assert q.shape[2] == Nq and k.shape[2] == Nk
    z = sage.quant_qk(q.cuda(), k.cuda(), True)
    assert sage.sage_get_device_status() == 0
    ref = oracle.quant_qk(q.numpy(), k.numpy(), oracle.Layout.dense(B, H, Nq, d), True,
                          kv_layout=oracle.Layout.dense(B, H, Nk, d))
    _check_qk(z, ref, f"kv {Nq}x{Nk}")


def test_quant_v_fp8_ws_matches_allocating_entries():
    B, H, N, d = 2, 3, 500, 128
    v = _v_with_offsets(B, H, N, d, 61).cuda()
    ws = torch.empty(B * H * d * 16, dtype=torch.uint8, device="cuda")
    for smooth in (False, True):
        ref = sage.quant_v_fp8(v, smooth_v=smooth)
        codes = torch.empty_like(ref[0])
        scales = torch.empty_like(ref[1])
        mean = torch.empty_like(ref[1]) if smooth else None
        sage.sage_quant_v_fp8_ws(v, codes, scales, mean, B, H, N, d, ws, ws.numel())
        assert sage.sage_get_device_status() == 0
        assert torch.equal(codes, ref[0]) and torch.equal(scales, ref[1])
        if smooth:
            assert torch.equal(mean, ref[2])
    with pytest.raises(sage.SageError):
        sage.sage_quant_v_fp8_ws(v, codes, scales, None, B, H, N, d, ws, ws.numel() - 16)


FINE_CASES = [(1, 2, 256, 64, 256), (2, 3, 300, 128, 300), (1, 2, 17, 128, 17),
              (2, 2, 200, 64, 700), (1, 1, 1, 128, 33)]


@pytest.mark.parametrize("B,H,Nq,d,Nk", FINE_CASES)
def test_quant_qk_fine_bit_exact(B, H, Nq, d, Nk):
    w = inputs.Workload("t", 81 + Nq + Nk, B, H, Nk, d, False, 2.0, nq=Nq)
    q, k, _ = inputs.make_dense(w)
    z = sage.quant_qk(q.cuda(), k.cuda(), True, fine=True)
    assert sage.sage_get_device_status() == 0
    ref = oracle.quant_qk(q.numpy(), k.numpy(), oracle.Layout.dense(B, H, Nq, d), True,
                          kv_layout=oracle.Layout.dense(B, H, Nk, d), fine=True)
    _check_qk(z, ref, f"fine {B}x{H}x{Nq}x{Nk}x{d}")


def test_quant_fine_varlen_bit_exact():
    H, d = 4, 128
    lens = [1, 127, 128, 0, 700, 33]
    w = inputs.Workload("t", 88, 0, H, 0, d, True, 2.0, nseq=len(lens))
    q, k, v, cu = inputs.make_varlen(w, lens=lens)
    z = sage.quant_qk_varlen(q.cuda(), k.cuda(), cu.cuda(), max(lens), True, fine=True)
    assert sage.sage_get_device_status() == 0
    ref = oracle.quant_qk(q.numpy(), k.numpy(), oracle.Layout.packed(cu.tolist(), H, d), True,
                          fine=True)
    _check_qk(z, ref, "fine varlen")


@pytest.mark.parametrize("Nq,Nk,d,fine", [(300, 300, 128, False), (129, 700, 64, True),
                                          (1, 200, 128, False)])
def test_quant_smooth_q(Nq, Nk, d, fine):
    B, H = 2, 2
    w = inputs.Workload("t", 121 + Nq, B, H, Nk, d, False, 2.0, nq=Nq)
    q, k, _ = inputs.make_dense(w)
    g = torch.Generator().manual_seed(122)
    q = (q.float() + (torch.rand(d, generator=g) * 2 - 1) * 8.0).half()   # Q channel offsets
    z = sage.quant_qk(q.cuda(), k.cuda(), True, fine=fine, smooth_q=True)
    assert sage.sage_get_device_status() == 0
    ref = oracle.quant_qk(q.numpy(), k.numpy(), oracle.Layout.dense(B, H, Nq, d), True,
                          kv_layout=oracle.Layout.dense(B, H, Nk, d), fine=fine, smooth_q=True)
    _check_qk(z, ref, f"smooth Q {Nq}x{Nk}")
    assert np.array_equal(_np(z["q_mean"]), ref["q_mean"])
    comp = _np(z["q_comp"])
    assert comp.shape == (B, H, (Nk + 127) // 128 * 128)
    assert not comp[:, :, Nk:].any()                     # padding past the keys is zero
    scale = np.abs(ref["q_comp"]).max()
    assert np.abs(comp[:, :, :Nk] - ref["q_comp"]).max() <= 1e-5 * scale
