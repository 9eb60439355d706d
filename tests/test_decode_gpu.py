"""The decode path (sage_attn_decode_quantized: Nq <= 16 queries, keys split over many
CTAs and the splits merged) vs the oracle, through the C ABI.

The codes come from the library's own quantization pass (bit-exact with the oracle's), so
the comparison covers the split-K attention: the quantized oracle within cosine >= 0.9999
and max |err| <= 1e-2, exact fp64 attention within cosine >= 0.999 and relative L1 <= 0.02,
and the tensor-core path on the same codes within the same bounds.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import quantized_attention_03_b200 as sage
from quantized_attention_03_b200 import inputs
from helpers import assert_vs_fp64, assert_vs_oracle

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().cpu().numpy()


def _decode(q, k, v, causal, fine):
    z = sage.quant_qk(q.cuda(), k.cuda(), True, fine=fine)
    out = sage.attn_decode(z["q_i8"], z["q_scale"], z["k_i8"], z["k_scale"], v.cuda(), causal,
                           fine=fine)
    status = sage.sage_get_device_status()
    assert status == 0, sage.status_string(status)
    return z, out


CASES = [
    # Nq, Nk, d, causal, fine
    (1, 1, 128, False, False), (1, 700, 128, True, False), (3, 129, 64, True, False),
    (16, 1000, 128, True, False), (16, 4100, 64, False, False), (5, 2000, 128, True, True),
    (1, 5000, 64, False, True), (16, 10, 128, True, False), (7, 1025, 128, False, False),
]


@pytest.mark.parametrize("Nq,Nk,d,causal,fine", CASES)
def test_decode_matches_oracle(Nq, Nk, d, causal, fine):
    B, H = 2, 3
    w = inputs.Workload("t", 700 + Nq + Nk, B, H, Nk, d, causal, 2.0, nq=Nq)
    q, k, v = inputs.make_dense(w)
    z, out = _decode(q, k, v, causal, fine)
    got = _np(out)
    lq, lk = oracle.Layout.dense(B, H, Nq, d), oracle.Layout.dense(B, H, Nk, d)
    ref = oracle.sage_attention(q.numpy(), k.numpy(), v.numpy(), lq, causal, True,
                                oracle.PV_FP16, kv_layout=lk, fine=fine)
    tag = f"decode Nq={Nq} Nk={Nk} d={d} causal={causal} fine={fine}"
    assert_vs_oracle(got, ref, tag)
    exact = oracle.attn_fp64(q.numpy(), k.numpy(), v.numpy(), lq, causal, 1 / math.sqrt(d),
                             kv_layout=lk)
    assert_vs_fp64(got, exact, False, tag)
    # the tensor-core path on the same codes
    tc = sage.attn_quantized(z["q_i8"], z["q_scale"], z["k_i8"], z["k_scale"], v.cuda(), None,
                             causal, sage.SAGE_PV_FP16, fine=fine)
    assert sage.sage_get_device_status() == 0
    assert_vs_oracle(got, _np(tc), tag + " vs tensor-core path")
    if causal and Nq > Nk:
        assert not got[:, :, :Nq - Nk].any()          # queries that see no key


def test_decode_no_keys_and_reused_workspace():
    # no keys: zeros; one workspace serves calls of different shapes up to its size
    B, H, d = 1, 2, 64
    q8 = torch.zeros((B, H, 4, d), dtype=torch.int8, device="cuda")
    qs = torch.ones((B, H, 1), device="cuda")
    out = torch.full((B, H, 4, d), 7.0, dtype=torch.float16, device="cuda")
    rc = sage.sage_attn_decode_quantized(q8, qs, q8, qs, out, out, B, H, 4, 0, d, True, 0.0, 0,
                                         None, 0)
    assert rc == sage.SAGE_OK and not out.any()
    big = sage.sage_attn_decode_workspace_size(2, 3, 16, 4100, 128)
    ws = torch.empty(big, dtype=torch.uint8, device="cuda")
    for Nq, Nk, dd in ((16, 4100, 128), (2, 300, 64), (16, 4100, 128)):
        w = inputs.Workload("t", 900 + Nq + Nk, 2, 3, Nk, dd, True, 2.0, nq=Nq)
        q, k, v = inputs.make_dense(w)
        z = sage.quant_qk(q.cuda(), k.cuda(), True)
        got = sage.attn_decode(z["q_i8"], z["q_scale"], z["k_i8"], z["k_scale"], v.cuda(), True,
                               workspace=ws)
        ref = sage.attn_decode(z["q_i8"], z["q_scale"], z["k_i8"], z["k_scale"], v.cuda(), True)
        assert sage.sage_get_device_status() == 0
        assert torch.equal(got, ref), (Nq, Nk, dd)       # same plan, same arithmetic


def test_decode_full_size_sampled():
    # a decode step of B=8 H=32 against 32768 cached keys (d=128), in the benchmark's
    # launch configuration; heads sampled against the oracle
    w = inputs.decode()
    q, k, v = inputs.make_dense(w)
    z, out = _decode(q, k, v, w.causal, False)
    got = _np(out)
    for s, h in ((0, 0), (w.B - 1, w.H - 1), (w.B // 2, 7)):
        # the oracle gets just that head (one contiguous block of each tensor)
        hq, hk, hv = (x[s:s + 1, h:h + 1].numpy() for x in (q, k, v))
        hlq = oracle.Layout.dense(1, 1, w.nq, w.d)
        hlk = oracle.Layout.dense(1, 1, w.N, w.d)
        ref = oracle.sage_attention(hq, hk, hv, hlq, w.causal, True, oracle.PV_FP16,
                                    kv_layout=hlk)
        tag = f"decode head {s},{h}"
        assert_vs_oracle(got[s:s + 1, h:h + 1], ref, tag)
        exact = oracle.attn_fp64(hq, hk, hv, hlq, w.causal, 1 / math.sqrt(w.d), kv_layout=hlk)
        assert_vs_fp64(got[s:s + 1, h:h + 1], exact, False, tag)
