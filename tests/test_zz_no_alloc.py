"""The allocation-free entry point sage_attn_fwd_noalloc, through the C ABI.

It serves callers that cannot allocate device memory while they run (for example a
serving process whose own allocator owns all GPU memory after start-up) and have no
scratch buffer of their own. Its scratch is a static device array inside the library,
shared by every call and keeping the previous call's contents. It runs the same kernels
as the allocating entry point sage_attn_fwd on the same inputs, so its output must be
the same bytes: three calls in a row with different shapes and modes (a large FP8 call,
then a smaller FP16 one, then a smaller FP8 one with smooth V that finds the large
call's statistics still in the array) are each compared bit for bit. A stale scale or
mean left in the array would change some output bits. This file is collected last so a
failure here cannot hide the other tests' results.
"""
import pytest
import torch

import quantized_attention_03_b200 as sage
from quantized_attention_03_b200 import inputs
from helpers import assert_vs_oracle

pytestmark = pytest.mark.gpu


def _inputs(B, H, N, d, seed):
    w = inputs.Workload("no-alloc", seed, B, H, N, d, False, 2.0)
    return [t.cuda() for t in inputs.make_dense(w)]


def test_noalloc_matches_allocating_entry_point_on_three_calls():
    smooth_kv = sage.SAGE_SMOOTH_K | sage.SAGE_SMOOTH_V
    cases = [
        # B, H, N, d, causal, pv_mode, flags
        (1, 8, 1500, 128, True, sage.SAGE_PV_FP8, sage.SAGE_SMOOTH_K),
        (2, 4, 700, 64, False, sage.SAGE_PV_FP16, sage.SAGE_SMOOTH_K),
        (1, 3, 900, 128, False, sage.SAGE_PV_FP8, smooth_kv),
    ]
    for seed, (B, H, N, d, causal, pv, flags) in enumerate(cases):
        q, k, v = _inputs(B, H, N, d, 300 + seed)
        assert sage.sage_workspace_size(B, H, N, B * N, d, pv) <= 64 * 1024 * 1024
        ref = torch.empty_like(q)
        sage.sage_attn_fwd(q, k, v, ref, B, H, N, d, causal, flags, pv, 0.0)
        got = torch.full_like(q, float("nan"))
        sage.sage_attn_fwd_noalloc(q, k, v, got, B, H, N, d, causal, flags, pv, 0.0)
        assert sage.sage_get_device_status() == sage.SAGE_OK
        if not torch.equal(got, ref):
            # say how far apart they are before failing
            assert_vs_oracle(got.cpu().numpy(), ref.cpu().numpy(), f"no-alloc call {seed}")
            raise AssertionError(f"no-alloc call {seed}: output differs from sage_attn_fwd "
                                 f"in {(got != ref).sum().item()} elements")


def test_noalloc_rejects_requests_beyond_its_scratch():
    B, H, N, d = 2, 32, 16384, 128          # needs ~270 MB of scratch, more than 64 MiB
    q = torch.empty((16,), dtype=torch.float16, device="cuda")   # never read: rejected first
    rc = sage.lib().sage_attn_fwd_noalloc(q.data_ptr(), q.data_ptr(), q.data_ptr(),
                                          q.data_ptr(), B, H, N, d, 0, 1, 0, 0.0, None)
    assert rc == sage.SAGE_ERR_WORKSPACE
