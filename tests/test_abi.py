"""The C-ABI library: it loads, exports every symbol include/sage.h declares, and rejects
bad arguments on the host before anything is enqueued (no GPU needed: these calls return
before any CUDA call)."""
import os
import re

import pytest

import quantized_attention_03_b200 as sage

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sage.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SAGE_API\s+[\w\s\*]*?\b(sage_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from quantized_attention_03_b200 import build
    build.build()
    return sage.lib()


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("sage_quant_qk", "sage_attn_fwd", "sage_attn_varlen_fwd", "sage_get_device_status"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name
        assert name in sage.SIGNATURES, f"binding lacks {name}"
        assert callable(getattr(sage, name)), name


def test_status_strings(lib):
    assert sage.status_string(0) == "SAGE_OK"
    assert sage.status_string(6) == "SAGE_ERR_TIMEOUT"
    assert sage.sage_version() >= 100


FAKE = 0x10000          # 16-byte aligned, never dereferenced: validation fails first
MIS = 0x10008           # 8-byte aligned only


def _fwd(lib, q=FAKE, k=FAKE, v=FAKE, o=FAKE, B=1, H=1, N=128, d=64, pv=0, smooth=1):
    return lib.sage_attn_fwd(q, k, v, o, B, H, N, d, 0, smooth, pv, 0.0, None)


def test_host_validation(lib):
    assert _fwd(lib, d=96) == sage.SAGE_ERR_UNSUPPORTED
    assert _fwd(lib, d=256) == sage.SAGE_ERR_UNSUPPORTED
    assert _fwd(lib, N=-1) == sage.SAGE_ERR_INVALID_ARG
    assert _fwd(lib, pv=2) == sage.SAGE_ERR_INVALID_ARG
    assert _fwd(lib, q=0) == sage.SAGE_ERR_INVALID_ARG
    assert _fwd(lib, v=MIS) == sage.SAGE_ERR_MISALIGNED
    assert _fwd(lib, o=MIS) == sage.SAGE_ERR_MISALIGNED
    assert _fwd(lib, H=70000) == sage.SAGE_ERR_UNSUPPORTED


def test_smoothing_flags(lib):
    # smooth V needs FP8 P.V (fp16 V is never quantized); unknown bits are rejected
    assert _fwd(lib, smooth=sage.SAGE_SMOOTH_V, pv=0) == sage.SAGE_ERR_UNSUPPORTED
    assert _fwd(lib, smooth=3, pv=0) == sage.SAGE_ERR_UNSUPPORTED
    assert _fwd(lib, smooth=16, pv=1) == sage.SAGE_ERR_INVALID_ARG
    # the self-attention quantization entry points take smooth K and the finer groups only
    assert lib.sage_quant_qk(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64,
                             sage.SAGE_SMOOTH_Q, None) == sage.SAGE_ERR_INVALID_ARG
    # smooth Q needs the mean and compensation outputs
    assert lib.sage_quant_qk_kv(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 1, 1, 128,
                                256, 64, sage.SAGE_SMOOTH_Q, None, 0, None) == \
        sage.SAGE_ERR_INVALID_ARG
    assert _fwd(lib, smooth=-1, pv=1) == sage.SAGE_ERR_INVALID_ARG
    assert _fwd(lib, smooth=3, pv=1, q=0) == sage.SAGE_ERR_INVALID_ARG      # flags accepted
    assert lib.sage_attn_fwd_noalloc(FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, 0, 2, 0, 0.0,
                                     None) == sage.SAGE_ERR_UNSUPPORTED
    # the pre-quantized smooth-V entry needs the V mean
    assert lib.sage_attn_fwd_quantized_smooth_v(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE,
                                                1, 1, 128, 64, 0, 0.0, None) == \
        sage.SAGE_ERR_INVALID_ARG
    assert lib.sage_quant_v_fp8_smooth(FAKE, FAKE, FAKE, None, 1, 1, 128, 64, None) == \
        sage.SAGE_ERR_INVALID_ARG


def test_size_limits(lib):
    # token counts are int32: B*N past 2^31 - 1 is refused before anything is enqueued
    assert _fwd(lib, B=65535, N=65536) == sage.SAGE_ERR_UNSUPPORTED
    assert lib.sage_attn_fwd_kv(FAKE, FAKE, FAKE, FAKE, 2, 1, 128, 2 ** 30 + 1, 64, 0, 1, 0, 0.0,
                                None, 0, None) == sage.SAGE_ERR_UNSUPPORTED
    assert lib.sage_attn_fwd_kv(FAKE, FAKE, FAKE, FAKE, 1, 1, 128, -1, 64, 0, 1, 0, 0.0, None, 0,
                                None) == sage.SAGE_ERR_INVALID_ARG
    # workspace sizes grow with the shapes and are zero for negative ones
    assert lib.sage_workspace_size_kv(1, 1, 128, 256, 128, 256, 64, 0) > \
        lib.sage_workspace_size_kv(1, 1, 128, 128, 128, 128, 64, 0)
    assert lib.sage_workspace_size_kv(-1, 1, 128, 256, 128, 256, 64, 0) == 0
    # the dense-layout form is the general one with total_tokens = B*N
    for pv in (0, 1):
        assert lib.sage_attn_workspace_size(2, 4, 300, 128, pv) == \
            lib.sage_workspace_size(2, 4, 300, 600, 128, pv)
    assert lib.sage_attn_workspace_size(-1, 4, 300, 128, 0) == 0
    assert lib.sage_attn_workspace_size(65535, 1, 65536, 64, 0) == 0   # B*N past int32


def test_empty_inputs_are_noops(lib):
    assert _fwd(lib, B=0) == sage.SAGE_OK
    assert _fwd(lib, N=0) == sage.SAGE_OK
    assert _fwd(lib, q=0, B=0) == sage.SAGE_OK
    assert lib.sage_quant_qk(0, 0, 0, 0, 0, 0, 0, 0, 4, 128, 64, 1, None) == sage.SAGE_OK


def test_workspace_checks(lib):
    need = lib.sage_workspace_size(2, 4, 300, 600, 128, 0)
    need8 = lib.sage_workspace_size(2, 4, 300, 600, 128, 1)
    # Q and K codes (one byte per element each) plus scales, means and fp64 sums
    assert need >= 2 * 600 * 4 * 128 and need8 >= need + 600 * 4 * 128
    rc = lib.sage_attn_fwd_ws(FAKE, FAKE, FAKE, FAKE, 2, 4, 300, 128, 0, 1, 0, 0.0, FAKE,
                              need - 1, None)
    assert rc == sage.SAGE_ERR_WORKSPACE
    rc = lib.sage_attn_fwd_ws(FAKE, FAKE, FAKE, FAKE, 2, 4, 300, 128, 0, 1, 0, 0.0, 0, 0, None)
    assert rc == sage.SAGE_ERR_WORKSPACE
    rc = lib.sage_attn_fwd_ws(FAKE, FAKE, FAKE, FAKE, 2, 4, 300, 128, 0, 1, 0, 0.0, FAKE + 16,
                              need, None)
    assert rc == sage.SAGE_ERR_MISALIGNED       # scratch must be 256-byte aligned


def test_varlen_requires_cu_seqlens(lib):
    rc = lib.sage_attn_varlen_fwd(FAKE, FAKE, FAKE, FAKE, 0, 2, 100, 60, 4, 64, 1, 1, 0, 0.0,
                                  0, 0, None)
    assert rc == sage.SAGE_ERR_INVALID_ARG


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(sage, "LIB_PATH", str(tmp_path / "absent.so"))
    monkeypatch.setattr(sage, "_lib", None)
    with pytest.raises(RuntimeError, match="no fallback"):
        sage.lib()


def _dec(lib, q=FAKE, o=FAKE, ws=FAKE, ws_bytes=1 << 30, B=1, H=2, Nq=1, Nk=700, d=128,
         flags=0):
    return lib.sage_attn_decode_quantized(q, FAKE, FAKE, FAKE, FAKE, o, B, H, Nq, Nk, d, 1, 0.0,
                                          flags, ws, ws_bytes, None)


def test_decode_host_validation(lib):
    # a few queries only, FP16 P.V, d 64 or 128; every check before anything is enqueued
    assert _dec(lib, Nq=17) == sage.SAGE_ERR_UNSUPPORTED
    assert _dec(lib, d=96) == sage.SAGE_ERR_UNSUPPORTED
    assert _dec(lib, Nk=-1) == sage.SAGE_ERR_INVALID_ARG
    assert _dec(lib, flags=sage.SAGE_SMOOTH_Q) == sage.SAGE_ERR_INVALID_ARG
    assert _dec(lib, q=0) == sage.SAGE_ERR_INVALID_ARG
    assert _dec(lib, ws=0) == sage.SAGE_ERR_INVALID_ARG
    assert _dec(lib, o=MIS) == sage.SAGE_ERR_MISALIGNED
    assert _dec(lib, ws=MIS) == sage.SAGE_ERR_MISALIGNED
    need = lib.sage_attn_decode_workspace_size(1, 2, 1, 700, 128)
    assert _dec(lib, ws_bytes=need - 1) == sage.SAGE_ERR_WORKSPACE
    assert _dec(lib, B=0) == sage.SAGE_OK and _dec(lib, Nq=0) == sage.SAGE_OK


def test_decode_workspace_size(lib):
    # per (sequence, head, split, query): the split's max, its sum and d output sums (fp32);
    # whole 128-key splits, so the size is a multiple of (2 + d) * 4 * B * H * Nq
    for B, H, Nq, Nk, d in ((1, 2, 1, 700, 128), (8, 32, 1, 32768, 128), (2, 3, 16, 4100, 64)):
        n = lib.sage_attn_decode_workspace_size(B, H, Nq, Nk, d)
        unit = (2 + d) * 4 * B * H * Nq
        assert n > 0 and n % unit == 0
        nsplit = n // unit
        assert 1 <= nsplit <= -(-Nk // 128)
    assert lib.sage_attn_decode_workspace_size(1, 1, 17, 100, 64) == 0
    assert lib.sage_attn_decode_workspace_size(1, 1, 1, 0, 64) == 0
    assert lib.sage_attn_decode_workspace_size(1, 1, 1, 100, 96) == 0
