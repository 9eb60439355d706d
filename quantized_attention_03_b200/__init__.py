"""Python binding of libsage.so, the B200 (sm_100a) SageAttention forward pass.

The C entry points declared in ``include/sage.h`` are exposed under the same names and
argument order (``sage_attn_fwd(q, k, v, out, B, H, N, d, causal, smooth_k, pv_mode,
sm_scale, stream)`` ...). Pointer arguments accept torch tensors (their device
pointer), plain integers or ``None``; ``stream=None`` means torch's current stream.
This module only marshals arguments: every step of the computation runs in the CUDA
library, and nothing falls back to another implementation. If the library is missing
the first call raises.

Convenience wrappers (``sageattn``, ``sageattn_varlen``, ``quant_qk``, ...) allocate
the output tensors with torch and call the same entry points.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsage.so")

SAGE_OK = 0
SAGE_ERR_INVALID_ARG = 1
SAGE_ERR_UNSUPPORTED = 2
SAGE_ERR_MISALIGNED = 3
SAGE_ERR_WORKSPACE = 4
SAGE_ERR_CUDA = 5
SAGE_ERR_TIMEOUT = 6
SAGE_ERR_BAD_SEQLENS = 7
SAGE_PV_FP16 = 0
SAGE_PV_FP8 = 1
SAGE_SMOOTH_K = 1     # flags of the fused entry points' smooth_k argument
SAGE_SMOOTH_V = 2
SAGE_SMOOTH_Q = 4
SAGE_QK_FINE = 8

Q_BLOCK = 128
K_BLOCK = 64
DECODE_MAX_Q = 16   # SAGE_DECODE_MAX_Q: most queries sage_attn_decode_quantized takes

# name -> (restype, argtypes) as declared in include/sage.h
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_Z = ctypes.c_size_t
_S = ctypes.c_int  # sage_status_t
SIGNATURES = {
    "sage_workspace_size": (_Z, [_I, _I, _I, _I, _I, _I]),
    "sage_attn_workspace_size": (_Z, [_I, _I, _I, _I, _I]),
    "sage_workspace_size_kv": (_Z, [_I, _I, _I, _I, _I, _I, _I, _I]),
    "sage_quant_qk_kv": (_S, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _Z,
                              _P]),
    "sage_attn_fwd_kv": (_S, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _P, _Z, _P]),
    "sage_attn_varlen_fwd_kv": (_S, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I,
                                     _I, _F, _P, _Z, _P]),
    "sage_attn_fwd_quantized_kv": (_S, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I,
                                        _I, _I, _F, _I, _P]),
    "sage_attn_decode_workspace_size": (_Z, [_I, _I, _I, _I, _I]),
    "sage_attn_decode_quantized": (_S, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I,
                                        _P, _Z, _P]),
    "sage_quant_qk": (_S, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "sage_quant_qk_ws": (_S, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _Z, _P]),
    "sage_quant_qk_varlen": (_S, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _I, _P]),
    "sage_quant_v_fp8": (_S, [_P, _P, _P, _I, _I, _I, _I, _P]),
    "sage_quant_v_fp8_varlen": (_S, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _P]),
    "sage_quant_v_fp8_smooth": (_S, [_P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "sage_quant_v_fp8_ws": (_S, [_P, _P, _P, _P, _I, _I, _I, _I, _P, _Z, _P]),
    "sage_quant_v_fp8_smooth_varlen": (_S, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P]),
    "sage_attn_fwd": (_S, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P]),
    "sage_attn_fwd_ws": (_S, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _Z, _P]),
    "sage_attn_varlen_fwd": (_S, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _P,
                                  _Z, _P]),
    "sage_attn_fwd_quantized": (_S, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F,
                                     _P]),
    "sage_attn_fwd_quantized_smooth_v": (_S, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I,
                                              _I, _F, _P]),
    "sage_debug_qk_int32": (_S, [_P, _P, _P, _I, _I, _I, _I, _P]),
    "sage_attn_fwd_noalloc": (_S, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P]),
    "sage_debug_wait_timeout": (_S, [ctypes.c_ulonglong, _P]),
    "sage_get_device_status": (_S, [_P]),
    "sage_status_string": (ctypes.c_char_p, [_I]),
    "sage_last_cuda_error": (_I, []),
    "sage_version": (_I, []),
}

_lib = None


class SageError(RuntimeError):
    def __init__(self, name: str, code: int):
        self.code = code
        msg = status_string(code) if _lib is not None else str(code)
        super().__init__(f"{name} failed: {msg} ({code})")


def lib() -> ctypes.CDLL:
    """Load libsage.so (built in-tree by ``build.py``); raise if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m quantized_attention_03_b200.build`"
                " (there is no fallback implementation)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().sage_status_string(int(code)).decode()


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s) -> Optional[int]:
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _call(name: str, *args):
    rc = getattr(lib(), name)(*args)
    if rc != SAGE_OK:
        raise SageError(name, rc)
    return rc


# ---------------------------------------------------------------- C-ABI names


def sage_workspace_size(nseq, H, max_seqlen, total_tokens, d, pv_mode) -> int:
    return int(lib().sage_workspace_size(nseq, H, max_seqlen, total_tokens, d, pv_mode))


def sage_attn_workspace_size(B, H, N, d, pv_mode) -> int:
    return int(lib().sage_attn_workspace_size(B, H, N, d, pv_mode))


def sage_workspace_size_kv(nseq, H, max_seqlen_q, max_seqlen_k, total_q, total_k, d,
                           pv_mode) -> int:
    return int(lib().sage_workspace_size_kv(nseq, H, max_seqlen_q, max_seqlen_k, total_q, total_k,
                                            d, pv_mode))


def sage_quant_qk_kv(q, k, q_i8, q_scale, k_i8, k_scale, k_mean, q_mean, q_comp, B, H, Nq, Nk,
                     d, flags, workspace=None, ws_bytes=0, stream=None):
    return _call("sage_quant_qk_kv", _ptr(q), _ptr(k), _ptr(q_i8), _ptr(q_scale), _ptr(k_i8),
                 _ptr(k_scale), _ptr(k_mean), _ptr(q_mean), _ptr(q_comp), B, H, Nq, Nk, d,
                 int(flags), _ptr(workspace), int(ws_bytes), _stream(stream))


def sage_attn_fwd_kv(q, k, v, out, B, H, Nq, Nk, d, causal, smooth_k, pv_mode, sm_scale,
                     workspace=None, ws_bytes=0, stream=None):
    return _call("sage_attn_fwd_kv", _ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, Nq, Nk, d,
                 int(causal), int(smooth_k), int(pv_mode), float(sm_scale), _ptr(workspace),
                 int(ws_bytes), _stream(stream))


def sage_attn_varlen_fwd_kv(q, k, v, out, cu_seqlens_q, cu_seqlens_k, nseq, total_q, total_k,
                            max_seqlen_q, max_seqlen_k, H, d, causal, smooth_k, pv_mode, sm_scale,
                            workspace=None, ws_bytes=0, stream=None):
    return _call("sage_attn_varlen_fwd_kv", _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                 _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), nseq, total_q, total_k, max_seqlen_q,
                 max_seqlen_k, H, d, int(causal), int(smooth_k), int(pv_mode), float(sm_scale),
                 _ptr(workspace), int(ws_bytes), _stream(stream))


def sage_attn_decode_workspace_size(B, H, Nq, Nk, d) -> int:
    return int(lib().sage_attn_decode_workspace_size(B, H, Nq, Nk, d))


def sage_attn_decode_quantized(q_i8, q_scale, k_i8, k_scale, v, out, B, H, Nq, Nk, d, causal,
                               sm_scale, flags, workspace, ws_bytes, stream=None):
    return _call("sage_attn_decode_quantized", _ptr(q_i8), _ptr(q_scale), _ptr(k_i8),
                 _ptr(k_scale), _ptr(v), _ptr(out), B, H, Nq, Nk, d, int(causal),
                 float(sm_scale), int(flags), _ptr(workspace), int(ws_bytes), _stream(stream))


def sage_attn_fwd_quantized_kv(q_i8, q_scale, k_i8, k_scale, v, v_scale, v_mean, q_comp, out, B,
                               H, Nq, Nk, d, causal, pv_mode, sm_scale, flags=0, stream=None):
    return _call("sage_attn_fwd_quantized_kv", _ptr(q_i8), _ptr(q_scale), _ptr(k_i8),
                 _ptr(k_scale), _ptr(v), _ptr(v_scale), _ptr(v_mean), _ptr(q_comp), _ptr(out), B,
                 H, Nq, Nk, d, int(causal), int(pv_mode), float(sm_scale), int(flags),
                 _stream(stream))


def sage_quant_qk(q, k, q_i8, q_scale, k_i8, k_scale, k_mean, B, H, N, d, smooth_k, stream=None):
    return _call("sage_quant_qk", _ptr(q), _ptr(k), _ptr(q_i8), _ptr(q_scale), _ptr(k_i8),
                 _ptr(k_scale), _ptr(k_mean), B, H, N, d, int(smooth_k), _stream(stream))


def sage_quant_qk_ws(q, k, q_i8, q_scale, k_i8, k_scale, k_mean, B, H, N, d, smooth_k, workspace,
                     ws_bytes, stream=None):
    return _call("sage_quant_qk_ws", _ptr(q), _ptr(k), _ptr(q_i8), _ptr(q_scale), _ptr(k_i8),
                 _ptr(k_scale), _ptr(k_mean), B, H, N, d, int(smooth_k), _ptr(workspace),
                 int(ws_bytes), _stream(stream))


def sage_quant_qk_varlen(q, k, cu_seqlens, nseq, total_tokens, max_seqlen, H, d, q_i8, q_scale,
                         k_i8, k_scale, k_mean, smooth_k, stream=None):
    return _call("sage_quant_qk_varlen", _ptr(q), _ptr(k), _ptr(cu_seqlens), nseq, total_tokens,
                 max_seqlen, H, d, _ptr(q_i8), _ptr(q_scale), _ptr(k_i8), _ptr(k_scale),
                 _ptr(k_mean), int(smooth_k), _stream(stream))


def sage_quant_v_fp8(v, v_e4m3, v_scale, B, H, N, d, stream=None):
    return _call("sage_quant_v_fp8", _ptr(v), _ptr(v_e4m3), _ptr(v_scale), B, H, N, d,
                 _stream(stream))


def sage_quant_v_fp8_varlen(v, cu_seqlens, nseq, total_tokens, max_seqlen, H, d, v_e4m3,
                            v_scale, stream=None):
    return _call("sage_quant_v_fp8_varlen", _ptr(v), _ptr(cu_seqlens), nseq, total_tokens,
                 max_seqlen, H, d, _ptr(v_e4m3), _ptr(v_scale), _stream(stream))


def sage_quant_v_fp8_ws(v, v_e4m3, v_scale, v_mean, B, H, N, d, workspace, ws_bytes,
                        stream=None):
    return _call("sage_quant_v_fp8_ws", _ptr(v), _ptr(v_e4m3), _ptr(v_scale), _ptr(v_mean), B, H,
                 N, d, _ptr(workspace), int(ws_bytes), _stream(stream))


def sage_quant_v_fp8_smooth(v, v_e4m3, v_scale, v_mean, B, H, N, d, stream=None):
    return _call("sage_quant_v_fp8_smooth", _ptr(v), _ptr(v_e4m3), _ptr(v_scale), _ptr(v_mean),
                 B, H, N, d, _stream(stream))


def sage_quant_v_fp8_smooth_varlen(v, cu_seqlens, nseq, total_tokens, max_seqlen, H, d, v_e4m3,
                                   v_scale, v_mean, stream=None):
    return _call("sage_quant_v_fp8_smooth_varlen", _ptr(v), _ptr(cu_seqlens), nseq,
                 total_tokens, max_seqlen, H, d, _ptr(v_e4m3), _ptr(v_scale), _ptr(v_mean),
                 _stream(stream))


def sage_attn_fwd(q, k, v, out, B, H, N, d, causal, smooth_k, pv_mode, sm_scale, stream=None):
    return _call("sage_attn_fwd", _ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, N, d, int(causal),
                 int(smooth_k), int(pv_mode), float(sm_scale), _stream(stream))


def sage_attn_fwd_ws(q, k, v, out, B, H, N, d, causal, smooth_k, pv_mode, sm_scale, workspace,
                     ws_bytes, stream=None):
    return _call("sage_attn_fwd_ws", _ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, N, d,
                 int(causal), int(smooth_k), int(pv_mode), float(sm_scale), _ptr(workspace),
                 int(ws_bytes), _stream(stream))


def sage_attn_varlen_fwd(q, k, v, out, cu_seqlens, nseq, total_tokens, max_seqlen, H, d, causal,
                         smooth_k, pv_mode, sm_scale, workspace=None, ws_bytes=0, stream=None):
    return _call("sage_attn_varlen_fwd", _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(cu_seqlens),
                 nseq, total_tokens, max_seqlen, H, d, int(causal), int(smooth_k), int(pv_mode),
                 float(sm_scale), _ptr(workspace), int(ws_bytes), _stream(stream))


def sage_attn_fwd_quantized(q_i8, q_scale, k_i8, k_scale, v, v_scale, out, B, H, N, d, causal,
                            pv_mode, sm_scale, stream=None):
    return _call("sage_attn_fwd_quantized", _ptr(q_i8), _ptr(q_scale), _ptr(k_i8), _ptr(k_scale),
                 _ptr(v), _ptr(v_scale), _ptr(out), B, H, N, d, int(causal), int(pv_mode),
                 float(sm_scale), _stream(stream))


def sage_attn_fwd_quantized_smooth_v(q_i8, q_scale, k_i8, k_scale, v_e4m3, v_scale, v_mean, out,
                                     B, H, N, d, causal, sm_scale, stream=None):
    return _call("sage_attn_fwd_quantized_smooth_v", _ptr(q_i8), _ptr(q_scale), _ptr(k_i8),
                 _ptr(k_scale), _ptr(v_e4m3), _ptr(v_scale), _ptr(v_mean), _ptr(out), B, H, N,
                 d, int(causal), float(sm_scale), _stream(stream))


def sage_debug_qk_int32(q_i8, k_i8, s_out, B, H, N, d, stream=None):
    return _call("sage_debug_qk_int32", _ptr(q_i8), _ptr(k_i8), _ptr(s_out), B, H, N, d,
                 _stream(stream))


def sage_attn_fwd_noalloc(q, k, v, out, B, H, N, d, causal, smooth_k, pv_mode, sm_scale,
                          stream=None):
    """sage_attn_fwd with the library's static scratch (no allocation; see sage.h)."""
    return _call("sage_attn_fwd_noalloc", _ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, N, d,
                 int(causal), int(smooth_k), int(pv_mode), float(sm_scale), _stream(stream))


def sage_debug_wait_timeout(timeout_ns, stream=None):
    return _call("sage_debug_wait_timeout", int(timeout_ns), _stream(stream))


def sage_get_device_status(stream=None) -> int:
    """Synchronize the stream and return (and clear) the device status code."""
    return int(lib().sage_get_device_status(_stream(stream)))


def sage_status_string(code: int) -> str:
    return status_string(code)


def sage_last_cuda_error() -> int:
    return int(lib().sage_last_cuda_error())


def sage_version() -> int:
    return int(lib().sage_version())


# ------------------------------------------------------------ torch conveniences


def _check_status(stream=None):
    code = sage_get_device_status(stream)
    if code != SAGE_OK:
        raise SageError("device", code)


def _smooth_flags(smooth_k: bool, smooth_v: bool, fine: bool = False,
                  smooth_q: bool = False) -> int:
    return ((SAGE_SMOOTH_K if smooth_k else 0) | (SAGE_SMOOTH_V if smooth_v else 0)
            | (SAGE_QK_FINE if fine else 0) | (SAGE_SMOOTH_Q if smooth_q else 0))


def sageattn(q, k, v, causal: bool = False, smooth_k: bool = True, pv_mode: int = SAGE_PV_FP16,
             sm_scale: float = 0.0, out=None, stream=None, smooth_v: bool = False,
             fine: bool = False, smooth_q: bool = False):
    """O = SageAttention(q, k, v) for fp16 CUDA tensors q [B, H, Nq, d], k and v
    [B, H, Nk, d] (Nq != Nk: sage_attn_fwd_kv, causal mask aligned at the bottom right)."""
    import torch
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    if out is None:
        out = torch.empty_like(q)
    flags = _smooth_flags(smooth_k, smooth_v, fine, smooth_q)
    if Nq == Nk:
        sage_attn_fwd(q, k, v, out, B, H, Nq, d, causal, flags, pv_mode, sm_scale, stream)
    else:
        sage_attn_fwd_kv(q, k, v, out, B, H, Nq, Nk, d, causal, flags, pv_mode, sm_scale, None, 0,
                         stream)
    return out


def sageattn_varlen_kv(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                       causal: bool = False, smooth_k: bool = True,
                       pv_mode: int = SAGE_PV_FP16, sm_scale: float = 0.0, out=None,
                       stream=None, smooth_v: bool = False, fine: bool = False,
                       smooth_q: bool = False):
    """Packed sequences with their own query and key lengths: q [Tq, H, d], k and v
    [Tk, H, d], cu_seqlens_q / cu_seqlens_k int32 [nseq+1] on the device. The options are
    sageattn's."""
    import torch
    Tq, H, d = q.shape
    Tk = k.shape[0]
    if out is None:
        out = torch.empty_like(q)
    sage_attn_varlen_fwd_kv(q, k, v, out, cu_seqlens_q, cu_seqlens_k, cu_seqlens_q.numel() - 1,
                            Tq, Tk, max_seqlen_q, max_seqlen_k, H, d, causal,
                            _smooth_flags(smooth_k, smooth_v, fine, smooth_q), pv_mode, sm_scale,
                            None, 0, stream)
    return out


def sageattn_varlen(q, k, v, cu_seqlens, max_seqlen: int, causal: bool = False,
                    smooth_k: bool = True, pv_mode: int = SAGE_PV_FP16, sm_scale: float = 0.0,
                    out=None, stream=None, smooth_v: bool = False, fine: bool = False,
                    smooth_q: bool = False):
    """SageAttention over packed sequences: q, k, v [T, H, d], cu_seqlens int32 [nseq+1].
    The options are sageattn's."""
    import torch
    T, H, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    sage_attn_varlen_fwd(q, k, v, out, cu_seqlens, cu_seqlens.numel() - 1, T, max_seqlen, H, d,
                         causal, _smooth_flags(smooth_k, smooth_v, fine, smooth_q), pv_mode,
                         sm_scale, None, 0, stream)
    return out


def quant_qk(q, k, smooth_k: bool = True, stream=None, fine: bool = False,
             smooth_q: bool = False):
    """Dense smooth-K + INT8: dict of q_i8, q_scale, k_i8, k_scale, k_mean (q [B,H,Nq,d]
    and k [B,H,Nk,d] may differ in length; fine: per-token Q and per-32-token K scales;
    smooth_q: also q_mean [B,H,d] and the score compensation q_comp [B,H,ceil(Nk/128)*128])."""
    import torch
    B, H, N, d = q.shape
    Nk = k.shape[2]
    dev = q.device
    qg, kg = (1, 32) if fine else (Q_BLOCK, K_BLOCK)
    z = dict(q_i8=torch.empty(q.shape, dtype=torch.int8, device=dev),
             q_scale=torch.empty((B, H, math.ceil(N / qg)), dtype=torch.float32, device=dev),
             k_i8=torch.empty(k.shape, dtype=torch.int8, device=dev),
             k_scale=torch.empty((B, H, math.ceil(Nk / kg)), dtype=torch.float32, device=dev),
             k_mean=torch.empty((B, H, d), dtype=torch.float32, device=dev))
    flags = ((SAGE_SMOOTH_K if smooth_k else 0) | (SAGE_QK_FINE if fine else 0)
             | (SAGE_SMOOTH_Q if smooth_q else 0))
    if smooth_q:
        z["q_mean"] = torch.empty((B, H, d), dtype=torch.float32, device=dev)
        z["q_comp"] = torch.empty((B, H, math.ceil(Nk / 128) * 128), dtype=torch.float32,
                                  device=dev)
    if N == Nk and not fine and not smooth_q:
        sage_quant_qk(q, k, z["q_i8"], z["q_scale"], z["k_i8"], z["k_scale"], z["k_mean"], B, H, N,
                      d, smooth_k, stream)
    else:
        sage_quant_qk_kv(q, k, z["q_i8"], z["q_scale"], z["k_i8"], z["k_scale"], z["k_mean"],
                         z.get("q_mean"), z.get("q_comp"), B, H, N, Nk, d, flags, None, 0, stream)
    return z


def quant_qk_varlen(q, k, cu_seqlens, max_seqlen: int, smooth_k: bool = True, stream=None,
                    fine: bool = False):
    import torch
    T, H, d = q.shape
    nseq = cu_seqlens.numel() - 1
    dev = q.device
    qg, kg = (1, 32) if fine else (Q_BLOCK, K_BLOCK)
    z = dict(q_i8=torch.empty(q.shape, dtype=torch.int8, device=dev),
             q_scale=torch.empty((nseq, H, math.ceil(max_seqlen / qg)), dtype=torch.float32,
                                 device=dev),
             k_i8=torch.empty(k.shape, dtype=torch.int8, device=dev),
             k_scale=torch.empty((nseq, H, math.ceil(max_seqlen / kg)), dtype=torch.float32,
                                 device=dev),
             k_mean=torch.empty((nseq, H, d), dtype=torch.float32, device=dev))
    flags = (SAGE_SMOOTH_K if smooth_k else 0) | (SAGE_QK_FINE if fine else 0)
    sage_quant_qk_varlen(q, k, cu_seqlens, nseq, T, max_seqlen, H, d, z["q_i8"], z["q_scale"],
                         z["k_i8"], z["k_scale"], z["k_mean"], flags, stream)
    return z


def quant_v_fp8(v, stream=None, smooth_v: bool = False):
    """Dense V -> (E4M3 codes as uint8 [B,H,N,d], per-channel scales [B,H,d]); with
    smooth_v, a third result: the channel mean of V [B,H,d] the codes are taken from."""
    import torch
    B, H, N, d = v.shape
    codes = torch.empty(v.shape, dtype=torch.uint8, device=v.device)
    scales = torch.empty((B, H, d), dtype=torch.float32, device=v.device)
    if not smooth_v:
        sage_quant_v_fp8(v, codes, scales, B, H, N, d, stream)
        return codes, scales
    mean = torch.empty((B, H, d), dtype=torch.float32, device=v.device)
    sage_quant_v_fp8_smooth(v, codes, scales, mean, B, H, N, d, stream)
    return codes, scales, mean


def quant_v_fp8_varlen(v, cu_seqlens, max_seqlen: int, stream=None, smooth_v: bool = False):
    import torch
    T, H, d = v.shape
    nseq = cu_seqlens.numel() - 1
    codes = torch.empty(v.shape, dtype=torch.uint8, device=v.device)
    scales = torch.empty((nseq, H, d), dtype=torch.float32, device=v.device)
    if not smooth_v:
        sage_quant_v_fp8_varlen(v, cu_seqlens, nseq, T, max_seqlen, H, d, codes, scales, stream)
        return codes, scales
    mean = torch.empty((nseq, H, d), dtype=torch.float32, device=v.device)
    sage_quant_v_fp8_smooth_varlen(v, cu_seqlens, nseq, T, max_seqlen, H, d, codes, scales, mean,
                                   stream)
    return codes, scales, mean


def attn_quantized(q_i8, q_scale, k_i8, k_scale, v, v_scale, causal: bool = False,
                   pv_mode: int = SAGE_PV_FP16, sm_scale: float = 0.0, out=None, stream=None,
                   v_mean=None, fine: bool = False, q_comp=None):
    """Step 3 on pre-quantized operands; v_mean (FP8 mode) selects the smooth-V epilogue,
    fine the per-token Q / per-32-token K scale layout, q_comp the smooth-Q compensation."""
    import torch
    B, H, N, d = q_i8.shape
    Nk = k_i8.shape[2]
    if out is None:
        out = torch.empty(q_i8.shape, dtype=torch.float16, device=q_i8.device)
    if Nk != N or fine or q_comp is not None:
        sage_attn_fwd_quantized_kv(q_i8, q_scale, k_i8, k_scale, v, v_scale, v_mean, q_comp, out,
                                   B, H, N, Nk, d, causal, pv_mode, sm_scale,
                                   SAGE_QK_FINE if fine else 0, stream)
        return out
    if v_mean is not None:
        if pv_mode != SAGE_PV_FP8:
            raise ValueError("v_mean needs the FP8 P.V mode")
        sage_attn_fwd_quantized_smooth_v(q_i8, q_scale, k_i8, k_scale, v, v_scale, v_mean, out,
                                         B, H, N, d, causal, sm_scale, stream)
        return out
    sage_attn_fwd_quantized(q_i8, q_scale, k_i8, k_scale, v, v_scale, out, B, H, N, d, causal,
                            pv_mode, sm_scale, stream)
    return out


def attn_decode(q_i8, q_scale, k_i8, k_scale, v, causal: bool = False, sm_scale: float = 0.0,
                out=None, stream=None, fine: bool = False, workspace=None):
    """Step 3 for a few queries (Nq <= DECODE_MAX_Q) on pre-quantized operands, FP16 P.V,
    split over the keys (sage_attn_decode_quantized); the workspace is allocated here
    unless given."""
    import torch
    B, H, Nq, d = q_i8.shape
    Nk = k_i8.shape[2]
    if out is None:
        out = torch.empty(q_i8.shape, dtype=torch.float16, device=q_i8.device)
    need = sage_attn_decode_workspace_size(B, H, Nq, Nk, d)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q_i8.device)
    sage_attn_decode_quantized(q_i8, q_scale, k_i8, k_scale, v, out, B, H, Nq, Nk, d, causal,
                               sm_scale, SAGE_QK_FINE if fine else 0, workspace,
                               workspace.numel() * workspace.element_size(), stream)
    return out


def qk_int32(q_i8, k_i8, stream=None):
    """Debug: the int32 score matrices S = q_i8 k_i8^T [B,H,N,N] from the tensor-core pass."""
    import torch
    B, H, N, d = q_i8.shape
    s = torch.zeros((B, H, N, N), dtype=torch.int32, device=q_i8.device)
    sage_debug_qk_int32(q_i8, k_i8, s, B, H, N, d, stream)
    return s
