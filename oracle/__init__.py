"""CPU oracle for the SageAttention forward pass (TEST INFRASTRUCTURE ONLY).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package. It wraps the plain-C restatement in ``sage_oracle.c`` (which
shares nothing with the CUDA library) and adds the per-head bookkeeping for the two
tensor layouts:

* dense  ``[B, H, N, d]`` (the layout of the ``scaled_dot_product_attention`` call the
  method replaces: 「SageAttention：低比特量化Attention，实现推理加速」, section "即插即用举例");
* packed varlen ``[T, H, d]`` with ``cu_seqlens`` (sequence s holds tokens
  ``cu[s]:cu[s+1]``); every per-head quantity (K mean, blocks, causal mask, V scale)
  is taken within one sequence.

Scales are returned as ``[nseq, H, nblk]`` with ``nblk = ceil(maxlen / blk)`` (dense:
nseq = B, maxlen = N); unused trailing entries are 0. K means and V scales are
``[nseq, H, d]``. Outputs of sampled calls are NaN outside the sampled heads/rows.
"""
from __future__ import annotations

import ctypes
import math
from dataclasses import dataclass
from typing import Iterable, List, Optional, Sequence, Tuple

import numpy as np

from . import build as _build

Q_BLOCK = 128   # Q tokens per INT8 scale block
K_BLOCK = 64    # K tokens per INT8 scale block
Q_FINE = 1      # finer groups: one Q scale per token ...
K_FINE = 32     # ... and one K scale per 32 tokens
PV_FP16 = 0
PV_FP8 = 1

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        i32 = ctypes.c_int
        f64 = ctypes.c_double
        L.oracle_head_channel_mean.argtypes = [P, i64, i64, i32, P]
        L.oracle_head_quant_int8.argtypes = [P, P, i64, i64, i32, i32, P, P]
        L.oracle_head_quant_v_fp8.argtypes = [P, P, i64, i64, i32, P, P]
        L.oracle_head_attn_quant.argtypes = [P, P, P, P, P, P, P, P, i64, i64, i64, i32, i32,
                                             i32, f64, i32, i32, i32, i64, i64, P]
        L.oracle_head_q_comp.argtypes = [P, P, P, i64, i64, i32, P]
        L.oracle_head_attn_fp64.argtypes = [P, P, P, i64, i64, i64, i32, i32, f64, i64, i64, P]
        L.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
        L.oracle_f16_to_f64.restype = f64
        L.oracle_round_f16.argtypes = [f64]
        L.oracle_round_f16.restype = f64
        L.oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_to_f64.restype = f64
        L.oracle_e4m3_encode.argtypes = [f64]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_num_threads.restype = i32
        _lib = L
    return _lib


def num_threads() -> int:
    return int(lib().oracle_num_threads())


# ------------------------------------------------------------------ layouts


@dataclass
class Layout:
    """Where each (sequence, head) lives in a flat buffer of one tensor."""
    nseq: int
    H: int
    d: int
    maxlen: int
    stride: int                      # elements between consecutive tokens of one head
    starts: List[int]                # token offset of each sequence
    lens: List[int]
    varlen: bool

    @staticmethod
    def dense(B: int, H: int, N: int, d: int) -> "Layout":
        return Layout(B, H, d, N, d, [0] * B, [N] * B, False)

    @staticmethod
    def packed(cu_seqlens: Sequence[int], H: int, d: int) -> "Layout":
        cu = [int(x) for x in cu_seqlens]
        lens = [cu[i + 1] - cu[i] for i in range(len(cu) - 1)]
        return Layout(len(lens), H, d, max(lens) if lens else 0, H * d, cu[:-1], lens, True)

    def offset(self, s: int, h: int) -> int:
        """Element offset of token 0 of head h of sequence s."""
        if self.varlen:
            return (self.starts[s] * self.H + h) * self.d
        return ((s * self.H) + h) * self.maxlen * self.d

    def heads(self, sel: Optional[Iterable[Tuple[int, int]]] = None):
        if sel is None:
            sel = [(s, h) for s in range(self.nseq) for h in range(self.H)]
        return [(s, h, self.offset(s, h), self.lens[s]) for (s, h) in sel]

    def nblk(self, blk: int) -> int:
        return max(1, math.ceil(self.maxlen / blk))


def _ptr(a: np.ndarray, off_elems: int = 0) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data + off_elems * a.itemsize


def _bits16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x)
    assert x.dtype == np.float16
    return x.view(np.uint16)


# ------------------------------------------------------------------ number formats


def round_f16(x: float) -> float:
    return lib().oracle_round_f16(float(x))


def e4m3_encode(x: float) -> int:
    return int(lib().oracle_e4m3_encode(float(x)))


def e4m3_decode(b: int) -> float:
    return lib().oracle_e4m3_to_f64(int(b))


def f16_to_f64(bits: int) -> float:
    return lib().oracle_f16_to_f64(int(bits))


# ------------------------------------------------------------------ method steps


def channel_mean(x: np.ndarray, layout: Layout, heads=None) -> np.ndarray:
    """Per-channel token mean of K (smooth K) or V (smooth V) for every (or each
    selected) (sequence, head): [nseq, H, d] fp32."""
    xb = _bits16(x)
    mu = np.zeros((layout.nseq, layout.H, layout.d), np.float32)
    for s, h, off, n in layout.heads(heads):
        lib().oracle_head_channel_mean(_ptr(xb, off), n, layout.stride, layout.d,
                                       _ptr(mu, (s * layout.H + h) * layout.d))
    return mu


k_mean = channel_mean
v_mean = channel_mean


def quant_int8(x: np.ndarray, layout: Layout, blk: int, mu: Optional[np.ndarray] = None,
               heads=None):
    """Per-block INT8 codes (same shape as x) and scales [nseq, H, nblk]."""
    xb = _bits16(x)
    codes = np.zeros(x.shape, np.int8)
    nb = layout.nblk(blk)
    scales = np.zeros((layout.nseq, layout.H, nb), np.float32)
    for s, h, off, n in layout.heads(heads):
        mup = _ptr(mu, (s * layout.H + h) * layout.d) if mu is not None else None
        lib().oracle_head_quant_int8(_ptr(xb, off), mup, n, layout.stride, layout.d, blk,
                                     _ptr(codes, off), _ptr(scales, (s * layout.H + h) * nb))
    return codes, scales


def q_comp(k: np.ndarray, kv_layout: Layout, muk: Optional[np.ndarray], muq: np.ndarray,
           heads=None) -> np.ndarray:
    """Smooth-Q compensation mean(Q) K^T per key: [nseq, H, maxlen_k] fp32."""
    kb = _bits16(k)
    comp = np.zeros((kv_layout.nseq, kv_layout.H, kv_layout.maxlen), np.float32)
    for s, h, off, n in kv_layout.heads(heads):
        sh = s * kv_layout.H + h
        mkp = _ptr(muk, sh * kv_layout.d) if muk is not None else None
        lib().oracle_head_q_comp(_ptr(kb, off), mkp, _ptr(muq, sh * kv_layout.d), n,
                                 kv_layout.stride, kv_layout.d, _ptr(comp, sh * kv_layout.maxlen))
    return comp


def quant_qk(q: np.ndarray, k: np.ndarray, layout: Layout, smooth_k: bool = True, heads=None,
             kv_layout: Optional[Layout] = None, fine: bool = False, smooth_q: bool = False):
    """Smooth K, then per-block INT8 of Q (128 tokens) and K (64 tokens), for every (or
    each selected) head; with ``fine``, one Q scale per token and one K scale per 32
    tokens. ``kv_layout`` places K when it has its own lengths (default: Q's layout).
    ``smooth_q``: Q - mean(Q) is quantized and the compensation mean(Q) K^T is returned
    as ``q_comp`` [nseq, H, maxlen_k] (with the Q mean as ``q_mean``)."""
    kvl = layout if kv_layout is None else kv_layout
    zeros = np.zeros((kvl.nseq, kvl.H, kvl.d), np.float32)
    mu = k_mean(k, kvl, heads) if smooth_k else zeros
    muq = channel_mean(q, layout, heads) if smooth_q else None
    q_i8, q_scale = quant_int8(q, layout, Q_FINE if fine else Q_BLOCK, muq, heads)
    k_i8, k_scale = quant_int8(k, kvl, K_FINE if fine else K_BLOCK, mu if smooth_k else None,
                               heads)
    z = dict(q_i8=q_i8, q_scale=q_scale, k_i8=k_i8, k_scale=k_scale, k_mean=mu)
    if smooth_q:
        z["q_mean"] = muq
        z["q_comp"] = q_comp(k, kvl, mu if smooth_k else None, muq, heads)
    return z


def quant_v_fp8(v: np.ndarray, layout: Layout, heads=None, mu: Optional[np.ndarray] = None):
    """E4M3 codes of V - mu (same shape) and per-channel scales [nseq, H, d]; mu is the
    channel mean of V [nseq, H, d] for smooth V, None for none."""
    vb = _bits16(v)
    codes = np.zeros(v.shape, np.uint8)
    scales = np.zeros((layout.nseq, layout.H, layout.d), np.float32)
    for s, h, off, n in layout.heads(heads):
        sh = (s * layout.H + h) * layout.d
        mup = _ptr(mu, sh) if mu is not None else None
        lib().oracle_head_quant_v_fp8(_ptr(vb, off), mup, n, layout.stride, layout.d,
                                      _ptr(codes, off), _ptr(scales, sh))
    return codes, scales


def attn_quant(q_i8, q_scale, k_i8, k_scale, v, v_scale, layout: Layout, causal: bool,
               pv_mode: int, sm_scale: float, tile_n: int = 128, heads=None,
               rows: Optional[Tuple[int, int]] = None,
               v_mean: Optional[np.ndarray] = None,
               kv_layout: Optional[Layout] = None, fine: bool = False,
               q_comp: Optional[np.ndarray] = None) -> np.ndarray:
    """Quantized attention from codes and scales; fp16 output, NaN where not computed.
    ``fine``: the scales are per Q token and per 32 K tokens (quant_qk(fine=True));
    ``q_comp`` [nseq, H, maxlen_k]: the smooth-Q compensation added to the scores.

    ``v`` is fp16 V (FP16 mode) or its E4M3 codes as uint8 (FP8 mode); ``v_mean``
    [nseq, H, d] (FP8 mode, smooth V) is added to every output row. ``kv_layout`` places
    K and V when their lengths differ from Q's (causal masks align at the bottom right)."""
    kvl = layout if kv_layout is None else kv_layout
    assert kvl.stride == layout.stride and kvl.nseq == layout.nseq
    out = np.full(q_i8.shape, np.nan, np.float16)
    ob = out.view(np.uint16)
    if pv_mode == PV_FP16:
        vv = _bits16(v)
    else:
        vv = np.ascontiguousarray(v)
        assert vv.dtype == np.uint8
    nqb, nkb = q_scale.shape[2], k_scale.shape[2]
    r0, r1 = rows if rows is not None else (0, layout.maxlen)
    for (s, h, off, n), (_, _, koff, nk) in zip(layout.heads(heads), kvl.heads(heads)):
        sh = s * layout.H + h
        vsp = _ptr(v_scale, sh * layout.d) if v_scale is not None else None
        vmp = _ptr(v_mean, sh * layout.d) if v_mean is not None else None
        cp = _ptr(q_comp, sh * kvl.maxlen) if q_comp is not None else None
        lib().oracle_head_attn_quant(_ptr(q_i8, off), _ptr(q_scale, sh * nqb), _ptr(k_i8, koff),
                                     _ptr(k_scale, sh * nkb), _ptr(vv, koff), vsp, vmp, cp, n, nk,
                                     layout.stride, layout.d, int(causal), int(pv_mode),
                                     float(sm_scale), int(tile_n),
                                     Q_FINE if fine else Q_BLOCK, K_FINE if fine else K_BLOCK,
                                     r0, r1, _ptr(ob, off))
    return out


def attn_fp64(q, k, v, layout: Layout, causal: bool, sm_scale: float, heads=None,
              rows: Optional[Tuple[int, int]] = None,
              kv_layout: Optional[Layout] = None) -> np.ndarray:
    """Exact attention in fp64 (inputs of any float dtype, upcast exactly); ``kv_layout``
    as in attn_quant."""
    kvl = layout if kv_layout is None else kv_layout
    assert kvl.stride == layout.stride and kvl.nseq == layout.nseq
    qf, kf, vf = (np.asarray(x).reshape(-1) for x in (q, k, v))
    out = np.full(np.shape(q), np.nan, np.float64)
    of = out.reshape(-1)
    r0, r1 = rows if rows is not None else (0, layout.maxlen)
    st, d = layout.stride, layout.d
    for (s, h, off, n), (_, _, koff, nk) in zip(layout.heads(heads), kvl.heads(heads)):
        # only the selected head's span of each tensor is widened to fp64 (the whole
        # tensors can be GBs); rows outside [r0, r1) stay NaN
        span_q = (n - 1) * st + d if n > 0 else 0
        span_k = (nk - 1) * st + d if nk > 0 else 0
        q64 = np.ascontiguousarray(qf[off:off + span_q], np.float64)
        k64 = np.ascontiguousarray(kf[koff:koff + span_k], np.float64)
        v64 = np.ascontiguousarray(vf[koff:koff + span_k], np.float64)
        o64 = np.full(span_q, np.nan, np.float64)
        if span_q:
            lib().oracle_head_attn_fp64(_ptr(q64), _ptr(k64) if span_k else 0,
                                        _ptr(v64) if span_k else 0, n, nk, st, d,
                                        int(causal), float(sm_scale), r0, r1, _ptr(o64))
        seg = of[off:off + span_q]
        np.copyto(seg, o64, where=~np.isnan(o64))
    return out


def default_sm_scale(d: int, sm_scale: Optional[float] = None) -> float:
    return float(sm_scale) if sm_scale is not None and sm_scale > 0 else 1.0 / math.sqrt(d)


def sage_attention(q, k, v, layout: Layout, causal: bool = False, smooth_k: bool = True,
                   pv_mode: int = PV_FP16, sm_scale: Optional[float] = None,
                   tile_n: int = 128, heads=None, rows=None,
                   smooth_v: bool = False, kv_layout: Optional[Layout] = None,
                   fine: bool = False, smooth_q: bool = False) -> np.ndarray:
    """The whole method from fp16 Q, K, V: smooth K (and, in FP8 mode, optionally V;
    optionally Q, with the mean(Q) K^T compensation), quantize, quantized attention.
    ``kv_layout`` places K and V when their lengths differ from Q's; ``fine`` selects
    per-token Q and per-32-token K scales."""
    if smooth_v and pv_mode != PV_FP8:
        raise ValueError("smooth V applies to the FP8 P.V mode")
    kvl = layout if kv_layout is None else kv_layout
    sm = default_sm_scale(layout.d, sm_scale)
    z = quant_qk(q, k, layout, smooth_k, heads, kvl, fine, smooth_q)
    qc = z.get("q_comp")
    if pv_mode == PV_FP8:
        vm = channel_mean(v, kvl, heads) if smooth_v else None
        v8, vs = quant_v_fp8(v, kvl, heads, vm)
        return attn_quant(z["q_i8"], z["q_scale"], z["k_i8"], z["k_scale"], v8, vs, layout,
                          causal, PV_FP8, sm, tile_n, heads, rows, vm, kvl, fine, qc)
    return attn_quant(z["q_i8"], z["q_scale"], z["k_i8"], z["k_scale"], v, None, layout,
                      causal, PV_FP16, sm, tile_n, heads, rows, None, kvl, fine, qc)
