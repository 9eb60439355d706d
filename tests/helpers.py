"""Shared helpers for the tests: accuracy metrics and the stated parity bounds.

Bounds (the method's accuracy targets for this implementation):
  vs the quantized oracle (same method, fp64 arithmetic): cosine >= 0.9999 and
      max |error| <= 1e-2 on the fp16 output;
  vs exact fp64 attention: cosine >= 0.999 and relative L1 <= 0.02 (FP16 PV mode).
FP8 PV mode cannot meet relative L1 <= 0.02 against fp64 on N(0,1) data: E4M3 keeps 3
mantissa bits, which alone costs about 2.5% relative L1 per operand; it is held to the
cosine bound against fp64 and to both bounds against the quantized oracle, and its
relative L1 is reported.
"""
import numpy as np

COS_VS_ORACLE = 0.9999
MAXABS_VS_ORACLE = 1e-2
COS_VS_FP64 = 0.999
RELL1_VS_FP64 = 0.02


def cos(a, b) -> float:
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b) + 1e-300))


def rel_l1(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.abs(a - b).sum() / (np.abs(b).sum() + 1e-300))


def max_abs(a, b) -> float:
    return float(np.max(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64))))


def assert_vs_oracle(gpu, ref, what=""):
    c, m = cos(gpu, ref), max_abs(gpu, ref)
    assert np.isfinite(np.asarray(gpu, np.float64)).all(), f"{what}: non-finite output"
    assert c >= COS_VS_ORACLE and m <= MAXABS_VS_ORACLE, f"{what}: cos={c:.6f} max_abs={m:.3g}"
    return c, m


def assert_vs_fp64(gpu, exact, fp8: bool, what=""):
    c, r = cos(gpu, exact), rel_l1(gpu, exact)
    assert c >= COS_VS_FP64, f"{what}: cos={c:.6f} rel_l1={r:.4f}"
    if not fp8:
        assert r <= RELL1_VS_FP64, f"{what}: cos={c:.6f} rel_l1={r:.4f}"
    return c, r
