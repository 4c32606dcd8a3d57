"""Shared checks of the GPU results against the fp64 oracle.

Acceptance (element by element):
  * fp32 result before rounding:  |Yf32 - Y_ref| <= 1e-3 * S + 1e-6,
    S = sum_k |X[m,k] W[n,k]| (the stated fp32 tolerance of the method);
  * bf16 result: within 1 bf16 ulp of round_bf16(Y_ref), ulps counted in
    the ordered integer encoding (so power-of-two boundaries and signs count
    right; +0 and -0 are equal) -- or, where the two stated tolerances
    disagree (outputs far smaller than S, whose fp32 error allowance spans
    several bf16 ulps), the correct rounding of SOME value inside the fp32
    bound: round(Y_ref - B) <= y <= round(Y_ref + B) in bf16 order,
    B = 1e-3 * S + 1e-6.  Any fp32 result meeting the fp32 bound, rounded once,
    meets this; a 1-ulp bound alone is unattainable there for any fp32
    accumulation order.
"""
import numpy as np
import torch

import oracle

ATOL = 1e-6
RTOL_S = 1e-3


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def ordered(bits: np.ndarray) -> np.ndarray:
    b = bits.astype(np.int64)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def ulp_distance(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    return np.abs(ordered(a_bits) - ordered(b_bits))


def check_full(x, w, y, yf32=None, Y_ref=None, S=None, what=""):
    """Compare complete outputs with the oracle; returns (max |err|/bound, max ulp)."""
    if Y_ref is None:
        Y_ref, S = oracle.gemm_ref(x.cpu(), w.cpu())
    worst = 0.0
    if yf32 is not None:
        yf = yf32.detach().cpu().double().numpy()
        bound = RTOL_S * S + ATOL
        err = np.abs(yf - Y_ref)
        ratio = err / bound
        bad = np.argwhere(~(err <= bound))
        assert bad.size == 0, (f"{what}: fp32 outside bound at {bad[:5].tolist()}: got {yf[tuple(bad[0])]}, "
                               f"ref {Y_ref[tuple(bad[0])]}, bound {bound[tuple(bad[0])]}")
        worst = float(ratio.max()) if ratio.size else 0.0
    got = bf16_bits(y)
    ok, d = bf16_ok(got, Y_ref, S)
    bad = np.argwhere(~ok)
    assert bad.size == 0, (f"{what}: bf16 off at {bad[:5].tolist()} "
                           f"(got {hex(int(got[tuple(bad[0])]))}, ref {hex(int(oracle.round_bf16(Y_ref)[tuple(bad[0])]))}, "
                           f"ulps {int(d[tuple(bad[0])])})")
    return worst, int(d.max()) if d.size else 0


def bf16_ok(got_bits, Y_ref, S):
    """Element-wise bf16 acceptance (see the module docstring) and ulp distances."""
    d = ulp_distance(got_bits, oracle.round_bf16(Y_ref))
    B = RTOL_S * S + ATOL
    lo = ordered(oracle.round_bf16(Y_ref - B))
    hi = ordered(oracle.round_bf16(Y_ref + B))
    g = ordered(got_bits)
    return (d <= 1) | ((g >= lo) & (g <= hi)), d


def check_sampled(x, w, y, yf32, ms, ns, what=""):
    """Compare sampled outputs (ms[i], ns[i]) with the oracle computed one by one."""
    Y_ref, S = oracle.gemm_ref_sampled(x.cpu(), w.cpu(), ms, ns)
    yc = y.detach().cpu()
    got_bits = bf16_bits(yc)[ms, ns]
    ok, d = bf16_ok(got_bits, Y_ref, S)
    assert ok.all(), f"{what}: bf16 off at samples {np.argwhere(~ok)[:5].ravel().tolist()}"
    if yf32 is not None:
        yf = yf32.detach().cpu().double().numpy()[ms, ns]
        assert (np.abs(yf - Y_ref) <= RTOL_S * S + ATOL).all(), f"{what}: fp32 outside bound"
    return int(d.max()) if d.size else 0


def check_bounded(y, yf32, ref, bound, what=""):
    """Fused outputs: |yf32 - ref| <= bound element-wise, and the bf16 result
    within 1 ulp of round_bf16(ref) or the rounding of some value inside the
    bound (the same acceptance as the plain GEMM, with the fused bound from
    oracle.fused_bounds)."""
    if yf32 is not None:
        yf = yf32.detach().cpu().double().numpy()
        err = np.abs(yf - ref)
        bad = np.argwhere(~(err <= bound))
        assert bad.size == 0, (f"{what}: fp32 outside bound at {bad[:5].tolist()}: got {yf[tuple(bad[0])]}, "
                               f"ref {ref[tuple(bad[0])]}, bound {bound[tuple(bad[0])]}")
    got = bf16_bits(y)
    d = ulp_distance(got, oracle.round_bf16(ref))
    g = ordered(got)
    ok = (d <= 1) | ((g >= ordered(oracle.round_bf16(ref - bound))) & (g <= ordered(oracle.round_bf16(ref + bound))))
    bad = np.argwhere(~ok)
    assert bad.size == 0, (f"{what}: bf16 off at {bad[:5].tolist()} (got {hex(int(got[tuple(bad[0])]))}, "
                           f"ref {hex(int(oracle.round_bf16(ref)[tuple(bad[0])]))}, ulps {int(d[tuple(bad[0])])})")
    return int(d.max()) if d.size else 0
