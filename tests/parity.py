"""Shared checks of the GPU results against the fp64 oracle.

Acceptance (element by element):
  * fp32 result before rounding:  |Yf32 - Y_ref| <= B,  B = 1e-3 * S + 1e-6,
    S = sum_k |X[m,k] W[n,k]| (the stated fp32 tolerance of the method);
  * bf16 result: within 1 bf16 ulp of round_bf16(Y_ref), ulps counted in
    the ordered integer encoding (so power-of-two boundaries and signs count
    right; +0 and -0 are equal).
  * The one place the two stated tolerances disagree is cancellation: where
    |Y_ref| < B the fp32 allowance reaches through zero and spans many bf16
    ulps of a value that small, so no fp32 accumulation order can promise
    1 ulp there.  Only those elements may instead be the correct rounding of
    SOME value inside the fp32 bound: round(Y_ref - B) <= y <= round(Y_ref + B)
    in bf16 order.  Every element with |Y_ref| >= B is held to 1 ulp.
  * Wherever the kernel also writes its fp32 result, the bf16 output must be
    exactly round_bf16(Yf32) (the one rounding of the kernel's own value).

Every check records the largest ulp distance it saw among the elements held
to 1 ulp, and how many elements fell in the cancellation window; the test
session prints both at its end.
"""
import numpy as np
import torch

import oracle

ATOL = 1e-6
RTOL_S = 1e-3

# largest ulp distance among elements held to 1 ulp, and the window count, over the session
STATS = {"checks": 0, "elements": 0, "max_ulp": 0, "cancel_elements": 0, "cancel_max_ulp": 0}


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def ordered(bits: np.ndarray) -> np.ndarray:
    b = bits.astype(np.int64)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def ulp_distance(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    return np.abs(ordered(a_bits) - ordered(b_bits))


def rne_bf16_of_f32(yf32: torch.Tensor) -> np.ndarray:
    """bf16 bits of the round-to-nearest-even of fp32 values (torch's
    conversion, a library routine independent of the kernels)."""
    return bf16_bits(yf32.detach().cpu().to(torch.bfloat16))


def bf16_ok(got_bits, ref, bound):
    """Element-wise bf16 acceptance (see the module docstring) against the
    fp64 reference `ref` with fp32 allowance `bound`; returns (ok, ulp
    distances, cancellation mask)."""
    ref = np.asarray(ref, dtype=np.float64)
    bound = np.asarray(bound, dtype=np.float64)
    d = ulp_distance(got_bits, oracle.round_bf16(ref))
    cancel = np.abs(ref) < bound
    g = ordered(got_bits)
    lo = ordered(oracle.round_bf16(ref - bound))
    hi = ordered(oracle.round_bf16(ref + bound))
    ok = (d <= 1) | (cancel & (g >= lo) & (g <= hi))
    return ok, d, cancel


def _record(d, cancel):
    STATS["checks"] += 1
    STATS["elements"] += int(d.size)
    held = d[~cancel]
    if held.size:
        STATS["max_ulp"] = max(STATS["max_ulp"], int(held.max()))
    if cancel.any():
        STATS["cancel_elements"] += int(cancel.sum())
        STATS["cancel_max_ulp"] = max(STATS["cancel_max_ulp"], int(d[cancel].max()))


def _check_bits(got, ref, bound, what):
    ok, d, cancel = bf16_ok(got, ref, bound)
    _record(d, cancel)
    bad = np.argwhere(~ok)
    held = d[~cancel]
    assert bad.size == 0, (f"{what}: bf16 off at {bad[:5].tolist()} "
                           f"(got {hex(int(got[tuple(bad[0])]))}, ref {hex(int(oracle.round_bf16(ref)[tuple(bad[0])]))}, "
                           f"ulps {int(d[tuple(bad[0])])}, |ref| {abs(float(ref[tuple(bad[0])])):.3g}, "
                           f"bound {float(bound[tuple(bad[0])]):.3g}; max ulp over held elements "
                           f"{int(held.max()) if held.size else 0})")
    return int(held.max()) if held.size else 0


def _check_f32(yf32, ref, bound, what, got_bits=None, sel=None):
    yfc = yf32.detach().cpu()
    yf = yfc.double().numpy()
    if sel is not None:
        yf = yf[sel]
    err = np.abs(yf - ref)
    bad = np.argwhere(~(err <= bound))
    assert bad.size == 0, (f"{what}: fp32 outside bound at {bad[:5].tolist()}: got {yf[tuple(bad[0])]}, "
                           f"ref {ref[tuple(bad[0])]}, bound {bound[tuple(bad[0])]}")
    if got_bits is not None:
        own = rne_bf16_of_f32(yfc)
        if sel is not None:
            own = own[sel]
        diff = np.argwhere(own != got_bits)
        assert diff.size == 0, (f"{what}: bf16 output is not the rounding of the kernel's own fp32 result at "
                                f"{diff[:5].tolist()}")
    return float((err / bound).max()) if err.size else 0.0


def check_full(x, w, y, yf32=None, Y_ref=None, S=None, what=""):
    """Compare complete outputs with the oracle; returns (max |err|/bound, max ulp over held elements)."""
    if Y_ref is None:
        Y_ref, S = oracle.gemm_ref(x.cpu(), w.cpu())
    B = RTOL_S * S + ATOL
    got = bf16_bits(y)
    worst = 0.0
    if yf32 is not None:
        worst = _check_f32(yf32, Y_ref, B, what, got_bits=got)
    return worst, _check_bits(got, Y_ref, B, what)


def check_sampled(x, w, y, yf32, ms, ns, what=""):
    """Compare sampled outputs (ms[i], ns[i]) with the oracle computed one by one."""
    Y_ref, S = oracle.gemm_ref_sampled(x.cpu(), w.cpu(), ms, ns)
    B = RTOL_S * S + ATOL
    got_bits = bf16_bits(y.detach().cpu())[ms, ns]
    if yf32 is not None:
        _check_f32(yf32, Y_ref, B, what, got_bits=got_bits, sel=(ms, ns))
    return _check_bits(got_bits, Y_ref, B, what)


def check_bounded(y, yf32, ref, bound, what=""):
    """Fused outputs: |yf32 - ref| <= bound element-wise, and the bf16 result
    within 1 ulp of round_bf16(ref) -- or, only where |ref| < bound, the
    rounding of some value inside the bound (the same acceptance as the plain
    GEMM, with the fused bound from oracle.fused_bounds)."""
    got = bf16_bits(y)
    if yf32 is not None:
        _check_f32(yf32, ref, bound, what, got_bits=got)
    return _check_bits(got, ref, bound, what)
