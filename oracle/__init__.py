"""Plain fp64 CPU oracle for the small-M decode GEMM ``Y = X @ W.T``.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product library
(``weight_streaming_megakernel_b200``) never imports it, and it never imports
the product: the two share no code.  Inputs for both come from ``synth``.

What it computes, and from which passage:

* ``gemm_ref`` -- for every output, the exact dot product of a row of X with a
  row of W over bf16 inputs widened exactly to fp64, summed in increasing k
  (``oracle.c``).  The decode-GEMM regime is the one named in "AMD: ROCm
  Low-Latency-GEMM-Kernel beschleunigen LLM-Inferenz ... MI355X", section "Was
  ist GEMM und die Decode-Phase eines LLMs?"; the pages never fix rounding or
  accumulation order, so the plain definition of the product is the reading.
* ``round_bf16`` -- one rounding of the fp64 result to bf16, to nearest with
  ties to even (IEEE-754 definition, written out in ``oracle.c``).
* ``chain_ref`` -- a chain of such GEMMs is the per-task product, each on that
  task's own input ("Fleet ..." reading notes, section 2a: the megakernel only
  changes when work runs, not what it computes).
* ``l2model`` -- Eq.(1) of the Fleet reading notes (section 3f), the L2 weight
  hit rate of M-major cooperative traversal, and AI_eff.
* ``silu`` / ``gate_up_rows`` / ``silu_mul_ref`` -- the fused SiLU epilogue of
  the gate+up GEMM ("Fleet ..." reading notes, sections 3f and 7b and the
  design summary: gate and up concatenated into one GEMM sharing one
  activation, with SiLU fused): ``H = silu(X Wg^T) * (X Wu^T)``, silu(z) =
  z / (1 + e^-z), evaluated in fp64 from the fp64 products.  The pages do not
  fix how gate and up rows are laid out in the one weight; the reading here
  interleaves them in blocks of 8 rows (gate rows 8b..8b+7, then the up rows
  8b..8b+7), so every weight tile holds matching gate and up rows.
* ``residual_ref`` -- the residual-add epilogue, ``Y = X W^T + R`` in fp64.
* ``fused_bounds`` -- the fp32 acceptance bounds of the fused outputs,
  propagated from the GEMM's per-element bound (see the function).

Every function here is pinned by ``tests/test_oracle_pins.py`` against
brute-force exact rational arithmetic, integer and permutation cases, library
routines (numpy int64/fp64 products, torch's fp32->bf16 rounding) and the
worked table printed beside Eq.(1).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC", "-std=c11"]


def build(src: str = _SRC, out: str = _LIB_PATH, force: bool = False) -> str:
    """Compile ``oracle.c`` with gcc into a shared library (in place)."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    cmd = ["gcc", *CFLAGS, "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _bind(lib):
    u16p = ctypes.POINTER(ctypes.c_uint16)
    f64p = ctypes.POINTER(ctypes.c_double)
    i32p = ctypes.POINTER(ctypes.c_int32)
    lib.wsmo_bf16_to_f64.argtypes = [ctypes.c_uint16]
    lib.wsmo_bf16_to_f64.restype = ctypes.c_double
    lib.wsmo_f64_to_bf16.argtypes = [ctypes.c_double]
    lib.wsmo_f64_to_bf16.restype = ctypes.c_uint16
    lib.wsmo_round_bf16.argtypes = [f64p, ctypes.c_int64, u16p]
    lib.wsmo_round_bf16.restype = None
    lib.wsmo_gemm.argtypes = [u16p, u16p, ctypes.c_int, ctypes.c_int, ctypes.c_int, f64p, f64p]
    lib.wsmo_gemm.restype = None
    lib.wsmo_gemm_sampled.argtypes = [u16p, u16p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                      i32p, i32p, ctypes.c_int64, f64p, f64p]
    lib.wsmo_gemm_sampled.restype = None
    lib.wsmo_set_threads.argtypes = [ctypes.c_int]
    lib.wsmo_set_threads.restype = ctypes.c_int
    return lib


def load(path: str | None = None):
    """Load (building if needed) the oracle library.  ``path`` loads another
    build of the same source, which the mutation tests use."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
        return _lib


def _u16(a) -> np.ndarray:
    """bf16 data as a C-contiguous uint16 numpy array of its bit patterns."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            assert a.dtype == torch.bfloat16, a.dtype
            return a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


def _p(a, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def bf16_to_f64(bits) -> np.ndarray:
    lib = load()
    b = _u16(bits).ravel()
    return np.array([lib.wsmo_bf16_to_f64(int(v)) for v in b], dtype=np.float64)


def round_bf16(y, lib=None) -> np.ndarray:
    """fp64 array -> uint16 bf16 bit patterns (RNE), same shape."""
    lib = lib or load()
    y = np.ascontiguousarray(y, dtype=np.float64)
    out = np.empty(y.shape, dtype=np.uint16)
    lib.wsmo_round_bf16(_p(y, ctypes.c_double), y.size, _p(out, ctypes.c_uint16))
    return out


def gemm_ref(X, W, lib=None):
    """(Y_ref, S) in fp64 for bf16 X [M,K] and W [N,K] (torch bf16 or uint16 bits)."""
    lib = lib or load()
    x = _u16(X)
    w = _u16(W)
    M, K = x.shape
    N, K2 = w.shape
    assert K == K2
    Y = np.empty((M, N), dtype=np.float64)
    S = np.empty((M, N), dtype=np.float64)
    lib.wsmo_gemm(_p(x, ctypes.c_uint16), _p(w, ctypes.c_uint16), M, N, K,
                  _p(Y, ctypes.c_double), _p(S, ctypes.c_double))
    return Y, S


def gemm_ref_sampled(X, W, ms, ns, lib=None):
    """(Y_ref, S) at the sampled output positions (ms[i], ns[i])."""
    lib = lib or load()
    x = _u16(X)
    w = _u16(W)
    M, K = x.shape
    N, _ = w.shape
    ms = np.ascontiguousarray(ms, dtype=np.int32)
    ns = np.ascontiguousarray(ns, dtype=np.int32)
    assert ms.shape == ns.shape
    assert ms.size == 0 or (ms.min() >= 0 and ms.max() < M and ns.min() >= 0 and ns.max() < N)
    Y = np.empty(ms.shape, dtype=np.float64)
    S = np.empty(ms.shape, dtype=np.float64)
    lib.wsmo_gemm_sampled(_p(x, ctypes.c_uint16), _p(w, ctypes.c_uint16), M, N, K,
                          _p(ms, ctypes.c_int32), _p(ns, ctypes.c_int32), ms.size,
                          _p(Y, ctypes.c_double), _p(S, ctypes.c_double))
    return Y, S


def chain_ref(tasks):
    """Per-task oracle of a GEMM chain: ``tasks`` is a list of (X, W) pairs,
    each task evaluated on its own input.  Returns a list of (Y_ref, S)."""
    return [gemm_ref(X, W) for (X, W) in tasks]


def set_threads(n: int = 0) -> int:
    """Set the OpenMP thread count (0 keeps the current one); returns it."""
    return load().wsmo_set_threads(int(n))


# --------------------------------------------------------------------------- fused epilogues

def silu(z):
    """silu(z) = z * sigmoid(z) = z / (1 + exp(-z)), fp64 (exp overflow for very
    negative z gives z / inf = -0.0, the limit)."""
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def gate_up_rows(I: int):
    """(gate, up) row indices of the fused gate+up weight [2I, K] for output
    column j < I: blocks of 8 rows, gate rows of block b then its up rows."""
    assert I % 8 == 0
    j = np.arange(I)
    gate = 16 * (j // 8) + (j % 8)
    return gate, gate + 8


def silu_mul_ref(X, W_gu, lib=None):
    """Fused gate+up GEMM with SiLU: returns (H_ref, G, U, Sg, Su), all [M, I]
    fp64: H = silu(G) * U with G, U the gate and up products and Sg, Su their
    sums of |products| (the scale of the GEMM bound)."""
    Y, S = gemm_ref(X, W_gu, lib)
    gi, ui = gate_up_rows(Y.shape[1] // 2)
    G, U = Y[:, gi], Y[:, ui]
    return silu(G) * U, G, U, S[:, gi], S[:, ui]


def residual_ref(X, W, R, lib=None):
    """Y = X W^T + R in fp64 (R: bf16 [M, N]); returns (Y_ref, S) with S the
    GEMM's sum of |products|."""
    Y, S = gemm_ref(X, W, lib)
    r = _u16(R)
    Rf = np.frombuffer((r.astype(np.uint32) << 16).tobytes(), dtype=np.float32).reshape(r.shape).astype(np.float64)
    return Y + Rf, S


def fused_bounds(kind, *, S=None, Y=None, G=None, U=None, Sg=None, Su=None):
    """Per-element fp32 acceptance bound of a fused output.

    The GEMM part of every output may differ from its fp64 value by
    d = 1e-3 * S + 1e-6 (the accumulation bound).  Residual: d plus one fp32
    rounding of the sum, 2^-23 |Y|.  SiLU*mul: with dg, du the bounds of G and
    U, and |silu'| <= 1.1 everywhere (its extremes are about 1.0998 and
    -0.0998), |dH| <= 1.1 |U| dg + (|silu(G)| + 1.1 dg) du, plus the fp32
    evaluation of silu and the product, 2^-19 |silu(G) U| + 1e-7."""
    if kind == "residual":
        return 1e-3 * S + 1e-6 + 2.0 ** -23 * np.abs(Y)
    if kind == "silu_mul":
        dg = 1e-3 * Sg + 1e-6
        du = 1e-3 * Su + 1e-6
        sg = np.abs(silu(G))
        return 1.1 * np.abs(U) * dg + (sg + 1.1 * dg) * du + 2.0 ** -19 * sg * np.abs(U) + 1e-7
    raise ValueError(kind)
