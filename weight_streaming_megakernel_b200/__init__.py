"""Python binding of libwsm, the weight-streaming decode GEMM library for B200.

Thin ctypes marshalling over the C ABI declared in ``include/wsm.h``: every
step of the computation runs in the library's CUDA kernels.  PyTorch supplies
device memory and streams only.  If ``libwsm.so`` is missing every call raises
(there is no fallback); build it with ``python -m
weight_streaming_megakernel_b200._build`` or ``__graft_entry__.build()``.

    Y[m, n] = sum_k X[m, k] * W[n, k]     (X [M,K], W [N,K], Y [M,N], bf16)
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import torch

__all__ = [
    "LIB_PATH", "WSM_OK", "WSM_ERR_INVALID", "WSM_ERR_UNSUPPORTED", "WSM_ERR_ALIGN", "WSM_ERR_NOMEM",
    "WSM_ERR_CUDA", "WSM_ERR_TIMEOUT", "PATH_AUTO", "PATH_STREAM", "PATH_UMMA", "ORDER_AUTO", "ORDER_M_MAJOR",
    "ORDER_NAIVE", "L2_AUTO", "L2_EVICT_FIRST", "L2_NORMAL", "FLAG_W_READONLY", "FLAG_NO_PDL", "FLAG_INDEPENDENT", "WsmError", "lib", "skinny_gemm", "plan",
    "workspace_bytes", "stream_status", "Task", "Chain", "gemm_chain", "chain_validate", "chain_plan", "last_error",
    "skinny_gemm_noalloc", "workspace_status", "gemm_chain_status", "debug_stall", "sm_die_map",
    "abi_version", "HEADER_SYMBOLS",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libwsm.so")

WSM_OK, WSM_ERR_INVALID, WSM_ERR_UNSUPPORTED, WSM_ERR_ALIGN, WSM_ERR_NOMEM, WSM_ERR_CUDA, WSM_ERR_TIMEOUT = range(7)
_STATUS_NAMES = {0: "WSM_OK", 1: "WSM_ERR_INVALID", 2: "WSM_ERR_UNSUPPORTED", 3: "WSM_ERR_ALIGN",
                 4: "WSM_ERR_NOMEM", 5: "WSM_ERR_CUDA", 6: "WSM_ERR_TIMEOUT"}
PATH_AUTO, PATH_STREAM, PATH_UMMA = 0, 1, 2
ORDER_AUTO, ORDER_M_MAJOR, ORDER_NAIVE = 0, 1, 2
L2_AUTO, L2_EVICT_FIRST, L2_NORMAL = 0, 1, 2
FLAG_W_READONLY, FLAG_NO_PDL, FLAG_INDEPENDENT = 1, 2, 4
EPI_NONE, EPI_SILU_MUL, EPI_RESIDUAL = 0, 1, 2
CHAIN_KERNELS_AUTO, CHAIN_KERNELS_ONE, CHAIN_KERNELS_SPLIT = 0, 1, 2
K_ORDER_AUTO, K_ORDER_INCREASING, K_ORDER_ROTATED = 0, 1, 2
CHAIN_CLUSTER_AUTO, CHAIN_CLUSTER_OFF, CHAIN_CLUSTER_ON = 0, 1, 2
DIE_GROUPS_AUTO, DIE_GROUPS_ON, DIE_GROUPS_OFF = 0, 1, 2

# Every function include/wsm.h declares (checked by the CPU tests).
HEADER_SYMBOLS = (
    "skinny_gemm", "skinny_gemm_ex", "wsm_plan", "wsm_workspace_bytes", "wsm_stream_status", "wsm_workspace_status",
    "wsm_debug_stall", "skinny_gemm_noalloc", "gemm_chain_status", "wsm_sm_die_map",
    "wsm_chain_plan", "wsm_chain_create", "wsm_chain_run", "wsm_chain_status", "wsm_chain_task_plan",
    "wsm_chain_trace",
    "wsm_chain_destroy",
    "gemm_chain", "wsm_chain_validate", "wsm_last_error", "wsm_abi_version",
)


class WsmError(RuntimeError):
    def __init__(self, code: int, where: str, msg: str):
        self.code = code
        super().__init__(f"{where}: {_STATUS_NAMES.get(code, code)}: {msg}")


class _Opts(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int), ("m_tile", ctypes.c_int), ("order", ctypes.c_int),
                ("l2_policy", ctypes.c_int), ("grid", ctypes.c_int), ("stage_k", ctypes.c_int),
                ("flags", ctypes.c_int), ("unit_stages", ctypes.c_int), ("tail_tiles", ctypes.c_int),
                ("tail_unit_stages", ctypes.c_int), ("l2_prefetch_stages", ctypes.c_int), ("tile_rows", ctypes.c_int),
                ("k_order", ctypes.c_int), ("epilogue", ctypes.c_int),
                ("R", ctypes.c_void_p), ("Yf32", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_size_t)]


class _PlanInfo(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int), ("grid", ctypes.c_int), ("tile_rows", ctypes.c_int),
                ("tile_k", ctypes.c_int), ("m_tile", ctypes.c_int), ("m_tiles", ctypes.c_int),
                ("n_tiles", ctypes.c_int), ("unit_stages", ctypes.c_int), ("tail_tiles", ctypes.c_int),
                ("tail_unit_stages", ctypes.c_int), ("units", ctypes.c_longlong),
                ("k_iters", ctypes.c_int), ("stages", ctypes.c_int),
                ("order", ctypes.c_int), ("l2_policy", ctypes.c_int), ("smem_bytes", ctypes.c_int),
                ("iters", ctypes.c_longlong), ("workspace_bytes", ctypes.c_size_t)]


class _Task(ctypes.Structure):
    _fields_ = [("X", ctypes.c_void_p), ("W", ctypes.c_void_p), ("Y", ctypes.c_void_p),
                ("M", ctypes.c_int), ("N", ctypes.c_int), ("K", ctypes.c_int), ("dep", ctypes.c_int),
                ("Yf32", ctypes.c_void_p), ("epilogue", ctypes.c_int), ("R", ctypes.c_void_p), ("dep_cols", ctypes.c_int),
                ("m_tile", ctypes.c_int)]


class _ChainTaskInfo(ctypes.Structure):
    _fields_ = [("plan", _PlanInfo), ("kernel", ctypes.c_int), ("l2_prefetch_stages", ctypes.c_int),
                ("k_order", ctypes.c_int), ("dep_ring_stages", ctypes.c_int), ("cluster", ctypes.c_int),
                ("die_split", ctypes.c_int)]


class _DieInfo(ctypes.Structure):
    _fields_ = [("num_sms", ctypes.c_int), ("dies", ctypes.c_int), ("sms_die0", ctypes.c_int),
                ("sms_die1", ctypes.c_int), ("agreement", ctypes.c_float), ("near_cycles", ctypes.c_float),
                ("far_cycles", ctypes.c_float)]


class _ChainOpts(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int), ("grid", ctypes.c_int), ("timeout_ns", ctypes.c_ulonglong),
                ("trace", ctypes.c_int), ("debug_unmet_dependency", ctypes.c_int), ("flags", ctypes.c_int),
                ("stage_k", ctypes.c_int), ("unit_stages", ctypes.c_int), ("tail_tiles", ctypes.c_int),
                ("tail_unit_stages", ctypes.c_int), ("l2_prefetch_stages", ctypes.c_int),
                ("counter_groups", ctypes.c_int), ("tile_rows", ctypes.c_int), ("k_order", ctypes.c_int),
                ("dep_ring_stages", ctypes.c_int), ("kernels", ctypes.c_int), ("cluster", ctypes.c_int),
                ("die_groups", ctypes.c_int)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libwsm.so is not built ({LIB_PATH}); run "
                               "`python -m weight_streaming_megakernel_b200._build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, st = ctypes.c_void_p, ctypes.c_int, ctypes.c_int
        L.skinny_gemm.argtypes = [vp, vp, vp, i, i, i, vp]
        L.skinny_gemm.restype = st
        L.skinny_gemm_ex.argtypes = [vp, vp, vp, i, i, i, ctypes.POINTER(_Opts), vp]
        L.skinny_gemm_ex.restype = st
        L.skinny_gemm_noalloc.argtypes = [vp, vp, vp, i, i, i, vp]
        L.skinny_gemm_noalloc.restype = st
        L.wsm_plan.argtypes = [i, i, i, i, ctypes.POINTER(_Opts), ctypes.POINTER(_PlanInfo)]
        L.wsm_plan.restype = st
        L.wsm_workspace_bytes.argtypes = [i, i, i, ctypes.POINTER(_Opts)]
        L.wsm_workspace_bytes.restype = ctypes.c_size_t
        L.wsm_stream_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
        L.wsm_stream_status.restype = st
        L.wsm_workspace_status.argtypes = [vp, ctypes.c_size_t, vp, ctypes.POINTER(ctypes.c_int)]
        L.wsm_workspace_status.restype = st
        L.wsm_debug_stall.argtypes = [i, ctypes.c_ulonglong]
        L.wsm_debug_stall.restype = st
        L.gemm_chain_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
        L.gemm_chain_status.restype = st
        L.wsm_sm_die_map.argtypes = [ctypes.POINTER(ctypes.c_int), i, ctypes.POINTER(_DieInfo)]
        L.wsm_sm_die_map.restype = st
        L.wsm_chain_task_plan.argtypes = [vp, i, ctypes.POINTER(_PlanInfo)]
        L.wsm_chain_task_plan.restype = st
        L.wsm_chain_create.argtypes = [ctypes.POINTER(_Task), i, ctypes.POINTER(_ChainOpts), ctypes.POINTER(vp)]
        L.wsm_chain_create.restype = st
        L.wsm_chain_run.argtypes = [vp, vp]
        L.wsm_chain_run.restype = st
        L.wsm_chain_status.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_int)]
        L.wsm_chain_status.restype = st
        L.wsm_chain_trace.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_ulonglong), ctypes.c_size_t]
        L.wsm_chain_trace.restype = ctypes.c_size_t
        L.wsm_chain_destroy.argtypes = [vp]
        L.wsm_chain_destroy.restype = None
        L.gemm_chain.argtypes = [ctypes.POINTER(_Task), i, vp]
        L.gemm_chain.restype = st
        L.wsm_chain_plan.argtypes = [ctypes.POINTER(_Task), i, ctypes.POINTER(_ChainOpts), i,
                                     ctypes.POINTER(_ChainTaskInfo), ctypes.POINTER(ctypes.c_int)]
        L.wsm_chain_plan.restype = st
        L.wsm_chain_validate.argtypes = [ctypes.POINTER(_Task), i]
        L.wsm_chain_validate.restype = st
        L.wsm_last_error.argtypes = []
        L.wsm_last_error.restype = ctypes.c_char_p
        L.wsm_abi_version.argtypes = []
        L.wsm_abi_version.restype = ctypes.c_int
        _lib = L
    return _lib


def last_error() -> str:
    return lib().wsm_last_error().decode()


def abi_version() -> int:
    return lib().wsm_abi_version()


def _check(code: int, where: str):
    if code != WSM_OK:
        raise WsmError(code, where, last_error())


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _check_operand(name, t, dtype=torch.bfloat16):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _opts(path=PATH_AUTO, m_tile=0, order=ORDER_AUTO, l2_policy=L2_AUTO, grid=0, yf32=None, workspace=None,
          stage_k=0, flags=0, unit_stages=0, tail_tiles=0, tail_unit_stages=0, l2_prefetch_stages=0, epilogue=0,
          r=None, tile_rows=0, k_order=0):
    o = _Opts()
    o.path, o.m_tile, o.order, o.l2_policy, o.grid, o.stage_k = path, m_tile, order, l2_policy, grid, stage_k
    o.flags, o.unit_stages, o.tail_tiles, o.tail_unit_stages = flags, unit_stages, tail_tiles, tail_unit_stages
    o.l2_prefetch_stages = l2_prefetch_stages
    o.epilogue = epilogue
    o.R = _ptr(r)
    o.tile_rows = tile_rows
    o.k_order = k_order
    o.Yf32 = _ptr(yf32)
    if workspace is not None:
        o.workspace = workspace.data_ptr()
        o.workspace_bytes = workspace.numel() * workspace.element_size()
    return o


def skinny_gemm(x: torch.Tensor, w: torch.Tensor, y: Optional[torch.Tensor] = None, *, path=PATH_AUTO,
                m_tile=0, order=ORDER_AUTO, l2_policy=L2_AUTO, grid=0, yf32: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None, stage_k=0, flags=0, unit_stages=0, tail_tiles=0,
                tail_unit_stages=0, l2_prefetch_stages=0, epilogue=EPI_NONE, r: Optional[torch.Tensor] = None,
                tile_rows=0, k_order=0, stream=None) -> torch.Tensor:
    """Y = X @ W.T on the current (or given) stream; returns Y.  With
    epilogue=EPI_SILU_MUL, W is the fused gate+up weight (rows interleaved in
    blocks of 8) and Y is [M, N/2] = silu(gate) * up; with EPI_RESIDUAL,
    Y = X @ W.T + r."""
    _check_operand("x", x)
    _check_operand("w", w)
    if x.dim() != 2 or w.dim() != 2 or x.shape[1] != w.shape[1]:
        raise ValueError(f"shapes x{tuple(x.shape)} w{tuple(w.shape)} do not form X[M,K] . W[N,K]^T")
    M, K = x.shape
    N = w.shape[0]
    ny = N // 2 if epilogue == EPI_SILU_MUL else N
    if y is None:
        y = torch.empty(M, ny, dtype=torch.bfloat16, device=x.device)
    _check_operand("y", y)
    if tuple(y.shape) != (M, ny):
        raise ValueError(f"y must be [{M}, {ny}]")
    if yf32 is not None:
        _check_operand("yf32", yf32, torch.float32)
        if tuple(yf32.shape) != (M, ny):
            raise ValueError(f"yf32 must be [{M}, {ny}]")
    if epilogue == EPI_RESIDUAL:
        if r is None:
            raise ValueError("the residual epilogue needs r")
        _check_operand("r", r)
        if tuple(r.shape) != (M, N):
            raise ValueError(f"r must be [{M}, {N}]")
    plain = (path, m_tile, order, l2_policy, grid, stage_k, flags, unit_stages, tail_tiles, tail_unit_stages,
             l2_prefetch_stages, epilogue, tile_rows, k_order) == (PATH_AUTO, 0, ORDER_AUTO, L2_AUTO, 0, 0, 0, 0, 0, 0, 0,
                                                                    0, 0, 0) \
        and yf32 is None and workspace is None
    s = _stream_handle(stream)
    if plain:
        _check(lib().skinny_gemm(x.data_ptr(), w.data_ptr(), y.data_ptr(), M, N, K, s), "skinny_gemm")
    else:
        o = _opts(path, m_tile, order, l2_policy, grid, yf32, workspace, stage_k, flags, unit_stages, tail_tiles,
                  tail_unit_stages, l2_prefetch_stages, epilogue, r, tile_rows, k_order)
        _check(lib().skinny_gemm_ex(x.data_ptr(), w.data_ptr(), y.data_ptr(), M, N, K, ctypes.byref(o), s),
               "skinny_gemm_ex")
    return y


def skinny_gemm_noalloc(x: torch.Tensor, w: torch.Tensor, y: torch.Tensor, stream=None) -> torch.Tensor:
    """Y = X @ W.T with the library's fixed device scratch array (no device
    allocation ever; calls that overlap on the GPU race on the array)."""
    _check_operand("x", x)
    _check_operand("w", w)
    _check_operand("y", y)
    M, K = x.shape
    N = w.shape[0]
    if w.shape[1] != K or tuple(y.shape) != (M, N):
        raise ValueError("shapes do not form Y[M,N] = X[M,K] . W[N,K]^T")
    _check(lib().skinny_gemm_noalloc(x.data_ptr(), w.data_ptr(), y.data_ptr(), M, N, K, _stream_handle(stream)),
           "skinny_gemm_noalloc")
    return y


def plan(M: int, N: int, K: int, num_sms: int = 148, **opts) -> dict:
    """The plan for a shape (pure host computation; no GPU needed)."""
    o = _opts(**opts)
    info = _PlanInfo()
    _check(lib().wsm_plan(M, N, K, num_sms, ctypes.byref(o), ctypes.byref(info)), "wsm_plan")
    return {f: getattr(info, f) for f, _ in _PlanInfo._fields_}


def workspace_bytes(M: int, N: int, K: int, **opts) -> int:
    o = _opts(**opts)
    n = lib().wsm_workspace_bytes(M, N, K, ctypes.byref(o))
    if n == 0:
        raise WsmError(WSM_ERR_INVALID, "wsm_workspace_bytes", last_error())
    return n


def stream_status(stream=None) -> int:
    """Synchronise the stream; 0, or WSM_ERR_TIMEOUT if a device-side wait of a
    call on it (or of a skinny_gemm_noalloc call on this device) ran out since
    the last check."""
    code = ctypes.c_int(0)
    rc = lib().wsm_stream_status(_stream_handle(stream), ctypes.byref(code))
    if rc not in (WSM_OK, WSM_ERR_TIMEOUT):
        raise WsmError(rc, "wsm_stream_status", last_error())
    return code.value


def workspace_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise the stream; 0, or WSM_ERR_TIMEOUT if a device-side wait of a
    skinny_gemm_ex call given this caller workspace ran out since the last check."""
    code = ctypes.c_int(0)
    rc = lib().wsm_workspace_status(workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                    _stream_handle(stream), ctypes.byref(code))
    if rc not in (WSM_OK, WSM_ERR_TIMEOUT):
        raise WsmError(rc, "wsm_workspace_status", last_error())
    return code.value


def gemm_chain_status(stream=None):
    """Synchronise the stream; (code, failed_task) for the one-shot gemm_chain
    runs on the current device since the last check."""
    ft = ctypes.c_int(-1)
    rc = lib().gemm_chain_status(_stream_handle(stream), ctypes.byref(ft))
    if rc not in (WSM_OK, WSM_ERR_TIMEOUT):
        raise WsmError(rc, "gemm_chain_status", last_error())
    return rc, ft.value


def sm_die_map(capacity: int = 1024):
    """Which die each SM of the current device sits on (measured once per
    device): (list die_of_sm indexed by SM id, -1 past the last SM; dict of
    the probe's findings)."""
    arr = (ctypes.c_int * capacity)()
    info = _DieInfo()
    _check(lib().wsm_sm_die_map(arr, capacity, ctypes.byref(info)), "wsm_sm_die_map")
    return list(arr), {f: getattr(info, f) for f, _ in _DieInfo._fields_}


def debug_stall(calls: int, limit_ns: int = 50_000_000) -> None:
    """Test hook: the next `calls` launches each stall CTA 0 on a flag nothing
    sets for limit_ns, then record WSM_ERR_TIMEOUT (no fault); 0 cancels."""
    _check(lib().wsm_debug_stall(calls, limit_ns), "wsm_debug_stall")


@dataclass
class Task:
    x: torch.Tensor
    w: torch.Tensor
    y: torch.Tensor
    dep: int = -1
    yf32: Optional[torch.Tensor] = None
    epilogue: int = EPI_NONE
    r: Optional[torch.Tensor] = None
    dep_cols: bool = False
    m_tile: int = 0


def _tasks_array(tasks: Sequence[Task]):
    arr = (_Task * len(tasks))()
    for i, t in enumerate(tasks):
        M, K = t.x.shape
        N = t.w.shape[0]
        arr[i].X, arr[i].W, arr[i].Y = t.x.data_ptr(), t.w.data_ptr(), t.y.data_ptr()
        arr[i].M, arr[i].N, arr[i].K, arr[i].dep = M, N, K, t.dep
        arr[i].Yf32 = _ptr(t.yf32)
        arr[i].epilogue, arr[i].R, arr[i].dep_cols = t.epilogue, _ptr(t.r), 1 if t.dep_cols else 0
        arr[i].m_tile = t.m_tile
    return arr


def chain_validate(tasks) -> None:
    """Host-side validation of a raw task list: sequence of dicts with keys
    X, W, Y (integer addresses), M, N, K and optionally dep, Yf32, epilogue, R,
    dep_cols."""
    arr = (_Task * len(tasks))()
    for i, t in enumerate(tasks):
        arr[i].X, arr[i].W, arr[i].Y = t["X"], t["W"], t["Y"]
        arr[i].M, arr[i].N, arr[i].K, arr[i].dep = t["M"], t["N"], t["K"], t.get("dep", -1)
        arr[i].Yf32 = t.get("Yf32")
        arr[i].epilogue, arr[i].R, arr[i].dep_cols = t.get("epilogue", 0), t.get("R"), int(bool(t.get("dep_cols")))
        arr[i].m_tile = t.get("m_tile", 0)
    _check(lib().wsm_chain_validate(arr, len(tasks)), "wsm_chain_validate")


def _chain_opts(path=PATH_AUTO, grid=0, timeout_ns=0, trace=False, debug_unmet_dependency=False, flags=0,
                stage_k=0, unit_stages=0, tail_tiles=0, tail_unit_stages=0, l2_prefetch_stages=0,
                counter_groups=0, kernels=0, tile_rows=0, k_order=0, dep_ring_stages=0, cluster=0,
                die_groups=0) -> "_ChainOpts":
    o = _ChainOpts()
    o.path, o.grid, o.timeout_ns, o.trace = path, grid, timeout_ns, (trace if trace in (1, 2) else 1) if trace else 0
    o.debug_unmet_dependency = 1 if debug_unmet_dependency else 0
    o.flags, o.stage_k = flags, stage_k
    o.unit_stages, o.tail_tiles, o.tail_unit_stages = unit_stages, tail_tiles, tail_unit_stages
    o.l2_prefetch_stages = l2_prefetch_stages
    o.counter_groups = counter_groups
    o.kernels = kernels
    o.tile_rows = tile_rows
    o.k_order = k_order
    o.dep_ring_stages = dep_ring_stages
    o.cluster = cluster
    o.die_groups = die_groups
    return o


def chain_plan(specs, num_sms: int = 148, **opts):
    """The plan gemm_chain / Chain would make (pure host computation, no GPU
    needed): specs is a sequence of dicts with keys M, N, K and optionally
    dep, epilogue, dep_cols.  The C call gets placeholder addresses (never
    dereferenced; a dep_cols task's X is its dependency's Y).  Returns
    (list of per-task dicts: the plan fields plus kernel, l2_prefetch_stages,
    k_order, dep_ring_stages; number of kernels)."""
    n = len(specs)
    arr = (_Task * n)()
    base = 1 << 32
    for i, t in enumerate(specs):
        x, w, y = base + (3 * i) * (1 << 24), base + (3 * i + 1) * (1 << 24), base + (3 * i + 2) * (1 << 24)
        dep = t.get("dep", -1)
        if t.get("dep_cols"):
            x = arr[dep].Y
        arr[i].X, arr[i].W, arr[i].Y = x, w, y
        arr[i].M, arr[i].N, arr[i].K, arr[i].dep = t["M"], t["N"], t["K"], dep
        arr[i].Yf32 = None
        arr[i].epilogue = t.get("epilogue", EPI_NONE)
        arr[i].R = base - (1 << 24) if arr[i].epilogue == EPI_RESIDUAL else None
        arr[i].dep_cols = 1 if t.get("dep_cols") else 0
        arr[i].m_tile = t.get("m_tile", 0)
    out = (_ChainTaskInfo * max(n, 1))()
    nk = ctypes.c_int(0)
    o = _chain_opts(**opts)
    _check(lib().wsm_chain_plan(arr, n, ctypes.byref(o), num_sms, out, ctypes.byref(nk)), "wsm_chain_plan")
    res = []
    for i in range(n):
        d = {f: getattr(out[i].plan, f) for f, _ in _PlanInfo._fields_}
        d.update(kernel=out[i].kernel, l2_prefetch_stages=out[i].l2_prefetch_stages, k_order=out[i].k_order,
                 dep_ring_stages=out[i].dep_ring_stages, cluster=out[i].cluster, die_split=out[i].die_split)
        res.append(d)
    return res, nk.value


class Chain:
    """A prepared chain of GEMMs run as one persistent kernel."""

    def __init__(self, tasks: Sequence[Task], *, path=PATH_AUTO, grid=0, timeout_ns=0, trace=False,
                 debug_unmet_dependency=False, flags=0, stage_k=0, unit_stages=0, tail_tiles=0,
                 tail_unit_stages=0, l2_prefetch_stages=0, counter_groups=0, kernels=0, tile_rows=0, k_order=0,
                 dep_ring_stages=0, cluster=0, die_groups=0):
        for i, t in enumerate(tasks):
            _check_operand(f"tasks[{i}].x", t.x)
            _check_operand(f"tasks[{i}].w", t.w)
            _check_operand(f"tasks[{i}].y", t.y)
        self.tasks = list(tasks)  # keeps the tensors alive
        arr = _tasks_array(self.tasks)
        o = _chain_opts(path=path, grid=grid, timeout_ns=timeout_ns, trace=trace,
                        debug_unmet_dependency=debug_unmet_dependency, flags=flags, stage_k=stage_k,
                        unit_stages=unit_stages, tail_tiles=tail_tiles, tail_unit_stages=tail_unit_stages,
                        l2_prefetch_stages=l2_prefetch_stages, counter_groups=counter_groups, kernels=kernels,
                        tile_rows=tile_rows, k_order=k_order, dep_ring_stages=dep_ring_stages, cluster=cluster,
                        die_groups=die_groups)
        h = ctypes.c_void_p()
        _check(lib().wsm_chain_create(arr, len(tasks), ctypes.byref(o), ctypes.byref(h)), "wsm_chain_create")
        self._h = h

    def run(self, stream=None):
        _check(lib().wsm_chain_run(self._h, _stream_handle(stream)), "wsm_chain_run")

    def status(self, stream=None):
        """Synchronise; returns (code, failed_task)."""
        ft = ctypes.c_int(-1)
        code = lib().wsm_chain_status(self._h, _stream_handle(stream), ctypes.byref(ft))
        return code, ft.value

    def task_plan(self, task: int) -> dict:
        """The plan of one task of the chain (as `plan` reports for a single call)."""
        info = _PlanInfo()
        _check(lib().wsm_chain_task_plan(self._h, task, ctypes.byref(info)), "wsm_chain_task_plan")
        return {f: getattr(info, f) for f, _ in _PlanInfo._fields_}

    def trace(self, stream=None):
        """Per-CTA, per-task stamps [grid, n_tasks, 8] (%globaltimer ns, 0 = no such event):
        first stage issued, dependency met, last unit's outputs written, SM id, last unit's
        accumulator at the epilogue, its split-K arrival counted, its reduction done (last
        arriver), first stage complete at the MMA issuer (the last four on the tensor-core
        path only); or None."""
        n = lib().wsm_chain_trace(self._h, _stream_handle(stream), None, 0)
        if n == 0:
            return None
        buf = (ctypes.c_ulonglong * n)()
        lib().wsm_chain_trace(self._h, _stream_handle(stream), buf, n)
        t = torch.tensor(list(buf), dtype=torch.int64)
        return t.view(-1, len(self.tasks), 8)

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            lib().wsm_chain_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def gemm_chain(tasks: Sequence[Task], stream=None):
    """One-shot chain run (prepared chains are cached by the library)."""
    arr = _tasks_array(tasks)
    _check(lib().gemm_chain(arr, len(tasks), _stream_handle(stream)), "gemm_chain")
