"""skinny_gemm_noalloc, the entry point for callers that cannot allocate
device memory once running: an inference loop that reserved its whole memory
budget at start-up, a host framework whose own allocator must own every
device allocation, or code that cannot afford cudaMalloc's implicit
synchronisation.  Its scratch is a fixed array in the library's device image.

Checked through the C ABI on two calls in a row (the second one finds the
first one's leftovers in the shared array): against the fp64 oracle with the
same acceptance as every other parity test, and bit for bit against
skinny_gemm (same plan, deterministic in-order split-K reduction).  Also: it
allocates no device memory (free memory unchanged across calls on a fresh
stream, while skinny_gemm on a fresh stream visibly allocates its
workspace), its refusal of shapes whose scratch does not fit, and the
reporting of a device-side time-out recorded in the array.

The file name makes pytest collect it last."""
import ctypes

import pytest
import torch

import synth
import weight_streaming_megakernel_b200 as wsm
from parity import bf16_bits, check_full

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield
    wsm.debug_stall(0)


def _new_cuda_stream():
    """A stream created just now with cudaStreamCreateWithFlags (torch's own
    streams come from a pool whose handles earlier tests may have used)."""
    import glob
    import os
    libdir = os.path.join(os.path.dirname(torch.__file__), "..", "nvidia", "cuda_runtime", "lib")
    rt = ctypes.CDLL(sorted(glob.glob(os.path.join(libdir, "libcudart.so*")))[0])
    h = ctypes.c_void_p()
    assert rt.cudaStreamCreateWithFlags(ctypes.byref(h), ctypes.c_uint(1)) == 0  # non-blocking
    return rt, h, torch.cuda.ExternalStream(h.value)


def _call_noalloc(x, w, y, stream=None):
    L = wsm.lib()
    M, K = x.shape
    N = w.shape[0]
    s = (stream or torch.cuda.current_stream()).cuda_stream
    return L.skinny_gemm_noalloc(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(w.data_ptr()),
                                 ctypes.c_void_p(y.data_ptr()), M, N, K, ctypes.c_void_p(s))


# FMA path, tensor-core path with split tiles, a skinny shape, M-tile padding, whole tiles
@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (16, 6144, 4096), (4, 2112, 7168), (32, 1000, 2048),
                                   (16, 24576, 4096)])
def test_noalloc_matches_oracle_and_skinny_gemm(M, N, K):
    x, w = synth.make_xw(M, N, K, seed=M + N)
    xd, wd = x.to(DEV), w.to(DEV)
    y_ref = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    wsm.skinny_gemm(xd, wd, y_ref)
    torch.cuda.synchronize()
    for call in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
        rc = _call_noalloc(xd, wd, y)
        assert rc == wsm.WSM_OK, wsm.last_error()
        torch.cuda.synchronize()
        check_full(x, w, y, what=f"noalloc call {call}")
        assert (bf16_bits(y) == bf16_bits(y_ref)).all(), f"call {call}: bits differ from skinny_gemm"
    assert wsm.stream_status() == 0


def test_noalloc_allocates_no_device_memory():
    M, N, K = 64, 8192, 8192   # a split-K plan with a 4 MiB scratch
    x, w = synth.make_xw(M, N, K, seed=7)
    xd, wd = x.to(DEV), w.to(DEV)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    assert _call_noalloc(xd, wd, y) == wsm.WSM_OK, wsm.last_error()  # first call: module and kernel set-up
    torch.cuda.synchronize()
    rt, h1, fresh = _new_cuda_stream()
    rt2, h2, other = _new_cuda_stream()
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(2):
        assert _call_noalloc(xd, wd, y, stream=fresh) == wsm.WSM_OK, wsm.last_error()
    fresh.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0, "skinny_gemm_noalloc allocated device memory"
    # the measurement is sensitive: skinny_gemm on another new stream allocates that stream's scratch
    free1 = torch.cuda.mem_get_info()[0]
    wsm.skinny_gemm(xd, wd, y, stream=other)
    other.synchronize()
    assert free1 - torch.cuda.mem_get_info()[0] >= (2 << 20)
    torch.cuda.synchronize()
    rt.cudaStreamDestroy(h1)
    rt2.cudaStreamDestroy(h2)


def test_noalloc_timeout_reported_once_then_correct():
    """A device-side time-out inside a noalloc call (the stall test hook) is
    kept in the array's status words -- later calls do not clear it -- and
    reported once by wsm_stream_status; the call after it is correct."""
    M, N, K = 16, 6144, 4096   # split tiles: the abandoned units leave tile counters mid-count
    x, w = synth.make_xw(M, N, K, seed=11)
    xd, wd = x.to(DEV), w.to(DEV)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    assert wsm.stream_status() == 0
    wsm.debug_stall(1, 50_000_000)
    assert _call_noalloc(xd, wd, y) == wsm.WSM_OK, wsm.last_error()
    y2 = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    assert _call_noalloc(xd, wd, y2) == wsm.WSM_OK, wsm.last_error()
    assert wsm.stream_status() == wsm.WSM_ERR_TIMEOUT
    assert "skinny_gemm_noalloc" in wsm.last_error()
    assert wsm.stream_status() == 0
    check_full(x, w, y2, what="the noalloc call after the time-out")


def test_noalloc_rejects_shapes_that_do_not_fit():
    M, N, K = 64, 57344, 8192
    assert wsm.workspace_bytes(M, N, K) > (16 << 20)
    x = torch.zeros(M, K, dtype=torch.bfloat16, device=DEV)
    w = torch.zeros(N, K, dtype=torch.bfloat16, device=DEV)
    y = torch.zeros(M, N, dtype=torch.bfloat16, device=DEV)
    rc = _call_noalloc(x, w, y)
    assert rc == wsm.WSM_ERR_UNSUPPORTED
    msg = wsm.last_error()
    assert "skinny_gemm_noalloc" in msg and str(16 << 20) in msg
