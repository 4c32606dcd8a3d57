"""skinny_gemm_noalloc, the entry point for callers that cannot allocate
device memory once running (a fixed memory budget, a foreign allocator that
must own all device memory, or no tolerance for cudaMalloc's implicit
synchronisation).  Its scratch is a fixed array in the library's device
image.  Checked through the C ABI against skinny_gemm on the same inputs, on
two calls in a row (the second one finds the first one's leftovers in the
shared array), and for its refusal of shapes whose scratch does not fit.

The file name makes pytest collect it last."""
import ctypes

import numpy as np
import pytest
import torch

import synth
import weight_streaming_megakernel_b200 as wsm
from parity import bf16_bits, ulp_distance

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    yield


def _call_noalloc(x, w, y):
    L = wsm.lib()
    M, K = x.shape
    N = w.shape[0]
    s = torch.cuda.current_stream().cuda_stream
    return L.skinny_gemm_noalloc(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(w.data_ptr()),
                                 ctypes.c_void_p(y.data_ptr()), M, N, K, ctypes.c_void_p(s))


# FMA path, tensor-core path with split tiles, a skinny shape, M-tile padding
@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (16, 6144, 4096), (4, 2112, 7168), (32, 1000, 2048),
                                   (16, 24576, 4096)])
def test_noalloc_matches_skinny_gemm(M, N, K):
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
        d = ulp_distance(bf16_bits(y), bf16_bits(y_ref))
        assert int(d.max()) <= 1, f"call {call}: differs from skinny_gemm by {int(d.max())} ulp"
        assert not torch.isnan(y.float()).any()


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
