// wsm_noalloc.cu -- skinny_gemm_noalloc: the same GEMM as skinny_gemm, with
// its scratch (status word, work-unit and tile counters, split-K partials) in
// one fixed-size array that lives in the library's device image instead of
// memory obtained with cudaMalloc.
//
// Who needs it: code that must not allocate device memory once it is running
// -- an inference loop that has reserved its whole memory budget up front, a
// host framework whose own allocator owns all device memory and must not see
// foreign allocations, or a caller on a latency-critical path where
// cudaMalloc's implicit synchronisation is unacceptable.  skinny_gemm would
// allocate a per-stream scratch buffer on the first call on each stream; this
// entry point never does.
#include "wsm_internal.cuh"
#include "../../include/wsm.h"

#include <cstdio>
#include <cstring>
#include <mutex>

namespace wsm {
void set_last_error_message(const char *msg);  // wsm_api.cu: what wsm_last_error() returns
}

namespace {

// The scratch: zero at module load, reused by every call on this device.
// Device memory held by every GPU that loads the library, until exit.
static __device__ __align__(256) unsigned char g_noalloc_scratch[WSM_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
// Per device: the device address of g_noalloc_scratch and the context it was looked up in.  After a
// device reset the primary context (and with it the module's memory) is new: the address is looked up
// again when the current context differs.
void *g_noalloc_ptr[kMaxDevices] = {};
CUcontext g_noalloc_ctx[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
CtxGetCurrentFn g_ctx_get_current = nullptr;

wsm_status noalloc_fail(wsm_status code, const char *msg) {
    wsm::set_last_error_message(msg);
    return code;
}

// The current context (nullptr if the driver entry point is unavailable).  Caller holds g_noalloc_mu.
CUcontext current_context() {
    if (!g_ctx_get_current) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &fn, 12000, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return nullptr;
        g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(fn);
    }
    CUcontext c = nullptr;
    if (g_ctx_get_current(&c) != CUDA_SUCCESS) return nullptr;
    return c;
}

}  // namespace

namespace wsm {
// The array's device address on `dev` if a call has set it up there in the current context, else nullptr
// (wsm_stream_status reads the array's status words through it).
void *noalloc_scratch_ptr(int dev) {
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev] || g_noalloc_ctx[dev] != current_context()) return nullptr;
    return g_noalloc_ptr[dev];
}
}  // namespace wsm

extern "C" {

wsm_status skinny_gemm_noalloc(const void *X, const void *W, void *Y, int M, int N, int K, wsm_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return noalloc_fail(WSM_ERR_CUDA, "skinny_gemm_noalloc: cudaGetDevice failed");
    if (dev < 0 || dev >= kMaxDevices) return noalloc_fail(WSM_ERR_UNSUPPORTED, "skinny_gemm_noalloc: device index too large");

    // Set-up, once per device (again after a device reset), with that device
    // current: the host-side name of the array is only a stand-in, so look up
    // its device address.
    void *scratch = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_noalloc_mu);
        const CUcontext ctx = current_context();
        if (!g_noalloc_ptr[dev] || g_noalloc_ctx[dev] != ctx) {
            void *p = nullptr;
            e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
            if (e != cudaSuccess || !p) {
                char buf[256];
                snprintf(buf, sizeof buf, "skinny_gemm_noalloc: cudaGetSymbolAddress failed on device %d: %s", dev,
                         cudaGetErrorString(e));
                return noalloc_fail(WSM_ERR_CUDA, buf);
            }
            g_noalloc_ptr[dev] = p;
            g_noalloc_ctx[dev] = ctx;
        }
        scratch = g_noalloc_ptr[dev];
    }

    // Arguments are checked before anything is queued.
    if (!X || !W || !Y) return noalloc_fail(WSM_ERR_INVALID, "X, W and Y must be non-null device pointers");
    if (((reinterpret_cast<uintptr_t>(X) | reinterpret_cast<uintptr_t>(W) | reinterpret_cast<uintptr_t>(Y)) & 15u) != 0)
        return noalloc_fail(WSM_ERR_ALIGN, "X, W and Y must be 16-byte aligned");

    // The same plan skinny_gemm would use; refuse shapes whose scratch does not fit.
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return noalloc_fail(WSM_ERR_CUDA, "skinny_gemm_noalloc: cannot read the SM count");
    wsm_plan_info info;
    wsm_status st = wsm_plan(M, N, K, sms, nullptr, &info);
    if (st != WSM_OK) return st;  // wsm_last_error() has the message
    if (info.workspace_bytes > (size_t)WSM_NOALLOC_SCRATCH_BYTES) {
        char buf[256];
        snprintf(buf, sizeof buf,
                 "skinny_gemm_noalloc: M=%d N=%d K=%d needs %zu bytes of scratch, more than the fixed %d bytes; "
                 "use skinny_gemm or skinny_gemm_ex with a workspace",
                 M, N, K, info.workspace_bytes, WSM_NOALLOC_SCRATCH_BYTES);
        return noalloc_fail(WSM_ERR_UNSUPPORTED, buf);
    }

    // The array keeps the previous call's contents: clear the counters this
    // call will use (they must start at zero).  The status words before them
    // are left alone: a time-out recorded by an earlier call stays there until
    // wsm_stream_status reads it.  Calls whose work overlaps on the GPU share
    // the array and race.
    const size_t counters = 4 * ((size_t)wsm::kSchedWords + (size_t)info.n_tiles * (size_t)info.m_tiles);
    e = cudaMemsetAsync(static_cast<unsigned char *>(scratch) + 256, 0, counters, stream);
    if (e != cudaSuccess) return noalloc_fail(WSM_ERR_CUDA, "skinny_gemm_noalloc: clearing the scratch failed");

    wsm_opts o;
    memset(&o, 0, sizeof o);
    o.workspace = scratch;
    o.workspace_bytes = (size_t)WSM_NOALLOC_SCRATCH_BYTES;
    return skinny_gemm_ex(X, W, Y, M, N, K, &o, stream_);
}

}  // extern "C"
