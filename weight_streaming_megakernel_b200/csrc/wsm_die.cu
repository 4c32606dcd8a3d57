// wsm_die.cu -- which die of the GPU each SM sits on, measured.
//
// A B200 is two dies, each with its own half of the L2; every global address
// is homed in one of them, and an SM reaches lines homed on the other die
// over the die-to-die link, a few hundred cycles further away.  CUDA does not
// say which SM is on which die, so this measures it: one CTA per SM times L2
// hits (ld.global.cg, serialised by a data dependency) to a set of lines;
// each line is fast for the SMs of its home die and slow for the others, so
// SMs of one die agree on which lines are near.  The first SM seen is the
// reference: an SM whose near/far pattern agrees with it on most lines is on
// its die.  Used to group CTAs by die, the chiplet-aware scheduling of
// "Fleet: Hierarchical Task-based Abstraction for Megakernels on Multi-Die
// GPUs" (reading notes, sections 3b and 3f), adapted: there, per-XCD private
// L2s; here, one coherent L2 split across two dies.
#include "wsm_internal.cuh"
#include "../../include/wsm.h"

#include <algorithm>
#include <cstdio>
#include <mutex>
#include <vector>

namespace wsm {
void set_last_error_message(const char *msg);

namespace {

constexpr int kProbeLines = 2048;      // lines timed per SM
constexpr int kProbeStrideWords = 128;  // 512 bytes between probed lines (a 1 MiB span)
constexpr int kProbeReps = 4;           // the fastest of these per line (the first one fills L2)
constexpr int kMaxSmId = 1024;

__device__ __forceinline__ unsigned long long clock_now() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%clock64;" : "=l"(t)::"memory");
    return t;
}
// The clock after `v` has arrived: a volatile shared store of v must wait for the load, and the volatile
// clock read is not moved above it (an arithmetic use of v would not hold the clock read back).
__device__ __forceinline__ unsigned long long clock_after(unsigned int v, unsigned int *sink) {
    asm volatile("st.volatile.shared.u32 [%0], %1;" ::"r"(smem_u32(sink)), "r"(v) : "memory");
    return clock_now();
}

// One CTA per SM (the dynamic shared memory keeps a second one off): thread 0 times its loads.
__global__ void __launch_bounds__(32, 1) sm_latency_probe(const unsigned int *lines, unsigned int *lat,
                                                          int *sm_of_cta) {
    __shared__ unsigned int sink;
    if (threadIdx.x != 0) return;
    const uint32_t sm = smid();
    sm_of_cta[blockIdx.x] = (int)sm;
    if (sm >= (uint32_t)kMaxSmId) return;
    unsigned int dep = 0;  // loaded values are all zero: adding them serialises the loads
    for (int i = 0; i < kProbeLines; ++i) {
        unsigned int best = 0xffffffffu;
        for (int r = 0; r < kProbeReps; ++r) {
            const unsigned int *a = lines + (size_t)i * kProbeStrideWords + dep;
            const unsigned long long t0 = clock_now();
            unsigned int v;
            asm volatile("ld.global.cg.u32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
            const unsigned long long t1 = clock_after(v, &sink);
            dep += v;
            best = min(best, (unsigned int)(t1 - t0));
        }
        lat[(size_t)sm * kProbeLines + i] = best;
    }
}

struct DieMap {
    bool done = false;
    std::vector<int> die;  // by SM id
    wsm_die_info info{};
};
std::mutex g_die_mu;
std::vector<DieMap> g_die_maps;

wsm_status die_fail(wsm_status code, const char *msg) {
    set_last_error_message(msg);
    return code;
}

#define DIE_CUDA(call)                                                                     \
    do {                                                                                   \
        cudaError_t e_ = (call);                                                           \
        if (e_ != cudaSuccess) {                                                           \
            char b_[256];                                                                  \
            snprintf(b_, sizeof b_, "wsm_sm_die_map: %s: %s", #call, cudaGetErrorString(e_)); \
            return die_fail(WSM_ERR_CUDA, b_);                                             \
        }                                                                                  \
    } while (0)

wsm_status measure(int dev, DieMap &m) {
    int sms = 0;
    DIE_CUDA(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    int smem_optin = 0;
    DIE_CUDA(cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev));
    unsigned int *lines = nullptr, *lat = nullptr;
    int *sm_of_cta = nullptr;
    const size_t line_bytes = (size_t)kProbeLines * kProbeStrideWords * 4 + 4096;
    const size_t lat_bytes = (size_t)kMaxSmId * kProbeLines * 4;
    DIE_CUDA(cudaMalloc(&lines, line_bytes));
    cudaError_t e = cudaMalloc(&lat, lat_bytes);
    if (e == cudaSuccess) e = cudaMalloc(&sm_of_cta, sizeof(int) * sms);
    if (e == cudaSuccess) e = cudaMemset(lines, 0, line_bytes);
    if (e == cudaSuccess) e = cudaMemset(lat, 0, lat_bytes);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(sm_latency_probe, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   smem_optin - 1024);
    if (e == cudaSuccess) {
        // one CTA per SM: each needs more than half an SM's shared memory; cooperative, so all are resident
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)sms);
        cfg.blockDim = dim3(32);
        cfg.dynamicSmemBytes = (size_t)(smem_optin - 1024);
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        void *args[3] = {&lines, &lat, &sm_of_cta};
        e = cudaLaunchKernelExC(&cfg, reinterpret_cast<const void *>(&sm_latency_probe), args);
    }
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    std::vector<unsigned int> h((size_t)kMaxSmId * kProbeLines);
    std::vector<int> ids(sms);
    if (e == cudaSuccess) e = cudaMemcpy(h.data(), lat, lat_bytes, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemcpy(ids.data(), sm_of_cta, sizeof(int) * sms, cudaMemcpyDeviceToHost);
    cudaFree(lines);
    cudaFree(lat);
    cudaFree(sm_of_cta);
    if (e != cudaSuccess) {
        char b[256];
        snprintf(b, sizeof b, "wsm_sm_die_map: the probe failed: %s", cudaGetErrorString(e));
        return die_fail(WSM_ERR_CUDA, b);
    }
    std::vector<int> seen;
    for (int id : ids)
        if (id >= 0 && id < kMaxSmId && std::find(seen.begin(), seen.end(), id) == seen.end()) seen.push_back(id);
    if ((int)seen.size() != sms)
        return die_fail(WSM_ERR_CUDA, "wsm_sm_die_map: the probe's CTAs did not land on every SM once");
    std::sort(seen.begin(), seen.end());
    // per line: near for an SM when below the line's median over the SMs
    const int n = (int)seen.size();
    std::vector<char> near((size_t)n * kProbeLines);
    for (int i = 0; i < kProbeLines; ++i) {
        std::vector<unsigned int> col(n);
        for (int s = 0; s < n; ++s) col[s] = h[(size_t)seen[s] * kProbeLines + i];
        std::vector<unsigned int> sorted = col;
        std::nth_element(sorted.begin(), sorted.begin() + n / 2, sorted.end());
        const unsigned int med = sorted[n / 2];
        for (int s = 0; s < n; ++s) near[(size_t)s * kProbeLines + i] = col[s] < med;
    }
    // agreement of every SM's pattern with the reference SM's
    m.die.assign(kMaxSmId, -1);
    double same = 0, other = 0;
    int n0 = 0, n1 = 0;
    double lat_near = 0, lat_far = 0;
    long long c_near = 0, c_far = 0;
    for (int s = 0; s < n; ++s) {
        int agree = 0;
        for (int i = 0; i < kProbeLines; ++i) agree += near[(size_t)s * kProbeLines + i] == near[i];
        const double a = (double)agree / kProbeLines;
        const int d = a >= 0.5 ? 0 : 1;
        m.die[seen[s]] = d;
        (d == 0 ? n0 : n1) += 1;
        (d == 0 ? same : other) += d == 0 ? a : 1.0 - a;
    }
    // near/far latencies: for each line, the lower of the two dies' mean latencies is the home die's
    for (int i = 0; i < kProbeLines; ++i) {
        double sum[2] = {0, 0};
        int cnt[2] = {0, 0};
        for (int s = 0; s < n; ++s) {
            const int d = m.die[seen[s]];
            sum[d] += h[(size_t)seen[s] * kProbeLines + i];
            ++cnt[d];
        }
        if (!cnt[0] || !cnt[1]) continue;
        const double a0 = sum[0] / cnt[0], a1 = sum[1] / cnt[1];
        lat_near += std::min(a0, a1);
        lat_far += std::max(a0, a1);
        ++c_near;
        ++c_far;
    }
    m.info.num_sms = n;
    m.info.sms_die0 = n0;
    m.info.sms_die1 = n1;
    m.info.agreement = (float)((same + other) / n);
    m.info.near_cycles = c_near ? (float)(lat_near / c_near) : 0.f;
    m.info.far_cycles = c_far ? (float)(lat_far / c_far) : 0.f;
    // two dies only if the patterns split the SMs cleanly in two groups
    m.info.dies = (n0 > 0 && n1 > 0 && m.info.agreement >= 0.75f) ? 2 : 1;
    if (m.info.dies == 1)
        for (int s = 0; s < n; ++s) m.die[seen[s]] = 0;
    m.done = true;
    return WSM_OK;
}

}  // namespace

// Die of each SM id on the current device (measured once per device, then cached); -1 for SM ids that do
// not exist.  Used by chain creation for die-grouped claims.
wsm_status die_map_of_device(int dev, const std::vector<int> **die, wsm_die_info *info) {
    std::lock_guard<std::mutex> lk(g_die_mu);
    if (dev < 0) return die_fail(WSM_ERR_INVALID, "bad device");
    if ((int)g_die_maps.size() <= dev) g_die_maps.resize(dev + 1);
    DieMap &m = g_die_maps[dev];
    if (!m.done) {
        wsm_status st = measure(dev, m);
        if (st != WSM_OK) return st;
    }
    if (die) *die = &m.die;
    if (info) *info = m.info;
    return WSM_OK;
}

}  // namespace wsm

extern "C" wsm_status wsm_sm_die_map(int *die_of_sm, int capacity, wsm_die_info *info) {
    if (capacity < 0 || (capacity > 0 && !die_of_sm))
        return wsm::die_fail(WSM_ERR_INVALID, "wsm_sm_die_map: die_of_sm must hold `capacity` ints");
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return wsm::die_fail(WSM_ERR_CUDA, "wsm_sm_die_map: no CUDA device");
    const std::vector<int> *die = nullptr;
    wsm_status st = wsm::die_map_of_device(dev, &die, info);
    if (st != WSM_OK) return st;
    for (int i = 0; i < capacity; ++i) die_of_sm[i] = i < (int)die->size() ? (*die)[i] : -1;
    wsm::set_last_error_message("");
    return WSM_OK;
}
