// Forward from host buffers with the copies overlapped: thd_attn_fwd_host.
//
// The pack is split into token ranges [t_c, t_{c+1}).  Range c's host-to-
// device copy of q, k, v rows runs on a copy stream, its attention
// (thd_attn_fwd_range: queries of the range against the keys before them)
// on the caller's stream once that copy has landed, and the device-to-host
// copy of its out / lse rows on a second copy stream once the attention is
// done.  A query row only sees keys of its own document at or before it, so
// range c needs no key rows past t_{c+1}: every row it reads was copied by
// range c or an earlier one, and the three engines (two copy directions and
// the SMs) work on different ranges at the same time.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "../../include/thd_attn.h"

namespace {

constexpr int kMaxChunks = 64;

struct Pipeline {
    cudaStream_t h2d = nullptr, d2h = nullptr;
    std::vector<cudaEvent_t> events;  // start, done, then h2d[c] and comp[c] per range
};

std::mutex g_mu;
std::unordered_map<int, Pipeline> g_pipes;

// The current device's copy streams and events (created on first use).
int get_pipeline(Pipeline** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return THD_ERR_CUDA;
    Pipeline& p = g_pipes[dev];
    if (p.h2d == nullptr) {
        if (cudaStreamCreateWithFlags(&p.h2d, cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&p.d2h, cudaStreamNonBlocking) != cudaSuccess)
            return THD_ERR_CUDA;
        p.events.resize(2 + 2 * kMaxChunks);
        for (auto& e : p.events)
            if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return THD_ERR_CUDA;
    }
    *out = &p;
    return THD_OK;
}

}  // namespace

extern "C" int thd_attn_fwd_host(const void* q_host, const void* k_host, const void* v_host,
                                 const int32_t* cu_seqlens, int n_docs, int Hq, int Hkv, int D,
                                 int window, float scale, const float* sinks_host_or_null,
                                 void* out_host, float* lse_host, void* q_dev, void* k_dev,
                                 void* v_dev, float* sinks_dev_or_null, void* out_dev,
                                 float* lse_dev, int n_chunks, void* stream_ptr) {
    if (cu_seqlens == nullptr || n_docs < 0 || Hq <= 0 || Hkv <= 0 || D <= 0) return THD_ERR_INVALID_ARG;
    if (n_chunks < 1 || n_chunks > kMaxChunks) return THD_ERR_INVALID_ARG;
    if ((sinks_host_or_null == nullptr) != (sinks_dev_or_null == nullptr)) return THD_ERR_INVALID_ARG;
    if (cu_seqlens[0] != 0) return THD_ERR_INVALID_ARG;
    for (int d = 0; d < n_docs; ++d)
        if (cu_seqlens[d + 1] < cu_seqlens[d]) return THD_ERR_INVALID_ARG;
    const int64_t T = cu_seqlens[n_docs];
    if (T == 0) return THD_OK;
    if (!q_host || !k_host || !v_host || !out_host || !lse_host || !q_dev || !k_dev || !v_dev ||
        !out_dev || !lse_dev)
        return THD_ERR_INVALID_ARG;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);

    // One call at a time per process: the streams and events are shared.
    std::lock_guard<std::mutex> lock(g_mu);
    Pipeline* p = nullptr;
    int rc = get_pipeline(&p);
    if (rc != THD_OK) return rc;
    cudaEvent_t ev_start = p->events[0], ev_done = p->events[1];
    const size_t q_row = static_cast<size_t>(Hq) * D * 2, kv_row = static_cast<size_t>(Hkv) * D * 2;
    const size_t o_row = q_row, l_row = static_cast<size_t>(Hq) * sizeof(float);
    auto at = [](const void* base, int64_t row, size_t row_bytes) {
        return static_cast<const char*>(base) + static_cast<size_t>(row) * row_bytes;
    };
    auto atw = [](void* base, int64_t row, size_t row_bytes) {
        return static_cast<char*>(base) + static_cast<size_t>(row) * row_bytes;
    };

    // The copies start after the work already queued on the caller's stream
    // (an earlier call may still read the device buffers).
    if (cudaEventRecord(ev_start, stream) != cudaSuccess ||
        cudaStreamWaitEvent(p->h2d, ev_start, 0) != cudaSuccess ||
        cudaStreamWaitEvent(p->d2h, ev_start, 0) != cudaSuccess)
        return THD_ERR_CUDA;
    if (sinks_host_or_null != nullptr &&
        cudaMemcpyAsync(sinks_dev_or_null, sinks_host_or_null, sizeof(float) * Hq,
                        cudaMemcpyHostToDevice, p->h2d) != cudaSuccess)
        return THD_ERR_CUDA;

    for (int c = 0; c < n_chunks && rc == THD_OK; ++c) {
        const int64_t t0 = T * c / n_chunks, t1 = T * (c + 1) / n_chunks;
        if (t1 == t0) continue;
        cudaEvent_t ev_h2d = p->events[2 + 2 * c], ev_comp = p->events[3 + 2 * c];
        const int64_t n = t1 - t0;
        if (cudaMemcpyAsync(atw(q_dev, t0, q_row), at(q_host, t0, q_row), n * q_row,
                            cudaMemcpyHostToDevice, p->h2d) != cudaSuccess ||
            cudaMemcpyAsync(atw(k_dev, t0, kv_row), at(k_host, t0, kv_row), n * kv_row,
                            cudaMemcpyHostToDevice, p->h2d) != cudaSuccess ||
            cudaMemcpyAsync(atw(v_dev, t0, kv_row), at(v_host, t0, kv_row), n * kv_row,
                            cudaMemcpyHostToDevice, p->h2d) != cudaSuccess ||
            cudaEventRecord(ev_h2d, p->h2d) != cudaSuccess ||
            cudaStreamWaitEvent(stream, ev_h2d, 0) != cudaSuccess) {
            rc = THD_ERR_CUDA;
            break;
        }
        rc = thd_attn_fwd_range(atw(q_dev, t0, q_row), k_dev, v_dev, cu_seqlens, n_docs, t0, t1, Hq,
                                Hkv, D, window, scale, sinks_dev_or_null, atw(out_dev, t0, o_row),
                                reinterpret_cast<float*>(atw(lse_dev, t0, l_row)), stream);
        if (rc != THD_OK) break;
        if (cudaEventRecord(ev_comp, stream) != cudaSuccess ||
            cudaStreamWaitEvent(p->d2h, ev_comp, 0) != cudaSuccess ||
            cudaMemcpyAsync(atw(out_host, t0, o_row), at(out_dev, t0, o_row), n * o_row,
                            cudaMemcpyDeviceToHost, p->d2h) != cudaSuccess ||
            cudaMemcpyAsync(atw(lse_host, t0, l_row), at(lse_dev, t0, l_row), n * l_row,
                            cudaMemcpyDeviceToHost, p->d2h) != cudaSuccess)
            rc = THD_ERR_CUDA;
    }
    // The caller's stream completes only after every copy queued above (the
    // last device-to-host copy follows all the others through the events).
    if (cudaEventRecord(ev_done, p->d2h) != cudaSuccess ||
        cudaStreamWaitEvent(stream, ev_done, 0) != cudaSuccess)
        return THD_ERR_CUDA;
    return rc;
}
