// C ABI of the packed-THD attention forward (declared in include/thd_attn.h):
// host validation, the per-device schedule cache and status word, TMA
// descriptor encoding and the kernel launch.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <list>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "../../include/thd_attn.h"
#include "scheduler.h"
#include "tma_map.h"
#include "thd_attn_kernel.cuh"
#include "thd_attn_split_kernel.cuh"
#include "thd_attn_bwd_kernels.cuh"

namespace {

using thd::KernelShape;

// ------------------------------------------------------------ kernel shapes --

using Cfg64x2 = thd::FwdConfig<64, 2, 1, 128, 8>;
using Cfg64x1 = thd::FwdConfig<64, 1, 2, 128, 8>;
using Cfg128x2 = thd::FwdConfig<128, 2, 1, 128, 5>;
using Cfg128x1 = thd::FwdConfig<128, 1, 2, 128, 6>;
using Cfg256x1 = thd::FwdConfig<256, 1, 2, 64, 5>;
using SplitCfg256 = thd::SplitConfig<256, 2, 4>;  // 2 heads per item over a CTA pair

constexpr int kNumVariants = 6;

int variant_index(const KernelShape& ks) {
    if (ks.pair) return 5;
    if (ks.D == 64) return ks.nq == 2 ? 0 : 1;
    if (ks.D == 128) return ks.nq == 2 ? 2 : 3;
    return 4;
}

// ---------------------------------------------------------- per-device state --

struct PlanEntry {
    std::vector<int32_t> cu;
    int Hq, Hkv, D, window;
    int64_t q_begin, q_end;  // query rows of the pack the plan covers
    int64_t k_end;           // keys j < k_end only (T: all)
    thd::WorkItem* d_items = nullptr;
    int64_t n_items = 0;
};

// Backward schedules: the dq kernel's items (one query head each) and the
// dk/dv kernel's items.
struct BwdPlanEntry {
    std::vector<int32_t> cu;
    int Hq, Hkv, D, window;
    thd::WorkItem* d_q_items = nullptr;
    int64_t n_q_items = 0;
    thd::BwdKVItem* d_kv_items = nullptr;
    int64_t n_kv_items = 0;
};

constexpr int kNumBwdVariants = 7;  // {dq, dkdv} x {D = 64, D = 128}, then dq, dv, dk at D = 256

struct DeviceState {
    int* d_status = nullptr;
    bool attr_set[kNumVariants] = {};
    bool bwd_attr_set[kNumBwdVariants] = {};
    std::list<PlanEntry> plans;         // most recently used first
    std::list<BwdPlanEntry> bwd_plans;  // most recently used first
};

constexpr size_t kMaxPlans = 40;  // per direction; the host pipeline's ranges each take one

std::mutex g_mu;
std::unordered_map<int, DeviceState> g_devices;

using thd::aligned16;
using thd::make_map;

// Returns the device state of the current device (created on first use).
// Caller holds g_mu.
int device_state(DeviceState** out, int* dev_out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return THD_ERR_CUDA;
    auto it = g_devices.find(dev);
    if (it == g_devices.end()) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return THD_ERR_CUDA;
        if (major != 10 || minor != 0) return THD_ERR_UNSUPPORTED;
        DeviceState st;
        if (cudaMalloc(&st.d_status, sizeof(int)) != cudaSuccess) return THD_ERR_NO_MEMORY;
        if (cudaMemset(st.d_status, 0, sizeof(int)) != cudaSuccess) return THD_ERR_CUDA;
        it = g_devices.emplace(dev, std::move(st)).first;
    }
    *out = &it->second;
    if (dev_out) *dev_out = dev;
    return THD_OK;
}

// Finds or builds (and uploads) the plan for these arguments.  Caller holds g_mu.
int get_plan(DeviceState* ds, const int32_t* cu, int n_docs, int64_t q_begin, int64_t q_end,
             int64_t k_end, int Hq, int Hkv, int D, int window, const KernelShape& ks,
             cudaStream_t stream, const PlanEntry** out) {
    for (auto it = ds->plans.begin(); it != ds->plans.end(); ++it) {
        if (it->Hq == Hq && it->Hkv == Hkv && it->D == D && it->window == window &&
            it->q_begin == q_begin && it->q_end == q_end && it->k_end == k_end &&
            it->cu.size() == static_cast<size_t>(n_docs) + 1 &&
            std::memcmp(it->cu.data(), cu, sizeof(int32_t) * (n_docs + 1)) == 0) {
            ds->plans.splice(ds->plans.begin(), ds->plans, it);
            *out = &ds->plans.front();
            return THD_OK;
        }
    }
    std::vector<thd_work_item> items =
        thd::build_plan_range(cu, n_docs, q_begin, q_end, Hq, Hkv, window, ks, k_end);
    PlanEntry e;
    e.cu.assign(cu, cu + n_docs + 1);
    e.q_begin = q_begin;
    e.q_end = q_end;
    e.k_end = k_end;
    e.Hq = Hq;
    e.Hkv = Hkv;
    e.D = D;
    e.window = window;
    e.n_items = static_cast<int64_t>(items.size());
    if (!items.empty()) {
        const size_t bytes = items.size() * sizeof(thd::WorkItem);
        if (cudaMalloc(&e.d_items, bytes) != cudaSuccess) return THD_ERR_NO_MEMORY;
        if (cudaMemcpyAsync(e.d_items, items.data(), bytes, cudaMemcpyHostToDevice, stream) !=
                cudaSuccess ||
            cudaStreamSynchronize(stream) != cudaSuccess) {
            cudaFree(e.d_items);
            return THD_ERR_CUDA;
        }
    }
    if (ds->plans.size() >= kMaxPlans) {
        // cudaFree waits for kernels that may still read the evicted plan.
        if (ds->plans.back().d_items) cudaFree(ds->plans.back().d_items);
        ds->plans.pop_back();
    }
    ds->plans.push_front(std::move(e));
    *out = &ds->plans.front();
    return THD_OK;
}

template <class C>
int launch(DeviceState* ds, int vidx, const PlanEntry& plan, const CUtensorMap& mq,
           const CUtensorMap& mk, const CUtensorMap& mv, const thd::FwdParams& prm,
           cudaStream_t stream) {
    auto kern = thd::thd_attn_fwd_kernel<C>;
    if (!ds->attr_set[vidx]) {
        if (!thd::launch_registers_ok<C>()) return THD_ERR_UNSUPPORTED;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::SMEM_ALLOC) != cudaSuccess)
            return THD_ERR_CUDA;
        ds->attr_set[vidx] = true;
    }
    kern<<<static_cast<unsigned>(plan.n_items), C::NUM_THREADS, C::SMEM_ALLOC, stream>>>(mq, mk, mv,
                                                                                      prm);
    return cudaGetLastError() == cudaSuccess ? THD_OK : THD_ERR_CUDA;
}

// CTA-pair shapes: two CTAs (one cluster) per work item.
template <class C>
int launch_pair(DeviceState* ds, int vidx, const PlanEntry& plan, const CUtensorMap& mq,
                const CUtensorMap& mk, const CUtensorMap& mv, const thd::FwdParams& prm,
                cudaStream_t stream) {
    auto kern = thd::thd_attn_fwd_split_kernel<C>;
    if (!ds->attr_set[vidx]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::SMEM_ALLOC) != cudaSuccess)
            return THD_ERR_CUDA;
        ds->attr_set[vidx] = true;
    }
    kern<<<static_cast<unsigned>(2 * plan.n_items), C::NUM_THREADS, C::SMEM_ALLOC, stream>>>(
        mq, mk, mv, prm);
    return cudaGetLastError() == cudaSuccess ? THD_OK : THD_ERR_CUDA;
}

// Uploads `n` items to a new device buffer (synchronously on `stream`).
template <class T>
int upload(const std::vector<T>& v, T** out, cudaStream_t stream) {
    *out = nullptr;
    if (v.empty()) return THD_OK;
    const size_t bytes = v.size() * sizeof(T);
    if (cudaMalloc(out, bytes) != cudaSuccess) {
        *out = nullptr;
        return THD_ERR_NO_MEMORY;
    }
    if (cudaMemcpyAsync(*out, v.data(), bytes, cudaMemcpyHostToDevice, stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess) {
        cudaFree(*out);
        *out = nullptr;
        return THD_ERR_CUDA;
    }
    return THD_OK;
}

// Finds or builds the backward schedules for these arguments.  Caller holds g_mu.
int get_bwd_plan(DeviceState* ds, const int32_t* cu, int n_docs, int Hq, int Hkv, int D, int window,
                 cudaStream_t stream, const BwdPlanEntry** out) {
    for (auto it = ds->bwd_plans.begin(); it != ds->bwd_plans.end(); ++it) {
        if (it->Hq == Hq && it->Hkv == Hkv && it->D == D && it->window == window &&
            it->cu.size() == static_cast<size_t>(n_docs) + 1 &&
            std::memcmp(it->cu.data(), cu, sizeof(int32_t) * (n_docs + 1)) == 0) {
            ds->bwd_plans.splice(ds->bwd_plans.begin(), ds->bwd_plans, it);
            *out = &ds->bwd_plans.front();
            return THD_OK;
        }
    }
    // dq items: the forward's query tiles and key ranges, one query head each
    // (64-key tiles at head dim 256).
    const KernelShape qs{D, 1, 1, D == 256 ? 64 : 128, 4, false};
    std::vector<thd_work_item> qi = thd::build_plan(cu, n_docs, Hq, Hkv, window, qs);
    std::vector<thd_bwd_kv_item> ki = thd::build_bwd_kv_plan(cu, n_docs, Hq, Hkv, D, window);
    std::vector<thd::WorkItem> qv(qi.size());
    std::memcpy(qv.data(), qi.data(), qi.size() * sizeof(thd::WorkItem));
    std::vector<thd::BwdKVItem> kv(ki.size());
    std::memcpy(kv.data(), ki.data(), ki.size() * sizeof(thd::BwdKVItem));
    BwdPlanEntry e;
    e.cu.assign(cu, cu + n_docs + 1);
    e.Hq = Hq;
    e.Hkv = Hkv;
    e.D = D;
    e.window = window;
    int rc = upload(qv, &e.d_q_items, stream);
    if (rc != THD_OK) return rc;
    rc = upload(kv, &e.d_kv_items, stream);
    if (rc != THD_OK) {
        if (e.d_q_items) cudaFree(e.d_q_items);
        return rc;
    }
    e.n_q_items = static_cast<int64_t>(qv.size());
    e.n_kv_items = static_cast<int64_t>(kv.size());
    if (ds->bwd_plans.size() >= kMaxPlans) {
        auto& old = ds->bwd_plans.back();
        if (old.d_q_items) cudaFree(old.d_q_items);
        if (old.d_kv_items) cudaFree(old.d_kv_items);
        ds->bwd_plans.pop_back();
    }
    ds->bwd_plans.push_front(std::move(e));
    *out = &ds->bwd_plans.front();
    return THD_OK;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

template <int D>
int launch_bwd(DeviceState* ds, const BwdPlanEntry& plan, const CUtensorMap& mq,
               const CUtensorMap& mdo, const CUtensorMap& mk, const CUtensorMap& mv,
               const thd::BwdParams& prm, const void* out, const void* dout, const float* sinks,
               float* dsinks, float* delta, float* sink_part, cudaStream_t stream) {
    using Cq = thd::BwdConfig<D, D == 64 ? 8 : 5>;  // one CTA per SM (all 512 TMEM columns)
    using Ckv = thd::BwdConfig<D, D == 64 ? 4 : 2>;
    auto kq = thd::thd_attn_bwd_dq_kernel<Cq>;
    auto kkv = thd::thd_attn_bwd_dkdv_kernel<Ckv>;
    const int vq = D == 64 ? 0 : 2, vkv = vq + 1;
    if (!ds->bwd_attr_set[vq]) {
        if (cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 thd::DqLayout<Cq>::SMEM_ALLOC) != cudaSuccess)
            return THD_ERR_CUDA;
        ds->bwd_attr_set[vq] = true;
    }
    if (!ds->bwd_attr_set[vkv]) {
        if (cudaFuncSetAttribute(kkv, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 thd::DkvLayout<Ckv>::SMEM_ALLOC) != cudaSuccess)
            return THD_ERR_CUDA;
        ds->bwd_attr_set[vkv] = true;
    }
    const int64_t rows = prm.T * prm.Hq;
    thd::thd_attn_bwd_preprocess_kernel<D><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(dout), prm.lse,
        sinks, delta, sink_part, rows, prm.Hq);
    if (dsinks != nullptr) {
        if (sinks != nullptr)
            thd::thd_attn_bwd_dsink_kernel<<<prm.Hq, 256, 0, stream>>>(sink_part, prm.T, prm.Hq, dsinks);
        else if (cudaMemsetAsync(dsinks, 0, sizeof(float) * prm.Hq, stream) != cudaSuccess)
            return THD_ERR_CUDA;
    }
    if (plan.n_q_items > 0)
        kq<<<static_cast<unsigned>(plan.n_q_items), Cq::NUM_THREADS, thd::DqLayout<Cq>::SMEM_ALLOC,
             stream>>>(mq, mdo, mk, mv, prm);
    if (plan.n_kv_items > 0)
        kkv<<<static_cast<unsigned>(plan.n_kv_items), Ckv::NUM_THREADS,
              thd::DkvLayout<Ckv>::SMEM_ALLOC, stream>>>(mq, mdo, mk, mv, prm);
    return cudaGetLastError() == cudaSuccess ? THD_OK : THD_ERR_CUDA;
}

// Head dim 256: dq with 64-key tiles, then the key side in two launches (dv
// alone, dk alone) with 64-query tiles.
template <class C>
int set_smem_attr(DeviceState* ds, int vidx, const void* kern, int bytes) {
    if (ds->bwd_attr_set[vidx]) return THD_OK;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return THD_ERR_CUDA;
    ds->bwd_attr_set[vidx] = true;
    return THD_OK;
}

int launch_bwd256(DeviceState* ds, const BwdPlanEntry& plan, const CUtensorMap& mq128,
                  const CUtensorMap& mdo128, const CUtensorMap& mk128, const CUtensorMap& mv128,
                  const CUtensorMap& mq64, const CUtensorMap& mdo64, const CUtensorMap& mk64,
                  const CUtensorMap& mv64, const thd::BwdParams& prm, const void* out,
                  const void* dout, const float* sinks, float* dsinks, float* delta,
                  float* sink_part, cudaStream_t stream) {
    using Cq = thd::BwdConfig<256, 3, 64>;
    using Cdv = thd::BwdConfig<256, 3, 64, thd::kDvOnly, 2, 2>;  // three Q slots, two dO, two S^T buffers
    using Cdk = thd::BwdConfig<256, 2, 64, thd::kDkOnly, 1>;  // two Q slots, one dO slot
    auto kq = thd::thd_attn_bwd_dq_kernel<Cq>;
    auto kdv = thd::thd_attn_bwd_dkdv_kernel<Cdv>;
    auto kdk = thd::thd_attn_bwd_dkdv_kernel<Cdk>;
    int rc = set_smem_attr<Cq>(ds, 4, reinterpret_cast<const void*>(kq), thd::DqLayout<Cq>::SMEM_ALLOC);
    if (rc == THD_OK)
        rc = set_smem_attr<Cdv>(ds, 5, reinterpret_cast<const void*>(kdv), thd::DkvLayout<Cdv>::SMEM_ALLOC);
    if (rc == THD_OK)
        rc = set_smem_attr<Cdk>(ds, 6, reinterpret_cast<const void*>(kdk), thd::DkvLayout<Cdk>::SMEM_ALLOC);
    if (rc != THD_OK) return rc;
    const int64_t rows = prm.T * prm.Hq;
    thd::thd_attn_bwd_preprocess_kernel<256><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(dout), prm.lse,
        sinks, delta, sink_part, rows, prm.Hq);
    if (dsinks != nullptr) {
        if (sinks != nullptr)
            thd::thd_attn_bwd_dsink_kernel<<<prm.Hq, 256, 0, stream>>>(sink_part, prm.T, prm.Hq, dsinks);
        else if (cudaMemsetAsync(dsinks, 0, sizeof(float) * prm.Hq, stream) != cudaSuccess)
            return THD_ERR_CUDA;
    }
    if (plan.n_q_items > 0)
        kq<<<static_cast<unsigned>(plan.n_q_items), Cq::NUM_THREADS, thd::DqLayout<Cq>::SMEM_ALLOC,
             stream>>>(mq128, mdo128, mk64, mv64, prm);
    if (plan.n_kv_items > 0) {
        kdv<<<static_cast<unsigned>(plan.n_kv_items), Cdv::NUM_THREADS,
              thd::DkvLayout<Cdv>::SMEM_ALLOC, stream>>>(mq64, mdo64, mk128, mv128, prm);
        kdk<<<static_cast<unsigned>(plan.n_kv_items), Cdk::NUM_THREADS,
              thd::DkvLayout<Cdk>::SMEM_ALLOC, stream>>>(mq64, mdo64, mk128, mv128, prm);
    }
    return cudaGetLastError() == cudaSuccess ? THD_OK : THD_ERR_CUDA;
}

// Stall-detector self-test: block 0 waits on an mbarrier that nothing
// signals, with the kernels' own bounded wait, and gives up after its limit,
// recording THD_ERR_TIMEOUT in the status word; block 1 starts waiting half a
// second later and must give up as soon as it sees that status, before its
// own limit runs out.  Plain waits on the wall clock: nothing faults or hangs.
__device__ long long g_selftest_waited[2];

__global__ void __launch_bounds__(32) thd_stall_selftest_kernel(int* status) {
    __shared__ __align__(8) uint64_t bar_storage;
    __shared__ int abort_flag;
    const uint32_t bar = thd::smem_addr(&bar_storage);
    if (threadIdx.x == 0) {
        thd::mbar_init(bar, 1);
        abort_flag = 0;
        thd::fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (blockIdx.x == 1) thd::spin_ns(500000000ull);
        const uint64_t t0 = thd::global_timer_ns();
        const bool ok = thd::mbar_wait(bar, 0, &abort_flag, status, thd::kStatusTimeout);
        g_selftest_waited[blockIdx.x] = ok ? -1 : static_cast<long long>(thd::global_timer_ns() - t0);
    }
}

}  // namespace

extern "C" {

int thd_attn_abi_version(void) { return (1 << 16) | 1; }

int thd_attn_selftest_stall(int64_t* waited_ns) {
    if (waited_ns == nullptr) return THD_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState* ds = nullptr;
    int rc = device_state(&ds, nullptr);
    if (rc != THD_OK) return rc;
    int status = 0;
    if (cudaMemcpy(&status, ds->d_status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return THD_ERR_CUDA;
    if (status != 0) return status;  // an earlier error is still unread
    cudaStream_t s = nullptr;
    if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess) return THD_ERR_CUDA;
    thd_stall_selftest_kernel<<<2, 32, 0, s>>>(ds->d_status);
    long long w[2] = {0, 0};
    const bool good = cudaGetLastError() == cudaSuccess && cudaStreamSynchronize(s) == cudaSuccess &&
                      cudaMemcpyFromSymbol(w, g_selftest_waited, sizeof(w)) == cudaSuccess;
    cudaStreamDestroy(s);
    if (!good) return THD_ERR_CUDA;
    waited_ns[0] = w[0];
    waited_ns[1] = w[1];
    return THD_OK;
}

const char* thd_attn_status_string(int status) {
    switch (status) {
        case THD_OK: return "ok";
        case THD_ERR_INVALID_ARG: return "invalid argument";
        case THD_ERR_UNSUPPORTED: return "unsupported head dim or device (needs sm_100 and D in {64,128,256})";
        case THD_ERR_CUDA: return "CUDA call failed";
        case THD_ERR_TIMEOUT: return "kernel wait timed out (pipeline stalled)";
        case THD_ERR_NO_MEMORY: return "out of device memory for the schedule cache";
        case THD_ERR_TOO_LARGE: return "schedule larger than the allocation-free scratch (65,536 work items)";
        case THD_ERR_STALE_SCRATCH: return "the allocation-free scratch held another call's schedule; nothing was computed";
        case THD_ERR_BAD_ITEM: return "debug build: a work item broke the schedule's invariants; nothing was computed";
        default: return "unknown status";
    }
}

int thd_attn_plan(const int32_t* cu_seqlens, int n_docs, int Hq, int Hkv, int D, int window,
                  thd_work_item* items, int64_t capacity, int64_t* n_items) {
    if (n_docs < 0 || cu_seqlens == nullptr) return THD_ERR_INVALID_ARG;
    return thd_attn_plan_range(cu_seqlens, n_docs, 0, cu_seqlens[n_docs], Hq, Hkv, D, window,
                               items, capacity, n_items);
}

int thd_attn_plan_range(const int32_t* cu_seqlens, int n_docs, int64_t q_begin, int64_t q_end,
                        int Hq, int Hkv, int D, int window, thd_work_item* items,
                        int64_t capacity, int64_t* n_items) {
    if (n_docs < 0 || cu_seqlens == nullptr) return THD_ERR_INVALID_ARG;
    return thd_attn_plan_range_keys(cu_seqlens, n_docs, q_begin, q_end, cu_seqlens[n_docs], Hq, Hkv,
                                    D, window, items, capacity, n_items);
}

int thd_attn_plan_range_keys(const int32_t* cu_seqlens, int n_docs, int64_t q_begin,
                             int64_t q_end, int64_t k_end, int Hq, int Hkv, int D, int window,
                             thd_work_item* items, int64_t capacity, int64_t* n_items) {
    if (n_items == nullptr || capacity < 0) return THD_ERR_INVALID_ARG;
    int rc = thd::validate_args(cu_seqlens, n_docs, Hq, Hkv, D, window);
    if (rc != THD_OK) return rc;
    if (q_begin < 0 || q_end < q_begin || q_end > cu_seqlens[n_docs] || k_end < 0 ||
        k_end > cu_seqlens[n_docs])
        return THD_ERR_INVALID_ARG;
    KernelShape ks;
    if (!thd::choose_kernel_shape(D, Hq / Hkv, &ks)) return THD_ERR_UNSUPPORTED;
    std::vector<thd_work_item> v =
        thd::build_plan_range(cu_seqlens, n_docs, q_begin, q_end, Hq, Hkv, window, ks, k_end);
    *n_items = static_cast<int64_t>(v.size());
    if (items != nullptr) {
        const int64_t n = std::min<int64_t>(capacity, static_cast<int64_t>(v.size()));
        std::memcpy(items, v.data(), sizeof(thd_work_item) * static_cast<size_t>(n));
    }
    return THD_OK;
}

int thd_attn_fwd_range(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                       int n_docs, int64_t q_begin, int64_t q_end, int Hq, int Hkv, int D,
                       int window, float scale, const float* sinks_or_null, void* out, float* lse,
                       void* stream_ptr) {
    if (n_docs < 0 || cu_seqlens == nullptr) return THD_ERR_INVALID_ARG;
    return thd_attn_fwd_range_keys(q, k, v, cu_seqlens, n_docs, q_begin, q_end, cu_seqlens[n_docs],
                                   Hq, Hkv, D, window, scale, sinks_or_null, out, lse, stream_ptr);
}

int thd_attn_fwd_range_keys(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                            int n_docs, int64_t q_begin, int64_t q_end, int64_t k_end, int Hq,
                            int Hkv, int D, int window, float scale, const float* sinks_or_null,
                            void* out, float* lse, void* stream_ptr) {
    int rc = thd::validate_args(cu_seqlens, n_docs, Hq, Hkv, D, window);
    if (rc != THD_OK) return rc;
    if (!(std::isfinite(scale) && scale > 0.0f)) return THD_ERR_INVALID_ARG;
    const int64_t T = cu_seqlens[n_docs];
    if (q_begin < 0 || q_end < q_begin || q_end > T || k_end < 0 || k_end > T)
        return THD_ERR_INVALID_ARG;
    if (T == 0 || q_end == q_begin) return THD_OK;
    if (!q || !k || !v || !out) return THD_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
        return THD_ERR_INVALID_ARG;
    if ((lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) ||
        (sinks_or_null && (reinterpret_cast<uintptr_t>(sinks_or_null) & 3u)))
        return THD_ERR_INVALID_ARG;
    KernelShape ks;
    if (!thd::choose_kernel_shape(D, Hq / Hkv, &ks)) return THD_ERR_UNSUPPORTED;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);

    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState* ds = nullptr;
    rc = device_state(&ds, nullptr);
    if (rc != THD_OK) return rc;
    const PlanEntry* plan = nullptr;
    rc = get_plan(ds, cu_seqlens, n_docs, q_begin, q_end, k_end, Hq, Hkv, D, window, ks, stream,
                  &plan);
    if (rc != THD_OK) return rc;
    if (plan->n_items == 0) return THD_OK;

    CUtensorMap mq, mk, mv;
    // The pair kernel loads half of each K tile (half the keys) per CTA.
    if (!make_map(&mq, q, q_end - q_begin, Hq, D, 128) ||
        !make_map(&mk, k, T, Hkv, D, ks.pair ? ks.block_n / 2 : ks.block_n) ||
        !make_map(&mv, v, T, Hkv, D, ks.block_n))
        return THD_ERR_CUDA;

    thd::FwdParams prm;
    prm.items = plan->d_items;
    prm.out = static_cast<__nv_bfloat16*>(out);
    prm.lse = lse;
    prm.sinks = sinks_or_null;
    prm.status = ds->d_status;
    prm.Hq = Hq;
    prm.G = Hq / Hkv;
    prm.window = window;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.q_offset = static_cast<int>(q_begin);

    switch (variant_index(ks)) {
        case 0: return launch<Cfg64x2>(ds, 0, *plan, mq, mk, mv, prm, stream);
        case 1: return launch<Cfg64x1>(ds, 1, *plan, mq, mk, mv, prm, stream);
        case 2: return launch<Cfg128x2>(ds, 2, *plan, mq, mk, mv, prm, stream);
        case 3: return launch<Cfg128x1>(ds, 3, *plan, mq, mk, mv, prm, stream);
        case 4: return launch<Cfg256x1>(ds, 4, *plan, mq, mk, mv, prm, stream);
        default: return launch_pair<SplitCfg256>(ds, 5, *plan, mq, mk, mv, prm, stream);
    }
}

int thd_attn_fwd(const void* q, const void* k, const void* v, const int32_t* cu_seqlens,
                 int n_docs, int Hq, int Hkv, int D, int window, float scale,
                 const float* sinks_or_null, void* out, float* lse, void* stream_ptr) {
    if (n_docs < 0 || cu_seqlens == nullptr) return THD_ERR_INVALID_ARG;
    return thd_attn_fwd_range(q, k, v, cu_seqlens, n_docs, 0, cu_seqlens[n_docs], Hq, Hkv, D,
                              window, scale, sinks_or_null, out, lse, stream_ptr);
}

size_t thd_attn_bwd_workspace_bytes(int64_t total_tokens, int Hq) {
    if (total_tokens <= 0 || Hq <= 0) return 0;
    return 2 * align256(static_cast<size_t>(total_tokens) * static_cast<size_t>(Hq) * sizeof(float));
}

int thd_attn_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse,
                 const void* dout, const int32_t* cu_seqlens, int n_docs, int Hq, int Hkv, int D,
                 int window, float scale, const float* sinks_or_null, void* dq, void* dk, void* dv,
                 float* dsinks_or_null, void* workspace, size_t workspace_bytes, void* stream_ptr) {
    int rc = thd::validate_args(cu_seqlens, n_docs, Hq, Hkv, D, window);
    if (rc != THD_OK) return rc;
    if (!(std::isfinite(scale) && scale > 0.0f)) return THD_ERR_INVALID_ARG;
    const int64_t T = cu_seqlens[n_docs];
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
    if ((dsinks_or_null && (reinterpret_cast<uintptr_t>(dsinks_or_null) & 3u)) ||
        (sinks_or_null && (reinterpret_cast<uintptr_t>(sinks_or_null) & 3u)))
        return THD_ERR_INVALID_ARG;
    if (T == 0) {
        if (dsinks_or_null &&
            cudaMemsetAsync(dsinks_or_null, 0, sizeof(float) * Hq, stream) != cudaSuccess)
            return THD_ERR_CUDA;
        return THD_OK;
    }
    if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv || !workspace)
        return THD_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(workspace) ||
        (reinterpret_cast<uintptr_t>(lse) & 3u))
        return THD_ERR_INVALID_ARG;
    if (workspace_bytes < thd_attn_bwd_workspace_bytes(T, Hq)) return THD_ERR_INVALID_ARG;

    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState* ds = nullptr;
    rc = device_state(&ds, nullptr);
    if (rc != THD_OK) return rc;
    const BwdPlanEntry* plan = nullptr;
    rc = get_bwd_plan(ds, cu_seqlens, n_docs, Hq, Hkv, D, window, stream, &plan);
    if (rc != THD_OK) return rc;

    CUtensorMap mq, mdo, mk, mv;
    if (!make_map(&mq, q, T, Hq, D, 128) || !make_map(&mdo, dout, T, Hq, D, 128) ||
        !make_map(&mk, k, T, Hkv, D, 128) || !make_map(&mv, v, T, Hkv, D, 128))
        return THD_ERR_CUDA;
    CUtensorMap mq64, mdo64, mk64, mv64;  // head dim 256: tiles of 64 rows
    if (D == 256 && (!make_map(&mq64, q, T, Hq, D, 64) || !make_map(&mdo64, dout, T, Hq, D, 64) ||
                     !make_map(&mk64, k, T, Hkv, D, 64) || !make_map(&mv64, v, T, Hkv, D, 64)))
        return THD_ERR_CUDA;
    float* delta = static_cast<float*>(workspace);
    float* sink_part = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                                align256(static_cast<size_t>(T) * Hq * sizeof(float)));
    thd::BwdParams prm;
    prm.q_items = plan->d_q_items;
    prm.kv_items = plan->d_kv_items;
    prm.lse = lse;
    prm.delta = delta;
    prm.dq = static_cast<__nv_bfloat16*>(dq);
    prm.dk = static_cast<__nv_bfloat16*>(dk);
    prm.dv = static_cast<__nv_bfloat16*>(dv);
    prm.status = ds->d_status;
    prm.T = T;
    prm.Hq = Hq;
    prm.Hkv = Hkv;
    prm.G = Hq / Hkv;
    prm.window = window;
    prm.scale = scale;
    prm.scale_log2 = scale * 1.4426950408889634f;
    if (D == 64)
        return launch_bwd<64>(ds, *plan, mq, mdo, mk, mv, prm, out, dout, sinks_or_null,
                              dsinks_or_null, delta, sink_part, stream);
    if (D == 128)
        return launch_bwd<128>(ds, *plan, mq, mdo, mk, mv, prm, out, dout, sinks_or_null,
                               dsinks_or_null, delta, sink_part, stream);
    return launch_bwd256(ds, *plan, mq, mdo, mk, mv, mq64, mdo64, mk64, mv64, prm, out, dout,
                         sinks_or_null, dsinks_or_null, delta, sink_part, stream);
}

int thd_attn_get_error(void* stream_ptr) {
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
    if (cudaStreamSynchronize(stream) != cudaSuccess) return THD_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState* ds = nullptr;
    int rc = device_state(&ds, nullptr);
    if (rc != THD_OK) return rc;
    int status = 0;
    if (cudaMemcpy(&status, ds->d_status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return THD_ERR_CUDA;
    if (status != 0 && cudaMemset(ds->d_status, 0, sizeof(int)) != cudaSuccess) return THD_ERR_CUDA;
    return status;
}

}  // extern "C"
