// thd_attn_fwd_noalloc: the same forward as thd_attn_fwd, for callers that
// must not allocate device memory.
//
// Who needs it: runtimes that reserve all device memory up front and hand
// out only pre-planned buffers (a cudaMalloc from inside the library would
// fail or fragment their pool), and latency-critical loops that cannot afford
// the device-wide synchronisation cudaMalloc/cudaFree may cause.  Such callers
// pass their inputs and outputs; the little scratch the kernel needs (the
// tile schedule and a status word) lives in a fixed-size array that is part
// of this library's device image, so no call allocates anything.
//
// Scratch: one file-scope static __device__ array per GPU that loads the
// library, held until the process exits.  Layout: bytes [0, 4) hold the
// status word, bytes [128, 136) the tag of the schedule in place, then from
// byte 256 up to kMaxItems work items of 32 bytes (2 MiB + 256 B in total).
// Every call shares it and it keeps the last call's contents: the schedule
// (with a new tag) is re-uploaded only when the arguments change, and every
// launch checks that the tag it was enqueued with is still in place, so a
// launch that would read another call's schedule records an error and does
// nothing instead.  The status word is kept until
// thd_attn_noalloc_get_error reads and clears it (while it is non-zero,
// launches skip their work), unless the caller supplies its own status word.
// Calls that overlap on the GPU (e.g. on two streams of one device) race on
// this array.
//
// Host side: the schedule is built into a static host array and sorted in
// place; no heap memory is taken either.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstddef>
#include <cstring>
#include <mutex>

#include "../../include/thd_attn.h"
#include "scheduler.h"
#include "tma_map.h"
#include "thd_attn_kernel.cuh"
#include "thd_attn_split_kernel.cuh"

namespace {

constexpr int64_t kMaxItems = 65536;
constexpr size_t kHeaderBytes = 256;
constexpr size_t kTagOffset = 128;  // the schedule's tag, uploaded with the items
constexpr size_t kScratchBytes = kHeaderBytes + kMaxItems * sizeof(thd::WorkItem);
constexpr int kMaxDevices = 64;
constexpr int kMaxCachedDocs = 4096;  // boundaries remembered to skip re-uploads

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

struct NoAllocDevice {
    bool ready = false;
    unsigned char* scratch = nullptr;  // device address of g_noalloc_scratch
    bool attr_set[6] = {};
    // arguments of the schedule now in the scratch (valid when have_plan)
    bool have_plan = false;
    int n_docs = 0, Hq = 0, Hkv = 0, D = 0, window = 0;
    int32_t cu[kMaxCachedDocs + 1];
    int64_t n_items = 0;
    unsigned long long tag = 0;       // tag of the schedule now in the scratch
    unsigned long long next_tag = 1;  // every upload gets a new one
};

// Host image of the scratch from byte kTagOffset on: the tag, padding to
// byte kHeaderBytes, then the work items; one copy uploads tag and items.
struct HostUpload {
    unsigned long long tag;
    unsigned char pad[kHeaderBytes - kTagOffset - sizeof(unsigned long long)];
    thd_work_item items[kMaxItems];
};
static_assert(offsetof(HostUpload, items) == kHeaderBytes - kTagOffset, "upload layout");

std::mutex g_mu;
NoAllocDevice g_dev[kMaxDevices];
HostUpload g_upload;
thd_work_item* const g_host_items = g_upload.items;

using NCfg64x2 = thd::FwdConfig<64, 2, 1, 128, 8>;
using NCfg64x1 = thd::FwdConfig<64, 1, 2, 128, 8>;
using NCfg128x2 = thd::FwdConfig<128, 2, 1, 128, 5>;
using NCfg128x1 = thd::FwdConfig<128, 1, 2, 128, 6>;
using NCfg256x1 = thd::FwdConfig<256, 1, 2, 64, 5>;
using NSplitCfg256 = thd::SplitConfig<256, 2, 4>;  // 2 heads per item over a CTA pair

using thd::aligned16;
using thd::make_map;

// Number of work items the schedule of these arguments has (no allocation).
int64_t count_items(const int32_t* cu, int n_docs, int Hq, const thd::KernelShape& ks) {
    int64_t tiles = 0;
    for (int d = 0; d < n_docs; ++d) tiles += (cu[d + 1] - cu[d] + 127) / 128;
    return tiles * (Hq / ks.nq);
}

// Writes the schedule into g_host_items (same items and order as the cached
// path's plan: chunk of kv groups, then longest first; the sort key below is unique
// and reproduces the generation order among items of equal length).
void write_plan(const int32_t* cu, int n_docs, int Hq, int Hkv, int window,
                const thd::KernelShape& ks, int64_t n) {
    const int G = Hq / Hkv, BN = ks.block_n;
    int64_t k = 0;
    for (int d = 0; d < n_docs; ++d) {
        const int s = cu[d], e = cu[d + 1];
        for (int q1 = e; q1 > s; q1 -= 128) {
            const int q0 = q1 - 128;
            const int r_lo = q0 > s ? q0 : s;
            int k_lo = s;
            if (window > 0 && r_lo - window + 1 > k_lo) k_lo = r_lo - window + 1;
            const int n_kv = (q1 - k_lo + BN - 1) / BN;
            for (int g = 0; g < Hkv; ++g)
                for (int hp = 0; hp < G / ks.nq; ++hp)
                    g_host_items[k++] = thd_work_item{q0, q1, s, g * G + hp * ks.nq,
                                                      q1 - n_kv * BN, n_kv, ks.nq, BN};
        }
    }
    const int c = thd::kv_groups_per_chunk(cu[n_docs], ks.D, Hkv);
    std::sort(g_host_items, g_host_items + n, [G, c](const thd_work_item& a, const thd_work_item& b) {
        if (a.head0 / G / c != b.head0 / G / c) return a.head0 / G / c < b.head0 / G / c;
        if (a.n_kv != b.n_kv) return a.n_kv > b.n_kv;
        if (a.doc_start != b.doc_start) return a.doc_start < b.doc_start;
        if (a.q1 != b.q1) return a.q1 > b.q1;
        return a.head0 < b.head0;
    });
}

// Once per device, with that device current: find the device address of the
// scratch array (the array's name is only a host-side stand-in) and zero its
// status word.
int setup_device(int dev, NoAllocDevice* st) {
    if (st->ready) return THD_OK;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return THD_ERR_CUDA;
    if (major != 10 || minor != 0) return THD_ERR_UNSUPPORTED;
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
        return THD_ERR_CUDA;
    if (cudaMemset(ptr, 0, kHeaderBytes) != cudaSuccess) return THD_ERR_CUDA;
    st->scratch = static_cast<unsigned char*>(ptr);
    st->ready = true;
    return THD_OK;
}

template <class C>
int launch(NoAllocDevice* st, int vidx, int64_t n_items, const CUtensorMap& mq,
           const CUtensorMap& mk, const CUtensorMap& mv, const thd::FwdParams& prm,
           cudaStream_t stream) {
    auto kern = thd::thd_attn_fwd_kernel<C>;
    if (!st->attr_set[vidx]) {
        if (!thd::launch_registers_ok<C>()) return THD_ERR_UNSUPPORTED;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::SMEM_ALLOC) != cudaSuccess)
            return THD_ERR_CUDA;
        st->attr_set[vidx] = true;
    }
    kern<<<static_cast<unsigned>(n_items), C::NUM_THREADS, C::SMEM_ALLOC, stream>>>(mq, mk, mv,
                                                                                  prm);
    return cudaGetLastError() == cudaSuccess ? THD_OK : THD_ERR_CUDA;
}

template <class C>
int launch_pair(NoAllocDevice* st, int vidx, int64_t n_items, const CUtensorMap& mq,
                const CUtensorMap& mk, const CUtensorMap& mv, const thd::FwdParams& prm,
                cudaStream_t stream) {
    auto kern = thd::thd_attn_fwd_split_kernel<C>;
    if (!st->attr_set[vidx]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::SMEM_ALLOC) != cudaSuccess)
            return THD_ERR_CUDA;
        st->attr_set[vidx] = true;
    }
    kern<<<static_cast<unsigned>(2 * n_items), C::NUM_THREADS, C::SMEM_ALLOC, stream>>>(mq, mk, mv,
                                                                                      prm);
    return cudaGetLastError() == cudaSuccess ? THD_OK : THD_ERR_CUDA;
}

}  // namespace

extern "C" int thd_attn_fwd_noalloc(const void* q, const void* k, const void* v,
                                    const int32_t* cu_seqlens, int n_docs, int Hq, int Hkv, int D,
                                    int window, float scale, const float* sinks_or_null, void* out,
                                    float* lse, int* device_status_or_null, void* stream_ptr) {
    int rc = thd::validate_args(cu_seqlens, n_docs, Hq, Hkv, D, window);
    if (rc != THD_OK) return rc;
    if (!(std::isfinite(scale) && scale > 0.0f)) return THD_ERR_INVALID_ARG;
    const int64_t T = cu_seqlens[n_docs];
    if (T == 0) return THD_OK;
    if (!q || !k || !v || !out) return THD_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
        return THD_ERR_INVALID_ARG;
    if ((lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) ||
        (sinks_or_null && (reinterpret_cast<uintptr_t>(sinks_or_null) & 3u)) ||
        (device_status_or_null && (reinterpret_cast<uintptr_t>(device_status_or_null) & 3u)))
        return THD_ERR_INVALID_ARG;
    thd::KernelShape ks;
    if (!thd::choose_kernel_shape(D, Hq / Hkv, &ks)) return THD_ERR_UNSUPPORTED;
    const int64_t n_items = count_items(cu_seqlens, n_docs, Hq, ks);
    if (n_items > kMaxItems) return THD_ERR_TOO_LARGE;
    if (n_items == 0) return THD_OK;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);

    std::lock_guard<std::mutex> lock(g_mu);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return THD_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return THD_ERR_UNSUPPORTED;
    NoAllocDevice* st = &g_dev[dev];
    rc = setup_device(dev, st);
    if (rc != THD_OK) return rc;

    thd::WorkItem* d_items = reinterpret_cast<thd::WorkItem*>(st->scratch + kHeaderBytes);
    const bool same_plan = st->have_plan && st->n_docs == n_docs && st->Hq == Hq &&
                           st->Hkv == Hkv && st->D == D && st->window == window &&
                           n_docs <= kMaxCachedDocs &&
                           std::memcmp(st->cu, cu_seqlens, sizeof(int32_t) * (n_docs + 1)) == 0;
    if (!same_plan) {
        write_plan(cu_seqlens, n_docs, Hq, Hkv, window, ks, n_items);
        st->have_plan = false;
        g_upload.tag = st->next_tag++;
        // Pageable source: the call returns once the host array is staged,
        // so the next call may overwrite it.
        if (cudaMemcpyAsync(st->scratch + kTagOffset, &g_upload,
                            (kHeaderBytes - kTagOffset) + sizeof(thd::WorkItem) * n_items,
                            cudaMemcpyHostToDevice, stream) != cudaSuccess)
            return THD_ERR_CUDA;
        st->tag = g_upload.tag;
        if (n_docs <= kMaxCachedDocs) {
            st->n_docs = n_docs;
            st->Hq = Hq;
            st->Hkv = Hkv;
            st->D = D;
            st->window = window;
            std::memcpy(st->cu, cu_seqlens, sizeof(int32_t) * (n_docs + 1));
            st->n_items = n_items;
            st->have_plan = true;
        }
    }

    // The scratch's own status word is not cleared here: an error stays
    // recorded (and later launches skip their work) until
    // thd_attn_noalloc_get_error reads it.
    int* status = device_status_or_null != nullptr ? device_status_or_null
                                                   : reinterpret_cast<int*>(st->scratch);

    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, q, T, Hq, D, 128) ||
        !make_map(&mk, k, T, Hkv, D, ks.pair ? ks.block_n / 2 : ks.block_n) ||
        !make_map(&mv, v, T, Hkv, D, ks.block_n))
        return THD_ERR_CUDA;

    thd::FwdParams prm;
    prm.items = d_items;
    prm.out = static_cast<__nv_bfloat16*>(out);
    prm.lse = lse;
    prm.sinks = sinks_or_null;
    prm.status = status;
    prm.Hq = Hq;
    prm.G = Hq / Hkv;
    prm.window = window;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.q_offset = 0;
    prm.plan_tag = reinterpret_cast<const unsigned long long*>(st->scratch + kTagOffset);
    prm.expected_tag = st->tag;

    if (ks.pair) return launch_pair<NSplitCfg256>(st, 5, n_items, mq, mk, mv, prm, stream);
    if (D == 64) {
        return ks.nq == 2 ? launch<NCfg64x2>(st, 0, n_items, mq, mk, mv, prm, stream)
                          : launch<NCfg64x1>(st, 1, n_items, mq, mk, mv, prm, stream);
    }
    if (D == 128) {
        return ks.nq == 2 ? launch<NCfg128x2>(st, 2, n_items, mq, mk, mv, prm, stream)
                          : launch<NCfg128x1>(st, 3, n_items, mq, mk, mv, prm, stream);
    }
    return launch<NCfg256x1>(st, 4, n_items, mq, mk, mv, prm, stream);
}

extern "C" int thd_attn_noalloc_get_error(void* stream_ptr) {
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
    if (cudaStreamSynchronize(stream) != cudaSuccess) return THD_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return THD_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return THD_ERR_UNSUPPORTED;
    NoAllocDevice* st = &g_dev[dev];
    if (!st->ready) return THD_OK;  // no launch on this device yet
    int status = 0;
    if (cudaMemcpy(&status, st->scratch, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return THD_ERR_CUDA;
    if (status != 0 && cudaMemset(st->scratch, 0, sizeof(int)) != cudaSuccess) return THD_ERR_CUDA;
    return status;
}
