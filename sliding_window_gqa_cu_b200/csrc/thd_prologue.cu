// Q/K prologue of the attention ("muse_glimmer.model" page): the
// parameter-free RMSNorm of every query and key head vector
// (MuseGlimmerScalelessRMSNorm: y = x / sqrt(mean(x^2) + eps)), then the
// split-half rotary embedding (MuseGlimmerRotaryEmbedding / apply_rotary_emb:
// element k pairs with k + D/2 and turns by position * theta^(-2k/D)), in
// place on the packed THD q [T, Hq, D] and k [T, Hkv, D].  Positions are the
// caller's, or each token's offset inside its own document.
//
// One warp per token: a lane holds D/32 consecutive elements of a head
// vector (so the split-half partner of lane l is lane l ^ 16) and computes
// the cos / sin of its own D/32 frequencies once, for all Hq + Hkv head
// vectors of the token; the warp loads four head vectors before it
// transforms any of them, to keep enough loads in flight.  Memory bound: each element is read and written
// once (16-bit loads and stores vectorised to 4, 8 or 16 bytes per lane).
// The angle is reduced modulo 2 pi in double precision before the fp32
// sine / cosine, so positions up to 2^31 keep full fp32 accuracy; everything
// else is fp32 and the result is rounded to bf16 once.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "../../include/thd_attn.h"
#include "tma_map.h"

namespace {

constexpr int kMaxHalf = 128;  // D / 2 for D = 256

struct PrologueParams {
    __nv_bfloat16* q;
    __nv_bfloat16* k;
    const int32_t* cu;         // device copy of cu_seqlens [n_docs + 1]
    const int32_t* positions;  // [T] or null
    int64_t T;
    int n_docs, Hq, Hkv, rope;
    float eps;
    double inv_freq[kMaxHalf];  // theta^(-2k/D), k < D/2
};

template <int D>
__global__ void __launch_bounds__(256) thd_qk_norm_rope_kernel(const PrologueParams p) {
    constexpr int E = D / 32;  // elements per lane
    constexpr int R = 4;       // head vectors loaded per warp before any is transformed
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + warp;
    if (t >= p.T) return;
    // cos / sin of this lane's E frequencies k = E (lane % 16) + e, shared by
    // all head vectors of the token (lane l and l ^ 16 hold a split-half pair).
    float cs[E], sn[E];
    if (p.rope) {
        int pos;
        if (p.positions != nullptr) {
            pos = p.positions[t];
        } else {  // last document starting at or before t
            int lo = 0, hi = p.n_docs - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (p.cu[mid] <= t) lo = mid; else hi = mid - 1;
            }
            pos = static_cast<int>(t - p.cu[lo]);
        }
        const int k0 = E * (lane & 15);
#pragma unroll
        for (int e = 0; e < E; ++e) {
            constexpr double kTwoPi = 6.283185307179586476925286766559;
            double a = static_cast<double>(pos) * p.inv_freq[k0 + e];
            a -= kTwoPi * rint(a * (1.0 / kTwoPi));
            sincosf(static_cast<float>(a), &sn[e], &cs[e]);
        }
    }
    const bool second = lane >= 16;
    const int rows = p.Hq + p.Hkv;
    for (int r0 = 0; r0 < rows; r0 += R) {
        uint32_t w[R][E / 2];
        __nv_bfloat16* mine[R];
#pragma unroll
        for (int i = 0; i < R; ++i) {
            const int r = r0 + i;
            mine[i] = nullptr;
            if (r < rows) {
                __nv_bfloat16* row = r < p.Hq ? p.q + (t * p.Hq + r) * D
                                              : p.k + (t * p.Hkv + (r - p.Hq)) * D;
                mine[i] = row + lane * E;
                if constexpr (E == 8) {
                    const uint4 x = *reinterpret_cast<const uint4*>(mine[i]);
                    w[i][0] = x.x; w[i][1] = x.y; w[i][2] = x.z; w[i][3] = x.w;
                } else if constexpr (E == 4) {
                    const uint2 x = *reinterpret_cast<const uint2*>(mine[i]);
                    w[i][0] = x.x; w[i][1] = x.y;
                } else {
                    w[i][0] = *reinterpret_cast<const uint32_t*>(mine[i]);
                }
            }
        }
#pragma unroll
        for (int i = 0; i < R; ++i) {
            if (r0 + i >= rows) break;  // warp-uniform
            float v[E];
#pragma unroll
            for (int u = 0; u < E / 2; ++u) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i][u]));
                v[2 * u] = f.x;
                v[2 * u + 1] = f.y;
            }
            float ss = 0.0f;
#pragma unroll
            for (int e = 0; e < E; ++e) ss = fmaf(v[e], v[e], ss);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
            const float inv = 1.0f / sqrtf(ss * (1.0f / D) + p.eps);
#pragma unroll
            for (int e = 0; e < E; ++e) v[e] *= inv;
            if (p.rope) {
                float o[E];
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const float partner = __shfl_xor_sync(0xffffffffu, v[e], 16);
                    o[e] = second ? fmaf(v[e], cs[e], partner * sn[e])
                                  : fmaf(v[e], cs[e], -partner * sn[e]);
                }
#pragma unroll
                for (int e = 0; e < E; ++e) v[e] = o[e];
            }
            uint32_t ow[E / 2];
#pragma unroll
            for (int u = 0; u < E / 2; ++u) {
                const __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * u], v[2 * u + 1]);
                ow[u] = *reinterpret_cast<const uint32_t*>(&b);
            }
            if constexpr (E == 8) {
                *reinterpret_cast<uint4*>(mine[i]) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
            } else if constexpr (E == 4) {
                *reinterpret_cast<uint2*>(mine[i]) = make_uint2(ow[0], ow[1]);
            } else {
                *reinterpret_cast<uint32_t*>(mine[i]) = ow[0];
            }
        }
    }
}

// Per device: a cached device copy of the last cu_seqlens.
struct CuCache {
    std::vector<int32_t> host;
    int32_t* dev = nullptr;
    size_t cap = 0;
};
std::mutex g_mu;
std::unordered_map<int, CuCache> g_cu;

int device_cu(const int32_t* cu, int n_docs, cudaStream_t stream, const int32_t** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return THD_ERR_CUDA;
    CuCache& c = g_cu[dev];
    const size_t n = static_cast<size_t>(n_docs) + 1;
    if (c.host.size() == n && std::memcmp(c.host.data(), cu, n * sizeof(int32_t)) == 0) {
        *out = c.dev;
        return THD_OK;
    }
    if (c.cap < n) {
        // cudaFree waits for kernels that may still read the old copy.
        if (c.dev) cudaFree(c.dev);
        c.dev = nullptr;
        c.cap = 0;
        c.host.clear();
        if (cudaMalloc(&c.dev, n * sizeof(int32_t)) != cudaSuccess) return THD_ERR_NO_MEMORY;
        c.cap = n;
    }
    // Synchronous with respect to the stream: earlier kernels may read the
    // previous contents.
    if (cudaStreamSynchronize(stream) != cudaSuccess ||
        cudaMemcpy(c.dev, cu, n * sizeof(int32_t), cudaMemcpyHostToDevice) != cudaSuccess) {
        c.host.clear();
        return THD_ERR_CUDA;
    }
    c.host.assign(cu, cu + n);
    *out = c.dev;
    return THD_OK;
}

}  // namespace

extern "C" int thd_qk_norm_rope(void* q, void* k, const int32_t* cu_seqlens, int n_docs,
                                const int32_t* positions_or_null, int Hq, int Hkv, int D,
                                float eps, float theta, int apply_rope, void* stream_ptr) {
    if (n_docs < 0 || cu_seqlens == nullptr || Hq <= 0 || Hkv < 0) return THD_ERR_INVALID_ARG;
    if (cu_seqlens[0] != 0) return THD_ERR_INVALID_ARG;
    for (int d = 0; d < n_docs; ++d)
        if (cu_seqlens[d + 1] < cu_seqlens[d]) return THD_ERR_INVALID_ARG;
    if (D != 64 && D != 128 && D != 256) return THD_ERR_UNSUPPORTED;
    if (!(std::isfinite(eps) && eps > 0.0f)) return THD_ERR_INVALID_ARG;
    if (apply_rope && !(std::isfinite(theta) && theta > 1.0f)) return THD_ERR_INVALID_ARG;
    const int64_t T = cu_seqlens[n_docs];
    if (T == 0) return THD_OK;
    if (T > 0x7fffffff) return THD_ERR_INVALID_ARG;
    if (!q || (Hkv > 0 && !k)) return THD_ERR_INVALID_ARG;
    if (!thd::aligned16(q) || (Hkv > 0 && !thd::aligned16(k)) ||
        (positions_or_null && (reinterpret_cast<uintptr_t>(positions_or_null) & 3u)))
        return THD_ERR_INVALID_ARG;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);

    PrologueParams p{};
    p.q = static_cast<__nv_bfloat16*>(q);
    p.k = static_cast<__nv_bfloat16*>(k);
    p.positions = positions_or_null;
    p.T = T;
    p.n_docs = n_docs;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.rope = apply_rope ? 1 : 0;
    p.eps = eps;
    for (int kk = 0; kk < D / 2; ++kk)
        p.inv_freq[kk] = std::pow(static_cast<double>(theta), -2.0 * kk / D);
    if (p.rope && positions_or_null == nullptr) {
        std::lock_guard<std::mutex> lock(g_mu);
        int rc = device_cu(cu_seqlens, n_docs, stream, &p.cu);
        if (rc != THD_OK) return rc;
    }
    const unsigned grid = static_cast<unsigned>((T + 7) / 8);  // 8 warps (tokens) per CTA
    switch (D) {
        case 64: thd_qk_norm_rope_kernel<64><<<grid, 256, 0, stream>>>(p); break;
        case 128: thd_qk_norm_rope_kernel<128><<<grid, 256, 0, stream>>>(p); break;
        default: thd_qk_norm_rope_kernel<256><<<grid, 256, 0, stream>>>(p); break;
    }
    return cudaGetLastError() == cudaSuccess ? THD_OK : THD_ERR_CUDA;
}
