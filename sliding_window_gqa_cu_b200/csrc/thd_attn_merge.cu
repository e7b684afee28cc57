// Merge of two partial attentions of the same query rows over disjoint key
// sets (thd_attn_merge).
//
// A context-parallel row ("muse_spark.magi_cp" page, MuseMagiPlan.attention:
// the local THD output with the keys exchanged between ranks) splits into the
// keys on its own rank and the keys on earlier ranks.  Each part is a
// softmax over its own keys, normalised by its own sum, with its log-sum-exp
// (natural log) beside it.  With m = max(lse_a, lse_b),
//   w_a = exp(lse_a - m),  w_b = exp(lse_b - m),
//   lse = m + log(w_a + w_b),  out = (w_a out_a + w_b out_b) / (w_a + w_b),
// which is the softmax over the union of the two key sets: the same identity
// the online softmax uses between key tiles, applied once to whole parts.  A
// part without keys has lse = -inf and weight 0; a row where both are -inf
// gets out = 0 and lse = -inf.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "../../include/thd_attn.h"

namespace {

// One thread per (row, head, 8 columns); the D / 8 threads of a (row, head)
// sit in one warp (D / 8 divides 32), so out and lse may alias out_a and
// lse_a: every thread of the warp reads both LSEs before any writes one.
__global__ void __launch_bounds__(256) thd_attn_merge_kernel(
    const __nv_bfloat16* out_a, const float* lse_a, const __nv_bfloat16* out_b, const float* lse_b,
    int64_t n_rh, int D, __nv_bfloat16* out, float* lse) {
    const int per = D / 8;
    const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const bool active = gid < n_rh * per;
    const int64_t rh = active ? gid / per : 0;
    const int c8 = active ? static_cast<int>(gid % per) : 0;
    float la = -INFINITY, lb = -INFINITY;
    uint4 xa = make_uint4(0u, 0u, 0u, 0u), xb = xa;
    if (active) {
        la = lse_a[rh];
        lb = lse_b[rh];
        xa = reinterpret_cast<const uint4*>(out_a + rh * D)[c8];
        xb = reinterpret_cast<const uint4*>(out_b + rh * D)[c8];
    }
    __syncwarp();
    if (!active) return;
    const float m = fmaxf(la, lb);
    float wa = 0.0f, wb = 0.0f, l = -INFINITY;
    if (m != -INFINITY) {
        wa = expf(la - m);
        wb = expf(lb - m);
        const float s = wa + wb;
        l = m + logf(s);
        wa /= s;
        wb /= s;
    }
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&xa);
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&xb);
    uint4 y;
    __nv_bfloat162* y2 = reinterpret_cast<__nv_bfloat162*>(&y);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const float2 fa = __bfloat1622float2(a2[u]);
        const float2 fb = __bfloat1622float2(b2[u]);
        y2[u] = __floats2bfloat162_rn(wa * fa.x + wb * fb.x, wa * fa.y + wb * fb.y);
    }
    reinterpret_cast<uint4*>(out + rh * D)[c8] = y;
    if (c8 == 0) lse[rh] = l;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" int thd_attn_merge(const void* out_a, const float* lse_a, const void* out_b,
                              const float* lse_b, int64_t rows, int Hq, int D, void* out,
                              float* lse, void* stream_ptr) {
    if (rows < 0 || Hq <= 0) return THD_ERR_INVALID_ARG;
    if (D != 64 && D != 128 && D != 256) return THD_ERR_UNSUPPORTED;
    if (rows == 0) return THD_OK;
    if (!out_a || !lse_a || !out_b || !lse_b || !out || !lse) return THD_ERR_INVALID_ARG;
    if (!aligned(out_a, 16) || !aligned(out_b, 16) || !aligned(out, 16) || !aligned(lse_a, 4) ||
        !aligned(lse_b, 4) || !aligned(lse, 4))
        return THD_ERR_INVALID_ARG;
    const int64_t n_rh = rows * Hq;
    const int64_t threads = n_rh * (D / 8);
    const int64_t blocks = (threads + 255) / 256;
    if (blocks > 0x7fffffffll) return THD_ERR_INVALID_ARG;
    thd_attn_merge_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream_ptr)>>>(
        static_cast<const __nv_bfloat16*>(out_a), lse_a, static_cast<const __nv_bfloat16*>(out_b), lse_b, n_rh,
        D, static_cast<__nv_bfloat16*>(out), lse);
    return cudaGetLastError() == cudaSuccess ? THD_OK : THD_ERR_CUDA;
}
