// Sparse MLA forward ("mistral_large4.attention" page, sparse_mla) on B200.
//
// For token t and head h: s_j = scale * <q[t, h, :576], kv[idx[t, j], :576]>
// over the valid index slots j (idx >= 0), p = softmax(s), latent =
// sum_j p_j kv[idx[t, j], :512], out[t, h, :] = value_weight[h] @ latent.
// A row without a valid slot is zero.  Three kernels:
//
// 0. Compaction (thd_sparse_mla_compact_kernel): one warp per token moves the
//    token's valid slots to the front of a copy of its index row (the order
//    of slots does not change the softmax) and records their count, so that
//    the attention processes ceil(count / 64) slot chunks, not K / 64.
//
// 1. Attention (thd_sparse_mla_attn_kernel): one CTA per (token, group of
//    128 heads, half of the 512 latent columns).  The token's 128 query rows
//    (128 x 576 bf16) are the A operand of S = Q kv^T: columns 0-255 in TMEM
//    (loaded by TMA into the second gather stage, which is still free, and
//    moved into TMEM by the softmax warps), columns 256-575 in shared memory
//    (128-byte swizzled).  The selected kv
//    rows are gathered 64 at a time by eight gather warps, four per stage
//    (16-byte cp.async copies, one kv row per warp instruction, into the
//    128-byte-swizzled layout the tensor core reads; two stages, each
//    refilled in two parts -- the columns PV does not read once S of the
//    stage's previous chunk is done, this CTA's latent half once its PV is
//    -- and published as soon as its copies land), so one shared-memory
//    tile serves S (K-major operand) and latent += P kv[:, half] (MN-major
//    operand, N = 256).
//    TMEM: Q 128 columns + two S / P buffers of 64 + the latent half 256 =
//    512, so S of the next chunk is computed while the softmax works on this
//    one; the two CTAs of a token each compute S (QK^T runs twice per
//    token).  Online softmax as in the attention forward (exp2 domain, lazy
//    rescale).  Writes the normalised latent (bf16) to a workspace
//    [T, H, 512].
// 2. Projection (thd_sparse_mla_proj_kernel): per head a GEMM
//    out[:, h, :] = latent[:, h, :] @ value_weight[h]^T, one CTA per
//    (128-token tile, head), TMA-fed tcgen05 MMAs with K = 512.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>

#include "../../include/thd_attn.h"
#include "sm100_ptx.cuh"
#include "thd_attn_kernel.cuh"
#include "tma_map.h"

namespace {

using thd::kStatusTimeout;

// --------------------------------------------------------- cp.async gather --

// One 16-byte global-to-shared copy.  No compiler memory barrier, so that
// the loads that compute the next copies' addresses may move ahead of it
// (the copied data is read only after cp_async_wait, which keeps one).
__device__ __forceinline__ void cp_async16_nc(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src));
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ld_shared_v4(uint32_t addr, uint32_t& a, uint32_t& b, uint32_t& c,
                                             uint32_t& d) {
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(a), "=r"(b), "=r"(c), "=r"(d) : "r"(addr)
                 : "memory");
}

struct SmlaParams {
    const __nv_bfloat16* q;    // [T, H, 576]
    const __nv_bfloat16* kv;   // [Tg, 576]
    const int32_t* idx;        // [T, K] valid slots first (compacted)
    const int32_t* count;      // [T] valid slots per token
    __nv_bfloat16* latent;     // [T, H, 512] (workspace)
    int* status;
    int64_t T, Tg;
    int H, K;
    float scale_log2;
};

constexpr int kQDim = 576, kLat = 512;
constexpr int kHalf = kLat / 2;                  // latent columns per CTA
constexpr int kBN = 64;                          // selected keys per chunk
constexpr int kNST = 2;                          // chunk stages
constexpr int kChunkBytes = kBN * 128;           // one 64-column chunk of a 64-row tile
constexpr int kStageBytes = 9 * kChunkBytes;     // 64 rows x 576 columns
constexpr int kQT = 256;                         // query columns held in TMEM
constexpr int kQSChunks = (kQDim - kQT) / 64;    // query chunks of 64 columns in shared memory
constexpr int kQSChunkBytes = 128 * 128;         // 128 rows x 64 columns
// TMEM columns: Q[:, :256] (bf16 pairs) 128, two S / P buffers of 64, the
// latent half 256: all 512.
constexpr int kTmQ = 0, kTmS = kQT / 2, kTmO = kTmS + 2 * kBN;
// Per stage: FULL (gathered), SFREE (S of its chunk done: the columns that
// PV does not read may be refilled), EMPTY (PV done: all of it).
constexpr int B_Q_READY = 0, B_QS_FULL = 1, B_FULL = 2, B_SFREE = B_FULL + kNST, B_EMPTY = B_SFREE + kNST,
              B_S_FULL = B_EMPTY + kNST,
              B_P_FULL = B_S_FULL + 2, B_O_FULL = B_P_FULL + 2, B_DRAIN = B_O_FULL + 1,
              B_QT_FULL = B_DRAIN + 1, kNumBars = B_QT_FULL + 1;
constexpr int kSmemQ = kNST * kStageBytes;                  // 1024-aligned
constexpr int kSmemBias = kSmemQ + kQSChunks * kQSChunkBytes;  // float [kNST][64]
constexpr int kSmemBar = kSmemBias + kNST * kBN * 4;
constexpr int kSmemTmem = kSmemBar + kNumBars * 8;
constexpr int kSmemAbort = kSmemTmem + 4;
constexpr int kSmemAlloc = kSmemAbort + 4 + 1024;
static_assert(kSmemAlloc <= 232448, "shared memory budget exceeded");
static_assert(kSmemQ % 1024 == 0 && kQSChunkBytes % 1024 == 0, "swizzled tiles need 1024-byte alignment");
static_assert(kTmO + kHalf <= 512, "TMEM budget exceeded");
// Warps: 0-3 softmax (thread = head), then kPW gather warps per stage, then
// the MMA issuer.
constexpr int kPW = 4;
constexpr int kMmaWarp = 4 + kNST * kPW;
constexpr int kThreads = (kMmaWarp + 1) * 32;
static_assert(kBN % kPW == 0 && kBN / kPW <= 32, "gather rows per warp");
static_assert((kQDim - kQT) % 64 == 0 && kQT % 64 == 0, "query split on 64-column chunks");

__global__ void __launch_bounds__(256) thd_sparse_mla_compact_kernel(const int32_t* __restrict__ idx,
                                                                      int64_t T, int K, int64_t Tg,
                                                                      int32_t* __restrict__ idx_c,
                                                                      int32_t* __restrict__ count) {
    const int lane = threadIdx.x & 31;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    const int32_t* src = idx + t * K;
    int32_t* dst = idx_c + t * K;
    int n = 0;
    for (int j0 = 0; j0 < K; j0 += 32) {
        const int j = j0 + lane;
        const int v = j < K ? src[j] : -1;
        const bool ok = v >= 0 && v < Tg;
        const unsigned m = __ballot_sync(0xffffffffu, ok);
        if (ok) dst[n + __popc(m & ((1u << lane) - 1u))] = v;
        n += __popc(m);
    }
    for (int j = n + lane; j < K; j += 32) dst[j] = -1;
    if (lane == 0) count[t] = n;
}

__global__ void __launch_bounds__(kThreads, 1) thd_sparse_mla_attn_kernel(const __grid_constant__ CUtensorMap tmap_q,
                                                                          const SmlaParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = thd::smem_addr(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
    const uint32_t sbase = thd::smem_addr(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int half = blockIdx.x & 1;
    const int hgroups = p.H / 128;
    const int hg = (blockIdx.x >> 1) % hgroups;
    const int64_t t = (blockIdx.x >> 1) / hgroups;
    const int nch = (p.count[t] + kBN - 1) / kBN;  // chunks holding valid slots
    auto bar = [&](int i) -> uint32_t { return sbase + kSmemBar + 8u * i; };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kSmemAbort);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kSmemTmem);
    float* bias = reinterpret_cast<float*>(smem + kSmemBias);

    if (threadIdx.x == 0) {
        thd::mbar_init(bar(B_Q_READY), 4);
        thd::mbar_init(bar(B_QT_FULL), 1);
        thd::mbar_init(bar(B_QS_FULL), 1);
        for (int s = 0; s < kNST; ++s) {
            thd::mbar_init(bar(B_FULL + s), kPW);  // the stage's gather warps
            thd::mbar_init(bar(B_SFREE + s), 1);
            thd::mbar_init(bar(B_EMPTY + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            thd::mbar_init(bar(B_S_FULL + b), 1);
            thd::mbar_init(bar(B_P_FULL + b), 4);
        }
        thd::mbar_init(bar(B_O_FULL), 1);
        thd::mbar_init(bar(B_DRAIN), 1);
        *abort_flag = *reinterpret_cast<volatile int*>(p.status) != 0 ? 1 : 0;
        thd::fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        thd::tmem_alloc(thd::smem_addr(tmem_slot), 512);
        thd::tmem_relinquish();
    }
    thd::tc_fence_before();
    __syncthreads();
    thd::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const bool skip = *abort_flag != 0;

    if (warp >= 4 && warp < kMmaWarp) {
        // ------------------------------------------------- gather producers
        // kPW warps per stage: stage 0 takes the even chunks, stage 1 the
        // odd ones.  Chunk c refills its stage in two parts: the columns that
        // PV does not read (the other latent half and the rotary part) once
        // S of chunk c - kNST is done, then this CTA's latent half once PV of
        // chunk c - kNST is done; it is published as soon as its copies have
        // landed, independently of the other stage.  Warp wi copies rows
        // [wi * kBN / kPW, +kBN / kPW) of the chunk, lane = 16-byte unit of a
        // row (units [32 k, 32 k + 32) of a row in copy k; this CTA's latent
        // half is exactly copy k = half), so each copy instruction moves 512
        // contiguous bytes of one kv row.  An invalid slot reads row 0 and
        // gets a -inf bias.
        constexpr int kRows = kBN / kPW;
        const int pw = warp - 4;
        const int s = pw / kPW;                 // this warp's stage
        // Stage 1 first holds Q's TMEM columns on their way into TMEM: its
        // gathers start once the softmax warps have read them.
        const int r0 = (pw % kPW) * kRows;
        const int32_t* irow = p.idx + t * p.K;
        bool ok = !skip;
        if (ok && s == 1 && nch > 1) ok = thd::warp_wait(bar(B_Q_READY), 0, abort_flag, p.status);
        for (int c = s; ok && c < nch; c += kNST) {
            const uint32_t par = ((c / kNST) & 1) ^ 1;
            ok = thd::warp_wait(bar(B_SFREE + s), par, abort_flag, p.status);
            if (!ok) break;
            const uint32_t stage = sbase + s * kStageBytes;
            const __nv_bfloat16* src[kRows];
#pragma unroll
            for (int rr = 0; rr < kRows; ++rr) {
                const int gi = irow[c * kBN + r0 + rr];
                src[rr] = p.kv + static_cast<int64_t>((gi >= 0 && gi < p.Tg) ? gi : 0) * kQDim;
            }
            auto copy = [&](int rr, int k) {
                const int r = r0 + rr;
                const int uu = lane + 32 * k;
                if (uu < 72)
                    cp_async16_nc(stage + r * 128 + (uu >> 3) * kChunkBytes +
                                      ((static_cast<uint32_t>(uu & 7) ^ static_cast<uint32_t>(r & 7)) << 4),
                                  src[rr] + uu * 8);
            };
#pragma unroll
            for (int rr = 0; rr < kRows; ++rr) {
#pragma unroll
                for (int k = 0; k < 3; ++k)
                    if (k != half) copy(rr, k);
            }
            ok = thd::warp_wait(bar(B_EMPTY + s), par, abort_flag, p.status);
            if (!ok) break;
            if (lane < kRows) {
                const int gi = irow[c * kBN + r0 + lane];
                bias[s * kBN + r0 + lane] = (gi >= 0 && gi < p.Tg) ? 0.0f : -INFINITY;
            }
#pragma unroll
            for (int rr = 0; rr < kRows; ++rr) copy(rr, half);
            cp_async_commit();
            cp_async_wait<0>();
            thd::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) thd::mbar_arrive(bar(B_FULL + s));
        }
        cp_async_wait<0>();
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------- MMA issuer
        // Order S(0) S(1) PV(0) S(2) PV(1) ...: S(c + 1) runs while the
        // softmax works on chunk c (two S / P buffers; S(c + 2) reuses the
        // buffer of P(c) only after PV(c), which the in-order tensor pipe
        // guarantees).
        if (lane == 0 && !skip) {
            constexpr uint32_t idesc_s = thd::idesc_bf16_f32(128, kBN, false);
            constexpr uint32_t idesc_o = thd::idesc_bf16_f32(128, kHalf, true);
            auto wait = [&](int i, uint32_t par) -> bool {
                return thd::mbar_wait(bar(i), par, abort_flag, p.status, kStatusTimeout);
            };
            const uint64_t dq0 = thd::smem_desc_sw128(sbase + kSmemQ, 16, 1024);
            // S(c) = Q kv^T: the first kQT columns of Q from TMEM, the rest
            // from shared memory (K steps of 16 columns = 32 bytes).
            auto issue_s = [&](int c) {
                const uint64_t dk = thd::smem_desc_sw128(sbase + (c % kNST) * kStageBytes, 16, 1024);
                const uint32_t d = tmem_base + kTmS + kBN * (c & 1);
#pragma unroll
                for (int kk = 0; kk < kQT / 16; ++kk)
                    thd::mma_bf16_ts(d, tmem_base + kTmQ + kk * 8,
                                     dk + (((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4), idesc_s,
                                     kk > 0 ? 1u : 0u);
#pragma unroll
                for (int kk = kQT / 16; kk < kQDim / 16; ++kk) {
                    const int qk = kk - kQT / 16;
                    thd::mma_bf16_ss(d, dq0 + (((qk >> 2) * kQSChunkBytes + (qk & 3) * 32) >> 4),
                                     dk + (((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4), idesc_s, 1u);
                }
            };
            // Issue whichever of the next S and the next PV can go first
            // (non-blocking tests): S(k) needs chunk k gathered and PV(k - 2)
            // issued (its S / P buffer), PV(k) needs P(k).  A PV that can go
            // is issued first: it frees the chunk's stage for the gather of
            // chunk k + 2.
            // Q[:, :kQT] of the token's 128 heads (four 64-column boxes) into
            // stage 1, on their way into TMEM; Q[:, kQT:] (five boxes)
            // straight into the swizzled layout the MMAs read.
            thd::tma_prefetch_desc(&tmap_q);
            thd::mbar_arrive_expect_tx(bar(B_QT_FULL), (kQT / 64) * kQSChunkBytes);
            for (int i = 0; i < kQT / 64; ++i)
                thd::tma_load_3d(sbase + kStageBytes + i * kQSChunkBytes, &tmap_q, bar(B_QT_FULL), 64 * i,
                                 hg * 128, static_cast<int>(t));
            thd::mbar_arrive_expect_tx(bar(B_QS_FULL), kQSChunks * kQSChunkBytes);
            for (int i = 0; i < kQSChunks; ++i)
                thd::tma_load_3d(sbase + kSmemQ + i * kQSChunkBytes, &tmap_q, bar(B_QS_FULL), kQT + 64 * i,
                                 hg * 128, static_cast<int>(t));
            bool ok = wait(B_QS_FULL, 0);
            if (!ok) thd::drain_wait(bar(B_QS_FULL), 0);
            ok = ok && wait(B_Q_READY, 0);
            int next_s = 0, next_pv = 0;
            uint64_t t_wait = 0;
            while (ok && next_pv < nch) {
                if (next_pv < next_s &&
                    thd::mbar_test(bar(B_P_FULL + (next_pv & 1)), (next_pv >> 1) & 1)) {
                    const int c = next_pv;
                    thd::tc_fence_after();
                    // latent half += P kv[:, half]: N = 256, the MN-major
                    // operand spans four 64-column chunks of the stage.
                    const uint64_t dv = thd::smem_desc_sw128(
                        sbase + (c % kNST) * kStageBytes + 4 * half * kChunkBytes, kChunkBytes, 1024);
#pragma unroll
                    for (int kk = 0; kk < kBN / 16; ++kk)
                        thd::mma_bf16_ts(tmem_base + kTmO, tmem_base + kTmS + kBN * (c & 1) + kk * 8,
                                         dv + ((kk * 16 * 128) >> 4), idesc_o, (c > 0 || kk > 0) ? 1u : 0u);
                    thd::mma_commit(bar(B_O_FULL));
                    thd::mma_commit(bar(B_EMPTY + c % kNST));
                    ++next_pv;
                    t_wait = 0;
                    continue;
                }
                if (next_s < nch && next_s <= next_pv + 1 &&
                    thd::mbar_test(bar(B_FULL + next_s % kNST), (next_s / kNST) & 1)) {
                    thd::tc_fence_after();
                    issue_s(next_s);
                    thd::mma_commit(bar(B_S_FULL + (next_s & 1)));
                    thd::mma_commit(bar(B_SFREE + next_s % kNST));
                    ++next_s;
                    t_wait = 0;
                    continue;
                }
                // Neither can go yet: bounded wait.
                const uint64_t now = thd::global_timer_ns();
                if (t_wait == 0) {
                    t_wait = now;
                } else if (now - t_wait > thd::kWaitLimitNs) {
                    atomicCAS(p.status, 0, kStatusTimeout);
                    *abort_flag = 1;
                    ok = false;
                } else if (*abort_flag || *reinterpret_cast<volatile int*>(p.status) != 0) {
                    *abort_flag = 1;
                    ok = false;
                }
            }
            thd::mma_commit(bar(B_DRAIN));
            thd::drain_wait(bar(B_DRAIN), 0);
            thd::drain_wait(bar(B_QT_FULL), 0);  // (landed long ago unless unwinding)
        }
        __syncwarp();
    } else {
        // --------------------------------------------------- softmax (128)
        const int row = warp * 32 + lane;
        const int h = hg * 128 + row;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
        bool ok = !skip;
        if (ok) ok = thd::warp_wait(bar(B_QT_FULL), 0, abort_flag, p.status);
        if (ok) {
            // Q row h, columns [0, kQT), into TMEM (bf16 pairs), from the
            // four 64-column boxes TMA put into stage 1 (128-byte swizzle:
            // 16-byte unit u of row r at r * 128 + ((u ^ (r % 8)) * 16)).
            // Arriving on Q_READY also hands stage 1 to its gather warps.
            const uint32_t qt = sbase + kStageBytes + static_cast<uint32_t>(row) * 128;
#pragma unroll
            for (int i = 0; i < kQT / 64; ++i) {
                uint32_t w[32];
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    ld_shared_v4(qt + i * kQSChunkBytes + ((static_cast<uint32_t>(u) ^ static_cast<uint32_t>(row & 7)) << 4),
                                 w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
                thd::tmem_st32(lane_base + kTmQ + 32 * i, w);
            }
            thd::tmem_wait_st();
            thd::tc_fence_before();
            __syncwarp();
            if (lane == 0) thd::mbar_arrive(bar(B_Q_READY));
        }
        float m_ref = -INFINITY, l = 0.0f;
        constexpr float kTau = 8.0f;
        const float sl2 = p.scale_log2;
        for (int c = 0; ok && c < nch; ++c) {
            const int s = c % kNST;
            const uint32_t ts = lane_base + kTmS + kBN * (c & 1);
            ok = thd::warp_wait(bar(B_FULL + s), (c / kNST) & 1, abort_flag, p.status) &&
                 thd::warp_wait(bar(B_S_FULL + (c & 1)), (c >> 1) & 1, abort_flag, p.status);
            if (!ok) break;
            thd::tc_fence_after();
            uint32_t sr[64];
            thd::tmem_ld32(ts, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
            thd::tmem_ld32(ts + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
            thd::tmem_wait_ld();
            thd::reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
            thd::reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
            const float4* b4 = reinterpret_cast<const float4*>(bias + s * kBN);
            float x[64];
            float mx = -INFINITY;
#pragma unroll
            for (int j4 = 0; j4 < 16; ++j4) {
                const float4 b = b4[j4];
                const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = 4 * j4 + e;
                    x[j] = fmaf(__uint_as_float(sr[j]), sl2, bv[e]);
                    mx = fmaxf(mx, x[j]);
                }
            }
            float alpha = 1.0f;
            bool rescale_o = false;
            if (c == 0 || m_ref == -INFINITY) {
                if (mx > m_ref) {
                    alpha = thd::ex2_approx(m_ref - mx);
                    m_ref = mx;
                    rescale_o = c > 0;
                }
            } else if (mx > m_ref + kTau) {
                alpha = thd::ex2_approx(m_ref - mx);
                m_ref = mx;
                rescale_o = true;
            }
            l *= alpha;
            const float neg_m = m_ref == -INFINITY ? 0.0f : -m_ref;
            uint32_t pk[32];
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                const float p0 = thd::ex2_approx(x[2 * u] + neg_m);
                const float p1 = thd::ex2_approx(x[2 * u + 1] + neg_m);
                l += p0 + p1;
                pk[u] = thd::pack_bf16x2(p0, p1);
            }
            thd::tmem_st16(ts, *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
            thd::tmem_st16(ts + 16, *reinterpret_cast<uint32_t(*)[16]>(&pk[16]));
            if (c > 0) {
                // The previous chunk's product must be done before O is
                // rescaled (and before this chunk's is issued); waiting every
                // chunk also keeps the P barriers within one phase of the
                // MMA issuer.
                ok = thd::warp_wait(bar(B_O_FULL), (c - 1) & 1, abort_flag, p.status);
                if (!ok) break;
                thd::tc_fence_after();
                if (__any_sync(0xffffffffu, rescale_o)) {
#pragma unroll 1
                    for (int cc = 0; cc < kHalf / 32; ++cc) {
                        uint32_t r[32];
                        thd::tmem_ld32(lane_base + kTmO + 32 * cc, r);
                        thd::tmem_wait_ld();
                        thd::reg_fence32(r);
#pragma unroll
                        for (int u = 0; u < 32; ++u) r[u] = __float_as_uint(__uint_as_float(r[u]) * alpha);
                        thd::tmem_st32(lane_base + kTmO + 32 * cc, r);
                    }
                }
            }
            thd::tmem_wait_st();
            thd::tc_fence_before();
            __syncwarp();
            if (lane == 0) thd::mbar_arrive(bar(B_P_FULL + (c & 1)));
        }
        if (ok && nch > 0) ok = thd::warp_wait(bar(B_O_FULL), (nch - 1) & 1, abort_flag, p.status);
        if (ok) {
            thd::tc_fence_after();
            const float inv_l = l > 0.0f ? 1.0f / l : 0.0f;
            __nv_bfloat16* dst = p.latent + (t * p.H + h) * kLat + kHalf * half;
#pragma unroll 1
            for (int cc = 0; cc < kHalf / 32; ++cc) {
                uint32_t r[32];
                if (nch > 0) {
                    thd::tmem_ld32(lane_base + kTmO + 32 * cc, r);
                    thd::tmem_wait_ld();
                    thd::reg_fence32(r);
                } else {
#pragma unroll
                    for (int u = 0; u < 32; ++u) r[u] = 0u;
                }
                uint32_t w[16];
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    w[u] = thd::pack_bf16x2(__uint_as_float(r[2 * u]) * inv_l,
                                            __uint_as_float(r[2 * u + 1]) * inv_l);
                uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * cc);
#pragma unroll
                for (int u = 0; u < 4; ++u) d4[u] = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
            }
        }
    }
    thd::tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        thd::tc_fence_after();
        thd::tmem_dealloc(tmem_base, 512);
    }
}

// --------------------------------------------------------------- projection --
// out[t, h, :vd] = latent[t, h, :512] @ W[h]^T: one CTA per (128 tokens,
// head); K = 512 in 8 chunks of 64 through a 3-stage TMA ring (at value dim
// 128, 99 KB of shared memory: two CTAs per SM overlap one's set-up and
// epilogue with the other's loads; 4 stages and one CTA measured ~1 % slower
// for the whole sparse MLA call).
struct ProjParams {
    __nv_bfloat16* out;  // [T, H, vd]
    int* status;
    int64_t T;
    int H, vd;
};

constexpr int kPNST = 3;
constexpr int kPA = 128 * 128;  // A chunk: 128 tokens x 64 latent columns

template <int VD>
__global__ void __launch_bounds__(192, 1) thd_sparse_mla_proj_kernel(
    const __grid_constant__ CUtensorMap map_lat, const __grid_constant__ CUtensorMap map_w,
    const ProjParams p) {
    constexpr int kPB = VD * 128;  // B chunk: VD rows x 64 columns
    constexpr int kStage = kPA + kPB;
    constexpr int BAR = kPNST * kStage;
    constexpr int TMEM_COLS = VD <= 32 ? 32 : VD <= 64 ? 64 : VD <= 128 ? 128 : 256;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = thd::smem_addr(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
    const uint32_t sbase = thd::smem_addr(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.x % p.H;
    const int64_t t0 = static_cast<int64_t>(blockIdx.x / p.H) * 128;
    auto bar = [&](int i) -> uint32_t { return sbase + BAR + 8u * i; };  // FULL[4], EMPTY[4], ACC, DRAIN
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + BAR + 8 * (2 * kPNST + 2));
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + BAR + 8 * (2 * kPNST + 2) + 4);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kPNST; ++s) {
            thd::mbar_init(bar(s), 1);
            thd::mbar_init(bar(kPNST + s), 1);
        }
        thd::mbar_init(bar(2 * kPNST), 1);
        thd::mbar_init(bar(2 * kPNST + 1), 1);
        *abort_flag = *reinterpret_cast<volatile int*>(p.status) != 0 ? 1 : 0;
        thd::fence_barrier_init();
    }
    if (warp == 5) {
        thd::tmem_alloc(thd::smem_addr(tmem_slot), TMEM_COLS);
        thd::tmem_relinquish();
    }
    thd::tc_fence_before();
    __syncthreads();
    thd::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const bool skip = *abort_flag != 0;
    constexpr int NCH = kLat / 64;
    if (warp == 4) {
        if (lane == 0 && !skip) {
            thd::tma_prefetch_desc(&map_lat);
            thd::tma_prefetch_desc(&map_w);
            int issued = 0;
            bool ok = true;
            for (int c = 0; c < NCH && ok; ++c) {
                const int s = c % kPNST;
                ok = thd::mbar_wait(bar(kPNST + s), ((c / kPNST) & 1) ^ 1, abort_flag, p.status,
                                    kStatusTimeout);
                if (!ok) break;
                thd::mbar_arrive_expect_tx(bar(s), kStage);
                thd::tma_load_3d(sbase + s * kStage, &map_lat, bar(s), c * 64, h, static_cast<int>(t0));
                thd::tma_load_3d(sbase + s * kStage + kPA, &map_w, bar(s), c * 64, 0, h);
                issued = c + 1;
            }
            if (!ok)
                for (int c = issued - kPNST > 0 ? issued - kPNST : 0; c < issued; ++c)
                    thd::drain_wait(bar(c % kPNST), (c / kPNST) & 1);
        }
        __syncwarp();
    } else if (warp == 5) {
        if (lane == 0 && !skip) {
            constexpr uint32_t idesc = thd::idesc_bf16_f32(128, VD, false);
            bool ok = true;
            for (int c = 0; c < NCH && ok; ++c) {
                const int s = c % kPNST;
                ok = thd::mbar_wait(bar(s), (c / kPNST) & 1, abort_flag, p.status, kStatusTimeout);
                if (!ok) break;
                thd::tc_fence_after();
                const uint64_t da = thd::smem_desc_sw128(sbase + s * kStage, 16, 1024);
                const uint64_t db = thd::smem_desc_sw128(sbase + s * kStage + kPA, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    thd::mma_bf16_ss(tmem_base, da + ((kk * 32) >> 4), db + ((kk * 32) >> 4), idesc,
                                     (c > 0 || kk > 0) ? 1u : 0u);
                thd::mma_commit(bar(kPNST + s));
            }
            if (ok) thd::mma_commit(bar(2 * kPNST));
            thd::mma_commit(bar(2 * kPNST + 1));
            thd::drain_wait(bar(2 * kPNST + 1), 0);
        }
        __syncwarp();
    } else if (warp < 4) {
        const int64_t t = t0 + warp * 32 + lane;
        bool ok = !skip && thd::warp_wait(bar(2 * kPNST), 0, abort_flag, p.status);
        if (ok) {
            thd::tc_fence_after();
            const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
#pragma unroll 1
            for (int cc = 0; cc < VD / 32; ++cc) {
                uint32_t r[32];
                thd::tmem_ld32(lane_base + 32 * cc, r);
                thd::tmem_wait_ld();
                thd::reg_fence32(r);
                uint32_t w[16];
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    w[u] = thd::pack_bf16x2(__uint_as_float(r[2 * u]), __uint_as_float(r[2 * u + 1]));
                if (t < p.T) {
                    uint4* d4 = reinterpret_cast<uint4*>(p.out + (t * p.H + h) * VD + 32 * cc);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        d4[u] = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
                }
            }
        }
    }
    thd::tc_fence_before();
    __syncthreads();
    if (warp == 5) {
        thd::tc_fence_after();
        thd::tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

template <int VD>
constexpr int proj_smem() {
    return kPNST * (kPA + VD * 128) + 8 * (2 * kPNST + 2) + 8 + 1024;
}

// 3-D map over q [T, H, 576]: dims (576, H, T), box (64, 128, 1): one token's
// 128 heads, 64 columns.
bool make_q_map(CUtensorMap* map, const void* base, int64_t T, int H) {
    auto fn = thd::encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(kQDim), static_cast<cuuint64_t>(H),
                          static_cast<cuuint64_t>(T)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(kQDim) * 2, static_cast<cuuint64_t>(H) * kQDim * 2};
    cuuint32_t box[3] = {64, 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over value_weight [H, VD, 512]: dims (512, VD, H), box (64, VD, 1).
bool make_w_map(CUtensorMap* map, const void* base, int H, int vd) {
    auto fn = thd::encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {512, static_cast<cuuint64_t>(vd), static_cast<cuuint64_t>(H)};
    cuuint64_t strides[2] = {512 * 2, static_cast<cuuint64_t>(vd) * 512 * 2};
    cuuint32_t box[3] = {64, static_cast<cuuint32_t>(vd), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int VD>
int launch_proj(const CUtensorMap& ml, const CUtensorMap& mw, const ProjParams& pp, cudaStream_t st) {
    auto k = thd_sparse_mla_proj_kernel<VD>;
    static bool attr[64] = {};  // per device
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return THD_ERR_CUDA;
    if (!attr[dev]) {
        if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, proj_smem<VD>()) !=
            cudaSuccess)
            return THD_ERR_CUDA;
        attr[dev] = true;
    }
    const int64_t tiles = (pp.T + 127) / 128;
    k<<<static_cast<unsigned>(tiles * pp.H), 192, proj_smem<VD>(), st>>>(ml, mw, pp);
    return cudaGetLastError() == cudaSuccess ? THD_OK : THD_ERR_CUDA;
}

int* g_status[64] = {};

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

}  // namespace

// Workspace: the bf16 latent [T, H, 512], the compacted indices [T, K] and
// the per-token valid-slot counts [T] (each part 256-byte aligned).
extern "C" size_t thd_sparse_mla_workspace_bytes(int64_t T, int H, int K) {
    if (T <= 0 || H <= 0 || K < 0) return 0;
    return align256(static_cast<size_t>(T) * static_cast<size_t>(H) * kLat * 2) +
           align256(static_cast<size_t>(T) * static_cast<size_t>(K) * 4) +
           align256(static_cast<size_t>(T) * 4);
}

extern "C" int thd_sparse_mla_fwd(const void* q, const void* kv, const int32_t* indices,
                                  const void* value_weight, int64_t T, int64_t Tg, int H, int K,
                                  int value_dim, float scale, void* out, void* workspace,
                                  size_t workspace_bytes, void* stream_ptr) {
    if (T < 0 || Tg < 0 || H <= 0 || K < 0) return THD_ERR_INVALID_ARG;
    if (H % 128 != 0 || K % kBN != 0) return THD_ERR_UNSUPPORTED;
    if (value_dim != 64 && value_dim != 128 && value_dim != 256) return THD_ERR_UNSUPPORTED;
    if (!(std::isfinite(scale) && scale >= 0.0f)) return THD_ERR_INVALID_ARG;
    if (T == 0) return THD_OK;
    if (T * (H / 128) * 2 > 0x7fffffffLL || Tg > 0x7fffffffLL) return THD_ERR_INVALID_ARG;
    if (!q || !kv || (!indices && K > 0) || !value_weight || !out || !workspace)
        return THD_ERR_INVALID_ARG;
    if (!thd::aligned16(q) || !thd::aligned16(kv) || !thd::aligned16(value_weight) ||
        !thd::aligned16(out) || !thd::aligned16(workspace) ||
        (reinterpret_cast<uintptr_t>(indices) & 3u))
        return THD_ERR_INVALID_ARG;
    if (workspace_bytes < thd_sparse_mla_workspace_bytes(T, H, K)) return THD_ERR_INVALID_ARG;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return THD_ERR_CUDA;
    if (g_status[dev] == nullptr) {
        if (cudaMalloc(&g_status[dev], sizeof(int)) != cudaSuccess) return THD_ERR_NO_MEMORY;
        if (cudaMemset(g_status[dev], 0, sizeof(int)) != cudaSuccess) return THD_ERR_CUDA;
    }
    static bool attr[64] = {};  // per device
    if (!attr[dev]) {
        if (cudaFuncSetAttribute(thd_sparse_mla_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kSmemAlloc) != cudaSuccess)
            return THD_ERR_CUDA;
        attr[dev] = true;
    }
    char* ws = static_cast<char*>(workspace);
    int32_t* idx_c = reinterpret_cast<int32_t*>(ws + align256(static_cast<size_t>(T) * H * kLat * 2));
    int32_t* cnt = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(idx_c) +
                                              align256(static_cast<size_t>(T) * K * 4));
    const int Keff = Tg > 0 ? K : 0;  // no key rows: every slot is invalid
    thd_sparse_mla_compact_kernel<<<static_cast<unsigned>((T + 7) / 8), 256, 0, stream>>>(
        indices, T, Keff, Tg, idx_c, cnt);
    SmlaParams p;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.kv = static_cast<const __nv_bfloat16*>(kv);
    p.idx = idx_c;
    p.count = cnt;
    p.latent = static_cast<__nv_bfloat16*>(workspace);
    p.status = g_status[dev];
    p.T = T;
    p.Tg = Tg;
    p.H = H;
    p.K = Keff;
    p.scale_log2 = scale * 1.4426950408889634f;
    CUtensorMap mq;
    if (!make_q_map(&mq, q, T, H)) return THD_ERR_CUDA;
    thd_sparse_mla_attn_kernel<<<static_cast<unsigned>(T * (H / 128) * 2), kThreads, kSmemAlloc, stream>>>(
        mq, p);
    if (cudaGetLastError() != cudaSuccess) return THD_ERR_CUDA;

    CUtensorMap ml, mw;
    if (!thd::make_map(&ml, workspace, T, H, kLat, 128) || !make_w_map(&mw, value_weight, H, value_dim))
        return THD_ERR_CUDA;
    ProjParams pp{static_cast<__nv_bfloat16*>(out), g_status[dev], T, H, value_dim};
    switch (value_dim) {
        case 64: return launch_proj<64>(ml, mw, pp, stream);
        case 128: return launch_proj<128>(ml, mw, pp, stream);
        default: return launch_proj<256>(ml, mw, pp, stream);
    }
}

extern "C" int thd_sparse_mla_get_error(void* stream_ptr) {
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
    if (cudaStreamSynchronize(stream) != cudaSuccess) return THD_ERR_CUDA;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return THD_ERR_CUDA;
    if (g_status[dev] == nullptr) return THD_OK;
    int s = 0;
    if (cudaMemcpy(&s, g_status[dev], sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return THD_ERR_CUDA;
    if (s != 0 && cudaMemset(g_status[dev], 0, sizeof(int)) != cudaSuccess) return THD_ERR_CUDA;
    return s;
}
