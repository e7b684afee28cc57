// Packed-THD sliding-window GQA attention BACKWARD for B200 (sm_100a).
//
// The gradient of the forward in thd_attn_kernel.cuh (same document, window
// and sink readings of the API pages).  With P_ij = exp(s_ij - lse_i), the
// forward's saved log-sum-exp, and dO the gradient of the output:
//   D_i   = sum_c dO_ic O_ic                        (preprocess kernel)
//   dP_ij = dO_i . v_j,  dS_ij = P_ij (dP_ij - D_i)
//   dq_i  = scale * sum_j dS_ij k_j                  (dq kernel)
//   dk_j  = scale * sum_{h in group} sum_i dS_ij q_i (dkdv kernel)
//   dv_j  = sum_{h in group} sum_i P_ij dO_i         (dkdv kernel)
//   dsink_h = -sum_i exp(sink_h - lse_i) D_i         (preprocess + reduce)
//
// Both main kernels recompute S and dP on the tensor core instead of sharing
// them through memory, so nothing is accumulated with atomics and the result
// is bitwise reproducible:
//   * dq kernel: one CTA per (128-row query tile, query head), looping over
//     the key tiles the tile sees: S = Q K^T, dP = dO V^T, dS written as bf16
//     over S in TMEM, dq += dS K (dS from TMEM, K from shared memory as an
//     MN-major operand).  S alternates between two TMEM buffers, so the
//     tensor core computes dq(j), dP(j + 1) and S(j + 2) while the
//     elementwise warps exponentiate S(j + 1).
//   * dkdv kernel: one CTA per (128-key tile, kv head), looping over the
//     query heads of the group and the 128-query tiles that see the keys:
//     S^T = K Q^T and dP^T = V dO^T (TMEM lane = key), P^T and dS^T written as
//     bf16 over them, dv += P^T dO and dk += dS^T Q (TMEM operands, dO and Q
//     as MN-major operands); dk and dv stay in TMEM for the whole group.
//
// Head dim 256: the operand that streams through the ring (K/V tiles in the
// dq kernel, Q/dO tiles in the dkdv kernel) comes in tiles of BN = 64 rows so
// that the resident 128-row tiles and the ring fit in shared memory, and the
// key-side kernel runs twice, once accumulating dv only and once dk only (two
// 256-column accumulators do not fit in TMEM together); the dk launch
// recomputes S^T.
//
// Warps (both kernels): 0-7 elementwise, 8 TMA producer, 9 MMA issuer, 10-11
// idle.  Elementwise warp w owns TMEM lanes [32 (w % 4), 32 (w % 4) + 32).
// No row-wide reduction is needed (the log-sum-exp is known), so the warps
// on a sub-partition work on independent halves of every tile: the 64
// columns [64 h, 64 h + 64) of S and dP (or S^T and dP^T), h = w / 4, with
// the half's 64 bf16 results (P, dS) written over its own columns
// [64 h, 64 h + 32).  Every wait is bounded and reports a timeout in the
// device status word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "sm100_ptx.cuh"
#include "thd_attn_kernel.cuh"

namespace thd {

struct BwdKVItem {  // identical layout to thd_bwd_kv_item in thd_attn.h
    int32_t k0, doc_start, doc_end, g;
    int32_t n_q, pad0, pad1, pad2;
};

struct BwdParams {
    const WorkItem* q_items;    // dq kernel: one query head per item
    const BwdKVItem* kv_items;  // dkdv kernel
    const float* lse;           // [T, Hq] natural log (forward output)
    const float* delta;         // [T, Hq] rowsum(dO * O)
    __nv_bfloat16* dq;          // [T, Hq, D]
    __nv_bfloat16* dk;          // [T, Hkv, D]
    __nv_bfloat16* dv;          // [T, Hkv, D]
    int* status;
    int64_t T;
    int Hq, Hkv, G, window;
    float scale;
    float scale_log2;  // scale * log2(e)
};

constexpr float kLog2e = 1.4426950408889634f;

// TMEM column (relative to S or dP) of the bf16 operand for K-step kk of an
// MMA over BN columns: half kk / (BN / 32) is packed into [BN/2 half,
// BN/2 half + BN/4), eight columns (16 values) per step.
template <int BN>
__device__ __forceinline__ constexpr uint32_t pcol(int kk) {
    return static_cast<uint32_t>((BN / 2) * (kk / (BN / 32)) + 8 * (kk % (BN / 32)));
}

// -------------------------------------------------------------- preprocess --
// One warp per (token, head) row: delta = sum_c dO * O in fp32; with sinks
// also the row's share of the sink gradient, -exp(sink_h - lse) * delta.
template <int D>
__global__ void __launch_bounds__(256) thd_attn_bwd_preprocess_kernel(
    const __nv_bfloat16* __restrict__ out, const __nv_bfloat16* __restrict__ dout,
    const float* __restrict__ lse, const float* __restrict__ sinks, float* __restrict__ delta,
    float* __restrict__ sink_part, int64_t rows, int Hq) {
    constexpr int PER_LANE = D / 32;  // 2, 4 or 8 bf16 per lane
    const int lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (row >= rows) return;
    const __nv_bfloat16* o = out + row * D + lane * PER_LANE;
    const __nv_bfloat16* g = dout + row * D + lane * PER_LANE;
    float acc = 0.0f;
    if constexpr (PER_LANE == 8) {
        const uint4 a = *reinterpret_cast<const uint4*>(o);
        const uint4 b = *reinterpret_cast<const uint4*>(g);
        const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&av[u]));
            const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bv[u]));
            acc = fmaf(x.x, y.x, fmaf(x.y, y.y, acc));
        }
    } else if constexpr (PER_LANE == 4) {
        const uint2 a = *reinterpret_cast<const uint2*>(o);
        const uint2 b = *reinterpret_cast<const uint2*>(g);
        const uint32_t av[2] = {a.x, a.y}, bv[2] = {b.x, b.y};
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&av[u]));
            const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bv[u]));
            acc = fmaf(x.x, y.x, fmaf(x.y, y.y, acc));
        }
    } else {
        const uint32_t a = *reinterpret_cast<const uint32_t*>(o);
        const uint32_t b = *reinterpret_cast<const uint32_t*>(g);
        const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&a));
        const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&b));
        acc = fmaf(x.x, y.x, x.y * y.y);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) {
        delta[row] = acc;
        if (sinks != nullptr) {
            const int h = static_cast<int>(row % Hq);
            sink_part[row] = -ex2_approx((sinks[h] - lse[row]) * kLog2e) * acc;
        }
    }
}

// dsink[h] = sum over tokens of sink_part[t, h], one block per head, in a
// fixed order (strided per-thread sums, then a tree): deterministic.
__global__ void __launch_bounds__(256) thd_attn_bwd_dsink_kernel(const float* __restrict__ sink_part,
                                                                 int64_t T, int Hq,
                                                                 float* __restrict__ dsink) {
    __shared__ float red[256];
    const int h = blockIdx.x;
    float acc = 0.0f;
    for (int64_t t = threadIdx.x; t < T; t += blockDim.x) acc += sink_part[t * Hq + h];
    red[threadIdx.x] = acc;
    __syncthreads();
    for (int s = blockDim.x / 2; s > 0; s >>= 1) {
        if (static_cast<int>(threadIdx.x) < s) red[threadIdx.x] += red[threadIdx.x + s];
        __syncthreads();
    }
    if (threadIdx.x == 0) dsink[h] = red[0];
}

// ------------------------------------------------------------ shared shape --

// What the key-side kernel accumulates: dk and dv together (head dim <= 128),
// or one of them (head dim 256, two launches).
enum BwdKvMode { kDkDv = 0, kDvOnly = 1, kDkOnly = 2 };

template <int D_, int NSLOT_, int BN_ = 128, int MODE_ = kDkDv, int NDSLOT_ = NSLOT_, int NBUF_ = 1>
struct BwdConfig {
    static constexpr int D = D_;
    static constexpr int NSLOT = NSLOT_;    // dq: K/V ring slots; dkdv: Q tile slots
    static constexpr int NDSLOT = NDSLOT_;  // dkdv: dO tile slots
    static constexpr int NBUF = NBUF_;      // dkdv: S^T / dP^T buffers (2: one accumulator, BN = 64)
    static constexpr int BM = 128;        // TMEM lanes (queries for dq, keys for dkdv)
    static constexpr int BN = BN_;        // columns of S per tile (keys for dq, queries for dkdv)
    static constexpr int MODE = MODE_;    // dkdv kernel only
    static constexpr int HALF = BN / 2;   // columns of S per elementwise warp
    static constexpr int KCH = D / 64;
    static constexpr int BOX_BYTES = 128 * 128;   // one 64-column chunk of a 128-row tile
    static constexpr int TILE_BYTES = 128 * D * 2;
    static constexpr int NBOX_BYTES = BN * 128;   // one 64-column chunk of a BN-row tile
    static constexpr int NTILE_BYTES = BN * D * 2;

    static constexpr int TM_S = 0;        // S (dq) or S^T (dkdv), then P / dS bf16
    static constexpr int TM_DP = 128;     // dP or dP^T, then dS^T (dkdv)
    static constexpr int TM_ACC0 = 256;   // dq (dq kernel) or dv (dkdv kernel)
    static constexpr int TM_ACC1 = MODE == kDkDv ? 256 + D : 256;  // dk (dkdv kernel)
    static constexpr int TM_S2 = BN == 128 ? 384 : BN;  // dq kernel: second S buffer (odd key tiles)
    static constexpr int TMEM_COLS = 512;

    static constexpr int PRODUCER_WARP = 8;
    static constexpr int MMA_WARP = 9;
    static constexpr int NUM_THREADS = 384;

    static_assert(D == 64 || D == 128 || D == 256, "backward kernels: head dim 64, 128 or 256");
    static_assert(BN == 128 || BN == 64, "S tiles of 128 or 64 columns");
    static_assert(TM_ACC0 + D <= 512, "TMEM budget exceeded");
    static_assert(BN == 64 ? (TM_S2 + BN <= TM_DP) : (TM_ACC0 + D <= TM_S2 && TM_S2 + BN <= TMEM_COLS),
                  "dq kernel TMEM budget exceeded");
    static_assert(NSLOT >= 1, "ring needs a slot");
};

// ------------------------------------------------------------------ dq ------
template <class C>
struct DqLayout {
    static constexpr int B_IN_FULL = 0;                       // Q and dO landed
    static constexpr int B_SLOT_FULL = 1;
    static constexpr int B_SLOT_EMPTY = B_SLOT_FULL + C::NSLOT;
    static constexpr int B_S_FULL = B_SLOT_EMPTY + C::NSLOT;  // [2] S of an even / odd tile done
    static constexpr int B_DP_FULL = B_S_FULL + 2;            // dP done
    static constexpr int B_DS_FULL = B_DP_FULL + 1;           // dS in TMEM (8 warps)
    static constexpr int B_ACC_FULL = B_DS_FULL + 1;          // dq accumulated
    static constexpr int B_DRAIN = B_ACC_FULL + 1;
    static constexpr int NUM_BARS = B_DRAIN + 1;
    static constexpr int SMEM_Q = 0;
    static constexpr int SMEM_DO = SMEM_Q + C::TILE_BYTES;
    static constexpr int SMEM_SLOTS = SMEM_DO + C::TILE_BYTES;  // [NSLOT] K or V tile of BN rows
    static constexpr int SMEM_BAR = SMEM_SLOTS + C::NSLOT * C::NTILE_BYTES;
    static constexpr int SMEM_TMEM_SLOT = SMEM_BAR + NUM_BARS * 8;
    static constexpr int SMEM_ABORT = SMEM_TMEM_SLOT + 4;
    static constexpr int SMEM_ALLOC = SMEM_ABORT + 4 + 1024;
    static_assert(SMEM_ALLOC <= 232448, "shared memory budget exceeded");
    static_assert(C::NSLOT >= 2, "dq ring needs two slots");
};

template <class C>
__global__ void __launch_bounds__(C::NUM_THREADS, 1)
thd_attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmap_q,
                       const __grid_constant__ CUtensorMap tmap_do,
                       const __grid_constant__ CUtensorMap tmap_k,
                       const __grid_constant__ CUtensorMap tmap_v, const BwdParams prm) {
    using L = DqLayout<C>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
    const uint32_t sbase = smem_addr(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const WorkItem it = prm.q_items[blockIdx.x];
    const int n = it.n_kv;
    const int h = it.head0;

    auto bar = [&](int idx) -> uint32_t { return sbase + L::SMEM_BAR + 8u * idx; };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::SMEM_ABORT);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::SMEM_TMEM_SLOT);

    if (threadIdx.x == 0) {
        mbar_init(bar(L::B_IN_FULL), 1);
        for (int s = 0; s < C::NSLOT; ++s) {
            mbar_init(bar(L::B_SLOT_FULL + s), 1);
            mbar_init(bar(L::B_SLOT_EMPTY + s), 1);
        }
        mbar_init(bar(L::B_S_FULL), 1);
        mbar_init(bar(L::B_S_FULL + 1), 1);
        mbar_init(bar(L::B_DP_FULL), 1);
        mbar_init(bar(L::B_DS_FULL), 8);
        mbar_init(bar(L::B_ACC_FULL), 1);
        mbar_init(bar(L::B_DRAIN), 1);
        *abort_flag = *reinterpret_cast<volatile int*>(prm.status) != 0 ? 1 : 0;
        fence_barrier_init();
    }
    if (warp == C::MMA_WARP) {
        tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const bool skip = *abort_flag != 0;

    if (warp == C::PRODUCER_WARP) {
        if (lane == 0 && !skip) {
            tma_prefetch_desc(&tmap_q);
            tma_prefetch_desc(&tmap_do);
            tma_prefetch_desc(&tmap_k);
            tma_prefetch_desc(&tmap_v);
            const int g = h / prm.G;
            mbar_arrive_expect_tx(bar(L::B_IN_FULL), 2 * C::TILE_BYTES);
            for (int c = 0; c < C::KCH; ++c) {
                tma_load_3d(sbase + L::SMEM_Q + c * C::BOX_BYTES, &tmap_q, bar(L::B_IN_FULL), c * 64,
                            h, it.q0);
                tma_load_3d(sbase + L::SMEM_DO + c * C::BOX_BYTES, &tmap_do, bar(L::B_IN_FULL),
                            c * 64, h, it.q0);
            }
            // Ring positions: 2j holds K(j), 2j+1 holds V(j).
            int issued = 0;
            bool ok = true;
            for (int pos = 0; pos < 2 * n && ok; ++pos) {
                const int slot = pos % C::NSLOT;
                ok = mbar_wait(bar(L::B_SLOT_EMPTY + slot), ((pos / C::NSLOT) & 1) ^ 1, abort_flag,
                               prm.status, kStatusTimeout);
                if (!ok) break;
                const CUtensorMap* map = (pos & 1) ? &tmap_v : &tmap_k;
                const int kt = it.kv_start + (pos >> 1) * C::BN;
                mbar_arrive_expect_tx(bar(L::B_SLOT_FULL + slot), C::NTILE_BYTES);
                for (int c = 0; c < C::KCH; ++c)
                    tma_load_3d(sbase + L::SMEM_SLOTS + slot * C::NTILE_BYTES + c * C::NBOX_BYTES, map,
                                bar(L::B_SLOT_FULL + slot), c * 64, g, kt);
                issued = pos + 1;
            }
            if (!ok) {
                drain_wait(bar(L::B_IN_FULL), 0);
                for (int pos = issued - C::NSLOT > 0 ? issued - C::NSLOT : 0; pos < issued; ++pos)
                    drain_wait(bar(L::B_SLOT_FULL + pos % C::NSLOT), (pos / C::NSLOT) & 1);
            }
        }
        __syncwarp();
    } else if (warp == C::MMA_WARP) {
        if (lane == 0 && !skip) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, C::BN, false);
            constexpr uint32_t idesc_acc = idesc_bf16_f32(128, C::D, true);
            const uint64_t dq0 = smem_desc_sw128(sbase + L::SMEM_Q, 16, 1024);
            const uint64_t ddo0 = smem_desc_sw128(sbase + L::SMEM_DO, 16, 1024);
            const uint64_t dkv0 = smem_desc_sw128(sbase + L::SMEM_SLOTS, 16, 1024);
            const uint64_t dkmn0 = smem_desc_sw128(sbase + L::SMEM_SLOTS, C::NBOX_BYTES, 1024);
            auto wait = [&](int idx, uint32_t parity) -> bool {
                return mbar_wait(bar(idx), parity, abort_flag, prm.status, kStatusTimeout);
            };
            auto wait_slot = [&](int pos) -> bool {
                return wait(L::B_SLOT_FULL + pos % C::NSLOT, (pos / C::NSLOT) & 1);
            };
            // Two S buffers: S(j + 2) and dP(j + 1) run on the tensor core
            // while the elementwise warps turn S(j + 1) into exponentials.
            auto issue_s = [&](int j) -> bool {  // S(j) = Q K(j)^T into buffer j % 2
                if (!wait_slot(2 * j)) return false;
                tc_fence_after();
                const uint64_t dk = dkv0 + ((((2 * j) % C::NSLOT) * C::NTILE_BYTES) >> 4);
                const uint32_t ts = tmem_base + ((j & 1) ? C::TM_S2 : C::TM_S);
#pragma unroll
                for (int kk = 0; kk < C::D / 16; ++kk) {
                    const uint32_t o = ((kk >> 2) * C::BOX_BYTES + (kk & 3) * 32) >> 4;
                    const uint32_t on = ((kk >> 2) * C::NBOX_BYTES + (kk & 3) * 32) >> 4;
                    mma_bf16_ss(ts, dq0 + o, dk + on, idesc_s, kk > 0 ? 1u : 0u);
                }
                mma_commit(bar(L::B_S_FULL + (j & 1)));
                return true;
            };
            auto issue_dp = [&](int j) -> bool {  // dP(j) = dO V(j)^T
                if (!wait_slot(2 * j + 1)) return false;
                tc_fence_after();
                const int vslot = (2 * j + 1) % C::NSLOT;
                const uint64_t dv = dkv0 + ((vslot * C::NTILE_BYTES) >> 4);
#pragma unroll
                for (int kk = 0; kk < C::D / 16; ++kk) {
                    const uint32_t o = ((kk >> 2) * C::BOX_BYTES + (kk & 3) * 32) >> 4;
                    const uint32_t on = ((kk >> 2) * C::NBOX_BYTES + (kk & 3) * 32) >> 4;
                    mma_bf16_ss(tmem_base + C::TM_DP, ddo0 + o, dv + on, idesc_s, kk > 0 ? 1u : 0u);
                }
                mma_commit(bar(L::B_DP_FULL));
                mma_commit(bar(L::B_SLOT_EMPTY + vslot));  // V(j) consumed
                return true;
            };
            bool ok = wait(L::B_IN_FULL, 0) && issue_s(0) && issue_dp(0) && (n < 2 || issue_s(1));
            for (int j = 0; ok && j < n; ++j) {
                ok = wait(L::B_DS_FULL, j & 1);
                if (!ok) break;
                tc_fence_after();
                const int kslot = (2 * j) % C::NSLOT;
                const uint64_t dkmn = dkmn0 + ((kslot * C::NTILE_BYTES) >> 4);
                const uint32_t ts = tmem_base + ((j & 1) ? C::TM_S2 : C::TM_S);
#pragma unroll
                for (int kk = 0; kk < C::BN / 16; ++kk)  // dq += dS K
                    mma_bf16_ts(tmem_base + C::TM_ACC0, ts + pcol<C::BN>(kk),
                                dkmn + ((kk * 16 * 128) >> 4), idesc_acc, (j > 0 || kk > 0) ? 1u : 0u);
                mma_commit(bar(L::B_SLOT_EMPTY + kslot));  // K(j) consumed
                // dP(j + 1) overwrites dP(j), read before dS(j) was signalled;
                // S(j + 2) overwrites dS(j), issued after the MMAs reading it.
                if (j + 1 < n) ok = issue_dp(j + 1);
                if (ok && j + 2 < n) ok = issue_s(j + 2);
            }
            if (ok) mma_commit(bar(L::B_ACC_FULL));
            mma_commit(bar(L::B_DRAIN));
            drain_wait(bar(L::B_DRAIN), 0);
        }
        __syncwarp();
    } else if (warp < 8) {
        const int h = warp >> 2;  // column half
        const int wq = warp & 3;
        const int row = wq * 32 + lane;
        const int i = it.q0 + row;
        const int s_doc = it.doc_start;
        const int r_lo = it.q0 > s_doc ? it.q0 : s_doc;
        const int r_hi = it.q1 - 1;
        const bool row_valid = i >= r_lo && i <= r_hi;
        const int W = prm.window;
        // Visible keys of this row: [lo_i, i]; none for rows outside the
        // document.
        int lo_i = (W > 0 && i - W + 1 > s_doc) ? i - W + 1 : s_doc;
        if (!row_valid) lo_i = i + 1;
        const int hq = it.head0;
        const float lse2 = row_valid ? prm.lse[static_cast<int64_t>(i) * prm.Hq + hq] * kLog2e : 0.0f;
        const float Di = row_valid ? prm.delta[static_cast<int64_t>(i) * prm.Hq + hq] : 0.0f;
        const float sl2 = prm.scale_log2;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(wq * 32) << 16);

        bool ok = !skip;
        for (int j = 0; ok && j < n; ++j) {
            ok = warp_wait(bar(L::B_S_FULL + (j & 1)), (j >> 1) & 1, abort_flag, prm.status);
            if (!ok) break;
            tc_fence_after();
            const uint32_t tm_s = (j & 1) ? C::TM_S2 : C::TM_S;
            constexpr int HALF = C::HALF;
            const int kh = it.kv_start + j * C::BN + HALF * h;  // first key of this half
            const bool full = row_valid && kh >= s_doc && kh + HALF - 1 <= r_lo &&
                              (W == 0 || kh >= r_hi - W + 1);
            const int c_lo = lo_i - kh, c_hi = i - kh;  // visible columns of the half
            // P of this half (HALF values) while the tensor core computes dP.
            float pv[HALF];
            {
                uint32_t sr[HALF];
#pragma unroll
                for (int cc = 0; cc < HALF / 32; ++cc)
                    tmem_ld32(lane_base + tm_s + HALF * h + 32 * cc,
                              *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * cc]));
                tmem_wait_ld();
#pragma unroll
                for (int cc = 0; cc < HALF / 32; ++cc)
                    reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&sr[32 * cc]));
#pragma unroll
                for (int c = 0; c < HALF; ++c) {
                    const float x = ex2_approx(fmaf(__uint_as_float(sr[c]), sl2, -lse2));
                    pv[c] = (full || (c >= c_lo && c <= c_hi)) ? x : 0.0f;
                }
            }
            ok = warp_wait(bar(L::B_DP_FULL), j & 1, abort_flag, prm.status);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int cc = 0; cc < HALF / 32; ++cc) {
                uint32_t dr[32];
                tmem_ld32(lane_base + C::TM_DP + HALF * h + 32 * cc, dr);
                tmem_wait_ld();
                reg_fence32(dr);
                uint32_t pk[16];
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    pk[u] = pack_bf16x2(pv[32 * cc + 2 * u] * (__uint_as_float(dr[2 * u]) - Di),
                                        pv[32 * cc + 2 * u + 1] * (__uint_as_float(dr[2 * u + 1]) - Di));
                // dS of this half's columns [32 cc, 32 cc + 32) goes to TMEM
                // columns HALF h + [16 cc, 16 cc + 16) (S of this half, read).
                tmem_st16(lane_base + tm_s + HALF * h + 16 * cc, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(L::B_DS_FULL));
        }
        if (ok) ok = warp_wait(bar(L::B_ACC_FULL), 0, abort_flag, prm.status);
        if (ok) {
            tc_fence_after();
            // Half h stores dq columns [h D / 2, (h + 1) D / 2).
            constexpr int HC = C::D / 2;
            __nv_bfloat16* orow = prm.dq + (static_cast<int64_t>(i) * prm.Hq + hq) * C::D + h * HC;
#pragma unroll 1
            for (int c = 0; c < HC / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(lane_base + C::TM_ACC0 + h * HC + c * 32, r);
                tmem_wait_ld();
                reg_fence32(r);
                uint32_t w[16];
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    w[u] = pack_bf16x2(__uint_as_float(r[2 * u]) * prm.scale,
                                       __uint_as_float(r[2 * u + 1]) * prm.scale);
                if (row_valid) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        dst[u] = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == C::MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------- dk, dv ----
template <class C>
struct DkvLayout {
    // Q tiles (with their lse / delta values) and dO tiles have rings of
    // their own: step s uses Q slot s % NQS and dO slot s % NDS; a slot is
    // released after the last product that reads it.
    static constexpr int NQS = C::NSLOT;
    static constexpr int NDS = C::NDSLOT;
    static constexpr int B_KV_FULL = 0;                    // K and V landed
    static constexpr int B_Q_FULL = 1;                     // [NQS] Q tile, lse, delta
    static constexpr int B_Q_EMPTY = B_Q_FULL + NQS;       // [NQS]
    static constexpr int B_DO_FULL = B_Q_EMPTY + NQS;      // [NDS] dO tile
    static constexpr int B_DO_EMPTY = B_DO_FULL + NDS;     // [NDS]
    // Score buffers: with one accumulator and 64-column score tiles, two
    // S^T (and two dP^T) buffers fit in TMEM beside it; step s uses buffer
    // s % NB.  The scores of step s + NB need Q(s + NB) while Q(s) is still
    // in use, so two buffers want a third Q slot.
    static constexpr int NB = C::NBUF;
    static_assert(NB == 1 || (NB == 2 && C::MODE != kDkDv && C::BN == 64 && NQS >= 3),
                  "two score buffers: one accumulator, 64-column tiles, three Q slots");
    static_assert(C::TM_S + NB * C::BN <= C::TM_DP && C::TM_DP + NB * C::BN <= C::TM_ACC0,
                  "score buffers overlap");
    static constexpr int B_S_FULL = B_DO_EMPTY + NDS;      // [NB] S^T done
    static constexpr int B_DP_FULL = B_S_FULL + NB;           // [NB] dP^T done
    static constexpr int B_P_READY = B_DP_FULL + NB;          // [NB] P^T in TMEM (8 warps)
    static constexpr int B_DS_READY = B_P_READY + NB;         // [NB] dS^T in TMEM (8 warps)
    static constexpr int B_ACC_FULL = B_DS_READY + NB;        // dk, dv accumulated
    static constexpr int B_DRAIN = B_ACC_FULL + 1;
    static constexpr int NUM_BARS = B_DRAIN + 1;
    static constexpr int SMEM_K = 0;
    static constexpr int SMEM_V = SMEM_K + C::TILE_BYTES;
    static_assert(C::MODE != kDkDv || C::TM_ACC1 + C::D <= 512, "dk and dv together exceed TMEM");
    static constexpr int V_BYTES = C::MODE == kDvOnly ? 0 : C::TILE_BYTES;  // dv alone needs no V
    static constexpr int SMEM_Q = SMEM_V + V_BYTES;               // [NQS] Q tiles of BN rows
    static constexpr int SMEM_DO = SMEM_Q + NQS * C::NTILE_BYTES;  // [NDS] dO tiles of BN rows
    static constexpr int SMEM_SIDE = SMEM_DO + NDS * C::NTILE_BYTES;  // [NQS][lse2 BN, delta BN]
    static constexpr int SIDE_BYTES = 2 * C::BN * 4;
    static constexpr int SMEM_BAR = SMEM_SIDE + NQS * SIDE_BYTES;
    static constexpr int SMEM_TMEM_SLOT = SMEM_BAR + NUM_BARS * 8;
    static constexpr int SMEM_ABORT = SMEM_TMEM_SLOT + 4;
    static constexpr int SMEM_ALLOC = SMEM_ABORT + 4 + 1024;
    static_assert(SMEM_ALLOC <= 232448, "shared memory budget exceeded");
};

template <class C>
__global__ void __launch_bounds__(C::NUM_THREADS, 1)
thd_attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmap_q,
                         const __grid_constant__ CUtensorMap tmap_do,
                         const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v, const BwdParams prm) {
    using L = DkvLayout<C>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
    const uint32_t sbase = smem_addr(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const BwdKVItem it = prm.kv_items[blockIdx.x];
    const int G = prm.G;
    const int nsub = it.n_q * (128 / C::BN);  // query tiles of BN rows per head
    const int n_steps = G * nsub;             // (query head, query tile) steps
    constexpr bool kDv = C::MODE != kDkOnly;  // accumulates dv
    constexpr bool kDk = C::MODE != kDvOnly;  // accumulates dk

    auto bar = [&](int idx) -> uint32_t { return sbase + L::SMEM_BAR + 8u * idx; };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::SMEM_ABORT);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::SMEM_TMEM_SLOT);
    float* side = reinterpret_cast<float*>(smem + L::SMEM_SIDE);

    if (threadIdx.x == 0) {
        mbar_init(bar(L::B_KV_FULL), 1);
        for (int s = 0; s < L::NQS; ++s) {
            mbar_init(bar(L::B_Q_FULL + s), 2);  // TMA bytes + the side values
            mbar_init(bar(L::B_Q_EMPTY + s), 1);
        }
        for (int s = 0; s < L::NDS; ++s) {
            mbar_init(bar(L::B_DO_FULL + s), 1);
            mbar_init(bar(L::B_DO_EMPTY + s), 1);
        }
        for (int b = 0; b < L::NB; ++b) {
            mbar_init(bar(L::B_S_FULL + b), 1);
            mbar_init(bar(L::B_DP_FULL + b), 1);
            mbar_init(bar(L::B_P_READY + b), 8);
            mbar_init(bar(L::B_DS_READY + b), 8);
        }
        mbar_init(bar(L::B_ACC_FULL), 1);
        mbar_init(bar(L::B_DRAIN), 1);
        *abort_flag = *reinterpret_cast<volatile int*>(prm.status) != 0 ? 1 : 0;
        fence_barrier_init();
    }
    if (warp == C::MMA_WARP) {
        tmem_alloc(smem_addr(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const bool skip = *abort_flag != 0;

    if (warp == C::PRODUCER_WARP) {
        // All 32 lanes stage the per-query lse / delta values; lane 0 issues
        // the copies.
        bool ok = !skip;
        int issued = 0;     // steps whose Q copies were issued
        int issued_do = 0;  // steps whose dO copies were issued
        if (ok && lane == 0) {
            tma_prefetch_desc(&tmap_q);
            tma_prefetch_desc(&tmap_do);
            tma_prefetch_desc(&tmap_k);
            tma_prefetch_desc(&tmap_v);
            mbar_arrive_expect_tx(bar(L::B_KV_FULL), (kDk ? 2 : 1) * C::TILE_BYTES);
            for (int c = 0; c < C::KCH; ++c) {
                tma_load_3d(sbase + L::SMEM_K + c * C::BOX_BYTES, &tmap_k, bar(L::B_KV_FULL), c * 64,
                            it.g, it.k0);
                if (kDk)
                    tma_load_3d(sbase + L::SMEM_V + c * C::BOX_BYTES, &tmap_v, bar(L::B_KV_FULL),
                                c * 64, it.g, it.k0);
            }
        }
        for (int s = 0; ok && s < n_steps; ++s) {
            const int qs = s % L::NQS, ds = s % L::NDS;
            const int h = it.g * G + s / nsub;
            const int i0 = it.k0 + (s % nsub) * C::BN;
            ok = warp_wait(bar(L::B_Q_EMPTY + qs), ((s / L::NQS) & 1) ^ 1, abort_flag, prm.status);
            if (!ok) break;
            if (lane == 0) {
                const uint32_t full = bar(L::B_Q_FULL + qs);
                const uint32_t dst = sbase + L::SMEM_Q + qs * C::NTILE_BYTES;
                mbar_arrive_expect_tx(full, C::NTILE_BYTES);
                for (int c = 0; c < C::KCH; ++c)
                    tma_load_3d(dst + c * C::NBOX_BYTES, &tmap_q, full, c * 64, h, i0);
            }
            float* sd = side + qs * 2 * C::BN;
#pragma unroll
            for (int u = 0; u < C::BN / 32; ++u) {
                const int col = lane * (C::BN / 32) + u;
                const int64_t i = static_cast<int64_t>(i0) + col;
                const bool in = i < prm.T;
                sd[col] = in ? prm.lse[i * prm.Hq + h] * kLog2e : 0.0f;
                sd[C::BN + col] = in ? prm.delta[i * prm.Hq + h] : 0.0f;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(L::B_Q_FULL + qs));
            issued = s + 1;
            ok = warp_wait(bar(L::B_DO_EMPTY + ds), ((s / L::NDS) & 1) ^ 1, abort_flag, prm.status);
            if (!ok) break;
            if (lane == 0) {
                const uint32_t full = bar(L::B_DO_FULL + ds);
                const uint32_t dst = sbase + L::SMEM_DO + ds * C::NTILE_BYTES;
                mbar_arrive_expect_tx(full, C::NTILE_BYTES);
                for (int c = 0; c < C::KCH; ++c)
                    tma_load_3d(dst + c * C::NBOX_BYTES, &tmap_do, full, c * 64, h, i0);
            }
            issued_do = s + 1;
        }
        if (!ok && !skip && lane == 0) {
            // Unwinding: let the copies already issued land before exit
            // (only the last ones into each slot can still be in flight).
            drain_wait(bar(L::B_KV_FULL), 0);
            for (int s = issued - L::NQS > 0 ? issued - L::NQS : 0; s < issued; ++s)
                drain_wait(bar(L::B_Q_FULL + s % L::NQS), (s / L::NQS) & 1);
            for (int s = issued_do - L::NDS > 0 ? issued_do - L::NDS : 0; s < issued_do; ++s)
                drain_wait(bar(L::B_DO_FULL + s % L::NDS), (s / L::NDS) & 1);
        }
        __syncwarp();
    } else if (warp == C::MMA_WARP) {
        if (lane == 0 && !skip) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, C::BN, false);
            constexpr uint32_t idesc_acc = idesc_bf16_f32(128, C::D, true);
            const uint64_t dk0 = smem_desc_sw128(sbase + L::SMEM_K, 16, 1024);
            const uint64_t dv0 = smem_desc_sw128(sbase + L::SMEM_V, 16, 1024);
            const uint64_t dq0 = smem_desc_sw128(sbase + L::SMEM_Q, 16, 1024);
            const uint64_t dqmn0 = smem_desc_sw128(sbase + L::SMEM_Q, C::NBOX_BYTES, 1024);
            const uint64_t ddo0 = smem_desc_sw128(sbase + L::SMEM_DO, 16, 1024);
            const uint64_t ddomn0 = smem_desc_sw128(sbase + L::SMEM_DO, C::NBOX_BYTES, 1024);
            auto wait = [&](int idx, uint32_t parity) -> bool {
                return mbar_wait(bar(idx), parity, abort_flag, prm.status, kStatusTimeout);
            };
            bool ok = wait(L::B_KV_FULL, 0);
            auto issue_st = [&](int s) {  // S^T(s) = K Q(s)^T
                const uint32_t qoff = ((s % L::NQS) * C::NTILE_BYTES) >> 4;
#pragma unroll
                for (int kk = 0; kk < C::D / 16; ++kk) {
                    const uint32_t o = ((kk >> 2) * C::BOX_BYTES + (kk & 3) * 32) >> 4;
                    const uint32_t on = ((kk >> 2) * C::NBOX_BYTES + (kk & 3) * 32) >> 4;
                    mma_bf16_ss(tmem_base + C::TM_S + C::BN * (s % L::NB), dk0 + o, dq0 + qoff + on, idesc_s,
                                kk > 0 ? 1u : 0u);
                }
            };
            auto issue_dpt = [&](int s) {  // dP^T(s) = V dO(s)^T
                const uint32_t dooff = ((s % L::NDS) * C::NTILE_BYTES) >> 4;
#pragma unroll
                for (int kk = 0; kk < C::D / 16; ++kk) {
                    const uint32_t o = ((kk >> 2) * C::BOX_BYTES + (kk & 3) * 32) >> 4;
                    const uint32_t on = ((kk >> 2) * C::NBOX_BYTES + (kk & 3) * 32) >> 4;
                    mma_bf16_ss(tmem_base + C::TM_DP + C::BN * (s % L::NB), dv0 + o, ddo0 + dooff + on, idesc_s,
                                kk > 0 ? 1u : 0u);
                }
            };
            if constexpr (C::MODE == kDkDv) {
                // Order dv(s) S^T(s+1) dk(s) dP^T(s+1): S^T(s+1) overwrites
                // P^T(s) only after dv(s) and dP^T(s+1) overwrites dS^T(s)
                // only after dk(s) (in-order tensor pipe), so the tensor core
                // works on S^T(s+1) while dS^T(s) is formed and on dk(s) and
                // dP^T(s+1) while P^T(s+1) is: each elementwise phase runs
                // under two products instead of one.
                if (ok && n_steps > 0) {
                    ok = wait(L::B_Q_FULL + 0, 0);
                    if (ok) {
                        tc_fence_after();
                        issue_st(0);
                        mma_commit(bar(L::B_S_FULL));
                        ok = wait(L::B_DO_FULL + 0, 0);
                    }
                    if (ok) {
                        tc_fence_after();
                        issue_dpt(0);
                        mma_commit(bar(L::B_DP_FULL));
                    }
                }
                for (int s = 0; ok && s < n_steps; ++s) {
                    const int qs = s % L::NQS, ds = s % L::NDS;
                    const uint32_t qoff = (qs * C::NTILE_BYTES) >> 4;
                    const uint32_t dooff = (ds * C::NTILE_BYTES) >> 4;
                    const bool more = s + 1 < n_steps;
                    ok = wait(L::B_P_READY, s & 1);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < C::BN / 16; ++kk)  // dv += P^T dO
                        mma_bf16_ts(tmem_base + C::TM_ACC0, tmem_base + C::TM_S + pcol<C::BN>(kk),
                                    ddomn0 + dooff + ((kk * 16 * 128) >> 4), idesc_acc,
                                    (s > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(bar(L::B_DO_EMPTY + ds));  // dO(s) done
                    if (more) {
                        ok = wait(L::B_Q_FULL + (s + 1) % L::NQS, ((s + 1) / L::NQS) & 1);
                        if (!ok) break;
                        tc_fence_after();
                        issue_st(s + 1);
                        mma_commit(bar(L::B_S_FULL));
                    }
                    ok = wait(L::B_DS_READY, s & 1);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < C::BN / 16; ++kk)  // dk += dS^T Q
                        mma_bf16_ts(tmem_base + C::TM_ACC1, tmem_base + C::TM_DP + pcol<C::BN>(kk),
                                    dqmn0 + qoff + ((kk * 16 * 128) >> 4), idesc_acc,
                                    (s > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(bar(L::B_Q_EMPTY + qs));  // Q(s) done
                    if (more) {
                        ok = wait(L::B_DO_FULL + (s + 1) % L::NDS, ((s + 1) / L::NDS) & 1);
                        if (!ok) break;
                        tc_fence_after();
                        issue_dpt(s + 1);
                        mma_commit(bar(L::B_DP_FULL));
                    }
                }
            }
            if constexpr (C::MODE != kDkDv) {
                // One accumulator: S^T(s + NB) (and dP^T(s + NB)) go out after
                // the product of step s that reads the buffer they
                // overwrite, so with two buffers the next step's scores are
                // computed while this step's elementwise work runs.
                auto issue_scores = [&](int s) -> bool {
                    if (!wait(L::B_Q_FULL + s % L::NQS, (s / L::NQS) & 1)) return false;
                    tc_fence_after();
                    issue_st(s);
                    mma_commit(bar(L::B_S_FULL + s % L::NB));
                    if constexpr (kDk) {
                        if (!wait(L::B_DO_FULL + s % L::NDS, (s / L::NDS) & 1)) return false;
                        tc_fence_after();
                        issue_dpt(s);
                        mma_commit(bar(L::B_DP_FULL + s % L::NB));
                        mma_commit(bar(L::B_DO_EMPTY + s % L::NDS));  // dO(s) read by dP^T only
                    }
                    return true;
                };
                for (int j = 0; ok && j < L::NB && j < n_steps; ++j) ok = issue_scores(j);
                for (int s = 0; ok && s < n_steps; ++s) {
                    const int qs = s % L::NQS, ds = s % L::NDS, b = s % L::NB;
                    const uint32_t ph = (s / L::NB) & 1;
                    if constexpr (kDv) {
                        ok = wait(L::B_DO_FULL + ds, (s / L::NDS) & 1) && wait(L::B_P_READY + b, ph);
                        if (!ok) break;
                        tc_fence_after();
                        const uint32_t dooff = (ds * C::NTILE_BYTES) >> 4;
#pragma unroll
                        for (int kk = 0; kk < C::BN / 16; ++kk)  // dv += P^T dO
                            mma_bf16_ts(tmem_base + C::TM_ACC0,
                                        tmem_base + C::TM_S + C::BN * b + pcol<C::BN>(kk),
                                        ddomn0 + dooff + ((kk * 16 * 128) >> 4), idesc_acc,
                                        (s > 0 || kk > 0) ? 1u : 0u);
                        mma_commit(bar(L::B_DO_EMPTY + ds));  // dO(s) done
                        // Q(s)'s slot also holds the lse / delta values the
                        // elementwise warps read before P_READY.
                        mma_commit(bar(L::B_Q_EMPTY + qs));
                    } else {
                        ok = wait(L::B_DS_READY + b, ph);
                        if (!ok) break;
                        tc_fence_after();
                        const uint32_t qoff = (qs * C::NTILE_BYTES) >> 4;
#pragma unroll
                        for (int kk = 0; kk < C::BN / 16; ++kk)  // dk += dS^T Q
                            mma_bf16_ts(tmem_base + C::TM_ACC1,
                                        tmem_base + C::TM_DP + C::BN * b + pcol<C::BN>(kk),
                                        dqmn0 + qoff + ((kk * 16 * 128) >> 4), idesc_acc,
                                        (s > 0 || kk > 0) ? 1u : 0u);
                        mma_commit(bar(L::B_Q_EMPTY + qs));  // Q(s) done
                    }
                    if (s + L::NB < n_steps) ok = issue_scores(s + L::NB);
                }
            }
            if (ok) mma_commit(bar(L::B_ACC_FULL));
            mma_commit(bar(L::B_DRAIN));
            drain_wait(bar(L::B_DRAIN), 0);
        }
        __syncwarp();
    } else if (warp < 8) {
        const int h = warp >> 2;  // column half
        const int wq = warp & 3;
        const int row = wq * 32 + lane;
        const int j = it.k0 + row;  // key of this TMEM lane
        const int e_doc = it.doc_end;
        const bool row_valid = j < e_doc;
        const int W = prm.window;
        const float sl2 = prm.scale_log2;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(wq * 32) << 16);
        const int k_last = it.k0 + 127 < e_doc - 1 ? it.k0 + 127 : e_doc - 1;
        // Queries that see key j: [j, i_hi]; none for keys past the document.
        int i_hi = e_doc - 1;
        if (W > 0 && j + W - 1 < i_hi) i_hi = j + W - 1;
        if (!row_valid) i_hi = j - 1;

        bool ok = !skip;
        constexpr int HALF = C::HALF;
        for (int s = 0; ok && s < n_steps; ++s) {
            const int qs = s % L::NQS;
            const int ih = it.k0 + (s % nsub) * C::BN + HALF * h;  // first query of this half
            // The side values of this step were stored before Q_FULL.
            const int b = s % L::NB;
            const uint32_t ph = (s / L::NB) & 1;
            const uint32_t tm_s = C::TM_S + C::BN * b, tm_dp = C::TM_DP + C::BN * b;
            ok = warp_wait(bar(L::B_Q_FULL + qs), (s / L::NQS) & 1, abort_flag, prm.status) &&
                 warp_wait(bar(L::B_S_FULL + b), ph, abort_flag, prm.status);
            if (!ok) break;
            tc_fence_after();
            const float* lse2 = side + qs * 2 * C::BN + HALF * h;
            const float* dlt = side + qs * 2 * C::BN + C::BN + HALF * h;
            // Every (key, query) of this half visible: its queries after every
            // key, inside the document and inside every key's window.
            const bool full = ih >= k_last && ih + HALF - 1 < e_doc && it.k0 + 127 < e_doc &&
                              (W == 0 || ih + HALF - 1 - it.k0 < W);
            const int c_lo = j - ih, c_hi = i_hi - ih;  // visible columns of the half
            // P^T of this half (while the tensor core computes dP^T) ...
            float pv[HALF];
            {
                uint32_t sr[HALF];
#pragma unroll
                for (int cc = 0; cc < HALF / 32; ++cc)
                    tmem_ld32(lane_base + tm_s + HALF * h + 32 * cc,
                              *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * cc]));
                tmem_wait_ld();
#pragma unroll
                for (int cc = 0; cc < HALF / 32; ++cc)
                    reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&sr[32 * cc]));
#pragma unroll
                for (int u = 0; u < HALF / 4; ++u) {
                    const float4 l4 = *reinterpret_cast<const float4*>(lse2 + 4 * u);
                    const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int c = 4 * u + e;
                        const float x = ex2_approx(fmaf(__uint_as_float(sr[c]), sl2, -lv[e]));
                        pv[c] = (full || (c >= c_lo && c <= c_hi)) ? x : 0.0f;
                    }
                }
                if constexpr (kDv) {
                    uint32_t pp[HALF / 2];
#pragma unroll
                    for (int u = 0; u < HALF / 2; ++u) pp[u] = pack_bf16x2(pv[2 * u], pv[2 * u + 1]);
                    // Over this half's own first S^T columns, all read.
#pragma unroll
                    for (int cc = 0; cc < HALF / 32; ++cc)
                        tmem_st16(lane_base + tm_s + HALF * h + 16 * cc,
                                  *reinterpret_cast<uint32_t(*)[16]>(&pp[16 * cc]));
                }
            }
            if constexpr (kDv) {
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(L::B_P_READY + b));
            }
            if constexpr (kDk) {
                // ... then dS^T = P^T (dP^T - delta) while it computes dv.
                ok = warp_wait(bar(L::B_DP_FULL + b), ph, abort_flag, prm.status);
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int cc = 0; cc < HALF / 32; ++cc) {
                    uint32_t dr[32];
                    tmem_ld32(lane_base + tm_dp + HALF * h + 32 * cc, dr);
                    tmem_wait_ld();
                    reg_fence32(dr);
                    uint32_t pd[16];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const float4 d4 = *reinterpret_cast<const float4*>(dlt + 32 * cc + 4 * u);
                        const float dv4[4] = {d4.x, d4.y, d4.z, d4.w};
                        float dsv[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            dsv[e] = pv[32 * cc + 4 * u + e] * (__uint_as_float(dr[4 * u + e]) - dv4[e]);
                        pd[2 * u] = pack_bf16x2(dsv[0], dsv[1]);
                        pd[2 * u + 1] = pack_bf16x2(dsv[2], dsv[3]);
                    }
                    // Over dP^T columns HALF h + [16 cc, 16 cc + 16), already read.
                    tmem_st16(lane_base + tm_dp + HALF * h + 16 * cc, pd);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(L::B_DS_READY + b));
            }
        }
        if (ok) ok = warp_wait(bar(L::B_ACC_FULL), 0, abort_flag, prm.status);
        if (ok && C::MODE != kDkDv) {
            // One accumulator (dv, or dk times the score scale); half h stores
            // its columns [h D / 2, (h + 1) D / 2).
            tc_fence_after();
            constexpr int HC = C::D / 2;
            __nv_bfloat16* dst_row = (kDv ? prm.dv : prm.dk) +
                                     (static_cast<int64_t>(j) * prm.Hkv + it.g) * C::D + h * HC;
            const float f = kDv ? 1.0f : prm.scale;
            const uint32_t acc = lane_base + (kDv ? C::TM_ACC0 : C::TM_ACC1) + h * HC;
#pragma unroll 1
            for (int c = 0; c < HC / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(acc + c * 32, r);
                tmem_wait_ld();
                reg_fence32(r);
                uint32_t w[16];
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    w[u] = pack_bf16x2(__uint_as_float(r[2 * u]) * f, __uint_as_float(r[2 * u + 1]) * f);
                if (row_valid) {
                    uint4* dst = reinterpret_cast<uint4*>(dst_row + c * 32);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        dst[u] = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
                }
            }
        } else if (ok) {
            tc_fence_after();
            // Half 0 stores dv, half 1 stores dk (times the score scale).
            __nv_bfloat16* dst_row = (h == 0 ? prm.dv : prm.dk) +
                                     (static_cast<int64_t>(j) * prm.Hkv + it.g) * C::D;
            const float f = h == 0 ? 1.0f : prm.scale;
            const uint32_t acc = lane_base + (h == 0 ? C::TM_ACC0 : C::TM_ACC1);
#pragma unroll 1
            for (int c = 0; c < C::D / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(acc + c * 32, r);
                tmem_wait_ld();
                reg_fence32(r);
                uint32_t w[16];
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    w[u] = pack_bf16x2(__uint_as_float(r[2 * u]) * f, __uint_as_float(r[2 * u + 1]) * f);
                if (row_valid) {
                    uint4* dst = reinterpret_cast<uint4*>(dst_row + c * 32);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        dst[u] = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == C::MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace thd
