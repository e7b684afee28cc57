// Packed-THD sliding-window GQA attention forward on CTA pairs with the
// softmax of every key tile split between two warpgroups (B200, sm_100a).
//
// Same computation as thd_attn_kernel.cuh (one work item = one 128-row query
// tile of one document for query heads that share one kv head; see that file
// for the masking and softmax readings of the API pages), organised so that
// the tensor core and the exponential unit can both stay busy:
//
// * Two CTAs (one cluster) share every tensor-core instruction: the leader
//   (rank 0) issues tcgen05.mma.cta_group::2 with M = 256, i.e. the same 128
//   query rows of one head in each CTA (two heads of one kv group per item).
//   Each CTA loads half of every K tile (half the keys: B of S = Q K^T is
//   split along N) and half of every V tile (half the head dim: B of
//   O += P V is split along N).
// * S has NSB buffers in TMEM: S(j+1) .. S(j+NSB-1) = Q K^T run while the
//   softmax works on tile j.  P (bf16) is written back into S(j) and read by
//   O += P V straight from TMEM.
// * Two softmax warpgroups share every tile: warpgroup h owns keys
//   [64h, 64h + 64) of the tile (TMEM columns [64h, 64h + 64) of S; its P
//   goes to columns [64h, 64h + 32)), so each thread handles 64 scores per
//   row.  The halves exchange their partial row maxima through shared memory
//   once per tile, so both apply the same running max to the one O, and each
//   rescales / stores half of its columns.  At head dim 256 the tensor core
//   needs twice the time of the exponentials per tile, which leaves room for
//   that exchange; at head dim 128 the two are equal and the one-CTA kernel
//   (thd_attn_kernel.cuh) is faster.
//
// Warps: 0-3 softmax half 0, 4-7 softmax half 1, 8 TMA producer (this CTA's
// halves of K/V), 9 MMA issuer (leader only), 10-11 idle.  Synchronisation:
//   * TMA loads of both CTAs complete on the LEADER's Q / slot barriers;
//   * MMA completion is committed to the same barrier in both CTAs (S ready,
//     O ready, slot free);
//   * the softmax warps of both CTAs arrive on the LEADER's P barrier;
//   * the two softmax halves of a CTA meet on a local exchange barrier.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "sm100_ptx.cuh"
#include "thd_attn_kernel.cuh"

// Element pairs (out of every 4) whose exponential runs on the FMA pipe
// (fit_exp2_poly.py) instead of MUFU.  At head dim 256 the exponential unit
// has slack, but moving a quarter of the work off it still measured ~1.5%
// faster.
#ifndef THD_SPLIT_EXP_EMU
#define THD_SPLIT_EXP_EMU 1
#endif

namespace thd {

template <int D_, int NSB_, int NSLOT_>
struct SplitConfig {
    static constexpr int D = D_;
    static constexpr int BN = 128;        // keys per key tile
    static constexpr int NSB = NSB_;      // S buffers in TMEM
    static constexpr int NSLOT = NSLOT_;  // ring slots (one K half or V half each)
    static constexpr int BM = 128;        // query rows per CTA (M = 256 per pair)
    static constexpr int HALF = BN / 2;   // keys per softmax warpgroup
    static constexpr int EXP_EMU = THD_SPLIT_EXP_EMU;

    static constexpr int KCH = D / 64;                  // 128-byte column chunks of a Q row
    static constexpr int Q_BOX_BYTES = BM * 128;
    static constexpr int Q_TILE_BYTES = BM * D * 2;
    static constexpr int KH_ROWS = BN / 2;              // keys of a K half
    static constexpr int KH_BOX_BYTES = KH_ROWS * 128;  // one 64-column chunk of a K half
    static constexpr int VH_COLS = D / 2;               // head-dim columns of a V half
    static constexpr int VH_CH = VH_COLS / 64;          // chunks of a V half
    static constexpr int VH_BOX_BYTES = BN * 128;       // one chunk of a V half
    static constexpr int SLOT_BYTES = BN * D;           // = K half bytes = V half bytes

    static constexpr int TMEM_S = 0;                    // S[b] at b*BN, b < NSB
    static constexpr int TMEM_O = NSB * BN;
    static constexpr int TMEM_USED = TMEM_O + D;
    static constexpr int TMEM_COLS = 512;

    static constexpr int PRODUCER_WARP = 8;
    static constexpr int MMA_WARP = 9;
    static constexpr int NUM_THREADS = 12 * 32;

    static constexpr int B_Q_FULL = 0;                          // leader: both CTAs' Q landed
    static constexpr int B_SLOT_FULL = 1;                       // leader: both halves landed
    static constexpr int B_SLOT_EMPTY = B_SLOT_FULL + NSLOT;    // both: slot may be refilled
    static constexpr int B_S_FULL = B_SLOT_EMPTY + NSLOT;       // both: S[b] = Q K^T done [NSB]
    static constexpr int B_P_FULL = B_S_FULL + NSB;             // leader: P written in both CTAs
    static constexpr int B_O_FULL = B_P_FULL + 1;               // both: PV done
    static constexpr int B_XCH = B_O_FULL + 1;                  // local: softmax halves met
    static constexpr int B_DRAIN = B_XCH + 1;
    static constexpr int NUM_BARS = B_DRAIN + 1;

    static constexpr int SMEM_Q = 0;
    static constexpr int SMEM_SLOTS = SMEM_Q + Q_TILE_BYTES;
    static constexpr int SMEM_XMAX = SMEM_SLOTS + NSLOT * SLOT_BYTES;  // float [2][2][BM]
    static constexpr int SMEM_XL = SMEM_XMAX + 2 * 2 * BM * 4;         // float [2][BM]
    static constexpr int SMEM_BAR = SMEM_XL + 2 * BM * 4;
    static constexpr int SMEM_TMEM_SLOT = SMEM_BAR + NUM_BARS * 8;
    static constexpr int SMEM_ABORT = SMEM_TMEM_SLOT + 4;
    static constexpr int SMEM_BYTES = SMEM_ABORT + 4;
    static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;

    static_assert(D == 128 || D == 256, "split pair kernel: head dim 128 or 256");
    static_assert(NSB == 2 || NSB == 3, "two or three S buffers");
    static_assert(TMEM_USED <= 512, "TMEM budget exceeded");
    static_assert(SMEM_ALLOC <= 232448, "shared memory budget exceeded");
    // Every wait of the MMA issuer is for a ring position whose slot was
    // released by an MMA it has already issued (issue order QK(0) .. QK(NSB-1),
    // then per tile j: PV(j), QK(j+NSB); V(j) is released after PV(j), K(j) after
    // QK(j)), so two slots cannot deadlock.
    static_assert(NSLOT >= 2, "ring needs two slots");
};

template <class C>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(C::NUM_THREADS, 1)
thd_attn_fwd_split_kernel(const __grid_constant__ CUtensorMap tmap_q,
                          const __grid_constant__ CUtensorMap tmap_k,
                          const __grid_constant__ CUtensorMap tmap_v,
                          const FwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
    const uint32_t sbase = smem_addr(smem);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const WorkItem it = p.items[blockIdx.x >> 1];
    const int n = it.n_kv;
    const int head = it.head0 + static_cast<int>(rank);  // this CTA's query head

    auto bar = [&](int idx) -> uint32_t { return sbase + C::SMEM_BAR + 8u * idx; };
    auto lead_bar = [&](int idx) -> uint32_t { return mapa_shared(bar(idx), 0); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::SMEM_ABORT);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SMEM_TMEM_SLOT);

    if (threadIdx.x == 0) {
        mbar_init(bar(C::B_Q_FULL), 1);
        for (int s = 0; s < C::NSLOT; ++s) {
            mbar_init(bar(C::B_SLOT_FULL + s), 1);
            mbar_init(bar(C::B_SLOT_EMPTY + s), 1);
        }
        for (int b = 0; b < C::NSB; ++b) mbar_init(bar(C::B_S_FULL + b), 1);
        mbar_init(bar(C::B_P_FULL), 16);  // the 8 softmax warps of each CTA
        mbar_init(bar(C::B_O_FULL), 1);
        mbar_init(bar(C::B_XCH), 8);  // the 8 softmax warps of this CTA
        mbar_init(bar(C::B_DRAIN), 1);
        *abort_flag = launch_should_skip(p) | debug_check_item(it, p, 2, C::BN);
        fence_barrier_init();
    }
    if (warp == C::MMA_WARP) {
        tmem_alloc_pair(smem_addr(tmem_slot), C::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers exist before anyone signals them
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const bool skip = *abort_flag != 0;

    if (warp == C::PRODUCER_WARP) {
        // ----------------------------------------- TMA producer (this CTA's half)
        if (lane == 0 && !skip) {
            tma_prefetch_desc(&tmap_q);
            tma_prefetch_desc(&tmap_k);
            tma_prefetch_desc(&tmap_v);
            const int g = it.head0 / p.G;
            if (leader) mbar_arrive_expect_tx(bar(C::B_Q_FULL), 2 * C::Q_TILE_BYTES);
            for (int c = 0; c < C::KCH; ++c)
                tma_load_3d_pair(sbase + C::SMEM_Q + c * C::Q_BOX_BYTES, &tmap_q,
                                 lead_bar(C::B_Q_FULL), c * 64, head, it.q0 - p.q_offset);
            // Ring positions: 2j holds K(j), 2j+1 holds V(j).  This CTA loads
            // keys [rank*BN/2, (rank+1)*BN/2) of K(j) and head-dim columns
            // [rank*D/2, (rank+1)*D/2) of V(j).
            bool ok = true;
            for (int pos = 0; pos < 2 * n && ok; ++pos) {
                const int slot = pos % C::NSLOT;
                ok = mbar_wait(bar(C::B_SLOT_EMPTY + slot), ((pos / C::NSLOT) & 1) ^ 1, abort_flag,
                               p.status, kStatusTimeout);
                if (!ok) break;
                if (leader) mbar_arrive_expect_tx(bar(C::B_SLOT_FULL + slot), 2 * C::SLOT_BYTES);
                const uint32_t full = lead_bar(C::B_SLOT_FULL + slot);
                const uint32_t dst = sbase + C::SMEM_SLOTS + slot * C::SLOT_BYTES;
                const int kt = it.kv_start + (pos >> 1) * C::BN;
                if ((pos & 1) == 0) {
                    for (int c = 0; c < C::KCH; ++c)
                        tma_load_3d_pair(dst + c * C::KH_BOX_BYTES, &tmap_k, full, c * 64, g,
                                         kt + static_cast<int>(rank) * C::KH_ROWS);
                } else {
                    for (int c = 0; c < C::VH_CH; ++c)
                        tma_load_3d_pair(dst + c * C::VH_BOX_BYTES, &tmap_v, full,
                                         static_cast<int>(rank) * C::VH_COLS + c * 64, g, kt);
                }
            }
            // On an abort, loads still in flight (they complete on the
            // leader's barriers, which this CTA cannot track) are given
            // 200 us to land before the pair reaches its closing barrier.
            if (!ok) spin_ns(200000);
        }
        __syncwarp();
    } else if (warp == C::MMA_WARP) {
        // ----------------------------------------------- MMA issuer (leader only)
        if (leader && lane == 0 && !skip) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(256, C::BN, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(256, C::D, true);
            const uint64_t dq = smem_desc_sw128(sbase + C::SMEM_Q, 16, 1024);
            const uint64_t dk0 = smem_desc_sw128(sbase + C::SMEM_SLOTS, 16, 1024);
            const uint64_t dv0 = smem_desc_sw128(sbase + C::SMEM_SLOTS, C::VH_BOX_BYTES, 1024);
            auto issue_qk = [&](int b, int slot) {
                const uint32_t d_tmem = tmem_base + C::TMEM_S + b * C::BN;
                const uint64_t dk = dk0 + ((slot * C::SLOT_BYTES) >> 4);
#pragma unroll
                for (int kk = 0; kk < C::D / 16; ++kk) {
                    const uint32_t qo = ((kk >> 2) * C::Q_BOX_BYTES + (kk & 3) * 32) >> 4;
                    const uint32_t ko = ((kk >> 2) * C::KH_BOX_BYTES + (kk & 3) * 32) >> 4;
                    mma2_bf16_ss(d_tmem, dq + qo, dk + ko, idesc_qk, kk > 0 ? 1u : 0u);
                }
            };
            // O += P V: the P of key half h sits in TMEM columns
            // [64h, 64h + 32) of S[b] (two keys per column); key k of the V
            // slot is its row k (128 bytes per row in each 64-column chunk).
            auto issue_pv = [&](int b, int slot, bool acc) {
                const uint32_t d_tmem = tmem_base + C::TMEM_O;
                const uint32_t p_tmem = tmem_base + C::TMEM_S + b * C::BN;
                const uint64_t dv = dv0 + ((slot * C::SLOT_BYTES) >> 4);
#pragma unroll
                for (int kk = 0; kk < C::BN / 16; ++kk)
                    mma2_bf16_ts(d_tmem, p_tmem + (kk >> 2) * C::HALF + (kk & 3) * 8,
                                 dv + ((kk * 16 * 128) >> 4), idesc_pv, (acc || kk > 0) ? 1u : 0u);
            };
            auto wait = [&](int idx, uint32_t parity) -> bool {
                return mbar_wait(bar(idx), parity, abort_flag, p.status, kStatusTimeout);
            };
            auto wait_slot = [&](int pos) -> bool {
                return wait(C::B_SLOT_FULL + pos % C::NSLOT, (pos / C::NSLOT) & 1);
            };

            bool ok = wait(C::B_Q_FULL, 0);
            for (int jj = 0; ok && jj < C::NSB && jj < n; ++jj) {
                ok = wait_slot(2 * jj);
                if (!ok) break;
                tc_fence_after();
                issue_qk(jj, (2 * jj) % C::NSLOT);
                mma2_commit_both(bar(C::B_S_FULL + jj));
                mma2_commit_both(bar(C::B_SLOT_EMPTY + (2 * jj) % C::NSLOT));
            }
            for (int j = 0; ok && j < n; ++j) {
                const int b = j % C::NSB;
                const int vslot = (2 * j + 1) % C::NSLOT;
                ok = wait_slot(2 * j + 1);
                if (!ok) break;
                ok = wait(C::B_P_FULL, j & 1);
                if (!ok) break;
                tc_fence_after();
                issue_pv(b, vslot, j > 0);
                mma2_commit_both(bar(C::B_O_FULL));
                mma2_commit_both(bar(C::B_SLOT_EMPTY + vslot));  // V(j) consumed
                const int jn = j + C::NSB;
                if (jn < n) {
                    // QK(j+NSB) overwrites S[b] (P(j)) only after PV(j) in
                    // issue order, which the tensor core keeps.
                    ok = wait_slot(2 * jn);
                    if (!ok) break;
                    tc_fence_after();
                    const int kslot = (2 * jn) % C::NSLOT;
                    issue_qk(b, kslot);
                    mma2_commit_both(bar(C::B_S_FULL + b));
                    mma2_commit_both(bar(C::B_SLOT_EMPTY + kslot));  // K(j+NSB) consumed
                }
            }
            mma2_commit_both(bar(C::B_DRAIN));
            drain_wait(bar(C::B_DRAIN), 0);
        }
        __syncwarp();
    } else if (warp < 8) {
        // ------------------------------------------------------------ softmax
        const int h = warp >> 2;  // key half of every tile
        const int wq = warp & 3;
        const int row = wq * 32 + lane;
        const int i = it.q0 + row;
        const int s_doc = it.doc_start;
        const int r_lo = it.q0 > s_doc ? it.q0 : s_doc;
        const int r_hi = it.q1 - 1;
        const bool row_valid = i >= r_lo && i <= r_hi;
        const int W = p.window;
        const int lo_i = (W > 0 && i - W + 1 > s_doc) ? i - W + 1 : s_doc;
        const float sl2 = p.scale_log2;
        constexpr float kTau = 8.0f;

        // The sink seeds the running max of both halves; its 2^0 = 1 joins
        // the sum of half 0 only.
        float m_ref = -INFINITY;
        float l = 0.0f;
        if (p.sinks != nullptr) {
            m_ref = p.sinks[head] * 1.4426950408889634f;
            l = h == 0 ? 1.0f : 0.0f;
        }
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(wq * 32) << 16);
        // This warp rescales and stores head-dim columns [h*D/2, (h+1)*D/2).
        constexpr int O_COLS = C::D / 2;
        const uint32_t o_tmem = lane_base + C::TMEM_O + h * O_COLS;
        const uint32_t p_full_leader = lead_bar(C::B_P_FULL);
        float* xmax = reinterpret_cast<float*>(smem + C::SMEM_XMAX);  // [2][2][BM]
        float* xl = reinterpret_cast<float*>(smem + C::SMEM_XL);      // [2][BM]

        bool ok = !skip;
        for (int j = 0; ok && j < n; ++j) {
            const int b = j % C::NSB;
            ok = warp_wait(bar(C::B_S_FULL + b), (j / C::NSB) & 1, abort_flag, p.status);
            if (!ok) break;
            tc_fence_after();
            const uint32_t s_tmem = lane_base + C::TMEM_S + b * C::BN + h * C::HALF;
            uint32_t sr[C::HALF];
#pragma unroll
            for (int c = 0; c < C::HALF / 32; ++c)
                tmem_ld32(s_tmem + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < C::HALF / 32; ++c)
                reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
            float sv[C::HALF];
#pragma unroll
            for (int c = 0; c < C::HALF; ++c) sv[c] = __uint_as_float(sr[c]);

            const int kh = it.kv_start + j * C::BN + h * C::HALF;  // first key of the half
            const bool full = kh >= s_doc && kh + C::HALF - 1 <= r_lo &&
                              (W == 0 || kh >= r_hi - W + 1);
            if (!full) {
                const int c_lo = lo_i - kh;
                const int c_hi = i - kh;
#pragma unroll
                for (int c = 0; c < C::HALF; ++c)
                    if (c < c_lo || c > c_hi) sv[c] = -INFINITY;
            }
            float mx[4] = {sv[0], sv[1], sv[2], sv[3]};
#pragma unroll
            for (int c = 4; c < C::HALF; c += 2)
                mx[(c >> 1) & 3] = max3f(mx[(c >> 1) & 3], sv[c], sv[c + 1]);
            float smax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            // Both halves must apply the same running max to O: exchange the
            // partial maxima (double-buffered by tile parity; a half can be at
            // most one tile ahead of the other).
            xmax[((j & 1) * 2 + h) * C::BM + row] = smax;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_XCH));
            ok = warp_wait(bar(C::B_XCH), j & 1, abort_flag, p.status);
            if (!ok) break;
            smax = fmaxf(smax, xmax[((j & 1) * 2 + (1 - h)) * C::BM + row]);
            const float m_tile = smax * sl2;

            float alpha = 1.0f;
            bool rescale_o = false;
            if (j == 0) {
                if (m_tile > m_ref) {
                    alpha = ex2_approx(m_ref - m_tile);
                    m_ref = m_tile;
                }
            } else if (m_tile > m_ref + kTau) {
                alpha = ex2_approx(m_ref - m_tile);
                m_ref = m_tile;
                rescale_o = true;
            }
            l *= alpha;
            const float neg_m = (m_ref == -INFINITY) ? 0.0f : -m_ref;

            // P for this half's 64 keys over the first 32 columns of its S half.
            const float2 sl2x2 = make_float2(sl2, sl2);
            const float2 negm2 = make_float2(neg_m, neg_m);
            float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
            exp_and_store_p<0, C::HALF / 32, C::HALF, C::EXP_EMU>(sv, sl2x2, negm2, s_tmem, acc0,
                                                                 acc1);
            l += (acc0.x + acc0.y) + (acc1.x + acc1.y);

            // PV(j-1) must be done before O is rescaled and before PV(j)
            // (waited every tile, which also keeps the O barrier's phases in
            // step with this warp).
            if (j > 0) {
                ok = warp_wait(bar(C::B_O_FULL), (j - 1) & 1, abort_flag, p.status);
                if (!ok) break;
                tc_fence_after();
                if (__any_sync(0xffffffffu, rescale_o)) {
#pragma unroll 1
                    for (int c = 0; c < O_COLS / 32; ++c) {
                        uint32_t r[32];
                        tmem_ld32(o_tmem + c * 32, r);
                        tmem_wait_ld();
                        reg_fence32(r);
#pragma unroll
                        for (int u = 0; u < 32; u += 2) {
                            const float2 y = __fmul2_rn(
                                make_float2(__uint_as_float(r[u]), __uint_as_float(r[u + 1])),
                                make_float2(alpha, alpha));
                            r[u] = __float_as_uint(y.x);
                            r[u + 1] = __float_as_uint(y.y);
                        }
                        tmem_st32(o_tmem + c * 32, r);
                    }
                }
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(p_full_leader);
        }

        // ---------------------------------------------------------- epilogue
        // Row sum = both halves' shares, exchanged on phase n of the exchange
        // barrier (the running max is already the same in both halves).
        if (ok) {
            xl[h * C::BM + row] = l;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_XCH));
            ok = warp_wait(bar(C::B_XCH), n & 1, abort_flag, p.status);
        }
        if (ok) {
            l += xl[(1 - h) * C::BM + row];
            ok = warp_wait(bar(C::B_O_FULL), (n - 1) & 1, abort_flag, p.status);
        }
        if (ok) {
            tc_fence_after();
            const float inv_l = l > 0.0f ? 1.0f / l : 0.0f;
            __nv_bfloat16* orow =
                p.out + (static_cast<int64_t>(i - p.q_offset) * p.Hq + head) * C::D + h * O_COLS;
#pragma unroll 1
            for (int c = 0; c < O_COLS / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(o_tmem + c * 32, r);
                tmem_wait_ld();
                reg_fence32(r);
                uint32_t w[16];
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    w[u] = pack_bf16x2(__uint_as_float(r[2 * u]) * inv_l,
                                       __uint_as_float(r[2 * u + 1]) * inv_l);
                if (row_valid) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        dst[u] = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
                }
            }
            if (h == 0 && row_valid && p.lse != nullptr)
                p.lse[static_cast<int64_t>(i - p.q_offset) * p.Hq + head] =
                    l > 0.0f ? (m_ref + log2f(l)) * 0.6931471805599453f : -INFINITY;
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // no CTA leaves while its peer may still signal or read it
    if (warp == C::MMA_WARP) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace thd
