// Packed-THD sliding-window GQA attention forward on CTA pairs, two query
// heads per CTA (B200, sm_100a), for head dim 128 and GQA groups that are a
// multiple of four.
//
// Same computation as thd_attn_kernel.cuh (see that file for the masking and
// softmax readings of the API pages: FlintMagiPlan.attention's window and
// sink, repeat_kv's head mapping).  One work item = one 128-row query tile of
// one document for four query heads of one kv group; the two CTAs of a
// cluster take two heads each:
//
// * Every tensor-core instruction is a tcgen05.mma.cta_group::2 with M = 256
//   issued by the leader (rank 0): instruction stream q (q = 0, 1) covers the
//   128 query rows of head head0 + q in CTA 0 and of head head0 + 2 + q in
//   CTA 1.  Each CTA loads half of every K tile (64 keys: B of S = Q K^T is
//   split along N) and half of every V tile (64 head-dim columns: B of
//   O += P V is split along N), so a QK instruction reads 96 instead of 128
//   bytes of shared memory per clock, and the K/V bytes each SM pulls from L2
//   halve.
// * Each CTA keeps whole score rows: S[q] (128 keys) and O[q] of its two
//   heads fill its 512 TMEM columns, so the softmax is the one-CTA kernel's,
//   one warpgroup per head (thread t = row t), with no exchange between the
//   CTAs except the "P written" arrivals on the leader's barrier.
// * MMA order per key tile j: PV0(j) QK0(j+1) | PV1(j) QK1(j+1): P(j)
//   overwrites S(j) and feeds PV(j) straight from TMEM, and QK(j+1) reuses the
//   S columns after PV(j) in the tensor core's issue order.
//
// Warps: 0-3 softmax of head stream 0, 4-7 head stream 1, 8 TMA producer
// (this CTA's Q tiles and K/V halves), 9 MMA issuer (leader only), 10-11 idle.
// Synchronisation:
//   * TMA loads of both CTAs complete on the LEADER's Q / slot barriers;
//   * MMA completion is committed to the same barrier in both CTAs (S ready,
//     O ready, slot free);
//   * the softmax warps of both CTAs arrive on the LEADER's P barriers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "sm100_ptx.cuh"
#include "thd_attn_kernel.cuh"

// Element pairs (out of every 4) whose exponential runs on the FMA pipe
// (fit_exp2_poly.py) instead of MUFU.  At head dim 128 the exponentials of a
// tile take as long as its MMAs at the tensor core's nominal rate.
#ifndef THD_PAIR_EXP_EMU
#define THD_PAIR_EXP_EMU 1
#endif

// 1: a persistent grid of one cluster per SM pair loops over the work items
// (the next item's Q load and first QK overlap the previous item's tail);
// 0: one cluster per item.
#ifndef THD_PAIR_PERSIST
#define THD_PAIR_PERSIST 1
#endif

namespace thd {

template <int D_, int NSLOT_, int EXP_EMU_>
struct PairConfig {
    static constexpr int D = D_;
    static constexpr int BN = 128;        // keys per key tile
    static constexpr int BM = 128;        // query rows per head tile (= TMEM lanes)
    static constexpr int NQ = 2;          // heads per CTA (4 per work item)
    static constexpr int NSLOT = NSLOT_;  // ring slots (one K half or V half each)
    // Element pairs (out of every 4) whose exponential runs on the FMA pipe.
    static constexpr int EXP_EMU = EXP_EMU_;

    static constexpr int KCH = D / 64;                  // 128-byte column chunks of a row
    static constexpr int Q_BOX_BYTES = BM * 128;
    static constexpr int Q_TILE_BYTES = BM * D * 2;
    static constexpr int KH_ROWS = BN / 2;              // keys of a K half
    static constexpr int KH_BOX_BYTES = KH_ROWS * 128;  // one 64-column chunk of a K half
    static constexpr int VH_COLS = D / 2;               // head-dim columns of a V half
    static constexpr int VH_CH = VH_COLS / 64;          // 64-column chunks of a V half
    static constexpr int VH_BOX_BYTES = BN * 128;       // one chunk of a V half
    static constexpr int SLOT_BYTES = BN * D;           // = K half bytes = V half bytes

    static constexpr int TMEM_S = 0;                    // S[q] at q*BN
    static constexpr int TMEM_O = NQ * BN;              // O[q] at TMEM_O + q*D
    static constexpr int TMEM_USED = TMEM_O + NQ * D;
    static constexpr int TMEM_COLS = 512;

    static constexpr int NUM_SOFTMAX_WARPS = 4 * NQ;
    static constexpr int PRODUCER_WARP = NUM_SOFTMAX_WARPS;
    static constexpr int MMA_WARP = NUM_SOFTMAX_WARPS + 1;
    static constexpr int NUM_THREADS = (NUM_SOFTMAX_WARPS + 4) * 32;
    // Register split as in the one-CTA kernel: 2*128*192 + 128*120 = 384*168.
    static constexpr int LAUNCH_REGS = 168;
    static constexpr int SOFTMAX_REGS = 192;
    static constexpr int CONTROL_REGS = 120;
    static_assert(NQ * 128 * SOFTMAX_REGS + 128 * CONTROL_REGS <= NUM_THREADS * LAUNCH_REGS,
                  "register split exceeds the launch");

    // mbarrier indices
    static constexpr int B_Q_FULL = 0;                        // leader: all four Q tiles landed
    static constexpr int B_Q_EMPTY = 1;                       // both: the item's last QK done
    static constexpr int B_SLOT_FULL = 2;                     // leader: both halves landed
    static constexpr int B_SLOT_EMPTY = B_SLOT_FULL + NSLOT;  // both: slot may be refilled
    static constexpr int B_S_FULL = B_SLOT_EMPTY + NSLOT;     // both: S[q] ready (and PV(j-1) done)
    static constexpr int B_P_FULL = B_S_FULL + NQ;            // leader: P[q] written in both CTAs
    static constexpr int B_O_FULL = B_P_FULL + NQ;            // both: last PV of stream q done
    static constexpr int B_O_FREE = B_O_FULL + NQ;            // leader: O[q] read in both CTAs
    static constexpr int B_DRAIN = B_O_FREE + NQ;
    static constexpr int NUM_BARS = B_DRAIN + 1;

    static constexpr int SMEM_Q = 0;
    static constexpr int SMEM_SLOTS = SMEM_Q + NQ * Q_TILE_BYTES;
    static constexpr int SMEM_BAR = SMEM_SLOTS + NSLOT * SLOT_BYTES;
    static constexpr int SMEM_TMEM_SLOT = SMEM_BAR + NUM_BARS * 8;
    static constexpr int SMEM_ABORT = SMEM_TMEM_SLOT + 4;
    static constexpr int SMEM_BYTES = SMEM_ABORT + 4;
    static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;

    static_assert(D == 128, "pair kernel with two heads per CTA: head dim 128");
    static_assert(VH_CH == 1, "a V half is one 64-column chunk");
    static_assert(TMEM_USED <= TMEM_COLS, "TMEM budget exceeded");
    static_assert(SMEM_ALLOC <= 232448, "shared memory budget exceeded");
    // Every wait of the MMA issuer is for a ring position whose slot was
    // released by an MMA it has already issued (V(j) after PV1(j), K(j+1)
    // after QK1(j+1)), so two slots cannot deadlock.
    static_assert(NSLOT >= 2, "ring needs two slots");
    static_assert(EXP_EMU >= 0 && EXP_EMU <= 4, "EXP_EMU counts element pairs out of 4");
};

template <class C>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(C::NUM_THREADS, 1)
thd_attn_fwd_pair_kernel(const __grid_constant__ CUtensorMap tmap_q,
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
    // Cluster c runs items c, c + n_clusters, ... (one item per cluster when
    // the grid has a cluster per item; a persistent grid of one cluster per
    // SM pair otherwise).  Barrier phases run on across items: S and P once
    // per key tile, Q, O and "O read" once per item.
    const int cluster_id = static_cast<int>(blockIdx.x >> 1);
    const int n_clusters = static_cast<int>(gridDim.x >> 1);
    const int n_items = p.n_items;

    auto bar = [&](int idx) -> uint32_t { return sbase + C::SMEM_BAR + 8u * idx; };
    auto lead_bar = [&](int idx) -> uint32_t { return mapa_shared(bar(idx), 0); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::SMEM_ABORT);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::SMEM_TMEM_SLOT);

    if (threadIdx.x == 0) {
        mbar_init(bar(C::B_Q_FULL), 1);
        mbar_init(bar(C::B_Q_EMPTY), 1);
        for (int s = 0; s < C::NSLOT; ++s) {
            mbar_init(bar(C::B_SLOT_FULL + s), 1);
            mbar_init(bar(C::B_SLOT_EMPTY + s), 1);
        }
        for (int q = 0; q < C::NQ; ++q) {
            mbar_init(bar(C::B_S_FULL + q), 1);
            mbar_init(bar(C::B_P_FULL + q), 8);  // 4 softmax warps of each CTA
            mbar_init(bar(C::B_O_FULL + q), 1);
            mbar_init(bar(C::B_O_FREE + q), 8);  // 4 softmax warps of each CTA
        }
        mbar_init(bar(C::B_DRAIN), 1);
        int bad = 0;
        if (THD_DEBUG)
            for (int w = cluster_id; w < n_items && !bad; w += n_clusters)
                bad = debug_check_item(p.items[w], p, 2 * C::NQ, C::BN);
        *abort_flag = launch_should_skip(p) | bad;
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

    if (warp >= C::NUM_SOFTMAX_WARPS) {
        regs_decrease<C::CONTROL_REGS>();
        if (warp == C::PRODUCER_WARP) {
            // --------------------------------- TMA producer (this CTA's part)
            if (lane == 0 && !skip) {
                tma_prefetch_desc(&tmap_q);
                tma_prefetch_desc(&tmap_k);
                tma_prefetch_desc(&tmap_v);
                bool ok = true;
                int pos = 0;  // ring position, continued across items
                int done = 0;  // items loaded so far
                for (int w = cluster_id; ok && w < n_items; w += n_clusters, ++done) {
                    const WorkItem it = p.items[w];
                    const int head_base = it.head0 + 2 * static_cast<int>(rank);
                    const int g = it.head0 / p.G;
                    // The previous item's Q tiles stay until its last QK is done.
                    if (done > 0) {
                        ok = mbar_wait(bar(C::B_Q_EMPTY), (done - 1) & 1, abort_flag, p.status,
                                       kStatusTimeout);
                        if (!ok) break;
                    }
                    if (leader) mbar_arrive_expect_tx(bar(C::B_Q_FULL), 2 * C::NQ * C::Q_TILE_BYTES);
                    for (int q = 0; q < C::NQ; ++q)
                        for (int c = 0; c < C::KCH; ++c)
                            tma_load_3d_pair(sbase + C::SMEM_Q + q * C::Q_TILE_BYTES + c * C::Q_BOX_BYTES,
                                             &tmap_q, lead_bar(C::B_Q_FULL), c * 64, head_base + q,
                                             it.q0 - p.q_offset);
                    // Ring positions: K(j) then V(j) for each key tile.  This
                    // CTA loads keys [rank*BN/2, (rank+1)*BN/2) of K(j) and
                    // head-dim columns [rank*D/2, (rank+1)*D/2) of V(j).
                    for (int jj = 0; jj < 2 * it.n_kv; ++jj, ++pos) {
                        const int slot = pos % C::NSLOT;
                        ok = mbar_wait(bar(C::B_SLOT_EMPTY + slot), ((pos / C::NSLOT) & 1) ^ 1,
                                       abort_flag, p.status, kStatusTimeout);
                        if (!ok) break;
                        if (leader) mbar_arrive_expect_tx(bar(C::B_SLOT_FULL + slot), 2 * C::SLOT_BYTES);
                        const uint32_t full = lead_bar(C::B_SLOT_FULL + slot);
                        const uint32_t dst = sbase + C::SMEM_SLOTS + slot * C::SLOT_BYTES;
                        const int kt = it.kv_start + (jj >> 1) * C::BN;
                        if ((jj & 1) == 0) {
                            for (int c = 0; c < C::KCH; ++c)
                                tma_load_3d_pair(dst + c * C::KH_BOX_BYTES, &tmap_k, full, c * 64, g,
                                                 kt + static_cast<int>(rank) * C::KH_ROWS);
                        } else {
                            tma_load_3d_pair(dst, &tmap_v, full, static_cast<int>(rank) * C::VH_COLS,
                                             g, kt);
                        }
                    }
                }
                // On an abort, loads still in flight (they complete on the
                // leader's barriers, which this CTA cannot track) are given
                // 200 us to land before the pair reaches its closing barrier.
                if (!ok) spin_ns(200000);
            }
            __syncwarp();
        } else if (warp == C::MMA_WARP) {
            // ------------------------------------------- MMA issuer (leader)
            if (leader && lane == 0 && !skip) {
                constexpr uint32_t idesc_qk = idesc_bf16_f32(256, C::BN, false);
                constexpr uint32_t idesc_pv = idesc_bf16_f32(256, C::D, true);
                const uint64_t dq0 = smem_desc_sw128(sbase + C::SMEM_Q, 16, 1024);
                const uint64_t dk0 = smem_desc_sw128(sbase + C::SMEM_SLOTS, 16, 1024);
                const uint64_t dv0 = smem_desc_sw128(sbase + C::SMEM_SLOTS, C::VH_BOX_BYTES, 1024);
                auto issue_qk = [&](int q, int slot) {
                    const uint32_t d_tmem = tmem_base + C::TMEM_S + q * C::BN;
                    const uint64_t dq = dq0 + ((q * C::Q_TILE_BYTES) >> 4);
                    const uint64_t dk = dk0 + ((slot * C::SLOT_BYTES) >> 4);
#pragma unroll
                    for (int kk = 0; kk < C::D / 16; ++kk) {
                        const uint32_t qo = ((kk >> 2) * C::Q_BOX_BYTES + (kk & 3) * 32) >> 4;
                        const uint32_t ko = ((kk >> 2) * C::KH_BOX_BYTES + (kk & 3) * 32) >> 4;
                        mma2_bf16_ss(d_tmem, dq + qo, dk + ko, idesc_qk, kk > 0 ? 1u : 0u);
                    }
                };
                // O += P V over the 128 keys of a tile: P (bf16, two keys per
                // column) in TMEM columns [0, 64) of S[q]; key k of the V half
                // is row k of the slot's 64-column chunk.
                auto issue_pv = [&](int q, int slot, bool acc) {
                    const uint32_t d_tmem = tmem_base + C::TMEM_O + q * C::D;
                    const uint32_t p_tmem = tmem_base + C::TMEM_S + q * C::BN;
                    const uint64_t dv = dv0 + ((slot * C::SLOT_BYTES) >> 4);
#pragma unroll
                    for (int kk = 0; kk < C::BN / 16; ++kk)
                        mma2_bf16_ts(d_tmem, p_tmem + kk * 8, dv + ((kk * 16 * 128) >> 4), idesc_pv,
                                     (acc || kk > 0) ? 1u : 0u);
                };
                auto wait = [&](int idx, uint32_t parity) -> bool {
                    return mbar_wait(bar(idx), parity, abort_flag, p.status, kStatusTimeout);
                };
                auto wait_slot = [&](int pos) -> bool {
                    return wait(C::B_SLOT_FULL + pos % C::NSLOT, (pos / C::NSLOT) & 1);
                };

                bool ok = true;
                int pos = 0;   // ring position of the item's K(0)
                int tile = 0;  // key tiles of earlier items (S / P phases)
                int done = 0;  // earlier items (Q / O phases)
                for (int w = cluster_id; ok && w < n_items; w += n_clusters, ++done) {
                    const int n = p.items[w].n_kv;
                    ok = wait(C::B_Q_FULL, done & 1) && wait_slot(pos);
                    if (!ok) break;
                    tc_fence_after();
                    for (int q = 0; q < C::NQ; ++q) {
                        issue_qk(q, pos % C::NSLOT);
                        mma2_commit_both(bar(C::B_S_FULL + q));
                    }
                    mma2_commit_both(bar(C::B_SLOT_EMPTY + pos % C::NSLOT));  // K(0) consumed
                    if (n == 1) mma2_commit_both(bar(C::B_Q_EMPTY));           // last QK of the item
                    for (int j = 0; ok && j < n; ++j) {
                        // PV(j) and QK(j+1) of a head stream go out as one run
                        // with one commit: S(j+1) ready also means O holds
                        // PV(j), so O gets its own commit only after the last
                        // tile.
                        const int vpos = pos + 2 * j + 1;
                        const int kpos = pos + 2 * j + 2;
                        const bool has_next = j + 1 < n;
                        ok = wait_slot(vpos) && (!has_next || wait_slot(kpos));
                        if (!ok) break;
                        for (int q = 0; q < C::NQ && ok; ++q) {
                            ok = wait(C::B_P_FULL + q, (tile + j) & 1);
                            // PV(0) overwrites O: the previous item's O must be read.
                            if (ok && j == 0 && done > 0) ok = wait(C::B_O_FREE + q, (done - 1) & 1);
                            if (!ok) break;
                            tc_fence_after();
                            issue_pv(q, vpos % C::NSLOT, j > 0);
                            if (has_next) {
                                issue_qk(q, kpos % C::NSLOT);
                                mma2_commit_both(bar(C::B_S_FULL + q));
                            } else {
                                mma2_commit_both(bar(C::B_O_FULL + q));
                            }
                        }
                        if (!ok) break;
                        mma2_commit_both(bar(C::B_SLOT_EMPTY + vpos % C::NSLOT));  // V(j) done
                        if (has_next) {
                            mma2_commit_both(bar(C::B_SLOT_EMPTY + kpos % C::NSLOT));  // K(j+1) done
                            if (j + 2 == n) mma2_commit_both(bar(C::B_Q_EMPTY));  // last QK of the item
                        }
                    }
                    pos += 2 * n;
                    tile += n;
                }
                // Every MMA issued by this thread has completed once this lands.
                mma2_commit_both(bar(C::B_DRAIN));
                drain_wait(bar(C::B_DRAIN), 0);
            }
            __syncwarp();
        }
    } else {
        // ---------------------------------------------------------- softmax
        regs_increase<C::SOFTMAX_REGS>();
        const int q = warp >> 2;
        const int wq = warp & 3;
        const int row = wq * 32 + lane;
        const int W = p.window;
        const float sl2 = p.scale_log2;
        constexpr float kTau = 8.0f;  // rescale only when the max grows by > 2^8
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(wq * 32) << 16);
        const uint32_t s_tmem = lane_base + C::TMEM_S + q * C::BN;
        const uint32_t o_tmem = lane_base + C::TMEM_O + q * C::D;
        const uint32_t p_full_leader = lead_bar(C::B_P_FULL + q);
        const uint32_t o_free_leader = lead_bar(C::B_O_FREE + q);

        bool ok = !skip;
        int tile = 0, done = 0;
        for (int w = cluster_id; ok && w < n_items; w += n_clusters, ++done) {
            const WorkItem it = p.items[w];
            const int n = it.n_kv;
            const int h = it.head0 + 2 * static_cast<int>(rank) + q;
            const int i = it.q0 + row;  // token of this row
            const int s_doc = it.doc_start;
            const int r_lo = it.q0 > s_doc ? it.q0 : s_doc;
            const int r_hi = it.q1 - 1;
            const bool row_valid = i >= r_lo && i <= r_hi;
            const int lo_i = (W > 0 && i - W + 1 > s_doc) ? i - W + 1 : s_doc;

            float m_ref = -INFINITY;
            float l = 0.0f;
            if (p.sinks != nullptr) {
                m_ref = p.sinks[h] * 1.4426950408889634f;
                l = 1.0f;
            }

            for (int j = 0; ok && j < n; ++j) {
                // S(j) ready; for j > 0 this also means PV(j-1) is in O.
                ok = warp_wait(bar(C::B_S_FULL + q), (tile + j) & 1, abort_flag, p.status);
                if (!ok) break;
                tc_fence_after();
                uint32_t sr[C::BN];
#pragma unroll
                for (int c = 0; c < C::BN / 32; ++c)
                    tmem_ld32(s_tmem + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < C::BN / 32; ++c)
                    reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
                float sv[C::BN];
#pragma unroll
                for (int c = 0; c < C::BN; ++c) sv[c] = __uint_as_float(sr[c]);

                const int kt = it.kv_start + j * C::BN;
                const bool full_tile = kt >= s_doc && kt + C::BN - 1 <= r_lo &&
                                       (W == 0 || kt >= r_hi - W + 1);
                if (!full_tile) {
                    const int c_lo = lo_i - kt;
                    const int c_hi = i - kt;
#pragma unroll
                    for (int c = 0; c < C::BN; ++c)
                        if (c < c_lo || c > c_hi) sv[c] = -INFINITY;
                }
                float mx[4] = {sv[0], sv[1], sv[2], sv[3]};
#pragma unroll
                for (int c = 4; c < C::BN; c += 2)
                    mx[(c >> 1) & 3] = max3f(mx[(c >> 1) & 3], sv[c], sv[c + 1]);
                const float smax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
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

                if (j > 0 && __any_sync(0xffffffffu, rescale_o)) {
#pragma unroll 1
                    for (int c = 0; c < C::D / 32; ++c) {
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
                    tmem_wait_st();
                }

                const float2 sl2x2 = make_float2(sl2, sl2);
                const float2 negm2 = make_float2(neg_m, neg_m);
                float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
                exp_and_store_p<0, C::BN / 32, C::BN, C::EXP_EMU>(sv, sl2x2, negm2, s_tmem, acc0, acc1);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(p_full_leader);
                l += (acc0.x + acc0.y) + (acc1.x + acc1.y);
            }

            if (ok) ok = warp_wait(bar(C::B_O_FULL + q), done & 1, abort_flag, p.status);
            if (!ok) break;
            tc_fence_after();
            const float inv_l = l > 0.0f ? 1.0f / l : 0.0f;
            __nv_bfloat16* orow = p.out + (static_cast<int64_t>(i - p.q_offset) * p.Hq + h) * C::D;
#pragma unroll 1
            for (int c = 0; c < C::D / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(o_tmem + c * 32, r);
                tmem_wait_ld();
                reg_fence32(r);
                if (c == C::D / 32 - 1) {
                    // O is read: the next item's PV(0) may overwrite it.
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(o_free_leader);
                }
                uint32_t wv[16];
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    wv[u] = pack_bf16x2(__uint_as_float(r[2 * u]) * inv_l,
                                        __uint_as_float(r[2 * u + 1]) * inv_l);
                if (row_valid) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        dst[u] = make_uint4(wv[4 * u], wv[4 * u + 1], wv[4 * u + 2], wv[4 * u + 3]);
                }
            }
            if (row_valid && p.lse != nullptr)
                p.lse[static_cast<int64_t>(i - p.q_offset) * p.Hq + h] =
                    l > 0.0f ? (m_ref + log2f(l)) * 0.6931471805599453f : -INFINITY;
            tile += n;
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

// Host check before the first launch: the register split assumes the kernel
// starts with LAUNCH_REGS registers per thread.
template <class C>
inline bool pair_launch_registers_ok() {
    cudaFuncAttributes a{};
    if (cudaFuncGetAttributes(&a, thd_attn_fwd_pair_kernel<C>) != cudaSuccess) return false;
    return a.numRegs >= C::LAUNCH_REGS;
}

// Clusters of the persistent grid: as many as can be resident at once (one
// per SM pair), found once per device after the shared-memory attribute is
// set.  Returns 0 on failure.
template <class C>
inline int pair_max_active_clusters() {
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(C::NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM_ALLOC;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, thd_attn_fwd_pair_kernel<C>, &cfg) != cudaSuccess) return 0;
    return n;
}

// Grid of a launch over n_items items: one cluster per item, or with the
// persistent grid at most max_clusters clusters that loop over the items.
inline unsigned pair_grid(int64_t n_items, int max_clusters) {
    int64_t c = n_items;
    if (THD_PAIR_PERSIST && max_clusters > 0 && c > max_clusters) c = max_clusters;
    return static_cast<unsigned>(2 * c);
}

}  // namespace thd
