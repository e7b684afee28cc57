// Packed-THD sliding-window GQA attention forward on CTA pairs (B200, sm_100a).
//
// Same computation as thd_attn_kernel.cuh (one work item = one 128-row query
// tile of one document for several query heads that share one kv head, see
// that file for the masking and softmax readings of the API pages), but a
// cluster of two CTAs shares every tensor-core instruction: the leader CTA
// (rank 0) issues tcgen05.mma.cta_group::2 with M = 256, i.e. the same 128
// query rows of NQ heads in each CTA.  An M = 256 instruction keeps the tensor
// core at its full rate with N = 128, which a one-CTA M = 128 instruction
// cannot, and each CTA loads only half of every K tile (half the keys: B of
// S = Q K^T is split along N) and half of every V tile (half of the head dim:
// B of O += P V is split along N).
//
// The probabilities P go to shared memory (128-byte swizzled, the A operand
// of O += P V), not back over S in TMEM.  S(j) is therefore free as soon as
// the softmax has loaded it into registers, and S(j+1) = Q K(j+1)^T runs on
// the tensor core while the softmax still works on tile j: a softmax
// warpgroup never waits for the whole MMA chain of its previous tile.
//
// Per CTA: NQ softmax warpgroups (TMEM lane = row of this CTA's query tile)
// and one control warpgroup (warp 0: TMA producer of this CTA's halves;
// warp 1: MMA issuer, active in the leader only, issuing whichever MMA is
// ready).  Synchronisation:
//   * TMA loads of both CTAs complete on the LEADER's Q / slot barriers;
//   * MMA completion is committed to the same barrier in both CTAs (S ready,
//     O ready, slot free);
//   * each CTA's softmax warps arrive on the LEADER's S-free and P barriers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "sm100_ptx.cuh"
#include "thd_attn_kernel.cuh"

namespace thd {

template <int D_, int NQ_, int BN_, int NSLOT_>
struct PairConfig {
    static constexpr int D = D_;
    static constexpr int NQ = NQ_;        // query tiles (heads) per CTA; 2*NQ per pair
    static constexpr int BN = BN_;        // keys per key tile
    static constexpr int NSLOT = NSLOT_;  // ring slots (one K half or V half each)
    static constexpr int BM = 128;        // query rows per CTA (M = 256 per pair)

    static constexpr int KCH = D / 64;                  // 128-byte column chunks of a Q row
    static constexpr int Q_BOX_BYTES = BM * 128;
    static constexpr int Q_TILE_BYTES = BM * D * 2;
    static constexpr int P_CH = BN / 64;                // 64-key chunks of a P row
    static constexpr int P_CHUNK_BYTES = BM * 128;
    static constexpr int P_TILE_BYTES = BM * BN * 2;
    static constexpr int KH_ROWS = BN / 2;              // keys of a K half
    static constexpr int KH_BOX_BYTES = KH_ROWS * 128;  // one 64-column chunk of a K half
    static constexpr int VH_COLS = D / 2;               // head-dim columns of a V half
    static constexpr int VH_CH = VH_COLS / 64;          // chunks of a V half
    static constexpr int VH_BOX_BYTES = BN * 128;       // one chunk of a V half
    static constexpr int SLOT_BYTES = BN * D;           // = K half bytes = V half bytes

    static constexpr int TMEM_S = 0;
    static constexpr int TMEM_O = NQ * BN;
    static constexpr int TMEM_USED = TMEM_O + NQ * D;
    static constexpr int TMEM_COLS = TMEM_USED <= 256 ? 256 : 512;

    static constexpr int NUM_SOFTMAX_WARPS = 4 * NQ;
    static constexpr int PRODUCER_WARP = NUM_SOFTMAX_WARPS;
    static constexpr int MMA_WARP = NUM_SOFTMAX_WARPS + 1;
    static constexpr int NUM_THREADS = (NUM_SOFTMAX_WARPS + 4) * 32;
    static constexpr bool REG_SPLIT = NQ == 2;
    static constexpr int LAUNCH_REGS = 168;
    static constexpr int SOFTMAX_REGS = 200;
    static constexpr int CONTROL_REGS = 104;
    static_assert(!REG_SPLIT || (NQ * 128 * SOFTMAX_REGS + 128 * CONTROL_REGS <=
                                 NUM_THREADS * LAUNCH_REGS), "register split exceeds the launch");

    static constexpr int B_Q_FULL = 0;                          // leader: both CTAs' Q landed
    static constexpr int B_SLOT_FULL = 1;                       // leader: both halves landed
    static constexpr int B_SLOT_EMPTY = B_SLOT_FULL + NSLOT;    // both: slot may be refilled
    static constexpr int B_S_FULL = B_SLOT_EMPTY + NSLOT;       // both: S = Q K^T done [NQ]
    static constexpr int B_S_FREE = B_S_FULL + NQ;              // leader: S read in both CTAs
    static constexpr int B_P_FULL = B_S_FREE + NQ;              // leader: P written in both CTAs
    static constexpr int B_O_FULL = B_P_FULL + NQ;              // both: PV done
    static constexpr int B_DRAIN = B_O_FULL + NQ;
    static constexpr int NUM_BARS = B_DRAIN + 1;

    static constexpr int SMEM_Q = 0;
    static constexpr int SMEM_P = SMEM_Q + NQ * Q_TILE_BYTES;
    static constexpr int SMEM_SLOTS = SMEM_P + NQ * P_TILE_BYTES;
    static constexpr int SMEM_BAR = SMEM_SLOTS + NSLOT * SLOT_BYTES;
    static constexpr int SMEM_TMEM_SLOT = SMEM_BAR + NUM_BARS * 8;
    static constexpr int SMEM_ABORT = SMEM_TMEM_SLOT + 4;
    static constexpr int SMEM_BYTES = SMEM_ABORT + 4;
    static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;

    static_assert(D == 128 || D == 256, "pair kernel: head dim 128 or 256");
    static_assert(BN % 64 == 0 && BN <= 256, "key tile must be a multiple of 64");
    static_assert(TMEM_USED <= 512, "TMEM budget exceeded");
    static_assert(SMEM_ALLOC <= 232448, "shared memory budget exceeded");
    static_assert(NSLOT >= 2, "ring needs two slots");
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
    const WorkItem it = p.items[blockIdx.x >> 1];
    const int n = it.n_kv;
    const int head_cta = it.head0 + static_cast<int>(rank) * C::NQ;  // first head of this CTA

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
        for (int q = 0; q < C::NQ; ++q) {
            mbar_init(bar(C::B_S_FULL + q), 1);
            mbar_init(bar(C::B_S_FREE + q), 8);  // 4 warps in each CTA
            mbar_init(bar(C::B_P_FULL + q), 8);
            mbar_init(bar(C::B_O_FULL + q), 1);
        }
        mbar_init(bar(C::B_DRAIN), 1);
        *abort_flag = *reinterpret_cast<volatile int*>(p.status) != 0 ? 1 : 0;
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
      if constexpr (C::REG_SPLIT) regs_decrease<C::CONTROL_REGS>();
      if (warp == C::PRODUCER_WARP) {
        // ------------------------------------- TMA producer (this CTA's half)
        if (lane == 0 && !skip) {
            tma_prefetch_desc(&tmap_q);
            tma_prefetch_desc(&tmap_k);
            tma_prefetch_desc(&tmap_v);
            const int g = it.head0 / p.G;
            if (leader) mbar_arrive_expect_tx(bar(C::B_Q_FULL), 2 * C::NQ * C::Q_TILE_BYTES);
            for (int q = 0; q < C::NQ; ++q)
                for (int c = 0; c < C::KCH; ++c)
                    tma_load_3d_pair(sbase + C::SMEM_Q + q * C::Q_TILE_BYTES + c * C::Q_BOX_BYTES,
                                     &tmap_q, lead_bar(C::B_Q_FULL), c * 64, head_cta + q, it.q0);
            // Ring positions: 2j holds K(j), 2j+1 holds V(j).  This CTA loads
            // keys [rank*BN/2, (rank+1)*BN/2) of K(j) and head-dim columns
            // [rank*D/2, (rank+1)*D/2) of V(j).
            bool ok = true;
            for (int pos = 0; pos < 2 * n && ok; ++pos) {
                const int slot = pos % C::NSLOT;
                ok = mbar_wait_cluster(bar(C::B_SLOT_EMPTY + slot), ((pos / C::NSLOT) & 1) ^ 1,
                                       abort_flag, p.status, kStatusTimeout);
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
      } else if (warp == C::MMA_WARP && leader) {
        // ------------------------------------------- MMA issuer (leader only)
        if (!skip) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(256, C::BN, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(256, C::D, true);
            const uint64_t dq0 = smem_desc_sw128(sbase + C::SMEM_Q, 16, 1024);
            const uint64_t dp0 = smem_desc_sw128(sbase + C::SMEM_P, 16, 1024);
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
                    if (elect_one()) mma2_bf16_ss(d_tmem, dq + qo, dk + ko, idesc_qk, kk > 0 ? 1u : 0u);
                }
            };
            auto issue_pv = [&](int q, int slot, bool acc) {
                const uint32_t d_tmem = tmem_base + C::TMEM_O + q * C::D;
                const uint64_t dp = dp0 + ((q * C::P_TILE_BYTES) >> 4);
                const uint64_t dv = dv0 + ((slot * C::SLOT_BYTES) >> 4);
#pragma unroll
                for (int kk = 0; kk < C::BN / 16; ++kk) {
                    const uint32_t po = ((kk >> 2) * C::P_CHUNK_BYTES + (kk & 3) * 32) >> 4;
                    if (elect_one())
                        mma2_bf16_ss(d_tmem, dp + po, dv + ((kk * 16 * 128) >> 4), idesc_pv,
                                     (acc || kk > 0) ? 1u : 0u);
                }
            };
            auto commit_both = [&](int idx) {
                if (elect_one()) mma2_commit_both(bar(idx));
                __syncwarp();
            };
            // Lane 0 probes, the warp follows (the issue loop stays converged).
            auto test = [&](int idx, uint32_t parity) -> bool {
                int r = 0;
                if (lane == 0) r = mbar_test(bar(idx), parity);
                return __shfl_sync(0xffffffffu, r, 0) != 0;
            };
            auto slot_ready = [&](int pos) -> bool {
                return test(C::B_SLOT_FULL + pos % C::NSLOT, (pos / C::NSLOT) & 1);
            };

            int ok = 1;
            if (lane == 0) ok = mbar_wait_cluster(bar(C::B_Q_FULL), 0, abort_flag, p.status, kStatusTimeout);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            int qk_next[C::NQ], pv_next[C::NQ];
#pragma unroll
            for (int q = 0; q < C::NQ; ++q) qk_next[q] = pv_next[q] = 0;
            int k_released = 0, v_released = 0;  // tiles whose K / V slot was handed back
            uint64_t idle_since = 0;
            bool idle = false;
            while (ok) {
                bool done = true, progress = false;
#pragma unroll
                for (int q = 0; q < C::NQ; ++q) {
                    if (pv_next[q] < n) done = false;
                    // O += P(t) V(t): P(t) written by both CTAs, V(t) landed.
                    const int tp = pv_next[q];
                    if (tp < qk_next[q] && test(C::B_P_FULL + q, tp & 1) && slot_ready(2 * tp + 1)) {
                        tc_fence_after();
                        issue_pv(q, (2 * tp + 1) % C::NSLOT, tp > 0);
                        commit_both(C::B_O_FULL + q);
                        pv_next[q] = tp + 1;
                        progress = true;
                    }
                    // S(t) = Q K(t)^T: S(t-1) read out by both CTAs, K(t) landed.
                    const int tq = qk_next[q];
                    if (tq < n && (tq == 0 || test(C::B_S_FREE + q, (tq - 1) & 1)) &&
                        slot_ready(2 * tq)) {
                        tc_fence_after();
                        issue_qk(q, (2 * tq) % C::NSLOT);
                        commit_both(C::B_S_FULL + q);
                        qk_next[q] = tq + 1;
                        progress = true;
                    }
                }
                if (done) break;
                // Hand slots back once every query tile has consumed them.
                int min_qk = n, min_pv = n;
#pragma unroll
                for (int q = 0; q < C::NQ; ++q) {
                    min_qk = qk_next[q] < min_qk ? qk_next[q] : min_qk;
                    min_pv = pv_next[q] < min_pv ? pv_next[q] : min_pv;
                }
                for (; k_released < min_qk; ++k_released)
                    commit_both(C::B_SLOT_EMPTY + (2 * k_released) % C::NSLOT);
                for (; v_released < min_pv; ++v_released)
                    commit_both(C::B_SLOT_EMPTY + (2 * v_released + 1) % C::NSLOT);
                if (progress) {
                    idle = false;
                } else {
                    // Bounded: give up (and record a timeout) if nothing became
                    // ready for the wait limit.
                    int give_up = 0;
                    if (lane == 0) {
                        const uint64_t now = global_timer_ns();
                        if (!idle) idle_since = now;
                        if (*abort_flag) {
                            give_up = 1;
                        } else if (*reinterpret_cast<volatile int*>(p.status) != 0) {
                            *abort_flag = 1;
                            give_up = 1;
                        } else if (idle && now - idle_since > kWaitLimitNs) {
                            atomicCAS(p.status, 0, kStatusTimeout);
                            *abort_flag = 1;
                            give_up = 1;
                        }
                    }
                    idle = true;
                    if (__shfl_sync(0xffffffffu, give_up, 0)) ok = 0;
                }
            }
            commit_both(C::B_DRAIN);
            if (lane == 0) drain_wait(bar(C::B_DRAIN), 0);
            __syncwarp();
        }
      }
    } else {
        // ------------------------------------------------------------ softmax
        if constexpr (C::REG_SPLIT) regs_increase<C::SOFTMAX_REGS>();
        const int q = warp >> 2;
        const int wq = warp & 3;
        const int row = wq * 32 + lane;
        const int h = head_cta + q;
        const int i = it.q0 + row;
        const int s_doc = it.doc_start;
        const int r_lo = it.q0 > s_doc ? it.q0 : s_doc;
        const int r_hi = it.q1 - 1;
        const bool row_valid = i >= r_lo && i <= r_hi;
        const int W = p.window;
        const int lo_i = (W > 0 && i - W + 1 > s_doc) ? i - W + 1 : s_doc;
        const float sl2 = p.scale_log2;
        constexpr float kTau = 8.0f;

        float m_ref = -INFINITY;
        float l = 0.0f;
        if (p.sinks != nullptr) {
            m_ref = p.sinks[h] * 1.4426950408889634f;
            l = 1.0f;
        }
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(wq * 32) << 16);
        const uint32_t s_tmem = lane_base + C::TMEM_S + q * C::BN;
        const uint32_t o_tmem = lane_base + C::TMEM_O + q * C::D;
        const uint32_t s_free_leader = lead_bar(C::B_S_FREE + q);
        const uint32_t p_full_leader = lead_bar(C::B_P_FULL + q);
        // This thread's row of P in shared memory (K-major, 128-byte swizzle:
        // 16-byte unit u of the row sits at unit u ^ (row % 8)).
        const uint32_t p_row = sbase + C::SMEM_P + q * C::P_TILE_BYTES + (row >> 3) * 1024 +
                               (row & 7) * 128;
        const uint32_t p_xor = static_cast<uint32_t>(row & 7);
        auto wait = [&](int idx, uint32_t parity) -> bool {
            int ok = 0;
            if (lane == 0) ok = mbar_wait_cluster(bar(idx), parity, abort_flag, p.status, kStatusTimeout);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            __syncwarp();
            return ok != 0;
        };

        bool ok = !skip;
        for (int j = 0; ok && j < n; ++j) {
            ok = wait(C::B_S_FULL + q, j & 1);
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
            // S(j) is in registers: the tensor core may overwrite it with S(j+1).
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(s_free_leader);

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
            for (int c = 4; c < C::BN; c += 2) mx[(c >> 1) & 3] = max3f(mx[(c >> 1) & 3], sv[c], sv[c + 1]);
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

            // Exponentials into registers (bf16 pairs) first ...
            const float2 sl2x2 = make_float2(sl2, sl2);
            const float2 negm2 = make_float2(neg_m, neg_m);
            float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
            uint32_t pk[C::BN / 2];
#pragma unroll
            for (int c = 0; c < C::BN / 2; ++c) {
                const float2 x = __ffma2_rn(make_float2(sv[2 * c], sv[2 * c + 1]), sl2x2, negm2);
                const float p0 = ex2_approx(x.x);
                const float p1 = ex2_approx(x.y);
                if (c & 1) acc1 = __fadd2_rn(acc1, make_float2(p0, p1));
                else acc0 = __fadd2_rn(acc0, make_float2(p0, p1));
                pk[c] = pack_bf16x2(p0, p1);
            }
            l += (acc0.x + acc0.y) + (acc1.x + acc1.y);

            // ... then wait until PV(j-1) is done: it has read P(j-1) from
            // shared memory, and O holds its contribution (for the rescale).
            if (j > 0) {
                ok = wait(C::B_O_FULL + q, (j - 1) & 1);
                if (!ok) break;
                tc_fence_after();
                if (__any_sync(0xffffffffu, rescale_o)) {
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
            }
            // P(j) to shared memory: 8 bf16 (16 bytes) per store.
#pragma unroll
            for (int u = 0; u < C::BN / 8; ++u) {
                const uint32_t addr = p_row + (u >> 3) * C::P_CHUNK_BYTES +
                                      ((static_cast<uint32_t>(u & 7) ^ p_xor) << 4);
                st_shared_v4(addr, pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(p_full_leader);
        }

        if (ok) ok = wait(C::B_O_FULL + q, (n - 1) & 1);
        if (ok) {
            tc_fence_after();
            const float inv_l = l > 0.0f ? 1.0f / l : 0.0f;
            __nv_bfloat16* orow = p.out + (static_cast<int64_t>(i) * p.Hq + h) * C::D;
#pragma unroll 1
            for (int c = 0; c < C::D / 32; ++c) {
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
            if (row_valid && p.lse != nullptr)
                p.lse[static_cast<int64_t>(i) * p.Hq + h] =
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

template <class C>
inline bool pair_launch_registers_ok() {
    if constexpr (!C::REG_SPLIT) {
        return true;
    } else {
        cudaFuncAttributes a{};
        if (cudaFuncGetAttributes(&a, thd_attn_fwd_pair_kernel<C>) != cudaSuccess) return false;
        return a.numRegs >= C::LAUNCH_REGS;
    }
}

}  // namespace thd
