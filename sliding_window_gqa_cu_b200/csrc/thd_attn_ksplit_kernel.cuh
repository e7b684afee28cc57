// Packed-THD sliding-window GQA attention forward, head dim 128, two query
// heads per CTA with the softmax of every key tile split between two
// warpgroups per head (B200, sm_100a).
//
// Same computation and work items as thd_attn_kernel.cuh with two heads per
// item (see that file for the masking and softmax readings of the API pages:
// FlintMagiPlan.attention's window and sink, repeat_kv's head mapping).  What
// differs is who runs the softmax: each head has two warpgroups, warpgroup
// (q, h) owning keys [64 h, 64 h + 64) of every 128-key tile of head q (TMEM
// columns [64 h, 64 h + 64) of S[q]; its P goes to columns [64 h, 64 h + 32)).
// A thread therefore exponentiates 64 scores per tile instead of 128, which
// halves the softmax leg of the per-head chain S ready -> P -> PV / next QK
// that the tensor core waits on.  The two halves exchange their partial row
// maxima through shared memory once per tile, so both apply one running max
// to the one O; each rescales and stores half of O's columns, and their row
// sums meet once at the end.
//
// Warps: 0-15 softmax (head q = w / 8, key half h = (w / 4) % 2, TMEM lane
// quadrant w % 4), 16 TMA producer, 17 MMA issuer (576 threads, 112 registers
// each).  TMEM: S[q] at
// 128 q, O[q] at 256 + 128 q (512 columns).  MMA order per key tile j, as in
// the two-head one-CTA kernel: PV0(j) QK0(j+1) | PV1(j) QK1(j+1).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "sm100_ptx.cuh"
#include "thd_attn_kernel.cuh"

// 1: head dim 128 with two heads per CTA runs on this kernel; 0: on the
// one-CTA kernel with one softmax warpgroup per head (thd_attn_kernel.cuh).
#ifndef THD_KSPLIT128
#define THD_KSPLIT128 0
#endif

namespace thd {

template <int NSLOT_>
struct KsplitConfig {
    static constexpr int D = 128;
    static constexpr int NQ = 2;          // heads per CTA
    static constexpr int BN = 128;        // keys per key tile
    static constexpr int BM = 128;        // query rows per tile (= TMEM lanes)
    static constexpr int HALF = BN / 2;   // keys per softmax warpgroup
    static constexpr int NSLOT = NSLOT_;  // K/V ring slots (one K or V tile each)
    static constexpr int EXP_EMU = THD_EXP_EMU;

    static constexpr int KCH = D / 64;
    static constexpr int Q_BOX_BYTES = BM * 128;
    static constexpr int Q_TILE_BYTES = BM * D * 2;
    static constexpr int KV_BOX_BYTES = BN * 128;
    static constexpr int KV_TILE_BYTES = BN * D * 2;

    static constexpr int TMEM_S = 0;
    static constexpr int TMEM_O = NQ * BN;
    static constexpr int TMEM_COLS = 512;

    static constexpr int NUM_SOFTMAX_WARPS = 8 * NQ;
    static constexpr int PRODUCER_WARP = NUM_SOFTMAX_WARPS;
    static constexpr int MMA_WARP = NUM_SOFTMAX_WARPS + 1;
    // 18 warps, no register split: 576 threads x 112 registers.
    static constexpr int NUM_THREADS = (NUM_SOFTMAX_WARPS + 2) * 32;

    static constexpr int B_Q_FULL = 0;
    static constexpr int B_SLOT_FULL = 1;
    static constexpr int B_SLOT_EMPTY = B_SLOT_FULL + NSLOT;
    static constexpr int B_S_FULL = B_SLOT_EMPTY + NSLOT;  // [NQ]
    static constexpr int B_P_FULL = B_S_FULL + NQ;         // [NQ] P of both halves, O rescaled
    static constexpr int B_O_FULL = B_P_FULL + NQ;         // [NQ] last PV done
    static constexpr int B_XCH = B_O_FULL + NQ;            // [NQ] the halves of a head met
    static constexpr int B_DRAIN = B_XCH + NQ;
    static constexpr int NUM_BARS = B_DRAIN + 1;

    static constexpr int SMEM_Q = 0;
    static constexpr int SMEM_SLOTS = SMEM_Q + NQ * Q_TILE_BYTES;
    static constexpr int SMEM_XMAX = SMEM_SLOTS + NSLOT * KV_TILE_BYTES;  // float [NQ][2][2][BM]
    static constexpr int SMEM_XL = SMEM_XMAX + NQ * 2 * 2 * BM * 4;       // float [NQ][2][BM]
    static constexpr int SMEM_BAR = SMEM_XL + NQ * 2 * BM * 4;
    static constexpr int SMEM_TMEM_SLOT = SMEM_BAR + NUM_BARS * 8;
    static constexpr int SMEM_ABORT = SMEM_TMEM_SLOT + 4;
    static constexpr int SMEM_BYTES = SMEM_ABORT + 4;
    static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;

    static_assert(TMEM_O + NQ * D <= TMEM_COLS, "TMEM budget exceeded");
    static_assert(SMEM_ALLOC <= 232448, "shared memory budget exceeded");
    static_assert(NSLOT >= 2, "K/V ring needs two slots");
};

template <class C>
__global__ void __maxnreg__(112)
thd_attn_fwd_ksplit_kernel(const __grid_constant__ CUtensorMap tmap_q,
                           const __grid_constant__ CUtensorMap tmap_k,
                           const __grid_constant__ CUtensorMap tmap_v,
                           const FwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_addr(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
    const uint32_t sbase = smem_addr(smem);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const WorkItem it = p.items[blockIdx.x];
    const int n = it.n_kv;

    auto bar = [&](int idx) -> uint32_t { return sbase + C::SMEM_BAR + 8u * idx; };
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
            mbar_init(bar(C::B_P_FULL + q), 8);  // the 8 softmax warps of the head
            mbar_init(bar(C::B_O_FULL + q), 1);
            mbar_init(bar(C::B_XCH + q), 8);
        }
        mbar_init(bar(C::B_DRAIN), 1);
        *abort_flag = launch_should_skip(p) | debug_check_item(it, p, C::NQ, C::BN);
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

    if (warp >= C::NUM_SOFTMAX_WARPS) {
        if (warp == C::PRODUCER_WARP) {
            // ---------------------------------------------------- TMA producer
            if (lane == 0 && !skip) {
                tma_prefetch_desc(&tmap_q);
                tma_prefetch_desc(&tmap_k);
                tma_prefetch_desc(&tmap_v);
                const int g = it.head0 / p.G;
                mbar_arrive_expect_tx(bar(C::B_Q_FULL), C::NQ * C::Q_TILE_BYTES);
                for (int q = 0; q < C::NQ; ++q)
                    for (int c = 0; c < C::KCH; ++c)
                        tma_load_3d(sbase + C::SMEM_Q + q * C::Q_TILE_BYTES + c * C::Q_BOX_BYTES,
                                    &tmap_q, bar(C::B_Q_FULL), c * 64, it.head0 + q,
                                    it.q0 - p.q_offset);
                // Ring positions: 2j holds K(j), 2j+1 holds V(j).
                int issued = 0;
                bool ok = true;
                for (int pos = 0; pos < 2 * n && ok; ++pos) {
                    const int slot = pos % C::NSLOT;
                    ok = mbar_wait(bar(C::B_SLOT_EMPTY + slot), ((pos / C::NSLOT) & 1) ^ 1,
                                   abort_flag, p.status, kStatusTimeout);
                    if (!ok) break;
                    const CUtensorMap* map = (pos & 1) ? &tmap_v : &tmap_k;
                    const int kt = it.kv_start + (pos >> 1) * C::BN;
                    mbar_arrive_expect_tx(bar(C::B_SLOT_FULL + slot), C::KV_TILE_BYTES);
                    for (int c = 0; c < C::KCH; ++c)
                        tma_load_3d(sbase + C::SMEM_SLOTS + slot * C::KV_TILE_BYTES + c * C::KV_BOX_BYTES,
                                    map, bar(C::B_SLOT_FULL + slot), c * 64, g, kt);
                    issued = pos + 1;
                }
                if (!ok) {
                    // Unwinding: let the loads already issued land before exit.
                    drain_wait(bar(C::B_Q_FULL), 0);
                    for (int pos = issued - C::NSLOT > 0 ? issued - C::NSLOT : 0; pos < issued; ++pos)
                        drain_wait(bar(C::B_SLOT_FULL + pos % C::NSLOT), (pos / C::NSLOT) & 1);
                }
            }
            __syncwarp();
        } else if (warp == C::MMA_WARP) {
            // ------------------------------------------------------ MMA issuer
            if (lane == 0 && !skip) {
                constexpr uint32_t idesc_qk = idesc_bf16_f32(128, C::BN, false);
                constexpr uint32_t idesc_pv = idesc_bf16_f32(128, C::D, true);
                const uint64_t dq0 = smem_desc_sw128(sbase + C::SMEM_Q, 16, 1024);
                const uint64_t dk0 = smem_desc_sw128(sbase + C::SMEM_SLOTS, 16, 1024);
                const uint64_t dv0 = smem_desc_sw128(sbase + C::SMEM_SLOTS, C::KV_BOX_BYTES, 1024);
                auto issue_qk = [&](int q, int slot) {
                    const uint32_t d_tmem = tmem_base + C::TMEM_S + q * C::BN;
                    const uint64_t dq = dq0 + ((q * C::Q_TILE_BYTES) >> 4);
                    const uint64_t dk = dk0 + ((slot * C::KV_TILE_BYTES) >> 4);
#pragma unroll
                    for (int kk = 0; kk < C::D / 16; ++kk) {
                        const uint32_t qo = ((kk >> 2) * C::Q_BOX_BYTES + (kk & 3) * 32) >> 4;
                        const uint32_t ko = ((kk >> 2) * C::KV_BOX_BYTES + (kk & 3) * 32) >> 4;
                        mma_bf16_ss(d_tmem, dq + qo, dk + ko, idesc_qk, kk > 0 ? 1u : 0u);
                    }
                };
                // O += P V: the P of key half h sits in TMEM columns
                // [64 h, 64 h + 32) of S[q] (two keys per column).
                auto issue_pv = [&](int q, int slot, bool acc) {
                    const uint32_t d_tmem = tmem_base + C::TMEM_O + q * C::D;
                    const uint32_t p_tmem = tmem_base + C::TMEM_S + q * C::BN;
                    const uint64_t dv = dv0 + ((slot * C::KV_TILE_BYTES) >> 4);
#pragma unroll
                    for (int kk = 0; kk < C::BN / 16; ++kk)
                        mma_bf16_ts(d_tmem, p_tmem + (kk >> 2) * C::HALF + (kk & 3) * 8,
                                    dv + ((kk * 16 * 128) >> 4), idesc_pv, (acc || kk > 0) ? 1u : 0u);
                };
                auto wait = [&](int idx, uint32_t parity) -> bool {
                    return mbar_wait(bar(idx), parity, abort_flag, p.status, kStatusTimeout);
                };
                auto wait_slot = [&](int pos) -> bool {
                    return wait(C::B_SLOT_FULL + pos % C::NSLOT, (pos / C::NSLOT) & 1);
                };
                bool ok = wait(C::B_Q_FULL, 0) && wait_slot(0);
                if (ok) {
                    tc_fence_after();
                    for (int q = 0; q < C::NQ; ++q) {
                        issue_qk(q, 0);
                        mma_commit(bar(C::B_S_FULL + q));
                    }
                    mma_commit(bar(C::B_SLOT_EMPTY + 0));  // K(0) consumed
                }
                for (int j = 0; ok && j < n; ++j) {
                    // PV(j) and QK(j+1) of a head go out as one run with one
                    // commit (S(j+1) ready also means O holds PV(j)).
                    const int vslot = (2 * j + 1) % C::NSLOT;
                    const bool has_next = j + 1 < n;
                    const int kslot = (2 * j + 2) % C::NSLOT;
                    ok = wait_slot(2 * j + 1) && (!has_next || wait_slot(2 * j + 2));
                    if (!ok) break;
                    for (int q = 0; q < C::NQ && ok; ++q) {
                        ok = wait(C::B_P_FULL + q, j & 1);
                        if (!ok) break;
                        tc_fence_after();
                        issue_pv(q, vslot, j > 0);
                        if (has_next) {
                            issue_qk(q, kslot);
                            mma_commit(bar(C::B_S_FULL + q));
                        } else {
                            mma_commit(bar(C::B_O_FULL + q));
                        }
                    }
                    if (!ok) break;
                    mma_commit(bar(C::B_SLOT_EMPTY + vslot));                   // V(j) done
                    if (has_next) mma_commit(bar(C::B_SLOT_EMPTY + kslot));   // K(j+1) done
                }
                mma_commit(bar(C::B_DRAIN));
                drain_wait(bar(C::B_DRAIN), 0);
            }
            __syncwarp();
        }
    } else {
        // ------------------------------------------------------------ softmax
        const int q = warp >> 3;        // head of the CTA
        const int h = (warp >> 2) & 1;  // key half of every tile
        const int wq = warp & 3;
        const int row = wq * 32 + lane;
        const int head = it.head0 + q;
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
        constexpr int O_COLS = C::D / 2;  // this warpgroup rescales / stores O's columns [h*64, h*64+64)
        const uint32_t s_tmem = lane_base + C::TMEM_S + q * C::BN + h * C::HALF;
        const uint32_t o_tmem = lane_base + C::TMEM_O + q * C::D + h * O_COLS;
        float* xmax = reinterpret_cast<float*>(smem + C::SMEM_XMAX) + q * 2 * 2 * C::BM;  // [2][2][BM]
        float* xl = reinterpret_cast<float*>(smem + C::SMEM_XL) + q * 2 * C::BM;          // [2][BM]

        bool ok = !skip;
        for (int j = 0; ok && j < n; ++j) {
            // S(j) ready; it also means PV(j-1) is in O.
            ok = warp_wait(bar(C::B_S_FULL + q), j & 1, abort_flag, p.status);
            if (!ok) break;
            tc_fence_after();
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
            for (int c = 4; c < C::HALF; c += 2) mx[(c >> 1) & 3] = max3f(mx[(c >> 1) & 3], sv[c], sv[c + 1]);
            float smax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            // Both halves apply the same running max to O: exchange the
            // partial maxima (double-buffered by tile parity; the halves meet
            // on this barrier every tile, so neither runs two tiles ahead).
            xmax[((j & 1) * 2 + h) * C::BM + row] = smax;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_XCH + q));
            ok = warp_wait(bar(C::B_XCH + q), j & 1, abort_flag, p.status);
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

            // P of this half's 64 keys over the first 32 columns of its S half.
            const float2 sl2x2 = make_float2(sl2, sl2);
            const float2 negm2 = make_float2(neg_m, neg_m);
            float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
            exp_and_store_p<0, C::HALF / 32, C::HALF, C::EXP_EMU>(sv, sl2x2, negm2, s_tmem, acc0, acc1);
            l += (acc0.x + acc0.y) + (acc1.x + acc1.y);

            // O holds PV(j-1) (S(j) is ready): rescale this half's columns
            // before PV(j), which waits for both halves' arrivals.
            if (j > 0 && __any_sync(0xffffffffu, rescale_o)) {
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
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_P_FULL + q));
        }

        // ---------------------------------------------------------- epilogue
        // Row sum = both halves' shares, exchanged on phase n of the exchange
        // barrier (the running max is already the same in both halves).
        if (ok) {
            xl[h * C::BM + row] = l;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::B_XCH + q));
            ok = warp_wait(bar(C::B_XCH + q), n & 1, abort_flag, p.status);
        }
        if (ok) {
            l += xl[(1 - h) * C::BM + row];
            ok = warp_wait(bar(C::B_O_FULL + q), 0, abort_flag, p.status);
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
    if (warp == C::MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

// Host check before the first launch (the kernel has no register split).
template <class C>
inline bool ksplit_launch_registers_ok() {
    return true;
}

}  // namespace thd
