// Packed-THD sliding-window GQA attention forward for B200 (sm_100a).
//
// One CTA computes one work item of the host tile schedule: a 128-row query
// tile of one document for NQ query heads that share one kv head (the
// repeat_kv grouping of the "muse_glimmer.model" page), against n_kv key
// tiles of BN keys.  Visible keys follow FlintMagiPlan.attention's window
// parameter ("flint.magi" page): s <= j <= i and (W == 0 or j > i - W) for a
// query i of document [s, e).  The per-head sink logit (FlintMagiPlan
// .attention, sink parameter) starts the running max/sum of every row and so
// joins the softmax denominator only.
//
// Warp roles (warp-specialised, all communication through mbarriers):
//   softmax warpgroups (one per query tile): thread t owns row t (= TMEM
//     lane t).  Reads S from TMEM, masks edge tiles, keeps the running max
//     and sum, rescales O in TMEM when the max grows by more than 2^8, and
//     writes P (bf16) back over S for O += P V.
//   control warpgroup: warp 0 is the TMA producer (Q tiles once, then K/V
//     tiles through a ring of 128-byte-swizzled shared-memory slots), warp 1
//     the MMA issuer: S = Q K^T (both operands from shared memory, K-major)
//     and O += P V (P from TMEM, V from shared memory, MN-major), fp32
//     accumulators in TMEM.
//
// TMEM columns: S[q][b] at (q*NSB + b)*BN (b < NSB buffers), O[q] after them.
// With NSB = 1 the MMA order QK(j) PV(j) QK(j+1) keeps S/P of one tile live;
// with NSB = 2, QK(j+1) runs while the softmax works on tile j.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "sm100_ptx.cuh"

#ifndef THD_EXP_EMU
#define THD_EXP_EMU 0
#endif

// 1: debug build.  Every forward CTA checks the work items it will run
// against the schedule's invariants before touching memory and, on a
// violation, records kStatusBadItem in the status word and does nothing
// (a status code instead of a trap or a fault).
#ifndef THD_DEBUG
#define THD_DEBUG 0
#endif



namespace thd {

struct WorkItem {  // identical layout to thd_work_item in thd_attn.h
    int32_t q0, q1, doc_start, head0;
    int32_t kv_start, n_kv, n_heads, block_n;
};

// Error code recorded in the device status word when a wait runs out.
constexpr int kStatusTimeout = -4;

template <int D_, int NQ_, int NSB_, int BN_, int NSLOT_>
struct FwdConfig {
    static constexpr int D = D_;
    static constexpr int NQ = NQ_;        // query tiles (heads) per CTA
    static constexpr int NSB = NSB_;      // S buffers per query tile
    static constexpr int BN = BN_;        // keys per key tile
    static constexpr int NSLOT = NSLOT_;  // K/V ring slots (one K or V tile each)
    static constexpr int BM = 128;        // query rows per tile (= TMEM lanes)
    // Element pairs (out of every 4) whose exponential runs on the FMA pipe.
    static constexpr int EXP_EMU = THD_EXP_EMU;

    static constexpr int KCH = D / 64;                 // 128-byte column chunks
    static constexpr int Q_BOX_BYTES = BM * 128;       // one chunk of a Q tile
    static constexpr int Q_TILE_BYTES = BM * D * 2;
    static constexpr int KV_BOX_BYTES = BN * 128;      // one chunk of a K/V tile
    static constexpr int KV_TILE_BYTES = BN * D * 2;

    static constexpr int TMEM_S = 0;
    static constexpr int TMEM_O = NQ * NSB * BN;
    static constexpr int TMEM_USED = TMEM_O + NQ * D;
    static constexpr int TMEM_COLS = TMEM_USED <= 32 ? 32 : TMEM_USED <= 64 ? 64
                                   : TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;

    // Warpgroups: NQ softmax warpgroups, then one control warpgroup whose
    // warp 0 is the TMA producer and warp 1 the MMA issuer (warps 2-3 idle).
    static constexpr int NUM_SOFTMAX_WARPS = 4 * NQ;
    static constexpr int PRODUCER_WARP = NUM_SOFTMAX_WARPS;
    static constexpr int MMA_WARP = NUM_SOFTMAX_WARPS + 1;
    static constexpr int NUM_THREADS = (NUM_SOFTMAX_WARPS + 4) * 32;
    // With three warpgroups a thread starts with 168 registers (3 warps per
    // SM sub-partition); the control warpgroup hands part of its share to the
    // softmax warpgroups: 2*128*192 + 128*120 = 384*168.  (With 208 / 88 the
    // control warps spilled; 192 / 120 spills nothing and measured 1-5 %
    // faster.)
    static constexpr bool REG_SPLIT = NQ == 2;
    static constexpr int LAUNCH_REGS = 168;
    static constexpr int SOFTMAX_REGS = 192;
    static constexpr int CONTROL_REGS = 120;
    static_assert(!REG_SPLIT || (NQ * 128 * SOFTMAX_REGS + 128 * CONTROL_REGS <=
                                 NUM_THREADS * LAUNCH_REGS), "register split exceeds the launch");

    // mbarrier indices
    static constexpr int B_Q_FULL = 0;
    static constexpr int B_SLOT_FULL = 1;
    static constexpr int B_SLOT_EMPTY = B_SLOT_FULL + NSLOT;
    static constexpr int B_S_FULL = B_SLOT_EMPTY + NSLOT;  // [NQ][NSB]
    static constexpr int B_P_FULL = B_S_FULL + NQ * NSB;   // [NQ][2] P (half) written, O rescaled
    static constexpr int B_O_FULL = B_P_FULL + 2 * NQ;     // PV done
    // With one S buffer per head the softmax publishes P in two halves (keys
    // [0, BN/2), then [BN/2, BN)), so PV starts on the first half while the
    // second half's exponentials still run (identical arithmetic).
    static constexpr bool P_SPLIT = NSB == 1;
    static constexpr int B_DRAIN = B_O_FULL + NQ;
    static constexpr int NUM_BARS = B_DRAIN + 1;

    // shared memory layout (offsets from a 1024-byte aligned base)
    static constexpr int SMEM_Q = 0;
    static constexpr int SMEM_SLOTS = SMEM_Q + NQ * Q_TILE_BYTES;
    static constexpr int SMEM_BAR = SMEM_SLOTS + NSLOT * KV_TILE_BYTES;
    static constexpr int SMEM_TMEM_SLOT = SMEM_BAR + NUM_BARS * 8;
    static constexpr int SMEM_ABORT = SMEM_TMEM_SLOT + 4;
    static constexpr int SMEM_BYTES = SMEM_ABORT + 4;
    static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;

    static_assert(D % 64 == 0 && D <= 256, "head dim must be 64, 128 or 256");
    static_assert(BN % 64 == 0 && BN <= 256, "key tile must be a multiple of 64");
    static_assert(TMEM_USED <= 512, "TMEM budget exceeded");
    static_assert(SMEM_ALLOC <= 232448, "shared memory budget exceeded");
    // Every wait of the MMA issuer is for a position whose slot was released
    // by an MMA it has already issued (V(j) is released right after PV(j),
    // K(j) right after QK(j)), so two slots already cannot deadlock; more
    // slots only let the producer run further ahead.
    static_assert(NSLOT >= 2, "K/V ring needs two slots");
};

struct FwdParams {
    const WorkItem* items;
    __nv_bfloat16* out;  // [T, Hq, D]
    float* lse;          // [T, Hq] or null
    const float* sinks;  // [Hq] or null
    int* status;         // device status word
    int Hq;
    int G;               // Hq / Hkv
    int window;
    float scale_log2;    // scale * log2(e)
    int q_offset;        // pack row of row 0 of q / out / lse (0 unless a token range)
    // Optional schedule check (allocation-free entry point): when set, the
    // launch runs only if *plan_tag equals expected_tag, i.e. the shared
    // scratch still holds the schedule this launch was enqueued for.
    const unsigned long long* plan_tag = nullptr;
    unsigned long long expected_tag = 0;
};

// Error code recorded when a launch finds another call's schedule in the
// allocation-free scratch (the launch then does nothing).
constexpr int kStatusStaleScratch = -7;

// Error code of the debug build's work-item checks.
constexpr int kStatusBadItem = -8;

// Debug build: the invariants every item of the host schedule satisfies
// (see scheduler.cpp): 1..128 query rows ending in the document, key tiles
// of block_n keys that end at the tile end (or before it, for a key-bounded
// range), whole GQA head groups of n_heads aligned heads inside [0, Hq).
__device__ __forceinline__ bool item_ok(const WorkItem& it, const FwdParams& p, int n_heads,
                                        int block_n) {
    return it.n_kv >= 1 && it.block_n == block_n && it.n_heads == n_heads &&
           it.q1 - it.q0 >= 1 && it.q1 - it.q0 <= 128 && it.doc_start < it.q1 &&
           it.q0 - p.q_offset >= -128 && it.kv_start + it.n_kv * block_n <= it.q1 &&
           it.head0 >= 0 && it.head0 % n_heads == 0 && it.head0 + n_heads <= p.Hq &&
           (it.head0 / p.G) == (it.head0 + n_heads - 1) / p.G;
}

// Debug build: record kStatusBadItem and return 1 if the item fails item_ok.
__device__ __forceinline__ int debug_check_item(const WorkItem& it, const FwdParams& p, int n_heads,
                                                int block_n) {
    if (THD_DEBUG && !item_ok(it, p, n_heads, block_n)) {
        atomicCAS(p.status, 0, kStatusBadItem);
        return 1;
    }
    return 0;
}

// CTA start-up decision, taken by one thread: skip the work if an earlier
// CTA or launch recorded an error that the host has not read yet, or if the
// schedule this launch was enqueued for is no longer in place.
__device__ __forceinline__ int launch_should_skip(const FwdParams& p) {
    if (p.plan_tag != nullptr &&
        *reinterpret_cast<const volatile unsigned long long*>(p.plan_tag) != p.expected_tag) {
        atomicCAS(p.status, 0, kStatusStaleScratch);
        return 1;
    }
    return *reinterpret_cast<volatile int*>(p.status) != 0 ? 1 : 0;
}

// Wait by lane 0 of the calling warp; the result is broadcast to the warp so
// that the warp-collective tcgen05 instructions after it stay convergent.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int* status) {
    int ok = 0;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort_flag, status, kStatusTimeout);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

// Bounded wait that ignores the abort flag: used while unwinding, to let
// operations already in flight finish before the CTA exits.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > kWaitLimitNs) return;
    }
}

// Exponentials of key columns [C0, C0 + 32*NCH) of one row: p = 2^(s*sl2 - m),
// two elements per packed FMA, summed into acc and written to TMEM as bf16
// pairs (key k goes to column k/2 of the S/P buffer).
// EMU of every 4 element pairs take the FMA-pipe polynomial instead of MUFU.
template <int C0, int NCH, int BN, int EMU>
__device__ __forceinline__ void exp_and_store_p(const float (&sv)[BN], float2 sl2x2, float2 negm2,
                                                uint32_t p_tmem, float2& acc0, float2& acc1) {
#pragma unroll
    for (int cc = 0; cc < NCH; ++cc) {
        uint32_t pk[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const int c = C0 + cc * 32 + 2 * u;
            const float2 x = __ffma2_rn(make_float2(sv[c], sv[c + 1]), sl2x2, negm2);
            float p0, p1;
            if ((u & 3) >= 4 - EMU) {
                const float2 e = exp2_poly2(x);
                p0 = e.x;
                p1 = e.y;
            } else {
                p0 = ex2_approx(x.x);
                p1 = ex2_approx(x.y);
            }
            if (u & 1) acc1 = __fadd2_rn(acc1, make_float2(p0, p1));
            else acc0 = __fadd2_rn(acc0, make_float2(p0, p1));
            pk[u] = pack_bf16x2(p0, p1);
        }
        tmem_st16(p_tmem + (C0 / 2) + cc * 16, pk);
    }
}

template <class C>
__global__ void __launch_bounds__(C::NUM_THREADS, 1)
thd_attn_fwd_kernel(const __grid_constant__ CUtensorMap tmap_q,
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
        for (int i = 0; i < C::NQ * C::NSB; ++i) mbar_init(bar(C::B_S_FULL + i), 1);
        for (int q = 0; q < C::NQ; ++q) {
            mbar_init(bar(C::B_P_FULL + 2 * q), 4);
            mbar_init(bar(C::B_P_FULL + 2 * q + 1), 4);
            mbar_init(bar(C::B_O_FULL + q), 1);
        }
        mbar_init(bar(C::B_DRAIN), 1);
        // A timeout recorded by an earlier CTA (or launch) makes every later
        // CTA skip its work until the host reads and clears the status.
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
      if constexpr (C::REG_SPLIT) regs_decrease<C::CONTROL_REGS>();
      if (warp == C::PRODUCER_WARP) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0 && !skip) {
            tma_prefetch_desc(&tmap_q);
            tma_prefetch_desc(&tmap_k);
            tma_prefetch_desc(&tmap_v);
            const int g = it.head0 / p.G;
            mbar_arrive_expect_tx(bar(C::B_Q_FULL), C::NQ * C::Q_TILE_BYTES);
            for (int q = 0; q < C::NQ; ++q)
                for (int c = 0; c < C::KCH; ++c)
                    tma_load_3d(sbase + C::SMEM_Q + q * C::Q_TILE_BYTES + c * C::Q_BOX_BYTES,
                                &tmap_q, bar(C::B_Q_FULL), c * 64, it.head0 + q, it.q0 - p.q_offset);
            // Ring positions: 2j holds K(j), 2j+1 holds V(j); position p uses
            // slot p % NSLOT.  A load waits only for the slot's previous tile.
            int issued = 0;
            bool ok = true;
            for (int pos = 0; pos < 2 * n && ok; ++pos) {
                const int slot = pos % C::NSLOT;
                ok = mbar_wait(bar(C::B_SLOT_EMPTY + slot), ((pos / C::NSLOT) & 1) ^ 1, abort_flag,
                               p.status, kStatusTimeout);
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
                // Only the last load issued into each slot can still be in
                // flight (earlier ones were consumed before the slot was reused).
                drain_wait(bar(C::B_Q_FULL), 0);
                for (int pos = issued - C::NSLOT > 0 ? issued - C::NSLOT : 0; pos < issued; ++pos)
                    drain_wait(bar(C::B_SLOT_FULL + pos % C::NSLOT), (pos / C::NSLOT) & 1);
            }
        }
        __syncwarp();
      } else if (warp == C::MMA_WARP) {
        // -------------------------------------------------------- MMA issuer
        if (lane == 0 && !skip) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, C::BN, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, C::D, true);
            // Descriptor bases; per instruction only the start address moves
            // (adding offset >> 4 to the low field cannot carry: shared
            // memory addresses stay below 2^18).
            const uint64_t dq0 = smem_desc_sw128(sbase + C::SMEM_Q, 16, 1024);
            const uint64_t dk0 = smem_desc_sw128(sbase + C::SMEM_SLOTS, 16, 1024);
            const uint64_t dv0 = smem_desc_sw128(sbase + C::SMEM_SLOTS, C::KV_BOX_BYTES, 1024);
            auto issue_qk = [&](int q, int b, int slot) {
                const uint32_t d_tmem = tmem_base + C::TMEM_S + (q * C::NSB + b) * C::BN;
                const uint64_t dq = dq0 + ((q * C::Q_TILE_BYTES) >> 4);
                const uint64_t dk = dk0 + ((slot * C::KV_TILE_BYTES) >> 4);
#pragma unroll
                for (int kk = 0; kk < C::D / 16; ++kk) {
                    // 16 bf16 = 32 bytes along K inside a 128-byte chunk
                    const uint32_t qo = ((kk >> 2) * C::Q_BOX_BYTES + (kk & 3) * 32) >> 4;
                    const uint32_t ko = ((kk >> 2) * C::KV_BOX_BYTES + (kk & 3) * 32) >> 4;
                    mma_bf16_ss(d_tmem, dq + qo, dk + ko, idesc_qk, kk > 0 ? 1u : 0u);
                }
            };
            // O += P V over the BN keys of one tile (K = 16 per instruction).
            auto issue_pv = [&](int q, int b, int slot, bool acc, int kk0 = 0, int kk1 = C::BN / 16) {
                const uint32_t d_tmem = tmem_base + C::TMEM_O + q * C::D;
                const uint32_t p_tmem = tmem_base + C::TMEM_S + (q * C::NSB + b) * C::BN;
                const uint64_t dv = dv0 + ((slot * C::KV_TILE_BYTES) >> 4);
#pragma unroll
                for (int kk = kk0; kk < kk1; ++kk) {
                    mma_bf16_ts(d_tmem, p_tmem + kk * 8, dv + ((kk * 16 * 128) >> 4), idesc_pv,
                                (acc || kk > 0) ? 1u : 0u);
                }
            };

            auto wait_slot = [&](int pos) -> bool {
                return mbar_wait(bar(C::B_SLOT_FULL + pos % C::NSLOT), (pos / C::NSLOT) & 1,
                                 abort_flag, p.status, kStatusTimeout);
            };
            bool ok = mbar_wait(bar(C::B_Q_FULL), 0, abort_flag, p.status, kStatusTimeout);
            for (int jj = 0; ok && jj < C::NSB && jj < n; ++jj) {
                ok = wait_slot(2 * jj);
                if (!ok) break;
                tc_fence_after();
                for (int q = 0; q < C::NQ; ++q) {
                    issue_qk(q, jj % C::NSB, (2 * jj) % C::NSLOT);
                    mma_commit(bar(C::B_S_FULL + q * C::NSB + jj % C::NSB));
                }
                mma_commit(bar(C::B_SLOT_EMPTY + (2 * jj) % C::NSLOT));
            }
            for (int j = 0; ok && j < n && C::NSB == 1; ++j) {
                // One S buffer per head: PV(j) and QK(j+1) of a head go out as
                // one run of 2 * 8 MMAs (QK(j+1) may overwrite S = P(j) only
                // after PV(j), which the in-order tensor pipe guarantees), with
                // one commit: S(j+1) ready also means O holds PV(j), so O gets
                // its own commit only after the last tile.  Fewer boundaries
                // between MMA runs keep the tensor pipe fed.
                const int vslot = (2 * j + 1) % C::NSLOT;
                const bool has_next = j + 1 < n;
                const int kslot = (2 * j + 2) % C::NSLOT;
                ok = wait_slot(2 * j + 1) && (!has_next || wait_slot(2 * j + 2));
                if (!ok) break;
                for (int q = 0; q < C::NQ && ok; ++q) {
                    ok = mbar_wait(bar(C::B_P_FULL + 2 * q), j & 1, abort_flag, p.status, kStatusTimeout);
                    if (!ok) break;
                    tc_fence_after();
                    if constexpr (C::P_SPLIT) {
                        issue_pv(q, 0, vslot, j > 0, 0, C::BN / 32);
                        ok = mbar_wait(bar(C::B_P_FULL + 2 * q + 1), j & 1, abort_flag, p.status,
                                       kStatusTimeout);
                        if (!ok) break;
                        tc_fence_after();
                        issue_pv(q, 0, vslot, true, C::BN / 32, C::BN / 16);
                    } else {
                        issue_pv(q, 0, vslot, j > 0);
                    }
                    if (has_next) {
                        issue_qk(q, 0, kslot);
                        mma_commit(bar(C::B_S_FULL + q));
                    } else {
                        mma_commit(bar(C::B_O_FULL + q));
                    }
                }
                if (!ok) break;
                mma_commit(bar(C::B_SLOT_EMPTY + vslot));                   // V(j) done
                if (has_next) mma_commit(bar(C::B_SLOT_EMPTY + kslot));   // K(j+1) done
            }
            for (int j = 0; ok && j < n && C::NSB == 2; ++j) {
                const int vslot = (2 * j + 1) % C::NSLOT;
                ok = wait_slot(2 * j + 1);
                if (!ok) break;
                const int jn = j + C::NSB;
                const bool has_next = jn < n;
                const int kslot = (2 * jn) % C::NSLOT;
                for (int q = 0; q < C::NQ && ok; ++q) {
                    ok = mbar_wait(bar(C::B_P_FULL + 2 * q), j & 1, abort_flag, p.status, kStatusTimeout);
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv(q, j % C::NSB, vslot, j > 0);
                    mma_commit(bar(C::B_O_FULL + q));
                    if (q == C::NQ - 1) mma_commit(bar(C::B_SLOT_EMPTY + vslot));  // V(j) done
                    if (has_next) {
                        if (q == 0) {
                            ok = wait_slot(2 * jn);
                            if (!ok) break;
                            tc_fence_after();
                        }
                        issue_qk(q, jn % C::NSB, kslot);
                        mma_commit(bar(C::B_S_FULL + q * C::NSB + jn % C::NSB));
                        if (q == C::NQ - 1) mma_commit(bar(C::B_SLOT_EMPTY + kslot));  // K(jn) done
                    }
                }
            }
            // Every MMA issued by this thread has completed once this lands.
            mma_commit(bar(C::B_DRAIN));
            drain_wait(bar(C::B_DRAIN), 0);
        }
        __syncwarp();
      }
    } else {
        // ------------------------------------------------------------ softmax
        if constexpr (C::REG_SPLIT) regs_increase<C::SOFTMAX_REGS>();
        const int q = warp >> 2;
        const int wq = warp & 3;
        const int row = wq * 32 + lane;
        const int h = it.head0 + q;
        const int i = it.q0 + row;  // token of this row
        const int s_doc = it.doc_start;
        const int r_lo = it.q0 > s_doc ? it.q0 : s_doc;
        const int r_hi = it.q1 - 1;
        const bool row_valid = i >= r_lo && i <= r_hi;
        const int W = p.window;
        const int lo_i = (W > 0 && i - W + 1 > s_doc) ? i - W + 1 : s_doc;
        const float sl2 = p.scale_log2;
        constexpr float kTau = 8.0f;  // rescale only when the max grows by > 2^8

        float m_ref = -INFINITY;
        float l = 0.0f;
        if (p.sinks != nullptr) {
            m_ref = p.sinks[h] * 1.4426950408889634f;
            l = 1.0f;
        }
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(wq * 32) << 16);
        const uint32_t o_tmem = lane_base + C::TMEM_O + q * C::D;

        bool ok = !skip;
        for (int j = 0; ok && j < n; ++j) {
            const int b = j % C::NSB;
            ok = warp_wait(bar(C::B_S_FULL + q * C::NSB + b), (j / C::NSB) & 1, abort_flag, p.status);
            if (!ok) break;
            tc_fence_after();
            const uint32_t s_tmem = lane_base + C::TMEM_S + (q * C::NSB + b) * C::BN;
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
            // Row max: 3-input max over pairs, four independent chains.
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

            // O must hold PV(j-1) before it is rescaled and before PV(j)
            // starts.  With one S buffer that is implied by S(j) being ready
            // (QK(j) was issued after PV(j-1)); with two it is waited for,
            // once per step: here if O is rescaled, else before P(j) is
            // published (which also keeps the P barriers from running two
            // phases ahead of the MMA issuer).
            const bool warp_rescale = j > 0 && __any_sync(0xffffffffu, rescale_o);
            bool o_ready = C::NSB == 1 || j == 0;
            if (warp_rescale) {
                if (!o_ready) {
                    ok = warp_wait(bar(C::B_O_FULL + q), (j - 1) & 1, abort_flag, p.status);
                    if (!ok) break;
                    tc_fence_after();
                    o_ready = true;
                }
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
            if constexpr (C::P_SPLIT) {
                // (one S buffer: O already holds PV(j-1), o_ready is true)
                exp_and_store_p<0, C::BN / 64, C::BN, C::EXP_EMU>(sv, sl2x2, negm2, s_tmem, acc0, acc1);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(C::B_P_FULL + 2 * q));
                exp_and_store_p<C::BN / 2, C::BN / 64, C::BN, C::EXP_EMU>(sv, sl2x2, negm2, s_tmem,
                                                                         acc0, acc1);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(C::B_P_FULL + 2 * q + 1));
            } else {
                exp_and_store_p<0, C::BN / 32, C::BN, C::EXP_EMU>(sv, sl2x2, negm2, s_tmem, acc0, acc1);
                tmem_wait_st();
                if (!o_ready) {
                    ok = warp_wait(bar(C::B_O_FULL + q), (j - 1) & 1, abort_flag, p.status);
                    if (!ok) break;
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(C::B_P_FULL + 2 * q));
            }
            l += (acc0.x + acc0.y) + (acc1.x + acc1.y);
        }

        // With one S buffer O_FULL completes once (after the last PV); with
        // two, once per tile.
        if (ok) ok = warp_wait(bar(C::B_O_FULL + q), C::NSB == 1 ? 0u : (n - 1) & 1, abort_flag, p.status);
        if (ok) {
            tc_fence_after();
            const float inv_l = l > 0.0f ? 1.0f / l : 0.0f;
            __nv_bfloat16* orow = p.out + (static_cast<int64_t>(i - p.q_offset) * p.Hq + h) * C::D;
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
                p.lse[static_cast<int64_t>(i - p.q_offset) * p.Hq + h] =
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

// Host check before the first launch of a shape: the register split above
// assumes the kernel starts with LAUNCH_REGS registers per thread; with fewer,
// setmaxnreg.inc could never be satisfied.
template <class C>
inline bool launch_registers_ok() {
    if constexpr (!C::REG_SPLIT) {
        return true;
    } else {
        cudaFuncAttributes a{};
        if (cudaFuncGetAttributes(&a, thd_attn_fwd_kernel<C>) != cudaSuccess) return false;
        return a.numRegs >= C::LAUNCH_REGS;
    }
}

}  // namespace thd
