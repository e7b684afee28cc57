// Host tile scheduler: see scheduler.h.
#include "scheduler.h"

#include <algorithm>

namespace thd {

bool choose_kernel_shape(int D, int group, KernelShape* out) {
    // One CTA per item with two heads of one kv group (even group) or one
    // head; at D = 256 with an even group, the CTA-pair kernel with the
    // key-split softmax (one head per CTA, two per item), whose M = 256
    // instructions keep N = 256 PV and N = 128 QK at the tensor core's full
    // rate.  (At D = 128 every CTA-pair design measured slower than the
    // one-CTA kernel, including one with whole score rows and two heads per
    // CTA: there the tensor core waits on the softmax, and the pair's
    // cross-CTA signals lengthen that chain.)
    const bool two = (group % 2) == 0;
    switch (D) {
        case 64:
            *out = two ? KernelShape{64, 2, 1, 128, 8, false} : KernelShape{64, 1, 2, 128, 8, false};
            return true;
        case 128:
            *out = two ? KernelShape{128, 2, 1, 128, 5, false} : KernelShape{128, 1, 2, 128, 6, false};
            return true;
        case 256:
            *out = two ? KernelShape{256, 2, 2, 128, 4, true} : KernelShape{256, 1, 2, 64, 5, false};
            return true;
        default:
            return false;
    }
}

int validate_args(const int32_t* cu_seqlens, int n_docs, int Hq, int Hkv, int D, int window) {
    if (n_docs < 0 || cu_seqlens == nullptr) return THD_ERR_INVALID_ARG;
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return THD_ERR_INVALID_ARG;
    if (window < 0) return THD_ERR_INVALID_ARG;
    if (cu_seqlens[0] != 0) return THD_ERR_INVALID_ARG;
    for (int d = 0; d < n_docs; ++d)
        if (cu_seqlens[d + 1] < cu_seqlens[d]) return THD_ERR_INVALID_ARG;
    if (D != 64 && D != 128 && D != 256) return THD_ERR_UNSUPPORTED;
    return THD_OK;
}

int kv_groups_per_chunk(int64_t T, int D, int Hkv) {
    // K and V of one kv head over the whole pack, bf16.
    const int64_t per_group = T * static_cast<int64_t>(D) * 2 * 2;
    constexpr int64_t kL2Budget = 48ll << 20;  // well inside the 126 MB L2
    int64_t c = per_group > 0 ? kL2Budget / per_group : Hkv;
    if (c < 1) c = 1;
    if (c > Hkv) c = Hkv;
    return static_cast<int>(c);
}

std::vector<thd_work_item> build_plan(const int32_t* cu, int n_docs, int Hq, int Hkv, int window,
                                      const KernelShape& ks) {
    return build_plan_range(cu, n_docs, 0, cu[n_docs], Hq, Hkv, window, ks);
}

std::vector<thd_work_item> build_plan_range(const int32_t* cu, int n_docs, int64_t q_begin,
                                            int64_t q_end, int Hq, int Hkv, int window,
                                            const KernelShape& ks, int64_t k_end) {
    constexpr int BM = 128;
    const int G = Hq / Hkv;
    const int BN = ks.block_n;
    std::vector<thd_work_item> items;
    size_t n_tiles = 0;
    for (int d = 0; d < n_docs; ++d) n_tiles += (cu[d + 1] - cu[d] + BM - 1) / BM + 1;
    items.reserve(n_tiles * static_cast<size_t>(Hq / ks.nq));

    for (int d = 0; d < n_docs; ++d) {
        const int s = cu[d], e = cu[d + 1];
        // The document's rows inside the range: [a, b).
        const int a = static_cast<int>(s > q_begin ? s : q_begin);
        const int b = static_cast<int>(e < q_end ? e : q_end);
        // Query tiles are aligned to the END of those rows, so a ragged tile
        // is the first (shortest key range) rather than the last; a tile that
        // would reach before a range start q_begin > 0 starts at q_begin
        // (fewer than 128 rows) so that no row outside the range is loaded.
        for (int q1 = b; q1 > a; q1 -= BM) {
            int q0 = q1 - BM;
            if (q_begin > 0 && q0 < q_begin) q0 = static_cast<int>(q_begin);
            const int r_lo = q0 > s ? q0 : s;
            int k_lo = s;  // lowest key any row of the tile can see
            if (window > 0 && r_lo - window + 1 > k_lo) k_lo = r_lo - window + 1;
            // Key tiles are aligned to the end of the keys the tile may read
            // (its end, or k_end before it): the last one sits on the causal
            // diagonal, keys below k_lo in the first one are masked.
            const int kv_end = static_cast<int>(q1 < k_end ? q1 : k_end);
            int n_kv = (kv_end - k_lo + BN - 1) / BN;
            if (n_kv < 1) n_kv = 1;  // no key below k_end: one wholly masked tile
            const int kv_start = kv_end - n_kv * BN;
            for (int g = 0; g < Hkv; ++g)
                for (int hp = 0; hp < G / ks.nq; ++hp)
                    items.push_back(thd_work_item{q0, q1, s, g * G + hp * ks.nq, kv_start, n_kv,
                                                  ks.nq, BN});
        }
    }
    // Kv groups in chunks whose K/V fits in L2, longest first within a chunk.
    // The CTAs in flight then read the K/V of a few kv heads only instead of
    // every group of the longest documents at once; where the whole pack's
    // K/V fits, this is plain longest-first (the best load balance).  The
    // stable sort keeps the items of one (query tile, kv group) adjacent.
    const int c = kv_groups_per_chunk(cu[n_docs], ks.D, Hkv);
    std::stable_sort(items.begin(), items.end(), [G, c](const thd_work_item& a, const thd_work_item& b) {
        const int ca = a.head0 / G / c, cb = b.head0 / G / c;
        if (ca != cb) return ca < cb;
        return a.n_kv > b.n_kv;
    });
    return items;
}

std::vector<thd_bwd_kv_item> build_bwd_kv_plan(const int32_t* cu, int n_docs, int Hq, int Hkv,
                                               int D, int window) {
    constexpr int BT = 128;
    std::vector<thd_bwd_kv_item> items;
    for (int d = 0; d < n_docs; ++d) {
        const int s = cu[d], e = cu[d + 1];
        for (int k0 = s; k0 < e; k0 += BT) {
            // Queries that see a key of [k0, k0 + 128): [k0, q_end), q_end =
            // the document end, or one past k0 + 127 + (W - 1) with a window.
            int64_t q_end = e;
            if (window > 0 && static_cast<int64_t>(k0) + 127 + window < q_end)
                q_end = static_cast<int64_t>(k0) + 127 + window;
            const int n_q = static_cast<int>((q_end - k0 + BT - 1) / BT);
            for (int g = 0; g < Hkv; ++g)
                items.push_back(thd_bwd_kv_item{k0, s, e, g, n_q, 0, 0, 0});
        }
    }
    // A dk/dv item streams the Q and dO rows of its group's G query heads,
    // G times the bytes of the group's K and V: chunk the groups by that
    // footprint, so that the CTAs in flight share the query tiles they read
    // in L2.
    const int64_t G = Hkv > 0 ? Hq / Hkv : 1;
    const int64_t per_group = static_cast<int64_t>(cu[n_docs]) * G * D * 2 * 2;
    constexpr int64_t kL2Budget = 48ll << 20;  // as for the forward's K / V
    int64_t cc = per_group > 0 ? kL2Budget / per_group : Hkv;
    if (cc < 1) cc = 1;
    if (cc > Hkv) cc = Hkv;
    const int c = static_cast<int>(cc);
    std::stable_sort(items.begin(), items.end(),
                     [c](const thd_bwd_kv_item& a, const thd_bwd_kv_item& b) {
                         if (a.g / c != b.g / c) return a.g / c < b.g / c;
                         return a.n_q > b.n_q;
                     });
    return items;
}

}  // namespace thd
