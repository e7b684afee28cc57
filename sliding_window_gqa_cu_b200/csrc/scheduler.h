// Host-side tile scheduler for the packed-THD attention forward.
//
// Turns the document boundaries of a pack (cu_seqlens, "CPU int32 padded
// document boundaries [documents + 1]" in _build_magi_plan) plus the window
// into the list of work items the kernel runs: one per (128-row query tile,
// group of query heads sharing a kv head).  The plan is the B200 counterpart
// of a per-microbatch Magi plan: built once per pack and reused by every
// layer that shares the same boundaries and window.
#pragma once

#include <cstdint>
#include <vector>

#include "../../include/thd_attn.h"

namespace thd {

// Kernel shape chosen for a head dim and GQA group size.
struct KernelShape {
    int D;
    int nq;       // query heads per work item (1 or 2)
    int nsb;      // S buffers per query tile
    int block_n;  // keys per key tile
    int nslot;    // K/V ring slots (one K or V tile each)
    bool pair;    // CTA-pair kernel (nq heads split over two CTAs)
};

// Returns false if the head dim is unsupported.
bool choose_kernel_shape(int D, int group, KernelShape* out);

// Number of consecutive kv groups whose items the plan mixes (longest first
// among them): as many as keep their K/V (T x D bf16 each for K and V) within
// 48 MB, at least one.
int kv_groups_per_chunk(int64_t T, int D, int Hkv);

// Host argument checks shared by every entry point (no CUDA calls).
int validate_args(const int32_t* cu_seqlens, int n_docs, int Hq, int Hkv, int D, int window);

// Builds the work list (kv head by kv head, longest first within a head).
// cu_seqlens must have passed validate_args.
std::vector<thd_work_item> build_plan(const int32_t* cu_seqlens, int n_docs, int Hq, int Hkv,
                                      int window, const KernelShape& ks);

// The same for the query rows [q_begin, q_end) of the pack only (keys from
// the whole pack): the local step of a context-parallel forward whose rank
// owns those rows.  build_plan is the range [0, T).  With k_end < T the rows
// see only keys j < k_end (the part of a context-parallel row that lies on
// earlier ranks): a tile's key range then ends at min(tile end, k_end), and a
// tile whose rows see no such key keeps one key tile, wholly masked.
std::vector<thd_work_item> build_plan_range(const int32_t* cu_seqlens, int n_docs, int64_t q_begin,
                                            int64_t q_end, int Hq, int Hkv, int window,
                                            const KernelShape& ks, int64_t k_end = INT64_MAX);

// Key-side work list of the backward (dk, dv): one item per (128-key tile of
// a document, kv head), with the query tiles that see any of its keys; same
// chunked kv-group order, longest first within a chunk.
std::vector<thd_bwd_kv_item> build_bwd_kv_plan(const int32_t* cu_seqlens, int n_docs, int Hq,
                                               int Hkv, int D, int window);

}  // namespace thd
