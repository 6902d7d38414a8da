// Expert parallelism: the layer's routed experts spread over `world` ranks, rank
// r holding experts [r * E/world, (r + 1) * E/world) ("DeepSeek-V3 notes"
// (knlb.dev), § infrastructure: expert parallelism with all-to-all dispatch and
// combine between the ranks; § architecture: a token is sent to a limited number
// of nodes — with contiguous expert blocks per rank and groups that do not
// straddle ranks, to at most topk_group ranks).
//
// A token crosses to a rank once, however many of its experts live there: the
// source sends one row per (token, destination rank) and the destination runs
// all of the token's experts it was sent and sums their weighted outputs before
// sending one row back.  An expert may live on several ranks (redundant copies
// of heavily loaded experts, "DeepSeek-V3 notes" § infrastructure, prefilling:
// redundant experts placed from live load statistics): slot (t, j) of expert e
// then goes to replica t mod n_e of e's n_e ranks, which splits e's rows evenly
// over its copies.  These kernels build the source side's rows; the row sort
// (dispatch.cuh) and the combine (combine.cuh) do the rest:
//   ep_rank_slots:  per slot, its destination rank, and the same rank again
//                   where the slot is the first of its token's slots bound for
//                   that rank (else -1: the token already has a row there);
//   ep_send_meta:   after the rows are sorted by destination, each row's routing
//                   data behind its H values — the token's k expert ids, each
//                   replaced by -1 unless that slot goes to this row's rank, and
//                   the k weights — and the number of rows for each rank.
#pragma once
#include <cstdint>

#include "device_status.cuh"

namespace moe {

// The rank that slot (t, j) of expert e is sent to: e's block without a placement
// table, else replica t mod n_e of the ranks listed for e (expert_ranks[e * max_rep
// + i], the first n_e entries >= 0).  -1 for a bad id or table entry (recorded).
__device__ __forceinline__ int slot_rank(int e, int64_t t, int E, int experts_per_rank,
                                         const int32_t* __restrict__ expert_ranks, int max_rep, int world) {
    if (static_cast<unsigned>(e) >= static_cast<unsigned>(E)) {
        record_error(kErrExpertId);
        return -1;
    }
    if (!expert_ranks) return e / experts_per_rank;
    const int32_t* reps = expert_ranks + static_cast<int64_t>(e) * max_rep;
    int n = 0;
    while (n < max_rep && reps[n] >= 0) ++n;
    const int d = n > 0 ? reps[t % n] : -1;
    if (static_cast<unsigned>(d) >= static_cast<unsigned>(world)) {
        record_error(kErrExpertId);
        return -1;
    }
    return d;
}

// One thread per token; K <= 32.  slot_dest[t, j] = the slot's rank (-1 for no
// row); rank_slot[t, j] = the same where j is the token's first slot bound there.
__global__ void __launch_bounds__(256) ep_rank_slots_kernel(const int32_t* __restrict__ topk_idx, int64_t T, int K,
                                                            int experts_per_rank, int E,
                                                            const int32_t* __restrict__ expert_ranks, int max_rep,
                                                            int world, int32_t* __restrict__ slot_dest,
                                                            int32_t* __restrict__ rank_slot) {
    const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (t >= T) return;
    const int32_t* in = topk_idx + t * K;
    unsigned seen[8] = {0, 0, 0, 0, 0, 0, 0, 0};  // ranks already given a row (world <= E <= 256)
    for (int j = 0; j < K; ++j) {
        const int r = slot_rank(in[j], t, E, experts_per_rank, expert_ranks, max_rep, world);
        int d = -1;
        if (r >= 0) {
            const unsigned bit = 1u << (r & 31);
            if (!(seen[r >> 5] & bit)) {
                seen[r >> 5] |= bit;
                d = r;
            }
        }
        slot_dest[t * K + j] = r;
        rank_slot[t * K + j] = d;
    }
}

// Rows [0, offsets[world]) of the send buffer (row_bytes apart): row r holds
// slot perm_src[r] = t * K + j0's token t, bound for rank slot_dest[t, j0]; its
// routing data goes at byte meta_off of the row: K int32 expert ids (slot j's id
// where slot_dest[t, j] is this row's rank, else -1), K fp32 weights, zeros up to
// meta_words words.  Threads cover (row, word) pairs of the rows' bound n_max;
// block 0 also writes counts[d] = offsets[d + 1] - offsets[d].
__global__ void __launch_bounds__(256) ep_send_meta_kernel(const int32_t* __restrict__ offsets, int world,
                                                           const int32_t* __restrict__ perm_src, int64_t n_slots,
                                                           int K, const int32_t* __restrict__ topk_idx,
                                                           const float* __restrict__ topk_w,
                                                           const int32_t* __restrict__ slot_dest, int64_t n_max,
                                                           uint8_t* __restrict__ rows, int64_t row_bytes,
                                                           int64_t meta_off, int meta_words,
                                                           int32_t* __restrict__ counts) {
    if (blockIdx.x == 0)
        for (int d = threadIdx.x; d < world; d += blockDim.x) counts[d] = offsets[d + 1] - offsets[d];
    const int64_t used = offsets[world];
    const int64_t n = n_max * meta_words;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / meta_words;
        const int w = static_cast<int>(i - r * meta_words);
        if (r >= used) break;
        const int64_t src = perm_src[r];
        uint32_t v = 0;
        if (src < 0 || src >= n_slots) {
            if (w == 0) record_error(kErrRowIndex);
        } else if (w < 2 * K) {
            const int64_t t = src / K;
            if (w < K) {
                const bool here = slot_dest[t * K + w] == slot_dest[src];
                v = here ? static_cast<uint32_t>(topk_idx[t * K + w]) : 0xffffffffu;
            } else {
                v = __float_as_uint(topk_w[t * K + (w - K)]);
            }
        }
        reinterpret_cast<uint32_t*>(rows + r * row_bytes + meta_off)[w] = v;
    }
}

}  // namespace moe
