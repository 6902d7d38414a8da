// Expert parallelism: the layer's routed experts spread over `world` ranks, rank
// r holding experts [r * E/world, (r + 1) * E/world) ("DeepSeek-V3 notes"
// (knlb.dev), § infrastructure: expert parallelism with all-to-all dispatch and
// combine between the ranks; § architecture: a token is sent to a limited number
// of nodes — with contiguous expert blocks per rank and groups that do not
// straddle ranks, to at most topk_group ranks).
//
// A token crosses to a rank once, however many of its experts live there: the
// source sends one row per (token, destination rank) and the destination runs
// all of the token's experts it holds and sums their weighted outputs before
// sending one row back.  These kernels build the source side's rows; the row
// sort (dispatch.cuh) and the combine (combine.cuh) do the rest:
//   ep_rank_slots:  per token, slot j's destination rank when slot j is the
//                   first of the token's slots on that rank, else -1;
//   ep_send_meta:   after the rows are sorted by destination, each row's routing
//                   data (the token's k expert ids and k weights) behind its H
//                   values, and the number of rows for each rank.
#pragma once
#include <cstdint>

#include "device_status.cuh"

namespace moe {

// One thread per token; K <= 32.  An expert id outside [0, E) is recorded and
// gives no row.
__global__ void __launch_bounds__(256) ep_rank_slots_kernel(const int32_t* __restrict__ topk_idx, int64_t T, int K,
                                                            int experts_per_rank, int E,
                                                            int32_t* __restrict__ rank_slot) {
    const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (t >= T) return;
    const int32_t* in = topk_idx + t * K;
    int32_t* out = rank_slot + t * K;
    unsigned seen[8] = {0, 0, 0, 0, 0, 0, 0, 0};  // ranks already given a row (world <= E <= 256)
    for (int j = 0; j < K; ++j) {
        const int e = in[j];
        int d = -1;
        if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) {
            const int r = e / experts_per_rank;
            const unsigned bit = 1u << (r & 31);
            if (!(seen[r >> 5] & bit)) {
                seen[r >> 5] |= bit;
                d = r;
            }
        } else {
            record_error(kErrExpertId);
        }
        out[j] = d;
    }
}

// Rows [0, offsets[world]) of the send buffer (row_bytes apart): row r holds
// slot perm_src[r] = t * K + j's token t; its routing data goes at byte meta_off
// of the row: K int32 expert ids, K fp32 weights, zeros up to meta_words words.
// Threads cover (row, word) pairs of the rows' bound n_max; block 0 also writes
// counts[d] = offsets[d + 1] - offsets[d].
__global__ void __launch_bounds__(256) ep_send_meta_kernel(const int32_t* __restrict__ offsets, int world,
                                                           const int32_t* __restrict__ perm_src, int64_t n_slots,
                                                           int K, const int32_t* __restrict__ topk_idx,
                                                           const float* __restrict__ topk_w, int64_t n_max,
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
            v = w < K ? static_cast<uint32_t>(topk_idx[t * K + w]) : __float_as_uint(topk_w[t * K + (w - K)]);
        }
        reinterpret_cast<uint32_t*>(rows + r * row_bytes + meta_off)[w] = v;
    }
}

}  // namespace moe
