// Token -> expert dispatch.  The teaching code of "The Evolving Transformer · 07"
// (§ 02, MoE.forward) selects, expert by expert and slot by slot, the tokens
// routed to that expert and gathers their rows; here the same grouping is done
// for all experts at once as a stable counting sort:
//   1. count:  per block of kDispTok tokens, how many slots go to each expert;
//   2. scan:   per expert, each block's starting row inside the expert's segment
//              and the expert's total (one warp per expert);
//   3. place:  expert offsets from the totals (optionally each segment padded to
//              a multiple of 128 rows), then the stable rank of every slot
//              (ascending (t, j)) -> row_of / perm_src;
//   4. scatter: each token's row is read once from x and written to its k rows
//              of x_perm with 16-byte vector stores.
// Routing indices come from the caller (moe_dispatch takes topk_idx as an
// argument): an index outside [0, E) is skipped — not counted, no row, row_of = -1
// — and recorded in the device error word (kErrExpertId).
//
// The same four kernels sort the rows of the expert-parallel exchange, where a
// slot's entry may name a bucket that is not this sort's (another rank's expert,
// or a destination rank the token already has a row for): SlotIndex says where
// slot (t, j)'s entry lives and which of its values are buckets, which have no
// row, and which are caller errors.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "device_status.cuh"

namespace moe {

constexpr int kDispTok = 32;      // tokens per dispatch block
constexpr int kDispThreads = 256;

// Slot (t, j)'s entry is v = idx[t * ld + j].  Its bucket is map[v] (map set) or
// v - base, when that lies in [0, E) (E is the kernel's bucket count); otherwise
// the slot has no row.  A value outside [lo, hi) is recorded in the device error
// word, except -1 when lo = -1 (a slot marked as having no row here); with
// `strict`, so is a value in [0, hi) that names no bucket.  The layer's dispatch
// uses {topk_idx, k, 0, 0, E}.
struct SlotIndex {
    const int32_t* idx;
    int ld;
    int base, lo, hi;
    const int32_t* map = nullptr;
    int strict = 0;
};

// The bucket of a slot's entry, or -1 (no row; caller errors recorded).
__device__ __forceinline__ int slot_bucket(const SlotIndex& s, int v, int E) {
    if (v < s.lo || v >= s.hi) {
        record_error(kErrExpertId);
        return -1;
    }
    if (v < 0) return -1;
    const int b = s.map ? s.map[v] : v - s.base;
    if (static_cast<unsigned>(b) < static_cast<unsigned>(E)) return b;
    if (s.strict) record_error(kErrExpertId);
    return -1;
}

// Per-block expert counts, stored expert-major: block_counts[e * nb + b].
__global__ void __launch_bounds__(kDispThreads) dispatch_count_kernel(
    SlotIndex si, int T, int K, int E, int32_t* __restrict__ block_counts) {
    extern __shared__ int cnt[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    const int t0 = blockIdx.x * kDispTok;
    const int n = min(kDispTok, T - t0) * K;
    const int32_t* idx = si.idx + (int64_t)t0 * si.ld;
    for (int q = threadIdx.x; q < n; q += blockDim.x) {
        const int tl = q / K;
        const int e = slot_bucket(si, idx[(int64_t)tl * si.ld + (q - tl * K)], E);
        if (e >= 0) atomicAdd(&cnt[e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        block_counts[(int64_t)e * gridDim.x + blockIdx.x] = cnt[e];
}

// One warp per expert: exclusive prefix of its counts over the blocks (the row
// each block starts at inside the expert's segment) and the expert's total.
__global__ void __launch_bounds__(256) dispatch_scan_kernel(const int32_t* __restrict__ block_counts, int nb,
                                                            int E, int32_t* __restrict__ block_base,
                                                            int32_t* __restrict__ totals) {
    const int lane = threadIdx.x & 31;
    const int e = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (e >= E) return;
    const int32_t* c = block_counts + (int64_t)e * nb;
    int32_t* out = block_base + (int64_t)e * nb;
    int carry = 0;
    for (int b0 = 0; b0 < nb; b0 += 32) {
        const int v = b0 + lane < nb ? c[b0 + lane] : 0;
        int incl = v;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += o;
        }
        if (b0 + lane < nb) out[b0 + lane] = carry + incl - v;
        carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) totals[e] = carry;
}

// w_src / w_perm (both null, or both set): w_perm[row] = w_src[t * ld + j] for the
// row slot (t, j) lands on (weights laid out like the entries).
__global__ void __launch_bounds__(kDispThreads) dispatch_place_kernel(
    SlotIndex si, int T, int K, int E, const int32_t* __restrict__ block_base,
    const int32_t* __restrict__ totals, int pad, int32_t* __restrict__ offsets, int32_t* __restrict__ perm_src,
    int32_t* __restrict__ row_of, const float* __restrict__ w_src = nullptr, float* __restrict__ w_perm = nullptr) {
    extern __shared__ int smem_i[];
    int* run = smem_i;              // [E] next free row of each expert for this block
    __shared__ int warp_sums[kDispThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int kWarps = kDispThreads / 32;
    // Expert offsets: exclusive scan of the totals (E <= 256 = one value per thread),
    // each segment rounded up to a multiple of `pad` rows (1, or 128 for MXFP8
    // operands whose scale atoms cover 128 rows).
    const int tot = tid < E ? (totals[tid] + pad - 1) / pad * pad : 0;
    int incl = tot;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += warp_sums[w];
    const int excl = base + incl - tot;
    if (tid < E) {
        run[tid] = excl + block_base[(int64_t)tid * gridDim.x + blockIdx.x];
        if (blockIdx.x == 0) {
            offsets[tid] = excl;
            if (tid == E - 1) offsets[E] = excl + tot;
        }
    }
    __syncthreads();
    const int t0 = blockIdx.x * kDispTok;
    const int ntok = min(kDispTok, T - t0);
    const int n = ntok * K;
    const int64_t q0 = (int64_t)t0 * K;
    const unsigned lt_mask = (1u << lane) - 1u;

    for (int r0 = 0; r0 < n; r0 += kDispThreads) {
        const int q = r0 + tid;
        const bool in_range = q < n;
        const int tl = q / K;
        const int64_t src = (int64_t)(t0 + tl) * si.ld + (q - tl * K);
        int e = in_range ? slot_bucket(si, si.idx[src], E) : -1;
        const bool valid = e >= 0;
        if (!valid) e = -1 - lane;  // lanes without a bucket never match another lane
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int lrank = __popc(peers & lt_mask);
        const bool leader = lrank == 0;
        const int wcnt = __popc(peers);
        int row = 0;
        // Warps take their turn in order, so ranks follow ascending slot index.
        for (int w = 0; w < kWarps; ++w) {
            if (warp == w && valid) {
                const int base = run[e];
                __syncwarp(peers);
                if (leader) run[e] = base + wcnt;
                row = base + lrank;
            }
            __syncthreads();
        }
        if (valid) {
            row_of[q0 + q] = row;
            perm_src[row] = (int32_t)(q0 + q);
            if (w_perm) w_perm[row] = w_src[src];
        } else if (in_range) {
            row_of[q0 + q] = -1;
        }
    }
}

// Row copy: block (t, c) moves 16-byte slices [256 c, 256 c + 256) of token t's
// row; each slice is loaded once and stored to the token's k rows of x_perm
// (slots the place step left without a row, row_of = -1, are skipped).
// The grid is T x ceil(H / 2048) blocks, so small batches still spread over
// every SM.  x_ld / out_ld: row strides in elements (H for dense rows; the
// expert-parallel rows carry routing data after their H values), multiples of 8.
__global__ void __launch_bounds__(256) dispatch_scatter_kernel(const __nv_bfloat16* __restrict__ x,
                                                               const int32_t* __restrict__ row_of, int K,
                                                               int H, __nv_bfloat16* __restrict__ x_perm,
                                                               int64_t x_ld, int64_t out_ld) {
    __shared__ int rows[32];
    const int t = blockIdx.x;
    if (threadIdx.x < K) rows[threadIdx.x] = row_of[(int64_t)t * K + threadIdx.x];
    __syncthreads();
    const int c = blockIdx.y * 256 + threadIdx.x;
    if (c >= H / 8) return;
    const uint4 v = reinterpret_cast<const uint4*>(x + (int64_t)t * x_ld)[c];
    for (int j = 0; j < K; ++j)
        if (rows[j] >= 0) reinterpret_cast<uint4*>(x_perm + (int64_t)rows[j] * out_ld)[c] = v;
}

}  // namespace moe
