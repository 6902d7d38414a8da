// Expert parallelism: the layer's routed experts spread over `world` ranks, rank
// r holding experts [r * E/world, (r + 1) * E/world) ("DeepSeek-V3 notes"
// (knlb.dev), § infrastructure: expert parallelism with all-to-all dispatch and
// combine between the ranks; § architecture: a token is sent to a limited number
// of nodes, which with contiguous expert blocks per rank is the topk_group limit).
// The exchange itself is a collective of the caller's communication library;
// these kernels prepare and consume its buffers:
//   ep_pack:          after moe_dispatch (rows in expert order, so the rows for
//                     rank d are one contiguous block), the per-expert row counts
//                     and each row's routing weight in row order, both sent along
//                     with the rows;
//   ep_recv_offsets:  the received per-(source rank, local expert) counts turned
//                     into segment offsets for the grouped GEMMs (segments in
//                     source-major order, which is the order the rows arrive in).
#pragma once
#include <cstdint>

#include "device_status.cuh"

namespace moe {

// Block 0 also writes the E per-expert counts; every thread handles rows of the
// routed row space [0, n_rows): w_perm[r] = topk_w[perm_src[r]] for the rows of
// some expert segment, 0 past them (rows skipped by the dispatch).
__global__ void __launch_bounds__(256) ep_pack_kernel(const int32_t* __restrict__ offsets, int E,
                                                      const int32_t* __restrict__ perm_src,
                                                      const float* __restrict__ topk_w, int64_t n_rows,
                                                      int32_t* __restrict__ counts, float* __restrict__ w_perm) {
    if (blockIdx.x == 0)
        for (int e = threadIdx.x; e < E; e += blockDim.x) counts[e] = offsets[e + 1] - offsets[e];
    const int64_t used = offsets[E];
    for (int64_t r = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; r < n_rows;
         r += (int64_t)gridDim.x * blockDim.x)
        w_perm[r] = r < used ? row_weight(perm_src, topk_w, r, n_rows) : 0.0f;
}

// One block: offsets[0] = 0, offsets[s + 1] = offsets[s] + counts[s] for the
// n = world * E/world segments (n <= 256).  A negative count is recorded and
// taken as 0.
__global__ void __launch_bounds__(256) ep_recv_offsets_kernel(const int32_t* __restrict__ counts, int n,
                                                              int32_t* __restrict__ offsets) {
    __shared__ int warp_sums[8];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int v = tid < n ? counts[tid] : 0;
    if (v < 0) {
        record_error(kErrSegment);
        v = 0;
    }
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += warp_sums[w];
    if (tid == 0) offsets[0] = 0;
    if (tid < n) offsets[tid + 1] = base + incl;
}

}  // namespace moe
