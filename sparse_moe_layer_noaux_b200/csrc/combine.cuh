// Combine: y[t] = shared_out[t] + sum_j w_j * expert_j(x[t]).  The routing
// weights are already applied by the down-projection epilogue, so this is a
// gather of k + 1 rows per token summed in fp32 in a fixed order (shared first,
// then slots 0..k-1) — the page's `output[mask] += w * expert_out` followed by
// `shared_expert_out + output` ("The Evolving Transformer · 07", § 02 / § 03),
// without atomics and therefore deterministic.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

namespace moe {

__device__ __forceinline__ void acc_bf16x8(float (&acc)[8], const uint4& v) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float2 f = __bfloat1622float2(p[q]);
        acc[2 * q] += f.x;
        acc[2 * q + 1] += f.y;
    }
}

// One warp per token; each lane owns 16-byte chunks (8 values) of the row.
__global__ void __launch_bounds__(256) combine_kernel(const __nv_bfloat16* __restrict__ y_perm,
                                                      const int32_t* __restrict__ row_of, int T,
                                                      int K, int H, int has_shared,
                                                      __nv_bfloat16* __restrict__ y) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    int rows[33];
    int nrows = 0;
    if (has_shared) rows[nrows++] = (int)((int64_t)T * K + t);
    for (int j = 0; j < K; ++j) rows[nrows++] = row_of[(int64_t)t * K + j];
    const int chunks = H / 8;
    for (int c = lane; c < chunks; c += 32) {
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.f;
        for (int r = 0; r < nrows; ++r) {
            const uint4 v = reinterpret_cast<const uint4*>(y_perm + (int64_t)rows[r] * H)[c];
            acc_bf16x8(acc, v);
        }
        uint4 out;
        __nv_bfloat162* o = reinterpret_cast<__nv_bfloat162*>(&out);
#pragma unroll
        for (int q = 0; q < 4; ++q) o[q] = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
        reinterpret_cast<uint4*>(y + (int64_t)t * H)[c] = out;
    }
}

}  // namespace moe
