// Combine: y[t] = shared_out[t] + sum_j w_j * expert_j(x[t]).  The routing
// weights are already applied by the down-projection epilogue, so this is a
// gather of k + 1 fp32 rows per token summed in fp32 in a fixed order (shared
// first, then slots 0..k-1), stored in fp32 or rounded once to bf16 — the page's
// `output[mask] += w * expert_out` followed by `shared_expert_out + output` ("The Evolving Transformer · 07", § 02 / § 03),
// without atomics and therefore deterministic.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

namespace moe {

__device__ __forceinline__ void store8(float* dst, const float (&a)[8]) {
    float4* d = reinterpret_cast<float4*>(dst);
    d[0] = make_float4(a[0], a[1], a[2], a[3]);
    d[1] = make_float4(a[4], a[5], a[6], a[7]);
}

__device__ __forceinline__ void store8(__nv_bfloat16* dst, const float (&a)[8]) {
    uint4 out;
    __nv_bfloat162* o = reinterpret_cast<__nv_bfloat162*>(&out);
#pragma unroll
    for (int q = 0; q < 4; ++q) o[q] = __floats2bfloat162_rn(a[2 * q], a[2 * q + 1]);
    *reinterpret_cast<uint4*>(dst) = out;
}

// One warp per token; each lane owns 8-value (32-byte) slices of the row.
// OutT = float (the layer output unrounded) or __nv_bfloat16 (rounded once, to nearest).
template <typename OutT>
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ y_perm,
                                                      const int32_t* __restrict__ row_of, int T,
                                                      int K, int H, int has_shared,
                                                      OutT* __restrict__ y) {
    __shared__ int rows_s[8][33];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const int t = blockIdx.x * (blockDim.x >> 5) + wib;
    if (t >= T) return;
    int* rows = rows_s[wib];
    const int nrows = K + has_shared;
    if (lane == 0 && has_shared) rows[0] = (int)((int64_t)T * K + t);
    if (lane < K) rows[has_shared + lane] = row_of[(int64_t)t * K + lane];
    __syncwarp();
    const int slices = H / 8;
    for (int c = lane; c < slices; c += 32) {
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.f;
        for (int r = 0; r < nrows; ++r) {
            const float4* src = reinterpret_cast<const float4*>(y_perm + (int64_t)rows[r] * H) + 2 * c;
            const float4 a = src[0], b = src[1];
            acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
            acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
        }
        store8(y + (int64_t)t * H + 8 * c, acc);
    }
}

}  // namespace moe
