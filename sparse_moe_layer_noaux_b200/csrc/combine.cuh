// Combine: y[t] = shared_out[t] + sum_j w_j * expert_j(x[t]).  The routing
// weights are already applied by the down-projection epilogue, so this is a
// gather of k + 1 block-scaled fp16 rows per token summed in fp32 in a fixed
// order (shared first, then slots 0..k-1), stored in fp32 or rounded once to
// bf16.  The teaching code of "The Evolving Transformer · 07" (§ 02, § 03) adds
// each expert's weighted output into the token's row and then the shared
// expert's output; gathering instead of scattering gives the same sum without
// atomics, and therefore deterministically.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "device_status.cuh"

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

// Block (t, c) combines 8-value (16-byte) slices [256 c, 256 c + 256) of token
// t's row, one slice per thread, so small batches still spread over every SM.
// Each y_perm row is block-scaled fp16: value = fp16 * 2^(code - 141), one code
// per 32 columns; the shared expert's output for token t is row shared_row0 + t.
// row_of comes from the caller (moe_combine): an entry outside [0, routed_rows)
// contributes nothing and is recorded in the device error word (kErrRowIndex).
// OutT = float (the layer output unrounded) or __nv_bfloat16 (rounded once, to
// nearest).
template <typename OutT>
__global__ void __launch_bounds__(256) combine_kernel(const __half* __restrict__ y_perm,
                                                      const uint8_t* __restrict__ y_scale, int64_t scale_ld,
                                                      const int32_t* __restrict__ row_of, int T, int K, int H,
                                                      int has_shared, int64_t shared_row0, int64_t routed_rows,
                                                      OutT* __restrict__ y) {
    __shared__ int rows[33];
    const int t = blockIdx.x;
    const int nrows = K + has_shared;
    if (threadIdx.x == 0 && has_shared) rows[0] = (int)(shared_row0 + t);
    if (threadIdx.x < K) {
        const int r = row_of[(int64_t)t * K + threadIdx.x];
        const bool ok = r >= 0 && r < routed_rows;
        if (!ok && blockIdx.y == 0) record_error(kErrRowIndex);
        rows[has_shared + threadIdx.x] = ok ? r : -1;
    }
    __syncthreads();
    const int c = blockIdx.y * 256 + threadIdx.x;
    if (c >= H / 8) return;
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.f;
    for (int r = 0; r < nrows; ++r) {
        const int64_t row = rows[r];
        if (row < 0) continue;
        const uint4 raw = reinterpret_cast<const uint4*>(y_perm + row * H)[c];
        const uint32_t code = y_scale[row * scale_ld + (c >> 2)];
        const float f = __uint_as_float((code - 14u) << 23);
        const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float2 v = __half22float2(h2[q]);
            acc[2 * q] += v.x * f;
            acc[2 * q + 1] += v.y * f;
        }
    }
    store8(y + (int64_t)t * H + 8 * c, acc);
}

}  // namespace moe
