// Combine: y[t] = shared_out[t] + sum_j w_j * expert_j(x[t]).  The routing
// weights are already applied by the down-projection epilogue, so this is a
// gather of k + 1 block-scaled fp16 rows per token summed in fp32 in a fixed
// order (shared first, then slots 0..k-1), stored in fp32 or rounded once to
// bf16 (the expert-parallel layer also sums a token's rows on the rank that ran
// them and re-encodes the partial sum as a block-scaled fp16 row to send back).
// The teaching code of "The Evolving Transformer · 07" (§ 02, § 03) adds
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

// A block-scaled fp16 row array: row r's H values at values + r * ld (halves) and
// its H/32 scale codes at scales + r * scale_ld (bytes); value = fp16 * 2^(code -
// 141).  The layer's y_perm has ld = H; the expert-parallel rows carry their
// codes after their values in one wire row.
struct ScaledRowsIn {
    const __half* values;
    int64_t ld;
    const uint8_t* scales;
    int64_t scale_ld;
};

struct ScaledRowsOut {
    __half* values;
    int64_t ld;
    uint8_t* scales;
    int64_t scale_ld;
};

enum CombineOut { kOutF32 = 0, kOutBF16 = 1, kOutScaled = 2 };

// Where the sums go: y [T, H] dense (fp32 or bf16), or block-scaled fp16 rows.
struct CombineDst {
    void* y;
    ScaledRowsOut rows;
};

// The encoding of the block-scaled rows (the down-projection epilogue writes the
// same): a block of 32 values whose largest magnitude has biased fp32 exponent
// E gets the code c = clamp(E, 15, 254) and stores fp16(v * 2^(141 - c)); both
// factors are exact powers of two, NaN and Inf keep their class.
__device__ __forceinline__ uint32_t combine_scale_code(uint32_t max_abs_bits) {
    return min(max(max_abs_bits >> 23, 15u), 254u);
}

// Block (t, c) combines 8-value (16-byte) slices [256 c, 256 c + 256) of token
// t's row, one slice per thread, so small batches still spread over every SM.
// The sum is the shared row t (when shared.values is set), then the routed rows
// row_of[t, 0..K) in slot order.  row_of comes from the caller: -1 marks a slot
// without a row when absent_ok (the expert-parallel sums), and any other entry
// outside [0, routed_rows) contributes nothing and is recorded in the device
// error word (kErrRowIndex).  kOut: kOutF32 stores the sums unrounded, kOutBF16
// rounds once to nearest, kOutScaled encodes them as block-scaled fp16 rows.
template <int kOut>
__global__ void __launch_bounds__(256) combine_kernel(ScaledRowsIn routed, int64_t routed_rows,
                                                      const int32_t* __restrict__ row_of, int T, int K, int H,
                                                      int absent_ok, ScaledRowsIn shared, CombineDst dst) {
    __shared__ const __half* vrow[33];
    __shared__ const uint8_t* srow[33];
    const int t = blockIdx.x;
    const int has_shared = shared.values != nullptr;
    const int nrows = K + has_shared;
    if (threadIdx.x == 0 && has_shared) {
        vrow[0] = shared.values + (int64_t)t * shared.ld;
        srow[0] = shared.scales + (int64_t)t * shared.scale_ld;
    }
    if (threadIdx.x < K) {
        const int r = row_of[(int64_t)t * K + threadIdx.x];
        const bool ok = r >= 0 && r < routed_rows;
        if (!ok && !(absent_ok && r == -1) && blockIdx.y == 0) record_error(kErrRowIndex);
        vrow[has_shared + threadIdx.x] = ok ? routed.values + (int64_t)r * routed.ld : nullptr;
        srow[has_shared + threadIdx.x] = ok ? routed.scales + (int64_t)r * routed.scale_ld : nullptr;
    }
    __syncthreads();
    const int c = blockIdx.y * 256 + threadIdx.x;
    const bool active = c < H / 8;
    if (kOut != kOutScaled && !active) return;
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.f;
    for (int r = 0; r < nrows && active; ++r) {
        const __half* v = vrow[r];
        if (!v) continue;
        const uint4 raw = reinterpret_cast<const uint4*>(v)[c];
        const uint32_t code = srow[r][c >> 2];
        const float f = __uint_as_float((code - 14u) << 23);
        const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float2 x = __half22float2(h2[q]);
            acc[2 * q] += x.x * f;
            acc[2 * q + 1] += x.y * f;
        }
    }
    if constexpr (kOut == kOutF32) {
        store8(static_cast<float*>(dst.y) + (int64_t)t * H + 8 * c, acc);
    } else if constexpr (kOut == kOutBF16) {
        store8(static_cast<__nv_bfloat16*>(dst.y) + (int64_t)t * H + 8 * c, acc);
    } else {
        // A 32-column block is the 4 consecutive lanes c = 4b .. 4b + 3 (H / 8 is a
        // multiple of 8, so a block is wholly active or wholly not).
        uint32_t mx = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) mx = max(mx, __float_as_uint(acc[q]) & 0x7fffffffu);
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        if (!active) return;
        const uint32_t code = combine_scale_code(mx);
        const float f = __uint_as_float((268u - code) << 23);
        uint4 out;
        __half2* o = reinterpret_cast<__half2*>(&out);
#pragma unroll
        for (int q = 0; q < 4; ++q) o[q] = __floats2half2_rn(acc[2 * q] * f, acc[2 * q + 1] * f);
        reinterpret_cast<uint4*>(dst.rows.values + (int64_t)t * dst.rows.ld)[c] = out;
        if ((c & 3) == 0) dst.rows.scales[(int64_t)t * dst.rows.scale_ld + (c >> 2)] = static_cast<uint8_t>(code);
    }
}

}  // namespace moe
