// MXFP8 operands for the expert GEMMs ("DeepSeek-V3 notes" (knlb.dev), § fp8:
// fine-grained block-wise quantisation, E4M3 throughout, scales derived online
// from each block's maximum; activations cached and dispatched in FP8).
//
// Format (the microscaling layout the tcgen05 block-scaled MMA reads):
//   * elements: E4M3 (bias 7, largest finite 448), one byte each, row-major
//     [rows, K] with K the contraction axis;
//   * scales:   one 8-bit power-of-two code per 32 consecutive elements of a row,
//     scale = 2^(code - 127); code = 127 + e for the smallest e with
//     amax <= 448 * 2^e (0 for an all-zero block), so no element saturates;
//   * scale layout: tiles of 128 rows x 128 K (4 codes per row) stored as
//     512-byte atoms, atom (rb, kb) at byte (rb * K/128 + kb) * 512, and inside
//     an atom the code of row r (0..127) and 32-block j (0..3) at byte
//     16 * (r % 32) + 4 * (r / 32) + j.  One atom is what one 128-row x 128-K
//     operand tile needs; tcgen05.cp moves it into four TMEM columns as is.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

namespace moe {

constexpr int kMxBlock = 32;      // elements per scale
constexpr int kMxAtomRows = 128;  // rows per scale atom
constexpr int kMxAtomK = 128;     // K per scale atom (4 codes per row)
constexpr int kMxAtomBytes = 512;

// Scale code of a block from the fp32 bit pattern of its largest magnitude.
// amax = (1 + f) 2^(E - 127): 448 = 1.75 * 2^8, so amax <= 448 * 2^e holds first
// at e = E - 127 - 8 when f <= 0.75 and at e = E - 127 - 7 otherwise.
__device__ __forceinline__ uint32_t mx_scale_code(uint32_t amax_bits) {
    if (amax_bits == 0) return 0;
    const int c = static_cast<int>(amax_bits >> 23) - ((amax_bits & 0x7fffffu) <= 0x600000u ? 8 : 7);
    return static_cast<uint32_t>(min(max(c, 0), 254));
}

// 2^(127 - code): the exact factor that maps a block into the E4M3 range.
__device__ __forceinline__ float mx_encode_factor(uint32_t code) { return __uint_as_float((254u - code) << 23); }

// Two fp32 values to two E4M3 bytes (round to nearest even), a in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
    return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}

// Byte offset of row r's code word (4 codes, K block kb) in a scale array whose
// rows have K / 128 atoms.
__device__ __forceinline__ int64_t mx_sf_word_offset(int64_t r, int kb, int k_atoms) {
    return ((r / kMxAtomRows) * k_atoms + kb) * kMxAtomBytes + 16 * (r % 32) + 4 * ((r / 32) % 4);
}

// Quantise 8 consecutive bf16 values held by one thread; four consecutive lanes
// (a 4-lane aligned group) form one 32-element block.  Returns the 8 E4M3 bytes
// and the block's code (the same in all four lanes).
__device__ __forceinline__ uint2 mx_quantize8(const uint4 v, uint32_t& code) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
    float f[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 t = __bfloat1622float2(p[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) m = max(m, __float_as_uint(fabsf(f[i])));
    m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
    code = mx_scale_code(m);
    const float s = mx_encode_factor(code);
    uint2 q;
    q.x = e4m3x2(f[0] * s, f[1] * s) | (e4m3x2(f[2] * s, f[3] * s) << 16);
    q.y = e4m3x2(f[4] * s, f[5] * s) | (e4m3x2(f[6] * s, f[7] * s) << 16);
    return q;
}

// The four codes of a 128-column slice gathered into the first of its 16 lanes
// (lanes 16i..16i+15 hold the slice; blocks start at lanes +0, +4, +8, +12).
__device__ __forceinline__ uint32_t mx_gather_codes(uint32_t code) {
    const int lane = threadIdx.x & 31;
    const int base = lane & 16;
    const uint32_t c0 = __shfl_sync(0xffffffffu, code, base + 0);
    const uint32_t c1 = __shfl_sync(0xffffffffu, code, base + 4);
    const uint32_t c2 = __shfl_sync(0xffffffffu, code, base + 8);
    const uint32_t c3 = __shfl_sync(0xffffffffu, code, base + 12);
    return c0 | (c1 << 8) | (c2 << 16) | (c3 << 24);
}

// Quantise a bf16 matrix [rows, K] (K a multiple of 128): block (r, c) of 256
// threads handles 2048 columns of row r, 8 per thread.
__global__ void __launch_bounds__(256) mx_quantize_rows_kernel(const __nv_bfloat16* __restrict__ src, int K,
                                                               uint8_t* __restrict__ q, uint8_t* __restrict__ sf) {
    const int64_t r = blockIdx.x;
    const int col = (blockIdx.y * 256 + threadIdx.x) * 8;
    const bool active = col < K;  // K % 128 == 0: whole 16-lane slices are active or not
    uint4 v = make_uint4(0, 0, 0, 0);
    if (active) v = *reinterpret_cast<const uint4*>(src + r * K + col);
    uint32_t code;
    const uint2 qv = mx_quantize8(v, code);
    const uint32_t word = mx_gather_codes(code);
    if (!active) return;
    *reinterpret_cast<uint2*>(q + r * K + col) = qv;
    if ((threadIdx.x & 15) == 0)
        *reinterpret_cast<uint32_t*>(sf + mx_sf_word_offset(r, col / kMxAtomK, K / kMxAtomK)) = word;
}

// Dispatch with quantisation: token t's row is read once, quantised, and written
// to its k rows of xq_perm (rows from row_of, expert segments 128-row aligned)
// and, when the layer has shared experts, to row t of xq_shared.
__global__ void __launch_bounds__(256) dispatch_scatter_mx_kernel(
    const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ row_of, int K, int H,
    uint8_t* __restrict__ xq_perm, uint8_t* __restrict__ xq_perm_sf, uint8_t* __restrict__ xq_shared,
    uint8_t* __restrict__ xq_shared_sf) {
    __shared__ int rows[32];
    const int64_t t = blockIdx.x;
    if (threadIdx.x < K) rows[threadIdx.x] = row_of[t * K + threadIdx.x];
    __syncthreads();
    const int col = (blockIdx.y * 256 + threadIdx.x) * 8;
    const bool active = col < H;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (active) v = *reinterpret_cast<const uint4*>(x + t * H + col);
    uint32_t code;
    const uint2 qv = mx_quantize8(v, code);
    const uint32_t word = mx_gather_codes(code);
    if (!active) return;
    const int kb = col / kMxAtomK, k_atoms = H / kMxAtomK;
    const bool writer = (threadIdx.x & 15) == 0;
    for (int j = 0; j < K; ++j) {
        const int64_t r = rows[j];
        if (r < 0) continue;  // a slot with an out-of-range expert index (skipped by the place step)
        *reinterpret_cast<uint2*>(xq_perm + r * H + col) = qv;
        if (writer) *reinterpret_cast<uint32_t*>(xq_perm_sf + mx_sf_word_offset(r, kb, k_atoms)) = word;
    }
    if (xq_shared != nullptr) {
        *reinterpret_cast<uint2*>(xq_shared + t * H + col) = qv;
        if (writer) *reinterpret_cast<uint32_t*>(xq_shared_sf + mx_sf_word_offset(t, kb, k_atoms)) = word;
    }
}

}  // namespace moe
