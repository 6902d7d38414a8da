// The memory-bound steps of the layer's backward pass (chain rule of the
// forward of "The Evolving Transformer · 07", § 02 / § 03, with the expert
// selection held fixed):
//   bwd_scatter_kernel     x and / or dO = w * dy of every (token, slot) into the
//                          expert-ordered rows (128-row aligned segments);
//   bwd_zero_pad_kernel    the padding rows of both to zero (the weight-gradient
//                          GEMMs sum over them);
//   bwd_router_kernel      per token: dL/dw_j = sum(dh h)_j / w_j (from the dh
//                          GEMM's per-tile partial sums), then through the weight
//                          normalisation and the sigmoid to dL/dlogit;
//   bwd_router_wgrad_kernel  dWr[e] = sum over expert e's rows of dlogit * x
//                          (row chunks in parallel, then an ordered reduction);
//   bwd_dx_kernel          dx[t] = shared row + sum_j expert rows (block-scaled
//                          fp16, the kDx GEMM's output) + sum_j dlogit_j Wr[e_j].
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace moe {

__global__ void __launch_bounds__(256) bwd_scatter_kernel(const __nv_bfloat16* __restrict__ x,
                                                          const __nv_bfloat16* __restrict__ dy,
                                                          const int32_t* __restrict__ row_of,
                                                          const float* __restrict__ topk_w, int K, int H,
                                                          __nv_bfloat16* __restrict__ x_perm,
                                                          __nv_bfloat16* __restrict__ do_perm) {
    __shared__ int rows[32];
    __shared__ float ws[32];
    const int64_t t = blockIdx.x;
    if (threadIdx.x < K) {
        rows[threadIdx.x] = row_of[t * K + threadIdx.x];
        ws[threadIdx.x] = topk_w[t * K + threadIdx.x];
    }
    __syncthreads();
    const int c = blockIdx.y * 256 + threadIdx.x;  // 8-element slice
    if (c >= H / 8) return;
    const uint4 xv = x_perm != nullptr ? reinterpret_cast<const uint4*>(x + t * H)[c] : make_uint4(0, 0, 0, 0);
    const uint4 dv = do_perm != nullptr ? reinterpret_cast<const uint4*>(dy + t * H)[c] : make_uint4(0, 0, 0, 0);
    const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
    float d[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float2 f = __bfloat1622float2(d2[q]);
        d[2 * q] = f.x;
        d[2 * q + 1] = f.y;
    }
    for (int j = 0; j < K; ++j) {
        const int64_t r = rows[j];
        if (x_perm != nullptr) reinterpret_cast<uint4*>(x_perm + r * H)[c] = xv;
        if (do_perm == nullptr) continue;
        uint4 o;
        __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
        for (int q = 0; q < 4; ++q) o2[q] = __floats2bfloat162_rn(ws[j] * d[2 * q], ws[j] * d[2 * q + 1]);
        reinterpret_cast<uint4*>(do_perm + r * H)[c] = o;
    }
}

// Block (e, b): rows offsets[e] + counts[e] .. offsets[e+1] of both buffers,
// 16-byte stores, blocks of one expert striding over its padding rows.  a and b
// may be the same buffer (only one needs zeroing), hence no __restrict__ on them.
__global__ void __launch_bounds__(256) bwd_zero_pad_kernel(const int32_t* __restrict__ offsets,
                                                           const int32_t* __restrict__ counts, int H,
                                                           __nv_bfloat16* a, __nv_bfloat16* b) {
    const int e = blockIdx.x;
    const int64_t r0 = offsets[e] + counts[e], r1 = offsets[e + 1];
    const int64_t n = (r1 - r0) * (H / 8);
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int64_t i = (int64_t)blockIdx.y * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.y * blockDim.x) {
        const int64_t r = r0 + i / (H / 8), c = i % (H / 8);
        reinterpret_cast<uint4*>(a + r * H)[c] = z;
        reinterpret_cast<uint4*>(b + r * H)[c] = z;
    }
}

// One thread per token.  logits: the router's fp32 logits [T, E] (partials
// summed over nsplit); dw_part [rows, ntile] partial sums of dh * h per row.
__global__ void __launch_bounds__(256) bwd_router_kernel(const float* __restrict__ part, int nsplit, int T, int E,
                                                         int K, int norm, float scale,
                                                         const int32_t* __restrict__ topk_idx,
                                                         const float* __restrict__ topk_w,
                                                         const int32_t* __restrict__ row_of,
                                                         const float* __restrict__ dw_part, int ntile,
                                                         float* __restrict__ dlogit) {
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T) return;
    float s[32], dw[32];
    float S = 0.0f, sdw = 0.0f;
    for (int j = 0; j < K; ++j) {
        const int e = topk_idx[(int64_t)t * K + j];
        float l = 0.0f;
        for (int q = 0; q < nsplit; ++q) l += part[((int64_t)q * T + t) * E + e];
        s[j] = 1.0f / (1.0f + __expf(-l));
        const int64_t r = row_of[(int64_t)t * K + j];
        float d = 0.0f;
        for (int q = 0; q < ntile; ++q) d += dw_part[r * ntile + q];
        dw[j] = d / topk_w[(int64_t)t * K + j];  // dh carries the routing weight w
        S += s[j];
        sdw += dw[j] * s[j];
    }
    for (int j = 0; j < K; ++j) {
        const float ds = norm ? scale / S * (dw[j] - sdw / S) : scale * dw[j];
        dlogit[(int64_t)t * K + j] = ds * s[j] * (1.0f - s[j]);
    }
}

// Block (e, c, q): 256 threads x 8 columns = 2048 columns c*2048.. of expert e,
// summed over the q-th of kRouterSplit row chunks of the expert's segment, eight
// rows per step with independent loads; partial sums go to
// part[q][e][H] and bwd_router_wgrad_reduce_kernel adds them in order
// (deterministic).
constexpr int kRouterSplit = 4;

__global__ void __launch_bounds__(256) bwd_router_wgrad_kernel(const int32_t* __restrict__ offsets,
                                                               const int32_t* __restrict__ counts,
                                                               const int32_t* __restrict__ perm_src,
                                                               const float* __restrict__ dlogit,
                                                               const __nv_bfloat16* __restrict__ x_perm, int H, int E,
                                                               float* __restrict__ part) {
    const int e = blockIdx.x, q = blockIdx.z;
    const int c = blockIdx.y * 256 + threadIdx.x;
    const int64_t n = counts[e];
    const int64_t chunk = (n + kRouterSplit - 1) / kRouterSplit;
    const int64_t i0 = q * chunk, i1 = min(n, i0 + chunk);
    const int64_t r0 = offsets[e];
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (c < H / 8) {
        for (int64_t i = i0; i < i1; i += 8) {
            float d[8];
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const bool in = i + u < i1;
                d[u] = in ? dlogit[perm_src[r0 + i + u]] : 0.0f;
                v[u] = in ? reinterpret_cast<const uint4*>(x_perm + (r0 + i + u) * H)[c] : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(&v[u]);
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    const float2 f = __bfloat1622float2(v2[w]);
                    acc[2 * w] += d[u] * f.x;
                    acc[2 * w + 1] += d[u] * f.y;
                }
            }
        }
        float4* out = reinterpret_cast<float4*>(part + ((int64_t)q * E + e) * H + 8 * c);
        out[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        out[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
}

__global__ void __launch_bounds__(256) bwd_router_wgrad_reduce_kernel(const float* __restrict__ part, int64_t n,
                                                                      float* __restrict__ d_router_w) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    float s = 0.0f;
#pragma unroll
    for (int q = 0; q < kRouterSplit; ++q) s += part[q * n + i];
    d_router_w[i] = s;
}

// Block (t, c): dx of token t, columns 8*(c*256 + thread) ..; expert rows are
// block-scaled fp16 (value = fp16 * 2^(code - 141), one code per 32 columns).
__global__ void __launch_bounds__(256) bwd_dx_kernel(const __half* __restrict__ dxq, const uint8_t* __restrict__ dxs,
                                                     int64_t scale_ld, const int32_t* __restrict__ row_of,
                                                     const int32_t* __restrict__ topk_idx,
                                                     const float* __restrict__ dlogit,
                                                     const float* __restrict__ router_w, int K, int H,
                                                     int has_shared, int64_t shared_row0, float* __restrict__ dx) {
    __shared__ int rows[33];
    __shared__ int experts[32];
    __shared__ float dl[32];
    const int64_t t = blockIdx.x;
    if (threadIdx.x < K) {
        rows[threadIdx.x] = row_of[t * K + threadIdx.x];
        experts[threadIdx.x] = topk_idx[t * K + threadIdx.x];
        dl[threadIdx.x] = dlogit[t * K + threadIdx.x];
    }
    if (threadIdx.x == 0) rows[K] = static_cast<int>(shared_row0 + t);
    __syncthreads();
    const int c = blockIdx.y * 256 + threadIdx.x;
    if (c >= H / 8) return;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    const int nrows = K + has_shared;
    for (int q = 0; q < nrows; ++q) {
        const int64_t r = q < K ? rows[q] : rows[K];
        const uint4 raw = reinterpret_cast<const uint4*>(dxq + r * H)[c];
        const float f = __uint_as_float((static_cast<uint32_t>(dxs[r * scale_ld + (c >> 2)]) - 14u) << 23);
        const __half2* h2 = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 v = __half22float2(h2[i]);
            acc[2 * i] += v.x * f;
            acc[2 * i + 1] += v.y * f;
        }
    }
    for (int j = 0; j < K; ++j) {
        const float4* w = reinterpret_cast<const float4*>(router_w + (int64_t)experts[j] * H + 8 * c);
        const float4 a = w[0], b = w[1];
        acc[0] += dl[j] * a.x; acc[1] += dl[j] * a.y; acc[2] += dl[j] * a.z; acc[3] += dl[j] * a.w;
        acc[4] += dl[j] * b.x; acc[5] += dl[j] * b.y; acc[6] += dl[j] * b.z; acc[7] += dl[j] * b.w;
    }
    float4* out = reinterpret_cast<float4*>(dx + t * H + 8 * c);
    out[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    out[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
}

}  // namespace moe
