// Router of the DeepSeekMoE layer (noaux_tc): logits, sigmoid scores, biased
// scores, group top-2 scores, group top-k, expert top-k, weights.
// "DeepSeekV3.2-Tiered-Implementations" README, § Architecture (sigmoid routing
// with correction bias, n_group / topk_group); "The Evolving Transformer · 07",
// § 02 (router(x) -> weights, indices) and § 06 (bias steers selection only).
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <math_constants.h>

namespace moe {

// ---------------------------------------------------------------------------
// K1 (CUDA cores): partial logits P[split][t][e] = sum_{h in split} x[t,h] * Wr[e,h]
// in fp32.  Block tile 128 tokens x 64 experts, 256 threads, 8x4 outputs each;
// the hidden axis is cut into `nsplit` slices when T is small so that the grid
// still covers the GPU.  Partials are summed by the select kernel in split
// order, so the result is deterministic.
// ---------------------------------------------------------------------------
constexpr int kRT = 128, kRE = 64, kRK = 32;

__global__ void __launch_bounds__(256) router_logits_kernel(
    const __nv_bfloat16* __restrict__ x, const float* __restrict__ wr, float* __restrict__ part,
    int T, int E, int H, int split_len) {
    __shared__ float xs[kRK][kRT + 4];
    __shared__ float ws[kRK][kRE + 4];
    const int tid = threadIdx.x;
    const int t0 = blockIdx.y * kRT, e0 = blockIdx.x * kRE;
    const int h_begin = blockIdx.z * split_len;
    const int h_end = min(H, h_begin + split_len);
    const int tr = tid / 16;  // 16 row groups of 8 tokens
    const int tc = tid % 16;  // 16 col groups of 4 experts
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    // Each thread moves two 8-element chunks of the x tile and two 4-element chunks
    // of the Wr tile per K step.  The next step's chunks are loaded into registers
    // while this step's FMAs run (same products, same summation order).
    static_assert(kRT * kRK / 8 == 2 * 256 && kRE * kRK / 4 == 2 * 256, "two chunks per thread");
    uint4 xr[2];
    float4 wv[2];
    auto fetch = [&](int h0) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int c = tid + 256 * u;
            const int r = c / (kRK / 8), kc = (c % (kRK / 8)) * 8;
            const int t = t0 + r;
            xr[u] = (t < T && h0 + kc < h_end)
                        ? *reinterpret_cast<const uint4*>(x + (int64_t)t * H + h0 + kc)
                        : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int c = tid + 256 * u;
            const int r = c / (kRK / 4), kc = (c % (kRK / 4)) * 4;
            const int e = e0 + r;
            wv[u] = (e < E && h0 + kc < h_end)
                        ? *reinterpret_cast<const float4*>(wr + (int64_t)e * H + h0 + kc)
                        : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    if (h_begin < h_end) fetch(h_begin);
    for (int h0 = h_begin; h0 < h_end; h0 += kRK) {
        // x tile 128 x 32 (bf16 -> fp32, transposed), Wr tile 64 x 32 (transposed).
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int c = tid + 256 * u;
            const int r = c / (kRK / 8), kc = (c % (kRK / 8)) * 8;
            const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&xr[u]);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float2 f = __bfloat1622float2(p[q]);
                xs[kc + 2 * q][r] = f.x;
                xs[kc + 2 * q + 1][r] = f.y;
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int c = tid + 256 * u;
            const int r = c / (kRK / 4), kc = (c % (kRK / 4)) * 4;
            ws[kc + 0][r] = wv[u].x;
            ws[kc + 1][r] = wv[u].y;
            ws[kc + 2][r] = wv[u].z;
            ws[kc + 3][r] = wv[u].w;
        }
        __syncthreads();
        if (h0 + kRK < h_end) fetch(h0 + kRK);
#pragma unroll 8
        for (int kk = 0; kk < kRK; ++kk) {
            float a[8], b[4];
#pragma unroll
            for (int i = 0; i < 8; ++i) a[i] = xs[kk][tr * 8 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = ws[kk][tc * 4 + j];
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
    float* out = part + (int64_t)blockIdx.z * T * E;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int t = t0 + tr * 8 + i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int e = e0 + tc * 4 + j;
            if (e < E) out[(int64_t)t * E + e] = acc[i][j];
        }
    }
}

// ---------------------------------------------------------------------------
// K1 (tensor cores), step 1: split each fp32 router weight exactly into three
// bf16 terms, w = hi + mid + lo (each term rounds the remainder of the previous
// ones to nearest; 3 x 8 significant bits cover fp32's 24).  A bf16 x times a
// bf16 term is exact in fp32, so x . Wr^T = x . hi^T + x . mid^T + x . lo^T is
// computed by one bf16 tensor-core GEMM with K = 3 H and fp32 accumulation.
// (Splitting a float into bfloat16 terms: Henry, Tang & Heinecke, "Leveraging
// the bfloat16 Artificial Intelligence Datatype For Higher-Precision
// Computations", ARITH 2019.)  Output planes: w3[p][e][h], p = 0, 1, 2.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) router_split_kernel(const float* __restrict__ wr,
                                                           __nv_bfloat16* __restrict__ w3, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float w = wr[i];
        const __nv_bfloat16 hi = __float2bfloat16_rn(w);
        const float r1 = w - __bfloat162float(hi);
        const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
        const float r2 = r1 - __bfloat162float(mid);
        w3[i] = hi;
        w3[n + i] = mid;
        w3[2 * n + i] = __float2bfloat16_rn(r2);
    }
}

// ---------------------------------------------------------------------------
// K2: one warp per token.  Expert e lives in lane e % 32, slot e / 32.
// ---------------------------------------------------------------------------
struct RouteArgs {
    const float* part;   // [nsplit][T][E] partial logits
    int nsplit;
    int T, E, G, TG, K;
    int norm;
    float scale;
    const float* bias;   // [E]
    int32_t* topk_idx;   // [T][K]
    float* topk_w;       // [T][K]
};

// (value, index) order: larger value first, lower index on equal values.
__device__ __forceinline__ bool route_beats(float va, int ia, float vb, int ib) {
    return va > vb || (va == vb && ia < ib);
}

// NaN (from a NaN in x, router_w or e_bias, or +inf - inf in a group score) is
// ranked as -inf, so the (value, index) order stays total: exactly topk_group
// groups are kept and k distinct valid experts are chosen whatever the inputs.
__device__ __forceinline__ float route_key(float v) { return v == v ? v : -CUDART_INF_F; }

template <int EPL>
__global__ void __launch_bounds__(256) router_select_kernel(RouteArgs a) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= a.T) return;
    const int E = a.E, gsize = E / a.G;

    // Logits: the split partials summed in split order.  The lane's EPL experts
    // are loaded side by side for each split (independent loads in flight, same
    // addition order per logit as a split-by-split sum).
    float l[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) l[i] = 0.f;
    const float* pt = a.part + (int64_t)t * E;
    const int64_t split_stride = (int64_t)a.T * E;
#pragma unroll 4
    for (int p = 0; p < a.nsplit; ++p) {
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const int e = lane + 32 * i;
            if (e < E) l[i] += pt[p * split_stride + e];
        }
    }

    // avail bit i: slot i holds an expert that may still be chosen.
    float s[EPL], cand[EPL];
    int grp[EPL];  // group of this lane's expert in slot i (-1: no expert)
    unsigned avail = 0;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        s[i] = 0.f;
        cand[i] = -CUDART_INF_F;
        grp[i] = e < E ? e / gsize : -1;
        if (e < E) {
            s[i] = 1.0f / (1.0f + expf(-l[i]));
            cand[i] = route_key(s[i] + a.bias[e]);  // biased score b_e
            avail |= 1u << i;
        }
    }

    // Group score: sum of the two largest biased scores of the group.
    float my_gscore = -CUDART_INF_F;  // lane g holds group g's score
    for (int g = 0; g < a.G; ++g) {
        float m1 = -CUDART_INF_F, m2 = -CUDART_INF_F;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            if (grp[i] == g) {
                const float v = cand[i];
                if (v > m1) { m2 = m1; m1 = v; }
                else if (v > m2) { m2 = v; }
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float o1 = __shfl_xor_sync(0xffffffffu, m1, off);
            const float o2 = __shfl_xor_sync(0xffffffffu, m2, off);
            const float n1 = fmaxf(m1, o1);
            const float n2 = fmaxf(fminf(m1, o1), fmaxf(m2, o2));
            m1 = n1;
            m2 = n2;
        }
        const float gs = route_key(gsize >= 2 ? m1 + m2 : m1);
        if (lane == g) my_gscore = gs;
    }

    // Keep the topk_group best groups (lower group index on equal scores).
    int rank = 0;
    for (int g = 0; g < a.G; ++g) {
        const float v = __shfl_sync(0xffffffffu, my_gscore, g);
        if (route_beats(v, g, my_gscore, lane)) ++rank;
    }
    const unsigned kept = __ballot_sync(0xffffffffu, lane < a.G && rank < a.TG);

    // Experts of dropped groups are excluded from the top-k.
#pragma unroll
    for (int i = 0; i < EPL; ++i)
        if (grp[i] < 0 || !((kept >> grp[i]) & 1u)) avail &= ~(1u << i);

    // k rounds of a warp arg-max over the available experts.  The kept groups hold
    // topk_group * E / n_group >= k experts, so every round finds one (bi < E).
    float my_s = 0.f;
    int my_idx = 0;
    for (int j = 0; j < a.K; ++j) {
        float bv = -CUDART_INF_F, bs = 0.f;
        int bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const int e = lane + 32 * i;
            if (((avail >> i) & 1u) && route_beats(cand[i], e, bv, bi)) {
                bv = cand[i];
                bi = e;
                bs = s[i];
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
            const float os = __shfl_xor_sync(0xffffffffu, bs, off);
            if (route_beats(ov, oi, bv, bi)) {
                bv = ov;
                bi = oi;
                bs = os;
            }
        }
#pragma unroll
        for (int i = 0; i < EPL; ++i)
            if (lane + 32 * i == bi) avail &= ~(1u << i);
        if (lane == j) {
            my_s = bs;
            my_idx = bi;
        }
    }

    float sum = lane < a.K ? my_s : 0.f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (lane < a.K) {
        float w = a.norm ? my_s / sum : my_s;
        w *= a.scale;
        a.topk_idx[(int64_t)t * a.K + lane] = my_idx;
        a.topk_w[(int64_t)t * a.K + lane] = w;
    }
}

}  // namespace moe
