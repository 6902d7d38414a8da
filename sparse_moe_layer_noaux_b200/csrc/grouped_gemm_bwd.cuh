// Grouped expert GEMMs of the layer's backward pass on tcgen05 (bf16 operands,
// fp32 accumulation in TMEM).  The chain rule of the SwiGLU experts
// ("The Evolving Transformer · 07", § 02; gradients checked by float64 finite
// differences as the "dsv3-native-reference" page's § NumPy Oracle does) needs
// four products per expert segment, all run by one persistent kernel template:
//   kRecompute  g = A Wg^T, u = A Wu^T (A = the segment's token rows), stored
//               as bf16, and optionally h = silu(g) u (the training forward);
//   kDh         dh = dO Wd (dO = w dy for routed rows, dy for shared rows), with
//               the SwiGLU backward in the epilogue: dg = dh u silu'(g),
//               du = dh silu(g), h = silu(g) u, and per row and half tile the
//               partial dot sum(dh h) that gives the routing-weight gradient;
//   kDx         dx_perm = dg Wg + du Wu (K = 2 I over the two weight maps),
//               block-scaled fp16 like the forward's y_perm;
//   kWgrad      dW = P^T Q for each expert over its rows (K = the segment's
//               rows): dWd = dO^T h and [dWg; dWu] = [dg du]^T x;
//   kFwdDown    the forward's down projection y = w (h Wd^T) on the same
//               128-row aligned segments (the training forward, which keeps g
//               and u for the backward), block-scaled fp16 like kDx.
// Weights are read in their stored (out, in) layout: where the product needs
// them transposed (kDh, kDx) the B operand is loaded MN-major (TMA boxes of 64
// contiguous elements by 64 K rows, 128-byte swizzle) and the instruction
// descriptor says so; kWgrad loads both operands MN-major.  Routed segments
// start on 128-row boundaries and their padding rows are zero, so K blocks of
// 64 rows never mix two experts.
#pragma once
#include "grouped_gemm.cuh"

namespace moe {

enum { kRecompute = 0, kDh = 1, kDx = 2, kWgrad = 3, kFwdDown = 4 };

struct BwdParams {
    const int32_t* offsets;      // [E+1] 128-aligned segment starts
    const int32_t* counts;       // [E]   rows of each segment
    int E;
    int T;                       // rows of the shared segment
    int has_shared;
    int n_tiles_routed, n_tiles_shared;     // output column tiles (kWgrad: N tiles)
    int m_tiles_wgrad_routed, m_tiles_wgrad_shared;  // kWgrad: output row tiles of one dW
    int kb_routed, kb_shared;               // K blocks of 64 (kRecompute / kDh / kDx)
    int b_rows_per_expert;                  // rows of one expert in the routed B maps
    int i_blocks_routed, i_blocks_shared;   // kDx: K blocks taken from the first B map (I / 64)
    // outputs
    __nv_bfloat16* out_routed;   // kRecompute: gu [rows, 2I]; kDh: dgu [rows, 2I]; kWgrad: dW rows
    int64_t ld_routed;
    __nv_bfloat16* out_shared;
    int64_t ld_shared;
    __nv_bfloat16* out2_routed;  // kDh: h [rows, I]; kWgrad: second half of the stacked output
    __nv_bfloat16* out2_shared;
    int64_t ld2_routed, ld2_shared;
    int split_rows_routed, split_rows_shared;   // kWgrad: output rows before out2 takes over
    int64_t out_expert_stride, out2_expert_stride;  // kWgrad: elements between experts' dW
    const __nv_bfloat16* gu_routed;  // kDh: recomputed g | u, [rows, 2I]
    const __nv_bfloat16* gu_shared;
    int64_t gu_ld_routed, gu_ld_shared;
    int half_routed, half_shared;    // kDh: I (where u starts inside a gu row)
    float* dw_part;                  // kDh: [rows, 2 n_tiles_routed] partial sum(dh h) of routed rows
    __half* yq_routed;               // kDx: block-scaled fp16 rows
    __half* yq_shared;
    uint8_t* ysc_routed;
    uint8_t* ysc_shared;
    int64_t yq_ld, ysc_ld;
    int n_valid_routed, n_valid_shared;
    const int32_t* perm_src;         // kFwdDown: routed row -> slot
    const float* topk_w;             // kFwdDown: slot -> routing weight
    uint32_t idesc;
};

struct BwdTile {
    int routed, expert;
    int m, n;        // tile coordinates (kWgrad: output row / column tile)
    int rows;        // rows of the segment
    int row0;        // first row of the segment
    int kb;          // K blocks of 64
};

struct BwdSmem {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t tmem_full[2];
    uint64_t tmem_empty[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort_flag;
    int total_tiles;
    int nseg;
    int seg_row0[kMaxSeg];
    int seg_rows[kMaxSeg];
    int tile_start[kMaxSeg + 1];
};

// Eight epilogue warps (two per TMEM lane quarter, each draining half of the 256
// accumulator columns): the weight-gradient tiles have only ~8 K blocks at the
// V3 prefill shape, so a four-warp epilogue was as long as the main loop.
constexpr int kBwdEpiWarps = 8;
constexpr int kBwdThreads = 64 + 32 * kBwdEpiWarps;
constexpr uint32_t kBwdStagePerWarp = 32 * kStagePitchH * 2;  // 32 rows x 80 B of 16-bit values
constexpr size_t kGemmBwdSmemBytes =
    1024 + kStages * (kTileABytes + kTileBBytes) + kBwdEpiWarps * kBwdStagePerWarp + sizeof(BwdSmem);

// Descriptor of an MN-major operand in the 128-byte swizzle layout: atoms of 64
// contiguous elements (128 B) by 8 K rows (1024 B); consecutive K groups of 8
// rows 1024 B apart, consecutive 64-element MN atoms `lbo` bytes apart.
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(uint32_t smem_addr, uint32_t lbo) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((smem_addr & 0x3FFFFu) >> 4);
    d |= static_cast<uint64_t>(lbo >> 4) << 16;
    d |= static_cast<uint64_t>(1024u >> 4) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    d |= static_cast<uint64_t>(2u) << 61;
    return d;
}

__host__ __device__ constexpr uint32_t idesc_bf16_f32_major(int M, int N, int a_mn, int b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(a_mn) << 15) |
           (static_cast<uint32_t>(b_mn) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}

template <int kMode>
__device__ __forceinline__ int bwd_tiles_of(const BwdParams& p, int seg, int rows) {
    const bool routed = !(p.has_shared && seg == 0);
    if (kMode == kWgrad)
        return (routed ? p.m_tiles_wgrad_routed * p.n_tiles_routed : p.m_tiles_wgrad_shared * p.n_tiles_shared);
    return ((rows + kBM - 1) / kBM) * (routed ? p.n_tiles_routed : p.n_tiles_shared);
}

template <int kMode>
__device__ __forceinline__ BwdTile decode_bwd(const BwdSmem& s, const BwdParams& p, int tile) {
    int lo = 0, hi = s.nseg - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s.tile_start[mid] <= tile) lo = mid;
        else hi = mid - 1;
    }
    BwdTile t;
    t.routed = !(p.has_shared && lo == 0);
    t.expert = lo - p.has_shared;
    t.rows = s.seg_rows[lo];
    t.row0 = s.seg_row0[lo];
    const int local = tile - s.tile_start[lo];
    if (kMode == kWgrad) {
        const int mt = t.routed ? p.m_tiles_wgrad_routed : p.m_tiles_wgrad_shared;
        t.n = local / mt;
        t.m = local - t.n * mt;
        t.kb = (t.rows + 63) / 64;
    } else {
        const int mt = (t.rows + kBM - 1) / kBM;
        t.n = local / mt;
        t.m = local - t.n * mt;
        t.kb = t.routed ? p.kb_routed : p.kb_shared;
    }
    return t;
}

template <int kMode>
__global__ void __launch_bounds__(kBwdThreads, 1)
    grouped_gemm_bwd_kernel(const __grid_constant__ CUtensorMap tmA_r, const __grid_constant__ CUtensorMap tmA_s,
                            const __grid_constant__ CUtensorMap tmB_r, const __grid_constant__ CUtensorMap tmB2_r,
                            const __grid_constant__ CUtensorMap tmB_s, const __grid_constant__ CUtensorMap tmB2_s,
                            const BwdParams p) {
    constexpr bool kAmn = kMode == kWgrad;                   // A loaded MN-major
    constexpr bool kBmn = kMode != kRecompute && kMode != kFwdDown;   // B loaded MN-major
    extern __shared__ uint8_t smem_raw[];
    uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t* smemA = tiles;
    uint8_t* smemB = tiles + kStages * kTileABytes;
    uint8_t* stage_base = tiles + kStages * (kTileABytes + kTileBBytes);
    BwdSmem& S = *reinterpret_cast<BwdSmem*>(stage_base + kBwdEpiWarps * kBwdStagePerWarp);
    volatile int* abort_flag = &S.abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (warp == 0 && lane == 0) {
        for (int i = 0; i < kStages; ++i) {
            ptx::mbar_init(ptx::smem_u32(&S.full[i]), 1);
            ptx::mbar_init(ptx::smem_u32(&S.empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(ptx::smem_u32(&S.tmem_full[i]), 1);
            ptx::mbar_init(ptx::smem_u32(&S.tmem_empty[i]), kBwdEpiWarps);
        }
        ptx::mbar_init(ptx::smem_u32(&S.mma_done), 1);
        ptx::fence_barrier_init();
        S.abort_flag = 0;
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_u32(&S.tmem_base), kTmemCols);
        ptx::tmem_relinquish();
    }
    if (warp == 2) {
        const int nseg = p.E + p.has_shared;
        const int per = (nseg + 31) / 32;
        const int s_begin = lane * per;
        int local = 0;
        for (int i = 0; i < per; ++i) {
            const int sg = s_begin + i;
            if (sg >= nseg) break;
            int rows, row0;
            if (p.has_shared && sg == 0) {
                rows = p.T; row0 = 0;
            } else {
                const int e = sg - p.has_shared;
                row0 = p.offsets[e];
                rows = p.counts[e];
            }
            S.seg_rows[sg] = rows;
            S.seg_row0[sg] = row0;
            local += bwd_tiles_of<kMode>(p, sg, rows);
        }
        int incl = local;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        int run = incl - local;
        for (int i = 0; i < per; ++i) {
            const int sg = s_begin + i;
            if (sg >= nseg) break;
            S.tile_start[sg] = run;
            run += bwd_tiles_of<kMode>(p, sg, S.seg_rows[sg]);
        }
        if (lane == 31) {
            S.total_tiles = incl;
            S.nseg = nseg;
            S.tile_start[nseg] = incl;
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const int total = S.total_tiles;
    const uint32_t tmem_base = S.tmem_base;

    if (warp == 0) {
        // ================= TMA producer =================
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued_mask = 0, issued_parity = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const BwdTile ti = decode_bwd<kMode>(S, p, tile);
                const CUtensorMap* mA = ti.routed ? &tmA_r : &tmA_s;
                const CUtensorMap* mB = ti.routed ? &tmB_r : &tmB_s;
                const CUtensorMap* mB2 = ti.routed ? &tmB2_r : &tmB2_s;
                const int b_base = ti.routed ? ti.expert * p.b_rows_per_expert : 0;
                const int i_blocks = ti.routed ? p.i_blocks_routed : p.i_blocks_shared;
                for (int kb = 0; kb < ti.kb; ++kb) {
                    if (!bounded_wait(ptx::smem_u32(&S.empty[stage]), phase ^ 1u, abort_flag, 0x141u)) {
                        ok = false;
                        break;
                    }
                    const uint32_t full = ptx::smem_u32(&S.full[stage]);
                    ptx::mbar_arrive_expect_tx(full, kTileABytes + kTileBBytes);
                    const uint32_t a_dst = ptx::smem_u32(smemA + stage * kTileABytes);
                    const uint32_t b_dst = ptx::smem_u32(smemB + stage * kTileBBytes);
                    if (kMode == kWgrad) {
                        // A: 128 output rows (MN) x 64 token rows (K); B: 256 output columns x 64 token rows.
                        const int krow = ti.row0 + kb * 64;
#pragma unroll
                        for (int j = 0; j < 2; ++j)
                            ptx::tma_load_2d(a_dst + j * (kTileABytes / 2), mA, full, ti.m * kBM + 64 * j, krow);
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            ptx::tma_load_2d(b_dst + j * (kTileBBytes / 4), mB, full, ti.n * kBN + 64 * j, krow);
                    } else {
                        const int a_row = ti.row0 + ti.m * kBM;
                        ptx::tma_load_2d(a_dst, mA, full, kb * kBK, a_row);
                        if (kMode == kRecompute) {
                            const int b_row = b_base + ti.n * (kBN / 2);
                            ptx::tma_load_2d(b_dst, mB, full, kb * kBK, b_row);
                            ptx::tma_load_2d(b_dst + kTileBBytes / 2, mB2, full, kb * kBK, b_row);
                        } else if (kMode == kFwdDown) {
                            ptx::tma_load_2d(b_dst, mB, full, kb * kBK, b_base + ti.n * kBN);
                        } else {
                            // B MN-major: 4 boxes of 64 output columns x 64 K rows of the weight.
                            const bool second = kMode == kDx && kb >= i_blocks;
                            const CUtensorMap* mb = second ? mB2 : mB;
                            const int krow = b_base + (second ? kb - i_blocks : kb) * kBK;
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                ptx::tma_load_2d(b_dst + j * (kTileBBytes / 4), mb, full, ti.n * kBN + 64 * j, krow);
                        }
                    }
                    issued_mask |= 1u << stage;
                    issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) {
                for (int s = 0; s < kStages; ++s)
                    if (issued_mask & (1u << s))
                        bounded_wait(ptx::smem_u32(&S.full[s]), (issued_parity >> s) & 1u, nullptr, 0x142u);
            }
        }
    } else if (warp == 1) {
        // ================= MMA issuer =================
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const BwdTile ti = decode_bwd<kMode>(S, p, tile);
                if (!bounded_wait(ptx::smem_u32(&S.tmem_empty[acc]), acc_phase ^ 1u, abort_flag, 0x241u)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBN);
                for (int kb = 0; kb < ti.kb; ++kb) {
                    if (!bounded_wait(ptx::smem_u32(&S.full[stage]), phase, abort_flag, 0x242u)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t a_addr = ptx::smem_u32(smemA + stage * kTileABytes);
                    const uint32_t b_addr = ptx::smem_u32(smemB + stage * kTileBBytes);
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k) {
                        // K-major: the next 16 K elements are 32 B further along the swizzled row;
                        // MN-major: 16 K rows of 128 B further.
                        const uint64_t ad = kAmn ? sw128_mnmajor_desc(a_addr + k * 2048, kTileABytes / 2)
                                                 : ptx::sw128_kmajor_desc(a_addr + k * 32);
                        const uint64_t bd = kBmn ? sw128_mnmajor_desc(b_addr + k * 2048, kTileBBytes / 4)
                                                 : ptx::sw128_kmajor_desc(b_addr + k * 32);
                        ptx::mma_bf16(d_tmem, ad, bd, p.idesc, (kb | k) != 0 ? 1u : 0u);
                    }
                    ptx::mma_commit(ptx::smem_u32(&S.empty[stage]));
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                ptx::mma_commit(ptx::smem_u32(&S.tmem_full[acc]));
                if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
            }
            ptx::mma_commit(ptx::smem_u32(&S.mma_done));
            bounded_wait(ptx::smem_u32(&S.mma_done), 0, nullptr, 0x243u);
        }
    } else {
        // ================= epilogue (warps 2..5) =================
        const int quarter = warp & 3;        // TMEM lanes 32*quarter .. +31
        const int half = (warp - 2) >> 2;    // accumulator columns 128*half .. +127
        const int c0 = half * (kBN / 64);    // first 32-column chunk of this warp
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            const BwdTile ti = decode_bwd<kMode>(S, p, tile);
            const bool got = bounded_wait(ptx::smem_u32(&S.tmem_full[acc]), acc_phase, abort_flag, 0x341u);
            __syncwarp();
            if (!__all_sync(0xffffffffu, got)) break;
            ptx::tc_fence_after();
            const uint32_t taddr = tmem_base + static_cast<uint32_t>(acc * kBN) +
                                   (static_cast<uint32_t>(quarter * 32) << 16);
            uint8_t* stage = stage_base + (warp - 2) * kBwdStagePerWarp;
            __nv_bfloat16* hs = reinterpret_cast<__nv_bfloat16*>(stage);
            const int r_warp0 = ti.m * kBM + quarter * 32;
            // Stage 32 bf16 values of this lane's row, then write 8 rows x 64 B per instruction.
            auto store_rows = [&](const float (&v)[32], __nv_bfloat16* base, int64_t ld, int col, int row_limit,
                                  int64_t row_origin) {
                uint4 pk[4];
                __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(pk);
#pragma unroll
                for (int q = 0; q < 16; ++q) h2[q] = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
                __syncwarp();
#pragma unroll
                for (int q = 0; q < 4; ++q) *reinterpret_cast<uint4*>(hs + lane * kStagePitchH + 8 * q) = pk[q];
                __syncwarp();
#pragma unroll
                for (int it = 0; it < 4; ++it) {
                    const int rw = it * 8 + (lane >> 2);
                    const int rl = r_warp0 + rw;
                    const uint4 val = *reinterpret_cast<const uint4*>(hs + rw * kStagePitchH + 8 * (lane & 3));
                    if (rl < row_limit)
                        *reinterpret_cast<uint4*>(base + (row_origin + rl) * ld + col + 8 * (lane & 3)) = val;
                }
            };
            const int r_local = r_warp0 + lane;
            if (kMode == kRecompute) {
                // Accumulator columns: g at 0..127, u at 128..255 for intermediate columns
                // n*128..; each warp takes two gate chunks and the matching up chunks, so it
                // can also form h = silu(g) u from the fp32 values (the training forward's h,
                // the same expression as the forward's SwiGLU epilogue).
                __nv_bfloat16* out = ti.routed ? p.out_routed : p.out_shared;
                const int64_t ld = ti.routed ? p.ld_routed : p.ld_shared;
                __nv_bfloat16* hout = ti.routed ? p.out2_routed : p.out2_shared;
                const int64_t ld2 = ti.routed ? p.ld2_routed : p.ld2_shared;
                const int ioff = ti.routed ? p.half_routed : p.half_shared;  // where u starts in a gu row
                const int limit = ti.rows;
#pragma unroll 1
                for (int i = 0; i < 2; ++i) {
                    const int c = 2 * half + i;
                    uint32_t gv[32], uv[32];
                    ptx::tmem_ld_32x32b_x32(taddr + c * 32, gv);
                    ptx::tmem_ld_32x32b_x32(taddr + (c + 4) * 32, uv);
                    ptx::tmem_wait_ld();
                    const int col = ti.n * (kBN / 2) + c * 32;
                    float f[32];
#pragma unroll
                    for (int q = 0; q < 32; ++q) f[q] = __uint_as_float(gv[q]);
                    store_rows(f, out, ld, col, limit, ti.row0);
#pragma unroll
                    for (int q = 0; q < 32; ++q) f[q] = __uint_as_float(uv[q]);
                    store_rows(f, out, ld, ioff + col, limit, ti.row0);
                    if (hout != nullptr) {
#pragma unroll
                        for (int q = 0; q < 32; ++q) {
                            const float g = __uint_as_float(gv[q]);
                            f[q] = g / (1.0f + __expf(-g)) * __uint_as_float(uv[q]);
                        }
                        store_rows(f, hout, ld2, col, limit, ti.row0);
                    }
                }
            } else if (kMode == kDh) {
                // dh for 256 intermediate columns n*256..; g and u of the same columns from gu.
                const bool routed = ti.routed;
                const __nv_bfloat16* gu = routed ? p.gu_routed : p.gu_shared;
                const int64_t gld = routed ? p.gu_ld_routed : p.gu_ld_shared;
                const int ioff = routed ? p.half_routed : p.half_shared;  // where u (du) starts in a row
                __nv_bfloat16* dgu = routed ? p.out_routed : p.out_shared;
                const int64_t ld = routed ? p.ld_routed : p.ld_shared;
                __nv_bfloat16* hout = routed ? p.out2_routed : p.out2_shared;
                const int64_t ld2 = routed ? p.ld2_routed : p.ld2_shared;
                // Padding rows of a routed segment get zeros (the weight-gradient sums run over them).
                const int limit = routed ? ((ti.rows + kBM - 1) / kBM) * kBM : ti.rows;
                const int n_valid = routed ? p.n_valid_routed : p.n_valid_shared;
                const bool row_ok = r_local < ti.rows;
                const int64_t grow = (int64_t)ti.row0 + r_local;
                float dot = 0.0f;
#pragma unroll 1
                for (int c = c0; c < c0 + kBN / 64; ++c) {
                    const int col = ti.n * kBN + c * 32;
                    if (col >= n_valid) break;  // uniform across the warp
                    uint32_t v[32];
                    ptx::tmem_ld_32x32b_x32(taddr + c * 32, v);
                    ptx::tmem_wait_ld();
                    // g and u of these 32 columns (packed bf16); zeros for rows past the segment.
                    uint4 gp[4], up[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        gp[q] = row_ok ? reinterpret_cast<const uint4*>(gu + grow * gld + col)[q] : make_uint4(0, 0, 0, 0);
                        up[q] = row_ok ? reinterpret_cast<const uint4*>(gu + grow * gld + ioff + col)[q]
                                       : make_uint4(0, 0, 0, 0);
                    }
                    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(gp);
                    const __nv_bfloat162* u2 = reinterpret_cast<const __nv_bfloat162*>(up);
                    float out[32];
                    // h = silu(g) u (and the routing-weight partial sum(dh h)), then du, then dg:
                    // one 32-value output live at a time.
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const float2 gf = __bfloat1622float2(g2[q]), uf = __bfloat1622float2(u2[q]);
                        const float s0 = 1.0f / (1.0f + __expf(-gf.x)), s1 = 1.0f / (1.0f + __expf(-gf.y));
                        out[2 * q] = gf.x * s0 * uf.x;
                        out[2 * q + 1] = gf.y * s1 * uf.y;
                        dot += __uint_as_float(v[2 * q]) * out[2 * q] + __uint_as_float(v[2 * q + 1]) * out[2 * q + 1];
                    }
                    store_rows(out, hout, ld2, col, limit, ti.row0);
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const float2 gf = __bfloat1622float2(g2[q]);
                        const float s0 = 1.0f / (1.0f + __expf(-gf.x)), s1 = 1.0f / (1.0f + __expf(-gf.y));
                        out[2 * q] = __uint_as_float(v[2 * q]) * gf.x * s0;
                        out[2 * q + 1] = __uint_as_float(v[2 * q + 1]) * gf.y * s1;
                    }
                    store_rows(out, dgu, ld, ioff + col, limit, ti.row0);
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const float2 gf = __bfloat1622float2(g2[q]), uf = __bfloat1622float2(u2[q]);
                        const float s0 = 1.0f / (1.0f + __expf(-gf.x)), s1 = 1.0f / (1.0f + __expf(-gf.y));
                        out[2 * q] = __uint_as_float(v[2 * q]) * uf.x * (s0 * (1.0f + gf.x * (1.0f - s0)));
                        out[2 * q + 1] = __uint_as_float(v[2 * q + 1]) * uf.y * (s1 * (1.0f + gf.y * (1.0f - s1)));
                    }
                    store_rows(out, dgu, ld, col, limit, ti.row0);
                }
                if (routed && row_ok) p.dw_part[grow * (2 * p.n_tiles_routed) + 2 * ti.n + half] = dot;
            } else if (kMode == kDx || kMode == kFwdDown) {
                const int n_valid = ti.routed ? p.n_valid_routed : p.n_valid_shared;
                __half* out_base = ti.routed ? p.yq_routed : p.yq_shared;
                uint8_t* sc_base = ti.routed ? p.ysc_routed : p.ysc_shared;
                __half* hq = reinterpret_cast<__half*>(stage);
                const bool row_ok = r_local < ti.rows;
                const int64_t grow = (int64_t)ti.row0 + r_local;
                float wrow = 1.0f;
                if (kMode == kFwdDown && ti.routed && row_ok) wrow = p.topk_w[p.perm_src[grow]];
                uint32_t codes[kBN / 64];
#pragma unroll
                for (int i = 0; i < kBN / 64; ++i) {
                    const int c = c0 + i;
                    __syncwarp();
                    uint32_t v[32];
                    ptx::tmem_ld_32x32b_x32(taddr + c * 32, v);
                    ptx::tmem_wait_ld();
                    const int col = ti.n * kBN + c * 32;
                    codes[i] = 0;
                    if (col >= n_valid) continue;
                    uint32_t mx = 0;
#pragma unroll
                    for (int q = 0; q < 32; ++q) mx = max(mx, __float_as_uint(fabsf(__uint_as_float(v[q]) * wrow)));
                    const uint32_t code = block_scale_code(mx);
                    const float f = block_encode_factor(code);
                    codes[i] = code;
                    uint4 pk[4];
                    __half2* h2 = reinterpret_cast<__half2*>(pk);
#pragma unroll
                    for (int q = 0; q < 16; ++q)
                        h2[q] = __floats2half2_rn(__uint_as_float(v[2 * q]) * wrow * f,
                                                  __uint_as_float(v[2 * q + 1]) * wrow * f);
#pragma unroll
                    for (int q = 0; q < 4; ++q) *reinterpret_cast<uint4*>(hq + lane * kStagePitchH + 8 * q) = pk[q];
                    __syncwarp();
#pragma unroll
                    for (int it = 0; it < 4; ++it) {
                        const int rw = it * 8 + (lane >> 2);
                        const int rl = r_warp0 + rw;
                        const uint4 val = *reinterpret_cast<const uint4*>(hq + rw * kStagePitchH + 8 * (lane & 3));
                        if (rl < ti.rows)
                            *reinterpret_cast<uint4*>(out_base + ((int64_t)ti.row0 + rl) * p.yq_ld + col +
                                                      8 * (lane & 3)) = val;
                    }
                }
                if (row_ok) {
                    uint8_t* dst = sc_base + grow * p.ysc_ld + ti.n * (kBN / 32);
                    const int nblk = min(kBN / 32, (n_valid - ti.n * kBN) / 32);
#pragma unroll
                    for (int i = 0; i < kBN / 64; ++i)
                        if (c0 + i < nblk) dst[c0 + i] = static_cast<uint8_t>(codes[i]);
                }
            } else {
                // kWgrad: output rows m*128 + r of this expert's dW (stacked outputs split at
                // split_rows), columns n*256..; a segment without rows gives zeros.
                const bool routed = ti.routed;
                const int split = routed ? p.split_rows_routed : p.split_rows_shared;
                const int orow = ti.m * kBM + quarter * 32;  // first output row of this warp
                __nv_bfloat16* base;
                int64_t ld, origin;
                if (orow < split) {
                    base = routed ? p.out_routed + ti.expert * p.out_expert_stride : p.out_shared;
                    ld = routed ? p.ld_routed : p.ld_shared;
                    origin = 0;
                } else {
                    base = routed ? p.out2_routed + ti.expert * p.out2_expert_stride : p.out2_shared;
                    ld = routed ? p.ld2_routed : p.ld2_shared;
                    origin = -split;
                }
#pragma unroll 1
                for (int c = c0; c < c0 + kBN / 64; ++c) {
                    float f[32];
                    if (ti.kb > 0) {
                        uint32_t v[32];
                        ptx::tmem_ld_32x32b_x32(taddr + c * 32, v);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int q = 0; q < 32; ++q) f[q] = __uint_as_float(v[q]);
                    } else {
#pragma unroll
                        for (int q = 0; q < 32; ++q) f[q] = 0.0f;
                    }
                    // Rows of a warp never straddle the split (split is a multiple of 128).
                    if (ti.n * kBN + c * 32 < (routed ? p.n_valid_routed : p.n_valid_shared))
                        store_rows(f, base, ld, ti.n * kBN + c * 32, 1 << 30, origin);
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&S.tmem_empty[acc]));
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace moe
