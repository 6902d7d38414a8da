// Grouped expert GEMMs on CTA pairs (tcgen05 .cta_group::2): the prefill path.
//
// Same computation and tile schedule idea as grouped_gemm.cuh, but two CTAs on
// neighbouring SMs (a cluster of 2) compute one 256-row x 256-column tile with
// one MMA stream issued by the pair's leader:
//   - each CTA loads its own 128 rows of A and its own half (128 rows) of the
//     256-row B tile, so every SM reads half of the weight tile it multiplies
//     with: per 128 x 256 x 64 block of work an SM brings in 32 KB instead of
//     48 KB;
//   - the last, partial row tile of a segment with at most 128 rows left runs as
//     an M = 128 pair tile (64 rows per CTA), so padding stays under 128 rows;
//   - accumulators live in each CTA's TMEM (two 256-column buffers); for
//     M = 128 tiles the hardware places a CTA's 64 rows on TMEM lanes 0-63 for
//     columns 0-127 and on lanes 64-127 for columns 128-255.
// The gate/up B tile is interleaved per 64 columns — gate 0-63, up 0-63 (CTA 0),
// gate 64-127, up 64-127 (CTA 1) — so every TMEM lane holds matching gate and up
// columns in both tile shapes.
//
// Protocol: both CTAs' TMA loads complete on the leader's full barrier (only the
// leader expects the bytes); the leader issues the MMAs and its commits arrive
// on the empty / tmem-full barriers of both CTAs; both CTAs' epilogue warps
// release an accumulator on the leader's tmem-empty barrier (8 arrivals).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "grouped_gemm.cuh"
#include "sm100_ptx.cuh"

namespace moe {

constexpr int kStages2 = 6;
constexpr uint32_t kTileA2Bytes = 128 * kBK * 2;  // 16 KB: this CTA's 128 rows of A
constexpr uint32_t kTileB2Bytes = 128 * kBK * 2;  // 16 KB: this CTA's half of B
constexpr uint32_t kPairStageBytes = 2 * (kTileA2Bytes + kTileB2Bytes);  // both CTAs, one stage

struct GemmSmem2 {
    uint64_t full[kStages2];
    uint64_t empty[kStages2];
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

constexpr size_t kGemm2SmemBytes =
    1024 + kStages2 * (kTileA2Bytes + kTileB2Bytes) + kStageBytes + sizeof(GemmSmem2);

struct PairTile {
    int routed, expert;
    int m, n;      // m counts 256-row tiles
    int rows;      // rows of the segment
    int row0;      // first row of the segment
    int kb;
    int r;         // rows of this pair tile (1..256)
    int m128;      // 1: M = 128 pair tile (64 rows per CTA)
};

__device__ __forceinline__ bool bounded_wait_cl(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                                unsigned code) {
    if (ptx::mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    for (uint32_t n = 1;; ++n) {
        if (ptx::mbar_try_wait_cluster(bar, parity)) return true;
        if ((n & 63u) == 0) {
            if (abort_flag && *abort_flag) return false;
            if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) {
                record_error(code);
                if (abort_flag) *abort_flag = 1;
                return false;
            }
        }
    }
}

__device__ __forceinline__ PairTile decode_pair_tile(const GemmSmem2& s, const GemmParams& p, int tile) {
    int lo = 0, hi = s.nseg - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s.tile_start[mid] <= tile) lo = mid;
        else hi = mid - 1;
    }
    PairTile t;
    t.routed = !(p.has_shared && lo == 0);
    t.expert = lo - p.has_shared;
    t.rows = s.seg_rows[lo];
    t.row0 = s.seg_row0[lo];
    const int mt = (t.rows + 255) / 256;
    const int local = tile - s.tile_start[lo];
    t.n = local / mt;
    t.m = local - t.n * mt;
    t.kb = t.routed ? p.kb_routed : p.kb_shared;
    t.r = min(256, t.rows - t.m * 256);
    t.m128 = t.r <= 128 ? 1 : 0;
    return t;
}

template <int kEpi>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_2sm_kernel(const __grid_constant__ CUtensorMap tmA_r, const __grid_constant__ CUtensorMap tmA_s,
                            const __grid_constant__ CUtensorMap tmB_r, const __grid_constant__ CUtensorMap tmB2_r,
                            const __grid_constant__ CUtensorMap tmB_s, const __grid_constant__ CUtensorMap tmB2_s,
                            const GemmParams p) {
    static_assert(kEpi == kSwiGLU || kEpi == kDown, "pair kernel: gate/up or down");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t* smemA = tiles;
    uint8_t* smemB = tiles + kStages2 * kTileA2Bytes;
    uint8_t* stage_base = tiles + kStages2 * (kTileA2Bytes + kTileB2Bytes);
    GemmSmem2& S = *reinterpret_cast<GemmSmem2*>(stage_base + kStageBytes);
    volatile int* abort_flag = &S.abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = ptx::cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;

    // ---- set-up ----
    if (warp == 0 && lane == 0) {
        for (int i = 0; i < kStages2; ++i) {
            ptx::mbar_init(ptx::smem_u32(&S.full[i]), 1);
            ptx::mbar_init(ptx::smem_u32(&S.empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(ptx::smem_u32(&S.tmem_full[i]), 1);
            ptx::mbar_init(ptx::smem_u32(&S.tmem_empty[i]), 8);  // 4 epilogue warps x 2 CTAs
        }
        ptx::mbar_init(ptx::smem_u32(&S.mma_done), 1);
        ptx::fence_barrier_init();
        S.abort_flag = 0;
        ptx::prefetch_tensormap(&tmA_r);
        ptx::prefetch_tensormap(&tmB_r);
        if (kEpi == kSwiGLU) ptx::prefetch_tensormap(&tmB2_r);
        if (p.has_shared) {
            ptx::prefetch_tensormap(&tmA_s);
            ptx::prefetch_tensormap(&tmB_s);
            if (kEpi == kSwiGLU) ptx::prefetch_tensormap(&tmB2_s);
        }
    }
    if (warp == 1) {
        ptx::tmem_alloc_pair(ptx::smem_u32(&S.tmem_base), kTmemCols);
        ptx::tmem_relinquish_pair();
    }
    if (warp == 2) {
        // Segment table; pair tiles of 256 rows per segment.
        const int nseg = p.E + p.has_shared;
        const int per = (nseg + 31) / 32;
        const int s_begin = lane * per;
        int local = 0;
        for (int i = 0; i < per; ++i) {
            const int sg = s_begin + i;
            if (sg >= nseg) break;
            int rows, row0, ntl;
            if (p.has_shared && sg == 0) {
                rows = p.T; row0 = 0; ntl = p.n_tiles_shared;
            } else {
                const int e = sg - p.has_shared;
                row0 = p.offsets[e];
                rows = p.offsets[e + 1] - row0;
                ntl = p.n_tiles_routed;
            }
            S.seg_rows[sg] = rows;
            S.seg_row0[sg] = row0;
            local += ((rows + 255) / 256) * ntl;
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
            const int ntl = (p.has_shared && sg == 0) ? p.n_tiles_shared : p.n_tiles_routed;
            run += ((S.seg_rows[sg] + 255) / 256) * ntl;
        }
        if (lane == 31) {
            S.total_tiles = incl;
            S.nseg = nseg;
            S.tile_start[nseg] = incl;
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();  // the peer's barriers and TMEM exist before anyone signals them
    ptx::tc_fence_after();

    const int total = S.total_tiles;
    const uint32_t tmem_base = S.tmem_base;

    if (warp == 0) {
        // ================= TMA producer (both CTAs) =================
        if (lane == 0) {
            const uint64_t pol_a = ptx::policy_evict_last();
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int tile = pair; tile < total && ok; tile += num_pairs) {
                const PairTile ti = decode_pair_tile(S, p, tile);
                const CUtensorMap* mA = ti.routed ? &tmA_r : &tmA_s;
                const CUtensorMap* mB = ti.routed ? &tmB_r : &tmB_s;
                const CUtensorMap* mB2 = ti.routed ? &tmB2_r : &tmB2_s;
                const int a_row = ti.row0 + ti.m * 256 + static_cast<int>(rank) * (ti.m128 ? 64 : 128);
                const int b_base = ti.routed ? ti.expert * p.b_rows_per_expert : 0;
                for (int kb = 0; kb < ti.kb; ++kb) {
                    if (!bounded_wait_cl(ptx::smem_u32(&S.empty[stage]), phase ^ 1u, abort_flag, 0x111u)) {
                        ok = false;
                        break;
                    }
                    const uint32_t full_local = ptx::smem_u32(&S.full[stage]);
                    const uint32_t full_leader = ptx::map_to_rank(full_local, 0);
                    if (leader) ptx::mbar_arrive_expect_tx(full_local, kPairStageBytes);
                    const uint32_t a_dst = ptx::smem_u32(smemA + stage * kTileA2Bytes);
                    const uint32_t b_dst = ptx::smem_u32(smemB + stage * kTileB2Bytes);
                    ptx::tma_load_2d_pair(a_dst, mA, full_leader, kb * kBK, a_row, pol_a);
                    if (kEpi == kSwiGLU) {
                        const int b_row = b_base + ti.n * (kBN / 2) + static_cast<int>(rank) * 64;
                        ptx::tma_load_2d_pair(b_dst, mB, full_leader, kb * kBK, b_row);
                        ptx::tma_load_2d_pair(b_dst + kTileB2Bytes / 2, mB2, full_leader, kb * kBK, b_row);
                    } else {
                        const int b_row = b_base + ti.n * kBN + static_cast<int>(rank) * 128;
                        ptx::tma_load_2d_pair(b_dst, mB, full_leader, kb * kBK, b_row);
                    }
                    if (++stage == kStages2) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) {
                // The loads complete on the leader's barrier, which this thread cannot
                // wait on from the follower: give copies in flight a bounded 50 us to land.
                const uint64_t t0 = ptx::globaltimer_ns();
                while (ptx::globaltimer_ns() - t0 < 50000ull) __nanosleep(1000);
            }
        }
    } else if (warp == 1) {
        // ================= MMA issuer (leader only) =================
        if (lane == 0 && leader) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = pair; tile < total && ok; tile += num_pairs) {
                const PairTile ti = decode_pair_tile(S, p, tile);
                if (!bounded_wait_cl(ptx::smem_u32(&S.tmem_empty[acc]), acc_phase ^ 1u, abort_flag, 0x211u)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBN);
                const uint32_t idesc = ptx::idesc_bf16_f32(ti.m128 ? 128 : 256, kBN);
                for (int kb = 0; kb < ti.kb; ++kb) {
                    if (!bounded_wait_cl(ptx::smem_u32(&S.full[stage]), phase, abort_flag, 0x212u)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t a_addr = ptx::smem_u32(smemA + stage * kTileA2Bytes);
                    const uint32_t b_addr = ptx::smem_u32(smemB + stage * kTileB2Bytes);
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)
                        ptx::mma_bf16_pair(d_tmem, ptx::sw128_kmajor_desc(a_addr + k * 32),
                                           ptx::sw128_kmajor_desc(b_addr + k * 32), idesc, (kb | k) != 0 ? 1u : 0u);
                    ptx::mma_commit_pair(ptx::smem_u32(&S.empty[stage]), 0x3);
                    if (++stage == kStages2) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                ptx::mma_commit_pair(ptx::smem_u32(&S.tmem_full[acc]), 0x3);
                if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
            }
            ptx::mma_commit_pair(ptx::smem_u32(&S.mma_done), 0x1);
            bounded_wait_cl(ptx::smem_u32(&S.mma_done), 0, nullptr, 0x213u);
        }
    } else {
        // ================= epilogue (warps 2..5, both CTAs) =================
        const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
        uint8_t* stage = stage_base + (warp - 2) * kStageBytesPerWarp;
        const uint32_t empty_leader[2] = {ptx::map_to_rank(ptx::smem_u32(&S.tmem_empty[0]), 0),
                                          ptx::map_to_rank(ptx::smem_u32(&S.tmem_empty[1]), 0)};
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = pair; tile < total; tile += num_pairs) {
            const PairTile ti = decode_pair_tile(S, p, tile);
            const bool got = bounded_wait_cl(ptx::smem_u32(&S.tmem_full[acc]), acc_phase, abort_flag, 0x311u);
            __syncwarp();
            if (!__all_sync(0xffffffffu, got)) break;
            ptx::tc_fence_after();
            // Rows of this warp and the TMEM column window it reads.
            //   M = 256: this CTA's rows 128*rank + 32*quarter + lane, all 256 columns.
            //   M = 128: rows 64*rank + 32*(quarter % 2) + lane; quarters 0-1 hold
            //            columns 0-127, quarters 2-3 columns 128-255, both at TMEM
            //            columns 0-127.
            const int half = ti.m128 ? (quarter >> 1) : 0;
            const int r_warp0 = ti.m * 256 + (ti.m128 ? 64 * static_cast<int>(rank) + 32 * (quarter & 1)
                                                      : 128 * static_cast<int>(rank) + 32 * quarter);
            const int r_local = r_warp0 + lane;
            const bool row_ok = r_local < ti.rows;
            const int64_t grow = (int64_t)ti.row0 + r_local;
            const uint32_t taddr = tmem_base + static_cast<uint32_t>(acc * kBN) +
                                   (static_cast<uint32_t>(quarter * 32) << 16);
            const int64_t ld = ti.routed ? p.ld_routed : p.ld_shared;
            const int n_valid = ti.routed ? p.n_valid_routed : p.n_valid_shared;
            if (kEpi == kSwiGLU) {
                __nv_bfloat16* out_base = ti.routed ? static_cast<__nv_bfloat16*>(p.out_routed)
                                                    : static_cast<__nv_bfloat16*>(p.out_shared);
                __nv_bfloat16* hs = reinterpret_cast<__nv_bfloat16*>(stage);
                const int npairs = ti.m128 ? 2 : 4;
#pragma unroll 1
                for (int q = 0; q < npairs; ++q) {
                    // Gate columns at TMEM g_col, matching up columns 64 further.
                    const int hf = ti.m128 ? half : (q >> 1);
                    const int sub = q & 1;
                    const int g_col = (ti.m128 ? 0 : hf * 128) + sub * 32;
                    const int col = ti.n * (kBN / 2) + hf * 64 + sub * 32;
                    __syncwarp();
                    uint32_t g[32], u[32];
                    ptx::tmem_ld_32x32b_x32(taddr + g_col, g);
                    ptx::tmem_ld_32x32b_x32(taddr + g_col + 64, u);
                    ptx::tmem_wait_ld();
                    if (col >= n_valid) continue;  // uniform across the warp
                    uint4 pk[4];
                    __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(pk);
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float g0 = __uint_as_float(g[2 * j]), g1 = __uint_as_float(g[2 * j + 1]);
                        const float u0 = __uint_as_float(u[2 * j]), u1 = __uint_as_float(u[2 * j + 1]);
                        h2[j] = __floats2bfloat162_rn(g0 / (1.0f + __expf(-g0)) * u0, g1 / (1.0f + __expf(-g1)) * u1);
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        *reinterpret_cast<uint4*>(hs + lane * kStagePitchH + 8 * j) = pk[j];
                    __syncwarp();
#pragma unroll
                    for (int it = 0; it < 4; ++it) {
                        const int rw = it * 8 + (lane >> 2);
                        const uint4 v = *reinterpret_cast<const uint4*>(hs + rw * kStagePitchH + 8 * (lane & 3));
                        if (r_warp0 + rw < ti.rows)
                            *reinterpret_cast<uint4*>(out_base + ((int64_t)ti.row0 + r_warp0 + rw) * ld + col +
                                                      8 * (lane & 3)) = v;
                    }
                }
            } else {
                __half* out_base = ti.routed ? static_cast<__half*>(p.out_routed) : static_cast<__half*>(p.out_shared);
                uint8_t* sc_base = ti.routed ? p.scale_routed : p.scale_shared;
                __half* hs = reinterpret_cast<__half*>(stage);
                float wrow = 1.0f;
                if (ti.routed && row_ok) wrow = p.topk_w[p.perm_src[grow]];
                const int nchunks = ti.m128 ? 4 : 8;
                const int col0 = ti.n * kBN + half * 128;  // first output column of this warp
                uint32_t codes[8];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    codes[c] = 0;
                    if (c >= nchunks) continue;  // uniform
                    __syncwarp();
                    uint32_t v[32];
                    ptx::tmem_ld_32x32b_x32(taddr + c * 32, v);
                    ptx::tmem_wait_ld();
                    const int col = col0 + c * 32;
                    if (col >= n_valid) continue;  // uniform across the warp
                    uint32_t mx = 0;
#pragma unroll
                    for (int j = 0; j < 32; ++j) mx = max(mx, __float_as_uint(fabsf(__uint_as_float(v[j]) * wrow)));
                    const uint32_t code = block_scale_code(mx);
                    const float f = block_encode_factor(code);
                    codes[c] = code;
                    uint4 pk[4];
                    __half2* h2 = reinterpret_cast<__half2*>(pk);
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        h2[j] = __floats2half2_rn(__uint_as_float(v[2 * j]) * wrow * f,
                                                  __uint_as_float(v[2 * j + 1]) * wrow * f);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        *reinterpret_cast<uint4*>(hs + lane * kStagePitchH + 8 * j) = pk[j];
                    __syncwarp();
#pragma unroll
                    for (int it = 0; it < 4; ++it) {
                        const int rw = it * 8 + (lane >> 2);
                        const uint4 val = *reinterpret_cast<const uint4*>(hs + rw * kStagePitchH + 8 * (lane & 3));
                        if (r_warp0 + rw < ti.rows)
                            *reinterpret_cast<uint4*>(out_base + ((int64_t)ti.row0 + r_warp0 + rw) * ld + col +
                                                      8 * (lane & 3)) = val;
                    }
                }
                if (row_ok) {
                    uint8_t* dst = sc_base + grow * p.scale_ld + col0 / 32;
                    const int nblk = min(nchunks, (n_valid - col0) / 32);
                    if (nblk == 8) {
                        uint2 pk;
                        pk.x = codes[0] | (codes[1] << 8) | (codes[2] << 16) | (codes[3] << 24);
                        pk.y = codes[4] | (codes[5] << 8) | (codes[6] << 16) | (codes[7] << 24);
                        *reinterpret_cast<uint2*>(dst) = pk;
                    } else if (nblk == 4) {
                        *reinterpret_cast<uint32_t*>(dst) = codes[0] | (codes[1] << 8) | (codes[2] << 16) | (codes[3] << 24);
                    } else {
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            if (c < nblk) dst[c] = static_cast<uint8_t>(codes[c]);
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive_remote(empty_leader[acc]);
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
    }

    // ---- teardown ----
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();  // the leader's MMAs into this CTA's TMEM and all remote signals are done
    if (warp == 1) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

}  // namespace moe
