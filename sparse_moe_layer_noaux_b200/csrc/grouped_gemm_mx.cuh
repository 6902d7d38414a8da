// MXFP8 grouped expert GEMMs ("DeepSeek-V3 notes" (knlb.dev), § fp8: E4M3
// operands with fine-grained block scales, higher-precision accumulation;
// "DeepSeekV3.2-Tiered-Implementations", § DeepGEMM: FP8 grouped GEMM for the
// MoE experts).  Same persistent warp-specialised structure and tile schedule as
// the bf16 kernels, on tcgen05.mma kind::mxf8f6f4.block_scale:
//   * operands E4M3 with one power-of-two scale per 32 K-elements of every row
//     (A: token rows, B: weight rows); the tensor core applies the scales and
//     accumulates in fp32 in TMEM;
//   * a stage is 128 K-elements: A 128x128 B, B 256x128 B (the same bytes as a
//     bf16 stage of 64), plus the two operands' scale atoms (512 B for A, 2 x 512 B
//     for B), copied into TMEM with tcgen05.cp before the stage's four MMAs;
//   * routed expert segments start on 128-row boundaries (the dispatch pads them)
//     so that every A tile has exactly one scale atom per K slice;
//   * TMEM: two fp32 accumulators of 256 columns overlapping in 16 columns
//     (0..255 and 240..495) plus 12 scale columns (496..507); the epilogue reads
//     the overlapping chunk first and releases it, so the next tile's MMAs can
//     start while the rest of the tile is drained.
// Epilogues:
//   kSwiGLU  h = silu(A Wg^T) * (A Wu^T), quantised to MXFP8 for the down GEMM
//            (the 128 columns of a tile are one scale atom column of h);
//   kDown    y = w_row * (h Wd^T), block-scaled fp16 (as the bf16 path).
#pragma once
#include "grouped_gemm.cuh"
#include "mx.cuh"

namespace moe {

constexpr int kBKq = 128;                              // fp8 elements per stage (128-byte rows)
constexpr uint32_t kSfaBytes = kMxAtomBytes;           // one atom: 128 rows x 4 codes
constexpr uint32_t kSfbBytes = 2 * kMxAtomBytes;       // 256 B rows = two atoms
constexpr uint32_t kSfStageBytes = kSfaBytes + kSfbBytes;
constexpr uint32_t kStageTxMx = kTileABytes + kTileBBytes + kSfStageBytes;
constexpr uint32_t kAccCol1 = 240;                     // second accumulator's first column
constexpr uint32_t kOverlapCols = 256 - kAccCol1;      // 16
constexpr uint32_t kSfaCol = 496, kSfbCol = 500;       // scale columns (4 for A, 8 for B)
static_assert(kSfbCol + 8 <= kTmemCols, "scale columns exceed the TMEM allocation");
static_assert(kAccCol1 + kBN <= kSfaCol, "accumulator overlaps the scale columns");

struct GemmParamsMx {
    const int32_t* offsets;      // [E+1] first row of each routed segment (multiples of 128)
    const int32_t* counts;       // [E]   rows of each routed segment
    int E;
    int T;                       // rows of the shared segment
    int has_shared;
    int n_tiles_routed, n_tiles_shared;
    int kb_routed, kb_shared;    // K slices of 128
    int n_valid_routed, n_valid_shared;
    int b_rows_per_expert;
    const uint8_t* sfa_routed;   // A scale atoms (x_perm or h), k-atoms per row block = kb
    const uint8_t* sfa_shared;
    const uint8_t* sfb_routed;   // B scale atoms: gate (kSwiGLU) or down weights
    const uint8_t* sfb2_routed;  // kSwiGLU: up weights
    const uint8_t* sfb_shared;
    const uint8_t* sfb2_shared;
    int64_t b_rows_routed, b_rows_shared;  // rows of the B matrices (bound for the second atom)
    void* out_routed;            // kSwiGLU: h E4M3 [rows, ld]; kDown: y_perm fp16
    int64_t ld_routed;
    void* out_shared;
    int64_t ld_shared;
    uint8_t* hsf_routed;         // kSwiGLU: scale atoms of h
    uint8_t* hsf_shared;
    int hsf_katoms_routed, hsf_katoms_shared;
    uint8_t* scale_routed;       // kDown: y_perm block codes
    uint8_t* scale_shared;
    int64_t scale_ld;
    const int32_t* perm_src;     // kDown: routed row -> slot
    const float* topk_w;
    int64_t max_rows;            // padded routed row space Rp: segments must lie in [0, Rp)
    int64_t n_slots;             // kDown: entries of topk_w (perm_src values < n_slots)
    int row_major_band;          // column tiles per band of a row-major segment (>= 1)
};

struct GemmSmemMx {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t tmem_full[2];
    uint64_t tmem_empty[2];
    uint64_t ovl_free[2];        // the overlapping columns of an accumulator have been read
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort_flag;
    int total_tiles;
    int nseg;
    int seg_row0[kMaxSeg];
    int seg_rows[kMaxSeg];
    int tile_start[kMaxSeg + 1];
};

constexpr size_t kGemmMxSmemBytes =
    1024 + kStages * (kTileABytes + kTileBBytes + kSfStageBytes) + kStageBytes + sizeof(GemmSmemMx);

__device__ __forceinline__ TileInfo decode_tile_mx(const GemmSmemMx& s, const GemmParamsMx& p, int tile) {
    int lo = 0, hi = s.nseg - 1;  // largest seg with tile_start[seg] <= tile
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s.tile_start[mid] <= tile) lo = mid;
        else hi = mid - 1;
    }
    TileInfo ti;
    ti.seg = lo;
    ti.routed = !(p.has_shared && lo == 0);
    ti.expert = lo - p.has_shared;
    ti.rows = s.seg_rows[lo];
    ti.row0 = s.seg_row0[lo];
    const int mt = (ti.rows + kBM - 1) / kBM;
    const int local = tile - s.tile_start[lo];
    ti.row_major = mt >= kRowMajorMinRowTiles ? 1 : 0;
    if (ti.row_major) {
        // Bands of row_major_band column tiles, each walked row tile by row tile: a
        // row tile's A rows are read once per band while the band's weight tiles
        // stay in L2 (the last band may be narrower).
        const int nt = ti.routed ? p.n_tiles_routed : p.n_tiles_shared;
        const int band = (p.row_major_band >= 1 && p.row_major_band < nt) ? p.row_major_band : nt;
        const int b = local / (mt * band);
        const int bw = min(band, nt - b * band);
        const int in_band = local - b * mt * band;
        ti.m = in_band / bw;
        ti.n = b * band + (in_band - ti.m * bw);
    } else {
        ti.n = local / mt;
        ti.m = local - ti.n * mt;
    }
    ti.kb = ti.routed ? p.kb_routed : p.kb_shared;
    ti.r = min(kBM, ti.rows - ti.m * kBM);
    ti.swap = 0;
    ti.rpad = 0;
    return ti;
}

template <int kEpi>
__global__ void __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_mx_kernel(const __grid_constant__ CUtensorMap tmA_r, const __grid_constant__ CUtensorMap tmA_s,
                           const __grid_constant__ CUtensorMap tmB_r, const __grid_constant__ CUtensorMap tmB2_r,
                           const __grid_constant__ CUtensorMap tmB_s, const __grid_constant__ CUtensorMap tmB2_s,
                           const GemmParamsMx p) {
    static_assert(kEpi == kSwiGLU || kEpi == kDown, "MXFP8 epilogues: SwiGLU and down");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t* smemA = tiles;
    uint8_t* smemB = smemA + kStages * kTileABytes;
    uint8_t* smemSF = smemB + kStages * kTileBBytes;
    uint8_t* stage_base = smemSF + kStages * kSfStageBytes;
    GemmSmemMx& S = *reinterpret_cast<GemmSmemMx*>(stage_base + kStageBytes);
    volatile int* abort_flag = &S.abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- set-up: barriers, TMEM, segment table ----
    if (warp == 0 && lane == 0) {
        for (int i = 0; i < kStages; ++i) {
            ptx::mbar_init(ptx::smem_u32(&S.full[i]), 1);
            ptx::mbar_init(ptx::smem_u32(&S.empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(ptx::smem_u32(&S.tmem_full[i]), 1);
            ptx::mbar_init(ptx::smem_u32(&S.tmem_empty[i]), 4);
            ptx::mbar_init(ptx::smem_u32(&S.ovl_free[i]), 4);
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
        ptx::tmem_alloc(ptx::smem_u32(&S.tmem_base), kTmemCols);
        ptx::tmem_relinquish();
    }
    if (warp == 2) {
        // Segment table and exclusive prefix of tiles per segment (one warp scan).
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
                rows = checked_segment_rows(row0, p.counts[e], p.max_rows, kMxAtomRows);
                ntl = p.n_tiles_routed;
            }
            S.seg_rows[sg] = rows;
            S.seg_row0[sg] = row0;
            local += ((rows + kBM - 1) / kBM) * ntl;
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
            run += ((S.seg_rows[sg] + kBM - 1) / kBM) * ntl;
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
            // L2 policy as in the bf16 kernel: keep what the tile order re-reads.
            const uint64_t pol_keep = ptx::policy_evict_last();
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued_mask = 0, issued_parity = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const TileInfo ti = decode_tile_mx(S, p, tile);
                const CUtensorMap* mA = ti.routed ? &tmA_r : &tmA_s;
                const CUtensorMap* mB = ti.routed ? &tmB_r : &tmB_s;
                const CUtensorMap* mB2 = ti.routed ? &tmB2_r : &tmB2_s;
                const int a_row = ti.row0 + ti.m * kBM;  // a multiple of 128
                const int b_base = ti.routed ? ti.expert * p.b_rows_per_expert : 0;
                const int64_t slice = static_cast<int64_t>(ti.kb) * kMxAtomBytes;  // bytes per atom row
                const uint8_t* sfa = (ti.routed ? p.sfa_routed : p.sfa_shared) + (a_row / kMxAtomRows) * slice;
                const uint8_t* sfb0;
                const uint8_t* sfb1;
                int b_row;
                if (kEpi == kSwiGLU) {
                    b_row = b_base + ti.n * (kBN / 2);
                    sfb0 = (ti.routed ? p.sfb_routed : p.sfb_shared) + (b_row / kMxAtomRows) * slice;
                    sfb1 = (ti.routed ? p.sfb2_routed : p.sfb2_shared) + (b_row / kMxAtomRows) * slice;
                } else {
                    b_row = b_base + ti.n * kBN;
                    const uint8_t* sfb = ti.routed ? p.sfb_routed : p.sfb_shared;
                    const int64_t b_rows = ti.routed ? p.b_rows_routed : p.b_rows_shared;
                    sfb0 = sfb + (b_row / kMxAtomRows) * slice;
                    // The second 128 rows of the tile; past the matrix their columns are
                    // never stored, so any in-bounds atom will do.
                    sfb1 = (b_row + kMxAtomRows < b_rows) ? sfb0 + slice : sfb0;
                }
                for (int kb = 0; kb < ti.kb; ++kb) {
                    if (!bounded_wait(ptx::smem_u32(&S.empty[stage]), phase ^ 1u, abort_flag, 0x121u)) {
                        ok = false;
                        break;
                    }
                    const uint32_t full = ptx::smem_u32(&S.full[stage]);
                    ptx::mbar_arrive_expect_tx(full, kStageTxMx);
                    const uint32_t a_dst = ptx::smem_u32(smemA + stage * kTileABytes);
                    const uint32_t b_dst = ptx::smem_u32(smemB + stage * kTileBBytes);
                    const uint32_t sf_dst = ptx::smem_u32(smemSF + stage * kSfStageBytes);
                    if (ti.row_major) {
                        ptx::tma_load_2d(a_dst, mA, full, kb * kBKq, a_row);
                        ptx::tma_load_2d(b_dst, mB, full, kb * kBKq, b_row, pol_keep);
                        if (kEpi == kSwiGLU)
                            ptx::tma_load_2d(b_dst + kTileBBytes / 2, mB2, full, kb * kBKq, b_row, pol_keep);
                    } else {
                        ptx::tma_load_2d(a_dst, mA, full, kb * kBKq, a_row, pol_keep);
                        ptx::tma_load_2d(b_dst, mB, full, kb * kBKq, b_row);
                        if (kEpi == kSwiGLU) ptx::tma_load_2d(b_dst + kTileBBytes / 2, mB2, full, kb * kBKq, b_row);
                    }
                    ptx::bulk_load(sf_dst, sfa + kb * kMxAtomBytes, kMxAtomBytes, full);
                    ptx::bulk_load(sf_dst + kSfaBytes, sfb0 + kb * kMxAtomBytes, kMxAtomBytes, full);
                    ptx::bulk_load(sf_dst + kSfaBytes + kMxAtomBytes, sfb1 + kb * kMxAtomBytes, kMxAtomBytes, full);
                    issued_mask |= 1u << stage;
                    issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) {
                for (int s = 0; s < kStages; ++s)
                    if (issued_mask & (1u << s))
                        bounded_wait(ptx::smem_u32(&S.full[s]), (issued_parity >> s) & 1u, nullptr, 0x122u);
            }
        }
    } else if (warp == 1) {
        // ================= MMA issuer =================
        if (lane == 0) {
            const uint32_t sfa_t = tmem_base + kSfaCol, sfb_t = tmem_base + kSfbCol;
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int j = 0;  // tiles of this CTA so far
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++j) {
                const TileInfo ti = decode_tile_mx(S, p, tile);
                const int acc = j & 1;
                // Accumulator `acc` was drained by the epilogue of tile j - 2, and the
                // columns it shares with the other accumulator by that of tile j - 1.
                if (!bounded_wait(ptx::smem_u32(&S.tmem_empty[acc]), ((j >> 1) & 1) ^ 1u, abort_flag, 0x221u) ||
                    (j > 0 && !bounded_wait(ptx::smem_u32(&S.ovl_free[acc ^ 1]), ((j - 1) >> 1) & 1, abort_flag,
                                            0x224u))) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t d_tmem = tmem_base + (acc ? kAccCol1 : 0u);
                for (int kb = 0; kb < ti.kb; ++kb) {
                    if (!bounded_wait(ptx::smem_u32(&S.full[stage]), phase, abort_flag, 0x222u)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t a_addr = ptx::smem_u32(smemA + stage * kTileABytes);
                    const uint32_t b_addr = ptx::smem_u32(smemB + stage * kTileBBytes);
                    const uint32_t sf_addr = ptx::smem_u32(smemSF + stage * kSfStageBytes);
                    // Scale atoms into TMEM (executed in order with the MMAs around them).
                    ptx::tmem_cp_32x128b_warpx4(sfa_t, ptx::plain_kmajor_desc(sf_addr, 128));
                    ptx::tmem_cp_32x128b_warpx4(sfb_t, ptx::plain_kmajor_desc(sf_addr + kSfaBytes, 128));
                    ptx::tmem_cp_32x128b_warpx4(sfb_t + 4, ptx::plain_kmajor_desc(sf_addr + kSfaBytes + kMxAtomBytes, 128));
#pragma unroll
                    for (int k = 0; k < kBKq / 32; ++k) {
                        const uint64_t ad = ptx::sw128_kmajor_desc(a_addr + k * 32);
                        const uint64_t bd = ptx::sw128_kmajor_desc(b_addr + k * 32);
                        ptx::mma_mxf8(d_tmem, ad, bd, ptx::idesc_mxf8(kBM, kBN, k, k), sfa_t, sfb_t,
                                      (kb | k) != 0 ? 1u : 0u);
                    }
                    ptx::mma_commit(ptx::smem_u32(&S.empty[stage]));
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                ptx::mma_commit(ptx::smem_u32(&S.tmem_full[acc]));
            }
            ptx::mma_commit(ptx::smem_u32(&S.mma_done));
            bounded_wait(ptx::smem_u32(&S.mma_done), 0, nullptr, 0x223u);
        }
    } else {
        // ================= epilogue (warps 2..5) =================
        const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
        int j = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++j) {
            const TileInfo ti = decode_tile_mx(S, p, tile);
            const int acc = j & 1;
            const bool got = bounded_wait(ptx::smem_u32(&S.tmem_full[acc]), (j >> 1) & 1, abort_flag, 0x321u);
            __syncwarp();
            if (!__all_sync(0xffffffffu, got)) break;
            ptx::tc_fence_after();
            const int r_local = ti.m * kBM + quarter * 32 + lane;
            const bool row_ok = r_local < ti.rows;
            const int64_t grow = (int64_t)ti.row0 + r_local;
            const uint32_t taddr = tmem_base + (acc ? kAccCol1 : 0u) + (static_cast<uint32_t>(quarter * 32) << 16);
            uint8_t* stage = stage_base + (warp - 2) * kStageBytesPerWarp;
            const int r_warp0 = ti.m * kBM + quarter * 32;
            auto release_overlap = [&]() {
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&S.ovl_free[acc]));
            };
            if (kEpi == kSwiGLU) {
                // Four chunks of 32 output columns: gate at c*32, up at 128 + c*32.  The
                // overlap (columns 240..255 of accumulator 0, 0..15 of accumulator 1)
                // lies in chunk 3 resp. chunk 0, which goes first.
                const int first = acc ? 0 : 3;
                constexpr int kPitch = 144;  // staging row pitch in bytes (128 + 16)
                uint32_t codes = 0;
#pragma unroll 1
                for (int ci = 0; ci < 4; ++ci) {
                    const int c = (first + ci) & 3;
                    __syncwarp();
                    uint32_t g[32], u[32];
                    ptx::tmem_ld_32x32b_x32(taddr + c * 32, g);
                    ptx::tmem_ld_32x32b_x32(taddr + kBN / 2 + c * 32, u);
                    ptx::tmem_wait_ld();
                    if (ci == 0) release_overlap();
                    float h[32];
                    uint32_t mx = 0;
#pragma unroll
                    for (int q = 0; q < 32; ++q) {
                        const float gv = __uint_as_float(g[q]), uv = __uint_as_float(u[q]);
                        h[q] = row_ok ? gv / (1.0f + __expf(-gv)) * uv : 0.0f;
                        mx = max(mx, __float_as_uint(fabsf(h[q])));
                    }
                    const uint32_t code = mx_scale_code(mx);
                    const float f = mx_encode_factor(code);
                    codes |= code << (8 * c);
                    uint4 pk[2];
                    uint32_t* w = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        w[q] = e4m3x2(h[4 * q] * f, h[4 * q + 1] * f) | (e4m3x2(h[4 * q + 2] * f, h[4 * q + 3] * f) << 16);
                    *reinterpret_cast<uint4*>(stage + lane * kPitch + c * 32) = pk[0];
                    *reinterpret_cast<uint4*>(stage + lane * kPitch + c * 32 + 16) = pk[1];
                }
                __syncwarp();
                // 4 rows x 128 B per instruction: lanes 8r..8r+7 write row r's 16-byte pieces.
                uint8_t* out_base = static_cast<uint8_t*>(ti.routed ? p.out_routed : p.out_shared);
                const int64_t ld = ti.routed ? p.ld_routed : p.ld_shared;
#pragma unroll
                for (int it = 0; it < 8; ++it) {
                    const int rw = it * 4 + (lane >> 3);
                    const uint4 v = *reinterpret_cast<const uint4*>(stage + rw * kPitch + (lane & 7) * 16);
                    *reinterpret_cast<uint4*>(out_base + ((int64_t)ti.row0 + r_warp0 + rw) * ld + ti.n * (kBN / 2) +
                                              (lane & 7) * 16) = v;
                }
                // This row's four codes are one 32-bit word of the h scale atom (row block
                // of the tile, K slice n of h).
                uint8_t* hsf = ti.routed ? p.hsf_routed : p.hsf_shared;
                const int katoms = ti.routed ? p.hsf_katoms_routed : p.hsf_katoms_shared;
                *reinterpret_cast<uint32_t*>(hsf + mx_sf_word_offset(grow, ti.n, katoms)) = codes;
            } else {
                const int n_valid = ti.routed ? p.n_valid_routed : p.n_valid_shared;
                __half* out_base = ti.routed ? static_cast<__half*>(p.out_routed) : static_cast<__half*>(p.out_shared);
                uint8_t* sc_base = ti.routed ? p.scale_routed : p.scale_shared;
                const int64_t ld = ti.routed ? p.ld_routed : p.ld_shared;
                __half* hs = reinterpret_cast<__half*>(stage);
                float wrow = 1.0f;
                if (ti.routed && row_ok) wrow = row_weight(p.perm_src, p.topk_w, grow, p.n_slots);
                const int first = acc ? 0 : kBN / 32 - 1;
                uint32_t codes_lo = 0, codes_hi = 0;
#pragma unroll 1
                for (int ci = 0; ci < kBN / 32; ++ci) {
                    const int c = (first + ci) & (kBN / 32 - 1);
                    __syncwarp();
                    uint32_t v[32];
                    ptx::tmem_ld_32x32b_x32(taddr + c * 32, v);
                    ptx::tmem_wait_ld();
                    if (ci == 0) release_overlap();
                    const int col = ti.n * kBN + c * 32;
                    if (col >= n_valid) continue;  // uniform across the warp
                    uint32_t mx = 0;
#pragma unroll
                    for (int q = 0; q < 32; ++q) mx = max(mx, __float_as_uint(fabsf(__uint_as_float(v[q]) * wrow)));
                    const uint32_t code = block_scale_code(mx);
                    const float f = block_encode_factor(code);
                    if (c < 4) codes_lo |= code << (8 * c);
                    else codes_hi |= code << (8 * (c - 4));
                    uint4 pk[4];
                    __half2* h2 = reinterpret_cast<__half2*>(pk);
#pragma unroll
                    for (int q = 0; q < 16; ++q)
                        h2[q] = __floats2half2_rn(__uint_as_float(v[2 * q]) * wrow * f,
                                                  __uint_as_float(v[2 * q + 1]) * wrow * f);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        *reinterpret_cast<uint4*>(hs + lane * kStagePitchH + 8 * q) = pk[q];
                    __syncwarp();
#pragma unroll
                    for (int it = 0; it < 4; ++it) {
                        const int rw = it * 8 + (lane >> 2);
                        const int rl = r_warp0 + rw;
                        const uint4 val = *reinterpret_cast<const uint4*>(hs + rw * kStagePitchH + 8 * (lane & 3));
                        if (rl < ti.rows)
                            *reinterpret_cast<uint4*>(out_base + ((int64_t)ti.row0 + rl) * ld + col + 8 * (lane & 3)) = val;
                    }
                }
                if (row_ok) {
                    uint8_t* dst = sc_base + grow * p.scale_ld + ti.n * (kBN / 32);
                    const int nblk = min(kBN / 32, (n_valid - ti.n * kBN) / 32);
                    if (nblk == kBN / 32) {
                        *reinterpret_cast<uint2*>(dst) = make_uint2(codes_lo, codes_hi);
                    } else {
                        for (int c = 0; c < nblk; ++c)
                            dst[c] = static_cast<uint8_t>((c < 4 ? codes_lo >> (8 * c) : codes_hi >> (8 * (c - 4))) & 0xffu);
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&S.tmem_empty[acc]));
        }
    }

    // ---- teardown ----
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace moe
