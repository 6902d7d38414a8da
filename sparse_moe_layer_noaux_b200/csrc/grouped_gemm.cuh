// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM),
// fed by TMA.  One persistent CTA per SM walks a static schedule of output
// tiles over variable-length expert segments read on the device (no host sync):
//   segment 0        the shared expert over all T tokens (when S > 0);
//   segment 1 + e    routed expert e, rows expert_offsets[e] .. expert_offsets[e+1].
// Two instantiations:
//   kSwiGLU  h = silu(A Wg^T) * (A Wu^T)   — gate and up tiles side by side in one
//            N = 256 accumulator (128 gate columns | 128 up columns), fused epilogue;
//   kDown    y = w_row * (h Wd^T)           — N = 256, routing weight in the epilogue,
//            output in block-scaled fp16 (fp16 values, one power-of-two scale per
//            32 consecutive columns of a row, chosen from the block's largest
//            magnitude): fp16's 11-bit precision relative to the block maximum, no
//            overflow, half the bytes of fp32;
//   kLogits  router logits l = x Wr^T in fp32 from an exact three-way bf16 split
//            Wr = hi + mid + lo (one segment of T rows, K = 3 H: each 64-column
//            block of x meets the three planes back to back, so its second and
//            third loads come from L2 and x streams from HBM once; N = E rounded
//            up to 16), fp32 output.
// ("The Evolving Transformer · 07", § 02: each routed expert is a SwiGLU FFN
// applied to the tokens sent to it; its output is multiplied by the routing
// weight.)
//
// Warp roles (192 threads): warp 0 issues TMA loads, warp 1 owns TMEM and issues
// the MMAs, warps 2..5 run the epilogue (warp w reads TMEM lanes 32*(w%4)..+31).
// Shared memory: kStages x (A 128x64 + B 256x64) bf16 tiles in the 128-byte
// swizzle layout; TMEM: two 256-column fp32 accumulators so the epilogue of one
// tile overlaps the main loop of the next.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "device_status.cuh"
#include "sm100_ptx.cuh"

namespace moe {

constexpr int kBM = 128;           // rows (tokens) per tile
constexpr int kBN = 256;           // accumulator columns per tile
constexpr int kBK = 64;            // K per stage (one 128-byte swizzle row of bf16)
constexpr int kStages = 4;
constexpr int kGemmThreads = 192;
constexpr int kMaxSeg = 258;       // 256 experts + shared
constexpr uint32_t kTileABytes = kBM * kBK * 2;   // 16 KB
constexpr uint32_t kTileBBytes = kBN * kBK * 2;   // 32 KB
constexpr uint32_t kTmemCols = 512;               // 2 accumulators x 256 columns
// Epilogue staging: each epilogue warp bounces its 32 rows x 32 columns through
// shared memory so that global stores write whole lines.  Row pitch 36 floats
// (144 B) keeps both the row-per-lane writes and the line-per-8-lanes reads of
// 16-byte vectors free of extra bank conflicts.
constexpr int kStagePitchF = 36;
constexpr uint32_t kStageBytesPerWarp = 32 * kStagePitchF * 4;   // 4608 B
constexpr uint32_t kStageBytes = 4 * kStageBytesPerWarp;         // 18 KB
constexpr int kStagePitchH = 40;                                 // bf16 row pitch (80 B)
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded device waits: 2 s
// Partial row tiles with at most this many valid rows are computed transposed.
#ifndef MOE_SWAP_MAX_ROWS
#define MOE_SWAP_MAX_ROWS 112
#endif
constexpr int kSwapMaxRows = MOE_SWAP_MAX_ROWS;

// A segment with at least this many 128-row tiles is walked row tile by row tile
// (all column tiles of a row tile in a row), so its A rows are read from HBM
// once while the segment's weight tiles are reused from L2; smaller segments walk
// column tile by column tile (the row tiles of a column share its weight tile and
// the segment's A rows stay in L2).  At the V3 shape the shared expert's 16384
// token rows are 235 MB of A: walked column-major they would be re-read from HBM
// once per column tile.
#ifndef MOE_ROW_MAJOR_MIN_ROW_TILES
#define MOE_ROW_MAJOR_MIN_ROW_TILES 16
#endif
constexpr int kRowMajorMinRowTiles = MOE_ROW_MAJOR_MIN_ROW_TILES;

// Weight bytes of one band of column tiles that a row-major segment keeps in L2.
constexpr int64_t kRowMajorBandBytes = 32ll << 20;

// Column tiles per band: as many whole weight tiles (rows_b x K elements of
// elt_bytes) as fit kRowMajorBandBytes, at least one.
__host__ __device__ inline int row_major_band(int rows_b, int64_t K, int elt_bytes) {
    const int64_t per = static_cast<int64_t>(rows_b) * K * elt_bytes;
    const int64_t b = per > 0 ? kRowMajorBandBytes / per : 1;
    return b < 1 ? 1 : (b > (1 << 20) ? (1 << 20) : static_cast<int>(b));
}

enum { kSwiGLU = 0, kDown = 1, kLogits = 2 };

struct GemmParams {
    const int32_t* offsets;      // [E+1] routed row offsets
    int E;
    int T;                       // rows of the shared segment
    int has_shared;
    int n_tiles_routed, n_tiles_shared;   // output column tiles
    int kb_routed, kb_shared;             // K blocks of 64
    int n_valid_routed, n_valid_shared;   // valid output columns
    int b_rows_per_expert;                // rows of one expert in the routed B map
    void* out_routed;                     // row r of routed segment -> out_routed + r*ld
    int64_t ld_routed;                    // (bf16 elements for kSwiGLU, fp16 for kDown)
    void* out_shared;                     // row t of the shared segment
    int64_t ld_shared;
    uint8_t* scale_routed;                // kDown: block scale codes, [rows][scale_ld]
    uint8_t* scale_shared;
    int64_t scale_ld;
    const int32_t* perm_src;              // kDown: routed row -> slot
    const float* topk_w;                  // kDown: slot -> routing weight
    uint32_t idesc;                       // MMA instruction descriptor (M = 128, N)
    uint32_t b_tile_bytes;                // bytes one B tile load brings in
    int b_plane_rows;                     // kLogits: rows of one plane in the B map (E)
    int allow_swap;                       // compute partial row tiles transposed
    int64_t max_rows;                     // routed row space: segments must lie in [0, max_rows)
    int64_t n_slots;                      // kDown: entries of topk_w (perm_src values < n_slots)
    int expert_mod;                       // routed segment s uses expert s % expert_mod (0: s)
    int row_major_band;                   // column tiles per band of a row-major segment (>= 1)
};

struct TileInfo {
    int seg;        // 0 = shared (if present) else routed
    int routed;     // 1 if routed expert segment
    int expert;
    int m, n;       // tile coordinates inside the segment
    int rows;       // rows of the segment
    int row0;       // first row of the segment in the A / output row space
    int kb;         // K blocks
    int r;          // valid rows in this tile (1..128)
    int swap;       // 1: computed transposed (weights as the M operand, see below)
    int rpad;       // swap: token columns of the MMA, r rounded up to 16
    int row_major;  // tiles of this segment are walked row tile by row tile
};

struct GemmSmem {
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

// Block-scaled fp16: a block of 32 values whose largest magnitude has biased
// fp32 exponent E gets the code c = clamp(E, 15, 254); values are stored as
// fp16(v * 2^(141 - c)), which puts the block maximum in [2^14, 2^15), and read
// back as fp16 * 2^(c - 141).  Both factors are normal fp32 powers of two, so
// scaling is exact; NaN and Inf keep their class.
__device__ __forceinline__ uint32_t block_scale_code(uint32_t max_abs_bits) {
    return min(max(max_abs_bits >> 23, 15u), 254u);
}
__device__ __forceinline__ float block_encode_factor(uint32_t code) { return __uint_as_float((268u - code) << 23); }

// Wait until the phase with parity `parity` of `bar` has completed.  Gives up
// (returns false) when the CTA is aborting or after kWaitLimitNs.
__device__ __forceinline__ bool bounded_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                             unsigned code, uint64_t limit_ns = kWaitLimitNs) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    for (uint32_t n = 1;; ++n) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if ((n & 63u) == 0) {
            if (abort_flag && *abort_flag) return false;
            if (ptx::globaltimer_ns() - t0 > limit_ns) {
                record_error(code);
                if (abort_flag) *abort_flag = 1;
                return false;
            }
        }
    }
}

__device__ __forceinline__ TileInfo decode_tile(const GemmSmem& s, const GemmParams& p, int tile) {
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
    if (p.expert_mod > 0 && ti.expert >= p.expert_mod) ti.expert %= p.expert_mod;
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
    // A segment that fits in one partial row tile (decode-sized: a few tokens per
    // expert) is computed transposed: the two 128-row halves of the weight tile
    // become the M = 128 operand and the r token rows the N operand (N = r rounded
    // up to 16); the operand tiles in shared memory are the same as for a normal
    // tile.  The last partial tile of a larger segment stays a normal 128-row tile:
    // measured on B200, narrow-N MMAs are not proportionally cheaper, and while
    // the gate/up GEMM is tensor-bound transposing those tails made it slower.
    ti.swap = (p.allow_swap && ti.rows <= kSwapMaxRows) ? 1 : 0;
    ti.rpad = (ti.r + 15) & ~15;
    return ti;
}

// Self-test of the bounded wait: one thread waits on an mbarrier that nothing
// arrives on; after limit_ns it records `code` in the device error word and the
// kernel returns normally.
__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns, unsigned code) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        ptx::mbar_init(ptx::smem_u32(&bar), 1);
        ptx::fence_barrier_init();
        abort_flag = 0;
    }
    __syncthreads();
    if (threadIdx.x == 0) bounded_wait(ptx::smem_u32(&bar), 0, &abort_flag, code, limit_ns);
}

template <int kEpi>
__global__ void __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA_r, const __grid_constant__ CUtensorMap tmA_s,
                        const __grid_constant__ CUtensorMap tmB_r, const __grid_constant__ CUtensorMap tmB2_r,
                        const __grid_constant__ CUtensorMap tmB_s, const __grid_constant__ CUtensorMap tmB2_s,
                        const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    // Operand tiles need 1024-byte alignment for the 128-byte swizzle pattern.
    uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t* smemA = tiles;
    uint8_t* smemB = tiles + kStages * kTileABytes;
    uint8_t* stage_base = tiles + kStages * (kTileABytes + kTileBBytes);
    GemmSmem& S = *reinterpret_cast<GemmSmem*>(stage_base + kStageBytes);
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
                rows = checked_segment_rows(row0, p.offsets[e + 1] - row0, p.max_rows, 1);
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
            // Column-major segments: the A rows are re-read by every column tile,
            // so they are kept in L2 preferentially (weight tiles are shared by the
            // CTAs on the segment's row tiles at the same time: default policy).
            // Row-major segments: the weight tiles are re-read by every row tile,
            // so those are kept instead.
            const uint64_t pol_keep = ptx::policy_evict_last();
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued_mask = 0, issued_parity = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const TileInfo ti = decode_tile(S, p, tile);
                const CUtensorMap* mA = ti.routed ? &tmA_r : &tmA_s;
                const CUtensorMap* mB = ti.routed ? &tmB_r : &tmB_s;
                const CUtensorMap* mB2 = ti.routed ? &tmB2_r : &tmB2_s;
                const int a_row = ti.row0 + ti.m * kBM;
                const int b_base = ti.routed ? ti.expert * p.b_rows_per_expert : 0;
                for (int kb = 0; kb < ti.kb; ++kb) {
                    if (!bounded_wait(ptx::smem_u32(&S.empty[stage]), phase ^ 1u, abort_flag, 0x101u)) {
                        ok = false;
                        break;
                    }
                    const uint32_t full = ptx::smem_u32(&S.full[stage]);
                    ptx::mbar_arrive_expect_tx(full, kTileABytes + p.b_tile_bytes);
                    const uint32_t a_dst = ptx::smem_u32(smemA + stage * kTileABytes);
                    const uint32_t b_dst = ptx::smem_u32(smemB + stage * kTileBBytes);
                    if (kEpi == kLogits) {
                        // K block 3 * (x column block) + plane: the same x tile is loaded
                        // for the three planes in a row (L2 hits after the first).  The
                        // column tile index is the split of K: tile n covers K blocks
                        // n * kb .. (n + 1) * kb, kb a multiple of 3.
                        const int kbg = ti.n * ti.kb + kb;
                        const int plane = kbg % 3;
                        const int kcol = (kbg / 3) * kBK;
                        ptx::tma_load_2d(a_dst, mA, full, kcol, a_row, pol_keep);
                        ptx::tma_load_2d(b_dst, mB, full, kcol, plane * p.b_plane_rows);
                    } else {
                        const int b_row = b_base + ti.n * (kEpi == kSwiGLU ? kBN / 2 : kBN);
                        if (ti.row_major) {
                            ptx::tma_load_2d(a_dst, mA, full, kb * kBK, a_row);
                            ptx::tma_load_2d(b_dst, mB, full, kb * kBK, b_row, pol_keep);
                            if (kEpi == kSwiGLU)
                                ptx::tma_load_2d(b_dst + kTileBBytes / 2, mB2, full, kb * kBK, b_row, pol_keep);
                        } else {
                            ptx::tma_load_2d(a_dst, mA, full, kb * kBK, a_row, pol_keep);
                            ptx::tma_load_2d(b_dst, mB, full, kb * kBK, b_row);
                            if (kEpi == kSwiGLU) ptx::tma_load_2d(b_dst + kTileBBytes / 2, mB2, full, kb * kBK, b_row);
                        }
                    }
                    issued_mask |= 1u << stage;
                    issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) {
                // Let this CTA's copies in flight land before the CTA exits.
                for (int s = 0; s < kStages; ++s)
                    if (issued_mask & (1u << s))
                        bounded_wait(ptx::smem_u32(&S.full[s]), (issued_parity >> s) & 1u, nullptr, 0x102u);
            }
        }
    } else if (warp == 1) {
        // ================= MMA issuer =================
        if (lane == 0) {
            const uint32_t idesc = p.idesc;
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const TileInfo ti = decode_tile(S, p, tile);
                if (!bounded_wait(ptx::smem_u32(&S.tmem_empty[acc]), acc_phase ^ 1u, abort_flag, 0x201u)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBN);
                for (int kb = 0; kb < ti.kb; ++kb) {
                    if (!bounded_wait(ptx::smem_u32(&S.full[stage]), phase, abort_flag, 0x202u)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t a_addr = ptx::smem_u32(smemA + stage * kTileABytes);
                    const uint32_t b_addr = ptx::smem_u32(smemB + stage * kTileBBytes);
                    if (!ti.swap) {
#pragma unroll
                        for (int k = 0; k < kBK / 16; ++k) {
                            const uint64_t ad = ptx::sw128_kmajor_desc(a_addr + k * 32);
                            const uint64_t bd = ptx::sw128_kmajor_desc(b_addr + k * 32);
                            ptx::mma_bf16(d_tmem, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
                        }
                    } else {
                        // D0[i][j] = W[i] . A[j] for weight rows i of the first B half,
                        // D1 (128 columns further) for the second half.
                        const uint32_t idesc_t = ptx::idesc_bf16_f32(kBM, ti.rpad);
#pragma unroll
                        for (int k = 0; k < kBK / 16; ++k) {
                            const uint64_t xd = ptx::sw128_kmajor_desc(a_addr + k * 32);
                            const uint64_t w0 = ptx::sw128_kmajor_desc(b_addr + k * 32);
                            const uint64_t w1 = ptx::sw128_kmajor_desc(b_addr + kTileBBytes / 2 + k * 32);
                            const uint32_t accum = (kb | k) != 0 ? 1u : 0u;
                            ptx::mma_bf16(d_tmem, w0, xd, idesc_t, accum);
                            ptx::mma_bf16(d_tmem + kBN / 2, w1, xd, idesc_t, accum);
                        }
                    }
                    ptx::mma_commit(ptx::smem_u32(&S.empty[stage]));
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                ptx::mma_commit(ptx::smem_u32(&S.tmem_full[acc]));
                if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
            }
            // Every MMA issued by this thread is complete once mma_done flips.
            ptx::mma_commit(ptx::smem_u32(&S.mma_done));
            bounded_wait(ptx::smem_u32(&S.mma_done), 0, nullptr, 0x203u);
        }
    } else {
        // ================= epilogue (warps 2..5) =================
        const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            const TileInfo ti = decode_tile(S, p, tile);
            const bool got = bounded_wait(ptx::smem_u32(&S.tmem_full[acc]), acc_phase, abort_flag, 0x301u);
            __syncwarp();
            if (!__all_sync(0xffffffffu, got)) break;
            ptx::tc_fence_after();
            const int r_local = ti.m * kBM + quarter * 32 + lane;
            const bool row_ok = r_local < ti.rows;
            const int64_t grow = (int64_t)ti.row0 + r_local;
            const uint32_t taddr = tmem_base + static_cast<uint32_t>(acc * kBN) +
                                   (static_cast<uint32_t>(quarter * 32) << 16);
            uint8_t* stage = stage_base + (warp - 2) * kStageBytesPerWarp;
            const int r_warp0 = ti.m * kBM + quarter * 32;  // first row of this warp
            const int64_t tile_row0 = (int64_t)ti.row0 + ti.m * kBM;
            if (ti.swap && kEpi == kSwiGLU) {
                // Transposed tile: TMEM lane = output column i of this 128-column tile,
                // TMEM column j = token row j (gate at 0.., up at 128..).
                const int n_valid = ti.routed ? p.n_valid_routed : p.n_valid_shared;
                __nv_bfloat16* out_base = ti.routed ? static_cast<__nv_bfloat16*>(p.out_routed)
                                                    : static_cast<__nv_bfloat16*>(p.out_shared);
                const int64_t ld = ti.routed ? p.ld_routed : p.ld_shared;
                const int col = ti.n * (kBN / 2) + quarter * 32 + lane;
                const bool col_ok = col < n_valid;
#pragma unroll 1
                for (int c = 0; c * 32 < ti.r; ++c) {
                    __syncwarp();
                    uint32_t g[32], u[32];
                    ptx::tmem_ld_32x32b_x32(taddr + c * 32, g);
                    ptx::tmem_ld_32x32b_x32(taddr + kBN / 2 + c * 32, u);
                    ptx::tmem_wait_ld();
                    const int jmax = min(32, ti.r - c * 32);
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        if (jj < jmax && col_ok) {
                            const float gv = __uint_as_float(g[jj]), uv = __uint_as_float(u[jj]);
                            out_base[(tile_row0 + c * 32 + jj) * ld + col] =
                                __float2bfloat16_rn(gv / (1.0f + __expf(-gv)) * uv);
                        }
                    }
                }
            } else if (ti.swap && kEpi == kDown) {
                // Transposed tile: TMEM lane = output column, column j = token row j;
                // the second 128 output columns sit 128 TMEM columns further.  The 32
                // lanes of a warp hold exactly one 32-column scale block of a row.
                const int n_valid = ti.routed ? p.n_valid_routed : p.n_valid_shared;
                __half* out_base = ti.routed ? static_cast<__half*>(p.out_routed) : static_cast<__half*>(p.out_shared);
                uint8_t* sc_base = ti.routed ? p.scale_routed : p.scale_shared;
                const int64_t ld = ti.routed ? p.ld_routed : p.ld_shared;
#pragma unroll 1
                for (int c = 0; c * 32 < ti.r; ++c) {
                    // Routing weight of token row c*32 + lane, shared across the warp below.
                    float wl = 1.0f;
                    if (ti.routed && c * 32 + lane < ti.r)
                        wl = row_weight(p.perm_src, p.topk_w, tile_row0 + c * 32 + lane, p.n_slots);
                    const int jmax = min(32, ti.r - c * 32);
#pragma unroll 1
                    for (int hh = 0; hh < 2; ++hh) {
                        const int col0 = ti.n * kBN + hh * (kBN / 2) + quarter * 32;  // block start
                        const bool blk_ok = col0 < n_valid;                            // warp-uniform
                        __syncwarp();
                        uint32_t v[32];
                        ptx::tmem_ld_32x32b_x32(taddr + hh * (kBN / 2) + c * 32, v);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) {
                            const float val = __uint_as_float(v[jj]) * __shfl_sync(0xffffffffu, wl, jj);
                            const uint32_t mx = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(val)));
                            if (jj < jmax && blk_ok) {
                                const uint32_t code = block_scale_code(mx);
                                const int64_t row = tile_row0 + c * 32 + jj;
                                out_base[row * ld + col0 + lane] = __float2half_rn(val * block_encode_factor(code));
                                if (lane == 0) sc_base[row * p.scale_ld + col0 / 32] = static_cast<uint8_t>(code);
                            }
                        }
                    }
                }
            } else if (kEpi == kSwiGLU) {
                const int n_valid = ti.routed ? p.n_valid_routed : p.n_valid_shared;
                __nv_bfloat16* out_base = ti.routed ? static_cast<__nv_bfloat16*>(p.out_routed)
                                                    : static_cast<__nv_bfloat16*>(p.out_shared);
                const int64_t ld = ti.routed ? p.ld_routed : p.ld_shared;
                __nv_bfloat16* hs = reinterpret_cast<__nv_bfloat16*>(stage);
#pragma unroll 1
                for (int c = 0; c < (kBN / 2) / 32; ++c) {
                    __syncwarp();
                    uint32_t g[32], u[32];
                    ptx::tmem_ld_32x32b_x32(taddr + c * 32, g);
                    ptx::tmem_ld_32x32b_x32(taddr + kBN / 2 + c * 32, u);
                    ptx::tmem_wait_ld();
                    const int col = ti.n * (kBN / 2) + c * 32;
                    if (col >= n_valid) continue;  // uniform across the warp
                    // h = silu(g) * u for this lane's row, 32 columns -> staging row `lane`.
                    uint4 pk[4];
                    __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(pk);
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const float g0 = __uint_as_float(g[2 * q]), g1 = __uint_as_float(g[2 * q + 1]);
                        const float u0 = __uint_as_float(u[2 * q]), u1 = __uint_as_float(u[2 * q + 1]);
                        const float h0 = g0 / (1.0f + __expf(-g0)) * u0;
                        const float h1 = g1 / (1.0f + __expf(-g1)) * u1;
                        h2[q] = __floats2bfloat162_rn(h0, h1);
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        *reinterpret_cast<uint4*>(hs + lane * kStagePitchH + 8 * q) = pk[q];
                    __syncwarp();
                    // 8 rows x 64 B per instruction: lanes 4r..4r+3 write row r's 32 values.
#pragma unroll
                    for (int it = 0; it < 4; ++it) {
                        const int rw = it * 8 + (lane >> 2);
                        const int r_local = r_warp0 + rw;
                        const uint4 v = *reinterpret_cast<const uint4*>(hs + rw * kStagePitchH + 8 * (lane & 3));
                        if (r_local < ti.rows)
                            *reinterpret_cast<uint4*>(out_base + ((int64_t)ti.row0 + r_local) * ld + col +
                                                      8 * (lane & 3)) = v;
                    }
                }
            } else if (kEpi == kDown) {
                const int n_valid = ti.routed ? p.n_valid_routed : p.n_valid_shared;
                __half* out_base = ti.routed ? static_cast<__half*>(p.out_routed) : static_cast<__half*>(p.out_shared);
                uint8_t* sc_base = ti.routed ? p.scale_routed : p.scale_shared;
                const int64_t ld = ti.routed ? p.ld_routed : p.ld_shared;
                __half* hs = reinterpret_cast<__half*>(stage);
                float wrow = 1.0f;
                if (ti.routed && row_ok) wrow = row_weight(p.perm_src, p.topk_w, grow, p.n_slots);
                uint32_t codes[kBN / 32];
#pragma unroll
                for (int c = 0; c < kBN / 32; ++c) {
                    __syncwarp();
                    uint32_t v[32];
                    ptx::tmem_ld_32x32b_x32(taddr + c * 32, v);
                    ptx::tmem_wait_ld();
                    const int col = ti.n * kBN + c * 32;
                    codes[c] = 0;
                    if (col >= n_valid) continue;  // uniform across the warp
                    // This lane's row, one 32-column block: scale from the block maximum.
                    uint32_t mx = 0;
#pragma unroll
                    for (int q = 0; q < 32; ++q) mx = max(mx, __float_as_uint(fabsf(__uint_as_float(v[q]) * wrow)));
                    const uint32_t code = block_scale_code(mx);
                    const float f = block_encode_factor(code);
                    codes[c] = code;
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
                    // 8 rows x 64 B per instruction: lanes 4r..4r+3 write row r's 32 values.
#pragma unroll
                    for (int it = 0; it < 4; ++it) {
                        const int rw = it * 8 + (lane >> 2);
                        const int r_local = r_warp0 + rw;
                        const uint4 val = *reinterpret_cast<const uint4*>(hs + rw * kStagePitchH + 8 * (lane & 3));
                        if (r_local < ti.rows)
                            *reinterpret_cast<uint4*>(out_base + ((int64_t)ti.row0 + r_local) * ld + col +
                                                      8 * (lane & 3)) = val;
                    }
                }
                // The row's scale codes of this 256-column tile: one 8-byte store when whole.
                if (row_ok) {
                    uint8_t* dst = sc_base + grow * p.scale_ld + ti.n * (kBN / 32);
                    const int nblk = min(kBN / 32, (n_valid - ti.n * kBN) / 32);
                    if (nblk == kBN / 32) {
                        uint2 pk;
                        pk.x = codes[0] | (codes[1] << 8) | (codes[2] << 16) | (codes[3] << 24);
                        pk.y = codes[4] | (codes[5] << 8) | (codes[6] << 16) | (codes[7] << 24);
                        *reinterpret_cast<uint2*>(dst) = pk;
                    } else {
#pragma unroll
                        for (int c = 0; c < kBN / 32; ++c)
                            if (c < nblk) dst[c] = static_cast<uint8_t>(codes[c]);
                    }
                }
            } else {
                // Logits of K split n into plane n of the partial sums [splits, T, E].
                const int n_valid = p.n_valid_shared;  // E
                float* out = static_cast<float*>(p.out_shared) + ((int64_t)ti.n * p.T + grow) * p.ld_shared;
#pragma unroll 1
                for (int c = 0; c * 32 < n_valid; ++c) {
                    __syncwarp();
                    uint32_t v[32];
                    ptx::tmem_ld_32x32b_x32(taddr + c * 32, v);
                    ptx::tmem_wait_ld();
                    if (row_ok) {
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const int col = c * 32 + 4 * q;
                            if (col < n_valid)
                                *reinterpret_cast<float4*>(out + col) =
                                    make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                                __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
                        }
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(ptx::smem_u32(&S.tmem_empty[acc]));
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
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
