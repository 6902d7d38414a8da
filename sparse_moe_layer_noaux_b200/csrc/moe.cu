// libmoe: C ABI of the DeepSeekMoE layer forward on B200 (see include/moe.h).
// Host side: argument validation, workspace carving, TMA tensor maps, launches.
// All kernels of the library are in this translation unit.
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <initializer_list>
#include <mutex>
#include <vector>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/moe.h"
#include "balance.cuh"
#include "combine.cuh"
#include "dispatch.cuh"
#include "ep.cuh"
#include "grouped_gemm.cuh"
#include "grouped_gemm_mx.cuh"
#include "grouped_gemm_bwd.cuh"
#include "bwd_small.cuh"
#include "mx.cuh"
#include "router.cuh"

namespace moe {
namespace {

std::atomic<uint64_t> g_launches{0};

inline void count_launch(int n = 1) { g_launches.fetch_add(static_cast<uint64_t>(n)); }

constexpr size_t kAlign = 256;
inline size_t align_up(size_t v, size_t a = kAlign) { return (v + a - 1) / a * a; }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Row pitch in bytes of the y_perm scale codes: one per 32 columns, padded to 8.
inline int64_t scale_ld(int64_t H) { return (H / 32 + 7) / 8 * 8; }

// --------------------------------------------------------------- validation
int validate_cfg(const moe_config* c, int64_t T) {
    if (!c || T < 0) return MOE_ERR_INVALID_ARG;
    const int H = c->hidden_size, E = c->n_routed_experts, K = c->num_experts_per_tok;
    const int G = c->n_group, TG = c->topk_group, I = c->moe_intermediate_size;
    if (H <= 0 || E <= 0 || G <= 0 || I <= 0 || c->n_shared_experts < 0) return MOE_ERR_INVALID_ARG;
    if (E % G != 0 || TG < 1 || TG > G || K < 1 || K > TG * (E / G)) return MOE_ERR_INVALID_ARG;
    if (c->norm_topk_prob != 0 && c->norm_topk_prob != 1) return MOE_ERR_INVALID_ARG;
    if (!(c->routed_scaling_factor == c->routed_scaling_factor)) return MOE_ERR_INVALID_ARG;
    if (H % 64 != 0 || I % 64 != 0) return MOE_ERR_UNSUPPORTED;
    if (E > 256 || G > 32 || K > 32) return MOE_ERR_UNSUPPORTED;
    const int64_t SI = static_cast<int64_t>(c->n_shared_experts) * I;
    if (SI > (1 << 24) || static_cast<int64_t>(E) * I > (1ll << 31) ||
        static_cast<int64_t>(E) * H > (1ll << 31))
        return MOE_ERR_UNSUPPORTED;
    // Every row index (routed rows with up to 127 padding rows per expert
    // segment, then the shared rows) must fit an int32 and a TMA coordinate.
    if (T * K + T + 128ll * E >= (1ll << 31) - 256) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

// --------------------------------------------------------------- router sizing
struct RouterPlan {
    int nsplit, split_len;
};

// The split count depends only on the shape (not on the device), so the
// workspace size computed before launch always matches what the launch uses.
constexpr int kRouterTargetBlocks = 296;  // two waves of blocks on 148 SMs

// Token counts from which the logits run on the tensor cores (below it, the
// CUDA-core kernel with a split hidden axis fills the GPU better).
constexpr int kRouterTensorCoreMinT = 2048;

RouterPlan plan_router(int T, int E, int H) {
    if (T <= 0) return RouterPlan{1, H};
    if (T >= kRouterTensorCoreMinT) {
        // Tensor-core logits: one tile per 128 rows, K (three planes of H) split in
        // s parts so that the row tiles times s fill up to 148 CTAs (s a power of
        // two dividing the H / 64 K blocks of a plane); the select kernel adds the
        // s partial sums.
        const int row_tiles = (T + kBM - 1) / kBM;
        int s = 1;
        while (row_tiles * s * 2 <= 148 && (H / kBK) % (s * 2) == 0) s *= 2;
        return RouterPlan{s, H};
    }
    const int tiles = ((T + kRT - 1) / kRT) * ((E + kRE - 1) / kRE);
    int want = (kRouterTargetBlocks + tiles - 1) / tiles;
    const int max_split = H / 256 > 0 ? H / 256 : 1;
    if (want > max_split) want = max_split;
    if (want < 1) want = 1;
    int split_len = (H + want - 1) / want;
    split_len = (split_len + kRK - 1) / kRK * kRK;
    RouterPlan r;
    r.split_len = split_len;
    r.nsplit = (H + split_len - 1) / split_len;
    return r;
}

constexpr size_t kGemmSmemBytes =
    1024 + kStages * (kTileABytes + kTileBBytes) + kStageBytes + sizeof(GemmSmem);
static_assert(kGemmSmemBytes <= 227 * 1024, "expert GEMM shared memory exceeds the 227 KB per-CTA limit");
static_assert(kGemmMxSmemBytes <= 227 * 1024, "MXFP8 GEMM shared memory exceeds the 227 KB per-CTA limit");
static_assert(kGemmBwdSmemBytes <= 227 * 1024, "backward GEMM shared memory exceeds the 227 KB per-CTA limit");

// --------------------------------------------------------------- device info
struct DeviceInfo {
    int num_sms = 0;
    bool attrs_set = false;
};
DeviceInfo g_dev[64];
std::mutex g_dev_mu;

int device_info(DeviceInfo** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceInfo& d = g_dev[dev];
    if (!d.attrs_set) {
        if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return MOE_ERR_CUDA;
        const int smem = static_cast<int>(kGemmSmemBytes);
        if (cudaFuncSetAttribute(grouped_gemm_kernel<kSwiGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 smem) != cudaSuccess ||
            cudaFuncSetAttribute(grouped_gemm_kernel<kDown>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 smem) != cudaSuccess ||
            cudaFuncSetAttribute(grouped_gemm_kernel<kLogits>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 smem) != cudaSuccess ||
            cudaFuncSetAttribute(grouped_gemm_mx_kernel<kSwiGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kGemmMxSmemBytes)) != cudaSuccess ||
            cudaFuncSetAttribute(grouped_gemm_mx_kernel<kDown>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kGemmMxSmemBytes)) != cudaSuccess ||
            cudaFuncSetAttribute(grouped_gemm_bwd_kernel<kRecompute>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kGemmBwdSmemBytes)) != cudaSuccess ||
            cudaFuncSetAttribute(grouped_gemm_bwd_kernel<kDh>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kGemmBwdSmemBytes)) != cudaSuccess ||
            cudaFuncSetAttribute(grouped_gemm_bwd_kernel<kDx>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kGemmBwdSmemBytes)) != cudaSuccess ||
            cudaFuncSetAttribute(grouped_gemm_bwd_kernel<kWgrad>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kGemmBwdSmemBytes)) != cudaSuccess ||
            cudaFuncSetAttribute(grouped_gemm_bwd_kernel<kFwdDown>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kGemmBwdSmemBytes)) != cudaSuccess)
            return MOE_ERR_CUDA;
        d.attrs_set = true;
    }
    *out = &d;
    return MOE_OK;
}

// --------------------------------------------------------------- workspace
struct Workspace {
    __nv_bfloat16* router_w3; // [3, E, H] exact bf16 split of router_w
    float* router_part;       // [nsplit, T, E]
    int32_t* block_counts;    // [E, nb]
    int32_t* block_base;      // [E, nb]
    int32_t* totals;          // [E]
    int32_t* topk_idx;        // [T, k]
    float* topk_w;            // [T, k]
    int32_t* offsets;         // [E + 1]
    int32_t* perm_src;        // [T*k]
    int32_t* row_of;          // [T, k]
    __nv_bfloat16* x_perm;    // [T*k, H]
    __nv_bfloat16* h_routed;  // [T*k, I]
    __nv_bfloat16* h_shared;  // [T, S*I]
    __half* y_perm;           // [T*k + T, H] block-scaled fp16 values
    uint8_t* y_scale;         // [T*k + T, scale_ld] block scale codes
    size_t bytes;
};

Workspace carve(const moe_config* c, int64_t T, uint8_t* base) {
    const int64_t H = c->hidden_size, E = c->n_routed_experts, K = c->num_experts_per_tok;
    const int64_t I = c->moe_intermediate_size, SI = static_cast<int64_t>(c->n_shared_experts) * I;
    const RouterPlan rp = plan_router(static_cast<int>(T), static_cast<int>(E), static_cast<int>(H));
    const int64_t nb = (T + kDispTok - 1) / kDispTok;
    Workspace w{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        uint8_t* p = base ? base + off : nullptr;
        off += align_up(bytes);
        return p;
    };
    w.router_w3 = reinterpret_cast<__nv_bfloat16*>(take(2 * 3 * E * H));
    w.router_part = reinterpret_cast<float*>(take(sizeof(float) * rp.nsplit * T * E));
    w.block_counts = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * nb * E));
    w.block_base = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * nb * E));
    w.totals = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * E));
    w.topk_idx = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * T * K));
    w.topk_w = reinterpret_cast<float*>(take(sizeof(float) * T * K));
    w.offsets = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (E + 1)));
    w.perm_src = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * T * K));
    w.row_of = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * T * K));
    w.x_perm = reinterpret_cast<__nv_bfloat16*>(take(2 * T * K * H));
    w.h_routed = reinterpret_cast<__nv_bfloat16*>(take(2 * T * K * I));
    w.h_shared = reinterpret_cast<__nv_bfloat16*>(take(2 * T * SI));
    w.y_perm = reinterpret_cast<__half*>(take(2 * (T * K + T) * H));
    w.y_scale = reinterpret_cast<uint8_t*>(take((T * K + T) * scale_ld(H)));
    w.bytes = off;
    return w;
}

size_t workspace_bytes_for(const moe_config* c, int64_t T) { return carve(c, T, nullptr).bytes; }

// --------------------------------------------------------------- TMA maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Row-major bf16 matrix [rows, cols]; box = box_rows x 64 columns, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    if (rows == 0) rows = 1;  // never addressed: the segment has no tiles
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// --------------------------------------------------------------- stages

// Router logits (fp32, [nsplit, T, E] partial sums) into `part`.
int launch_route_logits(const moe_config* c, int64_t T, const void* x, const float* wr, float* part,
                        __nv_bfloat16* w3, int num_sms, cudaStream_t st) {
    const int H = c->hidden_size, E = c->n_routed_experts;
    const RouterPlan rp = plan_router(static_cast<int>(T), E, H);
    if (T >= kRouterTensorCoreMinT) {
        // Logits on the tensor cores: exact 3-term bf16 split of Wr, one GEMM, K = 3 H.
        const int64_t n = static_cast<int64_t>(E) * H;
        router_split_kernel<<<static_cast<unsigned>((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096), 256, 0,
                              st>>>(wr, w3, n);
        const int npad = (E + 15) / 16 * 16;
        CUtensorMap a, b;
        if (!make_map(&a, x, T, H, kBM) || !make_map(&b, w3, 3ull * E, H, npad)) return MOE_ERR_CUDA;
        GemmParams p{};
        p.E = 0;
        p.T = static_cast<int>(T);
        p.has_shared = 1;
        p.n_tiles_shared = rp.nsplit;  // column tiles = splits of K
        p.kb_shared = 3 * (H / kBK) / rp.nsplit;
        p.n_valid_shared = E;
        p.out_shared = part;
        p.ld_shared = E;
        p.idesc = ptx::idesc_bf16_f32(kBM, npad);
        p.b_tile_bytes = static_cast<uint32_t>(npad) * kBK * 2;
        p.b_plane_rows = E;
        int64_t grid = (T + kBM - 1) / kBM * rp.nsplit;
        if (grid > num_sms) grid = num_sms;
        grouped_gemm_kernel<kLogits><<<static_cast<unsigned>(grid), kGemmThreads, kGemmSmemBytes, st>>>(
            a, a, b, b, b, b, p);
        count_launch(2);
    } else {
        dim3 g1((E + kRE - 1) / kRE, static_cast<unsigned>((T + kRT - 1) / kRT), rp.nsplit);
        router_logits_kernel<<<g1, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), wr, part,
                                                  static_cast<int>(T), E, H, rp.split_len);
        count_launch();
    }
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Scores, group limit, top-k and weights from the logits in `part`.
int launch_route_select(const moe_config* c, int64_t T, const float* bias, int32_t* idx, float* w,
                        const float* part, cudaStream_t st) {
    const int H = c->hidden_size, E = c->n_routed_experts;
    const RouterPlan rp = plan_router(static_cast<int>(T), E, H);
    RouteArgs a;
    a.part = part;
    a.nsplit = rp.nsplit;
    a.T = static_cast<int>(T);
    a.E = E;
    a.G = c->n_group;
    a.TG = c->topk_group;
    a.K = c->num_experts_per_tok;
    a.norm = c->norm_topk_prob;
    a.scale = c->routed_scaling_factor;
    a.bias = bias;
    a.topk_idx = idx;
    a.topk_w = w;
    const unsigned g2 = static_cast<unsigned>((T + 7) / 8);
    if (E <= 32) router_select_kernel<1><<<g2, 256, 0, st>>>(a);
    else if (E <= 64) router_select_kernel<2><<<g2, 256, 0, st>>>(a);
    else if (E <= 128) router_select_kernel<4><<<g2, 256, 0, st>>>(a);
    else router_select_kernel<8><<<g2, 256, 0, st>>>(a);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int launch_route(const moe_config* c, int64_t T, const void* x, const float* wr, const float* bias,
                 int32_t* idx, float* w, float* part, __nv_bfloat16* w3, int num_sms, cudaStream_t st) {
    const int v = launch_route_logits(c, T, x, wr, part, w3, num_sms, st);
    return v != MOE_OK ? v : launch_route_select(c, T, bias, idx, w, part, st);
}

// Rows of T tokens (K slots each, E buckets) sorted into bucket order: offsets
// [E + 1], perm_src, row_of and the bf16 rows (row strides x_ld / out_ld, in
// elements); with w_src / w_perm also each row's weight.
struct RowSort {
    SlotIndex si;
    int64_t T;
    int K, E, H;
    const void* x;
    int64_t x_ld;
    void* x_perm;
    int64_t out_ld;
    int32_t *offsets, *perm_src, *row_of;
    int32_t *block_counts, *block_base, *totals;
    const float* w_src;
    float* w_perm;
};

int launch_row_sort(const RowSort& a, cudaStream_t st) {
    const int E = a.E, K = a.K;
    const int nb = static_cast<int>((a.T + kDispTok - 1) / kDispTok);
    dispatch_count_kernel<<<nb, kDispThreads, sizeof(int) * E, st>>>(a.si, static_cast<int>(a.T), K, E,
                                                                      a.block_counts);
    dispatch_scan_kernel<<<(E + 7) / 8, 256, 0, st>>>(a.block_counts, nb, E, a.block_base, a.totals);
    dispatch_place_kernel<<<nb, kDispThreads, sizeof(int) * E, st>>>(a.si, static_cast<int>(a.T), K, E,
                                                                     a.block_base, a.totals, 1, a.offsets,
                                                                     a.perm_src, a.row_of, a.w_src, a.w_perm);
    const dim3 gs(static_cast<unsigned>(a.T), static_cast<unsigned>((a.H / 8 + 255) / 256));
    dispatch_scatter_kernel<<<gs, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(a.x), a.row_of, K, a.H,
                                                static_cast<__nv_bfloat16*>(a.x_perm), a.x_ld, a.out_ld);
    count_launch(4);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int launch_dispatch(const moe_config* c, int64_t T, const void* x, const int32_t* idx, int32_t* offsets,
                    void* x_perm, int32_t* perm_src, int32_t* row_of, int32_t* block_counts,
                    int32_t* block_base, int32_t* totals, cudaStream_t st) {
    const int E = c->n_routed_experts, K = c->num_experts_per_tok, H = c->hidden_size;
    RowSort a{};
    a.si = SlotIndex{idx, K, 0, 0, E};
    a.T = T;
    a.K = K;
    a.E = E;
    a.H = H;
    a.x = x;
    a.x_ld = H;
    a.x_perm = x_perm;
    a.out_ld = H;
    a.offsets = offsets;
    a.perm_src = perm_src;
    a.row_of = row_of;
    a.block_counts = block_counts;
    a.block_base = block_base;
    a.totals = totals;
    return launch_row_sort(a, st);
}

// Persistent grid: one CTA per SM, fewer when there cannot be that many tiles.
int64_t gemm_grid(int64_t T, int64_t R, int64_t E, int64_t n_cols_max, int has_shared, int num_sms,
                  int col_tile) {
    const int64_t m_tiles_bound = (R + kBM - 1) / kBM + E + (has_shared ? (T + kBM - 1) / kBM : 0);
    const int64_t n_tiles_bound = (n_cols_max + col_tile - 1) / col_tile;
    int64_t grid = m_tiles_bound * n_tiles_bound;
    if (grid > num_sms) grid = num_sms;
    if (grid < 1) grid = 1;
    return grid;
}

// Routed rows of the expert GEMMs: R rows (a bound: the segments may end earlier)
// in nseg consecutive segments, segment s = rows offsets[s] .. offsets[s+1],
// computed with expert s % n_local of the weight tensors (n_local = nseg: the
// layer's E experts on one GPU, or a rank's local experts under expert
// parallelism).
struct RoutedRows {
    int64_t R;
    int nseg;
    int n_local;
    const int32_t* offsets;
};

RoutedRows routed_rows_of(const moe_config* c, int64_t T, const int32_t* offsets) {
    return RoutedRows{T * c->num_experts_per_tok, c->n_routed_experts, c->n_routed_experts, offsets};
}

// K4: h = silu(A Wg^T) * (A Wu^T) for routed rows (A = x_perm) and shared rows (A = x).
int launch_gate_up(const moe_config* c, int64_t T, const void* x, const void* x_perm, const RoutedRows& rr,
                   const void* w_gate, const void* w_up, const void* ws_gate, const void* ws_up,
                   void* h_routed, void* h_shared, int num_sms, cudaStream_t st) {
    const int64_t H = c->hidden_size;
    const int64_t I = c->moe_intermediate_size, SI = static_cast<int64_t>(c->n_shared_experts) * I;
    const int64_t R = rr.R;
    const int has_shared = SI > 0 ? 1 : 0;
    CUtensorMap a_r, a_s, b_r, b2_r, b_s, b2_s;
    bool ok = make_map(&a_r, x_perm, R, H, kBM) && make_map(&b_r, w_gate, rr.n_local * I, H, kBN / 2) &&
              make_map(&b2_r, w_up, rr.n_local * I, H, kBN / 2);
    if (has_shared)
        ok = ok && make_map(&a_s, x, T, H, kBM) && make_map(&b_s, ws_gate, SI, H, kBN / 2) &&
             make_map(&b2_s, ws_up, SI, H, kBN / 2);
    else {
        a_s = a_r; b_s = b_r; b2_s = b2_r;
    }
    if (!ok) return MOE_ERR_CUDA;
    GemmParams p{};
    p.offsets = rr.offsets;
    p.E = rr.nseg;
    p.expert_mod = rr.n_local;
    p.T = static_cast<int>(T);
    p.has_shared = has_shared;
    p.n_tiles_routed = static_cast<int>((I + kBN / 2 - 1) / (kBN / 2));
    p.n_tiles_shared = static_cast<int>((SI + kBN / 2 - 1) / (kBN / 2));
    p.kb_routed = static_cast<int>(H / kBK);
    p.kb_shared = static_cast<int>(H / kBK);
    p.n_valid_routed = static_cast<int>(I);
    p.n_valid_shared = static_cast<int>(SI);
    p.b_rows_per_expert = static_cast<int>(I);
    p.out_routed = static_cast<__nv_bfloat16*>(h_routed);
    p.ld_routed = I;
    p.out_shared = static_cast<__nv_bfloat16*>(h_shared);
    p.ld_shared = SI;
    p.idesc = ptx::idesc_bf16_f32(kBM, kBN);
    p.b_tile_bytes = kTileBBytes;
    p.allow_swap = 1;
    p.max_rows = R;
    p.row_major_band = row_major_band(kBN, H, 2);
    const int64_t grid = gemm_grid(T, R, rr.nseg, I > SI ? I : SI, has_shared, num_sms, kBN / 2);
    grouped_gemm_kernel<kSwiGLU><<<static_cast<unsigned>(grid), kGemmThreads, kGemmSmemBytes, st>>>(
        a_r, a_s, b_r, b2_r, b_s, b2_s, p);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Block-scaled fp16 output rows (values [rows, H] and one scale code per 32 columns).
struct ScaledRows {
    __half* values;
    uint8_t* scales;
};

// K5: routed row r -> w_r * (h_r Wd^T), w_r = topk_w[perm_src[r]] (topk_w[r] when
// perm_src is null); shared row t -> h_shared[t] Wsd^T.
int launch_down(const moe_config* c, int64_t T, const void* h_routed, const void* h_shared, const RoutedRows& rr,
                const int32_t* perm_src, const float* topk_w, int64_t n_slots, const void* w_down,
                const void* ws_down, ScaledRows y_routed, ScaledRows y_shared, int num_sms, cudaStream_t st) {
    const int64_t H = c->hidden_size;
    const int64_t I = c->moe_intermediate_size, SI = static_cast<int64_t>(c->n_shared_experts) * I;
    const int64_t R = rr.R;
    const int has_shared = SI > 0 ? 1 : 0;
    CUtensorMap a_r, a_s, b_r, b_s;
    bool ok = make_map(&a_r, h_routed, R, I, kBM) && make_map(&b_r, w_down, rr.n_local * H, I, kBN);
    if (has_shared)
        ok = ok && make_map(&a_s, h_shared, T, SI, kBM) && make_map(&b_s, ws_down, H, SI, kBN);
    else {
        a_s = a_r; b_s = b_r;
    }
    if (!ok) return MOE_ERR_CUDA;
    GemmParams p{};
    p.offsets = rr.offsets;
    p.E = rr.nseg;
    p.expert_mod = rr.n_local;
    p.T = static_cast<int>(T);
    p.has_shared = has_shared;
    p.n_tiles_routed = static_cast<int>((H + kBN - 1) / kBN);
    p.n_tiles_shared = static_cast<int>((H + kBN - 1) / kBN);
    p.kb_routed = static_cast<int>(I / kBK);
    p.kb_shared = static_cast<int>(SI / kBK);
    p.n_valid_routed = static_cast<int>(H);
    p.n_valid_shared = static_cast<int>(H);
    p.b_rows_per_expert = static_cast<int>(H);
    p.out_routed = y_routed.values;
    p.ld_routed = H;
    p.out_shared = y_shared.values;
    p.ld_shared = H;
    p.scale_ld = scale_ld(H);
    p.scale_routed = y_routed.scales;
    p.scale_shared = y_shared.scales;
    p.perm_src = perm_src;
    p.topk_w = topk_w;
    p.idesc = ptx::idesc_bf16_f32(kBM, kBN);
    p.b_tile_bytes = kTileBBytes;
    p.allow_swap = 1;
    p.max_rows = R;
    p.row_major_band = row_major_band(kBN, I, 2);
    p.n_slots = n_slots;
    const int64_t grid = gemm_grid(T, R, rr.nseg, H, has_shared, num_sms, kBN);
    grouped_gemm_kernel<kDown><<<static_cast<unsigned>(grid), kGemmThreads, kGemmSmemBytes, st>>>(
        a_r, a_s, b_r, b_r, b_s, b_s, p);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// y_perm [R + T, H] and its scale codes as the routed rows followed by the shared rows.
void split_y_perm(const moe_config* c, int64_t R, void* y_perm, void* y_scale, ScaledRows* routed,
                  ScaledRows* shared) {
    const int64_t H = c->hidden_size;
    routed->values = static_cast<__half*>(y_perm);
    routed->scales = static_cast<uint8_t*>(y_scale);
    shared->values = static_cast<__half*>(y_perm) + R * H;
    shared->scales = static_cast<uint8_t*>(y_scale) + R * scale_ld(H);
}

int launch_combine_rows(int64_t T, int K, int H, ScaledRowsIn routed, int64_t routed_rows, const int32_t* row_of,
                        int absent_ok, ScaledRowsIn shared, CombineDst dst, int kind, cudaStream_t st) {
    const dim3 g(static_cast<unsigned>(T), static_cast<unsigned>((H / 8 + 255) / 256));
    const int Ti = static_cast<int>(T);
    if (kind == kOutBF16)
        combine_kernel<kOutBF16><<<g, 256, 0, st>>>(routed, routed_rows, row_of, Ti, K, H, absent_ok, shared, dst);
    else if (kind == kOutScaled)
        combine_kernel<kOutScaled><<<g, 256, 0, st>>>(routed, routed_rows, row_of, Ti, K, H, absent_ok, shared, dst);
    else
        combine_kernel<kOutF32><<<g, 256, 0, st>>>(routed, routed_rows, row_of, Ti, K, H, absent_ok, shared, dst);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int launch_combine(const moe_config* c, int64_t T, const void* y_perm, const void* y_scale,
                   const int32_t* row_of, void* y, int y_dtype, cudaStream_t st, int64_t shared_row0 = -1) {
    if (shared_row0 < 0) shared_row0 = T * c->num_experts_per_tok;
    const int64_t H = c->hidden_size, sld = scale_ld(c->hidden_size);
    const __half* v = static_cast<const __half*>(y_perm);
    const uint8_t* sc = static_cast<const uint8_t*>(y_scale);
    const ScaledRowsIn routed{v, H, sc, sld};
    const ScaledRowsIn shared = c->n_shared_experts > 0 ? ScaledRowsIn{v + shared_row0 * H, H, sc + shared_row0 * sld, sld}
                                                        : ScaledRowsIn{nullptr, 0, nullptr, 0};
    CombineDst dst{};
    dst.y = y;
    return launch_combine_rows(T, c->num_experts_per_tok, c->hidden_size, routed, shared_row0, row_of, 0, shared, dst,
                               y_dtype == MOE_DTYPE_BF16 ? kOutBF16 : kOutF32, st);
}


// ---------------------------------------------------------------- MXFP8 path
// Shapes the MXFP8 expert GEMMs take: scale atoms cover 128 K-elements, and the
// down GEMM's 256-column tiles must not straddle two experts' weight rows.
int validate_mx(const moe_config* c, int64_t T) {
    const int v = validate_cfg(c, T);
    if (v != MOE_OK) return v;
    if (c->hidden_size % 256 != 0 || c->moe_intermediate_size % 128 != 0) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

inline int64_t round128(int64_t v) { return (v + 127) / 128 * 128; }
inline int64_t mx_scale_bytes(int64_t rows, int64_t K) { return round128(rows) / 128 * (K / 128) * kMxAtomBytes; }

// Rows of the padded routed row space: every expert segment starts on a multiple
// of 128, so the segments of T*k rows take at most T*k + 127*E rows.
inline int64_t mx_routed_rows(const moe_config* c, int64_t T) {
    return round128(T * c->num_experts_per_tok + 127ll * c->n_routed_experts);
}

struct WorkspaceMx {
    __nv_bfloat16* router_w3;
    float* router_part;
    int32_t* block_counts;
    int32_t* block_base;
    int32_t* totals;          // [E] rows routed to each expert
    int32_t* topk_idx;
    float* topk_w;
    int32_t* offsets;         // [E + 1] padded segment starts
    int32_t* perm_src;        // [Rp]
    int32_t* row_of;          // [T, k]
    uint8_t* xq_perm;         // [Rp, H] E4M3
    uint8_t* xq_perm_sf;      // scale atoms of xq_perm
    uint8_t* xq_shared;       // [Tp, H]
    uint8_t* xq_shared_sf;
    uint8_t* hq_routed;       // [Rp, I]
    uint8_t* hq_routed_sf;
    uint8_t* hq_shared;       // [Tp, S*I]
    uint8_t* hq_shared_sf;
    __half* y_perm;           // [Rp + T, H] block-scaled fp16
    uint8_t* y_scale;
    int64_t rp;
    size_t bytes;
};

WorkspaceMx carve_mx(const moe_config* c, int64_t T, uint8_t* base) {
    const int64_t H = c->hidden_size, E = c->n_routed_experts, K = c->num_experts_per_tok;
    const int64_t I = c->moe_intermediate_size, SI = static_cast<int64_t>(c->n_shared_experts) * I;
    const RouterPlan rp = plan_router(static_cast<int>(T), static_cast<int>(E), static_cast<int>(H));
    const int64_t nb = (T + kDispTok - 1) / kDispTok;
    const int64_t Rp = mx_routed_rows(c, T), Tp = round128(T);
    WorkspaceMx w{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        uint8_t* p = base ? base + off : nullptr;
        off += align_up(bytes);
        return p;
    };
    w.router_w3 = reinterpret_cast<__nv_bfloat16*>(take(2 * 3 * E * H));
    w.router_part = reinterpret_cast<float*>(take(sizeof(float) * rp.nsplit * T * E));
    w.block_counts = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * nb * E));
    w.block_base = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * nb * E));
    w.totals = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * E));
    w.topk_idx = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * T * K));
    w.topk_w = reinterpret_cast<float*>(take(sizeof(float) * T * K));
    w.offsets = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (E + 1)));
    w.perm_src = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * Rp));
    w.row_of = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * T * K));
    w.xq_perm = take(Rp * H);
    w.xq_perm_sf = take(mx_scale_bytes(Rp, H));
    w.xq_shared = take(SI > 0 ? Tp * H : 0);
    w.xq_shared_sf = take(SI > 0 ? mx_scale_bytes(Tp, H) : 0);
    w.hq_routed = take(Rp * I);
    w.hq_routed_sf = take(mx_scale_bytes(Rp, I));
    w.hq_shared = take(Tp * SI);
    w.hq_shared_sf = take(SI > 0 ? mx_scale_bytes(Tp, SI) : 0);
    w.y_perm = reinterpret_cast<__half*>(take(2 * (Rp + T) * H));
    w.y_scale = take((Rp + T) * scale_ld(H));
    w.rp = Rp;
    w.bytes = off;
    return w;
}

// Row-major E4M3 matrix [rows, cols] (cols a multiple of 128); box = box_rows x 128
// bytes, 128-byte swizzle.
bool make_map_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    if (rows == 0) rows = 1;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBKq), box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int launch_mx_quantize(int64_t rows, int64_t K, const void* src, void* q, void* sf, cudaStream_t st) {
    const dim3 g(static_cast<unsigned>(rows), static_cast<unsigned>((K / 8 + 255) / 256));
    mx_quantize_rows_kernel<<<g, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(src), static_cast<int>(K),
                                               static_cast<uint8_t*>(q), static_cast<uint8_t*>(sf));
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Dispatch with quantisation: counting sort with 128-row aligned segments, then
// each token row quantised once and written to its k rows (and the shared rows).
int launch_dispatch_mx(const moe_config* c, int64_t T, const void* x, const int32_t* idx, int32_t* offsets,
                       uint8_t* xq_perm, uint8_t* xq_perm_sf, uint8_t* xq_shared, uint8_t* xq_shared_sf,
                       int32_t* perm_src, int32_t* row_of, int32_t* block_counts, int32_t* block_base,
                       int32_t* totals, cudaStream_t st) {
    const int E = c->n_routed_experts, K = c->num_experts_per_tok, H = c->hidden_size;
    const int nb = static_cast<int>((T + kDispTok - 1) / kDispTok);
    const SlotIndex si{idx, K, 0, 0, E};
    dispatch_count_kernel<<<nb, kDispThreads, sizeof(int) * E, st>>>(si, static_cast<int>(T), K, E, block_counts);
    dispatch_scan_kernel<<<(E + 7) / 8, 256, 0, st>>>(block_counts, nb, E, block_base, totals);
    dispatch_place_kernel<<<nb, kDispThreads, sizeof(int) * E, st>>>(si, static_cast<int>(T), K, E, block_base,
                                                                     totals, kMxAtomRows, offsets, perm_src, row_of);
    const dim3 gs(static_cast<unsigned>(T), static_cast<unsigned>((H / 8 + 255) / 256));
    dispatch_scatter_mx_kernel<<<gs, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), row_of, K, H, xq_perm,
                                                   xq_perm_sf, c->n_shared_experts > 0 ? xq_shared : nullptr,
                                                   xq_shared_sf);
    count_launch(4);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int64_t gemm_grid_mx(int64_t T, int64_t Rp, int64_t n_tiles_max, int has_shared, int num_sms) {
    int64_t grid = (Rp / kBM + (has_shared ? (T + kBM - 1) / kBM : 0)) * n_tiles_max;
    if (grid > num_sms) grid = num_sms;
    if (grid < 1) grid = 1;
    return grid;
}

// Device buffers of the MXFP8 expert stage (from the workspace, or the caller's).
struct MxBuffers {
    const int32_t* offsets;
    const int32_t* counts;
    const uint8_t* xq_perm;
    const uint8_t* xq_perm_sf;
    const uint8_t* xq_shared;
    const uint8_t* xq_shared_sf;
    uint8_t* hq_routed;
    uint8_t* hq_routed_sf;
    uint8_t* hq_shared;
    uint8_t* hq_shared_sf;
    const int32_t* perm_src;
    __half* y_perm;
    uint8_t* y_scale;
    int64_t rp;
};

MxBuffers buffers_of(const WorkspaceMx& w) {
    return MxBuffers{w.offsets,   w.totals,       w.xq_perm,   w.xq_perm_sf,   w.xq_shared, w.xq_shared_sf,
                     w.hq_routed, w.hq_routed_sf, w.hq_shared, w.hq_shared_sf, w.perm_src,  w.y_perm,
                     w.y_scale,   w.rp};
}

int launch_gate_up_mx(const moe_config* c, int64_t T, const MxBuffers& w, const moe_mx_weights* wt,
                      int num_sms, cudaStream_t st) {
    const int64_t H = c->hidden_size, E = c->n_routed_experts;
    const int64_t I = c->moe_intermediate_size, SI = static_cast<int64_t>(c->n_shared_experts) * I;
    const int has_shared = SI > 0 ? 1 : 0;
    CUtensorMap a_r, a_s, b_r, b2_r, b_s, b2_s;
    bool ok = make_map_u8(&a_r, w.xq_perm, w.rp, H, kBM) && make_map_u8(&b_r, wt->gate.q, E * I, H, kBN / 2) &&
              make_map_u8(&b2_r, wt->up.q, E * I, H, kBN / 2);
    if (has_shared)
        ok = ok && make_map_u8(&a_s, w.xq_shared, round128(T), H, kBM) &&
             make_map_u8(&b_s, wt->shared_gate.q, SI, H, kBN / 2) && make_map_u8(&b2_s, wt->shared_up.q, SI, H, kBN / 2);
    else {
        a_s = a_r; b_s = b_r; b2_s = b2_r;
    }
    if (!ok) return MOE_ERR_CUDA;
    GemmParamsMx p{};
    p.offsets = w.offsets;
    p.counts = w.counts;
    p.E = static_cast<int>(E);
    p.T = static_cast<int>(T);
    p.has_shared = has_shared;
    p.n_tiles_routed = static_cast<int>(I / (kBN / 2));
    p.n_tiles_shared = static_cast<int>(SI / (kBN / 2));
    p.kb_routed = static_cast<int>(H / kBKq);
    p.kb_shared = static_cast<int>(H / kBKq);
    p.n_valid_routed = static_cast<int>(I);
    p.n_valid_shared = static_cast<int>(SI);
    p.b_rows_per_expert = static_cast<int>(I);
    p.sfa_routed = w.xq_perm_sf;
    p.sfa_shared = w.xq_shared_sf;
    p.sfb_routed = static_cast<const uint8_t*>(wt->gate.sf);
    p.sfb2_routed = static_cast<const uint8_t*>(wt->up.sf);
    p.sfb_shared = has_shared ? static_cast<const uint8_t*>(wt->shared_gate.sf) : p.sfb_routed;
    p.sfb2_shared = has_shared ? static_cast<const uint8_t*>(wt->shared_up.sf) : p.sfb2_routed;
    p.b_rows_routed = E * I;
    p.b_rows_shared = SI;
    p.out_routed = w.hq_routed;
    p.ld_routed = I;
    p.out_shared = w.hq_shared;
    p.ld_shared = SI;
    p.hsf_routed = w.hq_routed_sf;
    p.hsf_shared = w.hq_shared_sf;
    p.hsf_katoms_routed = static_cast<int>(I / kMxAtomK);
    p.hsf_katoms_shared = static_cast<int>(SI / kMxAtomK);
    p.max_rows = w.rp;
    p.row_major_band = row_major_band(kBN, H, 1);
    const int64_t grid = gemm_grid_mx(T, w.rp, I > SI ? I / (kBN / 2) : SI / (kBN / 2), has_shared, num_sms);
    grouped_gemm_mx_kernel<kSwiGLU><<<static_cast<unsigned>(grid), kGemmThreads, kGemmMxSmemBytes, st>>>(
        a_r, a_s, b_r, b2_r, b_s, b2_s, p);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int launch_down_mx(const moe_config* c, int64_t T, const MxBuffers& w, const moe_mx_weights* wt,
                   const float* topk_w, int num_sms, cudaStream_t st) {
    const int64_t H = c->hidden_size, E = c->n_routed_experts;
    const int64_t I = c->moe_intermediate_size, SI = static_cast<int64_t>(c->n_shared_experts) * I;
    const int has_shared = SI > 0 ? 1 : 0;
    CUtensorMap a_r, a_s, b_r, b_s;
    bool ok = make_map_u8(&a_r, w.hq_routed, w.rp, I, kBM) && make_map_u8(&b_r, wt->down.q, E * H, I, kBN);
    if (has_shared)
        ok = ok && make_map_u8(&a_s, w.hq_shared, round128(T), SI, kBM) &&
             make_map_u8(&b_s, wt->shared_down.q, H, SI, kBN);
    else {
        a_s = a_r; b_s = b_r;
    }
    if (!ok) return MOE_ERR_CUDA;
    GemmParamsMx p{};
    p.offsets = w.offsets;
    p.counts = w.counts;
    p.E = static_cast<int>(E);
    p.T = static_cast<int>(T);
    p.has_shared = has_shared;
    p.n_tiles_routed = static_cast<int>(H / kBN);
    p.n_tiles_shared = static_cast<int>(H / kBN);
    p.kb_routed = static_cast<int>(I / kBKq);
    p.kb_shared = static_cast<int>(SI / kBKq);
    p.n_valid_routed = static_cast<int>(H);
    p.n_valid_shared = static_cast<int>(H);
    p.b_rows_per_expert = static_cast<int>(H);
    p.sfa_routed = w.hq_routed_sf;
    p.sfa_shared = w.hq_shared_sf;
    p.sfb_routed = static_cast<const uint8_t*>(wt->down.sf);
    p.sfb2_routed = p.sfb_routed;
    p.sfb_shared = has_shared ? static_cast<const uint8_t*>(wt->shared_down.sf) : p.sfb_routed;
    p.sfb2_shared = p.sfb_shared;
    p.b_rows_routed = E * H;
    p.b_rows_shared = H;
    p.out_routed = w.y_perm;
    p.ld_routed = H;
    p.out_shared = w.y_perm + w.rp * H;
    p.ld_shared = H;
    p.scale_ld = scale_ld(H);
    p.scale_routed = w.y_scale;
    p.scale_shared = w.y_scale + w.rp * p.scale_ld;
    p.perm_src = w.perm_src;
    p.topk_w = topk_w;
    p.max_rows = w.rp;
    p.row_major_band = row_major_band(kBN, I, 1);
    p.n_slots = T * c->num_experts_per_tok;
    const int64_t grid = gemm_grid_mx(T, w.rp, H / kBN, has_shared, num_sms);
    grouped_gemm_mx_kernel<kDown><<<static_cast<unsigned>(grid), kGemmThreads, kGemmMxSmemBytes, st>>>(
        a_r, a_s, b_r, b_r, b_s, b_s, p);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}


// ---------------------------------------------------------------- backward pass
struct WorkspaceBwd {
    __nv_bfloat16* router_w3;
    float* router_part;
    int32_t* block_counts;
    int32_t* block_base;
    int32_t* totals;          // [E] rows per expert
    int32_t* topk_idx;
    float* topk_w;
    int32_t* offsets;         // [E+1] 128-aligned segment starts
    int32_t* perm_src;        // [Rp]
    int32_t* row_of;          // [T, k]
    __nv_bfloat16* x_perm;    // [Rp, H]
    __nv_bfloat16* do_perm;   // [Rp, H]  w * dy
    __nv_bfloat16* gu_r;      // [Rp, 2I]
    __nv_bfloat16* gu_s;      // [T, 2SI]
    __nv_bfloat16* dgu_r;     // [Rp, 2I]
    __nv_bfloat16* dgu_s;     // [T, 2SI]
    __nv_bfloat16* h_r;       // [Rp, I]
    __nv_bfloat16* h_s;       // [T, SI]
    float* dw_part;           // [Rp, 2 ceil(I/256)]
    float* dlogit;            // [T, k]
    float* dwr_part;          // [kRouterSplit, E, H]
    __half* dxq;              // [Rp + T, H] block-scaled fp16
    uint8_t* dxs;             // [Rp + T, scale_ld]
    int64_t rp;
    size_t bytes;
};

WorkspaceBwd carve_bwd(const moe_config* c, int64_t T, uint8_t* base) {
    const int64_t H = c->hidden_size, E = c->n_routed_experts, K = c->num_experts_per_tok;
    const int64_t I = c->moe_intermediate_size, SI = static_cast<int64_t>(c->n_shared_experts) * I;
    const RouterPlan rp = plan_router(static_cast<int>(T), static_cast<int>(E), static_cast<int>(H));
    const int64_t nb = (T + kDispTok - 1) / kDispTok;
    const int64_t Rp = mx_routed_rows(c, T);
    WorkspaceBwd w{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        uint8_t* p = base ? base + off : nullptr;
        off += align_up(bytes);
        return p;
    };
    w.router_w3 = reinterpret_cast<__nv_bfloat16*>(take(2 * 3 * E * H));
    w.router_part = reinterpret_cast<float*>(take(sizeof(float) * rp.nsplit * T * E));
    w.block_counts = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * nb * E));
    w.block_base = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * nb * E));
    w.totals = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * E));
    w.topk_idx = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * T * K));
    w.topk_w = reinterpret_cast<float*>(take(sizeof(float) * T * K));
    w.offsets = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (E + 1)));
    w.perm_src = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * Rp));
    w.row_of = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * T * K));
    w.x_perm = reinterpret_cast<__nv_bfloat16*>(take(2 * Rp * H));
    w.do_perm = reinterpret_cast<__nv_bfloat16*>(take(2 * Rp * H));
    w.gu_r = reinterpret_cast<__nv_bfloat16*>(take(2 * Rp * 2 * I));
    w.gu_s = reinterpret_cast<__nv_bfloat16*>(take(2 * T * 2 * SI));
    w.dgu_r = reinterpret_cast<__nv_bfloat16*>(take(2 * Rp * 2 * I));
    w.dgu_s = reinterpret_cast<__nv_bfloat16*>(take(2 * T * 2 * SI));
    w.h_r = reinterpret_cast<__nv_bfloat16*>(take(2 * Rp * I));
    w.h_s = reinterpret_cast<__nv_bfloat16*>(take(2 * T * SI));
    w.dw_part = reinterpret_cast<float*>(take(sizeof(float) * Rp * 2 * ((I + kBN - 1) / kBN)));
    w.dlogit = reinterpret_cast<float*>(take(sizeof(float) * T * K));
    w.dwr_part = reinterpret_cast<float*>(take(sizeof(float) * kRouterSplit * E * H));
    w.dxq = reinterpret_cast<__half*>(take(2 * (Rp + T) * H));
    w.dxs = take((Rp + T) * scale_ld(H));
    w.rp = Rp;
    w.bytes = off;
    return w;
}

struct BwdArgs {
    const void *x, *dy, *w_gate, *w_up, *w_down, *ws_gate, *ws_up, *ws_down;
    void *d_w_gate, *d_w_up, *d_w_down, *d_ws_gate, *d_ws_up, *d_ws_down;
};

template <int kMode>
int launch_bwd_gemm(const CUtensorMap& a_r, const CUtensorMap& a_s, const CUtensorMap& b_r, const CUtensorMap& b2_r,
                    const CUtensorMap& b_s, const CUtensorMap& b2_s, const BwdParams& p, int64_t tiles_bound,
                    int num_sms, cudaStream_t st) {
    int64_t grid = tiles_bound < num_sms ? tiles_bound : num_sms;
    if (grid < 1) grid = 1;
    grouped_gemm_bwd_kernel<kMode><<<static_cast<unsigned>(grid), kBwdThreads, kGemmBwdSmemBytes, st>>>(
        a_r, a_s, b_r, b2_r, b_s, b2_s, p);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Route, dispatch into 128-row aligned segments, x into the expert rows (and dO =
// w dy when dy is given), padding rows zeroed.
int bwd_front(const moe_config* c, int64_t T, const float* router_w, const float* e_bias, const void* x,
              const void* dy, const WorkspaceBwd& w, int num_sms, cudaStream_t st) {
    const int64_t H = c->hidden_size, E = c->n_routed_experts, K = c->num_experts_per_tok;
    int v;
    if ((v = launch_route(c, T, x, router_w, e_bias, w.topk_idx, w.topk_w, w.router_part, w.router_w3, num_sms,
                          st)) != MOE_OK)
        return v;
    const int nb = static_cast<int>((T + kDispTok - 1) / kDispTok);
    const SlotIndex si{w.topk_idx, static_cast<int>(K), 0, 0, static_cast<int>(E)};
    dispatch_count_kernel<<<nb, kDispThreads, sizeof(int) * E, st>>>(si, static_cast<int>(T), static_cast<int>(K),
                                                                      static_cast<int>(E), w.block_counts);
    dispatch_scan_kernel<<<static_cast<unsigned>((E + 7) / 8), 256, 0, st>>>(w.block_counts, nb, static_cast<int>(E),
                                                                            w.block_base, w.totals);
    dispatch_place_kernel<<<nb, kDispThreads, sizeof(int) * E, st>>>(
        si, static_cast<int>(T), static_cast<int>(K), static_cast<int>(E), w.block_base, w.totals,
        kMxAtomRows, w.offsets, w.perm_src, w.row_of);
    const dim3 gs(static_cast<unsigned>(T), static_cast<unsigned>((H / 8 + 255) / 256));
    bwd_scatter_kernel<<<gs, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(dy),
                                            w.row_of, w.topk_w, static_cast<int>(K), static_cast<int>(H), w.x_perm,
                                            dy ? w.do_perm : nullptr);
    bwd_zero_pad_kernel<<<dim3(static_cast<unsigned>(E), 8), 256, 0, st>>>(w.offsets, w.totals, static_cast<int>(H),
                                                                          w.x_perm, dy ? w.do_perm : w.x_perm);
    count_launch(5);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// g, u of every routed and shared row (the gate/up GEMM keeping both products),
// and h = silu(g) u as well when `with_h` (the training forward).
int bwd_recompute(const moe_config* c, int64_t T, const BwdArgs& a, const WorkspaceBwd& w, int num_sms,
                  cudaStream_t st, bool with_h = false) {
    const int64_t H = c->hidden_size, E = c->n_routed_experts;
    const int64_t I = c->moe_intermediate_size, SI = static_cast<int64_t>(c->n_shared_experts) * I;
    const int has_shared = SI > 0 ? 1 : 0;
    const int64_t Rp = w.rp;
    CUtensorMap ar, as, br, b2r, bs, b2s;
    bool ok = make_map(&ar, w.x_perm, Rp, H, kBM) && make_map(&br, a.w_gate, E * I, H, kBN / 2) &&
              make_map(&b2r, a.w_up, E * I, H, kBN / 2);
    if (has_shared)
        ok = ok && make_map(&as, a.x, T, H, kBM) && make_map(&bs, a.ws_gate, SI, H, kBN / 2) &&
             make_map(&b2s, a.ws_up, SI, H, kBN / 2);
    else { as = ar; bs = br; b2s = b2r; }
    if (!ok) return MOE_ERR_CUDA;
    BwdParams p{};
    p.offsets = w.offsets; p.counts = w.totals; p.E = static_cast<int>(E); p.T = static_cast<int>(T);
    p.has_shared = has_shared;
    p.n_tiles_routed = static_cast<int>(I / (kBN / 2)); p.n_tiles_shared = static_cast<int>(SI / (kBN / 2));
    p.kb_routed = p.kb_shared = static_cast<int>(H / kBK);
    p.b_rows_per_expert = static_cast<int>(I);
    p.out_routed = w.gu_r; p.ld_routed = 2 * I; p.out_shared = w.gu_s; p.ld_shared = 2 * SI;
    if (with_h) {
        p.out2_routed = w.h_r; p.ld2_routed = I; p.out2_shared = w.h_s; p.ld2_shared = SI;
    }
    p.half_routed = static_cast<int>(I); p.half_shared = static_cast<int>(SI);
    p.idesc = idesc_bf16_f32_major(kBM, kBN, 0, 0);
    const int64_t m_bound = Rp / kBM + (has_shared ? (T + kBM - 1) / kBM : 0);
    return launch_bwd_gemm<kRecompute>(ar, as, br, b2r, bs, b2s, p, m_bound * (I / (kBN / 2)), num_sms, st);
}

int launch_backward(const moe_config* c, int64_t T, const float* router_w, const float* e_bias, const BwdArgs& a,
                    float* dx, float* d_router_w, const WorkspaceBwd& w, int num_sms, cudaStream_t st,
                    bool front_done = false) {
    const int64_t H = c->hidden_size, E = c->n_routed_experts, K = c->num_experts_per_tok;
    const int64_t I = c->moe_intermediate_size, SI = static_cast<int64_t>(c->n_shared_experts) * I;
    const int has_shared = SI > 0 ? 1 : 0;
    const int64_t Rp = w.rp;
    const int nti = static_cast<int>((I + kBN - 1) / kBN), nts = static_cast<int>((SI + kBN - 1) / kBN);
    int v;
    const int64_t m_bound = Rp / kBM + (has_shared ? (T + kBM - 1) / kBM : 0);
    const dim3 gs(static_cast<unsigned>(T), static_cast<unsigned>((H / 8 + 255) / 256));
    if (!front_done) {
        // 1-3. routing and dispatch recomputed (the same kernels and inputs as the
        // forward: the same selection), g and u recomputed
        if ((v = bwd_front(c, T, router_w, e_bias, a.x, a.dy, w, num_sms, st)) != MOE_OK) return v;
        if ((v = bwd_recompute(c, T, a, w, num_sms, st)) != MOE_OK) return v;
    } else {
        // Routing, rows and g | u kept by the training forward: only dO = w dy.
        bwd_scatter_kernel<<<gs, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(a.x),
                                                static_cast<const __nv_bfloat16*>(a.dy), w.row_of, w.topk_w,
                                                static_cast<int>(K), static_cast<int>(H), nullptr, w.do_perm);
        bwd_zero_pad_kernel<<<dim3(static_cast<unsigned>(E), 8), 256, 0, st>>>(w.offsets, w.totals,
                                                                              static_cast<int>(H), w.do_perm,
                                                                              w.do_perm);
        count_launch(2);
        if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
    }
    // 4. dh = dO Wd with the SwiGLU backward
    {
        CUtensorMap ar, as, br, bs;
        bool ok = make_map(&ar, w.do_perm, Rp, H, kBM) && make_map(&br, a.w_down, E * H, I, 64);
        if (has_shared) ok = ok && make_map(&as, a.dy, T, H, kBM) && make_map(&bs, a.ws_down, H, SI, 64);
        else { as = ar; bs = br; }
        if (!ok) return MOE_ERR_CUDA;
        BwdParams p{};
        p.offsets = w.offsets; p.counts = w.totals; p.E = static_cast<int>(E); p.T = static_cast<int>(T);
        p.has_shared = has_shared;
        p.n_tiles_routed = nti; p.n_tiles_shared = nts;
        p.kb_routed = p.kb_shared = static_cast<int>(H / kBK);
        p.b_rows_per_expert = static_cast<int>(H);
        p.out_routed = w.dgu_r; p.ld_routed = 2 * I; p.out_shared = w.dgu_s; p.ld_shared = 2 * SI;
        p.out2_routed = w.h_r; p.ld2_routed = I; p.out2_shared = w.h_s; p.ld2_shared = SI;
        p.gu_routed = w.gu_r; p.gu_ld_routed = 2 * I; p.gu_shared = w.gu_s; p.gu_ld_shared = 2 * SI;
        p.half_routed = static_cast<int>(I); p.half_shared = static_cast<int>(SI);
        p.n_valid_routed = static_cast<int>(I); p.n_valid_shared = static_cast<int>(SI);
        p.dw_part = w.dw_part;
        p.idesc = idesc_bf16_f32_major(kBM, kBN, 0, 1);
        if ((v = launch_bwd_gemm<kDh>(ar, as, br, br, bs, bs, p, m_bound * (nti > nts ? nti : nts), num_sms, st)) !=
            MOE_OK)
            return v;
    }
    // 5. dx_perm = dg Wg + du Wu (block-scaled fp16)
    {
        CUtensorMap ar, as, br, b2r, bs, b2s;
        bool ok = make_map(&ar, w.dgu_r, Rp, 2 * I, kBM) && make_map(&br, a.w_gate, E * I, H, 64) &&
                  make_map(&b2r, a.w_up, E * I, H, 64);
        if (has_shared)
            ok = ok && make_map(&as, w.dgu_s, T, 2 * SI, kBM) && make_map(&bs, a.ws_gate, SI, H, 64) &&
                 make_map(&b2s, a.ws_up, SI, H, 64);
        else { as = ar; bs = br; b2s = b2r; }
        if (!ok) return MOE_ERR_CUDA;
        BwdParams p{};
        p.offsets = w.offsets; p.counts = w.totals; p.E = static_cast<int>(E); p.T = static_cast<int>(T);
        p.has_shared = has_shared;
        p.n_tiles_routed = p.n_tiles_shared = static_cast<int>(H / kBN);
        p.kb_routed = static_cast<int>(2 * I / kBK); p.kb_shared = static_cast<int>(2 * SI / kBK);
        p.i_blocks_routed = static_cast<int>(I / kBK); p.i_blocks_shared = static_cast<int>(SI / kBK);
        p.b_rows_per_expert = static_cast<int>(I);
        p.n_valid_routed = p.n_valid_shared = static_cast<int>(H);
        p.yq_routed = w.dxq; p.yq_shared = w.dxq + Rp * H; p.yq_ld = H;
        p.ysc_routed = w.dxs; p.ysc_shared = w.dxs + Rp * scale_ld(H); p.ysc_ld = scale_ld(H);
        p.idesc = idesc_bf16_f32_major(kBM, kBN, 0, 1);
        if ((v = launch_bwd_gemm<kDx>(ar, as, br, b2r, bs, b2s, p, m_bound * (H / kBN), num_sms, st)) != MOE_OK)
            return v;
    }
    // 6. weight gradients: dWd = dO^T h, [dWg; dWu] = [dg du]^T x
    {
        CUtensorMap ar, as, br, bs;
        bool ok = make_map(&ar, w.do_perm, Rp, H, 64) && make_map(&br, w.h_r, Rp, I, 64);
        if (has_shared) ok = ok && make_map(&as, a.dy, T, H, 64) && make_map(&bs, w.h_s, T, SI, 64);
        else { as = ar; bs = br; }
        if (!ok) return MOE_ERR_CUDA;
        BwdParams p{};
        p.offsets = w.offsets; p.counts = w.totals; p.E = static_cast<int>(E); p.T = static_cast<int>(T);
        p.has_shared = has_shared;
        p.m_tiles_wgrad_routed = p.m_tiles_wgrad_shared = static_cast<int>(H / kBM);
        p.n_tiles_routed = nti; p.n_tiles_shared = nts;
        p.n_valid_routed = static_cast<int>(I); p.n_valid_shared = static_cast<int>(SI);
        p.out_routed = static_cast<__nv_bfloat16*>(a.d_w_down); p.ld_routed = I; p.out_expert_stride = H * I;
        p.out_shared = static_cast<__nv_bfloat16*>(a.d_ws_down); p.ld_shared = SI;
        p.split_rows_routed = p.split_rows_shared = static_cast<int>(H);
        p.idesc = idesc_bf16_f32_major(kBM, kBN, 1, 1);
        const int64_t tiles = (E + has_shared) * (H / kBM) * (nti > nts ? nti : nts);
        if ((v = launch_bwd_gemm<kWgrad>(ar, as, br, br, bs, bs, p, tiles, num_sms, st)) != MOE_OK) return v;
    }
    {
        CUtensorMap ar, as, br, bs;
        bool ok = make_map(&ar, w.dgu_r, Rp, 2 * I, 64) && make_map(&br, w.x_perm, Rp, H, 64);
        if (has_shared) ok = ok && make_map(&as, w.dgu_s, T, 2 * SI, 64) && make_map(&bs, a.x, T, H, 64);
        else { as = ar; bs = br; }
        if (!ok) return MOE_ERR_CUDA;
        BwdParams p{};
        p.offsets = w.offsets; p.counts = w.totals; p.E = static_cast<int>(E); p.T = static_cast<int>(T);
        p.has_shared = has_shared;
        p.m_tiles_wgrad_routed = static_cast<int>(2 * I / kBM);
        p.m_tiles_wgrad_shared = static_cast<int>(2 * SI / kBM);
        p.n_tiles_routed = p.n_tiles_shared = static_cast<int>(H / kBN);
        p.n_valid_routed = p.n_valid_shared = static_cast<int>(H);
        p.out_routed = static_cast<__nv_bfloat16*>(a.d_w_gate); p.ld_routed = H; p.out_expert_stride = I * H;
        p.out2_routed = static_cast<__nv_bfloat16*>(a.d_w_up); p.ld2_routed = H; p.out2_expert_stride = I * H;
        p.out_shared = static_cast<__nv_bfloat16*>(a.d_ws_gate); p.ld_shared = H;
        p.out2_shared = static_cast<__nv_bfloat16*>(a.d_ws_up); p.ld2_shared = H;
        p.split_rows_routed = static_cast<int>(I); p.split_rows_shared = static_cast<int>(SI);
        p.idesc = idesc_bf16_f32_major(kBM, kBN, 1, 1);
        const int64_t tiles = (E + has_shared) * (2 * (I > SI ? I : SI) / kBM) * (H / kBN);
        if ((v = launch_bwd_gemm<kWgrad>(ar, as, br, br, bs, bs, p, tiles, num_sms, st)) != MOE_OK) return v;
    }
    // 7. router backward, router weight gradient, dx
    const RouterPlan rp = plan_router(static_cast<int>(T), static_cast<int>(E), static_cast<int>(H));
    bwd_router_kernel<<<static_cast<unsigned>((T + 255) / 256), 256, 0, st>>>(
        w.router_part, rp.nsplit, static_cast<int>(T), static_cast<int>(E), static_cast<int>(K), c->norm_topk_prob,
        c->routed_scaling_factor, w.topk_idx, w.topk_w, w.row_of, w.dw_part, 2 * nti, w.dlogit);
    bwd_router_wgrad_kernel<<<dim3(static_cast<unsigned>(E), static_cast<unsigned>((H / 8 + 255) / 256),
                                   kRouterSplit),
                              256, 0, st>>>(w.offsets, w.totals, w.perm_src, w.dlogit, w.x_perm, static_cast<int>(H),
                                            static_cast<int>(E), w.dwr_part);
    bwd_router_wgrad_reduce_kernel<<<static_cast<unsigned>((E * H + 255) / 256), 256, 0, st>>>(w.dwr_part, E * H,
                                                                                             d_router_w);
    bwd_dx_kernel<<<gs, 256, 0, st>>>(w.dxq, w.dxs, scale_ld(H), w.row_of, w.topk_idx, w.dlogit, router_w,
                                      static_cast<int>(K), static_cast<int>(H), has_shared, Rp, dx);
    count_launch(4);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}


// The training forward: the layer's forward computed so that the backward can
// reuse its routing, expert rows and g | u (kept in a backward workspace, the
// "context"): route, dispatch into 128-row aligned segments, g and u (bf16) with
// h = silu(g) u from the same fp32 accumulators, the down projection with the
// routing weights, combine.
int launch_forward_train(const moe_config* c, int64_t T, const float* router_w, const float* e_bias,
                         const BwdArgs& a, void* y, int y_dtype, const WorkspaceBwd& w, int num_sms,
                         cudaStream_t st) {
    const int64_t H = c->hidden_size, E = c->n_routed_experts;
    const int64_t I = c->moe_intermediate_size, SI = static_cast<int64_t>(c->n_shared_experts) * I;
    const int has_shared = SI > 0 ? 1 : 0;
    const int64_t Rp = w.rp;
    int v;
    if ((v = bwd_front(c, T, router_w, e_bias, a.x, nullptr, w, num_sms, st)) != MOE_OK) return v;
    if ((v = bwd_recompute(c, T, a, w, num_sms, st, true)) != MOE_OK) return v;
    CUtensorMap ar, as, br, bs;
    bool ok = make_map(&ar, w.h_r, Rp, I, kBM) && make_map(&br, a.w_down, E * H, I, kBN);
    if (has_shared) ok = ok && make_map(&as, w.h_s, T, SI, kBM) && make_map(&bs, a.ws_down, H, SI, kBN);
    else { as = ar; bs = br; }
    if (!ok) return MOE_ERR_CUDA;
    BwdParams p{};
    p.offsets = w.offsets; p.counts = w.totals; p.E = static_cast<int>(E); p.T = static_cast<int>(T);
    p.has_shared = has_shared;
    p.n_tiles_routed = p.n_tiles_shared = static_cast<int>(H / kBN);
    p.kb_routed = static_cast<int>(I / kBK); p.kb_shared = static_cast<int>(SI / kBK);
    p.b_rows_per_expert = static_cast<int>(H);
    p.n_valid_routed = p.n_valid_shared = static_cast<int>(H);
    p.yq_routed = w.dxq; p.yq_shared = w.dxq + Rp * H; p.yq_ld = H;
    p.ysc_routed = w.dxs; p.ysc_shared = w.dxs + Rp * scale_ld(H); p.ysc_ld = scale_ld(H);
    p.perm_src = w.perm_src; p.topk_w = w.topk_w;
    p.idesc = idesc_bf16_f32_major(kBM, kBN, 0, 0);
    const int64_t m_bound = Rp / kBM + (has_shared ? (T + kBM - 1) / kBM : 0);
    if ((v = launch_bwd_gemm<kFwdDown>(ar, as, br, br, bs, bs, p, m_bound * (H / kBN), num_sms, st)) != MOE_OK)
        return v;
    return launch_combine(c, T, w.dxq, w.dxs, w.row_of, y, y_dtype, st, Rp);
}

// ---------------------------------------------------------------- host buffers
// moe_forward_host: the forward from pinned host x to host y, the batch cut into
// chunks of rows (rows are independent, so the result is the same as one call):
// chunk i's input copy and chunk i-1's output copy run on two internal copy
// streams while chunk i is computed on the caller's stream.  Two staging slots
// each for x and y in the workspace; an event per slot orders reuse.
struct HostStreams {
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t x_ready[2], computed[2], y_copied[2], start, done;
    std::mutex mu;
    bool ready = false;
};
HostStreams g_hs[64];

int host_streams(HostStreams** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
    HostStreams& h = g_hs[dev];
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!h.ready) {
        if (cudaStreamCreateWithFlags(&h.h2d, cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&h.d2h, cudaStreamNonBlocking) != cudaSuccess)
            return MOE_ERR_CUDA;
        cudaEvent_t* evs[] = {&h.x_ready[0], &h.x_ready[1], &h.computed[0], &h.computed[1],
                              &h.y_copied[0], &h.y_copied[1], &h.start, &h.done};
        for (cudaEvent_t* e : evs)
            if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return MOE_ERR_CUDA;
        h.ready = true;
    }
    *out = &h;
    return MOE_OK;
}

struct HostPlan {
    int64_t chunk;       // rows per chunk
    size_t x_slot, y_slot, fwd_bytes, bytes;
};

HostPlan plan_host(const moe_config* c, int64_t T, int64_t chunk_tokens, int y_dtype) {
    HostPlan hp{};
    hp.chunk = chunk_tokens > 0 && chunk_tokens < T ? chunk_tokens : T;
    if (hp.chunk < 1) hp.chunk = 1;
    const int64_t H = c->hidden_size;
    hp.x_slot = align_up(static_cast<size_t>(hp.chunk * H * 2));
    hp.y_slot = align_up(static_cast<size_t>(hp.chunk * H * (y_dtype == MOE_DTYPE_BF16 ? 2 : 4)));
    // The last chunk may be shorter, and a short batch can split the router's
    // hidden axis further: size for the larger of the two.
    const int64_t last = T - ((T + hp.chunk - 1) / hp.chunk - 1) * hp.chunk;
    const size_t a = workspace_bytes_for(c, hp.chunk), b = workspace_bytes_for(c, last > 0 ? last : hp.chunk);
    hp.fwd_bytes = align_up(a > b ? a : b);
    hp.bytes = 2 * hp.x_slot + 2 * hp.y_slot + hp.fwd_bytes;
    return hp;
}

// ---------------------------------------------------------------- no-allocation dispatch
// Scratch of moe_dispatch_noalloc: per-block expert counts, per-block bases and
// per-expert totals (2 x ceil(T / kDispTok) x E + E int32), held in this
// file-scope device array instead of a caller workspace.  Every GPU that loads
// the library keeps it until the process exits.
constexpr int64_t kStaticDispatchInts = (1 << 18) + 1024;  // 1 MiB + 4 KiB
static __device__ __align__(256) int32_t g_dispatch_scratch[kStaticDispatchInts];

int32_t* g_dispatch_scratch_addr[64];
std::mutex g_dispatch_scratch_mu;

// Device address of g_dispatch_scratch on the current device, looked up once per
// device (host code cannot use the symbol itself as a device pointer).
int dispatch_scratch(int32_t** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_dispatch_scratch_mu);
    if (!g_dispatch_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_dispatch_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
        g_dispatch_scratch_addr[dev] = static_cast<int32_t*>(p);
    }
    *out = g_dispatch_scratch_addr[dev];
    return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

int moe_workspace_size(const moe_config* cfg, int64_t T, size_t* bytes) {
    if (!bytes) return MOE_ERR_INVALID_ARG;
    const int v = validate_cfg(cfg, T);
    if (v != MOE_OK) return v;
    *bytes = workspace_bytes_for(cfg, T);
    return MOE_OK;
}

int moe_route(const moe_config* cfg, int64_t T, const void* x, const float* router_w, const float* e_bias,
              int32_t* topk_idx, float* topk_w, void* workspace, size_t workspace_bytes, void* stream) {
    int v = validate_cfg(cfg, T);
    if (v != MOE_OK) return v;
    if (T == 0) return MOE_OK;
    if (!x || !router_w || !e_bias || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(router_w)) return MOE_ERR_UNSUPPORTED;
    if (!workspace || workspace_bytes < workspace_bytes_for(cfg, T)) return MOE_ERR_WORKSPACE;
    DeviceInfo* d = nullptr;
    if ((v = device_info(&d)) != MOE_OK) return v;
    Workspace w = carve(cfg, T, static_cast<uint8_t*>(workspace));
    return launch_route(cfg, T, x, router_w, e_bias, topk_idx, topk_w, w.router_part, w.router_w3, d->num_sms,
                        static_cast<cudaStream_t>(stream));
}

int moe_dispatch(const moe_config* cfg, int64_t T, const void* x, const int32_t* topk_idx,
                 int32_t* expert_offsets, void* x_perm, int32_t* perm_src, int32_t* row_of, void* workspace,
                 size_t workspace_bytes, void* stream) {
    int v = validate_cfg(cfg, T);
    if (v != MOE_OK) return v;
    if (!expert_offsets) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        // No rows: every expert segment is empty.
        if (cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (cfg->n_routed_experts + 1), st) !=
            cudaSuccess)
            return MOE_ERR_CUDA;
        return MOE_OK;
    }
    if (!x || !topk_idx || !x_perm || !perm_src || !row_of) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(x_perm)) return MOE_ERR_UNSUPPORTED;
    if (!workspace || workspace_bytes < workspace_bytes_for(cfg, T)) return MOE_ERR_WORKSPACE;
    Workspace w = carve(cfg, T, static_cast<uint8_t*>(workspace));
    return launch_dispatch(cfg, T, x, topk_idx, expert_offsets, x_perm, perm_src, row_of, w.block_counts,
                           w.block_base, w.totals, st);
}

namespace {
int check_ptrs(std::initializer_list<const void*> ps) {
    for (const void* p : ps)
        if (!p) return MOE_ERR_INVALID_ARG;
    for (const void* p : ps)
        if (!aligned16(p)) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}
}  // namespace

int moe_dispatch_noalloc(const moe_config* cfg, int64_t T, const void* x, const int32_t* topk_idx,
                         int32_t* expert_offsets, void* x_perm, int32_t* perm_src, int32_t* row_of, void* stream) {
    int v = validate_cfg(cfg, T);
    if (v != MOE_OK) return v;
    if (!expert_offsets) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t E = cfg->n_routed_experts;
    const int64_t nb = (T + kDispTok - 1) / kDispTok;
    if (2 * nb * E + E > kStaticDispatchInts) return MOE_ERR_STATIC_LIMIT;
    if (T == 0) {
        if (cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (E + 1), st) != cudaSuccess) return MOE_ERR_CUDA;
        return MOE_OK;
    }
    if (!x || !topk_idx || !x_perm || !perm_src || !row_of) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(x_perm)) return MOE_ERR_UNSUPPORTED;
    int32_t* scratch = nullptr;
    if ((v = dispatch_scratch(&scratch)) != MOE_OK) return v;
    // Every part is fully written by the count and scan kernels before it is
    // read, so nothing has to be cleared between calls.
    return launch_dispatch(cfg, T, x, topk_idx, expert_offsets, x_perm, perm_src, row_of, scratch,
                           scratch + nb * E, scratch + 2 * nb * E, st);
}

int moe_experts_gate_up(const moe_config* cfg, int64_t T, const void* x, const void* x_perm,
                        const int32_t* expert_offsets, const void* w_gate, const void* w_up, const void* ws_gate,
                        const void* ws_up, void* h_routed, void* h_shared, void* stream) {
    int v = validate_cfg(cfg, T);
    if (v != MOE_OK) return v;
    if (T == 0) return MOE_OK;
    if (!expert_offsets) return MOE_ERR_INVALID_ARG;
    if ((v = check_ptrs({x_perm, w_gate, w_up, h_routed})) != MOE_OK) return v;
    if (cfg->n_shared_experts > 0 && (v = check_ptrs({x, ws_gate, ws_up, h_shared})) != MOE_OK) return v;
    DeviceInfo* d = nullptr;
    if ((v = device_info(&d)) != MOE_OK) return v;
    return launch_gate_up(cfg, T, x, x_perm, routed_rows_of(cfg, T, expert_offsets), w_gate, w_up, ws_gate, ws_up,
                          h_routed, h_shared,
                          d->num_sms, static_cast<cudaStream_t>(stream));
}

int moe_experts_down(const moe_config* cfg, int64_t T, const void* h_routed, const void* h_shared,
                     const int32_t* expert_offsets, const int32_t* perm_src, const float* topk_w,
                     const void* w_down, const void* ws_down, void* y_perm, void* y_perm_scale, void* stream) {
    int v = validate_cfg(cfg, T);
    if (v != MOE_OK) return v;
    if (T == 0) return MOE_OK;
    if (!expert_offsets || !perm_src || !topk_w) return MOE_ERR_INVALID_ARG;
    if ((v = check_ptrs({h_routed, w_down, y_perm, y_perm_scale})) != MOE_OK) return v;
    if (cfg->n_shared_experts > 0 && (v = check_ptrs({h_shared, ws_down})) != MOE_OK) return v;
    DeviceInfo* d = nullptr;
    if ((v = device_info(&d)) != MOE_OK) return v;
    ScaledRows yr, ys;
    split_y_perm(cfg, T * cfg->num_experts_per_tok, y_perm, y_perm_scale, &yr, &ys);
    return launch_down(cfg, T, h_routed, h_shared, routed_rows_of(cfg, T, expert_offsets), perm_src, topk_w,
                       T * cfg->num_experts_per_tok, w_down, ws_down, yr, ys, d->num_sms,
                       static_cast<cudaStream_t>(stream));
}

int moe_experts(const moe_config* cfg, int64_t T, const void* x, const void* x_perm,
                const int32_t* expert_offsets, const int32_t* perm_src, const float* topk_w, const void* w_gate,
                const void* w_up, const void* w_down, const void* ws_gate, const void* ws_up,
                const void* ws_down, void* h_routed, void* h_shared, void* y_perm, void* y_perm_scale,
                void* stream) {
    int v = validate_cfg(cfg, T);
    if (v != MOE_OK) return v;
    if (T == 0) return MOE_OK;
    if (!expert_offsets || !perm_src || !topk_w) return MOE_ERR_INVALID_ARG;
    if ((v = check_ptrs({x_perm, w_gate, w_up, w_down, h_routed, y_perm, y_perm_scale})) != MOE_OK) return v;
    if (cfg->n_shared_experts > 0 && (v = check_ptrs({x, ws_gate, ws_up, ws_down, h_shared})) != MOE_OK)
        return v;
    DeviceInfo* d = nullptr;
    if ((v = device_info(&d)) != MOE_OK) return v;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const RoutedRows rr = routed_rows_of(cfg, T, expert_offsets);
    if ((v = launch_gate_up(cfg, T, x, x_perm, rr, w_gate, w_up, ws_gate, ws_up, h_routed, h_shared, d->num_sms,
                            st)) != MOE_OK)
        return v;
    ScaledRows yr, ys;
    split_y_perm(cfg, rr.R, y_perm, y_perm_scale, &yr, &ys);
    return launch_down(cfg, T, h_routed, h_shared, rr, perm_src, topk_w, rr.R, w_down, ws_down, yr, ys, d->num_sms,
                       st);
}

int moe_combine(const moe_config* cfg, int64_t T, const void* y_perm, const void* y_perm_scale,
                const int32_t* row_of, void* y, int32_t y_dtype, void* stream) {
    int v = validate_cfg(cfg, T);
    if (v != MOE_OK) return v;
    if (y_dtype != MOE_DTYPE_F32 && y_dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!y_perm || !y_perm_scale || !row_of || !y) return MOE_ERR_INVALID_ARG;
    if (!aligned16(y_perm) || !aligned16(y) || !aligned16(y_perm_scale)) return MOE_ERR_UNSUPPORTED;
    return launch_combine(cfg, T, y_perm, y_perm_scale, row_of, y, y_dtype, static_cast<cudaStream_t>(stream));
}

int moe_forward(const moe_config* cfg, int64_t T, const void* x, const float* router_w, const float* e_bias,
                const void* w_gate, const void* w_up, const void* w_down, const void* ws_gate,
                const void* ws_up, const void* ws_down, void* y, int32_t y_dtype, int32_t* topk_idx_out,
                float* topk_w_out, void* workspace, size_t workspace_bytes, void* stream) {
    int v = validate_cfg(cfg, T);
    if (v != MOE_OK) return v;
    if (y_dtype != MOE_DTYPE_F32 && y_dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    const bool sh = cfg->n_shared_experts > 0;
    if (!x || !router_w || !e_bias || !w_gate || !w_up || !w_down || !y) return MOE_ERR_INVALID_ARG;
    if (sh && (!ws_gate || !ws_up || !ws_down)) return MOE_ERR_INVALID_ARG;
    const void* al[] = {x, router_w, w_gate, w_up, w_down, y};
    for (const void* p : al)
        if (!aligned16(p)) return MOE_ERR_UNSUPPORTED;
    if (sh) {
        const void* al2[] = {ws_gate, ws_up, ws_down};
        for (const void* p : al2)
            if (!aligned16(p)) return MOE_ERR_UNSUPPORTED;
    }
    if (!workspace || workspace_bytes < workspace_bytes_for(cfg, T) || !aligned16(workspace))
        return MOE_ERR_WORKSPACE;
    DeviceInfo* d = nullptr;
    if ((v = device_info(&d)) != MOE_OK) return v;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Workspace w = carve(cfg, T, static_cast<uint8_t*>(workspace));
    int32_t* idx = topk_idx_out ? topk_idx_out : w.topk_idx;
    float* tw = topk_w_out ? topk_w_out : w.topk_w;
    const RoutedRows rr = routed_rows_of(cfg, T, w.offsets);
    if ((v = launch_route(cfg, T, x, router_w, e_bias, idx, tw, w.router_part, w.router_w3, d->num_sms, st)) != MOE_OK)
        return v;
    if ((v = launch_dispatch(cfg, T, x, idx, w.offsets, w.x_perm, w.perm_src, w.row_of, w.block_counts,
                             w.block_base, w.totals, st)) != MOE_OK)
        return v;
    if ((v = launch_gate_up(cfg, T, x, w.x_perm, rr, w_gate, w_up, ws_gate, ws_up, w.h_routed, w.h_shared,
                            d->num_sms, st)) != MOE_OK)
        return v;
    ScaledRows yr, ys;
    split_y_perm(cfg, rr.R, w.y_perm, w.y_scale, &yr, &ys);
    if ((v = launch_down(cfg, T, w.h_routed, w.h_shared, rr, w.perm_src, tw, rr.R, w_down, ws_down, yr, ys,
                         d->num_sms, st)) != MOE_OK)
        return v;
    return launch_combine(cfg, T, w.y_perm, w.y_scale, w.row_of, y, y_dtype, st);
}

int64_t moe_mx_scale_bytes(int64_t rows, int64_t K) {
    if (rows < 0 || K <= 0 || K % 128 != 0) return -1;
    return mx_scale_bytes(rows, K);
}

int moe_mx_quantize(int64_t rows, int64_t K, const void* src, void* q, void* sf, void* stream) {
    if (rows < 0 || K <= 0) return MOE_ERR_INVALID_ARG;
    if (K % 128 != 0 || rows >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
    if (rows == 0) return MOE_OK;
    int v;
    if ((v = check_ptrs({src, q, sf})) != MOE_OK) return v;
    return launch_mx_quantize(rows, K, src, q, sf, static_cast<cudaStream_t>(stream));
}

int moe_workspace_size_mx(const moe_config* cfg, int64_t T, size_t* bytes) {
    if (!bytes) return MOE_ERR_INVALID_ARG;
    const int v = validate_mx(cfg, T);
    if (v != MOE_OK) return v;
    *bytes = carve_mx(cfg, T, nullptr).bytes;
    return MOE_OK;
}

int moe_mx_routed_rows(const moe_config* cfg, int64_t T, int64_t* rows) {
    if (!rows) return MOE_ERR_INVALID_ARG;
    const int v = validate_mx(cfg, T);
    if (v != MOE_OK) return v;
    *rows = mx_routed_rows(cfg, T);
    return MOE_OK;
}

int moe_dispatch_mx(const moe_config* cfg, int64_t T, const void* x, const int32_t* topk_idx,
                    int32_t* expert_offsets, int32_t* expert_counts, void* xq_perm, void* xq_perm_sf,
                    void* xq_shared, void* xq_shared_sf, int32_t* perm_src, int32_t* row_of, void* workspace,
                    size_t workspace_bytes, void* stream) {
    int v = validate_mx(cfg, T);
    if (v != MOE_OK) return v;
    if (!expert_offsets || !expert_counts) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t E = cfg->n_routed_experts;
    if (T == 0) {
        if (cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (E + 1), st) != cudaSuccess ||
            cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * E, st) != cudaSuccess)
            return MOE_ERR_CUDA;
        return MOE_OK;
    }
    if (!topk_idx || !perm_src || !row_of) return MOE_ERR_INVALID_ARG;
    if ((v = check_ptrs({x, xq_perm, xq_perm_sf})) != MOE_OK) return v;
    if (cfg->n_shared_experts > 0 && (v = check_ptrs({xq_shared, xq_shared_sf})) != MOE_OK) return v;
    if (!workspace || workspace_bytes < carve_mx(cfg, T, nullptr).bytes) return MOE_ERR_WORKSPACE;
    WorkspaceMx w = carve_mx(cfg, T, static_cast<uint8_t*>(workspace));
    if ((v = launch_dispatch_mx(cfg, T, x, topk_idx, expert_offsets, static_cast<uint8_t*>(xq_perm),
                                static_cast<uint8_t*>(xq_perm_sf), static_cast<uint8_t*>(xq_shared),
                                static_cast<uint8_t*>(xq_shared_sf), perm_src, row_of, w.block_counts,
                                w.block_base, w.totals, st)) != MOE_OK)
        return v;
    if (cudaMemcpyAsync(expert_counts, w.totals, sizeof(int32_t) * E, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

int moe_forward_mx(const moe_config* cfg, int64_t T, const void* x, const float* router_w, const float* e_bias,
                   const moe_mx_weights* weights, void* y, int32_t y_dtype, int32_t* topk_idx_out,
                   float* topk_w_out, void* workspace, size_t workspace_bytes, void* stream) {
    int v = validate_mx(cfg, T);
    if (v != MOE_OK) return v;
    if (y_dtype != MOE_DTYPE_F32 && y_dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!weights || !e_bias) return MOE_ERR_INVALID_ARG;
    const moe_mx_weights* wt = weights;
    if ((v = check_ptrs({x, router_w, y, wt->gate.q, wt->gate.sf, wt->up.q, wt->up.sf, wt->down.q, wt->down.sf})) !=
        MOE_OK)
        return v;
    if (cfg->n_shared_experts > 0 &&
        (v = check_ptrs({wt->shared_gate.q, wt->shared_gate.sf, wt->shared_up.q, wt->shared_up.sf,
                         wt->shared_down.q, wt->shared_down.sf})) != MOE_OK)
        return v;
    if (!workspace || workspace_bytes < carve_mx(cfg, T, nullptr).bytes || !aligned16(workspace))
        return MOE_ERR_WORKSPACE;
    DeviceInfo* d = nullptr;
    if ((v = device_info(&d)) != MOE_OK) return v;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    WorkspaceMx w = carve_mx(cfg, T, static_cast<uint8_t*>(workspace));
    int32_t* idx = topk_idx_out ? topk_idx_out : w.topk_idx;
    float* tw = topk_w_out ? topk_w_out : w.topk_w;
    if ((v = launch_route(cfg, T, x, router_w, e_bias, idx, tw, w.router_part, w.router_w3, d->num_sms, st)) != MOE_OK)
        return v;
    if ((v = launch_dispatch_mx(cfg, T, x, idx, w.offsets, w.xq_perm, w.xq_perm_sf, w.xq_shared, w.xq_shared_sf,
                                w.perm_src, w.row_of, w.block_counts, w.block_base, w.totals, st)) != MOE_OK)
        return v;
    const MxBuffers b = buffers_of(w);
    if ((v = launch_gate_up_mx(cfg, T, b, wt, d->num_sms, st)) != MOE_OK) return v;
    if ((v = launch_down_mx(cfg, T, b, wt, tw, d->num_sms, st)) != MOE_OK) return v;
    return launch_combine(cfg, T, w.y_perm, w.y_scale, w.row_of, y, y_dtype, st, w.rp);
}

namespace {
int check_mx_weights(const moe_config* cfg, const moe_mx_weights* wt, bool gate_up, bool down) {
    if (!wt) return MOE_ERR_INVALID_ARG;
    int v;
    if (gate_up && (v = check_ptrs({wt->gate.q, wt->gate.sf, wt->up.q, wt->up.sf})) != MOE_OK) return v;
    if (down && (v = check_ptrs({wt->down.q, wt->down.sf})) != MOE_OK) return v;
    if (cfg->n_shared_experts > 0) {
        if (gate_up && (v = check_ptrs({wt->shared_gate.q, wt->shared_gate.sf, wt->shared_up.q,
                                        wt->shared_up.sf})) != MOE_OK)
            return v;
        if (down && (v = check_ptrs({wt->shared_down.q, wt->shared_down.sf})) != MOE_OK) return v;
    }
    return MOE_OK;
}
}  // namespace

int moe_experts_gate_up_mx(const moe_config* cfg, int64_t T, const void* xq_perm, const void* xq_perm_sf,
                           const void* xq_shared, const void* xq_shared_sf, const int32_t* expert_offsets,
                           const int32_t* expert_counts, const moe_mx_weights* weights, void* hq_routed,
                           void* hq_routed_sf, void* hq_shared, void* hq_shared_sf, void* stream) {
    int v = validate_mx(cfg, T);
    if (v != MOE_OK) return v;
    if (T == 0) return MOE_OK;
    if (!expert_offsets || !expert_counts) return MOE_ERR_INVALID_ARG;
    if ((v = check_ptrs({xq_perm, xq_perm_sf, hq_routed, hq_routed_sf})) != MOE_OK) return v;
    if (cfg->n_shared_experts > 0 && (v = check_ptrs({xq_shared, xq_shared_sf, hq_shared, hq_shared_sf})) != MOE_OK)
        return v;
    if ((v = check_mx_weights(cfg, weights, true, false)) != MOE_OK) return v;
    DeviceInfo* d = nullptr;
    if ((v = device_info(&d)) != MOE_OK) return v;
    MxBuffers b{expert_offsets,
                expert_counts,
                static_cast<const uint8_t*>(xq_perm),
                static_cast<const uint8_t*>(xq_perm_sf),
                static_cast<const uint8_t*>(xq_shared),
                static_cast<const uint8_t*>(xq_shared_sf),
                static_cast<uint8_t*>(hq_routed),
                static_cast<uint8_t*>(hq_routed_sf),
                static_cast<uint8_t*>(hq_shared),
                static_cast<uint8_t*>(hq_shared_sf),
                nullptr,
                nullptr,
                nullptr,
                mx_routed_rows(cfg, T)};
    return launch_gate_up_mx(cfg, T, b, weights, d->num_sms, static_cast<cudaStream_t>(stream));
}

int moe_experts_down_mx(const moe_config* cfg, int64_t T, const void* hq_routed, const void* hq_routed_sf,
                        const void* hq_shared, const void* hq_shared_sf, const int32_t* expert_offsets,
                        const int32_t* expert_counts, const int32_t* perm_src, const float* topk_w,
                        const moe_mx_weights* weights, void* y_perm, void* y_perm_scale, void* stream) {
    int v = validate_mx(cfg, T);
    if (v != MOE_OK) return v;
    if (T == 0) return MOE_OK;
    if (!expert_offsets || !expert_counts || !perm_src || !topk_w) return MOE_ERR_INVALID_ARG;
    if ((v = check_ptrs({hq_routed, hq_routed_sf, y_perm, y_perm_scale})) != MOE_OK) return v;
    if (cfg->n_shared_experts > 0 && (v = check_ptrs({hq_shared, hq_shared_sf})) != MOE_OK) return v;
    if ((v = check_mx_weights(cfg, weights, false, true)) != MOE_OK) return v;
    DeviceInfo* d = nullptr;
    if ((v = device_info(&d)) != MOE_OK) return v;
    MxBuffers b{expert_offsets,
                expert_counts,
                nullptr,
                nullptr,
                nullptr,
                nullptr,
                const_cast<uint8_t*>(static_cast<const uint8_t*>(hq_routed)),
                const_cast<uint8_t*>(static_cast<const uint8_t*>(hq_routed_sf)),
                const_cast<uint8_t*>(static_cast<const uint8_t*>(hq_shared)),
                const_cast<uint8_t*>(static_cast<const uint8_t*>(hq_shared_sf)),
                perm_src,
                static_cast<__half*>(y_perm),
                static_cast<uint8_t*>(y_perm_scale),
                mx_routed_rows(cfg, T)};
    return launch_down_mx(cfg, T, b, weights, topk_w, d->num_sms, static_cast<cudaStream_t>(stream));
}

int moe_combine_mx(const moe_config* cfg, int64_t T, const void* y_perm, const void* y_perm_scale,
                   const int32_t* row_of, void* y, int32_t y_dtype, void* stream) {
    int v = validate_mx(cfg, T);
    if (v != MOE_OK) return v;
    if (y_dtype != MOE_DTYPE_F32 && y_dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!y_perm || !y_perm_scale || !row_of || !y) return MOE_ERR_INVALID_ARG;
    if (!aligned16(y_perm) || !aligned16(y) || !aligned16(y_perm_scale)) return MOE_ERR_UNSUPPORTED;
    return launch_combine(cfg, T, y_perm, y_perm_scale, row_of, y, y_dtype, static_cast<cudaStream_t>(stream),
                          mx_routed_rows(cfg, T));
}

int moe_workspace_size_bwd(const moe_config* cfg, int64_t T, size_t* bytes) {
    if (!bytes) return MOE_ERR_INVALID_ARG;
    const int v = validate_mx(cfg, T);
    if (v != MOE_OK) return v;
    *bytes = carve_bwd(cfg, T, nullptr).bytes;
    return MOE_OK;
}

int moe_backward(const moe_config* cfg, int64_t T, const void* x, const float* router_w, const float* e_bias,
                 const void* w_gate, const void* w_up, const void* w_down, const void* ws_gate, const void* ws_up,
                 const void* ws_down, const void* dy, float* dx, float* d_router_w, void* d_w_gate, void* d_w_up,
                 void* d_w_down, void* d_ws_gate, void* d_ws_up, void* d_ws_down, void* workspace,
                 size_t workspace_bytes, void* stream) {
    int v = validate_mx(cfg, T);
    if (v != MOE_OK) return v;
    const bool sh = cfg->n_shared_experts > 0;
    if ((v = check_ptrs({router_w, w_gate, w_up, w_down, d_router_w, d_w_gate, d_w_up, d_w_down})) != MOE_OK) return v;
    if (sh && (v = check_ptrs({ws_gate, ws_up, ws_down, d_ws_gate, d_ws_up, d_ws_down})) != MOE_OK) return v;
    if (!e_bias) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t H = cfg->hidden_size, E = cfg->n_routed_experts, I = cfg->moe_intermediate_size;
    const int64_t SI = static_cast<int64_t>(cfg->n_shared_experts) * I;
    if (T == 0) {
        // No tokens: every gradient is zero.
        const size_t wb = sizeof(uint16_t) * E * I * H, sb = sizeof(uint16_t) * SI * H;
        if (cudaMemsetAsync(d_router_w, 0, sizeof(float) * E * H, st) != cudaSuccess ||
            cudaMemsetAsync(d_w_gate, 0, wb, st) != cudaSuccess || cudaMemsetAsync(d_w_up, 0, wb, st) != cudaSuccess ||
            cudaMemsetAsync(d_w_down, 0, wb, st) != cudaSuccess ||
            (sh && (cudaMemsetAsync(d_ws_gate, 0, sb, st) != cudaSuccess ||
                    cudaMemsetAsync(d_ws_up, 0, sb, st) != cudaSuccess ||
                    cudaMemsetAsync(d_ws_down, 0, sb, st) != cudaSuccess)))
            return MOE_ERR_CUDA;
        return MOE_OK;
    }
    if ((v = check_ptrs({x, dy, dx})) != MOE_OK) return v;
    if (!workspace || workspace_bytes < carve_bwd(cfg, T, nullptr).bytes || !aligned16(workspace))
        return MOE_ERR_WORKSPACE;
    DeviceInfo* d = nullptr;
    if ((v = device_info(&d)) != MOE_OK) return v;
    const WorkspaceBwd w = carve_bwd(cfg, T, static_cast<uint8_t*>(workspace));
    const BwdArgs a{x, dy, w_gate, w_up, w_down, ws_gate, ws_up, ws_down,
                    d_w_gate, d_w_up, d_w_down, d_ws_gate, d_ws_up, d_ws_down};
    return launch_backward(cfg, T, router_w, e_bias, a, dx, d_router_w, w, d->num_sms, st);
}

int moe_workspace_size_host(const moe_config* cfg, int64_t T, int64_t chunk_tokens, int32_t y_dtype, size_t* bytes) {
    if (!bytes) return MOE_ERR_INVALID_ARG;
    const int v = validate_cfg(cfg, T);
    if (v != MOE_OK) return v;
    if (y_dtype != MOE_DTYPE_F32 && y_dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
    *bytes = plan_host(cfg, T, chunk_tokens, y_dtype).bytes;
    return MOE_OK;
}

int moe_forward_host(const moe_config* cfg, int64_t T, const void* x_host, const float* router_w, const float* e_bias,
                     const void* w_gate, const void* w_up, const void* w_down, const void* ws_gate, const void* ws_up,
                     const void* ws_down, void* y_host, int32_t y_dtype, int64_t chunk_tokens, void* workspace,
                     size_t workspace_bytes, void* stream) {
    int v = validate_cfg(cfg, T);
    if (v != MOE_OK) return v;
    if (y_dtype != MOE_DTYPE_F32 && y_dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x_host || !y_host || !e_bias) return MOE_ERR_INVALID_ARG;
    if ((v = check_ptrs({router_w, w_gate, w_up, w_down})) != MOE_OK) return v;
    if (cfg->n_shared_experts > 0 && (v = check_ptrs({ws_gate, ws_up, ws_down})) != MOE_OK) return v;
    const HostPlan hp = plan_host(cfg, T, chunk_tokens, y_dtype);
    if (!workspace || workspace_bytes < hp.bytes || !aligned16(workspace)) return MOE_ERR_WORKSPACE;
    HostStreams* hs = nullptr;
    if ((v = host_streams(&hs)) != MOE_OK) return v;
    std::lock_guard<std::mutex> lk(hs->mu);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* base = static_cast<uint8_t*>(workspace);
    uint8_t* xs[2] = {base, base + hp.x_slot};
    uint8_t* ys[2] = {base + 2 * hp.x_slot, base + 2 * hp.x_slot + hp.y_slot};
    void* fwd_ws = base + 2 * hp.x_slot + 2 * hp.y_slot;
    const int64_t H = cfg->hidden_size;
    const size_t ysz = y_dtype == MOE_DTYPE_BF16 ? 2 : 4;
    // The copy streams start after whatever the caller queued before this call.
    if (cudaEventRecord(hs->start, st) != cudaSuccess || cudaStreamWaitEvent(hs->h2d, hs->start, 0) != cudaSuccess ||
        cudaStreamWaitEvent(hs->d2h, hs->start, 0) != cudaSuccess)
        return MOE_ERR_CUDA;
    const int64_t n = (T + hp.chunk - 1) / hp.chunk;
    for (int64_t i = 0; i < n; ++i) {
        const int s = static_cast<int>(i & 1);
        const int64_t r0 = i * hp.chunk, rows = (r0 + hp.chunk <= T) ? hp.chunk : T - r0;
        // Input slot s was last read by chunk i-2's compute.
        if (i >= 2 && cudaStreamWaitEvent(hs->h2d, hs->computed[s], 0) != cudaSuccess) return MOE_ERR_CUDA;
        if (cudaMemcpyAsync(xs[s], static_cast<const uint8_t*>(x_host) + r0 * H * 2, rows * H * 2,
                            cudaMemcpyHostToDevice, hs->h2d) != cudaSuccess ||
            cudaEventRecord(hs->x_ready[s], hs->h2d) != cudaSuccess)
            return MOE_ERR_CUDA;
        // Output slot s was last read by chunk i-2's copy back.
        if (cudaStreamWaitEvent(st, hs->x_ready[s], 0) != cudaSuccess ||
            (i >= 2 && cudaStreamWaitEvent(st, hs->y_copied[s], 0) != cudaSuccess))
            return MOE_ERR_CUDA;
        if ((v = moe_forward(cfg, rows, xs[s], router_w, e_bias, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, ys[s],
                             y_dtype, nullptr, nullptr, fwd_ws, hp.fwd_bytes, stream)) != MOE_OK)
            return v;
        if (cudaEventRecord(hs->computed[s], st) != cudaSuccess ||
            cudaStreamWaitEvent(hs->d2h, hs->computed[s], 0) != cudaSuccess ||
            cudaMemcpyAsync(static_cast<uint8_t*>(y_host) + r0 * H * ysz, ys[s], rows * H * ysz,
                            cudaMemcpyDeviceToHost, hs->d2h) != cudaSuccess ||
            cudaEventRecord(hs->y_copied[s], hs->d2h) != cudaSuccess)
            return MOE_ERR_CUDA;
    }
    // The caller's stream reaches the end of this call once the last output copy is done.
    if (cudaEventRecord(hs->done, hs->d2h) != cudaSuccess || cudaStreamWaitEvent(st, hs->done, 0) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

int moe_forward_train(const moe_config* cfg, int64_t T, const void* x, const float* router_w, const float* e_bias,
                      const void* w_gate, const void* w_up, const void* w_down, const void* ws_gate,
                      const void* ws_up, const void* ws_down, void* y, int32_t y_dtype, void* context,
                      size_t context_bytes, void* stream) {
    int v = validate_mx(cfg, T);
    if (v != MOE_OK) return v;
    if (y_dtype != MOE_DTYPE_F32 && y_dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!e_bias) return MOE_ERR_INVALID_ARG;
    if ((v = check_ptrs({x, router_w, w_gate, w_up, w_down, y})) != MOE_OK) return v;
    if (cfg->n_shared_experts > 0 && (v = check_ptrs({ws_gate, ws_up, ws_down})) != MOE_OK) return v;
    if (!context || context_bytes < carve_bwd(cfg, T, nullptr).bytes || !aligned16(context)) return MOE_ERR_WORKSPACE;
    DeviceInfo* d = nullptr;
    if ((v = device_info(&d)) != MOE_OK) return v;
    const WorkspaceBwd w = carve_bwd(cfg, T, static_cast<uint8_t*>(context));
    const BwdArgs a{x, nullptr, w_gate, w_up, w_down, ws_gate, ws_up, ws_down,
                    nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
    return launch_forward_train(cfg, T, router_w, e_bias, a, y, y_dtype, w, d->num_sms,
                                static_cast<cudaStream_t>(stream));
}

int moe_backward_train(const moe_config* cfg, int64_t T, const void* x, const float* router_w,
                       const void* w_gate, const void* w_up, const void* w_down, const void* ws_gate,
                       const void* ws_up, const void* ws_down, const void* dy, float* dx, float* d_router_w,
                       void* d_w_gate, void* d_w_up, void* d_w_down, void* d_ws_gate, void* d_ws_up,
                       void* d_ws_down, void* context, size_t context_bytes, void* stream) {
    int v = validate_mx(cfg, T);
    if (v != MOE_OK) return v;
    const bool sh = cfg->n_shared_experts > 0;
    if ((v = check_ptrs({router_w, w_gate, w_up, w_down, d_router_w, d_w_gate, d_w_up, d_w_down})) != MOE_OK) return v;
    if (sh && (v = check_ptrs({ws_gate, ws_up, ws_down, d_ws_gate, d_ws_up, d_ws_down})) != MOE_OK) return v;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        const int64_t H = cfg->hidden_size, E = cfg->n_routed_experts, I = cfg->moe_intermediate_size;
        const int64_t SI = static_cast<int64_t>(cfg->n_shared_experts) * I;
        const size_t wb = sizeof(uint16_t) * E * I * H, sb = sizeof(uint16_t) * SI * H;
        if (cudaMemsetAsync(d_router_w, 0, sizeof(float) * E * H, st) != cudaSuccess ||
            cudaMemsetAsync(d_w_gate, 0, wb, st) != cudaSuccess || cudaMemsetAsync(d_w_up, 0, wb, st) != cudaSuccess ||
            cudaMemsetAsync(d_w_down, 0, wb, st) != cudaSuccess ||
            (sh && (cudaMemsetAsync(d_ws_gate, 0, sb, st) != cudaSuccess ||
                    cudaMemsetAsync(d_ws_up, 0, sb, st) != cudaSuccess ||
                    cudaMemsetAsync(d_ws_down, 0, sb, st) != cudaSuccess)))
            return MOE_ERR_CUDA;
        return MOE_OK;
    }
    if ((v = check_ptrs({x, dy, dx})) != MOE_OK) return v;
    if (!context || context_bytes < carve_bwd(cfg, T, nullptr).bytes || !aligned16(context)) return MOE_ERR_WORKSPACE;
    DeviceInfo* d = nullptr;
    if ((v = device_info(&d)) != MOE_OK) return v;
    const WorkspaceBwd w = carve_bwd(cfg, T, static_cast<uint8_t*>(context));
    const BwdArgs a{x, dy, w_gate, w_up, w_down, ws_gate, ws_up, ws_down,
                    d_w_gate, d_w_up, d_w_down, d_ws_gate, d_ws_up, d_ws_down};
    return launch_backward(cfg, T, router_w, nullptr, a, dx, d_router_w, w, d->num_sms, st, true);
}

const char* moe_status_string(int status) {
    switch (status) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported shape or alignment";
        case MOE_ERR_WORKSPACE: return "workspace missing or too small";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_TIMEOUT: return "a bounded device wait gave up";
        case MOE_ERR_DEVICE_CHECK: return "a device-side check found an index out of range (entry skipped)";
        case MOE_ERR_STATIC_LIMIT:
            return "size exceeds the fixed scratch of the no-allocation entry point "
                   "(2 * ceil(T / 32) * n_routed_experts + n_routed_experts must be <= 263168)";
        default: return "unknown status";
    }
}

int moe_device_status(void* stream, int32_t* device_error) {
    if (!device_error) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned int word = 0, zero = 0;
    if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&word, g_moe_error, sizeof(word)) != cudaSuccess) return MOE_ERR_CUDA;
    if (word != 0 && cudaMemcpyToSymbol(g_moe_error, &zero, sizeof(zero)) != cudaSuccess) return MOE_ERR_CUDA;
    *device_error = static_cast<int32_t>(word);
    if (word == 0) return MOE_OK;
    return (word >= kErrCheckFirst && word <= kErrCheckLast) ? MOE_ERR_DEVICE_CHECK : MOE_ERR_TIMEOUT;
}

uint64_t moe_launch_count(void) { return g_launches.load(); }

int moe_bias_update(const moe_config* cfg, int64_t T, const int32_t* topk_idx, float* e_bias, float gamma,
                    int32_t* expert_load, void* stream) {
    int v = validate_cfg(cfg, T);
    if (v != MOE_OK) return v;
    if (!topk_idx || !e_bias || !(gamma == gamma) || gamma < 0.0f || gamma > 3.0e38f) return MOE_ERR_INVALID_ARG;
    bias_update_kernel<<<1, 1024, 0, static_cast<cudaStream_t>(stream)>>>(
        topk_idx, T * cfg->num_experts_per_tok, cfg->n_routed_experts, gamma, e_bias, expert_load);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// ---------------------------------------------------------------- expert parallelism
namespace {
int validate_ep(const moe_config* c, int64_t T, int32_t world) {
    const int v = validate_cfg(c, T);
    if (v != MOE_OK) return v;
    if (world < 1 || c->n_routed_experts % world != 0) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

// Wire rows: a send row is the token's H bf16 values, then its k expert ids
// (int32) and k routing weights (fp32), zero-padded to 16 bytes; a return row is
// H block-scaled fp16 values, then their H/32 scale codes, padded to 16 bytes.
int64_t ep_send_row_bytes(const moe_config* c) {
    return 2ll * c->hidden_size + static_cast<int64_t>(align_up(8ull * c->num_experts_per_tok, 16));
}
int64_t ep_return_row_bytes(const moe_config* c) {
    return 2ll * c->hidden_size + static_cast<int64_t>(align_up(c->hidden_size / 32, 16));
}

// Rows one source sends for T tokens at most: one per (token, rank holding one of
// its experts), so at most min(k, world) per token.
int64_t ep_send_rows_max(const moe_config* c, int64_t T, int world) {
    return T * (c->num_experts_per_tok < world ? c->num_experts_per_tok : world);
}

// Expert rows of one rank for R received rows: at most one per received slot.
// (Rows from moe_ep_send name k distinct experts, so at most min(k, E/world) of
// them are local; the bound does not rely on that, since the rows are caller data.)
int64_t ep_local_rows_max(const moe_config* c, int64_t R) { return R * c->num_experts_per_tok; }

// Every received-row slot index and expert row (with up to 127 padding rows per
// segment and the shared rows) must fit an int32 and a TMA coordinate.
int check_ep_rows(const moe_config* c, int64_t T, int64_t R) {
    if (R < 0) return MOE_ERR_INVALID_ARG;
    if (R * c->num_experts_per_tok + T + 128ll * c->n_routed_experts >= (1ll << 31) - 256) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

struct WorkspaceEpSend {
    int32_t* slot_dest;     // [T, k] destination rank of each slot
    int32_t* rank_slot;     // [T, k] destination rank of a slot's row, or -1
    int32_t* perm_src;      // [T * min(k, world)] slot of each send row
    int32_t* offsets;       // [world + 1]
    int32_t* block_counts;  // [world, nb]
    int32_t* block_base;    // [world, nb]
    int32_t* totals;        // [world]
    size_t bytes;
};

WorkspaceEpSend carve_ep_send(const moe_config* c, int world, int64_t T, uint8_t* base) {
    const int64_t K = c->num_experts_per_tok, nb = (T + kDispTok - 1) / kDispTok;
    WorkspaceEpSend w{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        uint8_t* p = base ? base + off : nullptr;
        off += align_up(bytes);
        return p;
    };
    w.slot_dest = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * T * K));
    w.rank_slot = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * T * K));
    w.perm_src = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * ep_send_rows_max(c, T, world)));
    w.offsets = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (world + 1)));
    w.block_counts = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * nb * world));
    w.block_base = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * nb * world));
    w.totals = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * world));
    w.bytes = off;
    return w;
}

struct WorkspaceEpExperts {
    int32_t* offsets;         // [El + 1] segments of the El local experts
    int32_t* perm_src;        // [Rb] received slot (r * k + j) of each expert row
    int32_t* row_of;          // [R, k] expert row of each received slot, or -1
    int32_t* block_counts;    // [El, nb]
    int32_t* block_base;      // [El, nb]
    int32_t* totals;          // [El]
    float* w_perm;            // [Rb] routing weight of each expert row
    __nv_bfloat16* x_perm;    // [Rb, H]
    __nv_bfloat16* h_routed;  // [Rb, I]
    __nv_bfloat16* h_shared;  // [T, S*I]
    __half* y_perm;           // [Rb, H] block-scaled fp16
    uint8_t* y_scale;         // [Rb, scale_ld]
    size_t bytes;
};

WorkspaceEpExperts carve_ep_experts(const moe_config* c, int64_t El, int64_t T, int64_t R, uint8_t* base) {
    const int64_t K = c->num_experts_per_tok, H = c->hidden_size;
    const int64_t I = c->moe_intermediate_size, SI = static_cast<int64_t>(c->n_shared_experts) * I;
    const int64_t nb = (R + kDispTok - 1) / kDispTok, Rb = ep_local_rows_max(c, R);
    WorkspaceEpExperts w{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        uint8_t* p = base ? base + off : nullptr;
        off += align_up(bytes);
        return p;
    };
    w.offsets = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (El + 1)));
    w.perm_src = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * Rb));
    w.row_of = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * R * K));
    w.block_counts = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * nb * El));
    w.block_base = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * nb * El));
    w.totals = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * El));
    w.w_perm = reinterpret_cast<float*>(take(sizeof(float) * Rb));
    w.x_perm = reinterpret_cast<__nv_bfloat16*>(take(2 * Rb * H));
    w.h_routed = reinterpret_cast<__nv_bfloat16*>(take(2 * Rb * I));
    w.h_shared = reinterpret_cast<__nv_bfloat16*>(take(2 * T * SI));
    w.y_perm = reinterpret_cast<__half*>(take(2 * Rb * H));
    w.y_scale = reinterpret_cast<uint8_t*>(take(Rb * scale_ld(H)));
    w.bytes = off;
    return w;
}

// El = the most experts one rank holds (E/world without redundant copies).
size_t ep_workspace_bytes(const moe_config* c, int world, int64_t El, int64_t T, int64_t R) {
    const size_t a = carve_ep_send(c, world, T, nullptr).bytes, b = carve_ep_experts(c, El, T, R, nullptr).bytes;
    return a > b ? a : b;
}

// Number of replicas listed for expert e (the leading entries >= 0), 0 if the
// list is malformed (an entry outside [0, world), a repeated rank, or a valid
// entry after a -1).
int ep_replicas(const int32_t* reps, int max_rep, int world) {
    int n = 0;
    while (n < max_rep && reps[n] >= 0) {
        if (reps[n] >= world) return 0;
        for (int i = 0; i < n; ++i)
            if (reps[i] == reps[n]) return 0;
        ++n;
    }
    for (int i = n; i < max_rep; ++i)
        if (reps[i] >= 0) return 0;
    return n;
}
}  // namespace

int moe_ep_row_bytes(const moe_config* cfg, int64_t* send_row_bytes, int64_t* return_row_bytes) {
    const int v = validate_cfg(cfg, 0);
    if (v != MOE_OK) return v;
    if (!send_row_bytes || !return_row_bytes) return MOE_ERR_INVALID_ARG;
    *send_row_bytes = ep_send_row_bytes(cfg);
    *return_row_bytes = ep_return_row_bytes(cfg);
    return MOE_OK;
}

int moe_ep_workspace_size(const moe_config* cfg, int32_t world, int32_t n_local, int64_t T, int64_t R,
                          size_t* bytes) {
    int v = validate_ep(cfg, T, world);
    if (v != MOE_OK) return v;
    if (!bytes || n_local < 1 || n_local > cfg->n_routed_experts) return MOE_ERR_INVALID_ARG;
    if ((v = check_ep_rows(cfg, T, R)) != MOE_OK) return v;
    *bytes = ep_workspace_bytes(cfg, world, n_local, T, R);
    return MOE_OK;
}

int moe_ep_place(int32_t E, int32_t world, const int64_t* load, int32_t n_redundant, int32_t max_rep,
                 int32_t* expert_ranks) {
    if (E < 1 || world < 1 || E % world != 0 || max_rep < 1 || !load || !expert_ranks) return MOE_ERR_INVALID_ARG;
    if (n_redundant < 0) return MOE_ERR_INVALID_ARG;
    for (int e = 0; e < E; ++e)
        if (load[e] < 0) return MOE_ERR_INVALID_ARG;
    const int El = E / world;
    std::vector<int> n_rep(E, 1);
    std::vector<double> rank_load(world, 0.0);
    for (int e = 0; e < E; ++e) {
        expert_ranks[static_cast<int64_t>(e) * max_rep] = e / El;
        for (int i = 1; i < max_rep; ++i) expert_ranks[static_cast<int64_t>(e) * max_rep + i] = -1;
        rank_load[e / El] += static_cast<double>(load[e]);
    }
    for (int step = 0; step < n_redundant; ++step) {
        // The expert whose copies carry the most rows each (lowest id on ties)...
        int be = -1;
        double best = 0.0;
        for (int e = 0; e < E; ++e) {
            if (n_rep[e] >= max_rep || n_rep[e] >= world) continue;
            const double share = static_cast<double>(load[e]) / n_rep[e];
            if (share > best) {
                best = share;
                be = e;
            }
        }
        if (be < 0) break;  // nothing left that a copy would relieve
        // ...gets a copy on the least loaded rank that does not hold it (lowest rank on ties).
        int32_t* reps = expert_ranks + static_cast<int64_t>(be) * max_rep;
        int br = -1;
        for (int r = 0; r < world; ++r) {
            bool holds = false;
            for (int i = 0; i < n_rep[be]; ++i) holds = holds || reps[i] == r;
            if (!holds && (br < 0 || rank_load[r] < rank_load[br])) br = r;
        }
        const double s0 = static_cast<double>(load[be]) / n_rep[be], s1 = static_cast<double>(load[be]) / (n_rep[be] + 1);
        for (int i = 0; i < n_rep[be]; ++i) rank_load[reps[i]] -= s0 - s1;
        rank_load[br] += s1;
        reps[n_rep[be]++] = br;
    }
    return MOE_OK;
}

int moe_ep_local_experts(int32_t E, int32_t world, int32_t rank, const int32_t* expert_ranks, int32_t max_rep,
                         int32_t* local_of, int32_t* n_local) {
    if (E < 1 || world < 1 || E % world != 0 || rank < 0 || rank >= world || max_rep < 1 || !expert_ranks ||
        !local_of || !n_local)
        return MOE_ERR_INVALID_ARG;
    int n = 0;
    for (int e = 0; e < E; ++e) {
        const int32_t* reps = expert_ranks + static_cast<int64_t>(e) * max_rep;
        const int nr = ep_replicas(reps, max_rep, world);
        if (nr == 0) return MOE_ERR_INVALID_ARG;
        bool here = false;
        for (int i = 0; i < nr; ++i) here = here || reps[i] == rank;
        local_of[e] = here ? n++ : -1;
    }
    *n_local = n;
    return MOE_OK;
}

int moe_ep_send(const moe_config* cfg, int32_t world, int64_t T, const void* x, const int32_t* topk_idx,
                const float* topk_w, const int32_t* expert_ranks, int32_t max_rep, int32_t* send_counts,
                void* send_rows, int32_t* send_row_of, void* workspace, size_t workspace_bytes, void* stream) {
    int v = validate_ep(cfg, T, world);
    if (v != MOE_OK) return v;
    if (!send_counts || (expert_ranks && max_rep < 1)) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        if (cudaMemsetAsync(send_counts, 0, sizeof(int32_t) * world, st) != cudaSuccess) return MOE_ERR_CUDA;
        return MOE_OK;
    }
    if (!topk_idx || !topk_w || !send_row_of) return MOE_ERR_INVALID_ARG;
    if ((v = check_ptrs({x, send_rows})) != MOE_OK) return v;
    if (!workspace || workspace_bytes < carve_ep_send(cfg, world, T, nullptr).bytes || !aligned16(workspace))
        return MOE_ERR_WORKSPACE;
    const WorkspaceEpSend w = carve_ep_send(cfg, world, T, static_cast<uint8_t*>(workspace));
    const int K = cfg->num_experts_per_tok, E = cfg->n_routed_experts, H = cfg->hidden_size;
    const int64_t Wb = ep_send_row_bytes(cfg);
    ep_rank_slots_kernel<<<static_cast<unsigned>((T + 255) / 256), 256, 0, st>>>(
        topk_idx, T, K, E / world, E, expert_ranks, expert_ranks ? max_rep : 1, world, w.slot_dest, w.rank_slot);
    count_launch();
    // Sort the (token, rank) rows by rank: the rank-slot entries are the buckets,
    // -1 (a rank the token already has a row for) is no row.
    RowSort a{};
    a.si = SlotIndex{w.rank_slot, K, 0, -1, world};
    a.T = T;
    a.K = K;
    a.E = world;
    a.H = H;
    a.x = x;
    a.x_ld = H;
    a.x_perm = send_rows;
    a.out_ld = Wb / 2;
    a.offsets = w.offsets;
    a.perm_src = w.perm_src;
    a.row_of = send_row_of;
    a.block_counts = w.block_counts;
    a.block_base = w.block_base;
    a.totals = w.totals;
    if ((v = launch_row_sort(a, st)) != MOE_OK) return v;
    const int meta_words = static_cast<int>((Wb - 2ll * H) / 4);
    const int64_t n_max = ep_send_rows_max(cfg, T, world);
    int64_t blocks = (n_max * meta_words + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    ep_send_meta_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        w.offsets, world, w.perm_src, T * K, K, topk_idx, topk_w, w.slot_dest, n_max, static_cast<uint8_t*>(send_rows),
        Wb, 2ll * H, meta_words, send_counts);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_ep_experts(const moe_config* cfg, int32_t world, int32_t rank, const int32_t* local_of, int32_t n_local,
                   int64_t T, const void* x, int64_t R, const void* recv_rows, const void* w_gate, const void* w_up,
                   const void* w_down, const void* ws_gate, const void* ws_up, const void* ws_down,
                   void* return_rows, void* y_shared, void* y_shared_scale, void* workspace, size_t workspace_bytes,
                   void* stream) {
    int v = validate_ep(cfg, T, world);
    if (v != MOE_OK) return v;
    if (rank < 0 || rank >= world) return MOE_ERR_INVALID_ARG;
    const int El = local_of ? n_local : cfg->n_routed_experts / world;
    if (El < 1 || El > cfg->n_routed_experts) return MOE_ERR_INVALID_ARG;
    if ((v = check_ep_rows(cfg, T, R)) != MOE_OK) return v;
    const bool sh = cfg->n_shared_experts > 0 && T > 0;
    if (!sh && R == 0) return MOE_OK;
    if ((v = check_ptrs({w_gate, w_up, w_down})) != MOE_OK) return v;
    if (R > 0 && (v = check_ptrs({recv_rows, return_rows})) != MOE_OK) return v;
    if (sh && (v = check_ptrs({x, ws_gate, ws_up, ws_down, y_shared, y_shared_scale})) != MOE_OK) return v;
    if (!workspace || workspace_bytes < carve_ep_experts(cfg, El, T, R, nullptr).bytes || !aligned16(workspace))
        return MOE_ERR_WORKSPACE;
    DeviceInfo* d = nullptr;
    if ((v = device_info(&d)) != MOE_OK) return v;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const WorkspaceEpExperts w = carve_ep_experts(cfg, El, T, R, static_cast<uint8_t*>(workspace));
    const int K = cfg->num_experts_per_tok, E = cfg->n_routed_experts, H = cfg->hidden_size;
    const int64_t Wb = ep_send_row_bytes(cfg), Wr = ep_return_row_bytes(cfg);
    const int64_t Rb = ep_local_rows_max(cfg, R);
    // With no shared rows to compute (S = 0 or no local tokens) the shared members
    // are unused; the launches still take well-formed maps.
    moe_config c = *cfg;
    if (!sh) c.n_shared_experts = 0;
    if (R > 0) {
        // The received rows' slots sorted by local expert: -1 marks a slot sent
        // elsewhere; any other id must be one of this rank's experts (the block
        // rank * E/world.., or local_of[id] >= 0), else it is a caller error.
        const uint8_t* rows = static_cast<const uint8_t*>(recv_rows);
        RowSort a{};
        a.si = SlotIndex{reinterpret_cast<const int32_t*>(rows + 2ll * H), static_cast<int>(Wb / 4),
                         local_of ? 0 : rank * El, -1, E, local_of, 1};
        a.T = R;
        a.K = K;
        a.E = El;
        a.H = H;
        a.x = recv_rows;
        a.x_ld = Wb / 2;
        a.x_perm = w.x_perm;
        a.out_ld = H;
        a.offsets = w.offsets;
        a.perm_src = w.perm_src;
        a.row_of = w.row_of;
        a.block_counts = w.block_counts;
        a.block_base = w.block_base;
        a.totals = w.totals;
        a.w_src = reinterpret_cast<const float*>(rows + 2ll * H + 4ll * K);
        a.w_perm = w.w_perm;
        if ((v = launch_row_sort(a, st)) != MOE_OK) return v;
    } else if (cudaMemsetAsync(w.offsets, 0, sizeof(int32_t) * (El + 1), st) != cudaSuccess) {
        return MOE_ERR_CUDA;
    }
    const RoutedRows rr{Rb, El, El, w.offsets};
    if ((v = launch_gate_up(&c, T, x, w.x_perm, rr, w_gate, w_up, ws_gate, ws_up, w.h_routed, w.h_shared, d->num_sms,
                            st)) != MOE_OK)
        return v;
    const ScaledRows yr{w.y_perm, w.y_scale};
    const ScaledRows ys{static_cast<__half*>(y_shared), static_cast<uint8_t*>(y_shared_scale)};
    if ((v = launch_down(&c, T, w.h_routed, w.h_shared, rr, nullptr, w.w_perm, Rb, w_down, ws_down, yr, ys,
                         d->num_sms, st)) != MOE_OK)
        return v;
    if (R == 0) return MOE_OK;
    // Each received row's sum over its slots on this rank, re-encoded for the way back.
    CombineDst dst{};
    dst.rows = ScaledRowsOut{static_cast<__half*>(return_rows), Wr / 2, static_cast<uint8_t*>(return_rows) + 2ll * H,
                             Wr};
    return launch_combine_rows(R, K, H, ScaledRowsIn{w.y_perm, H, w.y_scale, scale_ld(H)}, Rb, w.row_of, 1,
                               ScaledRowsIn{nullptr, 0, nullptr, 0}, dst, kOutScaled, st);
}

int moe_ep_combine(const moe_config* cfg, int32_t world, int64_t T, int64_t n_back, const void* back_rows,
                   const int32_t* send_row_of, const void* y_shared, const void* y_shared_scale, void* y,
                   int32_t y_dtype, void* stream) {
    int v = validate_ep(cfg, T, world);
    if (v != MOE_OK) return v;
    if (y_dtype != MOE_DTYPE_F32 && y_dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
    if (n_back < 0 || n_back > ep_send_rows_max(cfg, T, world)) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!send_row_of) return MOE_ERR_INVALID_ARG;
    if ((v = check_ptrs({back_rows, y})) != MOE_OK) return v;
    const bool sh = cfg->n_shared_experts > 0;
    if (sh && (v = check_ptrs({y_shared, y_shared_scale})) != MOE_OK) return v;
    const int64_t H = cfg->hidden_size, Wr = ep_return_row_bytes(cfg);
    const uint8_t* b = static_cast<const uint8_t*>(back_rows);
    const ScaledRowsIn routed{reinterpret_cast<const __half*>(b), Wr / 2, b + 2 * H, Wr};
    const ScaledRowsIn shared = sh ? ScaledRowsIn{static_cast<const __half*>(y_shared), H,
                                                  static_cast<const uint8_t*>(y_shared_scale), scale_ld(H)}
                                   : ScaledRowsIn{nullptr, 0, nullptr, 0};
    CombineDst dst{};
    dst.y = y;
    return launch_combine_rows(T, cfg->num_experts_per_tok, cfg->hidden_size, routed, n_back, send_row_of, 1, shared,
                               dst, y_dtype == MOE_DTYPE_BF16 ? kOutBF16 : kOutF32, static_cast<cudaStream_t>(stream));
}

int moe_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
    if (limit_ns == 0 || limit_ns > 10000000000ull) return MOE_ERR_INVALID_ARG;
    wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, 0x901u);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // extern "C"
