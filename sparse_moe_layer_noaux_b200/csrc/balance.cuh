// Auxiliary-loss-free load balancing ("The Evolving Transformer · 07", § 06: the
// per-expert bias on the routing score is nudged down when the expert is
// overloaded and up when it is underloaded; no auxiliary loss).  After a batch,
// load_e = number of (token, slot) pairs routed to expert e, and
//   bias_e <- bias_e - gamma  if load_e > T*k/E,   bias_e + gamma  if load_e < T*k/E.
#pragma once
#include <cstdint>

#include "device_status.cuh"

namespace moe {

// One block: shared-memory histogram of the routing, then the update (E <= 256).
__global__ void __launch_bounds__(1024) bias_update_kernel(const int32_t* __restrict__ topk_idx, int64_t n,
                                                           int E, float gamma, float* __restrict__ bias,
                                                           int32_t* __restrict__ load_out) {
    __shared__ int cnt[256];
    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    // Routing indices come from the caller: one outside [0, E) is not counted and
    // is recorded in the device error word.
    for (int64_t q = threadIdx.x; q < n; q += blockDim.x) {
        const int e = topk_idx[q];
        if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) atomicAdd(&cnt[e], 1);
        else record_error(kErrExpertId);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        // load_e against the mean n / E, compared exactly as load_e * E against n.
        const int64_t lhs = static_cast<int64_t>(cnt[e]) * E;
        const float step = lhs > n ? -gamma : (lhs < n ? gamma : 0.0f);
        bias[e] = bias[e] + step;
        if (load_out) load_out[e] = cnt[e];
    }
}

}  // namespace moe
