// Device error word of the library and the device-side checks of caller data.
//
// The C ABI takes raw device pointers, so index arrays that a caller passes in
// (routing indices, expert offsets, row maps) cannot be checked on the host.
// Every kernel that indexes memory with such a value checks it first; an entry
// out of range is skipped (it reads or writes nothing) and the first failure's
// code is recorded here.  moe_device_status() reads and clears the word.
//   0x1xx .. 0x3xx, 0x9xx   a bounded wait gave up (TMA producer, MMA issuer,
//                           epilogue, self-test)
//   0x4xx                   caller data out of range (codes below)
#pragma once
#include <cstdint>

namespace moe {

__device__ unsigned int g_moe_error;

__device__ __forceinline__ void record_error(unsigned code) { atomicCAS(&g_moe_error, 0u, code); }

enum : unsigned {
    kErrExpertId = 0x401,  // a routing index outside [0, n_routed_experts)
    kErrRowIndex = 0x402,  // a row index (row_of) outside the rows of y_perm
    kErrSegment = 0x403,   // an expert segment (offsets / counts) outside the row space
    kErrSlot = 0x404,      // a slot index (perm_src) outside [0, T * k)
};

// First code of the caller-data range: moe_device_status reports words at or
// above it (and below the self-test codes) as MOE_ERR_DEVICE_CHECK.
constexpr unsigned kErrCheckFirst = 0x400, kErrCheckLast = 0x4ff;

// Rows of an expert segment [row0, row0 + rows) after the range check: the
// segment (its last tile rounded up to `align` rows when the kernel writes whole
// tiles) must lie in [0, max_rows) and start on a multiple of `align`; otherwise
// it gets no rows and kErrSegment is recorded.
__device__ __forceinline__ int checked_segment_rows(int row0, int rows, int64_t max_rows, int align) {
    const int64_t end = static_cast<int64_t>(row0) + (static_cast<int64_t>(rows) + align - 1) / align * align;
    if (row0 < 0 || rows < 0 || end > max_rows || row0 % align != 0) {
        record_error(kErrSegment);
        return 0;
    }
    return rows;
}

// Routing weight of routed row `row`: topk_w[perm_src[row]] (perm_src maps the
// row to its (token, slot) entry), or topk_w[row] when perm_src is null (rows
// already listed with their own weights).  A slot outside [0, n_slots) gives
// weight 0 and records kErrSlot.
__device__ __forceinline__ float row_weight(const int32_t* perm_src, const float* topk_w, int64_t row,
                                            int64_t n_slots) {
    const int64_t slot = perm_src ? static_cast<int64_t>(perm_src[row]) : row;
    if (slot < 0 || slot >= n_slots) {
        record_error(kErrSlot);
        return 0.0f;
    }
    return topk_w[slot];
}

}  // namespace moe
