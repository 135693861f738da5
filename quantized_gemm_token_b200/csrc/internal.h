// internal.h -- host-side helpers shared by the libdq translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/dq.h"

namespace dq {

// Per-device facts, filled on the first call that touches a device.
struct DeviceInfo {
  int device = -1;
  int sm_count = 0;
  int cc_major = 0, cc_minor = 0;
  size_t max_smem_optin = 0;
  uint32_t* err_word = nullptr;   // device address of the per-device error word
};

// Resolves the current device's info; DQ_ERR_UNSUPPORTED if it is not sm_100.
dq_status current_device(DeviceInfo** out);

// Raises `kernel`'s dynamic shared-memory limit to `bytes` on the current
// device, once per (device, kernel): the attribute belongs to a device's
// context, so every device the process launches on needs its own setting.
// Thread-safe; later calls for the same pair cost a short table scan.
dq_status smem_limit_once(const void* kernel, int bytes);

// Asks dq_int8_linear_noalloc to zero its static scratch on `device` again
// before its next use (a kernel that gave up a bounded wait may have left
// partial sums in it).
void noalloc_mark_dirty(int device);

// Records a CUDA error for dq_last_cuda_error() and returns DQ_ERR_CUDA.
dq_status cuda_fail(cudaError_t e);

// Launch-time wait limit (ns) for bounded waits.
unsigned long long wait_timeout_ns();

// cuTensorMapEncodeTiled through the runtime's driver entry point.
// 2-D, uint8 elements: dims {inner, outer}, outer stride in bytes, box
// {box_inner, box_outer}, swizzle = 128, 64 or 32 (bytes; anything else: none),
// zero fill out of bounds.
dq_status make_tmap_u8_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                          uint64_t stride_bytes, uint32_t box_inner, uint32_t box_outer,
                          int swizzle_bytes);

// 2-D tensor map for an output matrix [rows, cols] of 2- or 4-byte elements
// (row stride in bytes), box {32 cols, 32 rows}, swizzle matching a 32-column
// row: 64 B (2-byte elements) or 128 B (4-byte elements).
dq_status make_tmap_out_2d(CUtensorMap* map, void* base, uint64_t cols, uint64_t rows,
                           int elem_bytes);

inline bool aligned(const void* p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

}  // namespace dq

// Measurement knobs (declared in include/dq.h, "measurement knobs"): read at
// every launch, written by dq_debug_set_*; process-wide, relaxed atomics.
#include <atomic>
namespace dq {
extern std::atomic<int> g_schedule_override;
extern std::atomic<int> g_tile_n_override;
extern std::atomic<int> g_two_widths;
extern std::atomic<int> g_bsr_panel;
extern std::atomic<int> g_quant_kernel_override;
}  // namespace dq
