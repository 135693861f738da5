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

// Measurement knob, not part of the public header: 0 = automatic schedule,
// 1 = 1-SM kernel with whole tiles, 2 = 1-SM stream-K whenever a workspace
// allows it, 3 = the 2-SM pair kernel for every M, 4 = the dense arrangement
// also for M <= 128.
extern "C" DQ_API void dq_debug_set_schedule(int mode);
// Measurement knob: force the dense tile width (128, 160, 192, 224, 256; 0 = automatic).
extern "C" DQ_API void dq_debug_set_tile_n(int n);
// Measurement knob: 0 turns off the two-width (wave-balanced) dense schedule.
extern "C" DQ_API void dq_debug_set_two_widths(int on);
// Measurement knob: BSR panel variant (activation panel kept in shared memory,
// K <= 1280): 0 = never, 1 = automatic (blocks smaller than 64), 2 = always.
extern "C" DQ_API void dq_debug_set_bsr_panel(int mode);
// Measurement knob: quantize kernel (0 = automatic, 1 = register-resident,
// 2 = row-pipelined through shared memory).
extern "C" DQ_API void dq_debug_set_quant_kernel(int mode);
