// host.cu -- status codes, per-device state, the error word, tensor-map
// encoding, the bounded-wait self test and the tensor-pipe peak probe.
#include <cudaTypedefs.h>

#include <atomic>
#include <cstring>
#include <mutex>
#include <vector>

#include "internal.h"
#include "sm100.cuh"

namespace dq {

// One error word per device (each device holds its own copy of this module).
__device__ uint32_t g_err_word;

namespace {

constexpr int kMaxDevices = 64;
DeviceInfo g_devices[kMaxDevices];
std::mutex g_dev_mutex;
thread_local int t_last_cuda_error = 0;
std::atomic<unsigned long long> g_timeout_ns{2000000000ull};

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
cudaError_t g_encode_err = cudaSuccess;

void resolve_encoder() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  g_encode_err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (g_encode_err == cudaSuccess && q == cudaDriverEntryPointSuccess && fn != nullptr)
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  else if (g_encode_err == cudaSuccess)
    g_encode_err = cudaErrorNotSupported;
}

// Kernels whose shared-memory limit has been raised, per device.  Entries
// are appended under the mutex and published by the release store of n, so
// the scan needs no lock.
struct AttrEntry {
  const void* kernel;
  int bytes;
};
constexpr int kMaxAttr = 96;
struct DeviceAttrs {
  std::atomic<int> n{0};
  AttrEntry e[kMaxAttr];
};
DeviceAttrs g_attrs[kMaxDevices];
std::mutex g_attr_mutex;

bool attr_known(const DeviceAttrs& a, const void* kernel, int bytes) {
  const int n = a.n.load(std::memory_order_acquire);
  for (int i = 0; i < n; ++i)
    if (a.e[i].kernel == kernel && a.e[i].bytes >= bytes) return true;
  return false;
}

}  // namespace

std::atomic<int> g_schedule_override{0};
std::atomic<int> g_tile_n_override{0};
std::atomic<int> g_two_widths{1};
std::atomic<int> g_bsr_panel{1};
std::atomic<int> g_quant_kernel_override{0};

dq_status smem_limit_once(const void* kernel, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return DQ_ERR_UNSUPPORTED;
  DeviceAttrs& a = g_attrs[dev];
  if (attr_known(a, kernel, bytes)) return DQ_OK;
  std::lock_guard<std::mutex> lock(g_attr_mutex);
  if (attr_known(a, kernel, bytes)) return DQ_OK;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return cuda_fail(e);
  const int n = a.n.load(std::memory_order_relaxed);
  if (n < kMaxAttr) {               // a full table only costs a repeated (harmless) set
    a.e[n] = AttrEntry{kernel, bytes};
    a.n.store(n + 1, std::memory_order_release);
  }
  return DQ_OK;
}

dq_status cuda_fail(cudaError_t e) {
  t_last_cuda_error = static_cast<int>(e);
  return DQ_ERR_CUDA;
}

unsigned long long wait_timeout_ns() { return g_timeout_ns.load(std::memory_order_relaxed); }

dq_status current_device(DeviceInfo** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return DQ_ERR_UNSUPPORTED;
  DeviceInfo& d = g_devices[dev];
  if (d.device == dev) {
    *out = &d;
    return d.cc_major == 10 && d.cc_minor == 0 ? DQ_OK : DQ_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  if (d.device != dev) {
    DeviceInfo n;
    n.device = dev;
    if ((e = cudaDeviceGetAttribute(&n.sm_count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&n.cc_major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&n.cc_minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
      return cuda_fail(e);
    int optin = 0;
    if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
      return cuda_fail(e);
    n.max_smem_optin = static_cast<size_t>(optin);
    if (n.cc_major == 10 && n.cc_minor == 0) {
      void* p = nullptr;
      if ((e = cudaGetSymbolAddress(&p, g_err_word)) != cudaSuccess) return cuda_fail(e);
      n.err_word = static_cast<uint32_t*>(p);
    }
    d = n;
  }
  *out = &d;
  return d.cc_major == 10 && d.cc_minor == 0 ? DQ_OK : DQ_ERR_UNSUPPORTED;
}

dq_status make_tmap_u8_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                          uint64_t stride_bytes, uint32_t box_inner, uint32_t box_outer,
                          int swizzle_bytes) {
  std::call_once(g_encode_once, resolve_encoder);
  if (g_encode == nullptr) return cuda_fail(g_encode_err);
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUtensorMapSwizzle sw = swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                          : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                          : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    t_last_cuda_error = static_cast<int>(r);
    return DQ_ERR_CUDA;
  }
  return DQ_OK;
}

dq_status make_tmap_out_2d(CUtensorMap* map, void* base, uint64_t cols, uint64_t rows,
                           int elem_bytes) {
  std::call_once(g_encode_once, resolve_encoder);
  if (g_encode == nullptr) return cuda_fail(g_encode_err);
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * static_cast<uint64_t>(elem_bytes)};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  const bool four = elem_bytes == 4;
  CUresult r = g_encode(map, four ? CU_TENSOR_MAP_DATA_TYPE_INT32 : CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, base,
                        dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        four ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                        CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    t_last_cuda_error = static_cast<int>(r);
    return DQ_ERR_CUDA;
  }
  return DQ_OK;
}

// ------------------------------------------------------------ self test

__global__ void selftest_wait_kernel(WaitCtl ctl) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Nothing ever arrives on `bar`: the bounded wait must give up.
    mbar_wait(smem_u32(&bar), 0, ctl, &abort_flag);
  }
  __syncthreads();
}

// ------------------------------------------------------------ peak probe

// One CTA per SM; thread 0 issues `iters` 128x256x32 int8 MMAs from two
// fixed shared-memory tiles into one TMEM accumulator.
__global__ void __launch_bounds__(128, 1) mma_peak_kernel(int iters, WaitCtl ctl) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_tile = smem;                 // 128 x 128 B
  uint8_t* b_tile = smem + 128 * 128;     // 256 x 128 B
  __shared__ __align__(8) uint64_t done_bar;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  const int warp = threadIdx.x / 32;
  for (int i = threadIdx.x; i < (128 + 256) * 128 / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem)[i] = make_uint4(0x01010101u, 0x01010101u, 0x01010101u, 0x01010101u);
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&done_bar), 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_base), 256);
    tmem_relinquish();
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) {
    const uint32_t idesc = idesc_i8(128, 256);
    const uint64_t ad = smem_desc_kmajor<128>(smem_u32(a_tile));
    const uint64_t bd = smem_desc_kmajor<128>(smem_u32(b_tile));
#pragma unroll 1
    for (int i = 0; i < iters; ++i) {
      const uint32_t k = static_cast<uint32_t>(i & 3) * 2;   // 32-byte K step
      mma_i8(tmem_base, ad + k, bd + k, idesc, i > 0 ? 1u : 0u);
    }
    mma_commit(smem_u32(&done_bar));
    mbar_wait(smem_u32(&done_bar), 0, ctl, &abort_flag);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem_base, 256);
}

}  // namespace dq

using namespace dq;

extern "C" {

const char* dq_status_string(dq_status s) {
  switch (s) {
    case DQ_OK: return "DQ_OK";
    case DQ_ERR_INVALID_ARG: return "DQ_ERR_INVALID_ARG: invalid argument";
    case DQ_ERR_UNSUPPORTED: return "DQ_ERR_UNSUPPORTED: shape, alignment or device not supported";
    case DQ_ERR_CUDA: return "DQ_ERR_CUDA: a CUDA call failed (see dq_last_cuda_error)";
    case DQ_ERR_TIMEOUT: return "DQ_ERR_TIMEOUT: a bounded device wait ran out";
  }
  return "unknown dq_status";
}

int dq_last_cuda_error(void) { return t_last_cuda_error; }

int dq_version(void) { return 100; }

void dq_debug_set_schedule(int mode) { g_schedule_override.store(mode, std::memory_order_relaxed); }
void dq_debug_set_tile_n(int n) { g_tile_n_override.store(n, std::memory_order_relaxed); }
void dq_debug_set_two_widths(int on) { g_two_widths.store(on, std::memory_order_relaxed); }
void dq_debug_set_bsr_panel(int mode) { g_bsr_panel.store(mode, std::memory_order_relaxed); }
void dq_debug_set_quant_kernel(int mode) { g_quant_kernel_override.store(mode, std::memory_order_relaxed); }

void dq_set_wait_timeout_ns(uint64_t ns) {
  g_timeout_ns.store(ns == 0 ? 2000000000ull : static_cast<unsigned long long>(ns));
}

dq_status dq_sync_status(dq_stream_t stream) {
  DeviceInfo* d = nullptr;
  dq_status st = current_device(&d);
  if (st != DQ_OK) return st;
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  uint32_t word = 0;
  e = cudaMemcpyFromSymbol(&word, g_err_word, sizeof(word));
  if (e != cudaSuccess) return cuda_fail(e);
  if (word != 0) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(g_err_word, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_fail(e);
    if (word & kErrTimeout) noalloc_mark_dirty(d->device);
  }
  return (word & kErrTimeout) ? DQ_ERR_TIMEOUT : DQ_OK;
}

dq_status dq_selftest_wait_timeout(dq_stream_t stream) {
  DeviceInfo* d = nullptr;
  dq_status st = current_device(&d);
  if (st != DQ_OK) return st;
  WaitCtl ctl{d->err_word, wait_timeout_ns()};
  selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(ctl);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? DQ_OK : cuda_fail(e);
}

dq_status dq_mma_peak_probe(int grid, int iters, dq_stream_t stream) {
  DeviceInfo* d = nullptr;
  dq_status st = current_device(&d);
  if (st != DQ_OK) return st;
  if (iters < 1) return DQ_ERR_INVALID_ARG;
  if (grid <= 0) grid = d->sm_count;
  const int smem = (128 + 256) * 128 + 1024;
  if ((st = smem_limit_once(reinterpret_cast<const void*>(&mma_peak_kernel), smem)) != DQ_OK) return st;
  WaitCtl ctl{d->err_word, wait_timeout_ns()};
  mma_peak_kernel<<<grid, 128, smem, reinterpret_cast<cudaStream_t>(stream)>>>(iters, ctl);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? DQ_OK : cuda_fail(e);
}

}  // extern "C"
