// pipeline.cuh -- small device helpers for the warp-specialised kernels whose
// A operand is built in shared memory by worker warps (decompressed or
// dequantized weight tiles): sleeping bounded mbarrier waits, explicit
// shared-memory accesses, the 128B-swizzled K-major tile addressing and 1-D
// bulk copies.
#pragma once

#include <cstdint>

#include "sm100.cuh"

namespace dq {
namespace pipe {

// try_wait may suspend the thread (up to kSuspendNs) until the phase
// completes, so waiting warps take no issue slots from the working ones.
constexpr uint32_t kSuspendNs = 200000;

__device__ __forceinline__ bool try_wait_sleep(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(kSuspendNs)
      : "memory");
  return ok != 0;
}

// Bounded wait on the phase of `bar` with the given parity: gives up after
// ctl.timeout_ns (recording kErrTimeout and raising *abort) or as soon as
// another role has raised *abort.
__device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity, const WaitCtl& ctl, volatile int* abort) {
  if (try_wait_sleep(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    if (try_wait_sleep(bar, parity)) return true;
    if (*abort) return false;
    if (globaltimer() - t0 > ctl.timeout_ns) {
      atomicOr(ctl.err, kErrTimeout);
      *abort = 1;
      return false;
    }
  }
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds16(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds8(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Writes `width` (16 or 32) tokens of one output channel per lane, given as
// bf16 pairs (pk[i]: token 2i in the low half, 2i + 1 in the high half),
// into a staging buffer of 32 rows x 64 B (row j = token j; the warp's 32
// lanes = 32 neighbouring channels) for one 2-D TMA store.  Lanes exchange
// values in pairs so that each lane writes two neighbouring channels of one
// token (4 bytes; rows j and j + 1 of one instruction cover all 32 banks).
__device__ __forceinline__ void stage_bf16_pairs(uint32_t buf, const uint32_t (&pk)[16], int width, int lane) {
  const bool odd = lane & 1;
  const uint32_t col = static_cast<uint32_t>(lane & ~1) * 2u;
  const uint32_t sel = odd ? 0x3276u : 0x5410u;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    if (2 * i < width) {
      const uint32_t recv = __shfl_xor_sync(0xffffffffu, pk[i], 1);
      // even lane: (own token 2i, partner's token 2i); odd: (partner's 2i + 1, own 2i + 1)
      const uint32_t v = __byte_perm(pk[i], recv, sel);
      sts32(buf + static_cast<uint32_t>(2 * i + (odd ? 1 : 0)) * 64u + col, v);
    }
  }
}

// Byte offset of 16-byte chunk `c` (0..7) of row `r` in a 128B-swizzled
// K-major tile (rows of 128 B; the chunk index is XORed with r mod 8, as a
// SWIZZLE_128B tensor copy lays it out).  The tile must be 1024-byte aligned.
__device__ __forceinline__ uint32_t sw128_off(int r, int c) {
  return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

using dq::bulk_load_1d;

}  // namespace pipe
}  // namespace dq
