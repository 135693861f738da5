// hqq.cu -- weight-only int4 linear with the groupwise asymmetric
// dequantization fused into a bf16 tensor-core GEMM ("Fused HQQ Quantization
// Gemm", pytorch/ao PR 153: u4 / s4 codes are upcast to bf16, shifted by a
// zero point and scaled per group of in-features, then multiplied with the
// activations; forward and transposed products), plus the standalone
// dequantization and the packing of codes two to a byte.
//
// One persistent, warp-specialised kernel for sm_100a (448 threads):
//   warp 0       TMA producer: for each 64-deep contraction step, the packed
//                int4 weight tile (4 KB) and the activation tile (BN tokens x
//                64 bf16, 128B-swizzled) into a ring of NP stages.
//   warp 1       MMA issuer: tcgen05.mma kind::f16 (bf16 x bf16 -> fp32 in
//                TMEM), M = 128 weight rows, N = BN tokens, K = 16 per
//                instruction, four instructions per step.
//   warps 2..17  dequantizers, two groups of eight taking alternate steps
//                (one group's barrier and address work overlaps the other's
//                arithmetic): unpack the codes, w = bf16(bf16(q - z) * s)
//                in packed bf16x2 arithmetic, and write the 128 x 64 bf16 A
//                operand in the 128B-swizzled K-major layout into the stage
//                (the bf16 weight never reaches global memory).  Each thread
//                reads its own scales and zero points from global memory two
//                steps ahead of use: copying them into the stages with the
//                tiles cost the producer's copy engine about 100 ns per row
//                copy, twice the time of an activation or weight tile.
//   warps 18..21 epilogue, one warp per TMEM sub-partition, two 32-token
//                chunks per tensor-memory wait: tcgen05.ld the accumulator
//                (TMEM lane = output channel, column = token), convert to
//                bf16, write each 32 tokens x 32 channels block into a
//                staging buffer and store it with one TMA store (which clips
//                tokens >= M and channels >= the output width).
// The weight is the A operand (128 output channels per tile) and the tokens
// the B operand (up to 256): the dequantization work per MMA flop is then as
// small as a 128-row tile allows, and few-token calls need no padding to 128.
// Few tiles: the contraction is split over S <= 8 CTAs per tile, launched as
// one thread-block cluster; each split leaves its fp32 partial tile in its
// own shared memory and, after a cluster barrier, every CTA of the cluster
// adds all S partials (read through distributed shared memory, in split
// order, so the result does not depend on timing) for its share of the
// tile's tokens.  No global workspace and no atomics.
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>
#include <type_traits>

#include "internal.h"
#include "pipeline.cuh"
#include "sm100.cuh"

namespace dq {
namespace {

constexpr int HQ_THREADS = 704;
constexpr int HQ_DEQ_WARPS = 8;            // per group: warps 2..9 and 10..17
constexpr int HQ_EPI_WARP0 = 18;           // warps 18..21
constexpr int HQ_EPI_WARPS = 4;
constexpr int HQ_EPI_BUF = 2048;           // 32 tokens x 64 B; two per epilogue warp
constexpr int HQ_BK = 64;                  // contraction elements per step (128 B of bf16)
constexpr int HQ_A_BYTES = 128 * 128;      // dequantized weight tile: 128 rows x 128 B
constexpr int HQ_W_BYTES = 4096;           // packed int4 tile per step
constexpr int HQ_MAX_NP = 16;
constexpr int HQ_ACC_COLS = 256;           // TMEM columns per accumulator buffer
constexpr int HQ_TMEM_COLS = 512;          // two accumulator buffers
constexpr int HQ_SMEM_LIMIT = 227 * 1024;
constexpr int HQ_BAR_BYTES = 1024;

struct HqqArgs {
  int M;                  // tokens
  int n_out;              // output channels (N forward, K transposed)
  int kc;                 // contraction length (K forward, N transposed)
  int n_w, k_w;           // weight rows (N) and in-features (K)
  int group_log2;         // log2 of the group size (32 .. 256)
  int bn;                 // tokens per tile (multiple of 16, <= 256)
  int nt, tt;             // channel tiles (128 each), token tiles (bn each)
  int splits;             // contraction splits per tile
  int ks;                 // contraction steps per tile (ceil(kc / 64))
  int units;              // nt * tt * splits
  int np;                 // packed / activation ring stages
  uint32_t off_epi;       // shared-memory offset of the epilogue staging buffers (after the stages)
  uint32_t off_bar;       // shared-memory offset of the barriers (after the staging buffers)
  const uint16_t* scale;  // bf16 [K / group, n_w], group-major
  const uint16_t* zero;   // bf16 [K / group, n_w]
  uint16_t* out;          // bf16 [M, n_out]
  WaitCtl wait;
};

// bf16x2 arithmetic, each lane rounded once to nearest even (sm_90+ PTX).
__device__ __forceinline__ uint32_t bsub2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t bmul2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// bf16 bit patterns of 128 + c for a code nibble c put in the low mantissa
// bits (exact: the bf16 spacing at 128 is 1).  s4 codes are first offset by
// 8 (nibble ^ 8 = c + 8), so the exact subtraction takes 136 instead.
template <bool S4>
__device__ __forceinline__ uint32_t code_bias2() {
  return S4 ? 0x43084308u : 0x43004300u;
}

// Dequantizes the eight codes of one packed word (byte j = codes 2j, 2j+1
// in its low / high nibble) sharing one zero point and one scale (z2, s2:
// the bf16 pattern in both halves).  o[i] = bf16 pair (code 2i, code 2i+1).
template <bool S4>
__device__ __forceinline__ void dequant8(uint32_t w, uint32_t z2, uint32_t s2, uint32_t (&o)[4]) {
  if (S4) w ^= 0x88888888u;
  // nibbles at bit 0 and bit 16 of each shifted copy: codes (0,4) (1,5) (2,6) (3,7)
  uint32_t d[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t p = ((w >> (4 * i)) & 0x000F000Fu) | 0x43004300u;
    const uint32_t q = bsub2(p, code_bias2<S4>());          // exact: the codes as bf16
    d[i] = bmul2(bsub2(q, z2), s2);                         // bf16(bf16(q - z) * s)
  }
  o[0] = __byte_perm(d[0], d[1], 0x5410);   // codes 0, 1
  o[1] = __byte_perm(d[2], d[3], 0x5410);   // codes 2, 3
  o[2] = __byte_perm(d[0], d[1], 0x7632);   // codes 4, 5
  o[3] = __byte_perm(d[2], d[3], 0x7632);   // codes 6, 7
}

__device__ __forceinline__ uint32_t bf16_pair_of(uint16_t v) {
  return static_cast<uint32_t>(v) | (static_cast<uint32_t>(v) << 16);
}

// Instruction descriptor for kind::f16 with bf16 A and B, fp32 accumulator,
// both operands K-major, shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4)                                 // D format: f32
         | (1u << 7) | (1u << 10)                  // A, B format: bf16
         | (static_cast<uint32_t>(N >> 3) << 17)   // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);  // M / 16
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// A dequantizing thread's scales and zero points for one step, as loaded
// (zero where the channel or in-feature lies outside the weight or there is
// no step): forward one channel's s and z (bf16 bits) for its 32 codes;
// transposed eight weight rows' values (bf16 pairs) for each of its two byte
// columns.  The loads are predicated inline loads into the registers that
// hold them until use: any instruction that read or selected a loaded value
// here would wait for the load.
struct MetaFwd {
  uint32_t s, z;
};
// Forward with two 64-deep sub-tiles per step: one (s, z) per sub-tile.
struct MetaFwd2 {
  MetaFwd m[2];
};
struct MetaT {
  uint4 s8[2], z8[2];
};

__device__ __forceinline__ void ldg_u16_or0(uint32_t& v, const uint16_t* p, bool pred) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %1, 0;\n\tmov.b32 %0, 0;\n\t@q ld.global.nc.u16 %0, [%2];\n\t}"
      : "=r"(v)
      : "r"(static_cast<int>(pred)), "l"(p));
}
__device__ __forceinline__ void ldg_v4_or0(uint4& v, const uint16_t* p, bool pred) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %4, 0;\n\tmov.b32 %0, 0;\n\tmov.b32 %1, 0;\n\tmov.b32 %2, 0;\n\t"
      "mov.b32 %3, 0;\n\t@q ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%5];\n\t}"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "r"(static_cast<int>(pred)), "l"(p));
}

// Forward: thread t handles row t % 128 and codes 32 * (t / 128) .. +31 of
// the step, all inside one group (group sizes are >= 32).
__device__ __forceinline__ void load_meta_fwd(const HqqArgs& g, int dt, bool valid, int ntile, int kstep,
                                              MetaFwd& m) {
  const int n = ntile * 128 + (dt & 127);
  const int k = kstep * HQ_BK + (dt >> 7) * 32;   // kstep: 64-deep sub-tile index
  const bool in = valid && n < g.n_w && k < g.k_w;
  const int64_t gi = in ? static_cast<int64_t>(k >> g.group_log2) * g.n_w + n : 0;
  ldg_u16_or0(m.s, g.scale + gi, in);
  ldg_u16_or0(m.z, g.zero + gi, in);
}

// Transposed: warp w of the dequantizers handles weight rows n0 = 64 *
// kstep + 8 w .. +7 (16 contiguous bytes of a group row: n_w % 8 == 0, so
// the eight rows are all inside or all outside), lane l the output channels
// k = 2 b, 2 b + 1 for b = l and l + 32 (one group: groups are >= 32 wide
// and start at even k).
__device__ __forceinline__ void load_meta_t(const HqqArgs& g, int dt, bool valid, int ntile, int kstep, MetaT& m) {
  const int n0 = kstep * HQ_BK + (dt >> 5) * 8;
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int k = ntile * 128 + 2 * ((dt & 31) + 32 * u);
    const bool in = valid && n0 < g.n_w && k < g.k_w;
    const int64_t gi = in ? static_cast<int64_t>(k >> g.group_log2) * g.n_w + n0 : 0;
    ldg_v4_or0(m.s8[u], g.scale + gi, in);
    ldg_v4_or0(m.z8[u], g.zero + gi, in);
  }
}

// Forward: 256 threads turn the packed tile (128 channel rows x 32 B = 64
// codes) into the 128 x 64 bf16 A tile (thread t: row t % 128, codes
// 32 * (t / 128) .. +31).
template <bool S4>
__device__ __forceinline__ void dequant_tile_fwd(uint32_t atile, uint32_t wtile, int dt, const MetaFwd& m,
                                                 int wrow = 32) {
  const int r = dt & 127;
  const int h = dt >> 7;
  const uint4 pk = pipe::lds128(wtile + r * wrow + h * 16);
  const uint32_t s2 = m.s | (m.s << 16);
  const uint32_t z2 = m.z | (m.z << 16);
  const uint32_t words[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t o[4];
    dequant8<S4>(words[i], z2, s2, o);
    pipe::sts128(atile + pipe::sw128_off(r, 4 * h + i), o[0], o[1], o[2], o[3]);
  }
}

// Transposed: the packed tile holds 64 contraction rows (weight rows n) x
// 64 B (128 output channels k, two per byte); the A tile is 128 rows (k) x
// 64 bf16 (n).  Warp w handles n = 8w .. 8w+7; lane l the byte columns l and
// l + 32 (A rows 2l, 2l+1 and 2l+64, 2l+65): eight bytes from eight weight
// rows give two 16-byte chunks, one per A row.  The eight rows' scales and
// zero points (16 contiguous bytes of a group row each) are the bf16 pairs
// the packed arithmetic needs.
template <bool S4>
__device__ __forceinline__ void dequant_tile_t(uint32_t atile, uint32_t wtile, int dt, const MetaT& m) {
  const int nc = dt >> 5;       // n chunk (8 weight rows)
  const int lane = dt & 31;
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int b = lane + 32 * u;                 // byte column: k = 2b, 2b + 1 in the tile
    const uint32_t sp[4] = {m.s8[u].x, m.s8[u].y, m.s8[u].z, m.s8[u].w};
    const uint32_t zp[4] = {m.z8[u].x, m.z8[u].y, m.z8[u].z, m.z8[u].w};
    uint32_t lo[4], hi[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      // weight rows n0 + 2i and n0 + 2i + 1
      const uint32_t b0 = pipe::lds8(wtile + (nc * 8 + 2 * i) * 64 + b);
      const uint32_t b1 = pipe::lds8(wtile + (nc * 8 + 2 * i + 1) * 64 + b);
      uint32_t x = b0 | (b1 << 16);
      if (S4) x ^= 0x00880088u;
      const uint32_t pl = (x & 0x000F000Fu) | 0x43004300u;          // k = 2b: rows 2i, 2i + 1
      const uint32_t ph = ((x >> 4) & 0x000F000Fu) | 0x43004300u;   // k = 2b + 1
      lo[i] = bmul2(bsub2(bsub2(pl, code_bias2<S4>()), zp[i]), sp[i]);
      hi[i] = bmul2(bsub2(bsub2(ph, code_bias2<S4>()), zp[i]), sp[i]);
    }
    pipe::sts128(atile + pipe::sw128_off(2 * b, nc), lo[0], lo[1], lo[2], lo[3]);
    pipe::sts128(atile + pipe::sw128_off(2 * b + 1, nc), hi[0], hi[1], hi[2], hi[3]);
  }
}

struct Unit {
  int tile, split, ntile, ttile, k0, k1;
};

// Work unit u: tile = u / splits (channel tile major, token tile minor),
// contraction steps [k0, k1) of split u % splits.
__device__ __forceinline__ Unit decode_unit(const HqqArgs& g, int u) {
  Unit t;
  t.tile = u / g.splits;
  t.split = u - t.tile * g.splits;
  t.ntile = t.tile / g.tt;
  t.ttile = t.tile - t.ntile * g.tt;
  t.k0 = static_cast<int>(static_cast<int64_t>(t.split) * g.ks / g.splits);
  t.k1 = static_cast<int>(static_cast<int64_t>(t.split + 1) * g.ks / g.splits);
  return t;
}

// The CTA's contraction steps in order, across its units: (ntile, kk).
struct StepIt {
  int u, kk, k1, ntile;
  bool valid;
  __device__ __forceinline__ void start(const HqqArgs& g, int u0) {
    u = u0;
    valid = false;
    for (; u < g.units; u += gridDim.x) {
      const Unit t = decode_unit(g, u);
      if (t.k0 < t.k1) {
        kk = t.k0;
        k1 = t.k1;
        ntile = t.ntile;
        valid = true;
        return;
      }
    }
  }
  __device__ __forceinline__ void next(const HqqArgs& g) {
    if (!valid) return;
    if (++kk < k1) return;
    start(g, u + gridDim.x);
  }
};

__device__ __forceinline__ uint32_t bf16_bits(float f) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(f)));
}

// Converts `width` (16 or 32) fp32 accumulators of one output channel per
// lane to bf16 pairs and stages them (row j = token j of a 32 x 32 block).
__device__ __forceinline__ void stage_pairs(uint32_t buf, const uint32_t (&r)[32], int width, int lane) {
  uint32_t pk[16];
#pragma unroll
  for (int i = 0; i < 16; ++i)
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(pk[i]) : "f"(__uint_as_float(r[2 * i + 1])), "f"(__uint_as_float(r[2 * i])));
  pipe::stage_bf16_pairs(buf, pk, width, lane);
}

// SUB: 64-deep sub-tiles per contraction step (forward, few tokens: 2, so
// that each copy, barrier and hand-off serves 128 in-features; else 1).
template <bool TRANS, bool S4, int SUB = 1>
__global__ void __launch_bounds__(HQ_THREADS, 1)
    hqq_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                    const __grid_constant__ CUtensorMap tm_c32, const __grid_constant__ CUtensorMap tm_c16,
                    const HqqArgs g) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const smem = smem_raw + (base - raw);
  // stage s at base + s * stage_bytes: SUB dequantized A tiles (16 KB each),
  // then SUB activation tiles (bn x 128 B each), then the packed weight tile
  // (128 rows x 32 SUB bytes forward)
  static_assert(SUB == 1 || (SUB == 2 && !TRANS), "two sub-tiles per step: forward only");
  const uint32_t x_sub = static_cast<uint32_t>(g.bn) * 128u;
  const uint32_t x_bytes = x_sub * SUB;
  const uint32_t stage_bytes = HQ_A_BYTES * SUB + x_bytes + HQ_W_BYTES * SUB;
  uint64_t* const full = reinterpret_cast<uint64_t*>(smem + g.off_bar);   // TMA landed
  uint64_t* const deq = full + HQ_MAX_NP;                                 // A tile written
  uint64_t* const empty = deq + HQ_MAX_NP;                                // MMAs done with the stage
  uint64_t* const accf = empty + HQ_MAX_NP;
  uint64_t* const acce = accf + 2;
  uint64_t* const drain = acce + 2;
  uint32_t* const tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < g.np; ++i) {
      mbar_init(smem_u32(full + i), 1);
      mbar_init(smem_u32(deq + i), HQ_DEQ_WARPS);
      mbar_init(smem_u32(empty + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(accf + i), 1);
      mbar_init(smem_u32(acce + i), HQ_EPI_WARPS);
    }
    mbar_init(smem_u32(drain), 1);
    fence_barrier_init();
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), HQ_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // With a programmatic (early) launch, the previous kernel of the stream is
  // complete before any global memory is touched.
  griddep_wait();

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < g.units; u += gridDim.x) {
        const Unit t = decode_unit(g, u);
        for (int kk = t.k0; kk < t.k1; ++kk) {
          if (!pipe::wait(smem_u32(empty + stage), phase ^ 1, g.wait, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(full + stage);
          const uint32_t sx = base + stage * stage_bytes + HQ_A_BYTES * SUB;
          const uint32_t sw = sx + x_bytes;
          mbar_arrive_expect_tx(fb, x_bytes + HQ_W_BYTES * SUB);
#pragma unroll
          for (int sb = 0; sb < SUB; ++sb)
            tma_load_2d(sx + sb * x_sub, &tm_x, fb, (kk * SUB + sb) * 128, t.ttile * g.bn);
          if (TRANS)
            tma_load_2d(sw, &tm_w, fb, t.ntile * 64, kk * HQ_BK);
          else
            tma_load_2d(sw, &tm_w, fb, kk * 32 * SUB, t.ntile * 128);
          ++issued;
          if (++stage == g.np) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // every copy issued lands before the CTA can exit
      volatile int never = 0;
      for (long long i = issued > g.np ? issued - g.np : 0; i < issued; ++i)
        pipe::wait(smem_u32(full + static_cast<int>(i % g.np)), static_cast<uint32_t>((i / g.np) & 1), g.wait,
                &never);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, g.bn);
      int stage = 0, acc = 0;
      uint32_t phase = 0, aphase = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < g.units; u += gridDim.x) {
        const Unit t = decode_unit(g, u);
        if (!pipe::wait(smem_u32(acce + acc), aphase ^ 1, g.wait, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * HQ_ACC_COLS);
        for (int kk = t.k0; kk < t.k1; ++kk) {
          // the dequantizers waited for the copies, so deq implies full
          if (!pipe::wait(smem_u32(deq + stage), phase, g.wait, abort_flag) ||
              !pipe::wait(smem_u32(full + stage), phase, g.wait, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = base + stage * stage_bytes;
#pragma unroll
          for (int sb = 0; sb < SUB; ++sb) {
            const uint64_t ad = smem_desc_kmajor<128>(sa + sb * HQ_A_BYTES);
            const uint64_t bd = smem_desc_kmajor<128>(sa + HQ_A_BYTES * SUB + sb * x_sub);
#pragma unroll
            for (int j = 0; j < 4; ++j)   // K = 16 bf16 = 32 bytes per instruction
              mma_bf16(d_tmem, ad + 2 * j, bd + 2 * j, idesc, (kk > t.k0 || sb > 0 || j > 0) ? 1u : 0u);
          }
          mma_commit(smem_u32(empty + stage));
          if (++stage == g.np) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        mma_commit(smem_u32(accf + acc));
        if (++acc == 2) {
          acc = 0;
          aphase ^= 1;
        }
      }
      // every MMA issued has completed once drain flips
      mma_commit(smem_u32(drain));
      volatile int never = 0;
      pipe::wait(smem_u32(drain), 0, g.wait, &never);
    }
  } else if (warp < HQ_EPI_WARP0) {
    // ---------------------------------------------------------- dequantizers
    // A stage's A tile is free again once its copies have landed: the
    // producer refilled the stage only after the MMAs that read it completed.
    // Each thread's scales and zero points are loaded two steps ahead of use.
    using Meta = typename std::conditional<TRANS, MetaT, typename std::conditional<SUB == 2, MetaFwd2, MetaFwd>::type>::type;
    const int dt = (threadIdx.x - 64) & 255;
    const int grp = (threadIdx.x - 64) >> 8;     // group 1 takes the odd steps
    auto load_meta = [&](const StepIt& s, Meta& m) {
      if constexpr (TRANS) {
        load_meta_t(g, dt, s.valid, s.ntile, s.kk, m);
      } else if constexpr (SUB == 2) {
        load_meta_fwd(g, dt, s.valid, s.ntile, 2 * s.kk, m.m[0]);
        load_meta_fwd(g, dt, s.valid, s.ntile, 2 * s.kk + 1, m.m[1]);
      } else {
        load_meta_fwd(g, dt, s.valid, s.ntile, s.kk, m);
      }
    };
    // cur: this group's step; ahead: the group's step two of its own later
    StepIt cur, ahead;
    cur.start(g, blockIdx.x);
    if (grp) cur.next(g);
    ahead = cur;
    for (int i = 0; i < 4; ++i) ahead.next(g);
    int stage = grp;
    uint32_t phase = 0;
    if (stage >= g.np) {    // np >= 2: never, kept for clarity
      stage -= g.np;
      phase ^= 1;
    }
    // One step: `use` holds this step's values; the values of the step two
    // ahead are loaded into `fill` (free since the previous step).  Three
    // sets rotate by name, so no register is copied while its load is in
    // flight (a copy would wait for the load).
    auto step = [&](const Meta& use, Meta& fill) -> bool {
      if (!cur.valid) return false;
      load_meta(ahead, fill);
      const bool w = pipe::wait(smem_u32(full + stage), phase, g.wait, abort_flag);
      if (!__all_sync(0xffffffffu, w)) return false;
      const uint32_t sa = base + stage * stage_bytes;
      const uint32_t wt = sa + HQ_A_BYTES * SUB + x_bytes;
      if constexpr (TRANS) {
        dequant_tile_t<S4>(sa, wt, dt, use);
      } else if constexpr (SUB == 2) {
        dequant_tile_fwd<S4>(sa, wt, dt, use.m[0], 64);
        dequant_tile_fwd<S4>(sa + HQ_A_BYTES, wt + 32, dt, use.m[1], 64);
      } else {
        dequant_tile_fwd<S4>(sa, wt, dt, use);
      }
      fence_proxy_async_smem();     // generic-proxy writes -> visible to the MMA
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(deq + stage));
      stage += 2;
      if (stage >= g.np) {
        stage -= g.np;
        phase ^= 1;
      }
      cur.next(g);
      cur.next(g);
      ahead.next(g);
      ahead.next(g);
      return true;
    };
    Meta ma, mb, mc;
    load_meta(cur, ma);
    StepIt one = cur;
    one.next(g);
    one.next(g);
    load_meta(one, mb);
    while (step(ma, mc) && step(mb, ma) && step(mc, mb)) {
    }
  } else {
    // ---------------------------------------------------------- epilogue
    const int q = warp & 3;                 // TMEM sub-partition of this warp
    const int row = q * 32 + lane;          // accumulator row = output channel in the tile
    const uint32_t buf0 = base + g.off_epi + static_cast<uint32_t>(warp - HQ_EPI_WARP0) * 2 * HQ_EPI_BUF;
    int acc = 0;
    uint32_t aphase = 0;
    for (int u = blockIdx.x; u < g.units; u += gridDim.x) {
      const Unit t = decode_unit(g, u);
      const bool w = pipe::wait(smem_u32(accf + acc), aphase, g.wait, abort_flag);
      if (!__all_sync(0xffffffffu, w)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * HQ_ACC_COLS);
      const int ch0 = t.ntile * 128 + q * 32;
      const int tok0 = t.ttile * g.bn;
      // One 32-token chunk: with a split contraction the fp32 partial into
      // this CTA's shared memory ([bn][128], at the start of the stage ring:
      // the CTA's only unit, so every stage has been consumed once its
      // accumulator is ready), else bf16 through staging buffer `b` (free
      // once its previous store has read it: at most the other buffer's
      // store may still be reading).
      auto emit = [&](const uint32_t (&r)[32], int c0, int width, uint32_t b) {
        if (g.splits > 1) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < width) pipe::sts32(base + static_cast<uint32_t>((c0 + j) * 128 + row) * 4u, r[j]);
          return;
        }
        if (lane == 0) bulk_wait_group_read<1>();
        __syncwarp();
        stage_pairs(b, r, width, lane);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (ch0 < g.n_out && tok0 + c0 < g.M)      // boxes wholly outside are not issued
            tma_store_2d(width == 32 ? &tm_c32 : &tm_c16, b, 2 * ch0, tok0 + c0);
          bulk_commit_group();                       // (an empty group keeps the count in step)
        }
      };
      auto load = [&](uint32_t (&r)[32], int c0, int width) {
        if (width == 32) {
          tmem_ld_32x32b_x32(tb + c0, r);
        } else {
          uint32_t r16[16];
          tmem_ld_32x32b_x16(tb + c0, r16);
#pragma unroll
          for (int j = 0; j < 16; ++j) r[j] = r16[j];
#pragma unroll
          for (int j = 16; j < 32; ++j) r[j] = 0;
        }
      };
      for (int c0 = 0; c0 < g.bn; c0 += 64) {
        const int w0 = min(32, g.bn - c0);
        const int w1 = min(32, g.bn - c0 - 32);     // <= 0: no second chunk
        uint32_t r0[32], r1[32];
        load(r0, c0, w0);
        if (w1 > 0) load(r1, c0 + 32, w1);
        tmem_ld_wait();
        emit(r0, c0, w0, buf0);
        if (w1 > 0) emit(r1, c0 + 32, w1, buf0 + HQ_EPI_BUF);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(acce + acc));
      if (++acc == 2) {
        acc = 0;
        aphase ^= 1;
      }
    }
    if (lane == 0) bulk_wait_group<0>();         // every output store complete
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, HQ_TMEM_COLS);

  // Split contraction (one unit per CTA, the tile's S splits one cluster):
  // once every CTA of the cluster holds its partial tile, CTA r adds all S
  // partials for tokens [r * rows, (r + 1) * rows) of the tile, four
  // channels per thread, and stores them as bf16.  The second cluster
  // barrier keeps every CTA's shared memory alive until its peers have read
  // it.
  if (g.splits > 1) {
    cluster_sync_all();
    const Unit t = decode_unit(g, blockIdx.x);
    const int rank = static_cast<int>(cluster_ctarank());
    const int rows = (g.bn + g.splits - 1) / g.splits;
    const int r0 = rank * rows;
    const int r1 = min(g.bn, r0 + rows);
    for (int i = threadIdx.x; i < (r1 - r0) * 32; i += HQ_THREADS) {
      const int tok = r0 + (i >> 5);
      const int quad = i & 31;                        // channels 4 * quad .. + 3 of the tile
      const uint32_t off = base + static_cast<uint32_t>(tok * 128 + 4 * quad) * 4u;
      float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int sp = 0; sp < g.splits; ++sp) {
        const float4 v = ld_shared_cluster_f4(map_to_rank(off, static_cast<uint32_t>(sp)));
        sum.x += v.x;
        sum.y += v.y;
        sum.z += v.z;
        sum.w += v.w;
      }
      const int m = t.ttile * g.bn + tok;
      const int ch = t.ntile * 128 + 4 * quad;
      if (m < g.M && ch < g.n_out) {                  // n_out % 8 == 0: the quad is all in or all out
        const uint32_t lo = bf16_bits(sum.x) | (bf16_bits(sum.y) << 16);
        const uint32_t hi = bf16_bits(sum.z) | (bf16_bits(sum.w) << 16);
        *reinterpret_cast<uint2*>(g.out + static_cast<int64_t>(m) * g.n_out + ch) = make_uint2(lo, hi);
      }
    }
    cluster_sync_all();
  }
}

// Standalone dequantization: one thread per packed word (8 codes) -> 16 B of
// bf16.  Scales and zero points group-major ([K / group, N]).
template <bool S4>
__global__ void __launch_bounds__(256) hqq_dequant_kernel(const uint32_t* __restrict__ packed,
                                                          const uint16_t* __restrict__ scale,
                                                          const uint16_t* __restrict__ zero, int64_t N,
                                                          int64_t K, int group, uint16_t* __restrict__ w) {
  const int64_t words_per_row = K / 8;
  const int64_t total = N * words_per_row;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = i / words_per_row;
    const int64_t k = (i - n * words_per_row) * 8;
    const int64_t gi = (k / group) * N + n;
    uint32_t o[4];
    dequant8<S4>(__ldg(packed + i), bf16_pair_of(__ldg(zero + gi)), bf16_pair_of(__ldg(scale + gi)), o);
    *reinterpret_cast<uint4*>(w + n * K + k) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// [rows, cols] -> [cols, rows] for 16-bit elements, through a 32 x 33 tile.
__global__ void __launch_bounds__(256) transpose16_kernel(const uint16_t* __restrict__ src, int64_t rows,
                                                          int64_t cols, uint16_t* __restrict__ dst) {
  __shared__ uint16_t tile[32][33];
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * 32, c0 = static_cast<int64_t>(blockIdx.x) * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;     // 32 x 8 threads
  for (int i = ty; i < 32; i += 8) {
    const int64_t r = r0 + i, c = c0 + tx;
    if (r < rows && c < cols) tile[i][tx] = src[r * cols + c];
  }
  __syncthreads();
  for (int i = ty; i < 32; i += 8) {
    const int64_t c = c0 + i, r = r0 + tx;
    if (r < rows && c < cols) dst[c * rows + r] = tile[tx][i];
  }
}

__global__ void __launch_bounds__(256) hqq_pack_kernel(const int8_t* __restrict__ codes, int64_t n_bytes,
                                                       uint8_t* __restrict__ packed) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n_bytes;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint32_t lo = static_cast<uint8_t>(codes[2 * i]) & 0x0Fu;
    const uint32_t hi = static_cast<uint8_t>(codes[2 * i + 1]) & 0x0Fu;
    packed[i] = static_cast<uint8_t>(lo | (hi << 4));
  }
}

}  // namespace
}  // namespace dq

// ---------------------------------------------------------------- host side

namespace dq {
namespace {

struct HqqPlan {
  int bn, tt, nt, ks, splits, units, grid, np;
  size_t smem;
};

constexpr int HQ_MAX_SPLITS = 8;           // portable cluster size

// Tiles: 128 output channels x bn tokens, bn = the token count split evenly
// over ceil(M / 256) tiles and rounded up to 16.  When the tiles cannot fill
// the SMs the contraction is split over a cluster of up to 8 CTAs (at least
// 4 steps of 64 per split; the partial tile, bn x 128 fp32, must fit in the
// stage ring).
HqqPlan plan_hqq(int64_t M, int64_t n_out, int64_t kc, int sm_count, bool allow_split, int sub = 1) {
  HqqPlan p{};
  p.nt = static_cast<int>((n_out + 127) / 128);
  p.ks = static_cast<int>((kc + HQ_BK * sub - 1) / (HQ_BK * sub));
  p.tt = static_cast<int>((M + 255) / 256);
  const int64_t per = (M + p.tt - 1) / p.tt;
  p.bn = static_cast<int>(std::max<int64_t>(16, (per + 15) / 16 * 16));
  const int64_t tiles = static_cast<int64_t>(p.nt) * p.tt;
  p.splits = 1;
  if (allow_split && tiles < sm_count) {
    int s = static_cast<int>(sm_count / tiles);
    s = std::min(s, std::max(1, p.ks / 4));
    p.splits = std::max(1, std::min(s, HQ_MAX_SPLITS));
  }
  p.units = static_cast<int>(tiles * p.splits);
  p.grid = std::min(p.units, sm_count);
  const int stage = (HQ_A_BYTES + p.bn * 128 + HQ_W_BYTES) * sub;
  const int avail = HQ_SMEM_LIMIT - 1024 - 2 * HQ_EPI_WARPS * HQ_EPI_BUF - HQ_BAR_BYTES;
  p.np = std::min(HQ_MAX_NP, avail / stage);
  p.smem = 1024 + static_cast<size_t>(p.np) * stage + 2 * HQ_EPI_WARPS * HQ_EPI_BUF + HQ_BAR_BYTES;
  if (p.splits > 1 && p.np * stage < p.bn * 128 * 4) {    // no room for the partial tile
    p.splits = 1;
    p.units = static_cast<int>(tiles);
    p.grid = std::min(p.units, sm_count);
  }
  return p;
}

dq_status check_weights(const uint8_t* packed, const void* scale, const void* zero, int64_t N, int64_t K,
                        int group, int flags) {
  if (N <= 0 || K <= 0 || (flags & ~DQ_HQQ_S4) != 0) return DQ_ERR_INVALID_ARG;
  if (group != 32 && group != 64 && group != 128 && group != 256) return DQ_ERR_INVALID_ARG;
  if (K % group != 0) return DQ_ERR_INVALID_ARG;
  if (N % 8 != 0) return DQ_ERR_UNSUPPORTED;
  if (N > (int64_t{1} << 30) || K > (int64_t{1} << 30)) return DQ_ERR_UNSUPPORTED;
  if (packed == nullptr || scale == nullptr || zero == nullptr) return DQ_ERR_INVALID_ARG;
  if (!aligned(packed, 16) || !aligned(scale, 16) || !aligned(zero, 16)) return DQ_ERR_UNSUPPORTED;
  return DQ_OK;
}

template <bool TRANS, bool S4, int SUB = 1>
dq_status launch_hqq(const CUtensorMap& tx, const CUtensorMap& tw, const CUtensorMap& tc32, const CUtensorMap& tc16,
                     const HqqArgs& g, int grid, size_t smem, cudaStream_t stream) {
  const dq_status st =
      smem_limit_once(reinterpret_cast<const void*>(&hqq_gemm_kernel<TRANS, S4, SUB>), HQ_SMEM_LIMIT);
  if (st != DQ_OK) return st;
  // Programmatic stream serialization: the prologue (barriers, tensor-memory
  // allocation) overlaps the tail of the previous kernel of the stream.  A
  // split contraction runs each tile's splits as one cluster.
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = static_cast<unsigned>(g.splits);
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(HQ_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = g.splits > 1 ? 2 : 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, hqq_gemm_kernel<TRANS, S4, SUB>, tx, tw, tc32, tc16, g);
  return e == cudaSuccess ? DQ_OK : cuda_fail(e);
}

std::atomic<int> g_cluster_ok[64] = {};   // per device: 0 unknown, 1 yes, 2 no

// Whether a cluster of HQ_MAX_SPLITS CTAs with a full SM's shared memory
// each can be resident on the current device (then every smaller split
// cluster can too).  Asked once per device.
bool split_clusters_fit(const DeviceInfo& d) {
  int v = g_cluster_ok[d.device & 63].load(std::memory_order_relaxed);
  if (v == 0) {
    v = 2;
    if (smem_limit_once(reinterpret_cast<const void*>(&hqq_gemm_kernel<false, false>), HQ_SMEM_LIMIT) == DQ_OK) {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = HQ_MAX_SPLITS;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(HQ_MAX_SPLITS);
      cfg.blockDim = dim3(HQ_THREADS);
      cfg.dynamicSmemBytes = HQ_SMEM_LIMIT;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, hqq_gemm_kernel<false, false>, &cfg) == cudaSuccess && n >= 1) v = 1;
      else (void)cudaGetLastError();
    }
    g_cluster_ok[d.device & 63].store(v, std::memory_order_relaxed);
  }
  return v == 1;
}

dq_status hqq_linear_impl(bool trans, const void* x, int64_t M, const uint8_t* packed, const void* scale,
                          const void* zero, int64_t N, int64_t K, int group, int flags, void* out,
                          void* workspace, size_t workspace_bytes, dq_stream_t stream) {
  dq_status st = check_weights(packed, scale, zero, N, K, group, flags);
  if (st != DQ_OK) return st;
  if (M < 0) return DQ_ERR_INVALID_ARG;
  if (M > (int64_t{1} << 30)) return DQ_ERR_UNSUPPORTED;
  if (M == 0) return DQ_OK;
  if (x == nullptr || out == nullptr) return DQ_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(out, 16)) return DQ_ERR_UNSUPPORTED;
  DeviceInfo* d = nullptr;
  if ((st = current_device(&d)) != DQ_OK) return st;

  const int64_t n_out = trans ? K : N;
  const int64_t kc = trans ? N : K;
  (void)workspace;          // kept for the interface: the split contraction needs none
  (void)workspace_bytes;
  // Few tokens (forward): 128-deep steps of two 64-deep sub-tiles, half the
  // copies, barrier waits and hand-offs per in-feature.
  const int sub = (!trans && M <= 64) ? 2 : 1;
  const HqqPlan p = plan_hqq(M, n_out, kc, d->sm_count, split_clusters_fit(*d), sub);

  CUtensorMap tx, tw;
  // activations / output gradient: bf16 [M, kc] as bytes, 64-element k
  // slices of bn rows, 128B-swizzled (the MMA's K-major B layout)
  st = make_tmap_u8_2d(&tx, x, static_cast<uint64_t>(kc) * 2, static_cast<uint64_t>(M),
                       static_cast<uint64_t>(kc) * 2, 128, static_cast<uint32_t>(p.bn), 128);
  if (st != DQ_OK) return st;
  // packed codes [N, K/2]: forward 128 channels x 32 B (64 k); transposed
  // 64 weight rows x 64 B (128 output channels k)
  st = make_tmap_u8_2d(&tw, packed, static_cast<uint64_t>(K / 2), static_cast<uint64_t>(N),
                       static_cast<uint64_t>(K / 2), trans ? 64 : 32 * sub, trans ? 64 : 128, 0);
  if (st != DQ_OK) return st;

  // output bf16 [M, n_out] as bytes: 32 channels (64 B) x 32 or 16 tokens
  CUtensorMap tc32, tc16;
  st = make_tmap_u8_2d(&tc32, out, static_cast<uint64_t>(n_out) * 2, static_cast<uint64_t>(M),
                       static_cast<uint64_t>(n_out) * 2, 64, 32, 0);
  if (st != DQ_OK) return st;
  st = make_tmap_u8_2d(&tc16, out, static_cast<uint64_t>(n_out) * 2, static_cast<uint64_t>(M),
                       static_cast<uint64_t>(n_out) * 2, 64, 16, 0);
  if (st != DQ_OK) return st;

  HqqArgs g{};
  g.M = static_cast<int>(M);
  g.n_out = static_cast<int>(n_out);
  g.kc = static_cast<int>(kc);
  g.n_w = static_cast<int>(N);
  g.k_w = static_cast<int>(K);
  g.group_log2 = group == 32 ? 5 : group == 64 ? 6 : group == 128 ? 7 : 8;
  g.bn = p.bn;
  g.nt = p.nt;
  g.tt = p.tt;
  g.splits = p.splits;
  g.ks = p.ks;
  g.units = p.units;
  g.np = p.np;
  g.off_epi = static_cast<uint32_t>(p.np) * (HQ_A_BYTES + p.bn * 128 + HQ_W_BYTES) * sub;
  g.off_bar = g.off_epi + 2 * HQ_EPI_WARPS * HQ_EPI_BUF;
  g.scale = static_cast<const uint16_t*>(scale);
  g.zero = static_cast<const uint16_t*>(zero);
  g.out = static_cast<uint16_t*>(out);
  g.wait = WaitCtl{d->err_word, wait_timeout_ns()};
  const bool s4 = (flags & DQ_HQQ_S4) != 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (trans) return s4 ? launch_hqq<true, true>(tx, tw, tc32, tc16, g, p.grid, p.smem, s)
                       : launch_hqq<true, false>(tx, tw, tc32, tc16, g, p.grid, p.smem, s);
  if (sub == 2)
    return s4 ? launch_hqq<false, true, 2>(tx, tw, tc32, tc16, g, p.grid, p.smem, s)
              : launch_hqq<false, false, 2>(tx, tw, tc32, tc16, g, p.grid, p.smem, s);
  return s4 ? launch_hqq<false, true>(tx, tw, tc32, tc16, g, p.grid, p.smem, s)
            : launch_hqq<false, false>(tx, tw, tc32, tc16, g, p.grid, p.smem, s);
}

int grid_for(int64_t items, int sm_count) {
  const int64_t blocks = (items + 255) / 256;
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(blocks, static_cast<int64_t>(sm_count) * 16)));
}

}  // namespace
}  // namespace dq

using namespace dq;

extern "C" {

DQ_API dq_status dq_hqq_pack(const int8_t* codes, int64_t rows, int64_t cols, uint8_t* packed,
                             dq_stream_t stream) {
  if (rows < 0 || cols < 0 || (cols & 1) != 0) return DQ_ERR_INVALID_ARG;
  if (rows == 0 || cols == 0) return DQ_OK;
  if (codes == nullptr || packed == nullptr) return DQ_ERR_INVALID_ARG;
  DeviceInfo* d = nullptr;
  dq_status st = current_device(&d);
  if (st != DQ_OK) return st;
  const int64_t n_bytes = rows * (cols / 2);
  hqq_pack_kernel<<<grid_for(n_bytes, d->sm_count), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      codes, n_bytes, packed);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? DQ_OK : cuda_fail(e);
}

DQ_API dq_status dq_hqq_dequantize(const uint8_t* packed, const void* scale_bf16, const void* zero_bf16,
                                   int64_t N, int64_t K, int group, int flags, void* w_bf16,
                                   dq_stream_t stream) {
  dq_status st = check_weights(packed, scale_bf16, zero_bf16, N, K, group, flags);
  if (st != DQ_OK) return st;
  if (w_bf16 == nullptr) return DQ_ERR_INVALID_ARG;
  if (!aligned(w_bf16, 16)) return DQ_ERR_UNSUPPORTED;
  DeviceInfo* d = nullptr;
  if ((st = current_device(&d)) != DQ_OK) return st;
  const int64_t words = N * (K / 8);
  const auto* pw = reinterpret_cast<const uint32_t*>(packed);
  const auto* sc = static_cast<const uint16_t*>(scale_bf16);
  const auto* ze = static_cast<const uint16_t*>(zero_bf16);
  auto* w = static_cast<uint16_t*>(w_bf16);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (flags & DQ_HQQ_S4)
    hqq_dequant_kernel<true><<<grid_for(words, d->sm_count), 256, 0, s>>>(pw, sc, ze, N, K, group, w);
  else
    hqq_dequant_kernel<false><<<grid_for(words, d->sm_count), 256, 0, s>>>(pw, sc, ze, N, K, group, w);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? DQ_OK : cuda_fail(e);
}

DQ_API dq_status dq_hqq_group_major(const void* src_bf16, int64_t N, int64_t G, void* dst_bf16,
                                    dq_stream_t stream) {
  if (N < 0 || G < 0) return DQ_ERR_INVALID_ARG;
  if (N == 0 || G == 0) return DQ_OK;
  if (src_bf16 == nullptr || dst_bf16 == nullptr || N > (int64_t{1} << 30) || G > (int64_t{1} << 30))
    return DQ_ERR_INVALID_ARG;
  DeviceInfo* d = nullptr;
  dq_status st = current_device(&d);
  if (st != DQ_OK) return st;
  if ((G + 31) / 32 > 2147483647 || (N + 31) / 32 > 65535) return DQ_ERR_UNSUPPORTED;
  const dim3 grid(static_cast<unsigned>((G + 31) / 32), static_cast<unsigned>((N + 31) / 32));
  transpose16_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint16_t*>(src_bf16), N, G, static_cast<uint16_t*>(dst_bf16));
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? DQ_OK : cuda_fail(e);
}

// The split contraction reduces through distributed shared memory: no call
// needs a workspace (the query stays for the interface).
DQ_API size_t dq_hqq_workspace_size(int64_t M, int64_t N, int64_t K, int transposed) {
  (void)M;
  (void)N;
  (void)K;
  (void)transposed;
  return 0;
}

DQ_API dq_status dq_hqq_linear(const void* x_bf16, int64_t M, const uint8_t* packed, const void* scale_bf16,
                               const void* zero_bf16, int64_t N, int64_t K, int group, int flags,
                               void* out_bf16, void* workspace, size_t workspace_bytes, dq_stream_t stream) {
  return hqq_linear_impl(false, x_bf16, M, packed, scale_bf16, zero_bf16, N, K, group, flags, out_bf16,
                         workspace, workspace_bytes, stream);
}

DQ_API dq_status dq_hqq_linear_t(const void* y_bf16, int64_t M, const uint8_t* packed, const void* scale_bf16,
                                 const void* zero_bf16, int64_t N, int64_t K, int group, int flags,
                                 void* out_bf16, void* workspace, size_t workspace_bytes, dq_stream_t stream) {
  return hqq_linear_impl(true, y_bf16, M, packed, scale_bf16, zero_bf16, N, K, group, flags, out_bf16,
                         workspace, workspace_bytes, stream);
}

}  // extern "C"
