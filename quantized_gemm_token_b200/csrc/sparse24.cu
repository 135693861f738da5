// sparse24.cu -- the int8 dynamic-quantization linear layer with a 2:4
// semi-structured sparse weight ("sparse_fc supported", PaddlePaddle PR 41770:
// fully connected layers whose weights keep at most two nonzeros in every
// four consecutive in-features run a 2:4 sparse matmul after the weight is
// compressed on the device; its review asks for the int8 product with only
// the dequantization fused and a 16-bit output, which the library it used
// could not do).  Here the product runs on the sparse tensor-core MMA with
// the dequantization, bias and bf16 conversion fused, and no int32 matrix in
// global memory.
//
// Compressed weight (this library's own format, written by dq_s24_compress):
//   values [N, K/2] int8: the two kept values of each group of four, in
//     position order;
//   meta [N, K/8] uint8: one nibble per group, p0 | p1 << 2 (p0 < p1 the
//     kept positions), group 2b in the low nibble of byte b.
// This is the operand format of tcgen05.mma.sp with 8-bit operands: the
// values are the compressed A matrix as it is, and a 128-channel x 128
// in-feature block of the metadata (128 rows of 16 bytes) is one copy into
// tensor memory that serves two K = 64 MMAs (8 bytes per row each).
//
// One persistent, warp-specialised kernel for sm_100a (320 threads):
//   warp 0      TMA producer: per 128-deep contraction step the quantized
//               activation tile (bn tokens x 128 B, 128B-swizzled), the
//               step's compressed values (128 channel rows x 64 B,
//               64B-swizzled) and metadata (128 x 16 B, unswizzled).
//   warp 1      MMA issuer: tcgen05.cp of the step's metadata into a tensor
//               memory slot of the stage, then two tcgen05.mma.sp kind::i8
//               (M = 128 weight rows, N = bn tokens, logical K = 64 each,
//               int32 accumulator in TMEM, double-buffered).
//   warps 2..9  epilogue, two warps per TMEM sub-partition taking alternate
//               32-token chunks: out = bf16((acc * s_row) * s_col + bias),
//               each op rounded on its own, staged as a 32 x 32 block and
//               written by one TMA store; or the raw int32.
// Few tiles: the contraction is split; int32 partial tiles go to a
// workspace and, per epilogue warp, the last split of a tile to arrive adds
// them (exact, in split order) before the epilogue arithmetic.
// Many tokens (from 1536 with K >= 2048): a 2-SM pair version of the same
// kernel (s24_gemm2_kernel, 256-channel tiles over a cluster of two CTAs,
// each loading its own weight rows and half of the activation tile).
#include <cuda_bf16.h>

#include <algorithm>

#include "internal.h"
#include "pipeline.cuh"
#include "sm100.cuh"

namespace dq {
namespace {

constexpr int S4_THREADS = 320;
constexpr int S4_EPI_WARPS = 8;            // warps 2..9
constexpr int S4_BK = 128;                 // logical in-features per step (two sparse MMAs)
constexpr int S4_V_BYTES = 128 * 64;       // compressed values per step
constexpr int S4_M_BYTES = 128 * 16;       // metadata per step
constexpr int S4_MAX_NP = 16;
constexpr int S4_MAX_BN = 240;             // tokens per tile
// Tensor memory: two accumulators of bn columns at columns 0 and bn, then
// the metadata ring at column 2 * bn, 4 columns per stage (so bn = 240
// leaves room for 8 stages, bn <= 192 for all 16).
constexpr int S4_TMEM_COLS = 512;
constexpr int S4_SMEM_LIMIT = 227 * 1024;
constexpr int S4_BAR_BYTES = 1024;
constexpr int S4_CNT_PER_TILE = 8;         // split arrival counters per tile: one per epilogue warp
constexpr int S4_EPI_BUF = 2048;           // bf16 staging per epilogue warp: 32 tokens x 64 B
static_assert(2 * S4_MAX_BN + 4 * 8 <= S4_TMEM_COLS, "tensor memory");

struct S24Args {
  int M, N, K;
  int bn;                 // tokens per tile (multiple of 16, <= S4_MAX_BN)
  int nt, tt;             // channel tiles (128), token tiles (bn)
  int splits, ks, units, np;
  uint32_t off_epi;       // epilogue staging buffers (after the stages)
  uint32_t off_bar;       // barriers (after the staging buffers)
  const float* s_row;
  const float* s_col;
  const uint16_t* bias;   // bf16 bits or null
  void* out;              // bf16 or int32 [M, N]
  int out_s32;
  int32_t* ws;            // split partials [tile][split][bn][128] int32
  uint32_t* cnt;          // split arrival counters [tile][S4_CNT_PER_TILE]
  WaitCtl wait;
};

struct Unit {
  int tile, split, ntile, ttile, k0, k1;
};

__device__ __forceinline__ Unit decode_unit(const S24Args& g, int u) {
  Unit t;
  t.tile = u / g.splits;
  t.split = u - t.tile * g.splits;
  t.ntile = t.tile / g.tt;
  t.ttile = t.tile - t.ntile * g.tt;
  t.k0 = static_cast<int>(static_cast<int64_t>(t.split) * g.ks / g.splits);
  t.k1 = static_cast<int>(static_cast<int64_t>(t.split + 1) * g.ks / g.splits);
  return t;
}

// Instruction descriptor of the sparse kind::i8 MMA: the dense descriptor
// (signed A and B, int32 accumulator, both K-major) with the sparsity flag.
__host__ __device__ constexpr uint32_t idesc_i8_sparse(int M, int N) { return idesc_i8(M, N) | (1u << 2); }

// D[tmem] (+)= A * B^T with A 2:4-compressed (128 rows x 32 B per MMA, K = 64
// logical), its metadata at tensor-memory address `meta`; issued by one thread.
__device__ __forceinline__ void mma_i8_sparse(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t meta,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "tcgen05.mma.sp.cta_group::1.kind::i8 [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(meta), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Asynchronous copy of a 128-row x 16-byte shared-memory matrix (unswizzled:
// 8-row x 16-byte core matrices, 128 bytes apart) into 128 lanes x 4 columns
// of tensor memory; ordered before the MMAs this thread issues after it.
__device__ __forceinline__ void tmem_cp_128x128b(uint32_t taddr, uint32_t smem_addr) {
  const uint64_t desc = (static_cast<uint64_t>((smem_addr & 0x3FFFFu) >> 4))   // start address
                        | (static_cast<uint64_t>(128u >> 4) << 16)              // leading byte offset
                        | (static_cast<uint64_t>(128u >> 4) << 32)              // stride: 8-row groups
                        | (1ull << 46);                                         // version; no swizzle
  asm volatile("tcgen05.cp.cta_group::1.128x128b [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}

// Epilogue of one chunk: lane = channel ch (the warp's channels ch_w ..
// ch_w + 31), r[j] = int32 accumulator of token tok0 + j (j < width, width
// 16 or 32).  bf16 goes through the warp's staging buffer `buf` (free once
// its previous store has read it) and one TMA store of the 32 x 32 block,
// which clips tokens >= M and channels >= N; int32 is stored directly.
// bf16: out = bf16(((float)acc * s_row) * s_col + bias), each operation
// rounded on its own.
// PENDING: how many of this warp's earlier stores may still be reading their
// staging buffers (0: one buffer per warp; 1: two buffers used in turn, and
// every chunk commits a group, an empty one when it stores nothing, so that
// the count stays in step with the buffers).
template <int PENDING>
__device__ __forceinline__ void store_chunk_t(const S24Args& g, const uint32_t (&r)[32], int width, int tok0, int ch,
                                              int ch_w, int lane, uint32_t buf, const CUtensorMap* tm32,
                                              const CUtensorMap* tm16) {
  const bool ch_ok = ch < g.N;
  if (g.out_s32) {
    int32_t* o = static_cast<int32_t*>(g.out);
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j < width && ch_ok && tok0 + j < g.M) o[static_cast<int64_t>(tok0 + j) * g.N + ch] = static_cast<int32_t>(r[j]);
    return;
  }
  const float sc = ch_ok ? __ldg(g.s_col + ch) : 0.0f;
  const bool has_bias = g.bias != nullptr;
  const float b = (has_bias && ch_ok) ? __uint_as_float(static_cast<uint32_t>(__ldg(g.bias + ch)) << 16) : 0.0f;
  // the chunk's 32 token scales: one load per lane (lane j: token tok0 + j),
  // then handed out by shuffles; tokens past M get 0
  const int mj = tok0 + lane;
  const float sr_lane = mj < g.M ? __ldg(g.s_row + mj) : 0.0f;
  // ((float)acc * s_row) * s_col (+ bias) for the token pair (2i, 2i + 1) as
  // f32x2, each lane rounded like the scalar operation
  const uint64_t sc2 = pack_f2(sc, sc);
  const uint64_t b2 = pack_f2(b, b);
  uint32_t pk[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float sr0 = __shfl_sync(0xffffffffu, sr_lane, 2 * i);
    const float sr1 = __shfl_sync(0xffffffffu, sr_lane, 2 * i + 1);
    uint64_t f = mul_f2(mul_f2(pack_f2(__int2float_rn(static_cast<int32_t>(r[2 * i])),
                                       __int2float_rn(static_cast<int32_t>(r[2 * i + 1]))),
                               pack_f2(sr0, sr1)),
                        sc2);
    if (has_bias) f = add_f2(f, b2);
    float f0, f1;
    unpack_f2(f, f0, f1);
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(pk[i]) : "f"(f1), "f"(f0));
  }
  if (lane == 0) bulk_wait_group_read<PENDING>();
  __syncwarp();
  pipe::stage_bf16_pairs(buf, pk, width, lane);
  fence_proxy_async_smem();
  __syncwarp();
  if constexpr (PENDING == 0) {
    if (lane == 0 && ch_w < g.N && tok0 < g.M) {     // boxes wholly outside are not issued
      tma_store_2d(width == 32 ? tm32 : tm16, buf, 2 * ch_w, tok0);
      bulk_commit_group();
    }
  } else {
    if (lane == 0) {
      if (ch_w < g.N && tok0 < g.M) tma_store_2d(width == 32 ? tm32 : tm16, buf, 2 * ch_w, tok0);
      bulk_commit_group();
    }
  }
}

__device__ __forceinline__ void store_chunk(const S24Args& g, const uint32_t (&r)[32], int width, int tok0, int ch,
                                            int ch_w, int lane, uint32_t buf, const CUtensorMap* tm32,
                                            const CUtensorMap* tm16) {
  store_chunk_t<0>(g, r, width, tok0, ch, ch_w, lane, buf, tm32, tm16);
}

// Reads a chunk's accumulators (width 32, or 16 for a 16-token tail) from TMEM.
__device__ __forceinline__ void load_chunk(uint32_t taddr, int width, uint32_t (&r)[32]) {
  if (width == 32) {
    tmem_ld_32x32b_x32(taddr, r);
  } else {
    uint32_t r16[16];
    tmem_ld_32x32b_x16(taddr, r16);
#pragma unroll
    for (int j = 0; j < 16; ++j) r[j] = r16[j];
#pragma unroll
    for (int j = 16; j < 32; ++j) r[j] = 0;
  }
}

__global__ void __launch_bounds__(S4_THREADS, 1)
    s24_gemm_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_m, const __grid_constant__ CUtensorMap tm_c32,
                    const __grid_constant__ CUtensorMap tm_c16, const S24Args g) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const smem = smem_raw + (base - raw);
  // stage s at base + s * stage_bytes: activation tile (bn x 128 B), compressed
  // values (128 x 64 B), metadata (128 x 16 B); every part 1024-byte aligned
  const uint32_t q_bytes = static_cast<uint32_t>(g.bn) * 128u;
  const uint32_t stage_bytes = q_bytes + S4_V_BYTES + S4_M_BYTES;
  uint64_t* const full = reinterpret_cast<uint64_t*>(smem + g.off_bar);
  uint64_t* const empty = full + S4_MAX_NP;
  uint64_t* const accf = empty + S4_MAX_NP;
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
      mbar_init(smem_u32(empty + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(accf + i), 1);
      mbar_init(smem_u32(acce + i), S4_EPI_WARPS);
    }
    mbar_init(smem_u32(drain), 1);
    fence_barrier_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_m);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), S4_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // With a programmatic (early) launch, the kernel that produced A is done
  // before any global memory is touched.
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
          const uint32_t sq = base + stage * stage_bytes;
          const uint32_t sv = sq + q_bytes;
          mbar_arrive_expect_tx(fb, q_bytes + S4_V_BYTES + S4_M_BYTES);
          tma_load_2d(sq, &tm_q, fb, kk * S4_BK, t.ttile * g.bn);
          tma_load_2d(sv, &tm_v, fb, kk * (S4_BK / 2), t.ntile * 128);
          tma_load_2d(sv + S4_V_BYTES, &tm_m, fb, kk * (S4_BK / 8), t.ntile * 128);
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
      const uint32_t idesc = idesc_i8_sparse(128, g.bn);
      int stage = 0, acc = 0;
      uint32_t phase = 0, aphase = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < g.units; u += gridDim.x) {
        const Unit t = decode_unit(g, u);
        if (!pipe::wait(smem_u32(acce + acc), aphase ^ 1, g.wait, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * g.bn);
        for (int kk = t.k0; kk < t.k1; ++kk) {
          if (!pipe::wait(smem_u32(full + stage), phase, g.wait, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sq = base + stage * stage_bytes;
          const uint32_t sv = sq + q_bytes;
          // the step's metadata into this stage's tensor-memory slot (the
          // slot's previous MMAs completed before the stage was refilled)
          const uint32_t meta = tmem_base + static_cast<uint32_t>(2 * g.bn + 4 * stage);
          tmem_cp_128x128b(meta, sv + S4_V_BYTES);
          const uint64_t ad = smem_desc_kmajor<64>(sv);
          const uint64_t bd = smem_desc_kmajor<128>(sq);
#pragma unroll
          for (int j = 0; j < 2; ++j)   // logical K = 64 per MMA: 32 compressed bytes, 64 activation bytes
            mma_i8_sparse(d_tmem, ad + 2 * j, bd + 4 * j, meta + 2 * j, idesc, (kk > t.k0 || j > 0) ? 1u : 0u);
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
      mma_commit(smem_u32(drain));
      volatile int never = 0;
      pipe::wait(smem_u32(drain), 0, g.wait, &never);
    }
  } else {
    // ---------------------------------------------------------- epilogue
    // warp w reads TMEM sub-partition w % 4 (channels 32 (w % 4) .. + 31) and
    // takes every other 32-token chunk (grp = 0 or 1)
    const int ew = warp - 2;
    const int q = warp & 3;
    const int grp = ew >> 2;
    const int row = q * 32 + lane;
    const uint32_t buf = base + g.off_epi + static_cast<uint32_t>(ew) * S4_EPI_BUF;
    int acc = 0;
    uint32_t aphase = 0;
    for (int u = blockIdx.x; u < g.units; u += gridDim.x) {
      const Unit t = decode_unit(g, u);
      const bool w = pipe::wait(smem_u32(accf + acc), aphase, g.wait, abort_flag);
      if (!__all_sync(0xffffffffu, w)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * g.bn);
      const int ch = t.ntile * 128 + row;
      const int ch_w = t.ntile * 128 + q * 32;
      const int tok0 = t.ttile * g.bn;
      const int nch = (g.bn + 31) / 32;
      if (g.splits == 1) {
        for (int c = grp; c < nch; c += 2) {
          const int width = min(32, g.bn - 32 * c);
          uint32_t r[32];
          load_chunk(tb + 32 * c, width, r);
          tmem_ld_wait();
          if (c + 2 >= nch) {            // this warp's last chunk: the accumulator is free
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(acce + acc));
          }
          store_chunk(g, r, width, tok0 + 32 * c, ch, ch_w, lane, buf, &tm_c32, &tm_c16);
        }
        if (grp >= nch) {                 // no chunk for this warp (bn <= 32)
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(acce + acc));
        }
      } else {
        // Split contraction: this warp's chunks as an int32 partial tile
        // [token][channel], then the last of the tile's splits to arrive (per
        // warp: its own counter) adds the partials in split order and stores.
        int32_t* const part = g.ws + (static_cast<int64_t>(t.tile) * g.splits + t.split) * g.bn * 128;
        for (int c = grp; c < nch; c += 2) {
          const int width = min(32, g.bn - 32 * c);
          uint32_t r[32];
          load_chunk(tb + 32 * c, width, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < width) part[static_cast<int64_t>(32 * c + j) * 128 + row] = static_cast<int32_t>(r[j]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(acce + acc));
        __threadfence();
        __syncwarp();
        uint32_t prev = 0;
        if (lane == 0) prev = atomicAdd(g.cnt + t.tile * S4_CNT_PER_TILE + ew, 1u);
        prev = __shfl_sync(0xffffffffu, prev, 0);
        if (prev == static_cast<uint32_t>(g.splits - 1)) {
          __threadfence();
          const int32_t* const tile_ws = g.ws + static_cast<int64_t>(t.tile) * g.splits * g.bn * 128;
          for (int c = grp; c < nch; c += 2) {
            const int width = min(32, g.bn - 32 * c);
            uint32_t r[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) r[j] = 0u;
            // split by split, the chunk's loads all in flight together
            for (int sp = 0; sp < g.splits; ++sp) {
              const int32_t* src = tile_ws + (static_cast<int64_t>(sp) * g.bn + 32 * c) * 128 + row;
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (j < width) r[j] = static_cast<uint32_t>(static_cast<int32_t>(r[j]) + __ldcg(src + j * 128));
            }
            store_chunk(g, r, width, tok0 + 32 * c, ch, ch_w, lane, buf, &tm_c32, &tm_c16);
          }
          __syncwarp();
          if (lane == 0) g.cnt[t.tile * S4_CNT_PER_TILE + ew] = 0u;    // the counters are left zeroed
        }
      }
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
  if (warp == 1) tmem_dealloc(tmem_base, S4_TMEM_COLS);
}

// ---------------------------------------------------------------- 2-SM pair
// Many tokens: each 256-channel x bn-token tile's sparse MMAs run on a pair
// of SMs (a cluster of two CTAs, tcgen05.mma.sp.cta_group::2, M = 256).  Each
// CTA loads its own 128 weight rows (compressed values and metadata) and half
// of the activation tile (bn / 2 tokens); the pair MMA reads each CTA's half
// of the activations once for both SMs, so per SM and 128-deep step TMA
// writes 25 KB instead of 40 KB (bn = 240) and more stages fit.  The leader
// (rank 0) copies the step's metadata of both CTAs into their tensor memory
// (tcgen05.cp.cta_group::2: each CTA's rows from its own shared memory) and
// issues the MMAs; one commit multicast to both CTAs frees a stage or hands
// over an accumulator.  No split contraction.

__device__ __forceinline__ void mma_i8_sparse_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t meta,
                                                   uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "tcgen05.mma.sp.cta_group::2.kind::i8 [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(meta), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tmem_cp_128x128b_pair(uint32_t taddr, uint32_t smem_addr) {
  const uint64_t desc = (static_cast<uint64_t>((smem_addr & 0x3FFFFu) >> 4))
                        | (static_cast<uint64_t>(128u >> 4) << 16)
                        | (static_cast<uint64_t>(128u >> 4) << 32)
                        | (1ull << 46);
  asm volatile("tcgen05.cp.cta_group::2.128x128b [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}

__global__ void __launch_bounds__(S4_THREADS, 1)
    s24_gemm2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_m, const __grid_constant__ CUtensorMap tm_c32,
                     const __grid_constant__ CUtensorMap tm_c16, const S24Args g) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const smem = smem_raw + (base - raw);
  // stage s at base + s * stage_bytes: this CTA's half of the activation tile
  // (bn / 2 x 128 B), its compressed values (128 x 64 B) and metadata (128 x
  // 16 B); every part 1024-byte aligned
  const uint32_t q_bytes = static_cast<uint32_t>(g.bn / 2) * 128u;
  const uint32_t stage_bytes = q_bytes + S4_V_BYTES + S4_M_BYTES;
  uint64_t* const full = reinterpret_cast<uint64_t*>(smem + g.off_bar);
  uint64_t* const empty = full + S4_MAX_NP;
  uint64_t* const accf = empty + S4_MAX_NP;
  uint64_t* const acce = accf + 2;
  uint64_t* const drain = acce + 2;
  uint32_t* const tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = static_cast<int>(cluster_ctarank());
  const bool leader = rank == 0;
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int pairs = static_cast<int>(gridDim.x >> 1);
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < g.np; ++i) {
      mbar_init(smem_u32(full + i), 1);
      mbar_init(smem_u32(empty + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(accf + i), 1);
      mbar_init(smem_u32(acce + i), 2 * S4_EPI_WARPS);
    }
    mbar_init(smem_u32(drain), 1);
    fence_barrier_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_m);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_holder), S4_TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();            // both CTAs' barriers are initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  griddep_wait();

  if (warp == 0) {
    // ---------------------------------------------------------- producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      for (int u = pair; ok && u < g.units; u += pairs) {
        const int ntile = 2 * (u / g.tt) + rank;
        const int ttile = u % g.tt;
        for (int kk = 0; kk < g.ks; ++kk) {
          if (!pipe::wait(smem_u32(empty + stage), phase ^ 1, g.wait, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(full + stage);
          const uint32_t fb_leader = map_to_rank(fb, 0);
          const uint32_t sq = base + stage * stage_bytes;
          const uint32_t sv = sq + q_bytes;
          if (leader) mbar_arrive_expect_tx(fb, 2u * stage_bytes);
          tma_load_2d_pair(sq, &tm_q, fb_leader, kk * S4_BK, ttile * g.bn + rank * (g.bn / 2));
          tma_load_2d_pair(sv, &tm_v, fb_leader, kk * (S4_BK / 2), ntile * 128);
          tma_load_2d_pair(sv + S4_V_BYTES, &tm_m, fb_leader, kk * (S4_BK / 8), ntile * 128);
          ++issued;
          if (++stage == g.np) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        // Let the copies already issued land before the CTA leaves: the leader
        // waits on its full barriers (bounded); the follower, whose copies
        // complete on the leader's barriers, waits a fixed 100 us.
        if (leader) {
          WaitCtl quick = g.wait;
          quick.timeout_ns = quick.timeout_ns < 50000000ull ? quick.timeout_ns : 50000000ull;
          volatile int never = 0;
          for (long long i = issued > g.np ? issued - g.np : 0; i < issued; ++i)
            pipe::wait(smem_u32(full + static_cast<int>(i % g.np)), static_cast<uint32_t>((i / g.np) & 1), quick,
                       &never);
        } else {
          const uint64_t t0 = globaltimer();
          while (globaltimer() - t0 < 100000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer (leader)
    if (leader && lane == 0) {
      const uint32_t idesc = idesc_i8_sparse(256, g.bn);
      int stage = 0, acc = 0;
      uint32_t phase = 0, aphase = 0;
      bool ok = true;
      for (int u = pair; ok && u < g.units; u += pairs) {
        if (!pipe::wait(smem_u32(acce + acc), aphase ^ 1, g.wait, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * g.bn);
        for (int kk = 0; kk < g.ks; ++kk) {
          if (!pipe::wait(smem_u32(full + stage), phase, g.wait, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sq = base + stage * stage_bytes;
          const uint32_t sv = sq + q_bytes;
          // both CTAs' metadata of the step into their tensor-memory slot of
          // this stage (the slot's previous MMAs completed before the stage
          // was refilled)
          const uint32_t meta = tmem_base + static_cast<uint32_t>(2 * g.bn + 4 * stage);
          tmem_cp_128x128b_pair(meta, sv + S4_V_BYTES);
          const uint64_t ad = smem_desc_kmajor<64>(sv);
          const uint64_t bd = smem_desc_kmajor<128>(sq);
#pragma unroll
          for (int j = 0; j < 2; ++j)   // logical K = 64 per MMA: 32 compressed bytes, 64 activation bytes
            mma_i8_sparse_pair(d_tmem, ad + 2 * j, bd + 4 * j, meta + 2 * j, idesc, (kk > 0 || j > 0) ? 1u : 0u);
          mma_commit_pair_both(smem_u32(empty + stage));
          if (++stage == g.np) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        mma_commit_pair_both(smem_u32(accf + acc));
        if (++acc == 2) {
          acc = 0;
          aphase ^= 1;
        }
      }
      mma_commit_pair(map_to_rank(smem_u32(drain), 0));
      volatile int never = 0;
      pipe::wait(smem_u32(drain), 0, g.wait, &never);
    }
  } else {
    // ---------------------------------------------------------- epilogue (both CTAs)
    // This CTA's 128 channels (its TMEM lanes) x all bn tokens, as in the
    // 1-SM kernel; each warp frees the accumulator on the leader once it has
    // read its last chunk.
    const int ew = warp - 2;
    const int q = warp & 3;
    const int grp = ew >> 2;
    const int row = q * 32 + lane;
    const uint32_t buf0 = base + g.off_epi + static_cast<uint32_t>(ew) * 2u * S4_EPI_BUF;   // two per warp
    uint32_t flip = 0;
    const uint32_t acce_leader = map_to_rank(smem_u32(acce), 0);
    int acc = 0;
    uint32_t aphase = 0;
    for (int u = pair; u < g.units; u += pairs) {
      const int ntile = 2 * (u / g.tt) + rank;
      const int ttile = u % g.tt;
      const bool w = pipe::wait(smem_u32(accf + acc), aphase, g.wait, abort_flag);
      if (!__all_sync(0xffffffffu, w)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * g.bn);
      const int ch = ntile * 128 + row;
      const int ch_w = ntile * 128 + q * 32;
      const int tok0 = ttile * g.bn;
      const int nch = (g.bn + 31) / 32;
      // two of this warp's chunks per tensor-memory wait; the staging
      // buffers alternate, so a chunk waits only for the store before last
      for (int c0 = grp; c0 < nch; c0 += 4) {
        const int c1 = c0 + 2;
        const bool two = c1 < nch;
        const int w0 = min(32, g.bn - 32 * c0);
        const int w1 = two ? min(32, g.bn - 32 * c1) : 0;
        uint32_t r0[32], r1[32];
        load_chunk(tb + 32 * c0, w0, r0);
        if (two) load_chunk(tb + 32 * c1, w1, r1);
        tmem_ld_wait();
        if (c0 + 4 >= nch) {           // the batch with this warp's last chunk: the accumulator is free
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(acce_leader + static_cast<uint32_t>(acc) * 8u);
        }
        store_chunk_t<1>(g, r0, w0, tok0 + 32 * c0, ch, ch_w, lane, buf0 + flip * S4_EPI_BUF, &tm_c32, &tm_c16);
        flip ^= 1u;
        if (two) {
          store_chunk_t<1>(g, r1, w1, tok0 + 32 * c1, ch, ch_w, lane, buf0 + flip * S4_EPI_BUF, &tm_c32, &tm_c16);
          flip ^= 1u;
        }
      }
      if (grp >= nch) {                 // no chunk for this warp (bn <= 32)
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acce_leader + static_cast<uint32_t>(acc) * 8u);
      }
      if (++acc == 2) {
        acc = 0;
        aphase ^= 1;
      }
    }
    if (lane == 0) bulk_wait_group<0>();         // every output store complete
    __syncwarp();
  }

  tc_fence_before();
  cluster_sync_all();            // no CTA leaves while its peer may still read its shared memory or signal it
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, S4_TMEM_COLS);
}

// One thread per metadata byte (two groups): compress eight weight bytes.
__global__ void __launch_bounds__(256) s24_compress_kernel(const int8_t* __restrict__ w, int64_t N, int64_t K,
                                                           int8_t* __restrict__ values, uint8_t* __restrict__ meta,
                                                           int32_t* violations) {
  const int64_t per_row = K / 8;
  const int64_t total = N * per_row;
  for (int64_t b = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; b < total;
       b += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = b / per_row;
    const int64_t j = b - n * per_row;
    const uint2 src = *reinterpret_cast<const uint2*>(w + n * K + 8 * j);
    uint32_t vout = 0, mout = 0;
    int bad = 0;
#pragma unroll
    for (int gsub = 0; gsub < 2; ++gsub) {
      const uint32_t word = gsub ? src.y : src.x;
      int pos[2] = {0, 0};
      int cnt = 0, nz = 0;
#pragma unroll
      for (int p = 0; p < 4; ++p)
        if ((word >> (8 * p)) & 0xFFu) {
          ++nz;
          if (cnt < 2) pos[cnt++] = p;
        }
      if (nz > 2) ++bad;
      // fill with the lowest free (zero) positions
#pragma unroll
      for (int p = 0; p < 4; ++p)
        if (cnt < 2 && ((word >> (8 * p)) & 0xFFu) == 0u && !(cnt == 1 && pos[0] == p)) pos[cnt++] = p;
      const int p0 = min(pos[0], pos[1]), p1 = max(pos[0], pos[1]);
      const uint32_t v0 = (word >> (8 * p0)) & 0xFFu, v1 = (word >> (8 * p1)) & 0xFFu;
      vout |= (v0 | (v1 << 8)) << (16 * gsub);
      mout |= static_cast<uint32_t>(p0 | (p1 << 2)) << (4 * gsub);
    }
    *reinterpret_cast<uint32_t*>(values + n * (K / 2) + 4 * j) = vout;
    meta[b] = static_cast<uint8_t>(mout);
    if (bad && violations != nullptr) atomicAdd(violations, bad);
  }
}

// ---------------------------------------------------------------- host side

struct S24Plan {
  int bn, tt, nt, ks, splits, units, grid, np;
  size_t cnt_bytes, ws_bytes, smem;
};

// Token tile width: the multiple of 16 (<= S4_MAX_BN) whose whole waves of
// tiles over the SMs cost the least, a tile costing bn + 32 per step (a fixed
// share per step for the weight tile and the MMA issue).  The contraction is
// split only when the tiles cannot fill the SMs (few channels and tokens), at
// least four steps per split: each split writes and the last one reads back
// an int32 partial tile.
S24Plan plan_s24(int64_t M, int64_t N, int64_t K, int sm_count, bool allow_split) {
  S24Plan best{};
  long long best_cost = -1;
  const int nt = static_cast<int>((N + 127) / 128);
  const int ks = static_cast<int>(K / S4_BK);
  for (int bn = 16; bn <= S4_MAX_BN; bn += 16) {
    if (bn > 16 && bn - 16 >= M) break;                 // wider tiles only add empty tokens
    const int tt = static_cast<int>((M + bn - 1) / bn);
    const long long tiles = static_cast<long long>(nt) * tt;
    const long long waves = (tiles + sm_count - 1) / sm_count;
    const long long cost = waves * (bn + 32);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best.bn = bn;
      best.tt = tt;
    }
  }
  best.splits = 1;
  const long long tiles0 = static_cast<long long>(nt) * best.tt;
  if (allow_split && tiles0 < sm_count) {
    int sp = static_cast<int>(sm_count / tiles0);
    sp = std::min(sp, std::max(1, ks / 4));
    best.splits = std::max(1, std::min(sp, 32));
  }
  S24Plan& p = best;
  p.nt = nt;
  p.ks = ks;
  const long long tiles = static_cast<long long>(p.nt) * p.tt;
  p.cnt_bytes = (static_cast<size_t>(tiles) * S4_CNT_PER_TILE * sizeof(uint32_t) + 255) / 256 * 256;
  p.ws_bytes = p.splits > 1 ? p.cnt_bytes + static_cast<size_t>(tiles) * p.splits * p.bn * 128 * sizeof(int32_t) : 0;
  p.units = static_cast<int>(tiles * p.splits);
  p.grid = std::min(p.units, sm_count);
  const int stage = p.bn * 128 + S4_V_BYTES + S4_M_BYTES;
  p.np = std::min({S4_MAX_NP, (S4_SMEM_LIMIT - 1024 - S4_EPI_WARPS * S4_EPI_BUF - S4_BAR_BYTES) / stage,
                   (S4_TMEM_COLS - 2 * p.bn) / 4});
  p.smem = 1024 + static_cast<size_t>(p.np) * stage + S4_EPI_WARPS * S4_EPI_BUF + S4_BAR_BYTES;
  return p;
}

// 2-SM pair tiles: 256 channels (128 per CTA) x bn tokens, bn chosen as in
// plan_s24 over the CTA pairs; no split.  Each stage holds half the
// activation tile, so up to 8 stages fit at bn = 240.
S24Plan plan_s24_pair(int64_t M, int64_t N, int64_t K, int sm_count) {
  S24Plan best{};
  long long best_cost = -1;
  const int pairs = std::max(1, sm_count / 2);
  const int nt = static_cast<int>((N + 255) / 256);
  for (int bn = 16; bn <= S4_MAX_BN; bn += 16) {
    if (bn > 16 && bn - 16 >= M) break;
    const int tt = static_cast<int>((M + bn - 1) / bn);
    const long long tiles = static_cast<long long>(nt) * tt;
    const long long waves = (tiles + pairs - 1) / pairs;
    const long long cost = waves * (bn + 32);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best.bn = bn;
      best.tt = tt;
    }
  }
  S24Plan& p = best;
  p.splits = 1;
  p.nt = nt;
  p.ks = static_cast<int>(K / S4_BK);
  p.units = static_cast<int>(static_cast<long long>(p.nt) * p.tt);
  p.grid = 2 * std::min(p.units, pairs);
  const int stage = (p.bn / 2) * 128 + S4_V_BYTES + S4_M_BYTES;
  p.np = std::min({S4_MAX_NP, (S4_SMEM_LIMIT - 1024 - 2 * S4_EPI_WARPS * S4_EPI_BUF - S4_BAR_BYTES) / stage,
                   (S4_TMEM_COLS - 2 * p.bn) / 4});
  p.smem = 1024 + static_cast<size_t>(p.np) * stage + 2 * S4_EPI_WARPS * S4_EPI_BUF + S4_BAR_BYTES;
  return p;
}

int grid_for(int64_t items, int sm_count) {
  const int64_t blocks = (items + 255) / 256;
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(blocks, static_cast<int64_t>(sm_count) * 16)));
}

}  // namespace
}  // namespace dq

using namespace dq;

extern "C" {

DQ_API dq_status dq_s24_compress(const int8_t* wq, int64_t N, int64_t K, int8_t* values, uint8_t* meta,
                                 int32_t* violations, dq_stream_t stream) {
  if (N < 0 || K < 0 || K % 8 != 0) return DQ_ERR_INVALID_ARG;
  if (N == 0 || K == 0) return DQ_OK;
  if (wq == nullptr || values == nullptr || meta == nullptr) return DQ_ERR_INVALID_ARG;
  if (!aligned(wq, 8) || !aligned(values, 4)) return DQ_ERR_UNSUPPORTED;
  DeviceInfo* d = nullptr;
  dq_status st = current_device(&d);
  if (st != DQ_OK) return st;
  s24_compress_kernel<<<grid_for(N * (K / 8), d->sm_count), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      wq, N, K, values, meta, violations);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? DQ_OK : cuda_fail(e);
}

DQ_API size_t dq_s24_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0 || K % S4_BK != 0) return 0;
  DeviceInfo* d = nullptr;
  if (current_device(&d) != DQ_OK) return 0;
  return plan_s24(M, N, K, d->sm_count, true).ws_bytes;
}

DQ_API dq_status dq_s24_int8_linear(const int8_t* A, const float* s_row, int64_t M, int64_t K, const int8_t* values,
                                    const uint8_t* meta, const float* s_col, int64_t N, const void* bias_bf16,
                                    void* out, dq_out_dtype out_dtype, void* workspace, size_t workspace_bytes,
                                    dq_stream_t stream) {
  if (M < 0 || N <= 0 || K <= 0) return DQ_ERR_INVALID_ARG;
  if (out_dtype != DQ_OUT_BF16 && out_dtype != DQ_OUT_S32) return DQ_ERR_INVALID_ARG;
  if (K % S4_BK != 0 || N % 8 != 0) return DQ_ERR_UNSUPPORTED;
  if (M > (int64_t{1} << 30) || N > (int64_t{1} << 30) || K > (int64_t{1} << 30)) return DQ_ERR_UNSUPPORTED;
  if (values == nullptr || meta == nullptr) return DQ_ERR_INVALID_ARG;
  if (out_dtype == DQ_OUT_BF16 && s_col == nullptr) return DQ_ERR_INVALID_ARG;
  if (!aligned(values, 16) || !aligned(meta, 16)) return DQ_ERR_UNSUPPORTED;
  if (M == 0) return DQ_OK;
  if (A == nullptr || out == nullptr || (out_dtype == DQ_OUT_BF16 && s_row == nullptr)) return DQ_ERR_INVALID_ARG;
  if (!aligned(A, 16) || !aligned(out, 16)) return DQ_ERR_UNSUPPORTED;
  DeviceInfo* d = nullptr;
  dq_status st = current_device(&d);
  if (st != DQ_OK) return st;

  S24Plan p = plan_s24(M, N, K, d->sm_count, true);
  if (p.splits > 1 && (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < p.ws_bytes))
    p = plan_s24(M, N, K, d->sm_count, false);
  // Many tokens, no split: the 2-SM pair kernel (the dense int8 linear's rule;
  // schedule knob 3 forces it, 1 keeps the 1-SM kernel).
  const int sched = g_schedule_override.load(std::memory_order_relaxed);
  const bool pair = p.splits == 1 && N > 128 &&
                    (sched == 3 || (sched == 0 && M >= 1536 && K >= 2048));
  if (pair) p = plan_s24_pair(M, N, K, d->sm_count);

  CUtensorMap tq, tv, tm;
  st = make_tmap_u8_2d(&tq, A, static_cast<uint64_t>(K), static_cast<uint64_t>(M), static_cast<uint64_t>(K), 128,
                       static_cast<uint32_t>(pair ? p.bn / 2 : p.bn), 128);
  if (st != DQ_OK) return st;
  st = make_tmap_u8_2d(&tv, values, static_cast<uint64_t>(K / 2), static_cast<uint64_t>(N),
                       static_cast<uint64_t>(K / 2), 64, 128, 64);
  if (st != DQ_OK) return st;
  st = make_tmap_u8_2d(&tm, meta, static_cast<uint64_t>(K / 8), static_cast<uint64_t>(N),
                       static_cast<uint64_t>(K / 8), 16, 128, 0);
  if (st != DQ_OK) return st;
  // bf16 output [M, N] as bytes: 32 channels (64 B) x 32 or 16 tokens
  CUtensorMap tc32, tc16;
  st = make_tmap_u8_2d(&tc32, out, static_cast<uint64_t>(N) * 2, static_cast<uint64_t>(M),
                       static_cast<uint64_t>(N) * 2, 64, 32, 0);
  if (st != DQ_OK) return st;
  st = make_tmap_u8_2d(&tc16, out, static_cast<uint64_t>(N) * 2, static_cast<uint64_t>(M),
                       static_cast<uint64_t>(N) * 2, 64, 16, 0);
  if (st != DQ_OK) return st;

  S24Args g{};
  g.M = static_cast<int>(M);
  g.N = static_cast<int>(N);
  g.K = static_cast<int>(K);
  g.bn = p.bn;
  g.nt = p.nt;
  g.tt = p.tt;
  g.splits = p.splits;
  g.ks = p.ks;
  g.units = p.units;
  g.np = p.np;
  g.off_epi = static_cast<uint32_t>(p.np) * ((pair ? p.bn / 2 : p.bn) * 128 + S4_V_BYTES + S4_M_BYTES);
  g.off_bar = g.off_epi + (pair ? 2 : 1) * S4_EPI_WARPS * S4_EPI_BUF;   // the pair: two staging buffers per warp
  g.s_row = s_row;
  g.s_col = s_col;
  g.bias = out_dtype == DQ_OUT_BF16 ? static_cast<const uint16_t*>(bias_bf16) : nullptr;
  g.out = out;
  g.out_s32 = out_dtype == DQ_OUT_S32;
  if (p.splits > 1) {
    g.cnt = static_cast<uint32_t*>(workspace);
    g.ws = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + p.cnt_bytes);
  }
  g.wait = WaitCtl{d->err_word, wait_timeout_ns()};

  const void* kern = pair ? reinterpret_cast<const void*>(&s24_gemm2_kernel)
                          : reinterpret_cast<const void*>(&s24_gemm_kernel);
  const dq_status ast = smem_limit_once(kern, S4_SMEM_LIMIT);
  if (ast != DQ_OK) return ast;
  // Programmatic stream serialization: the prologue may overlap the tail of
  // the quantization that produced A; the kernel waits before global access.
  // The pair kernel runs as clusters of two CTAs.
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(p.grid));
  cfg.blockDim = dim3(S4_THREADS);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cfg.attrs = attr;
  cfg.numAttrs = pair ? 2 : 1;
  const cudaError_t e = pair ? cudaLaunchKernelEx(&cfg, s24_gemm2_kernel, tq, tv, tm, tc32, tc16, g)
                             : cudaLaunchKernelEx(&cfg, s24_gemm_kernel, tq, tv, tm, tc32, tc16, g);
  return e == cudaSuccess ? DQ_OK : cuda_fail(e);
}

}  // extern "C"
