// gemm_common.cuh -- pieces shared by the 1-SM and 2-SM int8 GEMM kernels:
// launch arguments, the per-CTA tile schedule, BSR index access and the
// dequantize / bf16 / store epilogue helpers.
#pragma once

#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace dq {

enum class Kind : int { Dense = 0, Swap = 1, Bsr = 2, Bsr32 = 3, Bsr16 = 4, DenseF8 = 5 };

// Contraction bytes per pipeline stage of the dense arrangements (1-SM and
// pair kernels): the K-major operand tiles are kDenseKB bytes wide, with the
// swizzle of that width.
constexpr int kDenseKB = 128;

// Dense arrangement with int8 (Dense) or e4m3 (DenseF8) operands; e4m3
// products accumulate in fp32 (kind::f8f6f4), int8 ones in int32.
__host__ __device__ constexpr bool is_dense_kind(Kind k) { return k == Kind::Dense || k == Kind::DenseF8; }

// Block-sparse weight kinds and their square block size (64, 32 or 16).
__host__ __device__ constexpr bool is_bsr(Kind k) { return k == Kind::Bsr || k == Kind::Bsr32 || k == Kind::Bsr16; }
__host__ __device__ constexpr int bsr_bs(Kind k) {
  return k == Kind::Bsr ? 64 : k == Kind::Bsr32 ? 32 : k == Kind::Bsr16 ? 16 : 0;
}

struct GemmArgs {
  int M, N, K;
  int a_tiles, b_tiles;   // tiles along the A slot (128 rows) and the B slot (BN rows)
  int kb_total;           // k blocks per tile (Dense / Swap)
  int num_tiles;
  int stream_k;           // 0: whole tiles round-robin; 1: stream-K ranges
  long long iters_total;  // num_tiles * kb_total (stream-K)
  const float* s_row;
  const float* s_col;
  const uint16_t* bias;   // bf16 bits or null
  void* out;
  int out_s32;
  int32_t* ws;            // stream-K partial tiles: [tile][BN][128] int32
  uint32_t* ws_cnt;       // stream-K arrival counters: [tile]
  const int32_t* crow;    // Bsr
  const int32_t* col;
  int nnzb;
  int nbr;                // Bsr: block rows (N / block size)
  int idx_smem;           // Bsr: crow and col staged in shared memory (they fit)
  // Dense, two tile widths (bn2 > 0): tiles [0, t1) are BN wide in row-major
  // tile order (a_tiles x b_tiles); tiles t1 .. num_tiles - 1 are bn2 wide and
  // cover the rest of the matrix: first_cnt tiles in 128-row block mb0 from
  // column c_start on, then per_row tiles in each later block row.
  int t1, bn2, mb0, c_start, first_cnt, per_row;
  // Each CTA takes a contiguous range of tiles (row-major tile order) instead
  // of every gridDim.x-th one: consecutive tiles then share their 128-row
  // block (the BSR panel kernel keeps that block's activations resident).
  int blocked;
  WaitCtl wait;
};


struct Seg {
  int tile;
  int kb0, kb1;
};

// Enumerates the (tile, k range) segments of one CTA; every role walks the
// same sequence.
struct SegIter {
  const GemmArgs* g;
  long long it, it_end;   // stream-K
  int next_tile;          // round-robin, or the next tile of a contiguous range
  int end_tile;           // contiguous range (g.blocked): one past the CTA's last tile
  __device__ SegIter(const GemmArgs& args) : g(&args) {
    const long long G = gridDim.x, c = blockIdx.x;
    if (args.stream_k) {
      it = c * args.iters_total / G;
      it_end = (c + 1) * args.iters_total / G;
    }
    if (args.blocked) {
      next_tile = static_cast<int>(c * args.num_tiles / G);
      end_tile = static_cast<int>((c + 1) * args.num_tiles / G);
    } else {
      next_tile = blockIdx.x;
      end_tile = args.num_tiles;
    }
  }
  __device__ bool next(Seg& s) {
    if (g->stream_k) {
      if (it >= it_end) return false;
      s.tile = static_cast<int>(it / g->kb_total);
      s.kb0 = static_cast<int>(it - static_cast<long long>(s.tile) * g->kb_total);
      const long long left = it_end - it;
      s.kb1 = static_cast<int>(min(static_cast<long long>(g->kb_total), s.kb0 + left));
      it += s.kb1 - s.kb0;
      return true;
    }
    if (next_tile >= end_tile) return false;
    s.tile = next_tile;
    next_tile += g->blocked ? 1 : static_cast<int>(gridDim.x);
    s.kb0 = 0;
    s.kb1 = g->kb_total;
    return true;
  }
};

// Where a tile lies: row block ta (128 rows for the 1-SM kernel, 256 for the
// pair kernel), B-slot tile tb, first output column n0 and the MMA width (bn,
// or g.bn2 for a Dense tile of the narrow second set).
struct TileGeom {
  int ta, tb, n0, width;
  bool narrow;
};
__device__ __forceinline__ TileGeom tile_geom(const GemmArgs& g, int tile, int bn, bool two_widths) {
  TileGeom t;
  if (two_widths && g.bn2 > 0 && tile >= g.t1) {
    int j = tile - g.t1;
    if (j < g.first_cnt) {
      t.ta = g.mb0;
      t.n0 = g.c_start + j * g.bn2;
    } else {
      j -= g.first_cnt;
      t.ta = g.mb0 + 1 + j / g.per_row;
      t.n0 = (j % g.per_row) * g.bn2;
    }
    t.tb = 0;
    t.width = g.bn2;
    t.narrow = true;
  } else {
    t.ta = tile / g.b_tiles;
    t.tb = tile % g.b_tiles;
    t.n0 = t.tb * bn;
    t.width = bn;
    t.narrow = false;
  }
  return t;
}

// Stream-K: number of CTAs whose ranges touch `tile`.
__device__ __forceinline__ int sk_contributors(const GemmArgs& g, int tile) {
  const long long G = gridDim.x, T = g.iters_total;
  const long long first = static_cast<long long>(tile) * g.kb_total;
  const long long last = first + g.kb_total - 1;
  const long long c0 = ((first + 1) * G - 1) / T;
  const long long c1 = ((last + 1) * G - 1) / T;
  return static_cast<int>(c1 - c0 + 1);
}

// Block range of one BSR block row, clamped to [0, nnzb].  `sidx` holds crow
// then col in shared memory, or is null (read global memory).
__device__ __forceinline__ void bsr_range(const GemmArgs& g, const int* sidx, int br, int& p0, int& p1) {
  int a = sidx ? sidx[br] : __ldg(g.crow + br);
  int b = sidx ? sidx[br + 1] : __ldg(g.crow + br + 1);
  a = min(max(a, 0), g.nnzb);
  b = min(max(b, a), g.nnzb);
  p0 = a;
  p1 = b;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// Column scales of one 32-column chunk as f32x2 pairs (s_col[n0 + 2i],
// s_col[n0 + 2i + 1]); zero past N (N % 8 == 0, so 8-column groups are wholly
// inside or outside).  All eight loads are issued before any is used.
struct ColScales {
  uint64_t sc[16];
};
// The same pairs out of a tile's staged slot (stage_tile_scales), c0 = the
// chunk's column offset from the tile's first column.
__device__ __forceinline__ void load_col_scales_staged(uint32_t slot, int c0, ColScales& p) {
#pragma unroll
  for (int v = 0; v < 8; ++v) {
    const uint4 w = lds_v4(slot + static_cast<uint32_t>(c0) * 4u + 16u * v);
    p.sc[2 * v] = (static_cast<uint64_t>(w.y) << 32) | w.x;
    p.sc[2 * v + 1] = (static_cast<uint64_t>(w.w) << 32) | w.z;
  }
}
__device__ __forceinline__ void load_col_scales(const GemmArgs& g, int n0, ColScales& p) {
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const int n = n0 + 8 * v;
    ulonglong2 c0 = make_ulonglong2(0ull, 0ull), c1 = c0;
    if (n < g.N) {
      c0 = __ldg(reinterpret_cast<const ulonglong2*>(g.s_col + n));
      c1 = __ldg(reinterpret_cast<const ulonglong2*>(g.s_col + n + 4));
    }
    p.sc[4 * v] = c0.x;
    p.sc[4 * v + 1] = c0.y;
    p.sc[4 * v + 2] = c1.x;
    p.sc[4 * v + 3] = c1.y;
  }
}

// A tile's column scales (fp32) and bias (bf16) staged in shared memory, so
// that the epilogue reads them there instead of issuing a dependent L2 load
// for every 32-column chunk.  One slot per tile in flight: s_col at +0 (up to
// 256 fp32), bias at +kScBiasOff (up to 256 bf16).  One thread copies them
// with 1-D bulk copies completing on the slot's mbarrier; columns past N are
// not copied (their outputs are clipped by the store).
constexpr int kScSlotBytes = 1536;
constexpr int kScBiasOff = 1024;

__device__ __forceinline__ void stage_tile_scales(const GemmArgs& g, uint32_t slot, int n0, int width,
                                                  uint32_t bar) {
  const int ncols = min(width, g.N - n0);          // a multiple of 8 (N % 8 == 0, n0 % 32 == 0)
  const bool need = !g.out_s32 && ncols > 0;
  const uint32_t sb = need ? static_cast<uint32_t>(ncols) * 4u : 0u;
  const uint32_t bb = need && g.bias != nullptr ? static_cast<uint32_t>(ncols) * 2u : 0u;
  mbar_arrive_expect_tx(bar, sb + bb);
  if (sb) bulk_load_1d(slot, g.s_col + n0, sb, bar);
  if (bb) bulk_load_1d(slot + kScBiasOff, g.bias + n0, bb, bar);
}

// Bias words of the 32-column chunk at column offset c0 (from the tile's
// first column) out of a staged slot.
__device__ __forceinline__ void load_bias_staged(uint32_t slot, int c0, uint4 (&b)[4]) {
#pragma unroll
  for (int v = 0; v < 4; ++v) b[v] = lds_v4(slot + kScBiasOff + static_cast<uint32_t>(c0) * 2u + 16u * v);
}
// Bias words of the chunk at output column n0 from global memory (zero past N).
__device__ __forceinline__ void load_bias_global(const GemmArgs& g, int n0, uint4 (&b)[4]) {
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const int n = n0 + 8 * v;
    b[v] = n < g.N ? __ldg(reinterpret_cast<const uint4*>(g.bias + n)) : make_uint4(0u, 0u, 0u, 0u);
  }
}

// Epilogue for one chunk of 32 columns of the Dense/Bsr layout: thread = row
// `row` (0..31 inside its warp's 32-row slab), output columns n0 .. n0+31.
// The 32x32 block is written into the warp's staging buffer with the tensor
// map's swizzle (64 B rows for bf16, 128 B rows for int32) and stored by one
// TMA bulk store, which also clips rows >= M and columns >= N.  `cs` holds the
// chunk's column scales (load_col_scales); with BIAS, g.bias is read for
// columns < N.  The output mode and the bias are template switches rather
// than run-time tests, so the code of the modes not taken is not executed
// predicated-off in every chunk.
template <bool S32, bool BIAS, bool F32ACC>
__device__ __forceinline__ void store_row_chunk_tma_t(const GemmArgs& g, const CUtensorMap* tm_c,
                                                      uint8_t* buf, int lane, int m0, int n0,
                                                      const uint32_t* r, float srow, const ColScales& cs,
                                                      const uint4 (&bias)[4]) {
  const uint32_t base = smem_u32(buf);
  if constexpr (S32) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t off = static_cast<uint32_t>(lane * 128 + ((j ^ (lane & 7)) << 4));
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(base + off), "r"(r[4 * j]),
                   "r"(r[4 * j + 1]), "r"(r[4 * j + 2]), "r"(r[4 * j + 3])
                   : "memory");
    }
  } else {
    // ((float)acc * s_row) * s_col (+ bias), as pairs: each lane of a pair
    // rounds like the scalar mul / add (RN), so the bits are those of the
    // scalar left-to-right evaluation.  All 16 output words are formed before
    // the shared-memory stores.
    const uint64_t srow2 = pack_f2(srow, srow);
    uint64_t f2[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      // int32 accumulators convert (round to nearest); fp32 ones are taken as they are
      const uint64_t a = F32ACC ? pack_f2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]))
                                : pack_f2(__int2float_rn(static_cast<int>(r[2 * j])),
                                          __int2float_rn(static_cast<int>(r[2 * j + 1])));
      f2[j] = mul_f2(mul_f2(a, srow2), cs.sc[j]);
    }
    if constexpr (BIAS) {
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint32_t bw[4] = {bias[v].x, bias[v].y, bias[v].z, bias[v].w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
          f2[4 * v + j] =
              add_f2(f2[4 * v + j], pack_f2(__uint_as_float(bw[j] << 16), __uint_as_float(bw[j] & 0xffff0000u)));
      }
    }
    uint32_t w[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      float lo, hi;
      unpack_f2(f2[j], lo, hi);
      w[j] = pack_bf16x2(lo, hi);
    }
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const uint32_t off = static_cast<uint32_t>(lane * 64 + ((v ^ ((lane >> 1) & 3)) << 4));
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(base + off), "r"(w[4 * v]),
                   "r"(w[4 * v + 1]), "r"(w[4 * v + 2]), "r"(w[4 * v + 3])
                   : "memory");
    }
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0 && n0 < g.N && m0 < g.M) {   // boxes wholly past the matrix are not issued
    tma_store_2d(tm_c, base, n0, m0);
    bulk_commit_group();
  }
}

// The same chunk epilogue with the column scales and bias read from the
// tile's staged shared-memory slot (stage_tile_scales) as they are needed,
// c0 = the chunk's column offset from the tile's first column: nothing is
// held in registers beyond the 32 accumulators and the 16 packed outputs.
template <bool S32, bool BIAS, bool F32ACC>
__device__ __forceinline__ void store_row_chunk_staged_t(const GemmArgs& g, const CUtensorMap* tm_c, uint8_t* buf,
                                                         int lane, int m0, int n0, const uint32_t* r, float srow,
                                                         uint32_t slot, int c0) {
  const uint32_t base = smem_u32(buf);
  if constexpr (S32) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t off = static_cast<uint32_t>(lane * 128 + ((j ^ (lane & 7)) << 4));
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(base + off), "r"(r[4 * j]),
                   "r"(r[4 * j + 1]), "r"(r[4 * j + 2]), "r"(r[4 * j + 3])
                   : "memory");
    }
  } else {
    // ((float)acc * s_row) * s_col (+ bias) as f32x2 pairs, left to right,
    // each lane rounded like the scalar op; 8 columns per step.
    const uint64_t srow2 = pack_f2(srow, srow);
    const uint32_t sc_addr = slot + static_cast<uint32_t>(c0) * 4u;
    const uint32_t b_addr = slot + kScBiasOff + static_cast<uint32_t>(c0) * 2u;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const uint4 s0 = lds_v4(sc_addr + 32u * v);
      const uint4 s1 = lds_v4(sc_addr + 32u * v + 16u);
      const uint64_t sc[4] = {(static_cast<uint64_t>(s0.y) << 32) | s0.x, (static_cast<uint64_t>(s0.w) << 32) | s0.z,
                              (static_cast<uint64_t>(s1.y) << 32) | s1.x, (static_cast<uint64_t>(s1.w) << 32) | s1.z};
      uint4 b = make_uint4(0u, 0u, 0u, 0u);
      if constexpr (BIAS) b = lds_v4(b_addr + 16u * v);
      const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
      uint32_t w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int e = 8 * v + 2 * j;
        const uint64_t a = F32ACC ? pack_f2(__uint_as_float(r[e]), __uint_as_float(r[e + 1]))
                                  : pack_f2(__int2float_rn(static_cast<int>(r[e])),
                                            __int2float_rn(static_cast<int>(r[e + 1])));
        uint64_t f = mul_f2(mul_f2(a, srow2), sc[j]);
        if constexpr (BIAS) f = add_f2(f, pack_f2(__uint_as_float(bw[j] << 16), __uint_as_float(bw[j] & 0xffff0000u)));
        float lo, hi;
        unpack_f2(f, lo, hi);
        w[j] = pack_bf16x2(lo, hi);
      }
      const uint32_t off = static_cast<uint32_t>(lane * 64 + ((v ^ ((lane >> 1) & 3)) << 4));
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(base + off), "r"(w[0]), "r"(w[1]), "r"(w[2]),
                   "r"(w[3])
                   : "memory");
    }
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0 && n0 < g.N && m0 < g.M) {   // boxes wholly past the matrix are not issued
    tma_store_2d(tm_c, base, n0, m0);
    bulk_commit_group();
  }
}

template <bool F32ACC = false>
__device__ __forceinline__ void store_row_chunk_staged(const GemmArgs& g, const CUtensorMap* tm_c, uint8_t* buf,
                                                       int lane, int m0, int n0, const uint32_t* r, float srow,
                                                       uint32_t slot, int c0) {
  if (g.out_s32) store_row_chunk_staged_t<true, false, F32ACC>(g, tm_c, buf, lane, m0, n0, r, srow, slot, c0);
  else if (g.bias != nullptr)
    store_row_chunk_staged_t<false, true, F32ACC>(g, tm_c, buf, lane, m0, n0, r, srow, slot, c0);
  else store_row_chunk_staged_t<false, false, F32ACC>(g, tm_c, buf, lane, m0, n0, r, srow, slot, c0);
}

// `bias` holds the chunk's 32 bf16 bias values (read only when g.bias is set).
template <bool F32ACC = false>
__device__ __forceinline__ void store_row_chunk_tma(const GemmArgs& g, const CUtensorMap* tm_c, uint8_t* buf,
                                                    int lane, int m0, int n0, const uint32_t* r, float srow,
                                                    const ColScales& cs, const uint4 (&bias)[4]) {
  // raw mode stores the accumulator bits (int32, or fp32 for e4m3 operands)
  if (g.out_s32) store_row_chunk_tma_t<true, false, F32ACC>(g, tm_c, buf, lane, m0, n0, r, srow, cs, bias);
  else if (g.bias != nullptr)
    store_row_chunk_tma_t<false, true, F32ACC>(g, tm_c, buf, lane, m0, n0, r, srow, cs, bias);
  else store_row_chunk_tma_t<false, false, F32ACC>(g, tm_c, buf, lane, m0, n0, r, srow, cs, bias);
}

// Epilogue for the Swap layout: thread = output channel n, columns are
// tokens m0 .. m0+CW-1.
template <int CW>
__device__ __forceinline__ void store_col_chunk(const GemmArgs& g, int n, int m0, const uint32_t* r) {
  if (n >= g.N) return;
  if (g.out_s32) {
    int32_t* o = static_cast<int32_t*>(g.out) + n;
#pragma unroll
    for (int j = 0; j < CW; ++j)
      if (m0 + j < g.M) o[static_cast<int64_t>(m0 + j) * g.N] = static_cast<int>(r[j]);
    return;
  }
  const float sc = __ldg(g.s_col + n);
  const bool has_bias = g.bias != nullptr;
  const float b = has_bias ? __uint_as_float(static_cast<uint32_t>(__ldg(g.bias + n)) << 16) : 0.0f;
  uint16_t* o = static_cast<uint16_t*>(g.out) + n;
#pragma unroll
  for (int j = 0; j < CW; ++j) {
    const int m = m0 + j;
    if (m < g.M) {
      float f = __fmul_rn(__fmul_rn(__int2float_rn(static_cast<int>(r[j])), __ldg(g.s_row + m)), sc);
      if (has_bias) f = __fadd_rn(f, b);
      __nv_bfloat16 h = __float2bfloat16_rn(f);
      o[static_cast<int64_t>(m) * g.N] = *reinterpret_cast<uint16_t*>(&h);
    }
  }
}

// Dense GEMM with each 256 x bn tile's MMA on a pair of SMs (gemm2sm.cu).
// g.a_tiles / g.b_tiles count 256-row / bn-column tiles; bn is 160, 192 or
// 256; with g.bn2 > 0 the tiles from g.t1 on are bn2 wide (tm_b2's box is
// bn2 / 2 weight rows).  `pairs` is the number of CTA pairs to launch; f8:
// e4m3 operands and an fp32 accumulator (bn 256 only).
dq_status launch_pair_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tb2,
                           const CUtensorMap& tc, const GemmArgs& g, int bn, int pairs, cudaStream_t stream,
                           bool f8 = false);
// CTA pairs of the pair kernel that fit on the current device at once.
dq_status pair_slots(const DeviceInfo& d, int* pairs);

}  // namespace dq
