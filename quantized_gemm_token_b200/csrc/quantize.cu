// quantize.cu -- per-row symmetric absmax int8 quantization.
//
// Per-token dynamic quantization of activations ("int8 dynamic quant + bsr
// support", pytorch/ao PR 821) with the absmax/127 symmetric scale (Paddle
// "sparse_fc supported", PR 41770, SpmmPluginDynamic), and the same formula
// per output channel for the weight:
//     s = fp32( max(absmax, 1e-8f) / 127 ),  q = clamp(rint(x / s), -127, 127)
// with IEEE round-to-nearest-even division: the codes are bit-identical to a
// scalar IEEE evaluation, computed without a division (bf16: Markstein's
// correction step gives the exact quotient; fp32: a flagged fallback).
//
// The default kernel keeps a whole row in registers: each row is owned by a
// power-of-two group of 32..256 threads, each thread loads up to 8 16-byte
// vectors (one HBM pass), the group reduces |x| (bf16x2 max per thread, then
// an integer max on the fp32 bit patterns across the group, exact for finite
// values: a non-negative IEEE value orders like its bits), and the codes are
// written straight from registers.  A row-pipelined kernel (bulk copies into a
// shared-memory ring) is kept as an alternative for 1-16 KB rows.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace dq {
namespace {

template <typename T>
struct Elem;
template <>
struct Elem<uint16_t> {          // bf16 bit patterns
  static constexpr int kPerVec = 8;
  __device__ static float to_float(uint32_t bits16) { return __uint_as_float(bits16 << 16); }
};
template <>
struct Elem<float> {
  static constexpr int kPerVec = 4;
};

__device__ __forceinline__ int8_t quant_one(float v, float s) {
  int r = __float2int_rn(__fdiv_rn(v, s));     // rint(fp32(v / s)), ties to even
  r = r > 127 ? 127 : (r < -127 ? -127 : r);
  return static_cast<int8_t>(r);
}

// fp32 inputs (the weight path): codes without a division, the same result as
// quant_one, with a flagged fallback to the IEEE division.
//
// Let inv = fp32(1 / s) and p = v * inv taken exactly (inside an FMA).  inv's
// rounding gives |p - v/s| <= |v/s| 2^-24 < 2^-17, because |v / s| <=
// 127 * (1 + 2^-23) (s >= absmax / 127 up to one rounding).  The correctly
// rounded quotient q* = fp32(v / s) is within half an fp32 ulp of v/s, at most
// 2^-18 below 128, so |p - q*| < 2^-16.  rint() can only tell p and q* apart if
// a half-integer lies between them (or q* is one); so when p is farther than
// 2^-15 from every half-integer, rint(p) == rint(q*) (and it lies in [-127,
// 127], so no clamp is needed).  Otherwise the caller redoes the vector with
// the exact IEEE division.
//
// rint(p) comes from t = fma(v, inv, 1.5 * 2^23): for |p| < 2^22 the exact sum
// lies in [2^23, 2^24) where the fp32 spacing is 1, so its round-to-nearest-
// even is 1.5 * 2^23 + rint_half_even(p) (1.5 * 2^23 is even); the low byte of
// t's bit pattern is rint(p) as a two's-complement int8, and r = t - 1.5 * 2^23
// is exact.  e = fma(v, inv, -r) is p - r (the distance to the nearest
// integer) with one rounding (error <= 2^-25); p is treated as near a
// half-integer when |e| >= 1/2 - 2^-14, a margin that covers that rounding.
// That test runs as d = fma(e, e, -c) with c = 1/4 - 2^-14 (exact in fp32,
// just below (1/2 - 2^-14)^2): d >= 0 (sign bit clear) whenever |e| >=
// 1/2 - 2^-14, so AND-ing the sign bits of a vector's d values flags it.
//
// The fp32 work runs as packed pairs (sm_100 f32x2 fma/sub, each lane of the
// pair rounded like the scalar instruction).
constexpr float kMagic = 12582912.0f;            // 1.5 * 2^23
constexpr float kNearSq = 0.24993896484375f;     // 1/4 - 2^-14

// Two codes (low bytes of the two t's) for the pair v; `tie` keeps the AND of
// the d sign bits (bit 31 clear once any code is near a tie), d0 / d1 the
// two d values' bits.
__device__ __forceinline__ void quant_pair(uint64_t v, uint64_t inv2, uint64_t magic2, uint64_t negc2,
                                           uint32_t& tie, uint32_t& t0, uint32_t& t1, uint32_t& d0,
                                           uint32_t& d1) {
  const uint64_t t = fma_f2(v, inv2, magic2);
  const uint64_t neg_r = sub_f2(magic2, t);          // -rint(p), exact
  const uint64_t e = fma_f2(v, inv2, neg_r);
  const uint64_t d = fma_f2(e, e, negc2);
  d0 = static_cast<uint32_t>(d);
  d1 = static_cast<uint32_t>(d >> 32);
  tie &= d0 & d1;
  t0 = static_cast<uint32_t>(t);
  t1 = static_cast<uint32_t>(t >> 32);
}

__device__ __forceinline__ uint32_t pack_low_bytes(uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
  return __byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410);
}

// bf16 inputs: the correctly rounded quotient without a division, by
// Markstein's correction step (P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1),
// 1990): q0 = fp32(v * inv), r = fma(-q0, s, v) (exact), q1 = fma(r, inv, q0)
// = fp32(v / s); then rint(q1) by the 1.5 * 2^23 addition (ties to even, as
// q1 is the exact fp32 quotient).  For every positive bf16 absmax and every
// bf16 value v with |v| <= absmax, rint(q1) equals rint(fp32(v / s)) (checked
// exhaustively against IEEE division; q1 itself differs only for quotients
// below 1/4, where r underflows, and those round to 0 either way).
__device__ __forceinline__ void quant_pair_bf16(uint64_t v, uint64_t inv2, uint64_t negs2, uint64_t magic2,
                                                uint32_t& t0, uint32_t& t1) {
  const uint64_t q0 = mul_f2(v, inv2);
  const uint64_t r = fma_f2(q0, negs2, v);
  const uint64_t q1 = fma_f2(r, inv2, q0);
  const uint64_t t = add_f2(q1, magic2);
  t0 = static_cast<uint32_t>(t);
  t1 = static_cast<uint32_t>(t >> 32);
}

// Codes of one 16-byte vector of 8 bf16 values (w = 4 packed words) as two
// words of int8 codes.
__device__ __forceinline__ uint2 quant_bf16x8(const uint32_t (&w)[4], uint64_t inv2, uint64_t negs2,
                                              uint64_t magic2) {
  uint32_t b[8];
#pragma unroll
  for (int h = 0; h < 4; ++h)
    quant_pair_bf16(pack_f2(__uint_as_float(w[h] << 16), __uint_as_float(w[h] & 0xffff0000u)), inv2, negs2,
                    magic2, b[2 * h], b[2 * h + 1]);
  return make_uint2(pack_low_bytes(b[0], b[1], b[2], b[3]), pack_low_bytes(b[4], b[5], b[6], b[7]));
}

// Output formats: int8 codes (absmax / 127) or e4m3 codes (absmax / 448, the
// largest e4m3 value; the vLLM quantization commits' dynamic FP8 scaling with
// the scaled values clamped to the e4m3 range).
enum class QFmt : int { I8 = 0, E4M3 = 1 };

template <QFmt F = QFmt::I8>
__device__ __forceinline__ float scale_from_absmax(float a) {
  return __fdiv_rn(fmaxf(a, 1e-8f), F == QFmt::E4M3 ? 448.0f : 127.0f);
}

// Two fp32 values -> two e4m3 codes (round to nearest even; magnitudes above
// 448 saturate to 448, which is the clamp), lo in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// e4m3 codes of 8 bf16 values (4 packed words): the quotient by Markstein's
// correction step as in the int8 path (for bf16 inputs and s = absmax / 448
// its e4m3 code equals the IEEE quotient's, checked for every bf16 pair), then
// one conversion per pair.
__device__ __forceinline__ uint2 quant_bf16x8_e4m3(const uint32_t (&w)[4], uint64_t inv2, uint64_t negs2) {
  uint32_t c[4];
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    const uint64_t v = pack_f2(__uint_as_float(w[h] << 16), __uint_as_float(w[h] & 0xffff0000u));
    const uint64_t q0 = mul_f2(v, inv2);
    const uint64_t r = fma_f2(q0, negs2, v);
    const uint64_t q1 = fma_f2(r, inv2, q0);
    float lo, hi;
    unpack_f2(q1, lo, hi);
    c[h] = e4m3x2(lo, hi);
  }
  return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

// e4m3 codes of 4 fp32 values (weights, offline): the IEEE quotient itself.
__device__ __forceinline__ uint32_t quant_f32x4_e4m3(uint4 v, float s) {
  return e4m3x2(__fdiv_rn(__uint_as_float(v.x), s), __fdiv_rn(__uint_as_float(v.y), s)) |
         (e4m3x2(__fdiv_rn(__uint_as_float(v.z), s), __fdiv_rn(__uint_as_float(v.w), s)) << 16);
}

__device__ __forceinline__ uint32_t pack4(int8_t a, int8_t b, int8_t c, int8_t d) {
  return (static_cast<uint32_t>(static_cast<uint8_t>(a))) |
         (static_cast<uint32_t>(static_cast<uint8_t>(b)) << 8) |
         (static_cast<uint32_t>(static_cast<uint8_t>(c)) << 16) |
         (static_cast<uint32_t>(static_cast<uint8_t>(d)) << 24);
}

// Exact codes (IEEE division) of one 16-byte vector of 4 fp32 values.  Out
// of line on purpose: it runs only for a vector holding a code near a tie
// (fp32 inputs rarely have one), and as a call the compiler cannot if-convert
// its divisions into the common path.
__device__ __noinline__ uint32_t quant_f32x4_exact(uint4 v, float s) {
  return pack4(quant_one(__uint_as_float(v.x), s), quant_one(__uint_as_float(v.y), s),
               quant_one(__uint_as_float(v.z), s), quant_one(__uint_as_float(v.w), s));
}

// Register-resident single-pass kernel.  256 threads; a row is owned by
// 2^tpr_log2 consecutive threads (32..256); VPT = max 16-byte vectors per
// thread.
template <typename T, int VPT, QFmt F = QFmt::I8>
__global__ void __launch_bounds__(256) quant_rows_vec_kernel(const T* __restrict__ x, int64_t M,
                                                             int64_t K, int64_t ldx,
                                                             int8_t* __restrict__ q, int64_t ldq,
                                                             float* __restrict__ scales,
                                                             int tpr_log2) {
  constexpr int E = Elem<T>::kPerVec;
  griddep_launch_dependents();     // the next kernel (e.g. the GEMM) may start its prologue
  // Launched with programmatic stream serialization: the previous kernel of
  // the stream (which may still read q or scales, or write x) is complete and
  // its writes visible before this kernel touches global memory.
  griddep_wait();
  const int tpr = 1 << tpr_log2;
  const int t = threadIdx.x & (tpr - 1);
  const int r_local = threadIdx.x >> tpr_log2;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (256 >> tpr_log2) + r_local;
  const int nv = static_cast<int>(K / E);
  __shared__ uint32_t warp_max[8];

  uint4 v[VPT];
  uint32_t amax = 0;
  if (row < M) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + row * ldx);
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int vi = t + i * tpr;
      if (vi < nv) v[i] = __ldcs(xr + vi);
    }
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int vi = t + i * tpr;
      if (vi < nv) {
        if constexpr (E == 8) {
          // |x| of both halves, max per half (bf16x2 max: exact for finite values)
          const uint32_t w4[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            __nv_bfloat162 xv = *reinterpret_cast<const __nv_bfloat162*>(&w4[h]);
            __nv_bfloat162 av = *reinterpret_cast<__nv_bfloat162*>(&amax);
            av = __hmax2(av, __habs2(xv));
            amax = *reinterpret_cast<uint32_t*>(&av);
          }
        } else {
          float af = __uint_as_float(amax);
          af = fmaxf(af, fabsf(__uint_as_float(v[i].x)));
          af = fmaxf(af, fabsf(__uint_as_float(v[i].y)));
          af = fmaxf(af, fabsf(__uint_as_float(v[i].z)));
          af = fmaxf(af, fabsf(__uint_as_float(v[i].w)));
          amax = __float_as_uint(af);
        }
      }
    }
    if constexpr (E == 8) amax = max(amax & 0xffffu, amax >> 16) << 16;   // to fp32 bits
  }
  amax = __reduce_max_sync(0xffffffffu, amax);
  if (tpr > 32) {
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) warp_max[warp] = amax;
    __syncthreads();
    const int wpr = tpr >> 5;
    const int w0 = r_local * wpr;
    amax = 0;
    for (int w = 0; w < wpr; ++w) amax = max(amax, warp_max[w0 + w]);
  }
  if (row >= M) return;
  const float s = scale_from_absmax<F>(__uint_as_float(amax));
  const float inv = __frcp_rn(s);
  if (t == 0) scales[row] = s;

  const float inv1 = inv;
  const uint64_t inv2 = pack_f2(inv1, inv1);
  const uint64_t magic2 = pack_f2(kMagic, kMagic);
  const uint64_t negc2 = pack_f2(-kNearSq, -kNearSq);
  const uint64_t negs2 = pack_f2(-s, -s);
  int8_t* qr = q + row * ldq;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int vi = t + i * tpr;
    if (vi < nv) {
      const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
      if constexpr (F == QFmt::E4M3) {
        if constexpr (E == 8)
          *reinterpret_cast<uint2*>(qr + static_cast<int64_t>(vi) * 8) = quant_bf16x8_e4m3(w, inv2, negs2);
        else
          *reinterpret_cast<uint32_t*>(qr + static_cast<int64_t>(vi) * 4) = quant_f32x4_e4m3(v[i], s);
      } else if constexpr (E == 8) {
        *reinterpret_cast<uint2*>(qr + static_cast<int64_t>(vi) * 8) = quant_bf16x8(w, inv2, negs2, magic2);
      } else {
        uint32_t tie = 0xffffffffu, b[4], dd[4];
        quant_pair(pack_f2(__uint_as_float(w[0]), __uint_as_float(w[1])), inv2, magic2, negc2, tie, b[0], b[1],
                   dd[0], dd[1]);
        quant_pair(pack_f2(__uint_as_float(w[2]), __uint_as_float(w[3])), inv2, magic2, negc2, tie, b[2], b[3],
                   dd[2], dd[3]);
        uint32_t out = pack_low_bytes(b[0], b[1], b[2], b[3]);
        if (!(tie >> 31)) out = quant_f32x4_exact(v[i], s);
        *reinterpret_cast<uint32_t*>(qr + static_cast<int64_t>(vi) * 4) = out;
      }
    }
  }
}

template <typename T>
__device__ __forceinline__ float load_as_float(const T* p);
template <>
__device__ __forceinline__ float load_as_float<uint16_t>(const uint16_t* p) {
  return __uint_as_float(static_cast<uint32_t>(*p) << 16);
}
template <>
__device__ __forceinline__ float load_as_float<float>(const float* p) {
  return *p;
}

// Any shape, stride or alignment: one CTA of 256 threads per row, two passes
// over the row (the second mostly from L2).
template <typename T, QFmt F = QFmt::I8>
__global__ void __launch_bounds__(256) quant_rows_generic_kernel(const T* __restrict__ x, int64_t M,
                                                                 int64_t K, int64_t ldx,
                                                                 int8_t* __restrict__ q,
                                                                 int64_t ldq,
                                                                 float* __restrict__ scales) {
  __shared__ float warp_max[8];
  for (int64_t row = blockIdx.x; row < M; row += gridDim.x) {
    const T* xr = x + row * ldx;
    float a = 0.0f;
    for (int64_t k = threadIdx.x; k < K; k += 256) a = fmaxf(a, fabsf(load_as_float<T>(xr + k)));
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = a;
    __syncthreads();
    a = warp_max[0];
    for (int w = 1; w < 8; ++w) a = fmaxf(a, warp_max[w]);
    __syncthreads();
    const float s = scale_from_absmax<F>(a);
    if (threadIdx.x == 0) scales[row] = s;
    int8_t* qr = q + row * ldq;
    for (int64_t k = threadIdx.x; k < K; k += 256) {
      if constexpr (F == QFmt::E4M3) {
        const float qv = __fdiv_rn(load_as_float<T>(xr + k), s);
        qr[k] = static_cast<int8_t>(e4m3x2(qv, 0.0f) & 0xffu);
      } else {
        qr[k] = quant_one(load_as_float<T>(xr + k), s);
      }
    }
  }
}

// ---------------------------------------------------------------- pipelined rows
//
// Memory-pipelined kernel for rows of 1 KB .. 16 KB: one CTA per SM walks a
// contiguous block of rows.  Lane 0 of warp 0 streams whole rows into a ring
// of shared-memory stages with 1-D bulk copies (cp.async.bulk, completion on
// the stage's mbarrier), so up to QT_RING_BYTES of loads stay in flight per SM
// while warps 1..16 compute.  Each consumer warp owns a row: pass 1 reduces
// |x| (bf16x2 max, then a warp max), pass 2 writes the codes with coalesced
// stores straight from the stage.
constexpr int QT_CONSUMERS = 24;
constexpr int QT_THREADS = 32 * (1 + QT_CONSUMERS);
constexpr int QT_RING_BYTES = 192 * 1024;
constexpr int QT_MAX_ROW_BYTES = 16 * 1024;

__device__ __forceinline__ void bulk_load_1d(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

template <typename T>
__global__ void __launch_bounds__(QT_THREADS, 1)
    quant_rows_tma_kernel(const T* __restrict__ x, int64_t M, int K, int64_t ldx, int8_t* __restrict__ q,
                          int64_t ldq, float* __restrict__ scales, int stages, int stage_bytes, int wpr,
                          WaitCtl wait) {
  constexpr int E = Elem<T>::kPerVec;             // elements per 16-byte chunk
  griddep_launch_dependents();     // the next kernel (e.g. the GEMM) may start its prologue
  extern __shared__ __align__(128) uint8_t qsmem[];
  __shared__ __align__(8) uint64_t full_bar[QT_RING_BYTES / 1024];
  __shared__ __align__(8) uint64_t empty_bar[QT_RING_BYTES / 1024];
  __shared__ int abort_flag;
  __shared__ uint32_t part_max[QT_CONSUMERS];
  __shared__ int group_ok[QT_CONSUMERS];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t G = gridDim.x;
  const int64_t r0 = blockIdx.x * M / G, r1 = (blockIdx.x + 1) * M / G;
  const int nrows = static_cast<int>(r1 - r0);
  const uint32_t row_bytes = static_cast<uint32_t>(K) * sizeof(T);
  const int nchunks = K / E;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int i = 0; i < stages; ++i) {
      mbar_init(smem_u32(full_bar + i), 1);
      mbar_init(smem_u32(empty_bar + i), 1);
    }
    fence_barrier_init();
  }
  __syncthreads();
  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int j = 0; j < nrows; ++j) {
        const int st = j % stages;
        const uint32_t ph = static_cast<uint32_t>(j / stages) & 1u;
        if (!mbar_wait(smem_u32(empty_bar + st), ph ^ 1u, wait, &abort_flag)) break;
        const uint32_t fb = smem_u32(full_bar + st);
        mbar_arrive_expect_tx(fb, row_bytes);
        bulk_load_1d(smem_u32(qsmem + st * stage_bytes), x + (r0 + j) * ldx, row_bytes, fb);
        ++issued;
      }
      if (issued < nrows) {
        // Gave up: let the loads already issued land (bounded, short waits).
        WaitCtl quick = wait;
        quick.timeout_ns = quick.timeout_ns < 50000000ull ? quick.timeout_ns : 50000000ull;
        volatile int never = 0;
        for (int j = issued - stages > 0 ? issued - stages : 0; j < issued; ++j)
          mbar_wait(smem_u32(full_bar + j % stages), static_cast<uint32_t>(j / stages) & 1u, quick, &never);
      }
    }
  } else {
    // Rows go round-robin to the QT_CONSUMERS / wpr groups of `wpr` warps
    // (wpr = 1, 2 or 4); the warps of a group split the row's 16-byte chunks
    // and combine their partial maxima through shared memory under the
    // group's named barrier.  `stages` is a multiple of the group count (the
    // launch checks it), so all rows of one stage belong to one group: the
    // group has consumed the stage's previous lap before it waits for the
    // next (try_wait.parity cannot tell lap L from lap L - 2).
    const int groups = QT_CONSUMERS / wpr;
    const int cw = warp - 1;
    const int grp = cw / wpr, wig = cw % wpr;
    const int bar_id = 1 + grp;                  // named barriers 1..groups
    const int cstep = 32 * wpr;
    for (int j = grp; grp < groups && j < nrows; j += groups) {
      const int st = j % stages;
      const uint32_t ph = static_cast<uint32_t>(j / stages) & 1u;
      if (wpr > 1) {
        // Only the group's first warp waits; the whole group then follows its
        // verdict, so no warp can be left alone at the group barrier.
        if (wig == 0) {
          const bool ok = mbar_wait(smem_u32(full_bar + st), ph, wait, &abort_flag);
          if (lane == 0) group_ok[grp] = ok ? 1 : 0;
        }
        named_bar_sync(bar_id, 32 * wpr);
        if (!group_ok[grp]) break;
      } else if (!mbar_wait(smem_u32(full_bar + st), ph, wait, &abort_flag)) {
        break;
      }
      const uint4* src = reinterpret_cast<const uint4*>(qsmem + st * stage_bytes);
      // pass 1: absmax
      uint32_t amax;
      if constexpr (E == 8) {
        __nv_bfloat162 am = __floats2bfloat162_rn(0.0f, 0.0f);
#pragma unroll 4
        for (int c = lane + 32 * wig; c < nchunks; c += cstep) {
          const uint4 v = src[c];
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) am = __hmax2(am, __habs2(*reinterpret_cast<const __nv_bfloat162*>(&w[h])));
        }
        const uint32_t ab = *reinterpret_cast<uint32_t*>(&am);
        amax = max(ab & 0xffffu, ab >> 16) << 16;
      } else {
        float af = 0.0f;
#pragma unroll 4
        for (int c = lane + 32 * wig; c < nchunks; c += cstep) {
          const uint4 v = src[c];
          af = fmaxf(af, fmaxf(fmaxf(fabsf(__uint_as_float(v.x)), fabsf(__uint_as_float(v.y))),
                               fmaxf(fabsf(__uint_as_float(v.z)), fabsf(__uint_as_float(v.w)))));
        }
        amax = __float_as_uint(af);
      }
      amax = __reduce_max_sync(0xffffffffu, amax);
      if (wpr > 1) {
        if (lane == 0) part_max[cw] = amax;
        named_bar_sync(bar_id, 32 * wpr);
        for (int w = 0; w < wpr; ++w) amax = max(amax, part_max[grp * wpr + w]);
      }
      const float s = scale_from_absmax(__uint_as_float(amax));
      const float inv = __frcp_rn(s);
      const int64_t row = r0 + j;
      if (lane == 0 && wig == 0) scales[row] = s;
      const uint64_t inv2 = pack_f2(inv, inv);
      const uint64_t magic2 = pack_f2(kMagic, kMagic);
      const uint64_t negc2 = pack_f2(-kNearSq, -kNearSq);
      int8_t* qr = q + row * ldq;
      const uint64_t negs2 = pack_f2(-s, -s);
      // pass 2: codes
#pragma unroll 2
      for (int c = lane + 32 * wig; c < nchunks; c += cstep) {
        const uint4 v = src[c];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        if constexpr (E == 8) {
          *reinterpret_cast<uint2*>(qr + static_cast<int64_t>(c) * 8) = quant_bf16x8(w, inv2, negs2, magic2);
        } else {
          uint32_t tie = 0xffffffffu, b[4], dd[4];
          quant_pair(pack_f2(__uint_as_float(w[0]), __uint_as_float(w[1])), inv2, magic2, negc2, tie, b[0], b[1],
                     dd[0], dd[1]);
          quant_pair(pack_f2(__uint_as_float(w[2]), __uint_as_float(w[3])), inv2, magic2, negc2, tie, b[2], b[3],
                     dd[2], dd[3]);
          uint32_t out = pack_low_bytes(b[0], b[1], b[2], b[3]);
          if (!(tie >> 31)) out = quant_f32x4_exact(v, s);
          *reinterpret_cast<uint32_t*>(qr + static_cast<int64_t>(c) * 4) = out;
        }
      }
      // every warp of the group is done with the stage (and with part_max)
      if (wpr > 1) named_bar_sync(bar_id, 32 * wpr);
      else __syncwarp();
      if (lane == 0 && wig == 0) mbar_arrive(smem_u32(empty_bar + st));
    }
  }
  __syncthreads();      // no CTA leaves with a bulk load still landing in its ring
}

template <typename T, QFmt F = QFmt::I8>
dq_status launch_quantize(const T* x, int64_t M, int64_t K, int64_t ldx, int8_t* q, int64_t ldq,
                          float* scales, cudaStream_t stream) {
  if (M < 0 || K < 1 || ldx < K || ldq < K) return DQ_ERR_INVALID_ARG;
  if (M > 0 && (x == nullptr || q == nullptr || scales == nullptr)) return DQ_ERR_INVALID_ARG;
  if (M > (int64_t(1) << 31) - 1) return DQ_ERR_UNSUPPORTED;
  DeviceInfo* d = nullptr;
  dq_status st = current_device(&d);
  if (st != DQ_OK) return st;
  if (M == 0) return DQ_OK;

  constexpr int E = Elem<T>::kPerVec;
  const int64_t nv = K / E;
  const bool vec_ok = (K % E == 0) && (ldx % E == 0) && aligned(x, 16) && (ldq % E == 0) &&
                      aligned(q, E) && nv <= 256 * 8;
  const int64_t row_bytes = K * static_cast<int64_t>(sizeof(T));
  // Measured on B200 (bf16 rows of 256 B .. 32 KB, 16 .. 65792 rows): with
  // the division-free rounding the register kernel is the faster one for every
  // shape (16384 x 8192: 6.0 TB/s against 5.6-5.8 for the pipelined kernel),
  // so the pipelined kernel runs only when asked for.
  const bool tma_ok = vec_ok && row_bytes >= 1024 && row_bytes <= QT_MAX_ROW_BYTES;
  const bool tma_pick = g_quant_kernel_override == 2 && F == QFmt::I8;   // int8 codes only
  if (tma_ok && tma_pick) {
    // stage = one row rounded up to 128 bytes; at most as many stages as the
    // ring holds (<= 192).
    const int stage_bytes = static_cast<int>((row_bytes + 127) / 128 * 128);
    int max_stages = QT_RING_BYTES / stage_bytes;
    if (max_stages > QT_RING_BYTES / 1024) max_stages = QT_RING_BYTES / 1024;
    // Rows go round-robin to QT_CONSUMERS / wpr groups of wpr warps.  The
    // stage count is a multiple of the group count, so a stage's rows (j,
    // j + stages, ...) all belong to one group, which therefore has consumed
    // the stage's previous lap before it waits for the next one: the parity
    // wait can never see lap L - 2 as lap L.  wpr grows until at least 4
    // stages stay loading beyond the rows being worked on (measured: 16 KB
    // rows best with 4 warps per row).
    int wpr = 1;
    while (wpr < 4) {
      const int grp = QT_CONSUMERS / wpr;
      if ((max_stages / grp) * grp - grp >= 4) break;
      wpr *= 2;
    }
    const int groups = QT_CONSUMERS / wpr;
    const int stages = (max_stages / groups) * groups;
    if (stages < groups) return DQ_ERR_UNSUPPORTED;    // not reachable for rows <= 16 KB
    const int smem = stages * stage_bytes;
    const dq_status ast = smem_limit_once(reinterpret_cast<const void*>(&quant_rows_tma_kernel<T>), QT_RING_BYTES);
    if (ast != DQ_OK) return ast;
    const int64_t grid = M < d->sm_count ? M : d->sm_count;
    WaitCtl wait{d->err_word, wait_timeout_ns()};
    quant_rows_tma_kernel<T><<<static_cast<unsigned>(grid), QT_THREADS, smem, stream>>>(
        x, M, static_cast<int>(K), ldx, q, ldq, scales, stages, stage_bytes, wpr, wait);
  } else if (vec_ok) {
    int tpr_log2 = 5;
    while ((int64_t(1) << tpr_log2) * 8 < nv) ++tpr_log2;     // tpr * 8 >= nv, tpr <= 256
    // Few rows: spread each row over more threads (fewer vectors each) so the
    // grid fills the SMs several times over and per-thread chains are short.
    while (tpr_log2 < 8 && ((int64_t(1) << tpr_log2) * 8 <= nv) &&
           (M * (int64_t(1) << tpr_log2)) / 256 < int64_t(d->sm_count) * 4)
      ++tpr_log2;
    // bf16 rows of 16 KB and more: at most four vectors per thread over up
    // to 256 threads (measured on B200, 16384 x 8192: 59.7 us with four
    // vectors per thread against 67.2 us with eight; 2.5 and 8 KB rows are
    // faster as chosen above).
    if (E == 8 && nv >= 1024)
      while (tpr_log2 < 8 && (int64_t(1) << tpr_log2) * 4 < nv) ++tpr_log2;
    const int64_t tpr = int64_t(1) << tpr_log2;
    const int64_t vpt = (nv + tpr - 1) / tpr;
    const int64_t rows_per_cta = 256 / tpr;
    const int64_t grid = (M + rows_per_cta - 1) / rows_per_cta;
    if (grid > 0x7fffffff) return DQ_ERR_UNSUPPORTED;
    // Programmatic stream serialization: the launch and the CTAs' start
    // overlap the tail of the previous kernel; the kernel waits for it
    // (griddepcontrol.wait) before its first global memory access.
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t le;
    if (vpt <= 1)
      le = cudaLaunchKernelEx(&cfg, quant_rows_vec_kernel<T, 1, F>, x, M, K, ldx, q, ldq, scales, tpr_log2);
    else if (vpt <= 2)
      le = cudaLaunchKernelEx(&cfg, quant_rows_vec_kernel<T, 2, F>, x, M, K, ldx, q, ldq, scales, tpr_log2);
    else if (vpt <= 4)
      le = cudaLaunchKernelEx(&cfg, quant_rows_vec_kernel<T, 4, F>, x, M, K, ldx, q, ldq, scales, tpr_log2);
    else
      le = cudaLaunchKernelEx(&cfg, quant_rows_vec_kernel<T, 8, F>, x, M, K, ldx, q, ldq, scales, tpr_log2);
    if (le != cudaSuccess) return cuda_fail(le);
  } else {
    const int64_t grid = M < int64_t(d->sm_count) * 16 ? M : int64_t(d->sm_count) * 16;
    quant_rows_generic_kernel<T, F><<<static_cast<unsigned>(grid), 256, 0, stream>>>(x, M, K, ldx, q,
                                                                                 ldq, scales);
  }
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? DQ_OK : cuda_fail(e);
}

}  // namespace
}  // namespace dq

extern "C" {

dq_status dq_quantize_rows(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, int8_t* q,
                           int64_t ldq, float* scales, dq_stream_t stream) {
  return dq::launch_quantize<uint16_t>(static_cast<const uint16_t*>(x_bf16), M, K, ldx, q, ldq,
                                       scales, reinterpret_cast<cudaStream_t>(stream));
}

dq_status dq_quantize_weight(const float* w, int64_t N, int64_t K, int64_t ldw, int8_t* wq,
                             int64_t ldwq, float* s_col, dq_stream_t stream) {
  return dq::launch_quantize<float>(w, N, K, ldw, wq, ldwq, s_col,
                                    reinterpret_cast<cudaStream_t>(stream));
}

dq_status dq_quantize_rows_fp8(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, uint8_t* q,
                               int64_t ldq, float* scales, dq_stream_t stream) {
  return dq::launch_quantize<uint16_t, dq::QFmt::E4M3>(static_cast<const uint16_t*>(x_bf16), M, K, ldx,
                                                       reinterpret_cast<int8_t*>(q), ldq, scales,
                                                       reinterpret_cast<cudaStream_t>(stream));
}

dq_status dq_quantize_weight_fp8(const float* w, int64_t N, int64_t K, int64_t ldw, uint8_t* wq,
                                 int64_t ldwq, float* s_col, dq_stream_t stream) {
  return dq::launch_quantize<float, dq::QFmt::E4M3>(w, N, K, ldw, reinterpret_cast<int8_t*>(wq), ldwq, s_col,
                                                    reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
