// quantize.cu -- per-row symmetric absmax int8 quantization.
//
// Per-token dynamic quantization of activations ("int8 dynamic quant + bsr
// support", pytorch/ao PR 821) with the absmax/127 symmetric scale (Paddle
// "sparse_fc supported", PR 41770, SpmmPluginDynamic), and the same formula
// per output channel for the weight:
//     s = fp32( max(absmax, 1e-8f) / 127 ),  q = clamp(rint(x / s), -127, 127)
// with IEEE round-to-nearest-even division (no reciprocal): the result is
// bit-identical to a scalar IEEE evaluation.
//
// The hot kernel keeps a whole row in registers: each row is owned by a
// power-of-two group of 32..256 threads, each thread loads up to 8 16-byte
// vectors (one HBM pass), the group reduces |x| with integer max on the bit
// patterns (exact for finite values: a non-negative IEEE value orders like its
// bits), and the codes are written straight from registers.
#include <cuda_bf16.h>

#include <mutex>

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

// Codes without a division, the same result as quant_one.
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
//
// The fp32 work runs as packed pairs (sm_100 f32x2 fma/sub, each lane of the
// pair rounded like the scalar instruction).
constexpr float kMagic = 12582912.0f;            // 1.5 * 2^23
constexpr float kNear = 0.49993896484375f;       // 1/2 - 2^-14

// Two codes (low bytes of the two t's) for the pair v; tracks max |e|.
__device__ __forceinline__ void quant_pair(uint64_t v, uint64_t inv2, uint64_t magic2, float& emax,
                                           uint32_t& t0, uint32_t& t1) {
  const uint64_t t = fma_f2(v, inv2, magic2);
  const uint64_t neg_r = sub_f2(magic2, t);          // -rint(p), exact
  const uint64_t e = fma_f2(v, inv2, neg_r);
  float e0, e1, f0, f1;
  unpack_f2(e, e0, e1);
  emax = fmaxf(emax, fmaxf(fabsf(e0), fabsf(e1)));
  unpack_f2(t, f0, f1);
  t0 = __float_as_uint(f0);
  t1 = __float_as_uint(f1);
}

__device__ __forceinline__ uint32_t pack_low_bytes(uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
  return __byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410);
}

__device__ __forceinline__ float scale_from_absmax(float a) {
  return __fdiv_rn(fmaxf(a, 1e-8f), 127.0f);
}

__device__ __forceinline__ uint32_t pack4(int8_t a, int8_t b, int8_t c, int8_t d) {
  return (static_cast<uint32_t>(static_cast<uint8_t>(a))) |
         (static_cast<uint32_t>(static_cast<uint8_t>(b)) << 8) |
         (static_cast<uint32_t>(static_cast<uint8_t>(c)) << 16) |
         (static_cast<uint32_t>(static_cast<uint8_t>(d)) << 24);
}

// Register-resident single-pass kernel.  256 threads; a row is owned by
// 2^tpr_log2 consecutive threads (32..256); VPT = max 16-byte vectors per
// thread.
template <typename T, int VPT>
__global__ void __launch_bounds__(256) quant_rows_vec_kernel(const T* __restrict__ x, int64_t M,
                                                             int64_t K, int64_t ldx,
                                                             int8_t* __restrict__ q, int64_t ldq,
                                                             float* __restrict__ scales,
                                                             int tpr_log2) {
  constexpr int E = Elem<T>::kPerVec;
  griddep_launch_dependents();     // the next kernel (e.g. the GEMM) may start its prologue
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
  const float s = scale_from_absmax(__uint_as_float(amax));
  const float inv = __frcp_rn(s);
  if (t == 0) scales[row] = s;

  const float inv1 = inv;
  const uint64_t inv2 = pack_f2(inv1, inv1);
  const uint64_t magic2 = pack_f2(kMagic, kMagic);
  int8_t* qr = q + row * ldq;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int vi = t + i * tpr;
    if (vi < nv) {
      const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
      float emax = 0.0f;
      if constexpr (E == 8) {
        uint32_t b[8];
#pragma unroll
        for (int h = 0; h < 4; ++h)
          quant_pair(pack_f2(__uint_as_float(w[h] << 16), __uint_as_float(w[h] & 0xffff0000u)), inv2, magic2,
                     emax, b[2 * h], b[2 * h + 1]);
        uint32_t out0 = pack_low_bytes(b[0], b[1], b[2], b[3]);
        uint32_t out1 = pack_low_bytes(b[4], b[5], b[6], b[7]);
        if (emax >= kNear) {   // rare: a code within 2^-14 of a tie, decide by IEEE division
          float f[8];
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            f[2 * h] = __uint_as_float(w[h] << 16);
            f[2 * h + 1] = __uint_as_float(w[h] & 0xffff0000u);
          }
          out0 = pack4(quant_one(f[0], s), quant_one(f[1], s), quant_one(f[2], s), quant_one(f[3], s));
          out1 = pack4(quant_one(f[4], s), quant_one(f[5], s), quant_one(f[6], s), quant_one(f[7], s));
        }
        *reinterpret_cast<uint2*>(qr + static_cast<int64_t>(vi) * 8) = make_uint2(out0, out1);
      } else {
        uint32_t b[4];
        quant_pair(pack_f2(__uint_as_float(w[0]), __uint_as_float(w[1])), inv2, magic2, emax, b[0], b[1]);
        quant_pair(pack_f2(__uint_as_float(w[2]), __uint_as_float(w[3])), inv2, magic2, emax, b[2], b[3]);
        uint32_t out = pack_low_bytes(b[0], b[1], b[2], b[3]);
        if (emax >= kNear)
          out = pack4(quant_one(__uint_as_float(w[0]), s), quant_one(__uint_as_float(w[1]), s),
                      quant_one(__uint_as_float(w[2]), s), quant_one(__uint_as_float(w[3]), s));
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
template <typename T>
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
    const float s = scale_from_absmax(a);
    if (threadIdx.x == 0) scales[row] = s;
    int8_t* qr = q + row * ldq;
    for (int64_t k = threadIdx.x; k < K; k += 256) qr[k] = quant_one(load_as_float<T>(xr + k), s);
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
    // A consumer must never get more than one ring lap ahead of the rows it
    // waits for (try_wait.parity cannot tell phase k from phase k-2), so only
    // min(QT_CONSUMERS, stages) warps take rows, each stepping by that count.
    // Rows go to groups of `wpr` warps (wpr = 1, 2 or 4; QT_CONSUMERS/wpr
    // groups, at most `stages` of them, see above); the warps of a group split
    // the row's 16-byte chunks and combine their partial maxima through
    // shared memory under the group's named barrier.
    const int groups_all = QT_CONSUMERS / wpr;
    const int groups = groups_all < stages ? groups_all : stages;
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
      int8_t* qr = q + row * ldq;
      // pass 2: codes
#pragma unroll 2
      for (int c = lane + 32 * wig; c < nchunks; c += cstep) {
        const uint4 v = src[c];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        float emax = 0.0f;
        if constexpr (E == 8) {
          uint32_t b[8];
#pragma unroll
          for (int h = 0; h < 4; ++h)
            quant_pair(pack_f2(__uint_as_float(w[h] << 16), __uint_as_float(w[h] & 0xffff0000u)), inv2, magic2,
                       emax, b[2 * h], b[2 * h + 1]);
          uint32_t out0 = pack_low_bytes(b[0], b[1], b[2], b[3]);
          uint32_t out1 = pack_low_bytes(b[4], b[5], b[6], b[7]);
          if (emax >= kNear) {
            float f[8];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              f[2 * h] = __uint_as_float(w[h] << 16);
              f[2 * h + 1] = __uint_as_float(w[h] & 0xffff0000u);
            }
            out0 = pack4(quant_one(f[0], s), quant_one(f[1], s), quant_one(f[2], s), quant_one(f[3], s));
            out1 = pack4(quant_one(f[4], s), quant_one(f[5], s), quant_one(f[6], s), quant_one(f[7], s));
          }
          *reinterpret_cast<uint2*>(qr + static_cast<int64_t>(c) * 8) = make_uint2(out0, out1);
        } else {
          uint32_t b[4];
          quant_pair(pack_f2(__uint_as_float(w[0]), __uint_as_float(w[1])), inv2, magic2, emax, b[0], b[1]);
          quant_pair(pack_f2(__uint_as_float(w[2]), __uint_as_float(w[3])), inv2, magic2, emax, b[2], b[3]);
          uint32_t out = pack_low_bytes(b[0], b[1], b[2], b[3]);
          if (emax >= kNear)
            out = pack4(quant_one(__uint_as_float(w[0]), s), quant_one(__uint_as_float(w[1]), s),
                        quant_one(__uint_as_float(w[2]), s), quant_one(__uint_as_float(w[3]), s));
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

// Measurement knob: 0 = automatic, 1 = register kernel, 2 = pipelined kernel.
int g_quant_kernel_override = 0;

template <typename T>
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
  // Measured on B200: the pipelined kernel wins for long rows (>= 9 KB); for
  // shorter rows its per-row fixed cost loses to the register kernel.
  const bool tma_ok = vec_ok && row_bytes >= 1024 && row_bytes <= QT_MAX_ROW_BYTES;
  const bool tma_pick = g_quant_kernel_override == 2 || (g_quant_kernel_override == 0 && row_bytes >= 9 * 1024);
  if (tma_ok && tma_pick) {
    // stage = one row rounded up to 128 bytes; as many stages as the ring holds (<= 192)
    const int stage_bytes = static_cast<int>((row_bytes + 127) / 128 * 128);
    int stages = QT_RING_BYTES / stage_bytes;
    if (stages > QT_RING_BYTES / 1024) stages = QT_RING_BYTES / 1024;
    const int smem = stages * stage_bytes;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
      attr_err = cudaFuncSetAttribute(quant_rows_tma_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      QT_RING_BYTES);
    });
    if (attr_err != cudaSuccess) return cuda_fail(attr_err);
    const int64_t grid = M < d->sm_count ? M : d->sm_count;
    // warps per row: leave at least 4 ring stages loading beyond the rows
    // being worked on (measured best: 16 KB rows 4 warps, 10 KB rows 2)
    int wpr = 1;
    while (wpr < 4 && QT_CONSUMERS / wpr > stages - 4) wpr *= 2;
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
    const int64_t tpr = int64_t(1) << tpr_log2;
    const int64_t vpt = (nv + tpr - 1) / tpr;
    const int64_t rows_per_cta = 256 / tpr;
    const int64_t grid = (M + rows_per_cta - 1) / rows_per_cta;
    if (grid > 0x7fffffff) return DQ_ERR_UNSUPPORTED;
    dim3 g(static_cast<unsigned>(grid));
    if (vpt <= 1)
      quant_rows_vec_kernel<T, 1><<<g, 256, 0, stream>>>(x, M, K, ldx, q, ldq, scales, tpr_log2);
    else if (vpt <= 2)
      quant_rows_vec_kernel<T, 2><<<g, 256, 0, stream>>>(x, M, K, ldx, q, ldq, scales, tpr_log2);
    else if (vpt <= 4)
      quant_rows_vec_kernel<T, 4><<<g, 256, 0, stream>>>(x, M, K, ldx, q, ldq, scales, tpr_log2);
    else
      quant_rows_vec_kernel<T, 8><<<g, 256, 0, stream>>>(x, M, K, ldx, q, ldq, scales, tpr_log2);
  } else {
    const int64_t grid = M < int64_t(d->sm_count) * 16 ? M : int64_t(d->sm_count) * 16;
    quant_rows_generic_kernel<T><<<static_cast<unsigned>(grid), 256, 0, stream>>>(x, M, K, ldx, q,
                                                                                 ldq, scales);
  }
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? DQ_OK : cuda_fail(e);
}

}  // namespace
}  // namespace dq

extern "C" {

void dq_debug_set_quant_kernel(int mode) { dq::g_quant_kernel_override = mode; }

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

}  // extern "C"
