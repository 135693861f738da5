// gemm2sm.cu -- the dense int8 x int8 -> int32 GEMM with the fused
// dequantization epilogue (pytorch/ao PR 821, "int8 dynamic quant + bsr
// support": i8i8->bf16 with no int32 intermediate in global memory), with
// each MMA spread over a pair of SMs (a thread-block cluster of 2 CTAs and
// tcgen05.mma.cta_group::2).
//
// Why a pair: with one SM per 128x256 tile, every 128-clock MMA step needs
// 12 KB of operands written into shared memory by TMA and read back by the
// tensor core, which the SM cannot sustain.  A pair computes a 256x256 tile:
// each CTA loads 128 rows of A and 128 rows (half) of B per k step, and the
// pair MMA reads each CTA's halves once for both SMs' tensor cores, so the
// per-SM shared-memory traffic per step drops by a third.
//
// Roles (both CTAs run the same code; rank 0 of the cluster leads):
//   warp 0      TMA producer in each CTA: its A and B halves into its own
//               stage ring; the loads complete on the LEADER's full barrier,
//               which expects the bytes of both CTAs.
//   warp 1      MMA issuer, leader only: tcgen05.mma.cta_group::2.kind::i8
//               (M = 256, N = tile width, K = 32); tcgen05.commit frees the
//               stage in both CTAs (one commit multicast to both) and hands the
//               accumulator to both CTAs' epilogues.
//   warps 2..9  epilogue in each CTA: at the start of a tile one thread
//               copies the tile's column scales and bias into shared memory
//               (1-D bulk copies, done while the MMAs still run); then its 128
//               accumulator rows out of its own TMEM, the same fp32
//               dequantization and TMA-store path as the 1-SM kernel; each
//               warp then tells the leader (remote arrive) that its part of
//               the accumulator is free.
// Schedule: whole tiles round-robin over the pairs.  When whole 256 x 256
// tiles leave a partial last wave (M=2048, N=4096: 128 tiles on 74 pairs),
// the full waves keep 256-wide tiles and the rest of the matrix is cut into
// one wave of narrower tiles (a second weight tensor map with half the box).
// Every load is a plain per-CTA load: each CTA fetches its own operand halves.
#include <atomic>

#include "gemm_common.cuh"

namespace dq {

// BN: pair tile width (output columns); each CTA holds BN/2 rows of B.
template <int BN>
struct Cfg2 {
  static constexpr int KB = kDenseKB;                   // k bytes per stage
  static constexpr int A_BYTES = 128 * KB;              // this CTA's 128 rows of A
  static constexpr int B_BYTES = (BN / 2) * KB;         // this CTA's half of B
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int EPI_WARPS = 8;
  static constexpr int OUT_BUF_BYTES = 32 * 32 * 4;     // per epilogue warp
  static constexpr int OUT_BYTES = EPI_WARPS * OUT_BUF_BYTES;
  static constexpr int BAR_BYTES = 512;                 // mbarriers, TMEM address, abort flag
  static constexpr int ALIGN_SLACK = 1024;              // the 1024-byte alignment of the base
  static constexpr int STAGES = (227 * 1024 - ALIGN_SLACK - BAR_BYTES - OUT_BYTES - kScSlotBytes) / STAGE_BYTES;
  static constexpr int ACC_BUFS = 512 / BN >= 3 ? 3 : 2;  // accumulators of BN TMEM columns
  static constexpr int TMEM_COLS = 512;
  static constexpr int K_STEPS = KB / 32;
  static constexpr int CW = 32;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int OFF_OUT = STAGES * STAGE_BYTES;
  static constexpr int OFF_SC = OFF_OUT + OUT_BYTES;
  static constexpr int OFF_BARS = OFF_SC + kScSlotBytes;
  static constexpr int SMEM_BYTES = OFF_BARS + BAR_BYTES + ALIGN_SLACK;
  static_assert(STAGES >= 3, "stages");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
  static_assert((2 * STAGES + 2 * ACC_BUFS + 3) * 8 + 8 <= BAR_BYTES, "barrier area");
  static_assert(BN % 32 == 0 && BN <= 256 && (BN / 2) % 8 == 0, "tile width");
};

// F8: e4m3 operands (kind::f8f6f4, fp32 accumulator; the epilogue takes the
// accumulator bits as fp32), else int8 (kind::i8, int32).
template <int BN, bool F8>
__global__ void __launch_bounds__(Cfg2<BN>::THREADS, 1)
    gemm2_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                 const __grid_constant__ CUtensorMap tm_b2, const __grid_constant__ CUtensorMap tm_c,
                 const __grid_constant__ GemmArgs g) {
  using C = Cfg2<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint8_t* sOut = smem + C::OFF_OUT;
  const uint32_t sc_slot = smem_u32(smem + C::OFF_SC);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BARS);
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + C::STAGES;
  uint64_t* accf_bar = bars + 2 * C::STAGES;
  uint64_t* acce_bar = accf_bar + C::ACC_BUFS;
  uint64_t* drain_bar = acce_bar + C::ACC_BUFS;
  uint64_t* sc_full = drain_bar + 1;           // the tile's scales have landed in the slot
  uint64_t* sc_free = sc_full + 1;             // every epilogue warp is done reading the slot
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sc_free + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int G = gridDim.x >> 1;                // CTA pairs
  const int pair = blockIdx.x >> 1;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(full_bar + s), 1);
      mbar_init(smem_u32(empty_bar + s), 1);
    }
    for (int a = 0; a < C::ACC_BUFS; ++a) {
      mbar_init(smem_u32(accf_bar + a), 1);
      mbar_init(smem_u32(acce_bar + a), 2 * C::EPI_WARPS);   // one arrive per epilogue warp of both CTAs
    }
    mbar_init(smem_u32(drain_bar), 1);
    mbar_init(smem_u32(sc_full), 1);
    mbar_init(smem_u32(sc_free), C::EPI_WARPS);
    fence_barrier_init();
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
    if (g.bn2 > 0) tma_prefetch_desc(&tm_b2);
    tma_prefetch_desc(&tm_c);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();            // both CTAs' barriers are initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  griddep_wait();                // programmatic launch: previous kernel done before global access

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      for (int t = pair; ok && t < g.num_tiles; t += G) {
        const TileGeom geo = tile_geom(g, t, BN, true);
        const int half = geo.width / 2;
        const uint32_t stage_tx = 2u * static_cast<uint32_t>(C::A_BYTES + half * C::KB);
        const void* tmb = geo.narrow ? &tm_b2 : &tm_b;
        for (int kb = 0; kb < g.kb_total; ++kb) {
          if (!mbar_wait(smem_u32(empty_bar + stage), phase ^ 1, g.wait, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(full_bar + stage);
          if (leader) mbar_arrive_expect_tx(fb, stage_tx);
          const uint32_t fb_leader = map_to_rank(fb, 0);
          tma_load_2d_pair(smem_u32(sA + stage * C::A_BYTES), &tm_a, fb_leader, kb * C::KB,
                           geo.ta * 256 + static_cast<int>(rank) * 128);
          tma_load_2d_pair(smem_u32(sB + stage * C::B_BYTES), tmb, fb_leader, kb * C::KB,
                           geo.n0 + static_cast<int>(rank) * half);
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        // Let loads already issued land before the CTA leaves: the leader
        // waits on its full barriers (bounded); the follower, whose loads
        // complete on the leader's barriers, waits a fixed 100 us.
        if (leader) {
          WaitCtl quick = g.wait;
          quick.timeout_ns = quick.timeout_ns < 50000000ull ? quick.timeout_ns : 50000000ull;
          volatile int never = 0;
          for (long long i = 0; i < issued && i < C::STAGES; ++i) {
            if (--stage < 0) {
              stage = C::STAGES - 1;
              phase ^= 1;
            }
            mbar_wait(smem_u32(full_bar + stage), phase, quick, &never);
          }
        } else {
          const uint64_t t0 = globaltimer();
          while (globaltimer() - t0 < 100000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (leader && lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int t = pair; ok && t < g.num_tiles; t += G) {
        const TileGeom geo = tile_geom(g, t, BN, true);
        const uint32_t idesc = F8 ? idesc_e4m3(256, geo.width) : idesc_i8(256, geo.width);
        if (!mbar_wait(smem_u32(acce_bar + acc), acc_phase ^ 1, g.wait, abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < g.kb_total; ++kb) {
          if (!mbar_wait(smem_u32(full_bar + stage), phase, g.wait, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = smem_desc_kmajor<C::KB>(smem_u32(sA + stage * C::A_BYTES));
          const uint64_t bd = smem_desc_kmajor<C::KB>(smem_u32(sB + stage * C::B_BYTES));
#pragma unroll
          for (int k = 0; k < C::K_STEPS; ++k)
            if constexpr (F8) mma_f8_pair(d, ad + 2 * k, bd + 2 * k, idesc, (kb > 0 || k > 0) ? 1u : 0u);
            else mma_i8_pair(d, ad + 2 * k, bd + 2 * k, idesc, (kb > 0 || k > 0) ? 1u : 0u);
          mma_commit_pair_both(smem_u32(empty_bar + stage));    // frees the stage in both CTAs
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        mma_commit_pair_both(smem_u32(accf_bar + acc));        // both CTAs' epilogues
        if (++acc == C::ACC_BUFS) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      mma_commit_pair(map_to_rank(smem_u32(drain_bar), 0));
      volatile int never = 0;
      mbar_wait(smem_u32(drain_bar), 0, g.wait, &never);
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    constexpr int GROUPS = C::EPI_WARPS / 4;
    const int ew = warp - 2;
    const int sp = warp & 3;
    const int grp = ew / 4;
    const int ep_tid = threadIdx.x - 64;
    uint8_t* my_out = sOut + ew * C::OUT_BUF_BYTES;
    int out_flip = 0;
    auto next_buf = [&]() -> uint8_t* {
      if (g.out_s32) {
        if (lane == 0) bulk_wait_group_read<0>();
        __syncwarp();
        return my_out;
      }
      if (lane == 0) bulk_wait_group_read<1>();
      __syncwarp();
      uint8_t* b = my_out + out_flip * (C::OUT_BUF_BYTES / 2);
      out_flip ^= 1;
      return b;
    };
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t sc_phase = 0;
    for (int t = pair; t < g.num_tiles; t += G) {
      const TileGeom geo = tile_geom(g, t, BN, true);
      const int m_slab = geo.ta * 256 + static_cast<int>(rank) * 128 + sp * 32;
      const int m = m_slab + lane;
      // Once every epilogue warp is done with the previous tile's scales,
      // one thread refills the slot for this tile while its MMAs still run.
      if (ep_tid == 0) {
        if (t != pair && !mbar_wait(smem_u32(sc_free), sc_phase ^ 1, g.wait, abort_flag)) break;
        stage_tile_scales(g, sc_slot, geo.n0, geo.width, smem_u32(sc_full));
      }
      const float srow = (!g.out_s32 && m < g.M) ? __ldg(g.s_row + m) : 0.0f;
      if (!mbar_wait(smem_u32(accf_bar + acc), acc_phase, g.wait, abort_flag)) break;
      if (!mbar_wait(smem_u32(sc_full), sc_phase, g.wait, abort_flag)) break;
      sc_phase ^= 1;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(sp * 32) << 16) + static_cast<uint32_t>(acc * BN);
      const int nch = geo.width / C::CW;
      const int last_c = grp + ((nch - 1 - grp) / GROUPS) * GROUPS;
      // Chunks are read from TMEM two at a time (one wait per pair); after
      // the pair holding its last chunk the warp hands the accumulator back
      // to the leader, then dequantizes and stores from registers.
#pragma unroll 1
      for (int c0 = grp; c0 < nch; c0 += 2 * GROUPS) {
        uint32_t r[2][C::CW];
        const bool two = c0 + GROUPS < nch;
        tmem_ld_32x32b_x32(tbase + c0 * C::CW, r[0]);
        if (two) tmem_ld_32x32b_x32(tbase + (c0 + GROUPS) * C::CW, r[1]);
        tmem_ld_wait();
        if (c0 == last_c || (two && c0 + GROUPS == last_c)) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(map_to_rank(smem_u32(acce_bar + acc), 0));
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int c = c0 + i * GROUPS;
          if (i == 1 && !two) break;
          store_row_chunk_staged<F8>(g, &tm_c, next_buf(), lane, m_slab, geo.n0 + c * C::CW, r[i], srow, sc_slot,
                                 c * C::CW);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(sc_free));
      if (++acc == C::ACC_BUFS) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    if (lane == 0) bulk_wait_group<0>();
    __syncwarp();
  }

  tc_fence_before();
  cluster_sync_all();            // no CTA leaves while its peer may still signal it
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
}

namespace {

std::atomic<int> g_pair_slots[64] = {};

template <int BN>
cudaLaunchConfig_t pair_config(cudaLaunchAttribute (&attr)[2], cudaStream_t stream) {
  using C = Cfg2<BN>;
  cudaLaunchConfig_t cfg = {};
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cfg;
}

template <int BN, bool F8>
dq_status launch_pair(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tb2, const CUtensorMap& tc,
                      const GemmArgs& g, int pairs, cudaStream_t stream) {
  using C = Cfg2<BN>;
  const dq_status st = smem_limit_once(reinterpret_cast<const void*>(&gemm2_kernel<BN, F8>), C::SMEM_BYTES);
  if (st != DQ_OK) return st;
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = pair_config<BN>(attr, stream);
  cfg.gridDim = dim3(2 * pairs);
  cudaError_t e = cudaLaunchKernelEx(&cfg, gemm2_kernel<BN, F8>, ta, tb, tb2, tc, g);
  return e == cudaSuccess ? DQ_OK : cuda_fail(e);
}

}  // namespace

// CTA pairs that fit at once (clusters of two, one CTA per SM; the same for
// every tile width, whose shared memory all but fills an SM), per device.
dq_status pair_slots(const DeviceInfo& d, int* pairs) {
  int n = g_pair_slots[d.device & 63].load(std::memory_order_relaxed);
  if (n == 0) {
    const dq_status st =
        smem_limit_once(reinterpret_cast<const void*>(&gemm2_kernel<256, false>), Cfg2<256>::SMEM_BYTES);
    if (st != DQ_OK) return st;
    cudaLaunchAttribute attr[2];
    cudaLaunchConfig_t cfg = pair_config<256>(attr, nullptr);
    cfg.numAttrs = 1;                         // the cluster shape only
    cfg.gridDim = dim3(2 * (d.sm_count / 2));
    cudaError_t e = cudaOccupancyMaxActiveClusters(&n, gemm2_kernel<256, false>, &cfg);
    if (e != cudaSuccess) return cuda_fail(e);
    if (n < 1) n = 1;
    g_pair_slots[d.device & 63].store(n, std::memory_order_relaxed);
  }
  *pairs = n;
  return DQ_OK;
}

// Launches gemm2_kernel with clusters of 2 CTAs, `pairs` pairs (persistent).
// bn: pair tile width (160, 192 or 256); f8: e4m3 operands (only with 256).
dq_status launch_pair_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tb2,
                           const CUtensorMap& tc, const GemmArgs& g, int bn, int pairs, cudaStream_t stream,
                           bool f8) {
  if (f8) return launch_pair<256, true>(ta, tb, tb2, tc, g, pairs, stream);
  switch (bn) {
    case 160: return launch_pair<160, false>(ta, tb, tb2, tc, g, pairs, stream);
    case 192: return launch_pair<192, false>(ta, tb, tb2, tc, g, pairs, stream);
    default: return launch_pair<256, false>(ta, tb, tb2, tc, g, pairs, stream);
  }
}

}  // namespace dq
