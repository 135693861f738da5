// gemm.cu -- the int8 x int8 -> int32 GEMM with the dequantization epilogue
// fused (pytorch/ao PR 821, "int8 dynamic quant + bsr support": i8i8->bf16,
// no int32 intermediate in global memory), dense and block-sparse weight,
// and its e4m3 x e4m3 -> fp32 sibling (the vLLM quantization commits'
// dynamic FP8, applied per token).
//
// One persistent, warp-specialised kernel template for sm_100a:
//   warp 0      TMA producer: streams K slices of both operands into a ring
//               of shared-memory stages (mbarrier full/empty pairs).
//   warp 1      MMA issuer: one thread issues tcgen05.mma (kind::i8, or
//               kind::f8f6f4 for e4m3; M = 128) into an accumulator in TMEM;
//               tcgen05.commit releases the stage and, at the end of a tile,
//               hands the accumulator over.
//   warps 2..9  epilogue (two warps per TMEM sub-partition, alternate
//               32-column chunks): tcgen05.ld the accumulator (thread = TMEM
//               lane = output row), dequantize in fp32 (acc * s_row * s_col +
//               bias, each op rounded to nearest even, no FMA), convert to
//               bf16, stage 32x32 blocks in shared memory and TMA-store them.
//               Accumulators are multi-buffered in TMEM so the epilogue of
//               tile i overlaps the MMAs of tile i+1.
//   last warp   streaming BSR only (warp 10): a second producer that issues the weight
//               block copies while warp 0 issues the activation slices.
//
// Operand arrangements sharing it:
//   Dense    A slot = 128 activation rows, B slot = BN weight channels
//            (DenseF8: the same with e4m3 operands).  When whole tiles leave
//            a partial last wave, the full waves keep BN-wide tiles and the
//            rest of the matrix goes in one wave of narrower tiles.
//   Swap     A slot = 128 weight channels, B slot = BN (16..128) tokens: for
//            few tokens and few channels the weight stream, not the token
//            count, fills MMA M.
//   Bsr*     A slot = 128 activation rows x the k slice of one block column,
//            B slot = one nonzero weight block (64x64, 32x32 or 16x16: kinds
//            Bsr, Bsr32, Bsr16); a tile spans 256 channels (4, 8 or 16 block
//            rows) and each block accumulates into its block row's slice of
//            the TMEM tile; the producer walks crow/col (PR 821: the kernel
//            takes crow_indices / col_indices / values directly).  A 16-wide
//            block is issued as a K = 32 MMA whose other 16 k bytes read
//            zeros.  The panel variant keeps a 128-row block's activations in
//            shared memory and streams only weight blocks.
//
// Many tokens (from 1536 with K >= 2048, and any K >= 8192) take the 2-SM
// pair kernel of gemm2sm.cu instead (int8 and e4m3); the 1-SM kernel keeps
// the rest and every BSR and swap call.
//
// Schedules: whole tiles round-robin over one CTA per SM (contiguous tile
// ranges for the BSR panel variant), or, for the swap arrangement when whole
// tiles would leave SMs idle, stream-K: the tile x k-block iteration space is
// cut into equal contiguous ranges, one per CTA; partial tiles meet in an
// int32 workspace through red.add, and the last arriving CTA (an arrival
// counter) runs the epilogue and zeroes the workspace again.  Integer adds
// are exact and associative, so every schedule gives identical bits.
#include <atomic>
#include <mutex>

#include "gemm_common.cuh"

namespace dq {

template <Kind KIND, int BN, bool PANEL = false>
struct Cfg {
  static constexpr int BM = 128;
  static constexpr bool BSR = is_bsr(KIND);
  static constexpr int BS = bsr_bs(KIND);                     // block size (BSR kinds)
  // k bytes per stage: dense 128 (128-byte swizzle); 64x64 blocks 64 (64-byte
  // swizzle); 32x32 and 16x16 blocks 32 (32-byte swizzle; a 16-wide block
  // uses the 32-byte A slice that contains it, the other half of the MMA's K
  // multiplying zeros, see the Bsr16 B descriptor).
  static constexpr int KB = !BSR ? kDenseKB : BS == 64 ? 64 : 32;
  // BSR panel variant: the 128 x K activation panel of the current 128-row
  // block stays in shared memory (K <= KP, chunks of 128 x 128 bytes with the
  // 128-byte swizzle) and the stages carry weight blocks only.
  static constexpr int KP = PANEL ? 1280 : 0;
  static constexpr int PANEL_CHUNKS = KP / 128;
  static constexpr int PANEL_BYTES = PANEL_CHUNKS * BM * 128;
  static constexpr int A_BYTES = PANEL ? 0 : BM * KB;         // per stage
  // BSR: a tile spans BN/BS block rows; each stage holds one BS x BS block
  // that accumulates into its block row's BS-column slice of the tile.
  static constexpr int B_ROWS = BSR ? BS : BN;
  static constexpr int MMA_N = B_ROWS;
  static constexpr int NSUB = BSR ? BN / BS : 1;
  static constexpr int B_BYTES = BSR ? BS * BS : B_ROWS * KB;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  // Row-layout epilogues (Dense, BSR) stage each warp's 32x32 output block in
  // shared memory for a TMA store: 2 buffers x 4 warps x 4 KB (int32 worst case).
  // Epilogue warps: two per TMEM sub-partition when a tile has at least two
  // 32-column chunks, so one warp's latency hides behind the other's work.
  // (Measured on B200 for the epilogue-bound BSR kernel: 12 or 16 epilogue
  // warps are slower than 8.)
  static constexpr int EPI_WARPS = BN >= 64 ? 8 : 4;
  static constexpr bool STAGED_OUT = KIND != Kind::Swap;
  static constexpr int OUT_BUF_BYTES = 32 * 32 * 4;           // per epilogue warp
  static constexpr int OUT_BYTES = STAGED_OUT ? EPI_WARPS * OUT_BUF_BYTES : 0;
  // BSR: crow and col are copied to shared memory when nbr + 1 + nnzb fits
  // (every tile and every block needs them; a global load per block would put
  // a dependent L2 round trip in front of each TMA issue).  The panel variant
  // has no room for them and reads them through L1.
  static constexpr int IDX_INTS = BSR && !PANEL ? 4096 : 0;
  static constexpr int IDX_BYTES = IDX_INTS * 4;
  // 16x16 blocks: two 256-byte zero regions, one below and one above the
  // stage buffers, that stand in for the half of the MMA's K the block does
  // not cover (the descriptor's leading-dimension offset must be positive).
  static constexpr int ZERO_BYTES = KIND == Kind::Bsr16 ? 1024 : 0;
  // Panel variant: a zero weight block, used in place of a block whose
  // column lies outside the matrix (it contributes zeros, as a load from
  // outside the matrix does in the streaming variant).
  static constexpr int ZB_BYTES = PANEL ? (B_BYTES > 256 ? B_BYTES : 256) : 0;
  static constexpr int STAGE_CAP = (BSR && (BS < 64 || PANEL)) || (!BSR && KB < 128) ? 24 : 12;
  static constexpr int ACC_RAW = 512 / BN;
  static constexpr int ACC_BUFS = ACC_RAW > 8 ? 8 : ACC_RAW;
  // mbarriers, the TMEM address, flags and (panel variant) stage columns
  static constexpr int BAR_BYTES = BSR || STAGE_CAP > 12 ? 1024 : 512;
  // Shared-memory layout for a given stage count and number of column-scale
  // slots (offsets from the 1024-aligned base; the last 1024 bytes are the
  // slack of aligning the dynamic shared-memory base).
  static constexpr int off_b(int st) { return ZERO_BYTES + PANEL_BYTES + st * A_BYTES; }
  static constexpr int off_out(int st) {
    return ((((off_b(st) + st * B_BYTES + ZERO_BYTES + 1023) / 1024 * 1024) + ZB_BYTES + 1023) / 1024) * 1024;
  }
  static constexpr int layout_bytes(int st, int slots) {
    return off_out(st) + OUT_BYTES + slots * kScSlotBytes + IDX_BYTES + BAR_BYTES + 1024;
  }
  static constexpr int pick_stages(int slots) {
    int st = STAGE_CAP;
    while (st > 2 && layout_bytes(st, slots) > 227 * 1024) --st;
    return st;
  }
  // Row-layout epilogues stage each tile's column scales and bias in shared
  // memory: two slots (the next tile's copy in flight while this tile is
  // stored) where that costs no operand stage, else one.
  static constexpr int SC_SLOTS = !STAGED_OUT ? 0 : pick_stages(2) == pick_stages(0) ? 2 : 1;
  static constexpr int STAGES = pick_stages(SC_SLOTS);
  static constexpr int OFF_ZLO = 0;
  static constexpr int OFF_PANEL = ZERO_BYTES;
  static constexpr int OFF_A = OFF_PANEL + PANEL_BYTES;
  static constexpr int OFF_B = off_b(STAGES);
  static constexpr int OFF_ZHI = OFF_B + STAGES * B_BYTES;
  static constexpr int OFF_ZB = (OFF_ZHI + ZERO_BYTES + 1023) / 1024 * 1024;
  static constexpr int OFF_OUT = off_out(STAGES);
  static constexpr int OFF_SC = OFF_OUT + OUT_BYTES;
  static constexpr int OFF_IDX = OFF_SC + SC_SLOTS * kScSlotBytes;
  static constexpr int OFF_BARS = OFF_IDX + IDX_BYTES;
  static constexpr int ACC_COLS = ACC_BUFS * BN;
  static constexpr int TMEM_COLS = ACC_COLS <= 32 ? 32 : ACC_COLS <= 64 ? 64 : ACC_COLS <= 128 ? 128
                                   : ACC_COLS <= 256 ? 256 : 512;
  static constexpr int K_STEPS = KB / 32;                     // MMA K = 32 bytes
  static constexpr int CW = BN >= 32 ? 32 : 16;               // epilogue chunk (columns)
  static constexpr int SMEM_BYTES = layout_bytes(STAGES, SC_SLOTS);
  // Streaming BSR stages carry a small activation slice and a small weight
  // block, so issuing their tensor copies bounds the K-heavy shapes (each
  // copy holds its issuing thread a few hundred cycles): there the two copies
  // of a stage come from two threads, warp 0 and one warp after the epilogue
  // warps.  Every other kind issues both from warp 0.
  static constexpr int NPROD = BSR && !PANEL ? 2 : 1;
  static constexpr int THREADS = 32 + 32 * NPROD + 32 * EPI_WARPS;
  static constexpr int NBARS = 2 * STAGES + 2 * ACC_BUFS + 3 + 2 * SC_SLOTS;
  static_assert(NBARS * 8 + 16 + (PANEL ? 4 * STAGES : 0) <= BAR_BYTES, "barrier area");
  static_assert(OFF_ZB + ZB_BYTES <= OFF_OUT, "layout");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
  static_assert(STAGES >= 2, "stages");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
  static_assert(!BSR || BN % (BSR ? BS : 1) == 0, "tile covers whole block rows");
  static_assert(!PANEL || BSR, "the panel variant is for BSR weights");
};

// The stream-K finishing store, kept out of line so that this rarely taken
// path does not add to the register pressure of the whole-tile epilogue.
__device__ __noinline__ void store_row_chunk_tma_cold(const GemmArgs& g, const CUtensorMap* tm_c, uint8_t* buf,
                                                      int lane, int m0, int n0, const uint32_t* r, float srow) {
  ColScales cs;
  uint4 bias[4];
  if (!g.out_s32) load_col_scales(g, n0, cs);
  if (!g.out_s32 && g.bias != nullptr) load_bias_global(g, n0, bias);
  store_row_chunk_tma(g, tm_c, buf, lane, m0, n0, r, srow, cs, bias);
}

template <Kind KIND, int BN, bool PANEL>
__global__ void __launch_bounds__(Cfg<KIND, BN, PANEL>::THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                const __grid_constant__ CUtensorMap tm_b2, const __grid_constant__ CUtensorMap tm_c,
                const __grid_constant__ GemmArgs g) {
  using C = Cfg<KIND, BN, PANEL>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem + C::OFF_A;
  uint8_t* sB = smem + C::OFF_B;
  uint8_t* sOut = smem + C::OFF_OUT;                          // 1024-aligned
  int* sIdx = reinterpret_cast<int*>(smem + C::OFF_IDX);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BARS);
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + C::STAGES;
  uint64_t* accf_bar = bars + 2 * C::STAGES;
  uint64_t* acce_bar = accf_bar + C::ACC_BUFS;
  uint64_t* drain_bar = acce_bar + C::ACC_BUFS;
  uint64_t* panel_full = drain_bar + 1;       // panel variant: activation panel landed
  uint64_t* panel_empty = panel_full + 1;     // panel variant: MMAs on the old panel done
  uint64_t* sc_full = panel_empty + 1;        // row epilogues: a tile's scales landed in slot i
  uint64_t* sc_free = sc_full + C::SC_SLOTS;   // every epilogue warp is done reading slot i
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sc_free + C::SC_SLOTS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* sk_last = const_cast<int*>(abort_flag + 1);
  // panel variant: each stage's block column, written by the producer before
  // it arms the stage's barrier (the MMA thread reads it after the wait)
  int* stage_col = sk_last + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(full_bar + s), 1);
      mbar_init(smem_u32(empty_bar + s), 1);
    }
    for (int a = 0; a < C::ACC_BUFS; ++a) {
      mbar_init(smem_u32(accf_bar + a), 1);
      mbar_init(smem_u32(acce_bar + a), 32 * C::EPI_WARPS);
    }
    mbar_init(smem_u32(drain_bar), 1);
    mbar_init(smem_u32(panel_full), 1);
    mbar_init(smem_u32(panel_empty), 1);
    for (int i = 0; i < C::SC_SLOTS; ++i) {
      mbar_init(smem_u32(sc_full + i), 1);
      mbar_init(smem_u32(sc_free + i), C::EPI_WARPS);
    }
    fence_barrier_init();
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
    if (is_dense_kind(KIND) && g.bn2 > 0) tma_prefetch_desc(&tm_b2);
    if constexpr (C::STAGED_OUT) tma_prefetch_desc(&tm_c);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), C::TMEM_COLS);
    tmem_relinquish();
  }
  // Everything above touched only shared memory, TMEM and the kernel
  // parameters; with a programmatic (early) launch, wait here for the
  // previous kernel of the stream before any global memory access.
  griddep_wait();
  const int* idx = nullptr;      // BSR: crow at idx[0..nbr], col at idx[nbr+1..]
  if constexpr (KIND == Kind::Bsr16 || PANEL) {
    // the zero regions the 16x16-block B descriptors and the panel variant's
    // out-of-matrix blocks point at, visible to the tensor core (async proxy)
    // before the first MMA
    for (int i = threadIdx.x; i < C::ZERO_BYTES / 16; i += blockDim.x) {
      reinterpret_cast<uint4*>(smem + C::OFF_ZLO)[i] = make_uint4(0u, 0u, 0u, 0u);
      reinterpret_cast<uint4*>(smem + C::OFF_ZHI)[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    for (int i = threadIdx.x; i < C::ZB_BYTES / 16; i += blockDim.x)
      reinterpret_cast<uint4*>(smem + C::OFF_ZB)[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
  if constexpr (C::BSR && !PANEL) {
    if (g.idx_smem) {
      const int nbr = g.nbr;
      for (int i = threadIdx.x; i <= nbr; i += blockDim.x) sIdx[i] = __ldg(g.crow + i);
      for (int i = threadIdx.x; i < g.nnzb; i += blockDim.x) sIdx[nbr + 1 + i] = __ldg(g.col + i);
      idx = sIdx;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0 || warp >= 2 + C::EPI_WARPS) {
    // ------------------------------------------------------------ producer
    // Warp 0 arms each stage's barrier with the stage's bytes and issues the
    // A copies; with two producers the other one issues the B copies (its
    // copies may land before the barrier is armed: the transaction count
    // then runs below zero until the arming, and the phase cannot complete
    // before that arrival).
    const bool a_side = warp == 0;
    const bool b_side = C::NPROD == 1 || warp != 0;
    if (lane == 0) {
      SegIter iter(g);
      Seg s;
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      int loaded_ta = -1;           // panel variant: block row whose panel is loaded
      int panel_loads = 0;
      const int panel_chunks = (g.K + 127) / 128;
      while (ok && iter.next(s)) {
        const TileGeom geo = tile_geom(g, s.tile, BN, is_dense_kind(KIND));
        const int ta = geo.ta, tb = geo.tb;
        const uint32_t stage_tx = C::A_BYTES + (is_dense_kind(KIND) ? geo.width * C::KB : C::B_BYTES);
        if constexpr (PANEL) {
          if (ta != loaded_ta) {
            // a new 128-row block: once the MMAs on the previous panel are
            // done, bring its 128 x K activations in (one box per 128 k bytes)
            if (panel_loads > 0) {
              if (!mbar_wait(smem_u32(panel_empty), static_cast<uint32_t>(panel_loads - 1) & 1u, g.wait,
                             abort_flag)) {
                ok = false;
                break;
              }
            }
            const uint32_t pf = smem_u32(panel_full);
            mbar_arrive_expect_tx(pf, static_cast<uint32_t>(panel_chunks) * (C::BM * 128));
            for (int ch = 0; ch < panel_chunks; ++ch)
              tma_load_2d(smem_u32(smem + C::OFF_PANEL + ch * (C::BM * 128)), &tm_a, pf, ch * 128, ta * 128);
            ++panel_loads;
            loaded_ta = ta;
          }
        }
        for (int j = 0; ok && j < C::NSUB; ++j) {
        int k0 = s.kb0, k1 = s.kb1;
        if constexpr (C::BSR) {
          const int br = tb * C::NSUB + j;
          if (br >= g.nbr) break;
          bsr_range(g, idx, br, k0, k1);
        }
        int c_next = (PANEL && k0 < k1) ? __ldg(g.col + k0) : 0;
        for (int kb = k0; kb < k1; ++kb) {
          const int c_cur = c_next;
          if (PANEL && kb + 1 < k1) c_next = __ldg(g.col + kb + 1);     // one block ahead
          if (!mbar_wait(smem_u32(empty_bar + stage), phase ^ 1, g.wait, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(full_bar + stage);
          if constexpr (PANEL) stage_col[stage] = c_cur;
          if (a_side) mbar_arrive_expect_tx(fb, stage_tx);
          const uint32_t da = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t db = smem_u32(sB + stage * C::B_BYTES);
          if constexpr (PANEL) {
            tma_load_2d(db, &tm_b, fb, 0, kb * C::BS);        // the block only; A is the panel
            (void)da;
          } else if constexpr (C::BSR) {
            // A: the KB-wide k slice holding block column c (for 16-wide
            // blocks the 32-byte slice that contains it); B: block kb
            if (a_side) {
              const int c = idx ? idx[g.nbr + 1 + kb] : __ldg(g.col + kb);
              const int ax = KIND == Kind::Bsr16 ? (c >> 1) * 32 : c * C::BS;
              tma_load_2d(da, &tm_a, fb, ax, ta * 128);
            }
            if (b_side) tma_load_2d(db, &tm_b, fb, 0, kb * C::BS);
          } else {
            tma_load_2d(da, &tm_a, fb, kb * C::KB, ta * 128);
            tma_load_2d(db, geo.narrow ? &tm_b2 : &tm_b, fb, kb * C::KB, geo.n0);
          }
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        }
      }
      if (!ok && !a_side) {
        // the B producer: its copies land on barriers warp 0 drains (below);
        // a fixed 100 us covers the ones whose stage was never armed
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 100000ull) {
        }
      } else if (!ok) {
        // Let the (at most STAGES) most recent loads land before the CTA
        // leaves; each wait is bounded by a short limit.
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
        if (PANEL && panel_loads > 0)
          mbar_wait(smem_u32(panel_full), static_cast<uint32_t>(panel_loads - 1) & 1u, quick, &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr bool F8 = KIND == Kind::DenseF8;
      constexpr uint32_t idesc_full = F8 ? idesc_e4m3(128, C::MMA_N) : idesc_i8(128, C::MMA_N);
      SegIter iter(g);
      Seg s;
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      int cur_ta = -1;               // panel variant: block row of the panel in use
      int panels = 0;
      while (ok && iter.next(s)) {
        if (!mbar_wait(smem_u32(acce_bar + acc), acc_phase ^ 1, g.wait, abort_flag)) break;
        tc_fence_after();
        const uint32_t idesc = (is_dense_kind(KIND) && g.bn2 > 0 && s.tile >= g.t1)
                                   ? (F8 ? idesc_e4m3(128, g.bn2) : idesc_i8(128, g.bn2)) : idesc_full;
        if constexpr (PANEL) {
          const int ta = s.tile / g.b_tiles;
          if (ta != cur_ta) {
            // hand the old panel back (once its MMAs are done), wait for the new one
            if (panels > 0) mma_commit(smem_u32(panel_empty));
            if (!mbar_wait(smem_u32(panel_full), static_cast<uint32_t>(panels) & 1u, g.wait, abort_flag)) break;
            tc_fence_after();
            ++panels;
            cur_ta = ta;
          }
        }
        for (int j = 0; ok && j < C::NSUB; ++j) {
        int k0 = s.kb0, k1 = s.kb1;
        if constexpr (C::BSR) {
          const int br = (s.tile % g.b_tiles) * C::NSUB + j;
          if (br >= g.nbr) break;
          bsr_range(g, idx, br, k0, k1);
        }
        // an empty block row leaves its slice untouched; the epilogue writes zeros there
        const uint32_t d = tmem_base + static_cast<uint32_t>(acc * BN + j * C::MMA_N);
        for (int kb = k0; kb < k1; ++kb) {
          if (!mbar_wait(smem_u32(full_bar + stage), phase, g.wait, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint64_t ad, bd;
          if constexpr (PANEL) {
            // A: the block column's k slice inside the resident panel (a start
            // address 32 / 64 / 96 bytes into a 128-byte swizzled row, as the
            // k steps of the dense kernel); a column outside [0, K / BS)
            // multiplies the zero block instead
            const int c = stage_col[stage];
            const bool valid = c >= 0 && c < g.K / C::BS;
            const int kbyte = !valid ? 0 : KIND == Kind::Bsr16 ? (c >> 1) * 32 : c * C::BS;
            ad = smem_desc_kmajor<128>(smem_u32(smem + C::OFF_PANEL + (kbyte >> 7) * (C::BM * 128))) +
                 static_cast<uint64_t>((kbyte & 127) >> 4);
            // (a 16-wide zero block is the low zero region itself, so that the
            // padded descriptor's offset stays positive)
            const uint32_t blk = valid ? smem_u32(sB + stage * C::B_BYTES)
                                       : smem_u32(smem + (KIND == Kind::Bsr16 ? C::OFF_ZLO : C::OFF_ZB));
            if constexpr (KIND == Kind::Bsr16)
              bd = smem_desc_b16_padded(blk, smem_u32(smem + C::OFF_ZLO), smem_u32(smem + C::OFF_ZHI), c & 1);
            else
              bd = smem_desc_kmajor<C::KB>(blk);
          } else if constexpr (KIND == Kind::Bsr16) {
            ad = smem_desc_kmajor<C::KB>(smem_u32(sA + stage * C::A_BYTES));
            // 16 channels x 16 k of the block, rows of 16 bytes (no swizzle):
            // the MMA's other 16 k bytes read a zero region, so the 32-byte A
            // slice's other half contributes nothing.
            const int c = idx ? idx[g.nbr + 1 + kb] : __ldg(g.col + kb);
            bd = smem_desc_b16_padded(smem_u32(sB + stage * C::B_BYTES), smem_u32(smem + C::OFF_ZLO),
                                      smem_u32(smem + C::OFF_ZHI), c & 1);
          } else {
            ad = smem_desc_kmajor<C::KB>(smem_u32(sA + stage * C::A_BYTES));
            bd = smem_desc_kmajor<C::KB>(smem_u32(sB + stage * C::B_BYTES));
          }
#pragma unroll
          for (int k = 0; k < C::K_STEPS; ++k) {
            if constexpr (F8) mma_f8(d, ad + 2 * k, bd + 2 * k, idesc, (kb > k0 || k > 0) ? 1u : 0u);
            else mma_i8(d, ad + 2 * k, bd + 2 * k, idesc, (kb > k0 || k > 0) ? 1u : 0u);
          }
          mma_commit(smem_u32(empty_bar + stage));
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        }
        if (!ok) break;
        mma_commit(smem_u32(accf_bar + acc));
        if (++acc == C::ACC_BUFS) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      // Every MMA issued by this thread has completed once drain_bar flips.
      mma_commit(smem_u32(drain_bar));
      volatile int never = 0;
      mbar_wait(smem_u32(drain_bar), 0, g.wait, &never);
    }
  } else if (warp < 2 + C::EPI_WARPS) {
    // ------------------------------------------------------------ epilogue
    // EPI_WARPS warps; warp w reads TMEM sub-partition w % 4 (rows 32*(w%4) ..
    // +31) and, with EPI_WARPS == 8, the two warps of a sub-partition take
    // alternate 32-column chunks of each tile.
    constexpr int CW = C::CW;
    constexpr int NCH = BN / CW;
    constexpr int GROUPS = C::EPI_WARPS / 4;
    constexpr int EPI_THREADS = 32 * C::EPI_WARPS;
    const int ew = warp - 2;
    const int sp = warp & 3;                 // TMEM sub-partition of this warp
    const int grp = ew / 4;                  // which chunks: c % GROUPS == grp
    const int row = sp * 32 + lane;          // TMEM lane = accumulator row
    const int ep_tid = threadIdx.x - 64;
    uint8_t* my_out = sOut + ew * C::OUT_BUF_BYTES;
    int out_flip = 0;
    // Staging buffer for the next 32x32 block, once the TMA store that last
    // read it is done: two 2 KB slots for bf16, one 4 KB slot for int32.
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
    SegIter iter(g);
    int k = 0;               // segments started
    const uint32_t sc_base = smem_u32(smem + C::OFF_SC);
    Seg s;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    while (ok && iter.next(s)) {
      const TileGeom geo = tile_geom(g, s.tile, BN, is_dense_kind(KIND));
      const int ta = geo.ta, tb = geo.tb, n0 = geo.n0;
      const int slot = C::SC_SLOTS > 0 ? k % C::SC_SLOTS : 0;
      const uint32_t sc_slot = sc_base + static_cast<uint32_t>(slot * kScSlotBytes);
      if constexpr (C::SC_SLOTS > 0) {
        // One thread copies each segment's scales into its slot once every
        // epilogue warp is done with the slot's previous contents: with one
        // slot at the start of the segment, with two one segment ahead (the
        // copy lands while the MMAs, or the previous segment's stores, run).
        if (ep_tid == 0) {
          if (C::SC_SLOTS == 1 || k == 0) {
            if (k > 0 && !mbar_wait(smem_u32(sc_free), static_cast<uint32_t>(k - 1) & 1u, g.wait, abort_flag))
              break;
            stage_tile_scales(g, sc_slot, n0, geo.width, smem_u32(sc_full + slot));
          }
          if constexpr (C::SC_SLOTS == 2) {
            SegIter peek = iter;
            Seg ns;
            if (peek.next(ns)) {
              const int k1 = k + 1, sl = k1 & 1;
              if (k1 >= 2 &&
                  !mbar_wait(smem_u32(sc_free + sl), static_cast<uint32_t>(k1 / 2 - 1) & 1u, g.wait, abort_flag))
                break;
              const TileGeom ng = tile_geom(g, ns.tile, BN, is_dense_kind(KIND));
              stage_tile_scales(g, sc_base + static_cast<uint32_t>(sl * kScSlotBytes), ng.n0, ng.width,
                                smem_u32(sc_full + sl));
            }
          }
        }
      }
      float srow = 0.0f;
      if constexpr (KIND != Kind::Swap) {
        const int m = ta * 128 + row;
        if (!g.out_s32 && m < g.M) srow = __ldg(g.s_row + m);
      }
      if (!mbar_wait(smem_u32(accf_bar + acc), acc_phase, g.wait, abort_flag)) break;
      if constexpr (C::SC_SLOTS > 0) {
        if (!mbar_wait(smem_u32(sc_full + slot), static_cast<uint32_t>(k / C::SC_SLOTS) & 1u, g.wait, abort_flag))
          break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(sp * 32) << 16) + static_cast<uint32_t>(acc * BN);
      const bool whole = !g.stream_k || (s.kb0 == 0 && s.kb1 == g.kb_total);
      // chunks of this tile (a narrow Dense tile has fewer; every warp still
      // has one, as bn2 >= 64); after reading its last chunk a warp releases
      // the accumulator
      const int nch = is_dense_kind(KIND) ? geo.width / CW : NCH;
      const int last_c = grp + ((nch - 1 - grp) / GROUPS) * GROUPS;

      if (whole) {
        // BATCH chunks per TMEM wait (row layouts: two); after the batch
        // holding its last chunk the warp hands the accumulator back to the
        // MMA warp, then dequantizes and stores from registers with the
        // column scales and bias from the tile's staged slot.
        constexpr int BATCH = C::STAGED_OUT ? 2 : 1;
#pragma unroll 1
        for (int c0 = grp; c0 < nch; c0 += BATCH * GROUPS) {
          uint32_t r[BATCH][CW];
          const bool two = BATCH > 1 && c0 + GROUPS < nch;
          // BSR: block rows of a chunk without blocks (their TMEM slice was
          // never written) read as zeros; a 32-column chunk holds one block
          // row's columns, or two 16-wide block rows
          bool empty_lo[BATCH], empty_hi[BATCH];
#pragma unroll
          for (int i = 0; i < BATCH; ++i) {
            empty_lo[i] = empty_hi[i] = false;
            if (i == 1 && !two) break;
            const int c = c0 + i * GROUPS;
            if constexpr (C::BSR) {
              auto row_empty = [&](int br) {
                int p0 = 0, p1 = 0;
                if (br < g.nbr) bsr_range(g, idx, br, p0, p1);
                return br >= g.nbr || p0 == p1;
              };
              const int br = tb * C::NSUB + (c * CW) / C::BS;
              empty_lo[i] = row_empty(br);
              empty_hi[i] = C::BS >= CW ? empty_lo[i] : row_empty(br + 1);
            }
            if (empty_lo[i] && empty_hi[i]) {
#pragma unroll
              for (int j = 0; j < CW; ++j) r[i][j] = 0;
            } else if constexpr (CW == 32) {
              tmem_ld_32x32b_x32(tbase + c * CW, r[i]);
            } else {
              tmem_ld_32x32b_x16(tbase + c * CW, r[i]);
            }
          }
          tmem_ld_wait();
          if constexpr (KIND == Kind::Bsr16) {
#pragma unroll
            for (int i = 0; i < BATCH; ++i) {
              if (!(empty_lo[i] && empty_hi[i]) && (empty_lo[i] || empty_hi[i])) {
#pragma unroll
                for (int j = 0; j < CW; ++j)
                  if (j < 16 ? empty_lo[i] : empty_hi[i]) r[i][j] = 0;
              }
            }
          }
          if (c0 == last_c || (two && c0 + GROUPS == last_c)) {
            tc_fence_before();
            mbar_arrive(smem_u32(acce_bar + acc));
          }
#pragma unroll
          for (int i = 0; i < BATCH; ++i) {
            if (i == 1 && !two) break;
            const int c = c0 + i * GROUPS;
            if constexpr (KIND == Kind::Swap) {
              store_col_chunk<CW>(g, ta * 128 + row, n0 + c * CW, r[i]);
            } else {
              store_row_chunk_staged<KIND == Kind::DenseF8>(g, &tm_c, next_buf(), lane, ta * 128 + sp * 32,
                                                            n0 + c * CW, r[i], srow, sc_slot, c * CW);
            }
          }
        }
      } else {
        // Stream-K partial tile: add into the workspace (coalesced: one
        // column of 128 rows is 512 contiguous bytes), then the last of the
        // contributing CTAs finishes the tile.
        int32_t* wt = g.ws + static_cast<int64_t>(s.tile) * BN * 128;
#pragma unroll 1
        for (int c = grp; c < NCH; c += GROUPS) {
          uint32_t r[CW];
          if constexpr (CW == 32) tmem_ld_32x32b_x32(tbase + c * CW, r);
          else tmem_ld_32x32b_x16(tbase + c * CW, r);
          tmem_ld_wait();
          if (c == last_c) {
            tc_fence_before();
            mbar_arrive(smem_u32(acce_bar + acc));
          }
#pragma unroll
          for (int j = 0; j < CW; ++j) atomicAdd(wt + (c * CW + j) * 128 + row, static_cast<int>(r[j]));
        }
        __threadfence();
        named_bar_sync(1, EPI_THREADS);
        if (ep_tid == 0) {
          const uint32_t prev = atomicAdd(g.ws_cnt + s.tile, 1u);
          *sk_last = (static_cast<int>(prev) == sk_contributors(g, s.tile) - 1) ? 1 : 0;
        }
        named_bar_sync(1, EPI_THREADS);
        if (*sk_last) {
          __threadfence();
#pragma unroll 1
          for (int c = grp; c < NCH; c += GROUPS) {
            uint32_t r[CW];
#pragma unroll
            for (int j = 0; j < CW; ++j) {
              int32_t* p = wt + (c * CW + j) * 128 + row;
              r[j] = static_cast<uint32_t>(__ldcg(p));
              __stcg(p, 0);
            }
            if constexpr (KIND == Kind::Swap) store_col_chunk<CW>(g, ta * 128 + row, tb * BN + c * CW, r);
            else store_row_chunk_tma_cold(g, &tm_c, next_buf(), lane, ta * 128 + sp * 32, tb * BN + c * CW, r, srow);
          }
          if (ep_tid == 0) g.ws_cnt[s.tile] = 0;
        }
        named_bar_sync(1, EPI_THREADS);   // sk_last is reused by the next partial tile
      }
      if constexpr (C::SC_SLOTS > 0) {
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(sc_free + slot));
      }
      ++k;
      if (++acc == C::ACC_BUFS) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    if constexpr (C::STAGED_OUT) {
      if (lane == 0) bulk_wait_group<0>();     // all output stores complete
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

// ---------------------------------------------------------------- BSR pack

__global__ void __launch_bounds__(256) bsr_pack_kernel(const int8_t* __restrict__ wq, int64_t K,
                                                       const int32_t* __restrict__ crow,
                                                       const int32_t* __restrict__ col, int nnzb,
                                                       int nbc, int bs, int8_t* __restrict__ values) {
  // one CTA per block row; a block's rows are split into 16-byte parts
  const int br = blockIdx.x;
  const int p0 = min(max(__ldg(crow + br), 0), nnzb);
  const int p1 = min(max(__ldg(crow + br + 1), p0), nnzb);
  const int parts = bs / 16;
  for (int p = p0; p < p1; ++p) {
    const int c = __ldg(col + p);
    for (int t = threadIdx.x; t < bs * parts; t += blockDim.x) {
      const int j = t / parts;             // row inside the block
      const int part = t % parts;          // 16-byte part of the row
      uint4 v = make_uint4(0, 0, 0, 0);
      if (c >= 0 && c < nbc)
        v = __ldg(reinterpret_cast<const uint4*>(wq + (static_cast<int64_t>(br) * bs + j) * K +
                                                 static_cast<int64_t>(c) * bs) + part);
      reinterpret_cast<uint4*>(values + (static_cast<int64_t>(p) * bs + j) * bs)[part] = v;
    }
  }
}

// ---------------------------------------------------------------- host side

namespace {

template <Kind KIND, int BN, bool PANEL = false>
dq_status launch(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tb2, const CUtensorMap& tc,
                 const GemmArgs& args, int grid, cudaStream_t stream) {
  using C = Cfg<KIND, BN, PANEL>;
  const dq_status st = smem_limit_once(reinterpret_cast<const void*>(&gemm_kernel<KIND, BN, PANEL>), C::SMEM_BYTES);
  if (st != DQ_OK) return st;
  // Programmatic stream serialization: the prologue may overlap the tail of
  // the previous kernel (e.g. the quantization that produced A); the kernel
  // waits (griddep_wait) before its first global memory access.
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_kernel<KIND, BN, PANEL>, ta, tb, tb2, tc, args);
  return e == cudaSuccess ? DQ_OK : cuda_fail(e);
}

constexpr int64_t kMaxK = 133144;   // floor((2^31 - 1) / 127^2): int32 accumulation is exact

// Measured on B200 (graphs of 20 launches, int8 data in [-40, 40]): with one
// multicast commit per stage the pair kernel (two thirds of the operand bytes
// per SM) is faster from about 1536 tokens and K = 2048 up (2048 x 4096 x
// 4096: 25.3 against 27.2 us; 4096^3: 46.1 against 52.1; 16384 x 4096 x 2048:
// 89 against 105), equal at 1024 tokens and at K = 1024 (38400 x 4096 x 1024:
// 143 us both), and from K = 8192 up at any token count above 128.
constexpr int64_t kPairMinK = 8192;
constexpr int64_t kPairMinKManyTokens = 2048;
constexpr int64_t kPairManyTokens = 1536;

// The measurement knobs, read once per call.
struct Knobs {
  int schedule, tile_n, two_widths, bsr_panel;
};
Knobs knobs() {
  return Knobs{g_schedule_override.load(std::memory_order_relaxed), g_tile_n_override.load(std::memory_order_relaxed),
               g_two_widths.load(std::memory_order_relaxed), g_bsr_panel.load(std::memory_order_relaxed)};
}

struct Plan {
  Kind kind;
  bool pair;         // the 2-SM pair kernel (gemm2sm.cu): 256-row tiles
  int bn;
  int a_tiles, b_tiles, kb_total, num_tiles;
  bool stream_k;
  size_t ws_bytes;   // bytes needed for stream-K (0 if it never splits)
  // Dense wave balance (bn2 > 0): the first t1 tiles (whole waves) are bn
  // wide; the rest of the matrix goes in one last wave of bn2-wide tiles.
  int t1, bn2, mb0, c_start, first_cnt, per_row;
};

// Whole tiles leave the SMs of a partial last wave idle (e.g. M=2048, N=4096:
// 256 tiles of 128 x 256 on 148 SMs, 1.73 waves).  Instead the full waves keep
// bn-wide tiles and the rest of the matrix is cut into at most `sms` tiles of
// the narrowest width (a multiple of 32, >= 64) that fits in one wave.  Every
// SM then does (waves - 1) wide tiles and at most one narrow one.
void plan_two_widths(Plan& p, int64_t N, int sms) {
  p.bn2 = 0;
  const int T = p.num_tiles;
  const int full = T / sms;
  if (full < 1 || T % sms == 0 || full > 8) return;     // one partial wave, or the tail is small
  const int t1 = full * sms;
  const int mb0 = t1 / p.b_tiles;
  const int c_start = (t1 % p.b_tiles) * p.bn;
  const int rows_after = p.a_tiles - mb0 - 1;
  for (int w = 64; w < p.bn; w += 32) {
    const int first = static_cast<int>((N - c_start + w - 1) / w);
    const int per_row = static_cast<int>((N + w - 1) / w);
    const long long t2 = static_cast<long long>(first) + static_cast<long long>(rows_after) * per_row;
    if (t2 <= sms) {
      p.t1 = t1;
      p.bn2 = w;
      p.mb0 = mb0;
      p.c_start = c_start;
      p.first_cnt = first;
      p.per_row = per_row;
      p.num_tiles = t1 + static_cast<int>(t2);
      return;
    }
  }
}

// Stream-K workspace: one int32 partial per tile ([BN][128], column-major so
// that red.add of one column by a warp is one 512-byte line) plus an arrival
// counter per tile.
size_t sk_workspace_bytes(const Plan& p, int /*ctas*/) {
  return static_cast<size_t>(p.num_tiles) * (static_cast<size_t>(p.bn) * 128 * 4 + 4);
}

// Few tokens (M <= 128): the weight stream dominates.  With enough output
// channels for about a wave of 128 x 224 tiles, the dense arrangement (tokens
// on MMA M, rows past M zero-filled by TMA and clipped on store) streams the
// weight faster than swap-AB, whose column-wise epilogue stores are
// scattered: measured at N = 28672, K = 8192: M = 128 47 us vs 57, M = 32
// 46.3 vs 48.9, M = 16 45.9 vs 46.7, but M = 1 54 vs 46, so from M = 17 on.
// For fewer channels swap-AB with stream-K keeps every SM busy.
bool small_m_dense(int64_t M, int64_t N, int sm_count, const Knobs& kn) {
  if (kn.schedule == 4 || kn.schedule == 5) return true;
  return M > 16 && M <= 128 && kn.schedule == 0 && kn.tile_n == 0 && (N + 223) / 224 >= sm_count * 3 / 4;
}

// Whether the pair kernel (256-row tiles over two SMs) takes a shape with
// more than 128 tokens when no schedule is forced.
bool pair_preferred(int64_t M, int64_t /*N*/, int64_t K) {
  return K >= kPairMinK || (M >= kPairManyTokens && K >= kPairMinKManyTokens);
}

// The schedule of one call: arrangement, kernel, tile widths and (swap-AB)
// stream-K with the workspace it needs.  `slots` is the number of CTA pairs
// that fit at once (the pair kernel's wave size), used only for the pair.
Plan make_plan(int64_t M, int64_t N, int64_t K, int sm_count, int pair_slots_n, const Knobs& kn) {
  Plan p{};
  p.kb_total = static_cast<int>((K + kDenseKB - 1) / kDenseKB);
  if (kn.schedule == 3 || (kn.schedule == 0 && M > 128 && pair_preferred(M, N, K))) {
    p.kind = Kind::Dense;
    p.pair = true;
    p.bn = (kn.tile_n == 160 || kn.tile_n == 192) ? kn.tile_n : 256;
    p.a_tiles = static_cast<int>((M + 255) / 256);
    p.b_tiles = static_cast<int>((N + p.bn - 1) / p.bn);
    p.num_tiles = p.a_tiles * p.b_tiles;
    if (p.bn == 256 && kn.two_widths && pair_slots_n > 0) plan_two_widths(p, N, pair_slots_n);
    return p;
  }
  const bool dense_small = M <= 128 && small_m_dense(M, N, sm_count, kn);
  if (M <= 128 && !dense_small) {
    p.kind = Kind::Swap;
    p.bn = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128;
    p.a_tiles = static_cast<int>((N + 127) / 128);
    p.b_tiles = static_cast<int>((M + p.bn - 1) / p.bn);
  } else {
    p.kind = Kind::Dense;
    p.bn = N <= 128 ? 128 : dense_small ? 224 : 256;
    if (kn.tile_n == 128 || kn.tile_n == 160 || kn.tile_n == 192 || kn.tile_n == 224 || kn.tile_n == 256)
      p.bn = kn.tile_n;
    p.a_tiles = static_cast<int>((M + 127) / 128);
    p.b_tiles = static_cast<int>((N + p.bn - 1) / p.bn);
  }
  p.num_tiles = p.a_tiles * p.b_tiles;
  const long long iters = static_cast<long long>(p.num_tiles) * p.kb_total;
  if (kn.schedule == 2 || kn.schedule == 5) {
    // forced stream-K (measurement): ranges over uniform tiles
    p.stream_k = iters >= sm_count;
    p.ws_bytes = p.stream_k ? sk_workspace_bytes(p, sm_count) : 0;
    return p;
  }
  // Stream-K pays when whole tiles would leave a large share of the SMs idle
  // in the last wave, and every CTA still gets a few k blocks.  Measured on
  // B200: for the dense arrangement splitting costs more than the idle SMs
  // of the last wave (both with red.add partials and with per-CTA partial
  // slots plus ready flags), so only swap-AB (few tokens, weight streaming)
  // splits.
  const int waves = (p.num_tiles + sm_count - 1) / sm_count;
  const double eff = static_cast<double>(p.num_tiles) / (static_cast<double>(waves) * sm_count);
  const bool worth = p.kind == Kind::Swap && eff < 0.9 && iters >= 4LL * sm_count;
  p.ws_bytes = worth ? sk_workspace_bytes(p, sm_count) : 0;
  p.stream_k = worth && kn.schedule != 1;
  if (!worth) p.ws_bytes = 0;
  if (p.kind == Kind::Dense && p.bn == 256 && kn.tile_n == 0 && kn.two_widths) plan_two_widths(p, N, sm_count);
  return p;
}

// Host-side checks of dq_int8_linear's arguments (shared with the
// allocation-free entry point, so both refuse the same calls).
dq_status check_linear_args(const int8_t* A, const float* s_row, int64_t M, int64_t K, const int8_t* W,
                            const float* s_col, int64_t N, const void* bias_bf16, const void* out,
                            dq_out_dtype out_dtype) {
  if (out_dtype != DQ_OUT_BF16 && out_dtype != DQ_OUT_S32) return DQ_ERR_INVALID_ARG;
  if (M < 0 || K < 1 || N < 1) return DQ_ERR_INVALID_ARG;
  if (M > 0 && (A == nullptr || W == nullptr || out == nullptr)) return DQ_ERR_INVALID_ARG;
  if (M > 0 && out_dtype == DQ_OUT_BF16 && (s_row == nullptr || s_col == nullptr))
    return DQ_ERR_INVALID_ARG;
  if (K % 16 != 0 || K > kMaxK || N % 8 != 0) return DQ_ERR_UNSUPPORTED;
  if (M > (int64_t(1) << 31) - 128 || N > (int64_t(1) << 31) - 256) return DQ_ERR_UNSUPPORTED;
  if (!aligned(A, 16) || !aligned(W, 16) || !aligned(out, 16)) return DQ_ERR_UNSUPPORTED;
  if (out_dtype == DQ_OUT_BF16 && (!aligned(s_col, 16) || (bias_bf16 && !aligned(bias_bf16, 16))))
    return DQ_ERR_UNSUPPORTED;
  return DQ_OK;
}

}  // namespace
}  // namespace dq

using namespace dq;

extern "C" {

size_t dq_int8_linear_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || N < 1 || K < 1) return 0;
  DeviceInfo* d = nullptr;
  if (current_device(&d) != DQ_OK) return 0;
  const Plan p = make_plan(M, N, K, d->sm_count, 0, knobs());
  return p.pair ? 0 : p.ws_bytes;
}

dq_status dq_int8_linear(const int8_t* A, const float* s_row, int64_t M, int64_t K, const int8_t* W,
                         const float* s_col, int64_t N, const void* bias_bf16, void* out,
                         dq_out_dtype out_dtype, void* workspace, size_t workspace_bytes,
                         dq_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  dq_status st0 = check_linear_args(A, s_row, M, K, W, s_col, N, bias_bf16, out, out_dtype);
  if (st0 != DQ_OK) return st0;
  DeviceInfo* d = nullptr;
  dq_status st = current_device(&d);
  if (st != DQ_OK) return st;
  if (M == 0) return DQ_OK;

  const Knobs kn = knobs();
  int pairs = 0;
  if (kn.schedule == 3 || (kn.schedule == 0 && M > 128 && pair_preferred(M, N, K))) {
    if ((st = pair_slots(*d, &pairs)) != DQ_OK) return st;
  }
  Plan p = make_plan(M, N, K, d->sm_count, pairs, kn);
  if (p.pair) {
    // Each 256-row tile's MMAs run on a pair of SMs (gemm2sm.cu).
    CUtensorMap ta, tb, tb2, tc;
    if ((st = make_tmap_u8_2d(&ta, A, K, M, K, kDenseKB, 128, kDenseKB)) != DQ_OK) return st;
    if ((st = make_tmap_u8_2d(&tb, W, K, N, K, kDenseKB, p.bn / 2, kDenseKB)) != DQ_OK) return st;
    if (p.bn2 > 0) {
      if ((st = make_tmap_u8_2d(&tb2, W, K, N, K, kDenseKB, p.bn2 / 2, kDenseKB)) != DQ_OK) return st;
    } else {
      tb2 = tb;
    }
    if ((st = make_tmap_out_2d(&tc, out, N, M, out_dtype == DQ_OUT_S32 ? 4 : 2)) != DQ_OK) return st;
    GemmArgs g{};
    g.M = static_cast<int>(M);
    g.N = static_cast<int>(N);
    g.K = static_cast<int>(K);
    g.a_tiles = p.a_tiles;
    g.b_tiles = p.b_tiles;
    g.kb_total = p.kb_total;
    g.num_tiles = p.num_tiles;
    g.t1 = p.t1;
    g.bn2 = p.bn2;
    g.mb0 = p.mb0;
    g.c_start = p.c_start;
    g.first_cnt = p.first_cnt;
    g.per_row = p.per_row;
    g.s_row = s_row;
    g.s_col = s_col;
    g.bias = static_cast<const uint16_t*>(bias_bf16);
    g.out = out;
    g.out_s32 = out_dtype == DQ_OUT_S32 ? 1 : 0;
    g.wait = WaitCtl{d->err_word, wait_timeout_ns()};
    return launch_pair_gemm(ta, tb, tb2, tc, g, p.bn, p.num_tiles < pairs ? p.num_tiles : pairs, stream);
  }

  // stream-K only with a large enough workspace (else whole tiles, same bits)
  const bool sk = p.stream_k && workspace != nullptr && workspace_bytes >= p.ws_bytes && aligned(workspace, 16);

  CUtensorMap ta, tb, tb2;
  const int8_t* a_src = p.kind == Kind::Swap ? W : A;
  const int8_t* b_src = p.kind == Kind::Swap ? A : W;
  const int64_t a_rows = p.kind == Kind::Swap ? N : M;
  const int64_t b_rows = p.kind == Kind::Swap ? M : N;
  if ((st = make_tmap_u8_2d(&ta, a_src, K, a_rows, K, kDenseKB, 128, kDenseKB)) != DQ_OK) return st;
  if ((st = make_tmap_u8_2d(&tb, b_src, K, b_rows, K, kDenseKB, p.bn, kDenseKB)) != DQ_OK) return st;
  if (p.bn2 > 0) {
    if ((st = make_tmap_u8_2d(&tb2, b_src, K, b_rows, K, kDenseKB, p.bn2, kDenseKB)) != DQ_OK) return st;
  } else {
    tb2 = tb;
  }
  CUtensorMap tc;
  if ((st = make_tmap_out_2d(&tc, out, N, M, out_dtype == DQ_OUT_S32 ? 4 : 2)) != DQ_OK) return st;
  const size_t slots_bytes = static_cast<size_t>(p.num_tiles) * p.bn * 128 * 4;

  GemmArgs g{};
  g.M = static_cast<int>(M);
  g.N = static_cast<int>(N);
  g.K = static_cast<int>(K);
  g.a_tiles = p.a_tiles;
  g.b_tiles = p.b_tiles;
  g.kb_total = p.kb_total;
  g.num_tiles = p.num_tiles;
  g.stream_k = sk ? 1 : 0;
  g.iters_total = static_cast<long long>(p.num_tiles) * p.kb_total;
  g.t1 = p.t1;
  g.bn2 = p.bn2;
  g.mb0 = p.mb0;
  g.c_start = p.c_start;
  g.first_cnt = p.first_cnt;
  g.per_row = p.per_row;
  g.s_row = s_row;
  g.s_col = s_col;
  g.bias = static_cast<const uint16_t*>(bias_bf16);
  g.out = out;
  g.out_s32 = out_dtype == DQ_OUT_S32 ? 1 : 0;
  if (sk) {
    g.ws = static_cast<int32_t*>(workspace);
    g.ws_cnt = reinterpret_cast<uint32_t*>(static_cast<char*>(workspace) + slots_bytes);
  }
  g.wait = WaitCtl{d->err_word, wait_timeout_ns()};
  const int grid = sk ? d->sm_count : (p.num_tiles < d->sm_count ? p.num_tiles : d->sm_count);

  if (p.kind == Kind::Dense) {
    switch (p.bn) {
      case 256: return launch<Kind::Dense, 256>(ta, tb, tb2, tc, g, grid, stream);
      case 224: return launch<Kind::Dense, 224>(ta, tb, tb2, tc, g, grid, stream);
      case 192: return launch<Kind::Dense, 192>(ta, tb, tb2, tc, g, grid, stream);
      case 160: return launch<Kind::Dense, 160>(ta, tb, tb2, tc, g, grid, stream);
      default: return launch<Kind::Dense, 128>(ta, tb, tb2, tc, g, grid, stream);
    }
  }
  switch (p.bn) {
    case 16: return launch<Kind::Swap, 16>(ta, tb, tb, tc, g, grid, stream);
    case 32: return launch<Kind::Swap, 32>(ta, tb, tb, tc, g, grid, stream);
    case 64: return launch<Kind::Swap, 64>(ta, tb, tb, tc, g, grid, stream);
    default: return launch<Kind::Swap, 128>(ta, tb, tb, tc, g, grid, stream);
  }
}

dq_status dq_fp8_linear(const uint8_t* A, const float* s_row, int64_t M, int64_t K, const uint8_t* W,
                        const float* s_col, int64_t N, const void* bias_bf16, void* out, dq_out_dtype out_dtype,
                        dq_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (out_dtype != DQ_OUT_BF16 && out_dtype != DQ_OUT_F32) return DQ_ERR_INVALID_ARG;
  if (M < 0 || K < 1 || N < 1) return DQ_ERR_INVALID_ARG;
  if (M > 0 && (A == nullptr || W == nullptr || out == nullptr)) return DQ_ERR_INVALID_ARG;
  if (M > 0 && out_dtype == DQ_OUT_BF16 && (s_row == nullptr || s_col == nullptr))
    return DQ_ERR_INVALID_ARG;
  const bool f32 = out_dtype == DQ_OUT_F32;
  if (K % 16 != 0 || N % (f32 ? 4 : 8) != 0) return DQ_ERR_UNSUPPORTED;
  if (M > (int64_t(1) << 31) - 128 || N > (int64_t(1) << 31) - 256 || K > (int64_t(1) << 20))
    return DQ_ERR_UNSUPPORTED;
  if (!aligned(A, 16) || !aligned(W, 16) || !aligned(out, 16)) return DQ_ERR_UNSUPPORTED;
  if (!f32 && (!aligned(s_col, 16) || (bias_bf16 && !aligned(bias_bf16, 16)))) return DQ_ERR_UNSUPPORTED;
  DeviceInfo* d = nullptr;
  dq_status st = current_device(&d);
  if (st != DQ_OK) return st;
  if (M == 0) return DQ_OK;

  // Many tokens (the int8 kernel's rule): the 2-SM pair kernel, 256 x 256
  // tiles over two SMs, two tile widths when the last wave is partial.
  const Knobs kn = knobs();
  if (N > 128 && (kn.schedule == 3 || (kn.schedule == 0 && M > 128 && pair_preferred(M, N, K)))) {
    int pairs = 0;
    if ((st = pair_slots(*d, &pairs)) != DQ_OK) return st;
    Plan p{};
    p.kind = Kind::DenseF8;
    p.pair = true;
    p.bn = 256;
    p.a_tiles = static_cast<int>((M + 255) / 256);
    p.b_tiles = static_cast<int>((N + p.bn - 1) / p.bn);
    p.kb_total = static_cast<int>((K + kDenseKB - 1) / kDenseKB);
    p.num_tiles = p.a_tiles * p.b_tiles;
    if (kn.two_widths) plan_two_widths(p, N, pairs);
    CUtensorMap ta, tb, tb2, tc;
    if ((st = make_tmap_u8_2d(&ta, A, K, M, K, kDenseKB, 128, kDenseKB)) != DQ_OK) return st;
    if ((st = make_tmap_u8_2d(&tb, W, K, N, K, kDenseKB, p.bn / 2, kDenseKB)) != DQ_OK) return st;
    if (p.bn2 > 0) {
      if ((st = make_tmap_u8_2d(&tb2, W, K, N, K, kDenseKB, p.bn2 / 2, kDenseKB)) != DQ_OK) return st;
    } else {
      tb2 = tb;
    }
    if ((st = make_tmap_out_2d(&tc, out, N, M, f32 ? 4 : 2)) != DQ_OK) return st;
    GemmArgs g{};
    g.M = static_cast<int>(M);
    g.N = static_cast<int>(N);
    g.K = static_cast<int>(K);
    g.a_tiles = p.a_tiles;
    g.b_tiles = p.b_tiles;
    g.kb_total = p.kb_total;
    g.num_tiles = p.num_tiles;
    g.t1 = p.t1;
    g.bn2 = p.bn2;
    g.mb0 = p.mb0;
    g.c_start = p.c_start;
    g.first_cnt = p.first_cnt;
    g.per_row = p.per_row;
    g.s_row = s_row;
    g.s_col = s_col;
    g.bias = static_cast<const uint16_t*>(bias_bf16);
    g.out = out;
    g.out_s32 = f32 ? 1 : 0;                   // raw accumulator bits
    g.wait = WaitCtl{d->err_word, wait_timeout_ns()};
    return launch_pair_gemm(ta, tb, tb2, tc, g, p.bn, p.num_tiles < pairs ? p.num_tiles : pairs, stream, true);
  }

  // The dense arrangement (tokens on MMA M), 128 x 256 tiles (128 x 128 for
  // N <= 128), two tile widths when the last wave is partial.
  Plan p{};
  p.kind = Kind::DenseF8;
  p.bn = N <= 128 ? 128 : 256;
  p.a_tiles = static_cast<int>((M + 127) / 128);
  p.b_tiles = static_cast<int>((N + p.bn - 1) / p.bn);
  p.kb_total = static_cast<int>((K + kDenseKB - 1) / kDenseKB);
  p.num_tiles = p.a_tiles * p.b_tiles;
  if (p.bn == 256 && kn.two_widths) plan_two_widths(p, N, d->sm_count);
  CUtensorMap ta, tb, tb2, tc;
  if ((st = make_tmap_u8_2d(&ta, A, K, M, K, kDenseKB, 128, kDenseKB)) != DQ_OK) return st;
  if ((st = make_tmap_u8_2d(&tb, W, K, N, K, kDenseKB, p.bn, kDenseKB)) != DQ_OK) return st;
  if (p.bn2 > 0) {
    if ((st = make_tmap_u8_2d(&tb2, W, K, N, K, kDenseKB, p.bn2, kDenseKB)) != DQ_OK) return st;
  } else {
    tb2 = tb;
  }
  if ((st = make_tmap_out_2d(&tc, out, N, M, f32 ? 4 : 2)) != DQ_OK) return st;
  GemmArgs g{};
  g.M = static_cast<int>(M);
  g.N = static_cast<int>(N);
  g.K = static_cast<int>(K);
  g.a_tiles = p.a_tiles;
  g.b_tiles = p.b_tiles;
  g.kb_total = p.kb_total;
  g.num_tiles = p.num_tiles;
  g.t1 = p.t1;
  g.bn2 = p.bn2;
  g.mb0 = p.mb0;
  g.c_start = p.c_start;
  g.first_cnt = p.first_cnt;
  g.per_row = p.per_row;
  g.s_row = s_row;
  g.s_col = s_col;
  g.bias = static_cast<const uint16_t*>(bias_bf16);
  g.out = out;
  g.out_s32 = f32 ? 1 : 0;                   // raw accumulator bits
  g.wait = WaitCtl{d->err_word, wait_timeout_ns()};
  const int grid = p.num_tiles < d->sm_count ? p.num_tiles : d->sm_count;
  if (p.bn == 256) return launch<Kind::DenseF8, 256>(ta, tb, tb2, tc, g, grid, stream);
  return launch<Kind::DenseF8, 128>(ta, tb, tb2, tc, g, grid, stream);
}

dq_status dq_bsr_int8_linear_blocked(const int8_t* A, const float* s_row, int64_t M, int64_t K, int64_t N,
                                     int64_t block, const int32_t* crow, const int32_t* col,
                                     const int8_t* values, int64_t nnzb, const float* s_col,
                                     const void* bias_bf16, void* out, dq_out_dtype out_dtype,
                                     dq_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (out_dtype != DQ_OUT_BF16 && out_dtype != DQ_OUT_S32) return DQ_ERR_INVALID_ARG;
  if (M < 0 || K < 1 || N < 1 || nnzb < 0) return DQ_ERR_INVALID_ARG;
  if (M > 0 && (A == nullptr || crow == nullptr || out == nullptr)) return DQ_ERR_INVALID_ARG;
  if (M > 0 && nnzb > 0 && (col == nullptr || values == nullptr)) return DQ_ERR_INVALID_ARG;
  if (M > 0 && out_dtype == DQ_OUT_BF16 && (s_row == nullptr || s_col == nullptr))
    return DQ_ERR_INVALID_ARG;
  if (block != 64 && block != 32 && block != 16) return DQ_ERR_UNSUPPORTED;
  if (K % block != 0 || N % block != 0 || K % 16 != 0 || K > 133120) return DQ_ERR_UNSUPPORTED;
  if (M > (int64_t(1) << 31) - 128 || N > (int64_t(1) << 31) - 256 || nnzb > (int64_t(1) << 24))
    return DQ_ERR_UNSUPPORTED;
  if (!aligned(A, 16) || !aligned(out, 16) || (values && !aligned(values, 16))) return DQ_ERR_UNSUPPORTED;
  if (out_dtype == DQ_OUT_BF16 && (!aligned(s_col, 16) || (bias_bf16 && !aligned(bias_bf16, 16))))
    return DQ_ERR_UNSUPPORTED;
  DeviceInfo* d = nullptr;
  dq_status st = current_device(&d);
  if (st != DQ_OK) return st;
  if (M == 0) return DQ_OK;

  // Panel variant (K <= 1280): each CTA keeps its 128 x K activation panel in
  // shared memory across consecutive tiles of the same 128-row block (A read
  // from L2 once per block row of tiles instead of once per weight block), so
  // A is described in 128 x 128-byte boxes with the 128-byte swizzle.
  // Streaming variant: A in k slices of 64 bytes (64-wide blocks) or 32 bytes
  // (32- and 16-wide blocks) x 128 rows, swizzled to the slice width.  B: the
  // blocks viewed as a [nnzb * block, block] byte matrix, one block per box;
  // 16-byte rows of 16-wide blocks are not swizzled.
  // Measured on B200 (ViT-H fc1, M=65792, K=1280): 32x32 blocks 627 us with
  // the panel vs 725 streaming, 16x16 2143 vs 2514; 64x64 blocks are as fast
  // or faster streaming (10 %: 266 vs 269 us, 20 %: 384 vs 396), where the
  // per-block MMA issue, not the activation traffic, bounds the kernel.
  const Knobs kn = knobs();
  const bool panel = K <= Cfg<Kind::Bsr, 256, true>::KP &&
                     (kn.bsr_panel == 2 || (kn.bsr_panel == 1 && block < 64));
  const int kb = panel ? 128 : block == 64 ? 64 : 32;
  const int bsw = block == 16 ? 0 : static_cast<int>(block);
  const uint32_t ub = static_cast<uint32_t>(block);
  CUtensorMap ta, tb;
  if ((st = make_tmap_u8_2d(&ta, A, K, M, K, kb, 128, kb)) != DQ_OK) return st;
  // With no blocks the B map is never read; describe A again to keep it valid.
  if (nnzb > 0) st = make_tmap_u8_2d(&tb, values, ub, static_cast<uint64_t>(nnzb) * ub, ub, ub, ub, bsw);
  else st = make_tmap_u8_2d(&tb, A, K, M, K, ub, ub, bsw);
  if (st != DQ_OK) return st;
  CUtensorMap tc;
  if ((st = make_tmap_out_2d(&tc, out, N, M, out_dtype == DQ_OUT_S32 ? 4 : 2)) != DQ_OK) return st;

  GemmArgs g{};
  g.M = static_cast<int>(M);
  g.N = static_cast<int>(N);
  g.K = static_cast<int>(K);
  g.a_tiles = static_cast<int>((M + 127) / 128);
  g.nbr = static_cast<int>(N / block);
  const int per_tile = static_cast<int>(256 / block);     // block rows per 256-channel tile
  g.b_tiles = (g.nbr + per_tile - 1) / per_tile;
  g.kb_total = 0;
  const int64_t tiles = static_cast<int64_t>(g.a_tiles) * g.b_tiles;
  if (tiles > 0x7fffffff) return DQ_ERR_UNSUPPORTED;
  g.num_tiles = static_cast<int>(tiles);
  g.stream_k = 0;
  g.s_row = s_row;
  g.s_col = s_col;
  g.bias = static_cast<const uint16_t*>(bias_bf16);
  g.out = out;
  g.out_s32 = out_dtype == DQ_OUT_S32 ? 1 : 0;
  g.crow = crow;
  g.col = col;
  g.nnzb = static_cast<int>(nnzb);
  g.idx_smem = !panel && (N / block + 1 + nnzb) <= Cfg<Kind::Bsr, 256>::IDX_INTS ? 1 : 0;
  g.blocked = panel ? 1 : 0;
  g.wait = WaitCtl{d->err_word, wait_timeout_ns()};
  const int grid = g.num_tiles < d->sm_count ? g.num_tiles : d->sm_count;
  if (panel) {
    if (block == 32) return launch<Kind::Bsr32, 256, true>(ta, tb, tb, tc, g, grid, stream);
    if (block == 16) return launch<Kind::Bsr16, 256, true>(ta, tb, tb, tc, g, grid, stream);
    return launch<Kind::Bsr, 256, true>(ta, tb, tb, tc, g, grid, stream);
  }
  if (block == 32) return launch<Kind::Bsr32, 256>(ta, tb, tb, tc, g, grid, stream);
  if (block == 16) return launch<Kind::Bsr16, 256>(ta, tb, tb, tc, g, grid, stream);
  return launch<Kind::Bsr, 256>(ta, tb, tb, tc, g, grid, stream);
}

dq_status dq_bsr_int8_linear(const int8_t* A, const float* s_row, int64_t M, int64_t K, int64_t N,
                             const int32_t* crow, const int32_t* col, const int8_t* values,
                             int64_t nnzb, const float* s_col, const void* bias_bf16, void* out,
                             dq_out_dtype out_dtype, dq_stream_t stream) {
  return dq_bsr_int8_linear_blocked(A, s_row, M, K, N, 64, crow, col, values, nnzb, s_col, bias_bf16, out,
                                    out_dtype, stream);
}

dq_status dq_bsr_pack_blocked(const int8_t* wq, int64_t N, int64_t K, int64_t block, const int32_t* crow,
                              const int32_t* col, int64_t nnzb, int8_t* values, dq_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (N < 1 || K < 1 || nnzb < 0 || wq == nullptr || crow == nullptr) return DQ_ERR_INVALID_ARG;
  if (nnzb > 0 && (col == nullptr || values == nullptr)) return DQ_ERR_INVALID_ARG;
  if (block != 64 && block != 32 && block != 16) return DQ_ERR_UNSUPPORTED;
  if (K % block != 0 || N % block != 0 || K % 16 != 0 || nnzb > (int64_t(1) << 24)) return DQ_ERR_UNSUPPORTED;
  if (!aligned(wq, 16) || (values && !aligned(values, 16))) return DQ_ERR_UNSUPPORTED;
  DeviceInfo* d = nullptr;
  dq_status st = current_device(&d);
  if (st != DQ_OK) return st;
  if (nnzb == 0) return DQ_OK;
  bsr_pack_kernel<<<static_cast<unsigned>(N / block), 256, 0, stream>>>(
      wq, K, crow, col, static_cast<int>(nnzb), static_cast<int>(K / block), static_cast<int>(block), values);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? DQ_OK : cuda_fail(e);
}

dq_status dq_bsr_pack(const int8_t* wq, int64_t N, int64_t K, const int32_t* crow, const int32_t* col,
                      int64_t nnzb, int8_t* values, dq_stream_t stream) {
  return dq_bsr_pack_blocked(wq, N, K, 64, crow, col, nnzb, values, stream);
}

dq_status dq_bsr_validate_blocked(const int32_t* crow, const int32_t* col, int64_t N, int64_t K, int64_t block,
                                  int64_t nnzb) {
  if (crow == nullptr || N < 1 || K < 1 || nnzb < 0 || block < 1 || N % block != 0 || K % block != 0)
    return DQ_ERR_INVALID_ARG;
  if (nnzb > 0 && col == nullptr) return DQ_ERR_INVALID_ARG;
  const int64_t nbr = N / block;
  int32_t* hc = new int32_t[nbr + 1];
  int32_t* hk = nnzb > 0 ? new int32_t[nnzb] : nullptr;
  dq_status st = DQ_OK;
  cudaError_t e = cudaMemcpy(hc, crow, (nbr + 1) * sizeof(int32_t), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && nnzb > 0) e = cudaMemcpy(hk, col, nnzb * sizeof(int32_t), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) {
    st = cuda_fail(e);
  } else {
    if (hc[0] != 0 || hc[nbr] != nnzb) st = DQ_ERR_INVALID_ARG;
    for (int64_t b = 0; st == DQ_OK && b < nbr; ++b)
      if (hc[b + 1] < hc[b]) st = DQ_ERR_INVALID_ARG;
    for (int64_t p = 0; st == DQ_OK && p < nnzb; ++p)
      if (hk[p] < 0 || hk[p] >= K / block) st = DQ_ERR_INVALID_ARG;
  }
  delete[] hc;
  delete[] hk;
  return st;
}

dq_status dq_bsr_validate(const int32_t* crow, const int32_t* col, int64_t N, int64_t K, int64_t nnzb) {
  return dq_bsr_validate_blocked(crow, col, N, K, 64, nnzb);
}

}  // extern "C"

// ---------------------------------------------------------------- no-alloc variant
//
// Scratch for dq_int8_linear_noalloc: callers that cannot allocate device
// memory get the stream-K workspace from this file-scope array instead.  In
// host code `g_noalloc_scratch` names a host-side stand-in, not the device
// array, so its device address is looked up once per device.
//
// The stream-K kernel leaves every partial tile and arrival counter it used
// at zero when it completes, so the array needs zeroing only before its first
// use on a device and after a kernel gave up a bounded wait (which can leave
// partial sums behind): dq_sync_status reports that as DQ_ERR_TIMEOUT and
// marks the device's array for re-zeroing by the next call.
namespace dq {
namespace {

static __device__ __align__(256) uint8_t g_noalloc_scratch[DQ_NOALLOC_SCRATCH_BYTES];

constexpr int kNoallocMaxDevices = 64;
void* g_noalloc_ptr[kNoallocMaxDevices] = {};
std::atomic<int> g_noalloc_dirty[kNoallocMaxDevices] = {};
std::mutex g_noalloc_mutex;

// Device address of the scratch array on the current device (set-up on the
// first call per device, with that device current): the address lookup and
// one zero-fill of the whole array on `stream`, which the call then waits
// for, so that later calls on any stream find it zero.  A re-zeroing asked
// for by dq_sync_status is queued on `stream` ahead of the call's kernel.
dq_status noalloc_scratch(cudaStream_t stream, void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kNoallocMaxDevices) return DQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    if ((e = cudaMemsetAsync(p, 0, DQ_NOALLOC_SCRATCH_BYTES, stream)) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaStreamSynchronize(stream)) != cudaSuccess) return cuda_fail(e);
    g_noalloc_ptr[dev] = p;
    g_noalloc_dirty[dev].store(0);
  } else if (g_noalloc_dirty[dev].exchange(0) != 0) {
    if ((e = cudaMemsetAsync(g_noalloc_ptr[dev], 0, DQ_NOALLOC_SCRATCH_BYTES, stream)) != cudaSuccess) {
      g_noalloc_dirty[dev].store(1);
      return cuda_fail(e);
    }
  }
  *out = g_noalloc_ptr[dev];
  return DQ_OK;
}

}  // namespace

void noalloc_mark_dirty(int device) {
  if (device >= 0 && device < kNoallocMaxDevices) g_noalloc_dirty[device].store(1);
}

}  // namespace dq

extern "C" dq_status dq_int8_linear_noalloc(const int8_t* A, const float* s_row, int64_t M, int64_t K,
                                            const int8_t* W, const float* s_col, int64_t N,
                                            const void* bias_bf16, void* out, dq_out_dtype out_dtype,
                                            dq_stream_t stream) {
  dq_status st = check_linear_args(A, s_row, M, K, W, s_col, N, bias_bf16, out, out_dtype);
  if (st != DQ_OK) return st;
  if (M == 0) return dq_int8_linear(A, s_row, M, K, W, s_col, N, bias_bf16, out, out_dtype, nullptr, 0, stream);
  DeviceInfo* d = nullptr;
  st = current_device(&d);
  if (st != DQ_OK) return st;
  const size_t need = dq_int8_linear_workspace_size(M, N, K);
  if (need > DQ_NOALLOC_SCRATCH_BYTES) return DQ_ERR_UNSUPPORTED;
  if (need == 0)
    return dq_int8_linear(A, s_row, M, K, W, s_col, N, bias_bf16, out, out_dtype, nullptr, 0, stream);
  void* scratch = nullptr;
  if ((st = noalloc_scratch(reinterpret_cast<cudaStream_t>(stream), &scratch)) != DQ_OK) return st;
  return dq_int8_linear(A, s_row, M, K, W, s_col, N, bias_bf16, out, out_dtype, scratch, need, stream);
}
