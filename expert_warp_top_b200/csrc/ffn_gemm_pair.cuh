// ffn_gemm_pair.cuh -- the grouped expert GEMM on CTA pairs (tcgen05 cta_group::2).
//
// Same computation as ffn_gemm.cuh (one expert group per tile, SwiGLU or
// gate-scaled epilogue), but a cluster of two CTAs works on a 256-row tile:
// each CTA holds its own 128 rows of A and one half (BN/2 rows) of the weight
// tile B, and one tcgen05.mma with M = 256 multiplies the pair's A by the whole
// B.  Per SM this halves the B bytes that TMA has to bring in (32 KB per
// k-block instead of 48 KB at BN = 256), which leaves room for a 6-deep
// shared-memory ring and lets the tensor pipe run closer to its peak.
//
// Roles, in both CTAs unless noted:
//   warp 0      TMA producer for this CTA's A rows and B half, into its own
//               shared memory (no multicast); both CTAs' loads count their
//               bytes on CTA 0's full barrier, which CTA 0 arms for the pair
//   warp 1      CTA 0 only: MMA issuer for the pair
//   warps 2..5  epilogue of this CTA's 128 accumulator rows (its own TMEM)
// Hand-offs across the pair: the MMA issuer's commits arrive on the empty and
// tfull barriers of both CTAs (multicast commit); CTA 1's epilogue warps
// arrive remotely on CTA 0's tempty barrier.  Every wait is bounded; a pair
// that gives up unwinds, drains its MMAs, meets at a cluster barrier and
// frees TMEM.
#pragma once
#include "ffn_gemm.cuh"

namespace moe {

constexpr int kPairBM = 256;  // rows per pair tile, 128 per CTA

// KCH: 128-byte K chunks per stage.  With 2, one 3-D load (the operand seen as
// 64-element strips {64, rows, K/64}) brings two consecutive K-major chunks of
// a tile, laid out one after the other as two 128-byte-swizzled tiles: half
// the TMA operations and barrier round trips per K of one chunk per stage.
template <int BN, bool TF32, int EPI, int KCH = 1>
struct PairCfg {
  static constexpr int kElemBytes = TF32 ? 4 : 2;
  static constexpr int kBK = KCH * 128 / kElemBytes;
  static constexpr int kMmaK = 32 / kElemBytes;
  static constexpr int kMmaPerStage = kBK / kMmaK;
  static constexpr int kAChunk = 128 * 128;          // this CTA's 128 rows x 128 bytes
  static constexpr int kBChunk = (BN / 2) * 128;     // its half of B x 128 bytes
  static constexpr int kABytes = KCH * kAChunk;      // this CTA's 128 rows of A
  static constexpr int kBBytes = KCH * kBChunk;      // this CTA's half of B
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kBoxesPerWarp = epi_boxes_per_warp<EPI>();
  static constexpr int kStages = ring_stages(kStageBytes, kBoxesPerWarp);
  // BN = 512 fills TMEM's 512 columns with one accumulator (no double buffer)
  static constexpr int kAccBufs = 2 * BN <= 512 ? 2 : 1;
  static constexpr int kTmemCols = kAccBufs * BN;
  // the MMA's N (at most 256) and the MMAs per K step that cover BN
  static constexpr int kMmaN = BN > 256 ? 256 : BN;
  static constexpr int kNSub = BN / kMmaN;
  static constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes +
                                       4 * kBoxesPerWarp * kEpiBoxBytes + 512 + kGroupTableBytes;
  static_assert(kSmemBytes <= (size_t)kSmemPerCta, "GEMM shared memory over the per-CTA limit");
};

// B_MN: B stored MN-major (B[g*K + k][n], n contiguous), seen by tmap_b as
// 64-column strips; each CTA loads its BN/2 columns in one 3-D load.
template <int BN, int EPI, bool TF32, bool B_MN = false, int KCH = 1>
__global__ void __launch_bounds__(kGemmThreads, 1)
    ffn_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a,
                         const __grid_constant__ CUtensorMap tmap_b,
                         const __grid_constant__ CUtensorMap tmap_out,
                         const __grid_constant__ CUtensorMap tmap_aux, const GemmArgs args) {
  static_assert(BN == 128 || BN == 256 || BN == 512, "pair tiles use BN = 128, 256 or 512");
  static_assert(BN <= 256 || (!B_MN && EPI != kEpiSwiGLUSave && EPI != kEpiSwiGLUBwd),
                "512-wide pair tiles: K-major weights, the inference epilogues");
  static_assert(!(B_MN && TF32), "MN-major B is bf16 only");
  static_assert(KCH == 1 || (KCH == 2 && !TF32 && BN <= 256),
                "two K chunks per stage: bf16, BN <= 256");
  using Cfg = PairCfg<BN, TF32, EPI, KCH>;
  using TOut = typename std::conditional<TF32, float, __nv_bfloat16>::type;
  constexpr int S = Cfg::kStages;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* tiles = smem;
  uint8_t* epi_boxes = smem + (size_t)S * Cfg::kStageBytes;  // 4 warps' boxes, 1024-aligned
  constexpr int kWarpBoxBytes = Cfg::kBoxesPerWarp * kEpiBoxBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(epi_boxes + 4 * kWarpBoxBytes);
  uint64_t* full_bar = bars;                 // [S] CTA 0: both CTAs' TMA -> MMA
  uint64_t* empty_bar = bars + S;            // [S] MMA (multicast) -> producers
  uint64_t* tfull_bar = bars + 2 * S;        // [2] MMA (multicast) -> epilogues
  uint64_t* tempty_bar = bars + 2 * S + 2;   // [2] CTA 0 only: 8 epilogue warps -> MMA
  uint64_t* drain_bar = bars + 2 * S + 4;    // [1] MMA drain at teardown
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_off = reinterpret_cast<int32_t*>(epi_boxes + 4 * kWarpBoxBytes + 512);
  int32_t* s_end = s_off + kGemmMaxGroups;
  int32_t* s_prefix = s_end + kGemmMaxGroups;

  const int warp = threadIdx.x >> 5;
  const unsigned lane = lane_id();
  const uint32_t rank = tc::cluster_ctarank();
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int G = args.G;
  const int n_blocks = args.N / BN;
  const int k_blocks = args.K / Cfg::kBK;

  if (warp == 0 && lane == 0) {
    tc::tma_prefetch_desc(&tmap_a);
    tc::tma_prefetch_desc(&tmap_b);
    for (int s = 0; s < S; ++s) {
      tc::mbar_init(tc::smem_u32(&full_bar[s]), 1);
      tc::mbar_init(tc::smem_u32(&empty_bar[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(tc::smem_u32(&tfull_bar[a]), 1);
      tc::mbar_init(tc::smem_u32(&tempty_bar[a]), 8);  // 4 epilogue warps x 2 CTAs
    }
    tc::mbar_init(tc::smem_u32(drain_bar), 1);
    *abort_flag = 0;
    tc::mbar_init_fence();
  }
  if (warp == 1) {
    tc::tmem_alloc_pair(tc::smem_u32(tmem_slot), Cfg::kTmemCols);
    tc::tmem_relinquish_pair();
  }
  pdl_enter();  // predecessors' outputs (group offsets, A rows) are visible from here
  if (warp == 2)
    group_tile_prefix(args.group_off, G, args.m_cap, kPairBM, n_blocks, args.tile_mode, s_off,
                      s_end, s_prefix, args.err);
  tc::fence_before_sync();
  __syncwarp();
  tc::cluster_sync();  // barriers of both CTAs initialised, TMEM allocated
  tc::fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const int total_tiles = s_prefix[G];
  const tc::WaitCtl wctl{abort_flag, args.err, args.wait_limit_ns};

  int last_mb = 0, last_nb = 0;  // the M and N block of the tile last located
  auto locate = [&](int tile, int& g, int& row0, int& gend, int& n0) {
    int lo = 0, hi = G;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_prefix[mid] <= tile) lo = mid;
      else hi = mid;
    }
    g = lo;
    const int local = tile - s_prefix[g];
    const int gstart = s_off[g];
    gend = s_end[g];
    const int m_blocks = group_m_blocks(gend - gstart, kPairBM, args.tile_mode);
    int nb, mb;
    if (args.raster) {
      mb = local / n_blocks;
      nb = local - mb * n_blocks;
    } else {
      nb = local / m_blocks;
      mb = local - nb * m_blocks;
    }
    row0 = gstart + mb * kPairBM;
    n0 = nb * BN;
    last_mb = mb;
    last_nb = nb;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_a = tc::policy_from_code(args.l2_a);
      const uint64_t pol_b = tc::policy_from_code(args.l2_b);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_parity = 0;
      bool skip_next = (args.debug & kDebugSkipFirstLoad) != 0 && rank == 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total_tiles; tile += n_pairs) {
        int g, row0, gend, n0;
        if (!B_MN && args.l2_prefetch && tile + n_pairs < total_tiles) {
          // This pair's next tile, one tile's time ahead: the first tile of its
          // M block (N block 0) brings this CTA's A rows, and the first tile of
          // its N block (M block 0) this CTA's half of the weight panel, into L2
          // (both contiguous: all K columns of consecutive rows).
          locate(tile + n_pairs, g, row0, gend, n0);
          const size_t kbytes = (size_t)args.K * Cfg::kElemBytes;
          const int r0 = row0 + (int)rank * 128;
          if (last_nb == 0 && r0 < gend)
            tc::bulk_prefetch_l2(static_cast<const uint8_t*>(args.a_ptr) + (size_t)r0 * kbytes,
                                 (uint32_t)(min(128, gend - r0) * kbytes));
          if (last_mb == 0)
            tc::bulk_prefetch_l2(static_cast<const uint8_t*>(args.b_ptr) +
                                     ((size_t)g * args.N + n0 + (int)rank * (BN / 2)) * kbytes,
                                 (uint32_t)((BN / 2) * kbytes));
        }
        locate(tile, g, row0, gend, n0);
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!tc::wait_bounded(tc::smem_u32(&empty_bar[stage]), phase ^ 1u, wctl)) {
            ok = false;
            break;
          }
          if (!skip_next) {
            const uint32_t fb = tc::smem_u32(&full_bar[stage]);
            const uint32_t fb_pair = tc::mapa_shared(fb, 0);  // the barrier in CTA 0
            uint8_t* sa = tiles + (size_t)stage * Cfg::kStageBytes;
            if (rank == 0) tc::mbar_arrive_expect_tx(fb, 2 * Cfg::kStageBytes);
            if (KCH == 2) {
              // strip map {element in chunk, row, chunk}: chunks 2kb, 2kb + 1
              tc::tma_load_3d_pair(tc::smem_u32(sa), &tmap_a, fb_pair, 0, row0 + (int)rank * 128,
                                   2 * kb, pol_a);
            } else {
              tc::tma_load_2d_pair(tc::smem_u32(sa), &tmap_a, fb_pair, kb * Cfg::kBK,
                                   row0 + (int)rank * 128, pol_a);
            }
            if (B_MN) {
              // strip map {column in strip, row, strip}: this CTA's BN/128 strips
              tc::tma_load_3d_pair(tc::smem_u32(sa + Cfg::kABytes), &tmap_b, fb_pair, 0,
                                   g * args.K + kb * Cfg::kBK, (n0 + (int)rank * (BN / 2)) / 64,
                                   pol_b);
            } else if (KCH == 2) {
              tc::tma_load_3d_pair(tc::smem_u32(sa + Cfg::kABytes), &tmap_b, fb_pair, 0,
                                   g * args.N + n0 + (int)rank * (BN / 2), 2 * kb, pol_b);
            } else if (BN > 256) {
              // two 256-column halves; CTA r loads rows [h*256 + r*128, +128) of the
              // panel, so that MMA h covers panel columns [h*256, h*256 + 256)
#pragma unroll
              for (int h = 0; h < Cfg::kNSub; ++h)
                tc::tma_load_2d_pair(tc::smem_u32(sa + Cfg::kABytes + h * 128 * 128), &tmap_b,
                                     fb_pair, kb * Cfg::kBK,
                                     g * args.N + n0 + h * 256 + (int)rank * 128, pol_b);
            } else {
              tc::tma_load_2d_pair(tc::smem_u32(sa + Cfg::kABytes), &tmap_b, fb_pair,
                                   kb * Cfg::kBK, g * args.N + n0 + (int)rank * (BN / 2), pol_b);
            }
            armed |= 1u << stage;
            armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          }
          skip_next = false;
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // CTA 0 waits for the last arming of every stage (its bytes include CTA 1's)
      if (rank == 0)
        for (int s = 0; s < S; ++s)
          if ((armed >> s) & 1u)
            tc::wait_bounded(tc::smem_u32(&full_bar[s]), (armed_parity >> s) & 1u, wctl, false);
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t idesc = tc::idesc_f32acc<TF32, 256, Cfg::kMmaN, false, B_MN>();
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total_tiles; tile += n_pairs) {
        if (!tc::wait_bounded_cluster(tc::smem_u32(&tempty_bar[acc]), acc_phase ^ 1u, wctl)) break;
        tc::fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!tc::wait_bounded_cluster(tc::smem_u32(&full_bar[stage]), phase, wctl)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t sa = tc::smem_u32(tiles + (size_t)stage * Cfg::kStageBytes);
          const uint64_t adesc = tc::desc_sw128_kmajor(sa);
          // MN-major B: strips of kBK rows x 128 bytes, one after the other
          const uint64_t bdesc = B_MN ? tc::desc_sw128_mnmajor(sa + Cfg::kABytes, Cfg::kBK * 128)
                                      : tc::desc_sw128_kmajor(sa + Cfg::kABytes);
#pragma unroll
          for (int kk = 0; kk < Cfg::kMmaPerStage; ++kk) {
            // +32 bytes per MMA along K inside a chunk's 128-byte rows (+2 in the
            // address field); the next chunk starts a whole chunk tile later
            constexpr int kPerChunk = 128 / 32;
            const int ch = kk / kPerChunk, ki = kk % kPerChunk;
            const uint64_t off = static_cast<uint64_t>(ch * (Cfg::kAChunk >> 4) + ki * 2);
            const uint64_t boff = B_MN ? static_cast<uint64_t>(kk * 128)
                                       : static_cast<uint64_t>(ch * (Cfg::kBChunk >> 4) + ki * 2);
#pragma unroll
            for (int h = 0; h < Cfg::kNSub; ++h) {
              // the h-th 256-column half: 16 KB further in shared memory, 256 TMEM columns on
              const uint64_t hoff = static_cast<uint64_t>(h * ((128 * 128) >> 4));
              const uint32_t dh = d_tmem + static_cast<uint32_t>(h * Cfg::kMmaN);
              if (TF32)
                tc::mma_tf32_pair(dh, adesc + off, bdesc + boff + hoff, idesc, (kb | kk) != 0);
              else
                tc::mma_f16_pair(dh, adesc + off, bdesc + boff + hoff, idesc, (kb | kk) != 0);
            }
          }
          // frees this stage in both CTAs once these MMAs have read it
          tc::commit_pair_multicast(tc::smem_u32(&empty_bar[stage]), 0x3);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc::commit_pair_multicast(tc::smem_u32(&tfull_bar[acc]), 0x3);
        if (++acc == Cfg::kAccBufs) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      tc::commit_pair_multicast(tc::smem_u32(drain_bar), 0x1);
      tc::wait_bounded(tc::smem_u32(drain_bar), 0u, wctl, false);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int r_in_half = quarter * 32 + (int)lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    const uint32_t tempty_local = tc::smem_u32(&tempty_bar[0]);
    for (int tile = pair; tile < total_tiles; tile += n_pairs) {
      int g, row0, gend, n0;
      if constexpr (EPI == kEpiSwiGLUBwd) {
        // this tile's saved rows (first tile only) and the next tile's, into L2
        for (int t = tile == pair ? tile : tile + n_pairs; t <= tile + n_pairs && t < total_tiles;
             t += n_pairs) {
          locate(t, g, row0, gend, n0);
          const int r = row0 + (int)rank * 128 + r_in_half;
          prefetch_aux_row<BN, EPI>(args, r < gend, (size_t)r, n0);
        }
      }
      locate(tile, g, row0, gend, n0);
      bool ok = true;
      if (lane == 0) ok = tc::wait_bounded(tc::smem_u32(&tfull_bar[acc]), acc_phase, wctl);
      ok = __shfl_sync(0xffffffffu, ok, 0) != 0;
      if (!ok) break;
      __syncwarp();
      tc::fence_after_sync();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(acc * BN);
      const int grow_i = row0 + (int)rank * 128 + r_in_half;
      const bool valid = grow_i < gend;
      epilogue_rows<BN, EPI, TOut>(taddr, valid, static_cast<size_t>(grow_i), n0, args,
                                   epi_boxes + quarter * kWarpBoxBytes, &tmap_out, &tmap_aux);
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        const uint32_t bar = tempty_local + static_cast<uint32_t>(acc * sizeof(uint64_t));
        if (rank == 0) tc::mbar_arrive(bar);
        else tc::mbar_arrive_remote(tc::mapa_shared(bar, 0));
      }
      if (++acc == Cfg::kAccBufs) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    // this warp's TMA stores have completed before the CTA exits
    if (lane == 0) tc::bulk_wait_all();
    __syncwarp();
  }

  // Both CTAs meet here only after their own work is done and the MMA issuer
  // has drained, so no MMA still reads the peer's shared memory or TMEM.
  tc::fence_before_sync();
  __syncwarp();
  tc::cluster_sync();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc_pair(tmem_base, Cfg::kTmemCols);
  }
}

}  // namespace moe
