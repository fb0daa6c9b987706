// wgrad_pair.cuh -- the weight-gradient GEMM of wgrad_gemm.cuh on CTA pairs
// (tcgen05 cta_group::2).
//
// C_g = A_g^T B_g per expert group, as in wgrad_gemm.cuh, but a cluster of two
// CTAs computes a 256 x BN output tile with one M = 256 MMA: CTA r holds
// output rows (columns of A) m0 + 128 r .. m0 + 128 r + 127 and half of the
// B tile (BN/2 columns of B).  Per SM this brings in 32 KB of operands per 64
// contracted rows instead of 48 KB, a third less of the L2 -> SM traffic that
// bounds the single-CTA kernel.
//
// Roles, in both CTAs unless noted:
//   warp 0      TMA producer: this CTA's A strips and B half, into its own
//               shared memory, completing on its own load barrier
//   warp 1      waits for its own stage, zeroes the rows past a ragged group's
//               end in its own boxes, and arrives on CTA 0's ready barrier;
//               in CTA 0 its lane 0 then waits for both CTAs' arrivals and
//               issues the pair MMAs, whose commits free the stage in both
//               CTAs (multicast) and hand the accumulator to both epilogues
//   warps 2..5  epilogue of this CTA's 128 accumulator rows, through TMA
//               stores as in wgrad_gemm.cuh; they arrive on CTA 0's tempty
//               barrier (remotely from CTA 1)
// Every wait is bounded; a pair that gives up unwinds, drains its MMAs, meets
// at a cluster barrier and frees TMEM.
#pragma once
#include "wgrad_gemm.cuh"

namespace moe {

template <int BN>
struct WgradPairCfg {
  static constexpr int kBK = 64;                    // contracted rows per stage
  static constexpr int kABytes = 128 * 128;         // this CTA's 128 columns of A x 64 rows
  static constexpr int kBBytes = (BN / 2) * 128;    // this CTA's BN/2 columns of B x 64 rows
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = (196608 / kStageBytes) > 8 ? 8 : (196608 / kStageBytes);
  static constexpr int kTmemCols = 2 * BN;
  static constexpr int kStoreBoxBytes = 32 * 128;
  static constexpr size_t kSmemBytes =
      1024 + (size_t)kStages * kStageBytes + 4 * kStoreBoxBytes + 512;
};

// tmap_a: A as 64-column strips, box 64 rows x 2 strips; tmap_b: B as strips,
// box 64 rows x BN/128 strips; tmap_out: the output [G*M, N], box 32 rows x
// 128 bytes.  M % 256 == 0, N % BN == 0.
template <int BN, typename TOut>
__global__ void __launch_bounds__(kGemmThreads, 1)
    wgrad_pair_kernel(const __grid_constant__ CUtensorMap tmap_a,
                      const __grid_constant__ CUtensorMap tmap_b,
                      const __grid_constant__ CUtensorMap tmap_out, const WgradArgs args) {
  static_assert(BN == 128 || BN == 256, "pair tiles use BN = 128 or 256");
  using Cfg = WgradPairCfg<BN>;
  constexpr int S = Cfg::kStages;
  constexpr int kChunks = Cfg::kStageBytes / 8192;  // 64-column boxes per stage

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* tiles = smem;
  uint8_t* store_boxes = smem + (size_t)S * Cfg::kStageBytes;  // 4 x 4 KB, 1024-aligned
  uint64_t* bars = reinterpret_cast<uint64_t*>(store_boxes + 4 * Cfg::kStoreBoxBytes);
  uint64_t* load_bar = bars;               // [S] this CTA's TMA -> its warp 1
  uint64_t* ready_bar = bars + S;          // [S] CTA 0: both warps 1 -> MMA issuer
  uint64_t* empty_bar = bars + 2 * S;      // [S] MMA (multicast) -> producers
  uint64_t* tfull_bar = bars + 3 * S;      // [2] MMA (multicast) -> epilogues
  uint64_t* tempty_bar = bars + 3 * S + 2; // [2] CTA 0: 8 epilogue warps -> MMA issuer
  uint64_t* drain_bar = bars + 3 * S + 4;  // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * S + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const unsigned lane = lane_id();
  const uint32_t rank = tc::cluster_ctarank();
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int G = args.G;
  const int m_blocks = args.M / 256, n_blocks = args.N / BN;
  const int tiles_per_group = m_blocks * n_blocks;
  const int total_tiles = G * tiles_per_group;

  if (warp == 0 && lane == 0) {
    tc::tma_prefetch_desc(&tmap_a);
    tc::tma_prefetch_desc(&tmap_b);
    tc::tma_prefetch_desc(&tmap_out);
    for (int s = 0; s < S; ++s) {
      tc::mbar_init(tc::smem_u32(&load_bar[s]), 1);
      tc::mbar_init(tc::smem_u32(&ready_bar[s]), 2);  // one arrival from each CTA
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
  pdl_enter();
  if (warp == 2 && blockIdx.x == 0) {
    bool bad = false;
    for (int g = (int)lane; g < G; g += 32) {
      const int lo = args.group_off[g], hi = args.group_off[g + 1];
      bad |= !(lo >= 0 && hi >= lo && hi <= args.rows);
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) raise_error(args.err, kErrIndex);
  }
  tc::fence_before_sync();
  __syncwarp();
  tc::cluster_sync();  // barriers of both CTAs initialised, TMEM allocated
  tc::fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const tc::WaitCtl wctl{abort_flag, args.err, args.wait_limit_ns};

  // pair tile -> (group, first output row m0 of the pair, n0); group batches
  // as in the single-CTA kernel
  auto locate = [&](int tile, int& g, int& m0, int& n0) {
    const int batch = tile / (kWgradGroupBatch * tiles_per_group);
    const int g0 = batch * kWgradGroupBatch;
    const int gb = min(kWgradGroupBatch, G - g0);
    const int r0 = tile - g0 * tiles_per_group;
    g = g0 + r0 % gb;
    const int r = r0 / gb;
    const int mb = r / n_blocks;
    m0 = mb * 256;
    n0 = (r - mb * n_blocks) * BN;
  };
  auto group_rows = [&](int g, int& r0, int& r1) {
    const int lo = __ldg(args.group_off + g), hi = __ldg(args.group_off + g + 1);
    const bool ok = lo >= 0 && hi >= lo && hi <= args.rows;
    r0 = ok ? lo : 0;
    r1 = ok ? hi : 0;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = tc::policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_parity = 0;
      bool skip_next = (args.debug & kDebugSkipFirstLoad) != 0 && rank == 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total_tiles; tile += n_pairs) {
        int g, m0, n0, r0, r1;
        locate(tile, g, m0, n0);
        group_rows(g, r0, r1);
        const int k_blocks = (r1 - r0 + Cfg::kBK - 1) / Cfg::kBK;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!tc::wait_bounded(tc::smem_u32(&empty_bar[stage]), phase ^ 1u, wctl)) {
            ok = false;
            break;
          }
          if (!skip_next) {
            const uint32_t lb = tc::smem_u32(&load_bar[stage]);
            uint8_t* sa = tiles + (size_t)stage * Cfg::kStageBytes;
            const int y = r0 + kb * Cfg::kBK;
            tc::mbar_arrive_expect_tx(lb, Cfg::kStageBytes);
            tc::tma_load_3d(tc::smem_u32(sa), &tmap_a, lb, 0, y, (m0 + (int)rank * 128) / 64, pol);
            tc::tma_load_3d(tc::smem_u32(sa + Cfg::kABytes), &tmap_b, lb, 0, y,
                            (n0 + (int)rank * (BN / 2)) / 64, pol);
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
      for (int s = 0; s < S; ++s)
        if ((armed >> s) & 1u)
          tc::wait_bounded(tc::smem_u32(&load_bar[s]), (armed_parity >> s) & 1u, wctl, false);
    }
  } else if (warp == 1) {
    // ------------------------------ stage check + tail zeroing; CTA 0: MMA
    constexpr uint32_t idesc = tc::idesc_f32acc<false, 256, BN, true, true>();
    const uint32_t ready0 = tc::mapa_shared(tc::smem_u32(&ready_bar[0]), 0);  // in CTA 0
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int tile = pair; ok && tile < total_tiles; tile += n_pairs) {
      int g, m0, n0, r0, r1;
      locate(tile, g, m0, n0);
      group_rows(g, r0, r1);
      const int k_blocks = (r1 - r0 + Cfg::kBK - 1) / Cfg::kBK;
      bool go = true;
      if (rank == 0 && lane == 0)
        go = tc::wait_bounded_cluster(tc::smem_u32(&tempty_bar[acc]), acc_phase ^ 1u, wctl);
      if (!__shfl_sync(0xffffffffu, go, 0)) break;
      tc::fence_after_sync();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
      for (int kb = 0; kb < k_blocks; ++kb) {
        if (lane == 0) go = tc::wait_bounded(tc::smem_u32(&load_bar[stage]), phase, wctl);
        if (!__shfl_sync(0xffffffffu, go, 0)) {
          ok = false;
          break;
        }
        uint8_t* sa = tiles + (size_t)stage * Cfg::kStageBytes;
        const int valid = min(Cfg::kBK, r1 - (r0 + kb * Cfg::kBK));
        if (valid % 16 != 0) {
          // rows valid.. of this CTA's strips belong to another group; only
          // those in the last 16-row block the MMAs read need zeroing
          const int n16 = (((valid + 15) & ~15) - valid) * 8;
          for (int c = 0; c < kChunks; ++c)
            for (int q = (int)lane; q < n16; q += 32)
              st_v4(sa + c * 8192 + valid * 128 + q * 16, make_uint4(0u, 0u, 0u, 0u));
          tc::fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) {
          const uint32_t rb = ready0 + static_cast<uint32_t>(stage * sizeof(uint64_t));
          if (rank == 0) tc::mbar_arrive(tc::smem_u32(&ready_bar[stage]));
          else tc::mbar_arrive_remote(rb);
        }
        if (rank == 0 && lane == 0) {
          go = tc::wait_bounded_cluster(tc::smem_u32(&ready_bar[stage]), phase, wctl);
          if (go) {
            tc::fence_after_sync();
            const uint32_t sa_u = tc::smem_u32(sa);
            const uint64_t adesc = tc::desc_sw128_mnmajor(sa_u, 8192);
            const uint64_t bdesc = tc::desc_sw128_mnmajor(sa_u + Cfg::kABytes, 8192);
            const int n_kk = (valid + 15) / 16;
            for (int kk = 0; kk < n_kk; ++kk) {
              const uint64_t off = static_cast<uint64_t>(kk * 128);
              tc::mma_f16_pair(d_tmem, adesc + off, bdesc + off, idesc, (kb | kk) != 0);
            }
            // frees the stage in both CTAs once these MMAs have read it
            tc::commit_pair_multicast(tc::smem_u32(&empty_bar[stage]), 0x3);
          }
        }
        if (!__shfl_sync(0xffffffffu, go, 0)) {
          ok = false;
          break;
        }
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (rank == 0 && lane == 0)  // also for an empty group
        tc::commit_pair_multicast(tc::smem_u32(&tfull_bar[acc]), 0x3);
      __syncwarp();
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (rank == 0 && lane == 0) {
      tc::commit_pair_multicast(tc::smem_u32(drain_bar), 0x1);
      tc::wait_bounded(tc::smem_u32(drain_bar), 0u, wctl, false);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    constexpr int VN = Vec16<TOut>::n;
    constexpr int kCols = 8 * VN;
    const bool tma_path = std::is_same<TOut, float>::value || !args.accumulate;
    uint8_t* box = store_boxes + quarter * Cfg::kStoreBoxBytes;
    const uint32_t box_u = tc::smem_u32(box);
    const uint32_t tempty_local = tc::smem_u32(&tempty_bar[0]);
    TOut* out = reinterpret_cast<TOut*>(args.out);
    for (int tile = pair; tile < total_tiles; tile += n_pairs) {
      int g, m0, n0, r0, r1;
      locate(tile, g, m0, n0);
      group_rows(g, r0, r1);
      const bool has_rows = r1 > r0;
      bool ok = true;
      if (lane == 0) ok = tc::wait_bounded(tc::smem_u32(&tfull_bar[acc]), acc_phase, wctl);
      ok = __shfl_sync(0xffffffffu, ok, 0) != 0;
      if (!ok) break;
      __syncwarp();
      tc::fence_after_sync();
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * BN);
      const int row0 = g * args.M + m0 + (int)rank * 128 + quarter * 32;
      if (has_rows || !args.accumulate) {
#pragma unroll 1
        for (int c = 0; c < BN / kCols; ++c) {
          float v[kCols];
#pragma unroll
          for (int h = 0; h < kCols / 32; ++h) {
            if (has_rows) {
              uint32_t vr[32];
              tc::tmem_ld32(taddr + c * kCols + h * 32, vr);
              tc::tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 32; ++i) v[h * 32 + i] = __uint_as_float(vr[i]);
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) v[h * 32 + i] = 0.f;
            }
          }
          if (tma_path) {
            if (lane == 0) tc::bulk_wait_read_all();
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 8; ++j)
              st_v4(box + lane * 128 + ((j ^ (lane & 7)) << 4), Vec16<TOut>::from_f32(v + j * VN));
            tc::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              if (args.accumulate) tc::tma_reduce_add_2d(&tmap_out, box_u, n0 + c * kCols, row0);
              else tc::tma_store_2d(&tmap_out, box_u, n0 + c * kCols, row0);
              tc::bulk_commit_group();
            }
          } else {
            TOut* p = out + ((size_t)row0 + lane) * args.N + n0 + c * kCols;
#pragma unroll
            for (int q = 0; q < kCols / VN; ++q) {
              float old[VN];
              Vec16<TOut>::to_f32(ld_v4(p + q * VN), old);
#pragma unroll
              for (int i = 0; i < VN; ++i) v[q * VN + i] += old[i];
              st_v4(p + q * VN, Vec16<TOut>::from_f32(v + q * VN));
            }
          }
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        const uint32_t bar = tempty_local + static_cast<uint32_t>(acc * sizeof(uint64_t));
        if (rank == 0) tc::mbar_arrive(bar);
        else tc::mbar_arrive_remote(tc::mapa_shared(bar, 0));
      }
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (lane == 0) tc::bulk_wait_all();
    __syncwarp();
  }

  // both CTAs meet after their own work and the MMA drain
  tc::fence_before_sync();
  __syncwarp();
  tc::cluster_sync();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc_pair(tmem_base, Cfg::kTmemCols);
  }
}

}  // namespace moe
