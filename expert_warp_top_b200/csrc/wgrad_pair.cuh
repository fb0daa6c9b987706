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
//               shared memory; both CTAs' loads count their bytes on CTA 0's
//               full barrier, which CTA 0 arms for the pair (no multicast)
//   warp 1      CTA 0 only, lane 0 alone: issues the pair MMAs, whose commits
//               free the stage in both CTAs (multicast) and hand the
//               accumulator to both epilogues
//   warp 6      CTA 0 only, tail fixer: once a stage holding a ragged group's
//               last 16-row block has landed in both CTAs, zeroes that block's
//               foreign rows in both CTAs' boxes (the peer's through
//               distributed shared memory) and signals the stage's fixed
//               barrier, which the issuer waits for on those stages only.  It
//               waits for every fill and its arrival is counted by CTA 0's
//               empty barrier, so its phase tracking stays exact.
//   warps 2..5  epilogue of this CTA's 128 accumulator rows, through TMA
//               stores as in wgrad_gemm.cuh; they arrive on CTA 0's tempty
//               barrier (remotely from CTA 1)
// No stage needs a per-stage handshake between the CTAs: the full barrier
// sees both CTAs' bytes.  Every wait is bounded; a pair that gives up unwinds,
// drains its MMAs, meets at a cluster barrier and frees TMEM.
#pragma once
#include "wgrad_gemm.cuh"

namespace moe {
namespace tc {
// Proxy fence for generic writes to any CTA's shared memory in the cluster.
__device__ __forceinline__ void fence_proxy_async_smem_cluster() {
  asm volatile("fence.proxy.async.shared::cluster;" ::: "memory");
}
// 16-byte store to shared memory of a CTA of this cluster (mapa address).
__device__ __forceinline__ void st_cluster_v4(uint32_t cluster_addr, const uint4& v) {
  asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(cluster_addr), "r"(v.x),
               "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
}  // namespace tc

// BK: contracted rows per stage.  128 halves the TMA operations per row but
// loads up to 127 rows past a group's end; the host takes it for long groups.
template <int BN, int BK = 64>
struct WgradPairCfg {
  static_assert(BK == 64 || BK == 128, "stages of 64 or 128 contracted rows");
  static constexpr int kBK = BK;                    // contracted rows per stage
  static constexpr int kStripBytes = kBK * 128;     // one 64-column strip of kBK rows
  static constexpr int kABytes = 2 * kStripBytes;   // this CTA's 128 columns of A
  static constexpr int kBBytes = (BN / 128) * kStripBytes;  // this CTA's BN/2 columns of B
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = (196608 / kStageBytes) > 8 ? 8 : (196608 / kStageBytes);
  static constexpr int kTmemCols = 2 * BN;
  static constexpr int kStoreBoxBytes = 32 * 128;
  static constexpr int kStoreBoxes = 8;             // two per epilogue warp
  static constexpr size_t kSmemBytes =
      1024 + (size_t)kStages * kStageBytes + kStoreBoxes * kStoreBoxBytes + 512;
  static_assert(kSmemBytes <= 232448, "over the per-CTA shared-memory limit");
};

// tmap_a: A as 64-column strips, box BK rows x 2 strips; tmap_b: B as strips,
// box BK rows x BN/128 strips; tmap_out: the output [G*M, N], box 32 rows x
// 128 bytes.  M % 256 == 0, N % BN == 0.
template <int BN, typename TOut, int BK = 64>
__global__ void __launch_bounds__(kWgradThreads, 1)
    wgrad_pair_kernel(const __grid_constant__ CUtensorMap tmap_a,
                      const __grid_constant__ CUtensorMap tmap_b,
                      const __grid_constant__ CUtensorMap tmap_out, const WgradArgs args) {
  static_assert(BN == 128 || BN == 256, "pair tiles use BN = 128 or 256");
  using Cfg = WgradPairCfg<BN, BK>;
  constexpr int S = Cfg::kStages;
  constexpr int kChunks = Cfg::kStageBytes / Cfg::kStripBytes;  // 64-column strips per stage

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* tiles = smem;
  uint8_t* store_boxes = smem + (size_t)S * Cfg::kStageBytes;  // 8 x 4 KB, 1024-aligned
  uint64_t* bars =
      reinterpret_cast<uint64_t*>(store_boxes + Cfg::kStoreBoxes * Cfg::kStoreBoxBytes);
  uint64_t* full_bar = bars;               // [S] CTA 0: both CTAs' TMA -> MMA issuer
  uint64_t* empty_bar = bars + S;          // [S] MMA (multicast) -> producers
  uint64_t* tfull_bar = bars + 2 * S;      // [2] MMA (multicast) -> epilogues
  uint64_t* tempty_bar = bars + 2 * S + 2; // [2] CTA 0: 8 epilogue warps -> MMA issuer
  uint64_t* drain_bar = bars + 2 * S + 4;  // [1]
  uint64_t* fixed_bar = bars + 2 * S + 5;  // [S] CTA 0: tail fixer -> MMA issuer
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
      tc::mbar_init(tc::smem_u32(&full_bar[s]), 1);
      // CTA 0's stage is released by the MMAs' commit and by the tail fixer
      tc::mbar_init(tc::smem_u32(&empty_bar[s]), rank == 0 ? 2 : 1);
      tc::mbar_init(tc::smem_u32(&fixed_bar[s]), 1);
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
            const uint32_t fb = tc::smem_u32(&full_bar[stage]);
            const uint32_t fb_pair = tc::mapa_shared(fb, 0);  // the barrier in CTA 0
            uint8_t* sa = tiles + (size_t)stage * Cfg::kStageBytes;
            const int y = r0 + kb * Cfg::kBK;
            if (rank == 0) tc::mbar_arrive_expect_tx(fb, 2 * Cfg::kStageBytes);
            tc::tma_load_3d_pair(tc::smem_u32(sa), &tmap_a, fb_pair, 0, y,
                                 (m0 + (int)rank * 128) / 64, pol);
            tc::tma_load_3d_pair(tc::smem_u32(sa + Cfg::kABytes), &tmap_b, fb_pair, 0, y,
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
      // CTA 0 waits for the last arming of every stage (its bytes include CTA 1's)
      if (rank == 0)
        for (int s = 0; s < S; ++s)
          if ((armed >> s) & 1u)
            tc::wait_bounded(tc::smem_u32(&full_bar[s]), (armed_parity >> s) & 1u, wctl, false);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------ CTA 0: MMA issuer
    // (CTA 1's warp 1 has nothing to do after allocating TMEM)
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc = tc::idesc_f32acc<false, 256, BN, true, true>();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t fixed_parity = 0;  // per stage: the next completion of its fixed barrier
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total_tiles; tile += n_pairs) {
        int g, m0, n0, r0, r1;
        locate(tile, g, m0, n0);
        group_rows(g, r0, r1);
        const int k_blocks = (r1 - r0 + Cfg::kBK - 1) / Cfg::kBK;
        if (!tc::wait_bounded_cluster(tc::smem_u32(&tempty_bar[acc]), acc_phase ^ 1u, wctl)) break;
        tc::fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < k_blocks; ++kb) {
          const int valid = min(Cfg::kBK, r1 - (r0 + kb * Cfg::kBK));
          bool got = tc::wait_bounded_cluster(tc::smem_u32(&full_bar[stage]), phase, wctl);
          if (got && valid % 16 != 0) {
            got = tc::wait_bounded_cluster(tc::smem_u32(&fixed_bar[stage]),
                                           (fixed_parity >> stage) & 1u, wctl);
            fixed_parity ^= 1u << stage;
          }
          if (!got) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t sa_u = tc::smem_u32(tiles + (size_t)stage * Cfg::kStageBytes);
          const uint64_t adesc = tc::desc_sw128_mnmajor(sa_u, Cfg::kStripBytes);
          const uint64_t bdesc = tc::desc_sw128_mnmajor(sa_u + Cfg::kABytes, Cfg::kStripBytes);
          // unrolled with a guard per MMA, as in the single-CTA kernel
          const int n_kk = (valid + 15) / 16;
#pragma unroll
          for (int kk = 0; kk < Cfg::kBK / 16; ++kk) {
            // +16 rows = two 1024-byte atoms = +128 in the address field
            const uint64_t off = static_cast<uint64_t>(kk * 128);
            if (kk < n_kk) tc::mma_f16_pair(d_tmem, adesc + off, bdesc + off, idesc, (kb | kk) != 0);
          }
          // frees the stage in both CTAs once these MMAs have read it
          tc::commit_pair_multicast(tc::smem_u32(&empty_bar[stage]), 0x3);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc::commit_pair_multicast(tc::smem_u32(&tfull_bar[acc]), 0x3);  // also for an empty group
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      tc::commit_pair_multicast(tc::smem_u32(drain_bar), 0x1);
      tc::wait_bounded(tc::smem_u32(drain_bar), 0u, wctl, false);
    }
    __syncwarp();
  } else if (warp == 6) {
    // ------------------------------------------------------ CTA 0: tail fixer
    if (rank == 0) {
      const uint32_t peer_tiles = tc::mapa_shared(tc::smem_u32(tiles), 1);  // CTA 1's ring
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total_tiles; tile += n_pairs) {
        int g, m0, n0, r0, r1;
        locate(tile, g, m0, n0);
        group_rows(g, r0, r1);
        const int k_blocks = (r1 - r0 + Cfg::kBK - 1) / Cfg::kBK;
        for (int kb = 0; kb < k_blocks; ++kb) {
          bool got = true;
          if (lane == 0) got = tc::wait_bounded_cluster(tc::smem_u32(&full_bar[stage]), phase, wctl);
          if (!__shfl_sync(0xffffffffu, got, 0)) {
            ok = false;
            break;
          }
          const int valid = min(Cfg::kBK, r1 - (r0 + kb * Cfg::kBK));
          if (valid % 16 != 0) {
            // Rows valid.. of every strip, in both CTAs, belong to another
            // group.  The MMAs read the stage in 16-row blocks up to the one
            // holding row valid - 1, so only that block's rows past valid are
            // zeroed.  The full barrier has seen both CTAs' bytes land, so
            // these stores come after the TMA writes; the proxy fence and the
            // cluster-scope arrive order them before the MMAs.
            const int n16 = (((valid + 15) & ~15) - valid) * 8;  // 16-byte pieces per strip
            const uint32_t peer = peer_tiles + static_cast<uint32_t>(stage * Cfg::kStageBytes);
            for (int c = 0; c < kChunks; ++c)
              for (int q = (int)lane; q < n16; q += 32) {
                const uint32_t off =
                    static_cast<uint32_t>(c * Cfg::kStripBytes + valid * 128 + q * 16);
                st_v4(tiles + (size_t)stage * Cfg::kStageBytes + off, make_uint4(0u, 0u, 0u, 0u));
                tc::st_cluster_v4(peer + off, make_uint4(0u, 0u, 0u, 0u));
              }
            tc::fence_proxy_async_smem_cluster();
            __syncwarp();
            if (lane == 0)
              tc::mbar_arrive_remote(tc::mapa_shared(tc::smem_u32(&fixed_bar[stage]), 0));
          }
          if (lane == 0) tc::mbar_arrive(tc::smem_u32(&empty_bar[stage]));
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    constexpr int VN = Vec16<TOut>::n;
    constexpr int kCols = 8 * VN;
    const bool tma_path = std::is_same<TOut, float>::value || !args.accumulate;
    uint8_t* my_boxes = store_boxes + quarter * 2 * Cfg::kStoreBoxBytes;  // this warp's two
    int n_stores = 0;
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
            // boxes alternate; at most one store (the other box's) may still
            // be reading when this box is rewritten
            uint8_t* box = my_boxes + (n_stores & 1) * Cfg::kStoreBoxBytes;
            const uint32_t box_u = tc::smem_u32(box);
            if (lane == 0) tc::bulk_wait_read_1();
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
            ++n_stores;
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
