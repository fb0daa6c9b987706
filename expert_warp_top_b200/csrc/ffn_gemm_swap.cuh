// ffn_gemm_swap.cuh -- the grouped expert GEMM with its operands swapped, for
// groups of few rows (the two inference epilogues, bf16).
//
// The same computation as ffn_gemm_pair.cuh, C[rows, n] = A[rows, :] . B[g*N + n, :]^T
// per group, but the weights are the MMA's M side and the group's rows its N
// side.  A CTA pair (tcgen05 cta_group::2) takes a tile of 256 weight rows
// (output features, 128 per CTA) by up to 256 of the group's rows, the N of the
// MMA being the tile's row count rounded up to 16.  A group of r rows is then
// padded to a multiple of 16 rows, not of 256: with a few hundred rows per group
// a quarter of the row-major tiles' MMA work can be padding.
//
// TMEM holds D^T: a lane per output feature, a column per row.  The epilogue
// turns it around through shared memory, 32 rows at a time: every warp writes
// its 32 features x 32 rows of fp32 accumulators into an exchange buffer, then
// reads it back one row per lane and writes whole output rows:
//   kEpiSwiGLU  the CTA's 128 weight rows are one gate/up interleave block
//               (64 gate rows, then the 64 matching up rows): warp q makes h
//               features 16q .. 16q + 15 of each row, silu(gate) * up
//   kEpiScale   warp q writes features 32q .. 32q + 31 of each row, times the
//               row's scale
// through a 128-byte-swizzled box and TMA stores; a 32-row chunk that runs past
// the group's end is stored row by row, so no row outside the group is written.
//
// The group's rows come in through one of five tensor maps whose boxes are 8,
// 16, 32, 64 and 128 rows high (per CTA), the smallest that covers the tile.
// Roles, barriers, bounded waits and teardown are those of ffn_gemm_pair.cuh.
#pragma once
#include "ffn_gemm_pair.cuh"

namespace moe {

constexpr int kSwapBM = 256;       // weight rows per pair tile (128 per CTA)
constexpr int kSwapMaxRows = 256;  // group rows per tile (the MMA's N, 16..256)
constexpr int kSwapMaps = 5;       // row-box heights 8 << i per CTA, i < 5
constexpr int kSwapMaxGroups = 256;
constexpr int kSwapExchStride = 33;  // floats per exchange row: 32 rows + 1 (no bank conflicts)

struct SwapCfg {
  static constexpr int kBK = 64;                 // bf16: one 128-byte swizzle row
  static constexpr int kMmaK = 16;
  static constexpr int kMmaPerStage = 4;
  static constexpr int kWBytes = 128 * 128;      // this CTA's 128 weight rows
  static constexpr int kABytes = 128 * 128;      // up to 128 of the group's rows
  static constexpr int kStageBytes = kWBytes + kABytes;
  static constexpr int kExchBytes = 128 * kSwapExchStride * 4;
  static constexpr int kBoxBytes = 2 * kEpiBoxBytes;  // 32 rows x 128 features (two boxes)
  static constexpr int kTableBytes = (int)sizeof(int32_t) * (3 * kSwapMaxGroups + 1);
  static constexpr int kStages =
      (kSmemPerCta - 1024 - 512 - kExchBytes - kBoxBytes - kTableBytes) / kStageBytes > 8
          ? 8
          : (kSmemPerCta - 1024 - 512 - kExchBytes - kBoxBytes - kTableBytes) / kStageBytes;
  static constexpr int kTmemCols = 2 * kSwapMaxRows;
  static constexpr size_t kSmemBytes =
      1024 + (size_t)kStages * kStageBytes + kExchBytes + kBoxBytes + 512 + kTableBytes;
  static_assert(kSmemBytes <= (size_t)kSmemPerCta, "GEMM shared memory over the per-CTA limit");
};

struct SwapMaps {
  CUtensorMap rows[kSwapMaps];  // A [m_cap, K], boxes of (8 << i) rows x 64 columns
};

// Named barrier of the four epilogue warps (id 1; __syncthreads uses 0).
__device__ __forceinline__ void epi_bar() {
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

template <int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
    ffn_gemm_swap_kernel(const __grid_constant__ SwapMaps tmap_rows,
                         const __grid_constant__ CUtensorMap tmap_w,
                         const __grid_constant__ CUtensorMap tmap_out, const GemmArgs args) {
  static_assert(EPI == kEpiSwiGLU || EPI == kEpiScale, "inference epilogues only");
  using Cfg = SwapCfg;
  constexpr int S = Cfg::kStages;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* tiles = smem;
  uint8_t* box = smem + (size_t)S * Cfg::kStageBytes;  // 1024-aligned
  float* exch = reinterpret_cast<float*>(box + Cfg::kBoxBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(box + Cfg::kBoxBytes + Cfg::kExchBytes);
  uint64_t* full_bar = bars;                 // [S] CTA 0: both CTAs' TMA -> MMA
  uint64_t* empty_bar = bars + S;            // [S] MMA (multicast) -> producers
  uint64_t* tfull_bar = bars + 2 * S;        // [2] MMA (multicast) -> epilogues
  uint64_t* tempty_bar = bars + 2 * S + 2;   // [2] CTA 0 only: 8 epilogue warps -> MMA
  uint64_t* drain_bar = bars + 2 * S + 4;    // [1] MMA drain at teardown
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* epi_ok = reinterpret_cast<volatile int*>(tmem_slot + 2);  // the tile's wait
  int32_t* s_off = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(bars) + 512);
  int32_t* s_end = s_off + kSwapMaxGroups;
  int32_t* s_prefix = s_end + kSwapMaxGroups;

  const int warp = threadIdx.x >> 5;
  const unsigned lane = lane_id();
  const uint32_t rank = tc::cluster_ctarank();
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int G = args.G;
  const int n_wblocks = args.N / kSwapBM;  // weight blocks of 256 rows per group
  const int k_blocks = args.K / Cfg::kBK;

  if (warp == 0 && lane == 0) {
    tc::tma_prefetch_desc(&tmap_w);
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
  pdl_enter();  // predecessors' outputs (group offsets, rows) are visible from here
  if (warp == 2)
    group_tile_prefix(args.group_off, G, args.m_cap, kSwapMaxRows, n_wblocks, kTilesAll, s_off,
                      s_end, s_prefix, args.err);
  tc::fence_before_sync();
  __syncwarp();
  tc::cluster_sync();  // barriers of both CTAs initialised, TMEM allocated
  tc::fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const int total_tiles = s_prefix[G];
  const tc::WaitCtl wctl{abort_flag, args.err, args.wait_limit_ns};

  // tile -> group g, weight rows [w0, w0 + 256), group rows [row0, row0 + nrows);
  // tiles run group by group, weight block by weight block, row chunk fastest,
  // so the pairs working at one time share a weight block in L2
  auto locate = [&](int tile, int& g, int& w0, int& row0, int& nrows) {
    int lo = 0, hi = G;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_prefix[mid] <= tile) lo = mid;
      else hi = mid;
    }
    g = lo;
    const int local = tile - s_prefix[g];
    const int gstart = s_off[g], gend = s_end[g];
    const int chunks = (gend - gstart + kSwapMaxRows - 1) / kSwapMaxRows;
    const int wb = local / chunks, ch = local - wb * chunks;
    w0 = wb * kSwapBM;
    row0 = gstart + ch * kSwapMaxRows;
    nrows = min(kSwapMaxRows, gend - row0);
  };
  // the MMA's N for a tile of n rows, and the box (8 << map) rows per CTA that covers it
  auto mma_n = [](int n) { return (n + 15) & ~15; };
  auto box_map = [](int half) {
    int m = 0;
    while ((8 << m) < half) ++m;
    return m;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_a = tc::policy_from_code(args.l2_a);
      const uint64_t pol_w = tc::policy_from_code(args.l2_b);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_parity = 0;
      bool skip_next = (args.debug & kDebugSkipFirstLoad) != 0 && rank == 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total_tiles; tile += n_pairs) {
        int g, w0, row0, nrows;
        locate(tile, g, w0, row0, nrows);
        const int half = mma_n(nrows) / 2;
        const int m = box_map(half);
        const uint32_t bytes = (uint32_t)(Cfg::kWBytes + (8 << m) * 128);
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!tc::wait_bounded(tc::smem_u32(&empty_bar[stage]), phase ^ 1u, wctl)) {
            ok = false;
            break;
          }
          if (!skip_next) {
            const uint32_t fb = tc::smem_u32(&full_bar[stage]);
            const uint32_t fb_pair = tc::mapa_shared(fb, 0);  // the barrier in CTA 0
            uint8_t* sw = tiles + (size_t)stage * Cfg::kStageBytes;
            if (rank == 0) tc::mbar_arrive_expect_tx(fb, 2 * bytes);
            tc::tma_load_2d_pair(tc::smem_u32(sw), &tmap_w, fb_pair, kb * Cfg::kBK,
                                 g * args.N + w0 + (int)rank * 128, pol_w);
            tc::tma_load_2d_pair(tc::smem_u32(sw + Cfg::kWBytes), &tmap_rows.rows[m], fb_pair,
                                 kb * Cfg::kBK, row0 + (int)rank * half, pol_a);
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
      constexpr uint32_t idesc0 = tc::idesc_f32acc<false, 256, 16>() & ~(0x3Fu << 17);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total_tiles; tile += n_pairs) {
        int g, w0, row0, nrows;
        locate(tile, g, w0, row0, nrows);
        const uint32_t idesc = idesc0 | (static_cast<uint32_t>(mma_n(nrows) >> 3) << 17);
        if (!tc::wait_bounded_cluster(tc::smem_u32(&tempty_bar[acc]), acc_phase ^ 1u, wctl)) break;
        tc::fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kSwapMaxRows);
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!tc::wait_bounded_cluster(tc::smem_u32(&full_bar[stage]), phase, wctl)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t sw = tc::smem_u32(tiles + (size_t)stage * Cfg::kStageBytes);
          const uint64_t wdesc = tc::desc_sw128_kmajor(sw);
          const uint64_t adesc = tc::desc_sw128_kmajor(sw + Cfg::kWBytes);
#pragma unroll
          for (int kk = 0; kk < Cfg::kMmaPerStage; ++kk) {
            const uint64_t off = static_cast<uint64_t>(kk * 2);  // +32 bytes along K
            tc::mma_f16_pair(d_tmem, wdesc + off, adesc + off, idesc, (kb | kk) != 0);
          }
          tc::commit_pair_multicast(tc::smem_u32(&empty_bar[stage]), 0x3);
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc::commit_pair_multicast(tc::smem_u32(&tfull_bar[acc]), 0x3);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      tc::commit_pair_multicast(tc::smem_u32(drain_bar), 0x1);
      tc::wait_bounded(tc::smem_u32(drain_bar), 0u, wctl, false);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lanes 32q .. 32q + 31 = local weight rows
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(args.out);
    const bool issuer = q == 0 && lane == 0;  // issues the chunk's tensor stores
    int acc = 0;
    uint32_t acc_phase = 0;
    const uint32_t tempty_local = tc::smem_u32(&tempty_bar[0]);
    for (int tile = pair; tile < total_tiles; tile += n_pairs) {
      int g, w0, row0, nrows;
      locate(tile, g, w0, row0, nrows);
      // one thread waits for the accumulator and tells the four warps, so that
      // they give up together (they meet at named barriers below)
      if (issuer) *epi_ok = tc::wait_bounded(tc::smem_u32(&tfull_bar[acc]), acc_phase, wctl);
      epi_bar();
      if (!*epi_ok) break;
      tc::fence_after_sync();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * kSwapMaxRows);
      const int n_chunks = (nrows + 31) / 32;
      // this CTA's 128 weight rows: output columns (kEpiScale) or h columns (kEpiSwiGLU)
      const int col0 = EPI == kEpiSwiGLU ? (w0 + (int)rank * 128) / 2 : w0 + (int)rank * 128;
      for (int c = 0; c < n_chunks; ++c) {
        uint32_t v[32];
        tc::tmem_ld32(taddr + c * 32, v);
        tc::tmem_ld_wait();
        if (c == n_chunks - 1) {
          // every accumulator column of the tile is in registers: free TMEM
          tc::fence_before_sync();
          __syncwarp();
          if (lane == 0) {
            const uint32_t bar = tempty_local + static_cast<uint32_t>(acc * sizeof(uint64_t));
            if (rank == 0) tc::mbar_arrive(bar);
            else tc::mbar_arrive_remote(tc::mapa_shared(bar, 0));
          }
        }
        // the last chunk's tensor stores have read the box before it is rewritten
        if (issuer) tc::bulk_wait_read_all();
        float* xrow = exch + (size_t)(q * 32 + (int)lane) * kSwapExchStride;
#pragma unroll
        for (int j = 0; j < 32; ++j) xrow[j] = __uint_as_float(v[j]);
        epi_bar();
        // one output row per lane
        const int r = c * 32 + (int)lane;  // row within the tile
        const bool valid = r < nrows;
        const bool full = c * 32 + 32 <= nrows;  // the same for every warp
        const size_t grow = (size_t)(row0 + r);
        if constexpr (EPI == kEpiSwiGLU) {
          float h[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float gv = exch[(size_t)(16 * q + i) * kSwapExchStride + lane];
            const float uv = exch[(size_t)(64 + 16 * q + i) * kSwapExchStride + lane];
            h[i] = gv * sigmoid_fast(gv) * uv;
          }
          const uint4 p0 = Vec16<__nv_bfloat16>::from_f32(h);
          const uint4 p1 = Vec16<__nv_bfloat16>::from_f32(h + 8);
          if (full) {
            // box: 32 rows x 128 bytes (64 h columns); warp q owns 16-byte pieces 2q, 2q + 1
            st_v4(box + lane * 128 + (((2 * q) ^ (lane & 7)) << 4), p0);
            st_v4(box + lane * 128 + (((2 * q + 1) ^ (lane & 7)) << 4), p1);
          } else if (valid) {
            __nv_bfloat16* dst = out + grow * args.ldo + col0 + 16 * q;
            st_v4(dst, p0);
            st_v4(dst + 8, p1);
          }
        } else {
          const float scale = (valid && args.row_scale) ? args.row_scale[grow] : 1.0f;
          float o[32];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            o[i] = exch[(size_t)(32 * q + i) * kSwapExchStride + lane] * scale;
          // two boxes of 32 rows x 64 columns; warp q owns pieces 4(q%2) .. 4(q%2)+3 of box q/2
          uint8_t* bq = box + (q >> 1) * kEpiBoxBytes;
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const uint4 pk = Vec16<__nv_bfloat16>::from_f32(o + 8 * t);
            if (full) {
              st_v4(bq + lane * 128 + (((4 * (q & 1) + t) ^ (lane & 7)) << 4), pk);
            } else if (valid) {
              st_v4(out + grow * args.ldo + col0 + 32 * q + 8 * t, pk);
            }
          }
        }
        tc::fence_proxy_async_smem();
        epi_bar();  // the exchange may be rewritten; the box is complete
        if (full && issuer) {
          const int grow0 = row0 + c * 32;
          if constexpr (EPI == kEpiSwiGLU) {
            tc::tma_store_2d(&tmap_out, tc::smem_u32(box), col0, grow0);
          } else {
            tc::tma_store_2d(&tmap_out, tc::smem_u32(box), col0, grow0);
            tc::tma_store_2d(&tmap_out, tc::smem_u32(box + kEpiBoxBytes), col0 + 64, grow0);
          }
          tc::bulk_commit_group();
        }
      }
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    // this CTA's tensor stores have completed before it exits
    if (issuer) tc::bulk_wait_all();
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
