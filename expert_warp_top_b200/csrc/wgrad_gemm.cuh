// wgrad_gemm.cuh -- per-expert weight gradients on tcgen05.
//
// For every expert group g (rows group_off[g] .. group_off[g+1]-1):
//   C_g[m, n] = sum over the group's rows p of A[p, m] * B[p, n]
// with A [rows, M] and B [rows, N] row-major, i.e. C_g = A_g^T B_g.  Both
// operands are therefore MN-major and the contraction runs over the group's
// rows, whose count is ragged.  This is the weight gradient of a grouped
// GEMM: dW_down[g] = dO_g^T (w h)_g and dW_gate/up[g] = dZ_g^T X_g.
//
// Kernel shape (one persistent CTA per SM, 224 threads):
//   warp 0      TMA producer: per stage 64 rows of A (128 columns) and of B (BN
//               columns), each one 3-D load of 64-column strips (the tensor
//               seen as {64, rows, cols/64}), 128-byte swizzle
//   warp 1      MMA issuer, lane 0 alone: four MMAs per stage, unrolled, with
//               no warp-wide step between stages (a per-stage shuffle and two
//               warp syncs held the MMA rate to two thirds of the lane-0 loop)
//   warp 6      tail fixer: in a group's last, partial row block the rows past
//               the group's end belong to the next group, so the MMAs stop at
//               the 16-row block that holds the group's last row, and this
//               warp zeroes that block's foreign rows in shared memory (a
//               128-byte row of a swizzled box holds exactly one row) and then
//               signals the stage's fixed barrier, which the issuer waits for
//               on those stages only; the zeroing overlaps earlier MMAs.  It
//               waits for every fill and takes part in releasing every stage,
//               so its phase tracking stays exact
//   warps 2..5  epilogue: tcgen05.ld of 32 accumulator rows (= 32 values of m),
//               staged 128 bytes per row (32 fp32 or 64 bf16 columns) into one
//               of two 128-byte-swizzled shared-memory boxes of this warp
//               (double-buffered against the store in flight), then written
//               by one TMA tensor store (or TMA reduce-add when accumulating
//               fp32): whole 128-byte lines reach L2 instead of 16-byte pieces
//               of 32 rows.  bf16 accumulation reads and rewrites the rows
//               with plain loads and stores.
// Tiles: group by group, M block, N block fastest.  A group without rows
// writes zeros (or leaves the output as it is when accumulating).  Every wait
// is bounded, as in the forward kernel.
#pragma once
#include "ffn_gemm.cuh"

namespace moe {

#ifndef MOE_WGRAD_GROUP_BATCH
#define MOE_WGRAD_GROUP_BATCH 1
#endif
constexpr int kWgradGroupBatch = MOE_WGRAD_GROUP_BATCH;

struct WgradArgs {
  const int32_t* group_off;  // [G+1] device
  int G;
  int M, N;                  // output of one group: [M, N]
  int rows;                  // rows of A and B
  void* out;                 // [G, M, N]
  int accumulate;            // 1: out += C, 0: out = C
  unsigned* err;
  uint64_t wait_limit_ns;
  int debug;
};

constexpr int kWgradThreads = 224;  // 7 warps: producer, issuer, 4 epilogue, tail fixer

template <int BN>
struct WgradCfg {
  static constexpr int kBK = 64;                     // rows (the K of this GEMM) per stage
  static constexpr int kABytes = 128 * 128;          // 128 columns of A x 64 rows
  static constexpr int kBBytes = BN * 128;           // BN columns of B x 64 rows
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = (196608 / kStageBytes) > 8 ? 8 : (196608 / kStageBytes);
  static constexpr int kTmemCols = 2 * BN;
  static constexpr int kStoreBoxBytes = 32 * 128;  // one staging box: 32 rows x 128 bytes
  static constexpr int kStoreBoxes = 8;             // two per epilogue warp
  static constexpr size_t kSmemBytes =
      1024 + (size_t)kStages * kStageBytes + kStoreBoxes * kStoreBoxBytes + 512;
};

// tmap_a / tmap_b: A and B as 64-column strips (encode_strips), boxes of 64
// rows x 2 strips (A) and 64 rows x BN/64 strips (B).  tmap_out: the output as
// a 2-D [G*M, N] tensor of TOut, box of 32 rows x 128 bytes, 128-byte swizzle.
template <int BN, typename TOut>
__global__ void __launch_bounds__(kWgradThreads, 1)
    wgrad_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                      const __grid_constant__ CUtensorMap tmap_b,
                      const __grid_constant__ CUtensorMap tmap_out, const WgradArgs args) {
  static_assert(BN == 64 || BN == 128 || BN == 256, "BN must be 64, 128 or 256");
  using Cfg = WgradCfg<BN>;
  constexpr int S = Cfg::kStages;
  constexpr int kChunks = (Cfg::kABytes + Cfg::kBBytes) / 8192;  // 64-column boxes per stage

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* tiles = smem;
  uint8_t* store_boxes = smem + (size_t)S * Cfg::kStageBytes;  // 8 x 4 KB, 1024-aligned
  uint64_t* bars =
      reinterpret_cast<uint64_t*>(store_boxes + Cfg::kStoreBoxes * Cfg::kStoreBoxBytes);
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + S;
  uint64_t* tfull_bar = bars + 2 * S;
  uint64_t* tempty_bar = bars + 2 * S + 2;
  uint64_t* drain_bar = bars + 2 * S + 4;
  uint64_t* fixed_bar = bars + 2 * S + 5;  // [S]: a tail stage's foreign rows are zeroed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * S + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const unsigned lane = lane_id();
  const int G = args.G;
  const int m_blocks = args.M / 128, n_blocks = args.N / BN;
  const int tiles_per_group = m_blocks * n_blocks;
  const int total_tiles = G * tiles_per_group;

  if (warp == 0 && lane == 0) {
    tc::tma_prefetch_desc(&tmap_a);
    tc::tma_prefetch_desc(&tmap_b);
    tc::tma_prefetch_desc(&tmap_out);
    for (int s = 0; s < S; ++s) {
      tc::mbar_init(tc::smem_u32(&full_bar[s]), 1);
      tc::mbar_init(tc::smem_u32(&empty_bar[s]), 2);  // the MMAs' commit and the tail fixer
      tc::mbar_init(tc::smem_u32(&fixed_bar[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      tc::mbar_init(tc::smem_u32(&tfull_bar[a]), 1);
      tc::mbar_init(tc::smem_u32(&tempty_bar[a]), 4);
    }
    tc::mbar_init(tc::smem_u32(drain_bar), 1);
    *abort_flag = 0;
    tc::mbar_init_fence();
  }
  if (warp == 1) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), Cfg::kTmemCols);
    tc::tmem_relinquish();
  }
  pdl_enter();
  if (warp == 2 && blockIdx.x == 0) {
    // a group that leaves [0, rows] or runs backwards is treated as empty
    // (see group_rows) and raises the index error bit
    bool bad = false;
    for (int g = (int)lane; g < G; g += 32) {
      const int lo = args.group_off[g], hi = args.group_off[g + 1];
      bad |= !(lo >= 0 && hi >= lo && hi <= args.rows);
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) raise_error(args.err, kErrIndex);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const tc::WaitCtl wctl{abort_flag, args.err, args.wait_limit_ns};

  // Tiles go group batch by group batch (kWgradGroupBatch groups each); inside
  // a batch the groups alternate, so the CTAs running at one time spread over
  // the batch's groups instead of all reading one group's rows.
  auto locate = [&](int tile, int& g, int& m0, int& n0) {
    const int batch = tile / (kWgradGroupBatch * tiles_per_group);
    const int g0 = batch * kWgradGroupBatch;
    const int gb = min(kWgradGroupBatch, G - g0);
    const int r0 = tile - g0 * tiles_per_group;
    g = g0 + r0 % gb;
    const int r = r0 / gb;
    const int mb = r / n_blocks;
    m0 = mb * 128;
    n0 = (r - mb * n_blocks) * BN;
  };
  // rows [r0, r1) of group g (empty if its bounds are invalid)
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
      bool skip_next = (args.debug & kDebugSkipFirstLoad) != 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
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
            uint8_t* sa = tiles + (size_t)stage * Cfg::kStageBytes;
            const int y = r0 + kb * Cfg::kBK;
            tc::mbar_arrive_expect_tx(fb, Cfg::kStageBytes);
            // strip maps: {column in strip, row, strip}; one load per operand
            tc::tma_load_3d(tc::smem_u32(sa), &tmap_a, fb, 0, y, m0 / 64, pol);
            tc::tma_load_3d(tc::smem_u32(sa + Cfg::kABytes), &tmap_b, fb, 0, y, n0 / 64, pol);
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
          tc::wait_bounded(tc::smem_u32(&full_bar[s]), (armed_parity >> s) & 1u, wctl, false);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_f32acc<false, 128, BN, true, true>();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t fixed_parity = 0;  // per stage: the next completion of its fixed barrier
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        int g, m0, n0, r0, r1;
        locate(tile, g, m0, n0);
        group_rows(g, r0, r1);
        const int k_blocks = (r1 - r0 + Cfg::kBK - 1) / Cfg::kBK;
        if (!tc::wait_bounded(tc::smem_u32(&tempty_bar[acc]), acc_phase ^ 1u, wctl)) break;
        tc::fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < k_blocks; ++kb) {
          const int valid = min(Cfg::kBK, r1 - (r0 + kb * Cfg::kBK));
          bool got = tc::wait_bounded(tc::smem_u32(&full_bar[stage]), phase, wctl);
          if (got && valid % 16 != 0) {
            got = tc::wait_bounded(tc::smem_u32(&fixed_bar[stage]), (fixed_parity >> stage) & 1u,
                                   wctl);
            fixed_parity ^= 1u << stage;
          }
          if (!got) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t sa_u = tc::smem_u32(tiles + (size_t)stage * Cfg::kStageBytes);
          const uint64_t adesc = tc::desc_sw128_mnmajor(sa_u, 8192);
          const uint64_t bdesc = tc::desc_sw128_mnmajor(sa_u + Cfg::kABytes, 8192);
          // Unrolled with a guard per MMA: a loop bounded at run time cost a
          // fifth of the MMA rate.
          const int n_kk = (valid + 15) / 16;
#pragma unroll
          for (int kk = 0; kk < Cfg::kBK / 16; ++kk) {
            // +16 rows = two 1024-byte atoms = +128 in the address field
            const uint64_t off = static_cast<uint64_t>(kk * 128);
            if (kk < n_kk) tc::mma_f16(d_tmem, adesc + off, bdesc + off, idesc, (kb | kk) != 0);
          }
          tc::commit(tc::smem_u32(&empty_bar[stage]));
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc::commit(tc::smem_u32(&tfull_bar[acc]));  // also for an empty group
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      tc::commit(tc::smem_u32(drain_bar));
      tc::wait_bounded(tc::smem_u32(drain_bar), 0u, wctl, false);
    }
    __syncwarp();
  } else if (warp == 6) {
    // ------------------------------------------------------------ tail fixer
    // The same stage sequence as the producer and the issuer.  It waits for
    // every fill in order and releases every stage (the empty barrier counts
    // its arrival beside the MMAs' commit), so it can neither run a fill ahead
    // of the loads nor be lapped by them; only stages holding a group's
    // partial last row block are written.
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
      int g, m0, n0, r0, r1;
      locate(tile, g, m0, n0);
      group_rows(g, r0, r1);
      const int k_blocks = (r1 - r0 + Cfg::kBK - 1) / Cfg::kBK;
      for (int kb = 0; kb < k_blocks; ++kb) {
        bool got = true;
        if (lane == 0) got = tc::wait_bounded(tc::smem_u32(&full_bar[stage]), phase, wctl);
        if (!__shfl_sync(0xffffffffu, got, 0)) {
          ok = false;
          break;
        }
        const int valid = min(Cfg::kBK, r1 - (r0 + kb * Cfg::kBK));
        if (valid % 16 != 0) {
          // Rows valid.. of every strip belong to another group (or lie past
          // the tensor).  The MMAs read the stage in 16-row blocks up to the
          // one holding row valid - 1, so only that block's rows past valid
          // are zeroed; later rows are never read.
          uint8_t* sa = tiles + (size_t)stage * Cfg::kStageBytes;
          const int n16 = (((valid + 15) & ~15) - valid) * 8;  // 16-byte pieces per strip
          for (int c = 0; c < kChunks; ++c)
            for (int q = (int)lane; q < n16; q += 32)
              st_v4(sa + c * 8192 + valid * 128 + q * 16, make_uint4(0u, 0u, 0u, 0u));
          tc::fence_proxy_async_smem();  // generic-proxy writes -> tensor-core reads
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(tc::smem_u32(&fixed_bar[stage]));
        }
        if (lane == 0) tc::mbar_arrive(tc::smem_u32(&empty_bar[stage]));
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    constexpr int VN = Vec16<TOut>::n;             // values per 16-byte piece
    constexpr int kCols = 8 * VN;                  // columns per 128-byte row of a box
    // TMA path: plain store, or reduce-add for fp32 accumulation
    const bool tma_path = std::is_same<TOut, float>::value || !args.accumulate;
    uint8_t* my_boxes = store_boxes + quarter * 2 * Cfg::kStoreBoxBytes;  // this warp's two
    int n_stores = 0;
    TOut* out = reinterpret_cast<TOut*>(args.out);
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
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
      const int row0 = g * args.M + m0 + quarter * 32;  // first output row of this warp
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
            // boxes alternate; the store issued two boxes ago (same box) must
            // have read it before it is rewritten: at most one store pending
            uint8_t* box = my_boxes + (n_stores & 1) * Cfg::kStoreBoxBytes;
            const uint32_t box_u = tc::smem_u32(box);
            if (lane == 0) tc::bulk_wait_read_1();
            __syncwarp();
            // row `lane` of the box: 8 pieces of 16 bytes, piece j at slot j ^ (row & 7)
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
            // bf16 accumulation: read, add, write this row's columns
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
      if (lane == 0) tc::mbar_arrive(tc::smem_u32(&tempty_bar[acc]));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    // every store issued by this warp has completed before the CTA exits
    if (lane == 0) tc::bulk_wait_all();
    __syncwarp();
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

}  // namespace moe
