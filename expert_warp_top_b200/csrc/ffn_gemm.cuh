// ffn_gemm.cuh -- grouped GEMM over ragged expert row groups on tcgen05.
//
// The expert computation of the Occult pipeline (Occult paper, TL;DR:
// "sparse-matrix-multiplication pipeline"): every expert multiplies only its
// own compact EPD rows.  Group g covers rows group_off[g] .. group_off[g+1]-1
// of A and uses weight block g of B:
//   C[rows, n] = sum_k A[rows, k] * B[g*N + n, k]      (both K-major)
//
// Kernel shape (one persistent CTA per SM, 192 threads):
//   warp 0      TMA producer: A tile 128 x 64 and B tile BN x 64 (bf16; 32 wide
//               for fp32/TF32) per stage, 128-byte swizzle, STAGES-deep ring.
//               With a row index (GATHER), the A tile's rows are gathered:
//               each of the 32 lanes issues one tile::gather4 of 4 rows, so the
//               compact EPD rows are read straight out of the SFD payload.
//   warp 1      TMEM owner and MMA issuer: tcgen05.mma M=128, N=BN, K=16 (8 for
//               TF32), accumulators double-buffered in TMEM (2 x BN columns)
//   warps 2..5  epilogue: tcgen05.ld of its 32 TMEM lanes (= 32 tile rows),
//               fused SwiGLU (GEMM 1) or gate-weight scaling (GEMM 2), or
//               the training variants below; the warp's 32 rows go through
//               128-byte-swizzled staging boxes and TMA stores, except in a
//               warp that straddles its group's end, which stores its valid
//               rows directly (a tile never writes past its group)
// Tiles are ordered group by group, N block by N block, M block fastest, and
// dealt round-robin to the CTAs; the same weight block is then read by
// neighbouring CTAs at the same time and stays in L2.
//
// Every mbarrier wait is bounded (globaltimer); a wait that expires raises the
// timeout bit of the device error flag and the CTA unwinds: the producer
// waits for its own TMA copies in flight, the MMA issuer drains its MMAs, and
// TMEM is freed before the kernel returns.
#pragma once
#include <type_traits>

#include "tc_ptx.cuh"

namespace moe {

constexpr int kGemmBM = 128;
constexpr int kGemmThreads = 192;
constexpr int kGemmMaxGroups = 1024;
constexpr int kEpiSwiGLU = 0;  // out[:, n0/2 + j] = silu(gate) * up   (64-row interleave)
constexpr int kEpiScale = 1;   // out[:, n0 + j]   = row_scale * acc
// Training forward of GEMM 1: the pre-activations (gate and up columns, in the
// GEMM's own interleaved column order) are kept, rounded to bf16, in aux_out
// [rows, ld_aux], and out receives silu(gate) * up of those rounded values.
constexpr int kEpiSwiGLUSave = 2;
// Backward of the SwiGLU and of the gate scaling, fused behind the dgrad GEMM
// dH' = dO_rows . W_down (the un-gated gradient of h).  With z = the saved
// pre-activations (aux_in, interleaved like kEpiSwiGLUSave), s = sigmoid(z_g),
// h = bf16(z_g s z_u) and w = row_scale (1 if null):
//   aux_out  dZ: dz_g = w dH' z_u s (1 + z_g (1 - s)),  dz_u = w dH' z_g s
//   out      w h                     (the A^T operand of the down weight gradient)
//   partial  sum over this tile's columns of dH' h  (the gate gradient, per
//            row and N block: partial[row * n_part + n0 / BN])
constexpr int kEpiSwiGLUBwd = 3;

// Debug switch used by the timeout test: the producer skips the first stage it
// would load, so the MMA issuer's wait can never complete.
constexpr int kDebugSkipFirstLoad = 1;


// The logistic sigmoid of SiLU, 1 / (1 + e^-x), with the fast division
// (__fdividef: a reciprocal and a multiply).  The IEEE division is a
// subroutine with a special-case branch, and the epilogues take one per
// element.  x -> -inf gives 0, x -> +inf gives 1.
__device__ __forceinline__ float sigmoid_fast(float x) {
  return __fdividef(1.0f, 1.0f + __expf(-x));
}

// Shared-memory staging of one epilogue warp: a box of 32 rows x 128 bytes in
// the 128-byte swizzle, written out by a TMA tensor store.
constexpr int kEpiBoxBytes = 32 * 128;

// Staging boxes per epilogue warp.  The training epilogues write three row
// pieces per 64 columns of h (gate and up pre-activations or their gradients,
// and h or w h), so they get three; the others write one.
#ifndef MOE_STAGE_SAVE_EPI
#define MOE_STAGE_SAVE_EPI 1
#endif
template <int EPI>
__host__ __device__ constexpr int epi_boxes_per_warp() {
  return (EPI == kEpiSwiGLUBwd || (EPI == kEpiSwiGLUSave && MOE_STAGE_SAVE_EPI != 0)) ? 3 : 1;
}

// Shared memory of one GEMM CTA: 1 KB alignment slack, the operand ring, the
// epilogue boxes of 4 warps, 512 bytes of barriers and the group tables.  The
// ring takes as many stages (up to 8) as the opt-in limit per CTA on sm_100
// (227 KB) leaves.
constexpr int kSmemPerCta = 232448;
constexpr int kGroupTableBytes = (int)sizeof(int32_t) * (3 * kGemmMaxGroups + 1);
__host__ __device__ constexpr int ring_stages(int stage_bytes, int boxes_per_warp) {
  return (kSmemPerCta - 1024 - 512 - kGroupTableBytes - 4 * boxes_per_warp * kEpiBoxBytes) /
                     stage_bytes > 8
             ? 8
             : (kSmemPerCta - 1024 - 512 - kGroupTableBytes - 4 * boxes_per_warp * kEpiBoxBytes) /
                   stage_bytes;
}

template <int BN, bool TF32, int EPI>
struct GemmCfg {
  static constexpr int kElemBytes = TF32 ? 4 : 2;
  static constexpr int kBK = 128 / kElemBytes;       // one 128-byte swizzle row
  static constexpr int kMmaK = 32 / kElemBytes;      // K of one tcgen05.mma
  static constexpr int kMmaPerStage = kBK / kMmaK;   // = 4
  static constexpr int kABytes = kGemmBM * 128;
  static constexpr int kBBytes = BN * 128;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kBoxesPerWarp = epi_boxes_per_warp<EPI>();
  static constexpr int kStages = ring_stages(kStageBytes, kBoxesPerWarp);
  static constexpr int kTmemCols = (2 * BN) < 32 ? 32 : 2 * BN;  // a power of two here
  static constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes +
                                       4 * kBoxesPerWarp * kEpiBoxBytes + 512 + kGroupTableBytes;
  static_assert(kSmemBytes <= (size_t)kSmemPerCta, "GEMM shared memory over the per-CTA limit");
};

struct GemmArgs {
  const int32_t* group_off;  // [G+1] device
  const int32_t* a_row_index;  // GATHER: row of A feeding each of the m_cap rows
  int a_rows;                // GATHER: rows of A
  int G;
  int N;                     // output columns per group (B rows per group)
  int K;
  int m_cap;                 // rows of A and of out
  const float* row_scale;    // kEpiScale: per-row factor (nullable)
  void* out;
  int ldo;                   // out row stride, elements
  unsigned* err;
  uint64_t wait_limit_ns;
  int debug;
  // kEpiSwiGLUSave / kEpiSwiGLUBwd only
  const void* aux_in = nullptr;  // saved pre-activations [rows, ld_aux]
  void* aux_out = nullptr;       // pre-activations (save) or their gradient (bwd)
  int ld_aux = 0;
  float* partial = nullptr;      // gate-gradient partials [rows, n_part] (nullable)
  int n_part = 0;
  int tile_mode = 0;             // kTilesAll / kTilesPairNoSmallTail / kTilesSmallTail
  // L2 policies (0 evict_normal, 1 evict_last, 2 evict_first): of the A-row
  // loads, the weight loads and the epilogue's tensor stores of `out`
  int l2_a = 0, l2_b = 1, l2_out = 0;
  // tile order inside a group: 0 M blocks fastest (concurrently running CTAs
  // share one weight block in L2), 1 N blocks fastest (they share A rows)
  int raster = 0;
  // L2 prefetch of the next tile's first-use operand panels (CTA-pair kernel,
  // K-major operands): the base addresses of A [m_cap, K] and B [G*N, K]
  const void* a_ptr = nullptr;
  const void* b_ptr = nullptr;
  int l2_prefetch = 0;
};

// Which rows of each group a launch covers, for mixing CTA-pair and single-CTA
// tiles: a group of r rows has r / 256 full pair tiles and a tail of r % 256.
//   kTilesAll              every row, in tiles of the kernel's own height
//   kTilesPairNoSmallTail  pair tiles (256 rows): the full ones, and the tail
//                          only when it is longer than 128 rows
//   kTilesSmallTail        single-CTA tiles (128 rows): only a tail of 1..128
//                          rows, which then needs half a pair tile's MMA work
constexpr int kTilesAll = 0;
constexpr int kTilesPairNoSmallTail = 1;
constexpr int kTilesSmallTail = 2;

__device__ __forceinline__ int group_m_blocks(int rows, int bm, int mode) {
  if (mode == kTilesPairNoSmallTail) return rows / 256 + (rows % 256 > 128 ? 1 : 0);
  if (mode == kTilesSmallTail) return (rows % 256 > 0 && rows % 256 <= 128) ? 1 : 0;
  return (rows + bm - 1) / bm;
}
// First row of a group's first tile in the launch.
__device__ __forceinline__ int group_first_row(int gstart, int rows, int mode) {
  return mode == kTilesSmallTail ? gstart + (rows / 256) * 256 : gstart;
}

__device__ __forceinline__ float round_bf16(float v) {
  return __bfloat162float(__float2bfloat16_rn(v));
}

// Writes 64 bf16 values of this thread's row at column `col` of `out`.  When
// the warp's 32 rows are all inside the group (`full`), the rows go through
// the warp's box and one TMA store (whole 128-byte lines); otherwise each
// valid row is stored directly, so that no row past the group's end is
// touched.  Warp-collective.
__device__ __forceinline__ void store_row64_bf16(const float* v, bool valid, bool full,
                                                 size_t grow, int wrow0, int col,
                                                 __nv_bfloat16* out, int ldo, uint8_t* box,
                                                 const CUtensorMap* tmap_out, int l2_out) {
  const unsigned lane = lane_id();
  if (full) {
    if (lane == 0) tc::bulk_wait_read_all();  // the box's previous store has read it
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 8; ++j)
      st_v4(box + lane * 128 + ((j ^ (lane & 7)) << 4), Vec16<__nv_bfloat16>::from_f32(v + j * 8));
    tc::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      if (l2_out) tc::tma_store_2d_hint(tmap_out, tc::smem_u32(box), col, wrow0,
                                        tc::policy_from_code(l2_out));
      else tc::tma_store_2d(tmap_out, tc::smem_u32(box), col, wrow0);
      tc::bulk_commit_group();
    }
  } else if (valid) {
    __nv_bfloat16* dst = out + grow * ldo + col;
#pragma unroll
    for (int j = 0; j < 8; ++j) st_v4(dst + j * 8, Vec16<__nv_bfloat16>::from_f32(v + j * 8));
  }
}

// kEpiSwiGLUBwd reads, for its row, the saved pre-activations of the tile's BN
// columns of h: 2 BN contiguous bf16 values (gate and up).  The epilogue warps
// ask L2 for them one tile ahead, so those loads wait on L2, not on HBM.
template <int BN, int EPI>
__device__ __forceinline__ void prefetch_aux_row(const GemmArgs& args, bool valid, size_t grow,
                                                 int n0) {
  if constexpr (EPI == kEpiSwiGLUBwd) {
    if (valid)
      tc::bulk_prefetch_l2(
          reinterpret_cast<const __nv_bfloat16*>(args.aux_in) + grow * args.ld_aux + 2 * n0,
          4 * BN);
  }
}

// Epilogue of one accumulator tile for this thread's TMEM lane (= one tile
// row): tcgen05.ld 32 columns at a time, fused SwiGLU or row scaling, and the
// row's stores (bf16 SwiGLU / scale: through the warp's staging box and TMA
// stores, see store_row64_bf16).  Every lane of the warp must call it
// (tcgen05.ld is warp-collective); `valid` masks the stores.
template <int BN, int EPI, typename TOut>
__device__ __forceinline__ void epilogue_rows(uint32_t taddr, bool valid, size_t grow, int n0,
                                              const GemmArgs& args, uint8_t* box,
                                              const CUtensorMap* tmap_out,
                                              const CUtensorMap* tmap_aux) {
  TOut* out = reinterpret_cast<TOut*>(args.out);
  const int ldo = args.ldo;
  const float* row_scale = args.row_scale;
  constexpr bool kBf16 = std::is_same<TOut, __nv_bfloat16>::value;
  const bool full = __all_sync(0xffffffffu, valid);
  const int wrow0 = __shfl_sync(0xffffffffu, (int)grow, 0);  // the warp's rows are consecutive
  const unsigned lane = lane_id();
  // The training epilogues stage 64 columns of h at a time in the warp's three
  // boxes (gate piece, up piece, h piece), as two halves of 32, then write
  // them with three TMA stores; a warp that straddles a group's end stores
  // its valid rows directly.  put(b, j, v) writes 16-byte piece j of this
  // lane's 128-byte row of box b (swizzled).
  [[maybe_unused]] auto put = [&](int b, int j, const uint4& v) {
    st_v4(box + b * kEpiBoxBytes + lane * 128 + ((j ^ (lane & 7)) << 4), v);
  };
  [[maybe_unused]] auto boxes_free = [&]() {  // the boxes' previous stores have read them
    if (lane == 0) tc::bulk_wait_read_all();
    __syncwarp();
  };
  [[maybe_unused]] auto store_boxes = [&](int zcol, int hcol) {
    tc::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tc::tma_store_2d(tmap_aux, tc::smem_u32(box), zcol, wrow0);
      tc::tma_store_2d(tmap_aux, tc::smem_u32(box + kEpiBoxBytes), zcol + 64, wrow0);
      tc::tma_store_2d(tmap_out, tc::smem_u32(box + 2 * kEpiBoxBytes), hcol, wrow0);
      tc::bulk_commit_group();
    }
  };
  if constexpr (EPI == kEpiSwiGLUSave) {
    static_assert(std::is_same<TOut, __nv_bfloat16>::value,
                  "the training epilogue is bf16 only");
    constexpr bool kStaged = epi_boxes_per_warp<EPI>() == 3;
    TOut* z = reinterpret_cast<TOut*>(args.aux_out);
#pragma unroll 1
    for (int p = 0; p < BN / 128; ++p) {
      if (kStaged && full) boxes_free();
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        uint32_t gr[32], ur[32];
        tc::tmem_ld32(taddr + p * 128 + h * 32, gr);
        tc::tmem_ld32(taddr + p * 128 + 64 + h * 32, ur);
        tc::tmem_ld_wait();
        if (valid) {
          float gv[32], uv[32], hv[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            gv[i] = round_bf16(__uint_as_float(gr[i]));
            uv[i] = round_bf16(__uint_as_float(ur[i]));
            hv[i] = gv[i] * sigmoid_fast(gv[i]) * uv[i];
          }
          if (kStaged && full) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              put(0, h * 4 + v, Vec16<TOut>::from_f32(gv + v * 8));
              put(1, h * 4 + v, Vec16<TOut>::from_f32(uv + v * 8));
              put(2, h * 4 + v, Vec16<TOut>::from_f32(hv + v * 8));
            }
          } else {
            TOut* zg = z + grow * args.ld_aux + n0 + p * 128 + h * 32;
            TOut* dst = out + grow * ldo + (n0 >> 1) + p * 64 + h * 32;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              st_v4(zg + v * 8, Vec16<TOut>::from_f32(gv + v * 8));
              st_v4(zg + 64 + v * 8, Vec16<TOut>::from_f32(uv + v * 8));
              st_v4(dst + v * 8, Vec16<TOut>::from_f32(hv + v * 8));
            }
          }
        }
      }
      if (kStaged && full) store_boxes(n0 + p * 128, (n0 >> 1) + p * 64);
    }
  } else if constexpr (EPI == kEpiSwiGLUBwd) {
    static_assert(std::is_same<TOut, __nv_bfloat16>::value,
                  "the training epilogue is bf16 only");
    static_assert(BN % 64 == 0, "the SwiGLU backward epilogue works in 64-column steps");
    const TOut* z = reinterpret_cast<const TOut*>(args.aux_in);
    TOut* dz = reinterpret_cast<TOut*>(args.aux_out);
    const float w = (valid && row_scale) ? row_scale[grow] : 1.0f;
    float dgp = 0.f;
    // z offset of h column i0 (a multiple of 32): gate and up 64 apart
    auto z_off = [&](int i0) {
      return grow * args.ld_aux + (size_t)((i0 >> 6) * 128 + (i0 & 63));
    };
    // the saved pre-activations of chunk c + 1 are loaded while chunk c computes
    uint4 zn[8];
    if (valid) {
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        zn[v] = ld_v4(z + z_off(n0) + v * 8);
        zn[4 + v] = ld_v4(z + z_off(n0) + 64 + v * 8);
      }
    }
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      uint32_t vr[32];
      tc::tmem_ld32(taddr + c * 32, vr);
      uint4 zc[8];
#pragma unroll
      for (int v = 0; v < 8; ++v) zc[v] = zn[v];
      if (valid && c + 1 < BN / 32) {
        const size_t zo = z_off(n0 + (c + 1) * 32);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          zn[v] = ld_v4(z + zo + v * 8);
          zn[4 + v] = ld_v4(z + zo + 64 + v * 8);
        }
      }
      tc::tmem_ld_wait();
      if (full && (c & 1) == 0) boxes_free();
      const int i0 = n0 + c * 32;  // column of h (= of W_down's f axis)
      if (valid) {
        float zg[32], zu[32], dg[32], du[32], hg[32];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          Vec16<TOut>::to_f32(zc[v], zg + v * 8);
          Vec16<TOut>::to_f32(zc[4 + v], zu + v * 8);
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float dh = __uint_as_float(vr[i]);
          const float sg = sigmoid_fast(zg[i]);
          const float silu = zg[i] * sg;
          const float hv = round_bf16(silu * zu[i]);
          dgp += dh * hv;
          const float dhw = w * dh;
          dg[i] = dhw * zu[i] * sg * (1.0f + zg[i] * (1.0f - sg));
          du[i] = dhw * silu;
          hg[i] = w * hv;
        }
        if (full) {
          const int jb = (c & 1) * 4;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            put(0, jb + v, Vec16<TOut>::from_f32(dg + v * 8));
            put(1, jb + v, Vec16<TOut>::from_f32(du + v * 8));
            put(2, jb + v, Vec16<TOut>::from_f32(hg + v * 8));
          }
        } else {
          const size_t zoff = z_off(i0);
          TOut* dst = out + grow * ldo + i0;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            st_v4(dz + zoff + v * 8, Vec16<TOut>::from_f32(dg + v * 8));
            st_v4(dz + zoff + 64 + v * 8, Vec16<TOut>::from_f32(du + v * 8));
            st_v4(dst + v * 8, Vec16<TOut>::from_f32(hg + v * 8));
          }
        }
      }
      // after the second half of a 64-column step: gate and up of h columns
      // [i0 - 32, i0 + 32) sit at z columns 2 (i0 - 32) and 2 (i0 - 32) + 64
      if (full && (c & 1) == 1) store_boxes(2 * (i0 - 32), i0 - 32);
    }
    if (valid && args.partial) args.partial[grow * args.n_part + n0 / BN] = dgp;
  } else if constexpr (EPI == kEpiSwiGLU && kBf16) {
    // columns [128p, 128p+64) are gate rows, [128p+64, 128p+128) the matching
    // up rows: 64 h columns per p, one 128-byte row of bf16
#pragma unroll 1
    for (int p = 0; p < BN / 128; ++p) {
      float hv[64];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t gr[32], ur[32];
        tc::tmem_ld32(taddr + p * 128 + h * 32, gr);
        tc::tmem_ld32(taddr + p * 128 + 64 + h * 32, ur);
        tc::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float gv = __uint_as_float(gr[i]);
          const float uv = __uint_as_float(ur[i]);
          hv[h * 32 + i] = gv * sigmoid_fast(gv) * uv;
        }
      }
      store_row64_bf16(hv, valid, full, grow, wrow0, (n0 >> 1) + p * 64, out, ldo, box, tmap_out,
                       args.l2_out);
    }
  } else if constexpr (EPI == kEpiScale && kBf16) {
    const float scale = (valid && row_scale) ? row_scale[grow] : 1.0f;
#pragma unroll 1
    for (int c = 0; c < BN / 64; ++c) {
      float v[64];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t vr[32];
        tc::tmem_ld32(taddr + c * 64 + h * 32, vr);
        tc::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) v[h * 32 + i] = __uint_as_float(vr[i]) * scale;
      }
      store_row64_bf16(v, valid, full, grow, wrow0, n0 + c * 64, out, ldo, box, tmap_out,
                       args.l2_out);
    }
  } else if constexpr (EPI == kEpiSwiGLU) {
    // (fp32 output) columns [128p, 128p+64) gate, [128p+64, 128p+128) up
#pragma unroll 1
    for (int p = 0; p < BN / 128; ++p) {
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        uint32_t gr[32], ur[32];
        tc::tmem_ld32(taddr + p * 128 + h * 32, gr);
        tc::tmem_ld32(taddr + p * 128 + 64 + h * 32, ur);
        tc::tmem_ld_wait();
        if (valid) {
          float hv[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float gv = __uint_as_float(gr[i]);
            const float uv = __uint_as_float(ur[i]);
            hv[i] = gv * sigmoid_fast(gv) * uv;
          }
          TOut* dst = out + grow * ldo + (n0 >> 1) + p * 64 + h * 32;
#pragma unroll
          for (int v = 0; v < 32 / Vec16<TOut>::n; ++v)
            st_v4(dst + v * Vec16<TOut>::n, Vec16<TOut>::from_f32(hv + v * Vec16<TOut>::n));
        }
      }
    }
  } else {
    const float scale = (valid && row_scale) ? row_scale[grow] : 1.0f;
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      uint32_t vr[32];
      tc::tmem_ld32(taddr + c * 32, vr);
      tc::tmem_ld_wait();
      if (valid) {
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(vr[i]) * scale;
        TOut* dst = out + grow * ldo + n0 + c * 32;
#pragma unroll
        for (int q = 0; q < 32 / Vec16<TOut>::n; ++q)
          st_v4(dst + q * Vec16<TOut>::n, Vec16<TOut>::from_f32(v + q * Vec16<TOut>::n));
      }
    }
  }
}

// Tile prefix of the groups (one warp): s_off/s_end hold each group's rows
// (a group whose bounds leave [0, m_cap] or run backwards is treated as empty
// and raises the index error bit); s_prefix[g] = first tile of group g, where
// group g has group_m_blocks(rows, bm, mode) * n_blocks tiles; s_prefix[G] =
// all tiles.
__device__ __forceinline__ void group_tile_prefix(const int32_t* group_off, int G, int m_cap,
                                                  int bm, int n_blocks, int mode, int32_t* s_off,
                                                  int32_t* s_end, int32_t* s_prefix,
                                                  unsigned* err) {
  const unsigned lane = lane_id();
  int carry = 0;
  bool bad = false;
  for (int g0 = 0; g0 < G; g0 += 32) {
    const int g = g0 + (int)lane;
    int tiles_g = 0;
    if (g < G) {
      const int lo = group_off[g], hi = group_off[g + 1];
      const bool ok = lo >= 0 && hi >= lo && hi <= m_cap;
      bad |= !ok;
      s_off[g] = lo;
      s_end[g] = ok ? hi : lo;
      const int rows = ok ? hi - lo : 0;
      tiles_g = group_m_blocks(rows, bm, mode) * n_blocks;
    }
    int inc = tiles_g;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, inc, o);
      if ((int)lane >= o) inc += y;
    }
    if (g < G) s_prefix[g] = carry + inc - tiles_g;
    carry += __shfl_sync(0xffffffffu, inc, 31);
  }
  if (lane == 0) s_prefix[G] = carry;
  if (__any_sync(0xffffffffu, bad) && lane == 0 && blockIdx.x == 0) raise_error(err, kErrIndex);
}

// B_MN: B is stored MN-major -- B[g*K + k][n], n contiguous (a weight used
// transposed, as in the input-gradient GEMMs) -- and tmap_b sees it as
// 64-column strips {64, G*K, N/64}: one load brings BN/64 strips of 64 K rows.
template <int BN, int EPI, bool TF32, bool GATHER, bool B_MN = false>
__global__ void __launch_bounds__(kGemmThreads, 1)
    ffn_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                    const __grid_constant__ CUtensorMap tmap_b,
                    const __grid_constant__ CUtensorMap tmap_out,
                    const __grid_constant__ CUtensorMap tmap_aux, const GemmArgs args) {
  using Cfg = GemmCfg<BN, TF32, EPI>;
  using TOut = typename std::conditional<TF32, float, __nv_bfloat16>::type;
  constexpr int S = Cfg::kStages;
  static_assert(!(B_MN && TF32), "MN-major B is bf16 only");
  static_assert(!B_MN || BN % 64 == 0, "MN-major B needs BN a multiple of 64");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* tiles = smem;
  uint8_t* epi_boxes = smem + (size_t)S * Cfg::kStageBytes;  // 4 warps' boxes, 1024-aligned
  constexpr int kWarpBoxBytes = Cfg::kBoxesPerWarp * kEpiBoxBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(epi_boxes + 4 * kWarpBoxBytes);
  uint64_t* full_bar = bars;            // [S]   TMA -> MMA
  uint64_t* empty_bar = bars + S;       // [S]   MMA -> TMA
  uint64_t* tfull_bar = bars + 2 * S;   // [2]   MMA -> epilogue
  uint64_t* tempty_bar = bars + 2 * S + 2;  // [2] epilogue -> MMA
  uint64_t* drain_bar = bars + 2 * S + 4;   // [1] MMA drain at teardown
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_off = reinterpret_cast<int32_t*>(epi_boxes + 4 * kWarpBoxBytes + 512);
  int32_t* s_end = s_off + kGemmMaxGroups;
  int32_t* s_prefix = s_end + kGemmMaxGroups;

  const int warp = threadIdx.x >> 5;
  const unsigned lane = lane_id();
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
      tc::mbar_init(tc::smem_u32(&tempty_bar[a]), 4);  // one arrive per epilogue warp
    }
    tc::mbar_init(tc::smem_u32(drain_bar), 1);
    *abort_flag = 0;
    tc::mbar_init_fence();
  }
  if (warp == 1) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), Cfg::kTmemCols);
    tc::tmem_relinquish();
  }
  if (args.tile_mode == kTilesSmallTail) {
    // The small-tail launch follows the pair launch of the same GEMM, whose
    // CTAs all passed their own wait (the inputs are complete) before this
    // launch could start; it works alongside the pair launch's last tiles and
    // waits for that launch only before it exits (end of the kernel).
    pdl_trigger();
  } else {
    pdl_enter();  // predecessors' outputs (group offsets, A rows) are visible from here
  }
  if (warp == 2)
    group_tile_prefix(args.group_off, G, args.m_cap, kGemmBM, n_blocks, args.tile_mode, s_off,
                      s_end, s_prefix, args.err);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const int total_tiles = s_prefix[G];
  const tc::WaitCtl wctl{abort_flag, args.err, args.wait_limit_ns};

  // tile -> (group, m block, n block)
  auto locate = [&](int tile, int& g, int& row0, int& rows, int& n0) {
    int lo = 0, hi = G;  // largest g with s_prefix[g] <= tile
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_prefix[mid] <= tile) lo = mid;
      else hi = mid;
    }
    g = lo;
    const int local = tile - s_prefix[g];
    const int gstart = s_off[g], gend = s_end[g];
    const int m_blocks = group_m_blocks(gend - gstart, kGemmBM, args.tile_mode);
    int nb, mb;
    if (args.raster) {
      mb = local / n_blocks;
      nb = local - mb * n_blocks;
    } else {
      nb = local / m_blocks;
      mb = local - nb * m_blocks;
    }
    row0 = group_first_row(gstart, gend - gstart, args.tile_mode) + mb * kGemmBM;
    rows = min(kGemmBM, gend - row0);
    n0 = nb * BN;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // The whole warp runs the loop: lane 0 waits, arms the stage and loads B;
    // in GATHER mode every lane then gathers 4 of the tile's 128 A rows.
    if (GATHER || lane == 0) {
      const uint64_t pol_a = tc::policy_from_code(args.l2_a);
      const uint64_t pol_b = tc::policy_from_code(args.l2_b);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_parity = 0;  // per stage: armed at least once, parity of the last arming
      bool skip_next = (args.debug & kDebugSkipFirstLoad) != 0;
      bool ok = true;
      bool bad_row = false;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        int g, row0, rows, n0;
        locate(tile, g, row0, rows, n0);
        int ri[4] = {0, 0, 0, 0};
        if (GATHER) {
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int i = (int)lane * 4 + r;
            if (i < rows) {
              const int v = __ldg(args.a_row_index + row0 + i);
              if (v >= 0 && v < args.a_rows) ri[r] = v;
              else bad_row = true;
            }
          }
        }
        for (int kb = 0; kb < k_blocks; ++kb) {
          bool go = true;
          if (lane == 0) go = tc::wait_bounded(tc::smem_u32(&empty_bar[stage]), phase ^ 1u, wctl);
          if (GATHER) go = __shfl_sync(0xffffffffu, go, 0) != 0;
          if (!go) {
            ok = false;
            break;
          }
          if (!skip_next) {
            const uint32_t fb = tc::smem_u32(&full_bar[stage]);
            uint8_t* sa = tiles + (size_t)stage * Cfg::kStageBytes;
            if (lane == 0) {
              tc::mbar_arrive_expect_tx(fb, Cfg::kStageBytes);
              if (!GATHER)
                tc::tma_load_2d(tc::smem_u32(sa), &tmap_a, fb, kb * Cfg::kBK, row0, pol_a);
              if (B_MN) {
                // strip map {column in strip, row, strip}: BN/64 strips in one load
                tc::tma_load_3d(tc::smem_u32(sa + Cfg::kABytes), &tmap_b, fb, 0,
                                g * args.K + kb * Cfg::kBK, n0 / 64, pol_b);
              } else {
                tc::tma_load_2d(tc::smem_u32(sa + Cfg::kABytes), &tmap_b, fb, kb * Cfg::kBK,
                                g * args.N + n0, pol_b);
              }
            }
            if (GATHER) {
              __syncwarp();
              tc::tma_gather4(tc::smem_u32(sa + lane * 512), &tmap_a, fb, kb * Cfg::kBK, ri[0],
                              ri[1], ri[2], ri[3], pol_a);
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
      if (GATHER && __any_sync(0xffffffffu, bad_row) && lane == 0) raise_error(args.err, kErrIndex);
      // Leave no TMA write in flight into this CTA's shared memory: wait for
      // the last arming of every stage (already complete on the normal path,
      // where the MMA issuer consumed it; maybe not if the CTA is unwinding).
      if (lane == 0)
        for (int s = 0; s < S; ++s)
          if ((armed >> s) & 1u)
            tc::wait_bounded(tc::smem_u32(&full_bar[s]), (armed_parity >> s) & 1u, wctl, false);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = tc::idesc_f32acc<TF32, 128, BN, false, B_MN>();
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        if (!tc::wait_bounded(tc::smem_u32(&tempty_bar[acc]), acc_phase ^ 1u, wctl)) break;
        tc::fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!tc::wait_bounded(tc::smem_u32(&full_bar[stage]), phase, wctl)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t sa = tc::smem_u32(tiles + (size_t)stage * Cfg::kStageBytes);
          const uint64_t adesc = tc::desc_sw128_kmajor(sa);
          const uint64_t bdesc = B_MN ? tc::desc_sw128_mnmajor(sa + Cfg::kABytes, 8192)
                                      : tc::desc_sw128_kmajor(sa + Cfg::kABytes);
#pragma unroll
          for (int kk = 0; kk < Cfg::kMmaPerStage; ++kk) {
            // K-major: +32 bytes along K inside the swizzled row = +2 in the
            // address field; MN-major: +16 K rows = two 1024-byte atoms = +128
            const uint64_t off = static_cast<uint64_t>(kk * 2);
            const uint64_t boff = B_MN ? static_cast<uint64_t>(kk * 128) : off;
            if (TF32)
              tc::mma_tf32(d_tmem, adesc + off, bdesc + boff, idesc, (kb | kk) != 0);
            else
              tc::mma_f16(d_tmem, adesc + off, bdesc + boff, idesc, (kb | kk) != 0);
          }
          tc::commit(tc::smem_u32(&empty_bar[stage]));  // frees the stage when these MMAs finish
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc::commit(tc::smem_u32(&tfull_bar[acc]));  // accumulator ready
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // drain: every MMA this thread issued has finished before TMEM is freed
      tc::commit(tc::smem_u32(drain_bar));
      tc::wait_bounded(tc::smem_u32(drain_bar), 0u, wctl, false);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int r_in_tile = quarter * 32 + (int)lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      int g, row0, rows, n0;
      if constexpr (EPI == kEpiSwiGLUBwd) {
        // this tile's saved rows (first tile only) and the next tile's, into L2
        for (int t = tile == (int)blockIdx.x ? tile : tile + (int)gridDim.x;
             t <= tile + (int)gridDim.x && t < total_tiles; t += gridDim.x) {
          locate(t, g, row0, rows, n0);
          prefetch_aux_row<BN, EPI>(args, r_in_tile < rows, (size_t)(row0 + r_in_tile), n0);
        }
      }
      locate(tile, g, row0, rows, n0);
      // lane 0 waits for the accumulator; the warp then proceeds converged
      bool ok = true;
      if (lane == 0) ok = tc::wait_bounded(tc::smem_u32(&tfull_bar[acc]), acc_phase, wctl);
      ok = __shfl_sync(0xffffffffu, ok, 0) != 0;
      if (!ok) break;
      __syncwarp();
      tc::fence_after_sync();
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * BN);
      const bool valid = r_in_tile < rows;
      const size_t grow = static_cast<size_t>(row0 + r_in_tile);
      epilogue_rows<BN, EPI, TOut>(taddr, valid, grow, n0, args, epi_boxes + quarter * kWarpBoxBytes,
                                   &tmap_out, &tmap_aux);
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(tc::smem_u32(&tempty_bar[acc]));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    // this warp's TMA stores have completed before the CTA exits
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
  // the small-tail launch completes only after the pair launch before it, so
  // that the next kernel's wait covers both
  if (args.tile_mode == kTilesSmallTail) pdl_wait();
}

}  // namespace moe
