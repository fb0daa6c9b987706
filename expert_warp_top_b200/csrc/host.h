// host.h -- host-side helpers shared by the library's translation units:
// error reporting, per-device state, tensor maps, launch helpers and the
// launchers of the tcgen05 GEMM kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <mutex>
#include <type_traits>
#include <utility>
#include <vector>

#include "../../include/moe_occult.h"
#include "ffn_gemm.cuh"
#include "ffn_gemm_pair.cuh"
#include "ffn_gemm_swap.cuh"
#include "wgrad_gemm.cuh"
#include "wgrad_pair.cuh"

namespace moe_host {

// Sets this thread's error message (moe_last_error) and returns code.
int fail(int code, const char* fmt, ...);
const char* last_message();

#define MOE_REQUIRE(cond, code, ...)                       \
  do {                                                     \
    if (!(cond)) return ::moe_host::fail(code, __VA_ARGS__); \
  } while (0)

#define MOE_CUDA(call)                                                                     \
  do {                                                                                     \
    cudaError_t e_ = (call);                                                               \
    if (e_ != cudaSuccess)                                                                 \
      return ::moe_host::fail(MOE_ERR_CUDA, "%s: %s (%s:%d)", #call, cudaGetErrorString(e_), \
                              __FILE__, __LINE__);                                         \
  } while (0)

#define MOE_LAUNCHED(what)                                                                 \
  do {                                                                                     \
    cudaError_t e_ = cudaGetLastError();                                                   \
    if (e_ != cudaSuccess)                                                                 \
      return ::moe_host::fail(MOE_ERR_CUDA, "launch of %s failed: %s", what,               \
                              cudaGetErrorString(e_));                                     \
  } while (0)

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
  unsigned* err_flag = nullptr;  // the device error flag the kernels raise
  std::mutex mu;
  std::vector<const void*> smem_raised;                   // kernels with the smem limit raised
  std::vector<std::pair<const void*, int>> pair_clusters;  // CTA-pair kernels: clusters that fit
};

// The current device's state (checks that it is an sm_100 part).
int device_info(DeviceInfo** out);

// Raises kern's dynamic shared-memory limit to `bytes`, once per device.
int ensure_smem(DeviceInfo* di, const void* kern, size_t bytes);

// Test-only knobs, set by moe_set_debug.
extern int g_debug_flags;
extern double g_wait_limit_ms;
inline uint64_t wait_limit_ns() { return static_cast<uint64_t>(g_wait_limit_ms * 1.0e6); }
constexpr int kDebugForceSingle = 2;  // GEMMs on single CTAs
constexpr int kDebugForcePair = 4;    // GEMMs on CTA pairs only where the shape allows
constexpr int kDebugForceHybrid = 8;  // pair tiles plus single-CTA small tails
constexpr int kDebugBulkMovers = 16;  // dispatch and combine through TMA bulk copies
// Tuning knobs of the expert GEMMs: with kDebugGemmPolicy set, bits 20..21, 22..23
// and 24..25 of the flags give the L2 policy of the A loads, the weight loads and
// the output stores (0 evict_normal, 1 evict_last, 2 evict_first; output 0 = no
// hint), bit 26 the N-fastest tile order and bit 27 the L2 prefetch of the next
// tile's first-use panels.  (They sit above every switch below.)
constexpr int kDebugGemmPolicy = 32;
constexpr int kDebugForceSwap = 64;   // inference GEMMs on the swapped-operand kernel
constexpr int kDebugNoSwap = 128;     // never on the swapped-operand kernel
constexpr int kDebugWideTiles = 256;  // inference GEMMs on 256 x 512 pair tiles where N allows
constexpr int kDebugNoWideTiles = 512;
constexpr int kDebugKch1 = 65536;  // pair GEMMs with one K chunk per stage only
constexpr int kDebugWgradShortStages = 131072;  // weight-gradient pairs on 64-row stages only

// 2-D row-major [rows, cols] tensor, box [box_rows, box_cols], 128-byte swizzle.
int encode_2d(CUtensorMap* map, const void* base, int dtype, uint64_t cols, uint64_t rows,
              uint32_t box_cols, uint32_t box_rows);

// The same [rows, cols] tensor seen as 64-column strips: a 3-D map with dims
// {64, rows, cols / 64} and strides {row pitch, 128 bytes}, box
// {64, box_rows, box_strips}, 128-byte swizzle.  One load brings box_strips
// strips of box_rows rows, strip after strip (each box_rows x 128 bytes): the
// layout of an MN-major operand tile, in one instruction instead of one per
// strip.  bf16 only; cols % 64 == 0.
int encode_strips(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                  uint32_t box_rows, uint32_t box_strips);

int check_common(int T, int E, int k, int R);
int check_dtype(int dtype);
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int esize(int dtype) { return dtype == MOE_BF16 ? 2 : 4; }
inline int pick_bn(int N) { return N % 256 == 0 ? 256 : (N % 128 == 0 ? 128 : 64); }
inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Every kernel is launched with programmatic stream serialization, so the next
// kernel on the stream can be scheduled while this one finishes; each kernel
// starts with griddepcontrol.wait (moe::pdl_enter) before it touches memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                     Args&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ---- the grouped GEMM (ffn_gemm.cuh / ffn_gemm_pair.cuh) --------------------
// Arguments of the training epilogues (kEpiSwiGLUSave, kEpiSwiGLUBwd).
struct GemmExtra {
  const void* aux_in = nullptr;
  void* aux_out = nullptr;
  int ld_aux = 0;
  float* partial = nullptr;
  int n_part = 0;
  int tile_mode = 0;  // moe::kTilesAll / kTilesPairNoSmallTail / kTilesSmallTail
};

inline moe::GemmArgs gemm_args(const DeviceInfo* di, const int32_t* group_off,
                               const int32_t* a_row_index, int a_rows, int G, int N, int K,
                               int m_cap, const float* row_scale, void* out, int ldo,
                               const GemmExtra& ex) {
  moe::GemmArgs a{group_off, a_row_index, a_rows, G, N, K, m_cap, row_scale, out, ldo,
                  di->err_flag, wait_limit_ns(), g_debug_flags};
  a.aux_in = ex.aux_in;
  a.aux_out = ex.aux_out;
  a.ld_aux = ex.ld_aux;
  a.partial = ex.partial;
  a.n_part = ex.n_part;
  a.tile_mode = ex.tile_mode;
  if (g_debug_flags & kDebugGemmPolicy) {
    a.l2_a = (g_debug_flags >> 20) & 3;
    a.l2_b = (g_debug_flags >> 22) & 3;
    a.l2_out = (g_debug_flags >> 24) & 3;
    a.raster = (g_debug_flags >> 26) & 1;
    a.l2_prefetch = (g_debug_flags >> 27) & 1;
  }
  return a;
}

// B's tensor map: K-major [G*N, K] with box [box_n rows, 64 cols], or
// MN-major [G*K, N] as 64-column strips with box [64 K rows, box_n / 64 strips].
template <bool B_MN>
int encode_b(CUtensorMap* tb, const void* b, int dtype, int G, int N, int K, int bk,
             uint32_t box_n) {
  if (B_MN) return encode_strips(tb, b, (uint64_t)N, (uint64_t)G * K, bk, box_n / 64);
  return encode_2d(tb, b, dtype, (uint64_t)K, (uint64_t)G * N, bk, box_n);
}

// The GEMM output [m_cap, ldo] for the epilogue's TMA stores: boxes of 32 rows
// x 128 bytes, 128-byte swizzle.
inline int encode_out(CUtensorMap* to, const void* out, int dtype, int m_cap, int ldo) {
  return encode_2d(to, out, dtype, (uint64_t)ldo, (uint64_t)(m_cap > 0 ? m_cap : 1),
                   dtype == MOE_BF16 ? 64 : 32, 32);
}

// The training epilogues' second output, aux_out [m_cap, ld_aux] (the
// pre-activations or their gradient), for their TMA stores; the other
// epilogues never read this map and get a copy of the output's.
template <int EPI>
int encode_aux(CUtensorMap* tx, const CUtensorMap& to, const GemmExtra& ex, int dtype, int m_cap) {
  constexpr bool kTraining = EPI == moe::kEpiSwiGLUSave || EPI == moe::kEpiSwiGLUBwd;
  MOE_REQUIRE(!kTraining || (ex.aux_out && ex.ld_aux > 0), MOE_ERR_INVALID_ARG,
              "the training epilogues need their second output");
  if (!kTraining) {
    *tx = to;
    return MOE_OK;
  }
  return encode_out(tx, ex.aux_out, dtype, m_cap, ex.ld_aux);
}

// A is [a_rows, K]; with a_row_index the m_cap rows fed to the GEMM are
// gathered from it (row p = a[a_row_index[p]]), else they are a's first m_cap.
template <int BN, int EPI, bool TF32, bool GATHER, bool B_MN>
int launch_gemm(DeviceInfo* di, const void* a, int a_rows, const int32_t* a_row_index, int m_cap,
                int K, const void* b, int G, int N, const int32_t* group_off,
                const float* row_scale, void* out, int ldo, const GemmExtra& ex,
                cudaStream_t st) {
  using Cfg = moe::GemmCfg<BN, TF32, EPI>;
  const int dtype = TF32 ? MOE_F32 : MOE_BF16;
  CUtensorMap ta, tb;
  int rc = encode_2d(&ta, a, dtype, (uint64_t)K, (uint64_t)a_rows, Cfg::kBK,
                     GATHER ? 1u : (uint32_t)moe::kGemmBM);
  if (rc) return rc;
  if ((rc = encode_b<B_MN>(&tb, b, dtype, G, N, K, Cfg::kBK, BN))) return rc;
  CUtensorMap to, tx;
  if ((rc = encode_out(&to, out, dtype, m_cap, ldo))) return rc;
  if ((rc = encode_aux<EPI>(&tx, to, ex, dtype, m_cap))) return rc;
  auto kern = moe::ffn_gemm_kernel<BN, EPI, TF32, GATHER, B_MN>;
  if ((rc = ensure_smem(di, reinterpret_cast<const void*>(kern), Cfg::kSmemBytes))) return rc;
  const long long ub = ((long long)m_cap / moe::kGemmBM + G) * (N / BN);
  const int grid = (int)(ub < di->num_sms ? (ub < 1 ? 1 : ub) : di->num_sms);
  const moe::GemmArgs args =
      gemm_args(di, group_off, a_row_index, a_rows, G, N, K, m_cap, row_scale, out, ldo, ex);
  MOE_CUDA(launch_k(kern, dim3(grid), dim3(moe::kGemmThreads), Cfg::kSmemBytes, st, ta, tb, to,
                    tx, args));
  MOE_LAUNCHED("ffn_gemm_kernel");
  return MOE_OK;
}

template <int EPI, bool TF32, bool GATHER, bool B_MN>
int launch_gemm_bn(DeviceInfo* di, int bn, const void* a, int a_rows,
                   const int32_t* a_row_index, int m_cap, int K, const void* b, int G, int N,
                   const int32_t* group_off, const float* row_scale, void* out, int ldo,
                   const GemmExtra& ex, cudaStream_t st) {
  if (bn == 256)
    return launch_gemm<256, EPI, TF32, GATHER, B_MN>(di, a, a_rows, a_row_index, m_cap, K, b, G,
                                                     N, group_off, row_scale, out, ldo, ex, st);
  if (bn == 128)
    return launch_gemm<128, EPI, TF32, GATHER, B_MN>(di, a, a_rows, a_row_index, m_cap, K, b, G,
                                                     N, group_off, row_scale, out, ldo, ex, st);
  return launch_gemm<64, EPI, TF32, GATHER, B_MN>(di, a, a_rows, a_row_index, m_cap, K, b, G, N,
                                                  group_off, row_scale, out, ldo, ex, st);
}

// The same GEMM on CTA pairs (cluster of 2, M = 256 tiles).  Needs BN/2 >= 64.
// KCH = 2: two 128-byte K chunks per stage through 3-D strip maps (K % 128 == 0).
template <int BN, int EPI, bool TF32, bool B_MN, int KCH = 1>
int launch_gemm_pair(DeviceInfo* di, const void* a, int a_rows, int m_cap, int K, const void* b,
                     int G, int N, const int32_t* group_off, const float* row_scale, void* out,
                     int ldo, const GemmExtra& ex, cudaStream_t st) {
  using Cfg = moe::PairCfg<BN, TF32, EPI, KCH>;
  const int dtype = TF32 ? MOE_F32 : MOE_BF16;
  CUtensorMap ta, tb;
  int rc;
  if (KCH == 2) {
    // {element in chunk, row, chunk}: boxes of 128 rows (A) or BN/2 rows (B) x 2 chunks
    if ((rc = encode_strips(&ta, a, (uint64_t)K, (uint64_t)a_rows, 128, 2))) return rc;
    if (B_MN) {
      if ((rc = encode_b<true>(&tb, b, dtype, G, N, K, Cfg::kBK, BN / 2))) return rc;
    } else if ((rc = encode_strips(&tb, b, (uint64_t)K, (uint64_t)G * N, BN / 2, 2))) {
      return rc;
    }
  } else {
    if ((rc = encode_2d(&ta, a, dtype, (uint64_t)K, (uint64_t)a_rows, Cfg::kBK, 128))) return rc;
    // each CTA loads its BN/2 weight rows in one box, or (BN = 512) in two of 128
    if ((rc = encode_b<B_MN>(&tb, b, dtype, G, N, K, Cfg::kBK, BN > 256 ? 128 : BN / 2)))
      return rc;
  }
  CUtensorMap to, tx;
  if ((rc = encode_out(&to, out, dtype, m_cap, ldo))) return rc;
  if ((rc = encode_aux<EPI>(&tx, to, ex, dtype, m_cap))) return rc;
  auto kern = moe::ffn_gemm_pair_kernel<BN, EPI, TF32, B_MN, KCH>;
  const void* key = reinterpret_cast<const void*>(kern);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(moe::kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = Cfg::kSmemBytes;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;  // the occupancy query below sees the cluster shape only
  if ((rc = ensure_smem(di, key, Cfg::kSmemBytes))) return rc;
  int max_clusters = 0;
  {
    std::lock_guard<std::mutex> lk(di->mu);
    for (auto& pc : di->pair_clusters)
      if (pc.first == key) max_clusters = pc.second;
  }
  if (max_clusters == 0) {
    cfg.gridDim = dim3(2 * (di->num_sms / 2), 1, 1);
    MOE_CUDA(cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg));
    MOE_REQUIRE(max_clusters >= 1, MOE_ERR_UNSUPPORTED, "no CTA pair fits on this device");
    std::lock_guard<std::mutex> lk(di->mu);
    di->pair_clusters.emplace_back(key, max_clusters);
  }
  const long long ub = ((long long)m_cap / moe::kPairBM + G) * (N / BN);
  const long long pairs = ub < max_clusters ? (ub < 1 ? 1 : ub) : max_clusters;
  cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
  cfg.numAttrs = 2;
  moe::GemmArgs args =
      gemm_args(di, group_off, nullptr, a_rows, G, N, K, m_cap, row_scale, out, ldo, ex);
  args.a_ptr = a;
  args.b_ptr = b;
  MOE_CUDA(cudaLaunchKernelEx(&cfg, kern, ta, tb, to, tx, args));
  return MOE_OK;
}

// The same GEMM with the operands swapped (ffn_gemm_swap.cuh): CTA pairs on
// 256 weight rows x up to 256 of a group's rows.  bf16, K-major weights, the
// two inference epilogues; N % 256 == 0, G <= kSwapMaxGroups.
template <int EPI>
int launch_gemm_swap(DeviceInfo* di, const void* a, int a_rows, int m_cap, int K, const void* b,
                     int G, int N, const int32_t* group_off, const float* row_scale, void* out,
                     int ldo, cudaStream_t st) {
  using Cfg = moe::SwapCfg;
  moe::SwapMaps rows;
  int rc;
  for (int i = 0; i < moe::kSwapMaps; ++i)
    if ((rc = encode_2d(&rows.rows[i], a, MOE_BF16, (uint64_t)K, (uint64_t)a_rows, Cfg::kBK,
                        8u << i)))
      return rc;
  CUtensorMap tw, to;
  if ((rc = encode_2d(&tw, b, MOE_BF16, (uint64_t)K, (uint64_t)G * N, Cfg::kBK, 128))) return rc;
  if ((rc = encode_out(&to, out, MOE_BF16, m_cap, ldo))) return rc;
  auto kern = moe::ffn_gemm_swap_kernel<EPI>;
  const void* key = reinterpret_cast<const void*>(kern);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(moe::kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = Cfg::kSmemBytes;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;  // the occupancy query below sees the cluster shape only
  if ((rc = ensure_smem(di, key, Cfg::kSmemBytes))) return rc;
  int max_clusters = 0;
  {
    std::lock_guard<std::mutex> lk(di->mu);
    for (auto& pc : di->pair_clusters)
      if (pc.first == key) max_clusters = pc.second;
  }
  if (max_clusters == 0) {
    cfg.gridDim = dim3(2 * (di->num_sms / 2), 1, 1);
    MOE_CUDA(cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg));
    MOE_REQUIRE(max_clusters >= 1, MOE_ERR_UNSUPPORTED, "no CTA pair fits on this device");
    std::lock_guard<std::mutex> lk(di->mu);
    di->pair_clusters.emplace_back(key, max_clusters);
  }
  const long long ub = ((long long)m_cap / moe::kSwapMaxRows + G) * (N / moe::kSwapBM);
  const long long pairs = ub < max_clusters ? (ub < 1 ? 1 : ub) : max_clusters;
  cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
  cfg.numAttrs = 2;
  const moe::GemmArgs args =
      gemm_args(di, group_off, nullptr, a_rows, G, N, K, m_cap, row_scale, out, ldo, GemmExtra{});
  MOE_CUDA(cudaLaunchKernelEx(&cfg, kern, rows, tw, to, args));
  return MOE_OK;
}

// Groups this short (rows on average) go to the swapped-operand kernel.  It
// measured slower than the row-major pair kernel on every workload (the
// OLMoE-shaped layer's GEMMs 0.43 against 0.41 ms, DSV2-Lite-shaped 1.52 against
// 1.43 ms): its tail tiles still stream the full weight tile into each SM, and
// its epilogue turns the accumulators around through shared memory.  So it
// runs only when asked for (kDebugForceSwap), tested.
#ifndef MOE_SWAP_MAX_AVG_ROWS
#define MOE_SWAP_MAX_AVG_ROWS 0
#endif

// Groups at least this tall (rows on average) take the 256 x 512 pair tiles
// when N allows (0: only when asked for, kDebugWideTiles).  Measured against the
// 256 x 256 tiles on one B200 (GEMM-only replays, three rounds): level on the
// correlated prefill layer (8.12-8.14 against 8.07-8.22 ms) and the
// Mixtral-shaped one (4.76 against 4.79 ms), slower on the DSV2-Lite-shaped
// (1.52 against 1.45 ms) and OLMoE-shaped (0.463 against 0.414 ms) layers.  They
// ran ~100 MHz higher under the same power cap: fewer bytes into each SM per
// FLOP, but the accumulator is not double-buffered, so every tile's epilogue
// stalls the tensor pipe.
#ifndef MOE_WIDE_MIN_AVG_ROWS
#define MOE_WIDE_MIN_AVG_ROWS 0
#endif

// GEMM over the groups, on CTA pairs when the groups are tall enough to fill
// 256-row tiles (and the rows are read in place), else on single CTAs.  In
// hybrid mode a group's tail of at most 128 rows goes to a second,
// single-CTA launch (128-row tiles), which halves that tail's MMA work.
#ifndef MOE_PAIR_MIN_ROWS
#define MOE_PAIR_MIN_ROWS 192
#endif
#ifndef MOE_PAIR_KCH2
#define MOE_PAIR_KCH2 1
#endif
template <int EPI, bool TF32, bool B_MN = false>
int launch_gemm_auto(DeviceInfo* di, const void* a, int a_rows, const int32_t* a_row_index,
                     int m_cap, int K, const void* b, int G, int N, const int32_t* group_off,
                     const float* row_scale, void* out, int ldo, cudaStream_t st,
                     const GemmExtra& ex = GemmExtra{}) {
  const bool tall = (long long)m_cap >= (long long)MOE_PAIR_MIN_ROWS * G;
  const bool pair_ok = !a_row_index && N % 128 == 0;
  if constexpr (!TF32 && !B_MN && (EPI == moe::kEpiSwiGLU || EPI == moe::kEpiScale)) {
    const bool swap_ok = !a_row_index && N % moe::kSwapBM == 0 && G <= moe::kSwapMaxGroups &&
                         K % 64 == 0 && !(g_debug_flags & kDebugNoSwap);
    const bool short_groups = (long long)m_cap < (long long)MOE_SWAP_MAX_AVG_ROWS * G;
    if (swap_ok && ((g_debug_flags & kDebugForceSwap) || short_groups))
      return launch_gemm_swap<EPI>(di, a, a_rows, m_cap, K, b, G, N, group_off, row_scale, out,
                                   ldo, st);
  }
  bool pair = pair_ok && tall;
  // Hybrid tiling (a group's tail of <= 128 rows on single-CTA tiles, in a
  // second launch) cuts the OLMoE-shaped layer's padded MMA rows from 20% to
  // 11% but measured no faster (482-485 vs 490 us for both GEMMs): it stays
  // opt-in, tested, behind kDebugForceHybrid.
  bool hybrid = false;
  if (g_debug_flags & kDebugForceSingle) pair = false;
  if ((g_debug_flags & kDebugForcePair) && pair_ok) pair = true;
  if ((g_debug_flags & kDebugForceHybrid) && pair_ok) {
    pair = true;
    hybrid = true;
  }
  if constexpr (!TF32 && !B_MN && (EPI == moe::kEpiSwiGLU || EPI == moe::kEpiScale)) {
    // 256 x 512 pair tiles, one accumulator: half the row-operand bytes into each
    // SM per FLOP of the 256 x 256 tiles, for tall groups
    const bool wide_tall = MOE_WIDE_MIN_AVG_ROWS > 0 &&
                           (long long)m_cap >= (long long)MOE_WIDE_MIN_AVG_ROWS * G;
    if (pair && !hybrid && N % 512 == 0 && !(g_debug_flags & kDebugNoWideTiles) &&
        ((g_debug_flags & kDebugWideTiles) || wide_tall))
      return launch_gemm_pair<512, EPI, TF32, B_MN>(di, a, a_rows, m_cap, K, b, G, N, group_off,
                                                    row_scale, out, ldo, ex, st);
  }
  // two K chunks per stage (3-D strip loads) where K allows and the ring keeps
  // three stages: the epilogues with three staging boxes per warp would be left
  // with two, which measured slower than five single-chunk stages
  if constexpr (!TF32 && moe::PairCfg<256, TF32, EPI, 2>::kStages >= 3) {
    if (pair && !hybrid && MOE_PAIR_KCH2 && K % 128 == 0 && !(g_debug_flags & kDebugKch1)) {
      GemmExtra exp = ex;
      exp.tile_mode = moe::kTilesAll;
      return N % 256 == 0
                 ? launch_gemm_pair<256, EPI, TF32, B_MN, 2>(di, a, a_rows, m_cap, K, b, G, N,
                                                             group_off, row_scale, out, ldo, exp,
                                                             st)
                 : launch_gemm_pair<128, EPI, TF32, B_MN, 2>(di, a, a_rows, m_cap, K, b, G, N,
                                                             group_off, row_scale, out, ldo, exp,
                                                             st);
    }
  }
  if (pair) {
    GemmExtra exp = ex;
    exp.tile_mode = hybrid ? moe::kTilesPairNoSmallTail : moe::kTilesAll;
    int rc = N % 256 == 0
                 ? launch_gemm_pair<256, EPI, TF32, B_MN>(di, a, a_rows, m_cap, K, b, G, N,
                                                          group_off, row_scale, out, ldo, exp, st)
                 : launch_gemm_pair<128, EPI, TF32, B_MN>(di, a, a_rows, m_cap, K, b, G, N,
                                                          group_off, row_scale, out, ldo, exp, st);
    if (rc || !hybrid) return rc;
    GemmExtra ext = ex;
    ext.tile_mode = moe::kTilesSmallTail;
    return launch_gemm_bn<EPI, TF32, false, B_MN>(di, pick_bn(N), a, a_rows, nullptr, m_cap, K, b,
                                                  G, N, group_off, row_scale, out, ldo, ext, st);
  }
  const int bn = pick_bn(N);
  if constexpr (!B_MN) {
    if (a_row_index)
      return launch_gemm_bn<EPI, TF32, true, false>(di, bn, a, a_rows, a_row_index, m_cap, K, b,
                                                    G, N, group_off, row_scale, out, ldo, ex, st);
  }
  return launch_gemm_bn<EPI, TF32, false, B_MN>(di, bn, a, a_rows, nullptr, m_cap, K, b, G, N,
                                                group_off, row_scale, out, ldo, ex, st);
}

// ---- the weight-gradient GEMM (wgrad_gemm.cuh) -------------------------------
// out[g] (+)= A_g^T B_g with A [rows, M], B [rows, N] bf16 row-major and the
// groups' rows given by group_off.  M % 128 == 0, N % 64 == 0.
template <int BN, typename TOut>
int launch_wgrad_bn(DeviceInfo* di, const void* a, const void* b, int rows, int M, int N,
                    const int32_t* group_off, int G, void* out, int accumulate, cudaStream_t st) {
  using Cfg = moe::WgradCfg<BN>;
  CUtensorMap ta, tb;
  int rc = encode_strips(&ta, a, (uint64_t)M, (uint64_t)rows, 64, 2);
  if (rc) return rc;
  if ((rc = encode_strips(&tb, b, (uint64_t)N, (uint64_t)rows, 64, BN / 64))) return rc;
  // the output [G*M, N]: boxes of 32 rows x 128 bytes for the epilogue's TMA stores
  constexpr bool kF32 = std::is_same<TOut, float>::value;
  CUtensorMap to;
  if ((rc = encode_2d(&to, out, kF32 ? MOE_F32 : MOE_BF16, (uint64_t)N, (uint64_t)G * M,
                      kF32 ? 32 : 64, 32)))
    return rc;
  auto kern = moe::wgrad_gemm_kernel<BN, TOut>;
  if ((rc = ensure_smem(di, reinterpret_cast<const void*>(kern), Cfg::kSmemBytes))) return rc;
  const long long tiles = (long long)G * (M / 128) * (N / BN);
  const int grid = (int)(tiles < di->num_sms ? (tiles < 1 ? 1 : tiles) : di->num_sms);
  moe::WgradArgs args{group_off, G, M, N, rows, out, accumulate, di->err_flag, wait_limit_ns(),
                      g_debug_flags};
  MOE_CUDA(launch_k(kern, dim3(grid), dim3(moe::kWgradThreads), Cfg::kSmemBytes, st, ta, tb, to,
                    args));
  MOE_LAUNCHED("wgrad_gemm_kernel");
  return MOE_OK;
}

// The same on CTA pairs: 256 x BN output tiles (M % 256 == 0, N % BN == 0),
// stages of BK contracted rows.
template <int BN, typename TOut, int BK = 64>
int launch_wgrad_pair(DeviceInfo* di, const void* a, const void* b, int rows, int M, int N,
                      const int32_t* group_off, int G, void* out, int accumulate,
                      cudaStream_t st) {
  using Cfg = moe::WgradPairCfg<BN, BK>;
  CUtensorMap ta, tb, to;
  int rc = encode_strips(&ta, a, (uint64_t)M, (uint64_t)rows, Cfg::kBK, 2);
  if (rc) return rc;
  if ((rc = encode_strips(&tb, b, (uint64_t)N, (uint64_t)rows, Cfg::kBK, BN / 128))) return rc;
  constexpr bool kF32 = std::is_same<TOut, float>::value;
  if ((rc = encode_2d(&to, out, kF32 ? MOE_F32 : MOE_BF16, (uint64_t)N, (uint64_t)G * M,
                      kF32 ? 32 : 64, 32)))
    return rc;
  auto kern = moe::wgrad_pair_kernel<BN, TOut, BK>;
  const void* key = reinterpret_cast<const void*>(kern);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(moe::kWgradThreads, 1, 1);
  cfg.dynamicSmemBytes = Cfg::kSmemBytes;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;  // the occupancy query below sees the cluster shape only
  if ((rc = ensure_smem(di, key, Cfg::kSmemBytes))) return rc;
  int max_clusters = 0;
  {
    std::lock_guard<std::mutex> lk(di->mu);
    for (auto& pc : di->pair_clusters)
      if (pc.first == key) max_clusters = pc.second;
  }
  if (max_clusters == 0) {
    cfg.gridDim = dim3(2 * (di->num_sms / 2), 1, 1);
    MOE_CUDA(cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg));
    MOE_REQUIRE(max_clusters >= 1, MOE_ERR_UNSUPPORTED, "no CTA pair fits on this device");
    std::lock_guard<std::mutex> lk(di->mu);
    di->pair_clusters.emplace_back(key, max_clusters);
  }
  const long long tiles = (long long)G * (M / 256) * (N / BN);
  const long long pairs = tiles < max_clusters ? (tiles < 1 ? 1 : tiles) : max_clusters;
  cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
  cfg.numAttrs = 2;
  moe::WgradArgs args{group_off, G, M, N, rows, out, accumulate, di->err_flag, wait_limit_ns(),
                      g_debug_flags};
  MOE_CUDA(cudaLaunchKernelEx(&cfg, kern, ta, tb, to, args));
  return MOE_OK;
}

template <typename TOut>
int launch_wgrad(DeviceInfo* di, const void* a, const void* b, int rows, int M, int N,
                 const int32_t* group_off, int G, void* out, int accumulate, cudaStream_t st) {
  // The CTA-pair kernel moves a third less operand traffic per FLOP into each
  // SM, so its six stages cover more of the load latency than the single-CTA
  // kernel's four.  Alone on one B200 (fp32 out, ragged groups) it measured
  // 1175 against 1250 us on the DSV2-Lite-shaped gate/up gradient and 219
  // against 225 us on the OLMoE-shaped down gradient, so it is the default
  // where the shape allows; kDebugForceSingle keeps the single-CTA kernel.
  const bool pair = M % 256 == 0 && N % 128 == 0 && !(g_debug_flags & kDebugForceSingle);
  if (pair) {
    // Stages of 128 contracted rows (half the TMA operations) for groups that
    // average 1024 rows or more: 4-8% faster there on one B200 (DSV2-Lite-shaped
    // gate/up gradient 1048 against 1089 us), 1-2% slower on 512-row groups,
    // where a group's last block loads more rows past its end.
    const bool long_groups = (long long)rows >= 1024LL * (G > 0 ? G : 1) &&
                             !(g_debug_flags & kDebugWgradShortStages);
    if (long_groups) {
      if (N % 256 == 0)
        return launch_wgrad_pair<256, TOut, 128>(di, a, b, rows, M, N, group_off, G, out,
                                                 accumulate, st);
      return launch_wgrad_pair<128, TOut, 128>(di, a, b, rows, M, N, group_off, G, out,
                                               accumulate, st);
    }
    if (N % 256 == 0)
      return launch_wgrad_pair<256, TOut>(di, a, b, rows, M, N, group_off, G, out, accumulate, st);
    return launch_wgrad_pair<128, TOut>(di, a, b, rows, M, N, group_off, G, out, accumulate, st);
  }
  const int bn = pick_bn(N);
  if (bn == 256)
    return launch_wgrad_bn<256, TOut>(di, a, b, rows, M, N, group_off, G, out, accumulate, st);
  if (bn == 128)
    return launch_wgrad_bn<128, TOut>(di, a, b, rows, M, N, group_off, G, out, accumulate, st);
  return launch_wgrad_bn<64, TOut>(di, a, b, rows, M, N, group_off, G, out, accumulate, st);
}

}  // namespace moe_host
