// api.cu -- the C ABI (include/moe_occult.h): argument checks, launch
// configuration and the tensor-map set-up of every kernel of the layer.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <type_traits>
#include <vector>

#include "../../include/moe_occult.h"
#include "brim.cuh"
#include "dispatch.cuh"
#include "ep.cuh"
#include "host.h"
#include "route.cuh"
#include "route_brim.cuh"
#include "shuffle.cuh"

// The device error flag the kernels raise (bits moe::kErrIndex, kErrTimeout).
__device__ unsigned g_moe_err_flag;
// moe_get_device_status's reading of the flag, taken and cleared in one step.
__device__ unsigned g_moe_err_snapshot;

__global__ void take_error_flag_kernel() {
  moe::pdl_enter();
  g_moe_err_snapshot = atomicExch(&g_moe_err_flag, 0u);
}

// Fixed scratch of moe_brim_build_noalloc (1 MiB, held by every GPU that loads
// this library until the process exits).
constexpr size_t kNoAllocScratchInts = size_t(1) << 18;
static __device__ __align__(256) int32_t g_brim_noalloc_scratch[kNoAllocScratchInts];

namespace moe_host {

namespace {
thread_local char g_msg[512];
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;
}  // namespace
std::mutex g_status_mu;

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof g_msg, fmt, ap);
  va_end(ap);
  return code;
}

const char* last_message() { return g_msg; }

int device_info(DeviceInfo** out) {
  int dev = 0;
  MOE_CUDA(cudaGetDevice(&dev));
  MOE_REQUIRE(dev >= 0 && dev < kMaxDevices, MOE_ERR_UNSUPPORTED, "device index %d too large", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& di = g_dev[dev];
  if (!di.ready) {
    MOE_CUDA(cudaDeviceGetAttribute(&di.num_sms, cudaDevAttrMultiProcessorCount, dev));
    int major = 0, minor = 0;
    MOE_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
    MOE_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
    MOE_REQUIRE(major == 10 && minor == 0, MOE_ERR_UNSUPPORTED,
                "this library is built for sm_100a (B200); device %d is sm_%d%d", dev, major,
                minor);
    void* p = nullptr;
    MOE_CUDA(cudaGetSymbolAddress(&p, g_moe_err_flag));
    di.err_flag = static_cast<unsigned*>(p);
    di.ready = true;
  }
  *out = &di;
  return MOE_OK;
}

int ensure_smem(DeviceInfo* di, const void* kern, size_t bytes) {
  std::lock_guard<std::mutex> lk(di->mu);
  for (const void* k : di->smem_raised)
    if (k == kern) return MOE_OK;
  MOE_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes));
  di->smem_raised.push_back(kern);
  return MOE_OK;
}

int g_debug_flags = 0;
double g_wait_limit_ms = 4000.0;

namespace {
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

int get_encode_fn(EncodeTiledFn* fn) {
  static EncodeTiledFn cached = nullptr;
  static std::mutex mu;
  std::lock_guard<std::mutex> lk(mu);
  if (!cached) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    MOE_CUDA(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q));
    MOE_REQUIRE(q == cudaDriverEntryPointSuccess && p, MOE_ERR_CUDA,
                "cuTensorMapEncodeTiled is not available from the driver");
    cached = reinterpret_cast<EncodeTiledFn>(p);
  }
  *fn = cached;
  return MOE_OK;
}
}  // namespace

int encode_2d(CUtensorMap* map, const void* base, int dtype, uint64_t cols, uint64_t rows,
              uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn fn = nullptr;
  int rc = get_encode_fn(&fn);
  if (rc) return rc;
  const int esz = dtype == MOE_BF16 ? 2 : 4;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * (cuuint64_t)esz};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dtype == MOE_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                  2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  MOE_REQUIRE(r == CUDA_SUCCESS, MOE_ERR_CUDA,
              "cuTensorMapEncodeTiled failed (%d) for a [%llu x %llu] tensor", (int)r,
              (unsigned long long)rows, (unsigned long long)cols);
  return MOE_OK;
}

int encode_strips(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                  uint32_t box_rows, uint32_t box_strips) {
  EncodeTiledFn fn = nullptr;
  int rc = get_encode_fn(&fn);
  if (rc) return rc;
  cuuint64_t dims[3] = {64, rows, cols / 64};
  cuuint64_t strides[2] = {cols * 2, 128};
  cuuint32_t box[3] = {64, box_rows, box_strips};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  MOE_REQUIRE(r == CUDA_SUCCESS, MOE_ERR_CUDA,
              "cuTensorMapEncodeTiled failed (%d) for a [%llu x %llu] strip tensor", (int)r,
              (unsigned long long)rows, (unsigned long long)cols);
  return MOE_OK;
}

int check_common(int T, int E, int k, int R) {
  MOE_REQUIRE(T >= 0, MOE_ERR_INVALID_ARG, "T must be >= 0 (got %d)", T);
  MOE_REQUIRE(E >= 1 && E <= moe::kMaxE, MOE_ERR_UNSUPPORTED, "E must be in [1, 256] (got %d)", E);
  MOE_REQUIRE(k >= 1 && k <= E && k <= moe::kMaxK, MOE_ERR_UNSUPPORTED,
              "k must be in [1, min(E, 16)] (got k=%d, E=%d)", k, E);
  MOE_REQUIRE(R >= 1 && R <= E && E % R == 0, MOE_ERR_UNSUPPORTED,
              "R must divide E (got E=%d, R=%d)", E, R);
  return MOE_OK;
}

int check_dtype(int dtype) {
  MOE_REQUIRE(dtype == MOE_BF16 || dtype == MOE_F32, MOE_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  return MOE_OK;
}

}  // namespace moe_host

using namespace moe_host;

namespace {

// Device address of g_brim_noalloc_scratch on the current device.  The
// array's name in host code is only a host-side stand-in, so the address is
// looked up with cudaGetSymbolAddress, once per device, with that device
// current, and cached.
int32_t* g_noalloc_ptr[kMaxDevices];
std::mutex g_noalloc_mu;

int noalloc_scratch(int32_t** out) {
  int dev = 0;
  MOE_CUDA(cudaGetDevice(&dev));
  MOE_REQUIRE(dev >= 0 && dev < kMaxDevices, MOE_ERR_UNSUPPORTED, "device index %d too large", dev);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    MOE_CUDA(cudaGetSymbolAddress(&p, g_brim_noalloc_scratch));
    MOE_REQUIRE(p != nullptr, MOE_ERR_CUDA, "no device address for the fixed scratch array");
    g_noalloc_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return MOE_OK;
}

// How many warps share one token row in the movers: one warp per token when
// the batch gives every SM warps_per_sm warps, more for small batches.  The
// combine takes 16 (its 126 registers a thread keep 16 warps on an SM, and
// each extra part repeats the token's BRIM reads): one warp per token
// measured 52.0 against 56.1 us on the OLMoE-shaped combine (T = 4096).
int mover_parts(const DeviceInfo* di, int T, int max_parts, int warps_per_sm = 32) {
  const long long want = (long long)di->num_sms * warps_per_sm;
  int P = (int)((want + T - 1) / (T > 0 ? T : 1));
  if (P > max_parts) P = max_parts;
  return P < 1 ? 1 : P;
}




// The BRIM passes, compiled for a bound KMAX >= k so per-token state stays in
// registers.
template <int KMAX>
int launch_brim_passes(const int32_t* topk_idx, const float* topk_w, int T, int k,
                       const int32_t* slot_of, int E, int R, int32_t* brim0, int32_t* sfd_token,
                       int32_t* sfd_off, int32_t* brim1, int32_t* epd_off, int32_t* epd_sfd,
                       float* epd_gate, int32_t* c_t, uint32_t* scratch, unsigned* err,
                       cudaStream_t stream) {
  const int n_tiles = (T + moe::kBrimTileTokens - 1) / moe::kBrimTileTokens;
  const int blocks = (n_tiles + 3) / 4;
  const int ncol = R + E;
  int32_t* totals = reinterpret_cast<int32_t*>(scratch) + (size_t)ncol * n_tiles;
  MOE_CUDA(launch_k(moe::brim_mask_kernel<KMAX>, blocks, 128, 0, stream, topk_idx, slot_of, T, k, E, R, n_tiles,
                                                          scratch, err));
  MOE_LAUNCHED("brim_mask_kernel");
  // the column scan writes the tiles' bases over the masks
  MOE_CUDA(launch_k(moe::brim_colscan_kernel, ncol, moe::kColscanThreads, 0, stream,
                    static_cast<const uint32_t*>(scratch), scratch, n_tiles, ncol, totals, T, R,
                    static_cast<int32_t*>(nullptr)));
  MOE_LAUNCHED("brim_colscan_kernel");
  MOE_CUDA(launch_k(moe::brim_scatter_kernel<KMAX>, n_tiles, 32 * moe::kScatterWarps, 0, stream,
      topk_idx, topk_w, slot_of, T, k, E, R, n_tiles, reinterpret_cast<const int32_t*>(scratch),
      static_cast<const int32_t*>(totals), sfd_off, epd_off, c_t, brim0, sfd_token, brim1,
      epd_sfd, epd_gate, moe::BrimExtras{}));
  MOE_LAUNCHED("brim_scatter_kernel");
  return MOE_OK;
}

int brim_passes(const int32_t* topk_idx, const float* topk_w, int T, int k, const int32_t* slot_of,
                int E, int R, int32_t* brim0, int32_t* sfd_token, int32_t* sfd_off, int32_t* brim1,
                int32_t* epd_off, int32_t* epd_sfd, float* epd_gate, int32_t* c_t,
                uint32_t* scratch, unsigned* err, cudaStream_t stream) {
#define MOE_BRIM_K(KM)                                                                        \
  return launch_brim_passes<KM>(topk_idx, topk_w, T, k, slot_of, E, R, brim0, sfd_token,      \
                                sfd_off, brim1, epd_off, epd_sfd, epd_gate, c_t, scratch, err, \
                                stream)
  if (k <= 2) MOE_BRIM_K(2);
  if (k <= 4) MOE_BRIM_K(4);
  if (k <= 8) MOE_BRIM_K(8);
  MOE_BRIM_K(16);
#undef MOE_BRIM_K
}

// Scratch entries of a BRIM build: one 32-bit word per column per 32-token
// tile (the masks, which the column scan overwrites with the tiles' bases),
// then one total per column.
size_t brim_scratch_entries(int T, int E, int R) {
  const size_t n_tiles = ((size_t)T + moe::kBrimTileTokens - 1) / moe::kBrimTileTokens;
  return (n_tiles + 1) * (size_t)(R + E);
}

}  // namespace

// ---------------------------------------------------------------------------
namespace moe_host {
namespace {
// Shared memory the bulk combine takes per block, for its piece size.
size_t combine_bulk_smem(int kmax, int piece_bytes) {
  return (size_t)moe::kBulkWarps * (3 * kmax + 1) * piece_bytes;
}

template <typename TA, int KM>
int launch_combine_bulk(DeviceInfo* di, const void* o_epd, int T, int d, int R, int L,
                        size_t cap, int tk, const int32_t* brim0, const int32_t* brim1,
                        const void* shared_out, void* y_sfd, void* y, cudaStream_t stream) {
  // piece: as large as two blocks per SM allow (~110 KB each), 512 B .. 8 KB;
  // shorter for batches too small to give every SM 16 units of work
  const int row_bytes = d * (int)sizeof(TA);
  int piece = (110 * 1024) / (moe::kBulkWarps * (3 * KM + 1));
  piece = piece / 512 * 512;
  if (piece < 512) piece = 512;
  if (piece > moe::kBulkPiece) piece = moe::kBulkPiece;
  if (piece > row_bytes) piece = row_bytes;
  const long long want = (long long)di->num_sms * 16;
  while ((long long)T * ((row_bytes + piece - 1) / piece) < want && piece >= 1024) piece /= 2;
  piece = piece / 128 * 128;
  const int n_pieces = (row_bytes + piece - 1) / piece;
  const size_t smem = combine_bulk_smem(KM, piece);
  // the kernel's limit is raised once per device, to the most any piece size
  // above can ask for (110 KB)
  constexpr size_t kMaxSmem = 110 * 1024;
  MOE_REQUIRE(smem <= kMaxSmem, MOE_ERR_UNSUPPORTED, "combine staging too large");
  auto kern = moe::combine_bulk_kernel<TA, KM>;
  int rc = ensure_smem(di, reinterpret_cast<const void*>(kern), kMaxSmem);
  if (rc) return rc;
  const long long units = (long long)T * n_pieces;
  long long blocks = (units + moe::kBulkWarps - 1) / moe::kBulkWarps;
  if (blocks > 2LL * di->num_sms) blocks = 2LL * di->num_sms;
  MOE_CUDA(launch_k(kern, (int)blocks, moe::kBulkWarps * 32, smem, stream,
                    static_cast<const TA*>(o_epd), T, d, piece / (int)sizeof(TA), n_pieces, R, L,
                    cap, tk, brim0, brim1, static_cast<const TA*>(shared_out),
                    static_cast<TA*>(y_sfd), static_cast<TA*>(y), di->err_flag,
                    wait_limit_ns()));
  MOE_LAUNCHED("combine_bulk_kernel");
  return MOE_OK;
}

// The combine kernel (register path, or the copy engine's under
// kDebugBulkMovers) for every combine entry point: the whole return path,
// y_sfd only (y == NULL), or the returned rows summed into y (brim1 == NULL,
// L == 1, rows = the SFD rows).
int launch_combine(const void* o_epd, int T, int d, int dtype, int k, int R, int L,
                   size_t cap, int tk, const int32_t* brim0, const int32_t* brim1,
                   const void* shared_out, void* y_sfd, void* y, cudaStream_t stream) {
  DeviceInfo* di;
  int rc = device_info(&di);
  if (rc) return rc;
  if (g_debug_flags & kDebugBulkMovers) {
#define MOE_CB(TA, KM)                                                                         \
  return launch_combine_bulk<TA, KM>(di, o_epd, T, d, R, L, cap, tk, brim0, brim1, shared_out, \
                                     y_sfd, y, stream)
    if (dtype == MOE_BF16) {
      using B = __nv_bfloat16;
      if (k <= 2) MOE_CB(B, 2);
      if (k <= 4) MOE_CB(B, 4);
      if (k <= 8) MOE_CB(B, 8);
      MOE_CB(B, 16);
    } else {
      if (k <= 2) MOE_CB(float, 2);
      if (k <= 4) MOE_CB(float, 4);
      if (k <= 8) MOE_CB(float, 8);
      MOE_CB(float, 16);
    }
#undef MOE_CB
  }
  const int P = mover_parts(di, T, (d * esize(dtype) + 511) / 512, 16);
  const long long warps = (long long)T * P;
  const int blocks = (int)((warps + moe::kMoverWarps - 1) / moe::kMoverWarps);
#define MOE_COMBINE(TA, KM)                                                                    \
  MOE_CUDA(launch_k(moe::combine_kernel<TA, KM>, blocks, moe::kMoverWarps * 32, 0, stream,     \
      static_cast<const TA*>(o_epd), T, d, P, R, L, cap, tk, brim0, brim1,                     \
      static_cast<const TA*>(shared_out), static_cast<TA*>(y_sfd), static_cast<TA*>(y),        \
      di->err_flag))
  if (dtype == MOE_BF16) {
    using B = __nv_bfloat16;
    if (k <= 2) MOE_COMBINE(B, 2);
    else if (k <= 4) MOE_COMBINE(B, 4);
    else if (k <= 8) MOE_COMBINE(B, 8);
    else MOE_COMBINE(B, 16);
  } else {
    if (k <= 2) MOE_COMBINE(float, 2);
    else if (k <= 4) MOE_COMBINE(float, 4);
    else if (k <= 8) MOE_COMBINE(float, 8);
    else MOE_COMBINE(float, 16);
  }
#undef MOE_COMBINE
  MOE_LAUNCHED("combine_kernel");
  return MOE_OK;
}
}  // namespace
}  // namespace moe_host

// ===========================================================================
extern "C" {

int moe_abi_version(void) { return 1; }

const char* moe_last_error(void) { return last_message(); }

// Test-only knobs: debug flags of the GEMM (1 = skip the first TMA load, so a
// bounded wait expires) and the device wait limit in milliseconds.
int moe_set_debug(int flags, double wait_limit_ms) {
  MOE_REQUIRE(wait_limit_ms > 0.0, MOE_ERR_INVALID_ARG, "wait limit must be positive");
  g_debug_flags = flags;
  g_wait_limit_ms = wait_limit_ms;
  return MOE_OK;
}

int moe_get_device_status(moe_stream_t stream) {
  DeviceInfo* di;
  int rc = device_info(&di);
  if (rc) return rc;
  // One atomic exchange on the device reads the flag and clears it, ordered
  // after the stream's earlier work: a bit that a kernel on another stream
  // raises at any moment is either in this reading or left for the next one.
  // The host lock keeps two callers from sharing the snapshot word.
  std::lock_guard<std::mutex> lk(g_status_mu);
  MOE_CUDA(launch_k(take_error_flag_kernel, 1, 1, 0, stream));
  MOE_LAUNCHED("take_error_flag_kernel");
  unsigned v = 0;
  MOE_CUDA(cudaMemcpyFromSymbolAsync(&v, g_moe_err_snapshot, sizeof v, 0,
                                     cudaMemcpyDeviceToHost, stream));
  MOE_CUDA(cudaStreamSynchronize(stream));
  if (v & moe::kErrTimeout) return fail(MOE_ERR_TIMEOUT, "a bounded device wait expired");
  if (v & moe::kErrIndex) return fail(MOE_ERR_DEVICE_CHECK, "a kernel met an out-of-range index");
  return MOE_OK;
}

// ---------------------------------------------------------------------------
int moe_route_topk(const float* logits, int T, int E, int k, int renorm, int32_t* topk_idx,
                   float* topk_w, moe_stream_t stream) {
  int rc = check_common(T, E, k, 1);
  if (rc) return rc;
  MOE_REQUIRE(renorm == 0 || renorm == 1, MOE_ERR_INVALID_ARG, "renorm must be 0 or 1");
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(logits && topk_idx && topk_w, MOE_ERR_INVALID_ARG, "null pointer");
  DeviceInfo* di;
  if ((rc = device_info(&di))) return rc;
  // G lanes per token (the result does not depend on G)
  const int G = moe::route_lanes_per_token(T, di->num_sms);
  const int blocks = (int)(((long long)T * G + 255) / 256);
#define MOE_ROUTE_TOPK(KM, GG)                                                                \
  MOE_CUDA(launch_k(moe::route_topk_kernel<KM, GG>, blocks, 256, 0, stream, logits, T, E, k,  \
                    renorm, topk_idx, topk_w))
#define MOE_ROUTE_TOPK_G(KM)                                                                   \
  do {                                                                                        \
    if (G == 8) MOE_ROUTE_TOPK(KM, 8);                                                        \
    else if (G == 4) MOE_ROUTE_TOPK(KM, 4);                                                   \
    else if (G == 2) MOE_ROUTE_TOPK(KM, 2);                                                   \
    else MOE_ROUTE_TOPK(KM, 1);                                                               \
  } while (0)
  if (k <= 2) MOE_ROUTE_TOPK_G(2);
  else if (k <= 4) MOE_ROUTE_TOPK_G(4);
  else if (k <= 8) MOE_ROUTE_TOPK_G(8);
  else MOE_ROUTE_TOPK_G(16);
#undef MOE_ROUTE_TOPK_G
#undef MOE_ROUTE_TOPK
  MOE_LAUNCHED("route_topk_kernel");
  return MOE_OK;
}

// ---------------------------------------------------------------------------
size_t moe_brim_workspace_size(int T, int E, int R) {
  if (T < 0 || E < 1 || R < 1) return 0;
  return align256(sizeof(int32_t) * brim_scratch_entries(T, E, R)) + 256;
}

int moe_brim_build(const int32_t* topk_idx, const float* topk_w, int T, int k,
                   const int32_t* slot_of, int E, int R, int32_t* brim0, int32_t* sfd_token,
                   int32_t* sfd_off, int32_t* brim1, int32_t* epd_off, int32_t* epd_sfd,
                   float* epd_gate, int32_t* c_t, void* ws, size_t ws_bytes,
                   moe_stream_t stream) {
  int rc = check_common(T, E, k, R);
  if (rc) return rc;
  MOE_REQUIRE(slot_of && sfd_off && epd_off && c_t, MOE_ERR_INVALID_ARG, "null pointer");
  DeviceInfo* di;
  if ((rc = device_info(&di))) return rc;
  if (T == 0) {
    MOE_CUDA(cudaMemsetAsync(sfd_off, 0, sizeof(int32_t) * (R + 1), stream));
    MOE_CUDA(cudaMemsetAsync(epd_off, 0, sizeof(int32_t) * (E + 1), stream));
    MOE_CUDA(cudaMemsetAsync(c_t, 0, sizeof(int32_t), stream));
    return MOE_OK;
  }
  MOE_REQUIRE(topk_idx && topk_w && brim0 && sfd_token && brim1 && epd_sfd && epd_gate && ws,
              MOE_ERR_INVALID_ARG, "null pointer");
  MOE_REQUIRE(ws_bytes >= moe_brim_workspace_size(T, E, R), MOE_ERR_INVALID_ARG,
              "workspace too small: %zu < %zu bytes", ws_bytes, moe_brim_workspace_size(T, E, R));
  return brim_passes(topk_idx, topk_w, T, k, slot_of, E, R, brim0, sfd_token, sfd_off, brim1,
                     epd_off, epd_sfd, epd_gate, c_t, static_cast<uint32_t*>(ws), di->err_flag,
                     stream);
}

// ---------------------------------------------------------------------------
// moe_brim_build_noalloc: the BRIM build for callers that cannot allocate
// device memory or lend a workspace (see the header).  Its scratch is a fixed
// file-scope device array; host code only ever uses the device address that
// cudaGetSymbolAddress returns for it, looked up once per device.
int moe_brim_build_noalloc(const int32_t* topk_idx, const float* topk_w, int T, int k,
                           const int32_t* slot_of, int E, int R, int32_t* brim0,
                           int32_t* sfd_token, int32_t* sfd_off, int32_t* brim1,
                           int32_t* epd_off, int32_t* epd_sfd, float* epd_gate, int32_t* c_t,
                           moe_stream_t stream) {
  int rc = check_common(T, E, k, R);
  if (rc) return rc;
  MOE_REQUIRE(slot_of && sfd_off && epd_off && c_t, MOE_ERR_INVALID_ARG, "null pointer");
  const size_t need = brim_scratch_entries(T, E, R);
  MOE_REQUIRE(need <= kNoAllocScratchInts, MOE_ERR_UNSUPPORTED,
              "moe_brim_build_noalloc: T=%d, R=%d, E=%d needs %zu scratch entries, more than "
              "its fixed %zu (1 MiB); use moe_brim_build with a workspace",
              T, R, E, need, kNoAllocScratchInts);
  DeviceInfo* di;
  if ((rc = device_info(&di))) return rc;
  int32_t* counts = nullptr;
  if ((rc = noalloc_scratch(&counts))) return rc;
  if (T == 0) {
    MOE_CUDA(cudaMemsetAsync(sfd_off, 0, sizeof(int32_t) * (R + 1), stream));
    MOE_CUDA(cudaMemsetAsync(epd_off, 0, sizeof(int32_t) * (E + 1), stream));
    MOE_CUDA(cudaMemsetAsync(c_t, 0, sizeof(int32_t), stream));
    return MOE_OK;
  }
  MOE_REQUIRE(topk_idx && topk_w && brim0 && sfd_token && brim1 && epd_sfd && epd_gate,
              MOE_ERR_INVALID_ARG, "null pointer");
  return brim_passes(topk_idx, topk_w, T, k, slot_of, E, R, brim0, sfd_token, sfd_off, brim1,
                     epd_off, epd_sfd, epd_gate, c_t, reinterpret_cast<uint32_t*>(counts),
                     di->err_flag, stream);
}

// ---------------------------------------------------------------------------
int moe_prune_topk(int32_t* topk_idx, float* topk_w, int T, int k, const int32_t* slot_of, int E,
                   int R, int m, moe_stream_t stream) {
  int rc = check_common(T, E, k, R);
  if (rc) return rc;
  MOE_REQUIRE(m >= 1, MOE_ERR_INVALID_ARG, "m must be >= 1 (got %d)", m);
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(topk_idx && topk_w && slot_of, MOE_ERR_INVALID_ARG, "null pointer");
  DeviceInfo* di;
  if ((rc = device_info(&di))) return rc;
  const dim3 grid((T + 255) / 256), block(256);
#define MOE_PRUNE(KM) \
  MOE_CUDA(launch_k(moe::prune_kernel<KM>, grid, block, 0, stream, topk_idx, topk_w, T, k, slot_of, E, R, m))
  if (k <= 2) {
    MOE_PRUNE(2);
  } else if (k <= 4) {
    MOE_PRUNE(4);
  } else if (k <= 8) {
    MOE_PRUNE(8);
  } else {
    MOE_PRUNE(16);
  }
#undef MOE_PRUNE
  MOE_LAUNCHED("prune_kernel");
  return MOE_OK;
}

// ---------------------------------------------------------------------------
// Scratch of the fused index path: the masks, the tiles' bases (kept apart so
// that the histogram can read the masks after the column scan), the column
// totals and the rank columns' own-rank hits.
size_t route_brim_scratch_entries(int T, int E, int R) {
  const size_t n_tiles = ((size_t)T + moe::kBrimTileTokens - 1) / moe::kBrimTileTokens;
  return (2 * n_tiles + 1) * (size_t)(R + E) + (size_t)R;
}

size_t moe_route_brim_workspace_size(int T, int E, int R) {
  if (T < 0 || E < 1 || R < 1) return 0;
  return align256(sizeof(int32_t) * route_brim_scratch_entries(T, E, R)) + 256;
}

int moe_route_brim(const float* logits, int T, int E, int k, int renorm, const int32_t* slot_of,
                   int R, int prune_m, int32_t* topk_idx, float* topk_w, int32_t* brim0, int32_t* sfd_token,
                   int32_t* sfd_off, int32_t* brim1, int32_t* epd_off, int32_t* epd_sfd,
                   float* epd_gate, int32_t* c_t, int32_t* per_rank, int64_t* total,
                   int64_t* remote, uint32_t* hist, int hist_accumulate, void* ws,
                   size_t ws_bytes, moe_stream_t stream) {
  int rc = check_common(T, E, k, R);
  if (rc) return rc;
  MOE_REQUIRE(renorm == 0 || renorm == 1, MOE_ERR_INVALID_ARG, "renorm must be 0 or 1");
  MOE_REQUIRE(prune_m >= 0, MOE_ERR_INVALID_ARG, "prune_m must be >= 0 (0 = no pruning)");
  MOE_REQUIRE(slot_of && sfd_off && epd_off && c_t, MOE_ERR_INVALID_ARG, "null pointer");
  MOE_REQUIRE((per_rank == nullptr) == (total == nullptr) && (total == nullptr) == (remote == nullptr),
              MOE_ERR_INVALID_ARG, "per_rank, total and remote are given together or not at all");
  DeviceInfo* di;
  if ((rc = device_info(&di))) return rc;
  if (hist && !hist_accumulate)
    MOE_CUDA(cudaMemsetAsync(hist, 0, sizeof(uint32_t) * E * E, stream));
  if (T == 0) {
    if (per_rank) {
      MOE_CUDA(cudaMemsetAsync(per_rank, 0, sizeof(int32_t) * R, stream));
      MOE_CUDA(cudaMemsetAsync(total, 0, sizeof(int64_t), stream));
      MOE_CUDA(cudaMemsetAsync(remote, 0, sizeof(int64_t), stream));
    }
    MOE_CUDA(cudaMemsetAsync(sfd_off, 0, sizeof(int32_t) * (R + 1), stream));
    MOE_CUDA(cudaMemsetAsync(epd_off, 0, sizeof(int32_t) * (E + 1), stream));
    MOE_CUDA(cudaMemsetAsync(c_t, 0, sizeof(int32_t), stream));
    return MOE_OK;
  }
  MOE_REQUIRE(logits && topk_idx && topk_w && brim0 && sfd_token && brim1 && epd_sfd && epd_gate &&
                  ws,
              MOE_ERR_INVALID_ARG, "null pointer");
  MOE_REQUIRE(ws_bytes >= moe_route_brim_workspace_size(T, E, R), MOE_ERR_INVALID_ARG,
              "workspace too small: %zu < %zu bytes", ws_bytes,
              moe_route_brim_workspace_size(T, E, R));
  MOE_REQUIRE(aligned16(ws), MOE_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  uint32_t* masks = static_cast<uint32_t*>(ws);
  const int n_tiles = (T + moe::kBrimTileTokens - 1) / moe::kBrimTileTokens;
  const int ncol = R + E;
  uint32_t* bases = masks + (size_t)ncol * n_tiles;
  int32_t* totals = reinterpret_cast<int32_t*>(bases + (size_t)ncol * n_tiles);
  int32_t* own = totals + ncol;
  moe::BrimExtras extras{};
  if (per_rank) {
    extras.per_rank = per_rank;
    extras.total = reinterpret_cast<unsigned long long*>(total);
    extras.remote = reinterpret_cast<unsigned long long*>(remote);
    extras.own = own;
  }
  if (hist) {
    extras.hist = hist;
    extras.masks = masks;
    const int ct = moe::hist_chunk_tiles(E);
    extras.n_hist = (n_tiles + ct - 1) / ct;
  }
  const int G = moe::route_lanes_per_token(T, di->num_sms);
#define MOE_ROUTE_TILE(KM, GG)                                                                \
  MOE_CUDA(launch_k(moe::route_brim_tile_kernel<KM, GG>,                                     \
                    dim3((n_tiles + moe::RouteTile<GG>::kTiles - 1) / moe::RouteTile<GG>::kTiles), \
                    dim3(moe::RouteTile<GG>::kThreads), 0, stream, logits, T, E, k, renorm,    \
                    slot_of, R, prune_m, n_tiles, topk_idx, topk_w, masks, di->err_flag))
#define MOE_ROUTE_TILE_G(KM)                                                                   \
  do {                                                                                        \
    if (G == 8) MOE_ROUTE_TILE(KM, 8);                                                        \
    else if (G == 4) MOE_ROUTE_TILE(KM, 4);                                                   \
    else if (G == 2) MOE_ROUTE_TILE(KM, 2);                                                   \
    else MOE_ROUTE_TILE(KM, 1);                                                               \
  } while (0)
#define MOE_ROUTE_BRIM(KM)                                                                    \
  MOE_ROUTE_TILE_G(KM);                                                                       \
  MOE_CUDA(launch_k(moe::brim_colscan_kernel, dim3(ncol), dim3(moe::kColscanThreads), 0,      \
                    stream, static_cast<const uint32_t*>(masks), bases, n_tiles, ncol, totals,  \
                    T, R, per_rank ? own : static_cast<int32_t*>(nullptr)));                    \
  MOE_CUDA(launch_k(moe::brim_scatter_kernel<KM>, dim3(extras.n_hist + n_tiles),              \
                    dim3(32 * moe::kScatterWarps), 0, stream, static_cast<const int32_t*>(topk_idx), \
                    static_cast<const float*>(topk_w), slot_of, T, k, E, R, n_tiles,            \
                    reinterpret_cast<const int32_t*>(bases), static_cast<const int32_t*>(totals), \
                    sfd_off, epd_off, c_t, brim0, sfd_token, brim1, epd_sfd, epd_gate, extras))
  if (k <= 2) {
    MOE_ROUTE_BRIM(2);
  } else if (k <= 4) {
    MOE_ROUTE_BRIM(4);
  } else if (k <= 8) {
    MOE_ROUTE_BRIM(8);
  } else {
    MOE_ROUTE_BRIM(16);
  }
#undef MOE_ROUTE_BRIM
#undef MOE_ROUTE_TILE_G
#undef MOE_ROUTE_TILE
  MOE_LAUNCHED("route_brim_tile_kernel");
  return MOE_OK;
}

// ---------------------------------------------------------------------------
// Token shuffling across layers.
int moe_interlayer_histogram(const int32_t* idx_l, const int32_t* idx_next, int T, int k, int E,
                             uint32_t* hist, int accumulate, moe_stream_t stream) {
  int rc = check_common(T, E, k, 1);
  if (rc) return rc;
  MOE_REQUIRE(hist, MOE_ERR_INVALID_ARG, "null pointer");
  if (!accumulate) MOE_CUDA(cudaMemsetAsync(hist, 0, sizeof(uint32_t) * E * E, stream));
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(idx_l && idx_next, MOE_ERR_INVALID_ARG, "null pointer");
  DeviceInfo* di;
  if ((rc = device_info(&di))) return rc;
  const dim3 grid((T + 255) / 256), block(256);
#define MOE_IL(KM)                                                                            \
  MOE_CUDA(launch_k(moe::interlayer_hist_kernel<KM>, grid, block, 0, stream, idx_l, idx_next, T, \
                    k, E, hist, di->err_flag))
  if (k <= 2) MOE_IL(2);
  else if (k <= 4) MOE_IL(4);
  else if (k <= 8) MOE_IL(8);
  else MOE_IL(16);
#undef MOE_IL
  MOE_LAUNCHED("interlayer_hist_kernel");
  return MOE_OK;
}

int moe_rank_affinity(const uint32_t* hist, int E, const int32_t* slot_of_next, int R,
                      uint32_t* table, moe_stream_t stream) {
  int rc = check_common(0, E, 1, R);
  if (rc) return rc;
  MOE_REQUIRE(hist && slot_of_next && table, MOE_ERR_INVALID_ARG, "null pointer");
  DeviceInfo* di;
  if ((rc = device_info(&di))) return rc;
  MOE_CUDA(launch_k(moe::rank_affinity_kernel, dim3((E * R + 255) / 256), dim3(256), 0, stream,
                    hist, E, slot_of_next, R, table, di->err_flag));
  MOE_LAUNCHED("rank_affinity_kernel");
  return MOE_OK;
}

int moe_predict_home(const int32_t* idx_l, int T, int k, int E, const uint32_t* table, int R,
                     int32_t* home, moe_stream_t stream) {
  int rc = check_common(T, E, k, R);
  if (rc) return rc;
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(idx_l && table && home, MOE_ERR_INVALID_ARG, "null pointer");
  DeviceInfo* di;
  if ((rc = device_info(&di))) return rc;
  const dim3 grid((unsigned)(((long long)T * 32 + 255) / 256)), block(256);
#define MOE_PH(KM) \
  MOE_CUDA(launch_k(moe::predict_home_kernel<KM>, grid, block, 0, stream, idx_l, T, k, E, table, R, home))
  if (k <= 2) MOE_PH(2);
  else if (k <= 4) MOE_PH(4);
  else if (k <= 8) MOE_PH(8);
  else MOE_PH(16);
#undef MOE_PH
  MOE_LAUNCHED("predict_home_kernel");
  return MOE_OK;
}

int moe_count_local(const int32_t* idx, int T, int k, const int32_t* slot_of, int E, int R,
                    const int32_t* home, int64_t* out, moe_stream_t stream) {
  int rc = check_common(T, E, k, R);
  if (rc) return rc;
  MOE_REQUIRE(out, MOE_ERR_INVALID_ARG, "null pointer");
  MOE_CUDA(cudaMemsetAsync(out, 0, 2 * sizeof(int64_t), stream));
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(idx && slot_of, MOE_ERR_INVALID_ARG, "null pointer");
  DeviceInfo* di;
  if ((rc = device_info(&di))) return rc;
  const dim3 grid((T + 255) / 256), block(256);
  auto* o = reinterpret_cast<unsigned long long*>(out);
#define MOE_CL(KM)                                                                             \
  MOE_CUDA(launch_k(moe::count_local_kernel<KM>, grid, block, 0, stream, idx, T, k, slot_of, E, R, \
                    home, o, di->err_flag))
  if (k <= 2) MOE_CL(2);
  else if (k <= 4) MOE_CL(4);
  else if (k <= 8) MOE_CL(8);
  else MOE_CL(16);
#undef MOE_CL
  MOE_LAUNCHED("count_local_kernel");
  return MOE_OK;
}

namespace {
struct ShuffleCarve {
  uint32_t* scratch; int32_t *brim0, *brim1, *epd_off, *epd_sfd, *c_t; float* epd_gate;
};
size_t carve_shuffle(char* base, int T, int R, ShuffleCarve* out) {
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + off : nullptr;
    off += align256(bytes ? bytes : 1);
    return p;
  };
  ShuffleCarve c{};
  c.scratch = reinterpret_cast<uint32_t*>(take(sizeof(int32_t) * brim_scratch_entries(T, R, R)));
  c.brim0 = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (size_t)R * T));
  c.brim1 = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (size_t)T));
  c.epd_off = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (R + 1)));
  c.epd_sfd = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (size_t)T));
  c.epd_gate = reinterpret_cast<float*>(take(sizeof(float) * (size_t)T));
  c.c_t = reinterpret_cast<int32_t*>(take(sizeof(int32_t)));
  if (out) *out = c;
  return off + 256;
}
}  // namespace

size_t moe_token_shuffle_workspace_size(int T, int R) {
  if (T < 0 || R < 1 || R > moe::kMaxE) return 0;
  return carve_shuffle(nullptr, T, R, nullptr);
}

int moe_token_shuffle(const int32_t* home, int T, int R, const void* x, int d, int dtype,
                      void* x_out, int32_t* perm, int32_t* rank_off, int32_t* inv, void* ws,
                      size_t ws_bytes, moe_stream_t stream) {
  int rc = check_common(T, R, 1, R);
  if (rc) return rc;
  MOE_REQUIRE(rank_off, MOE_ERR_INVALID_ARG, "null pointer");
  MOE_REQUIRE(!x || ((rc = check_dtype(dtype)) == 0 && d >= 64 && d % 64 == 0 && x_out),
              MOE_ERR_INVALID_ARG, "x needs x_out, a known dtype and d a positive multiple of 64");
  if (T == 0) {
    MOE_CUDA(cudaMemsetAsync(rank_off, 0, sizeof(int32_t) * (R + 1), stream));
    return MOE_OK;
  }
  MOE_REQUIRE(perm, MOE_ERR_INVALID_ARG, "null pointer");
  MOE_REQUIRE(home && ws && aligned16(ws), MOE_ERR_INVALID_ARG, "null or misaligned pointer");
  MOE_REQUIRE(!x || (aligned16(x) && aligned16(x_out)), MOE_ERR_INVALID_ARG,
              "rows must be 16-byte aligned");
  const size_t need = carve_shuffle(nullptr, T, R, nullptr);
  MOE_REQUIRE(ws_bytes >= need, MOE_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes",
              ws_bytes, need);
  DeviceInfo* di;
  if ((rc = device_info(&di))) return rc;
  char* base = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~uintptr_t(255));
  ShuffleCarve c;
  carve_shuffle(base, T, R, &c);
  // the home-rank order: BRIM_0 over one "expert" per rank (k = 1, E = R,
  // identity placement), so the order within a rank is ascending token order
  if ((rc = brim_passes(home, nullptr, T, 1, nullptr, R, R, c.brim0, perm, rank_off, c.brim1,
                        c.epd_off, c.epd_sfd, c.epd_gate, c.c_t, c.scratch, di->err_flag, stream)))
    return rc;
  if (x || inv) {
    const int row_bytes = x ? d * esize(dtype) : 0;
    MOE_CUDA(launch_k(moe::gather_rows_kernel, dim3((unsigned)(((long long)T * 32 + 255) / 256)),
                      dim3(256), 0, stream, static_cast<const uint8_t*>(x), perm, T, row_bytes,
                      static_cast<uint8_t*>(x_out), inv, di->err_flag));
    MOE_LAUNCHED("gather_rows_kernel");
  }
  return MOE_OK;
}

// ---------------------------------------------------------------------------
int moe_dispatch_gather(const void* x, int T, int d, int dtype, int k, int R, int L,
                        const int32_t* brim0, const int32_t* brim1, void* x_sfd, void* x_epd,
                        moe_stream_t stream) {
  int rc = check_dtype(dtype);
  if (rc) return rc;
  MOE_REQUIRE(T >= 0 && k >= 1 && k <= moe::kMaxK && R >= 1 && L >= 1 && R * L <= moe::kMaxE,
              MOE_ERR_UNSUPPORTED, "bad shape (T=%d k=%d R=%d L=%d)", T, k, R, L);
  MOE_REQUIRE(d >= 64 && d % 64 == 0, MOE_ERR_UNSUPPORTED, "d must be a positive multiple of 64");
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(x && brim0 && brim1 && (x_sfd || x_epd), MOE_ERR_INVALID_ARG, "null pointer");
  MOE_REQUIRE(aligned16(x) && aligned16(x_sfd) && aligned16(x_epd), MOE_ERR_INVALID_ARG,
              "row buffers must be 16-byte aligned");
  DeviceInfo* di;
  if ((rc = device_info(&di))) return rc;
  const size_t cap = (size_t)T * (k < R ? k : R);
  const int row_bytes = d * esize(dtype);
  if (g_debug_flags & kDebugBulkMovers) {
    // copy-engine dispatch: whole rows (up to 8 KB) per unit when the batch
    // fills the GPU, shorter pieces (>= 512 bytes) when it does not
    const long long want = (long long)di->num_sms * 16;
    int n_pieces = (row_bytes + moe::kBulkPiece - 1) / moe::kBulkPiece;
    while ((long long)T * n_pieces < want && row_bytes / (2 * n_pieces) >= 512) n_pieces *= 2;
    int piece = (row_bytes + n_pieces - 1) / n_pieces;
    piece = (piece + 127) & ~127;
    if (piece > moe::kBulkPiece) piece = moe::kBulkPiece;
    n_pieces = (row_bytes + piece - 1) / piece;
    const long long units = (long long)T * n_pieces;
    long long blocks = (units + moe::kBulkWarps - 1) / moe::kBulkWarps;
    if (blocks > 2LL * di->num_sms) blocks = 2LL * di->num_sms;
    if ((rc = ensure_smem(di, reinterpret_cast<const void*>(moe::dispatch_bulk_kernel),
                          moe::kBulkSmem)))
      return rc;
    MOE_CUDA(launch_k(moe::dispatch_bulk_kernel, (int)blocks, moe::kBulkWarps * 32,
                      moe::kBulkSmem, stream, static_cast<const uint8_t*>(x), T, row_bytes, piece,
                      n_pieces, R, L, cap, T * k, brim0, brim1, static_cast<uint8_t*>(x_sfd),
                      static_cast<uint8_t*>(x_epd), di->err_flag, wait_limit_ns()));
    MOE_LAUNCHED("dispatch_bulk_kernel");
    return MOE_OK;
  }
  constexpr int CH = 4;  // 512-byte chunks in flight per warp
  const int P = mover_parts(di, T, (row_bytes + CH * 512 - 1) / (CH * 512));
  const long long warps = (long long)T * P;
  const int blocks = (int)((warps + moe::kMoverWarps - 1) / moe::kMoverWarps);
  MOE_CUDA(launch_k(moe::dispatch_kernel<CH>, blocks, moe::kMoverWarps * 32, 0, stream, 
      static_cast<const uint8_t*>(x), T, row_bytes, P, R, L, cap, T * k, brim0, brim1,
      static_cast<uint8_t*>(x_sfd), static_cast<uint8_t*>(x_epd), di->err_flag));
  MOE_LAUNCHED("dispatch_kernel");
  return MOE_OK;
}

// ---------------------------------------------------------------------------
int moe_combine_scatter(const void* o_epd, int T, int d, int dtype, int k, int R, int L,
                        const int32_t* brim0, const int32_t* brim1, const void* shared_out,
                        void* y_sfd, void* y, moe_stream_t stream) {
  int rc = check_dtype(dtype);
  if (rc) return rc;
  MOE_REQUIRE(T >= 0 && k >= 1 && k <= moe::kMaxK && R >= 1 && L >= 1 && R * L <= moe::kMaxE,
              MOE_ERR_UNSUPPORTED, "bad shape (T=%d k=%d R=%d L=%d)", T, k, R, L);
  MOE_REQUIRE(d >= 64 && d % 64 == 0, MOE_ERR_UNSUPPORTED, "d must be a positive multiple of 64");
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(o_epd && brim0 && brim1 && y, MOE_ERR_INVALID_ARG, "null pointer");
  MOE_REQUIRE(aligned16(o_epd) && aligned16(y) && aligned16(y_sfd) && aligned16(shared_out),
              MOE_ERR_INVALID_ARG, "row buffers must be 16-byte aligned");
  DeviceInfo* di;
  if ((rc = device_info(&di))) return rc;
  const size_t cap = (size_t)T * (k < R ? k : R);
  return launch_combine(o_epd, T, d, dtype, k, R, L, cap, T * k, brim0, brim1, shared_out, y_sfd,
                        y, stream);
}

// ---------------------------------------------------------------------------
// Real expert parallelism: the device steps around the all-to-all exchanges.
int moe_ep_pack_routing(const int32_t* topk_idx, const float* topk_w, int T, int k,
                        const int32_t* slot_of, int E, int R, const int32_t* sfd_token,
                        const int32_t* sfd_off, const int32_t* c_t, int32_t* idx_send,
                        float* w_send, moe_stream_t stream) {
  int rc = check_common(T, E, k, R);
  if (rc) return rc;
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(topk_idx && topk_w && slot_of && sfd_token && sfd_off && c_t && idx_send && w_send,
              MOE_ERR_INVALID_ARG, "null pointer");
  DeviceInfo* di;
  if ((rc = device_info(&di))) return rc;
  const long long cap = (long long)T * (k < R ? k : R);
  long long blocks = (cap + 255) / 256;
  if (blocks > 8LL * di->num_sms) blocks = 8LL * di->num_sms;
  MOE_CUDA(launch_k(moe::ep_pack_routing_kernel, (int)blocks, 256, 0, stream, topk_idx, topk_w,
                    T, k, slot_of, E, R, E / R, sfd_token, sfd_off, c_t, cap, idx_send, w_send,
                    di->err_flag));
  MOE_LAUNCHED("ep_pack_routing_kernel");
  return MOE_OK;
}


int moe_ep_return_rows(const void* o_epd, int T, int d, int dtype, int k, int R, int L,
                       const int32_t* brim0, const int32_t* brim1, void* y_ret,
                       moe_stream_t stream) {
  int rc = check_dtype(dtype);
  if (rc) return rc;
  MOE_REQUIRE(T >= 0 && k >= 1 && k <= moe::kMaxK && R >= 1 && L >= 1 && R * L <= moe::kMaxE,
              MOE_ERR_UNSUPPORTED, "bad shape (T=%d k=%d R=%d L=%d)", T, k, R, L);
  MOE_REQUIRE(d >= 64 && d % 64 == 0, MOE_ERR_UNSUPPORTED, "d must be a positive multiple of 64");
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(o_epd && brim0 && brim1 && y_ret, MOE_ERR_INVALID_ARG, "null pointer");
  MOE_REQUIRE(aligned16(o_epd) && aligned16(y_ret), MOE_ERR_INVALID_ARG,
              "row buffers must be 16-byte aligned");
  const size_t cap = (size_t)T * (k < R ? k : R);
  return launch_combine(o_epd, T, d, dtype, k, R, L, cap, T * k, brim0, brim1, nullptr, y_ret,
                        nullptr, stream);
}

int moe_ep_combine(const void* y_ret, int T, int d, int dtype, int k, int R,
                   const int32_t* brim0, const void* shared_out, void* y, moe_stream_t stream) {
  int rc = check_dtype(dtype);
  if (rc) return rc;
  MOE_REQUIRE(T >= 0 && k >= 1 && k <= moe::kMaxK && R >= 1 && R <= moe::kMaxE,
              MOE_ERR_UNSUPPORTED, "bad shape (T=%d k=%d R=%d)", T, k, R);
  MOE_REQUIRE(d >= 64 && d % 64 == 0, MOE_ERR_UNSUPPORTED, "d must be a positive multiple of 64");
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(y_ret && brim0 && y, MOE_ERR_INVALID_ARG, "null pointer");
  MOE_REQUIRE(aligned16(y_ret) && aligned16(y) && aligned16(shared_out), MOE_ERR_INVALID_ARG,
              "row buffers must be 16-byte aligned");
  const int kr = k < R ? k : R;  // at most this many ranks per token
  const size_t cap = (size_t)T * kr;
  return launch_combine(y_ret, T, d, dtype, kr, R, 1, cap, (int)cap, brim0, nullptr, shared_out,
                        nullptr, y, stream);
}

// ---------------------------------------------------------------------------
// The exchange over peer memory.  The host struct is copied, as it is, into
// the kernels' parameter of the same layout.
static_assert(sizeof(moe_ep_peers) == sizeof(moe::EpPeers) &&
                  offsetof(moe_ep_peers, row0) == offsetof(moe::EpPeers, row0) &&
                  offsetof(moe_ep_peers, seg) == offsetof(moe::EpPeers, seg) &&
                  MOE_EP_MAX_PEERS == moe::kMaxEpPeers,
              "moe_ep_peers and the device table must match");

static int check_peers(const moe_ep_peers* peers, int R, size_t row_bytes, bool lists) {
  MOE_REQUIRE(peers, MOE_ERR_INVALID_ARG, "null peer table");
  MOE_REQUIRE(R <= MOE_EP_MAX_PEERS, MOE_ERR_UNSUPPORTED, "R = %d peers, at most %d", R,
              MOE_EP_MAX_PEERS);
  for (int q = 0; q < R; ++q) {
    MOE_REQUIRE(peers->rows[q] && aligned16(peers->rows[q]) && peers->row0[q] >= -(1LL << 40),
                MOE_ERR_INVALID_ARG, "peer %d: row buffer missing or not 16-byte aligned", q);
    MOE_REQUIRE(!lists || (peers->idx[q] && peers->w[q]), MOE_ERR_INVALID_ARG,
                "peer %d: routing-list buffers missing", q);
  }
  (void)row_bytes;
  return MOE_OK;
}

int moe_ep_send_peer(const void* x, int T, int d, int dtype, int k, int R, int L,
                     const int32_t* topk_idx, const float* topk_w, const int32_t* slot_of,
                     const int32_t* brim0, const int32_t* brim1, const int32_t* sfd_token,
                     const int32_t* sfd_off, const int32_t* c_t, const moe_ep_peers* peers,
                     moe_stream_t stream) {
  int rc = check_dtype(dtype);
  if (rc) return rc;
  MOE_REQUIRE(T >= 0 && k >= 1 && k <= moe::kMaxK && R >= 1 && L >= 1 && R * L <= moe::kMaxE,
              MOE_ERR_UNSUPPORTED, "bad shape (T=%d k=%d R=%d L=%d)", T, k, R, L);
  MOE_REQUIRE(d >= 64 && d % 64 == 0, MOE_ERR_UNSUPPORTED, "d must be a positive multiple of 64");
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(x && topk_idx && topk_w && slot_of && brim0 && brim1 && sfd_token && sfd_off && c_t,
              MOE_ERR_INVALID_ARG, "null pointer");
  MOE_REQUIRE(aligned16(x), MOE_ERR_INVALID_ARG, "row buffers must be 16-byte aligned");
  const int row_bytes = d * esize(dtype);
  if ((rc = check_peers(peers, R, (size_t)row_bytes, true))) return rc;
  DeviceInfo* di;
  if ((rc = device_info(&di))) return rc;
  moe::EpPeers pe;
  std::memcpy(&pe, peers, sizeof pe);
  const size_t cap = (size_t)T * (k < R ? k : R);
  constexpr int CH = 4;  // 512-byte chunks in flight per warp
  const int P = mover_parts(di, T, (row_bytes + CH * 512 - 1) / (CH * 512));
  const long long warps = (long long)T * P;
  const int blocks = (int)((warps + moe::kMoverWarps - 1) / moe::kMoverWarps);
  MOE_CUDA(launch_k(moe::dispatch_peer_kernel<CH>, blocks, moe::kMoverWarps * 32, 0, stream,
                    static_cast<const uint8_t*>(x), T, row_bytes, P, R, L, cap, T * k, brim0,
                    brim1, static_cast<uint8_t*>(nullptr), di->err_flag, pe));
  MOE_LAUNCHED("dispatch_peer_kernel");
  long long pblocks = ((long long)cap + 255) / 256;
  if (pblocks > 8LL * di->num_sms) pblocks = 8LL * di->num_sms;
  MOE_CUDA(launch_k(moe::ep_pack_routing_peer_kernel, (int)pblocks, 256, 0, stream, topk_idx,
                    topk_w, T, k, slot_of, R * L, R, L, sfd_token, sfd_off, c_t,
                    (long long)cap, di->err_flag, pe));
  MOE_LAUNCHED("ep_pack_routing_peer_kernel");
  return MOE_OK;
}

int moe_ep_return_peer(const void* o_epd, int T, int d, int dtype, int k, int R, int L,
                       const int32_t* brim0, const int32_t* brim1, const moe_ep_peers* peers,
                       moe_stream_t stream) {
  int rc = check_dtype(dtype);
  if (rc) return rc;
  MOE_REQUIRE(T >= 0 && k >= 1 && k <= moe::kMaxK && R >= 1 && L >= 1 && R * L <= moe::kMaxE,
              MOE_ERR_UNSUPPORTED, "bad shape (T=%d k=%d R=%d L=%d)", T, k, R, L);
  MOE_REQUIRE(d >= 64 && d % 64 == 0, MOE_ERR_UNSUPPORTED, "d must be a positive multiple of 64");
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(o_epd && brim0 && brim1, MOE_ERR_INVALID_ARG, "null pointer");
  MOE_REQUIRE(aligned16(o_epd), MOE_ERR_INVALID_ARG, "row buffers must be 16-byte aligned");
  if ((rc = check_peers(peers, R, (size_t)d * esize(dtype), false))) return rc;
  for (int q = 0; q < R; ++q)
    MOE_REQUIRE(peers->seg[q] <= peers->seg[q + 1], MOE_ERR_INVALID_ARG,
                "peer segments must not run backwards");
  DeviceInfo* di;
  if ((rc = device_info(&di))) return rc;
  moe::EpPeers pe;
  std::memcpy(&pe, peers, sizeof pe);
  const size_t cap = (size_t)T * (k < R ? k : R);
  const int P = mover_parts(di, T, (d * esize(dtype) + 511) / 512, 16);
  const long long warps = (long long)T * P;
  const int blocks = (int)((warps + moe::kMoverWarps - 1) / moe::kMoverWarps);
#define MOE_RET(TA, KM)                                                                        \
  MOE_CUDA(launch_k(moe::combine_peer_kernel<TA, KM>, blocks, moe::kMoverWarps * 32, 0, stream, \
                    static_cast<const TA*>(o_epd), T, d, P, R, L, cap, T * k, brim0, brim1,    \
                    di->err_flag, pe))
  if (dtype == MOE_BF16) {
    using B = __nv_bfloat16;
    if (k <= 2) MOE_RET(B, 2);
    else if (k <= 4) MOE_RET(B, 4);
    else if (k <= 8) MOE_RET(B, 8);
    else MOE_RET(B, 16);
  } else {
    if (k <= 2) MOE_RET(float, 2);
    else if (k <= 4) MOE_RET(float, 4);
    else if (k <= 8) MOE_RET(float, 8);
    else MOE_RET(float, 16);
  }
#undef MOE_RET
  MOE_LAUNCHED("combine_peer_kernel");
  return MOE_OK;
}

// ---------------------------------------------------------------------------
int moe_prepare_weights(const void* wg, const void* wu, const void* wd, int E, int d, int f,
                        int dtype, const int32_t* slot_of, void* w_gu, void* w_dn,
                        moe_stream_t stream) {
  int rc = check_dtype(dtype);
  if (rc) return rc;
  MOE_REQUIRE(E >= 1 && E <= moe::kMaxE, MOE_ERR_UNSUPPORTED, "E must be in [1, 256]");
  MOE_REQUIRE(d >= 64 && d % 64 == 0 && f >= 64 && f % 64 == 0, MOE_ERR_UNSUPPORTED,
              "d and f must be positive multiples of 64 (d=%d f=%d)", d, f);
  MOE_REQUIRE(wg && wu && wd && w_gu && w_dn, MOE_ERR_INVALID_ARG, "null pointer");
  MOE_REQUIRE(aligned16(wg) && aligned16(wu) && aligned16(wd) && aligned16(w_gu) && aligned16(w_dn),
              MOE_ERR_INVALID_ARG, "weights must be 16-byte aligned");
  DeviceInfo* di;
  if ((rc = device_info(&di))) return rc;
  const int es = esize(dtype);
  const int grid = di->num_sms * 4;
  MOE_CUDA(launch_k(moe::pack_gate_up_kernel, grid, 256, 0, stream, static_cast<const uint8_t*>(wg),
                                                     static_cast<const uint8_t*>(wu), E, d, f, es,
                                                     slot_of, static_cast<uint8_t*>(w_gu)));
  MOE_LAUNCHED("pack_gate_up_kernel");
  MOE_CUDA(launch_k(moe::pack_down_kernel, grid, 256, 0, stream, static_cast<const uint8_t*>(wd), E, d, f, es,
                                                  slot_of, static_cast<uint8_t*>(w_dn)));
  MOE_LAUNCHED("pack_down_kernel");
  return MOE_OK;
}

int moe_prepare_shared_weights(const void* sg, const void* su, const void* sd, int S, int d,
                               int fs, int dtype, void* w_gu, void* w_dn, moe_stream_t stream) {
  int rc = check_dtype(dtype);
  if (rc) return rc;
  MOE_REQUIRE(S >= 1 && d >= 64 && d % 64 == 0 && fs >= 64 && fs % 64 == 0, MOE_ERR_UNSUPPORTED,
              "need S >= 1 and d, fs positive multiples of 64 (S=%d d=%d fs=%d)", S, d, fs);
  MOE_REQUIRE(sg && su && sd && w_gu && w_dn, MOE_ERR_INVALID_ARG, "null pointer");
  MOE_REQUIRE(aligned16(sg) && aligned16(su) && aligned16(sd) && aligned16(w_gu) && aligned16(w_dn),
              MOE_ERR_INVALID_ARG, "weights must be 16-byte aligned");
  DeviceInfo* di;
  if ((rc = device_info(&di))) return rc;
  const int es = esize(dtype);
  const int grid = di->num_sms * 4;
  MOE_CUDA(launch_k(moe::pack_shared_gate_up_kernel, grid, 256, 0, stream, static_cast<const uint8_t*>(sg),
                                                            static_cast<const uint8_t*>(su), S, d,
                                                            fs, es, static_cast<uint8_t*>(w_gu)));
  MOE_LAUNCHED("pack_shared_gate_up_kernel");
  MOE_CUDA(launch_k(moe::pack_shared_down_kernel, grid, 256, 0, stream, static_cast<const uint8_t*>(sd), S, d,
                                                         fs, es, static_cast<uint8_t*>(w_dn)));
  MOE_LAUNCHED("pack_shared_down_kernel");
  return MOE_OK;
}

// ---------------------------------------------------------------------------
size_t moe_expert_ffn_workspace_size(int m_cap, int f, int dtype) {
  if (m_cap < 0 || f < 0) return 0;
  return align256((size_t)m_cap * f * (dtype == MOE_BF16 ? 2 : 4)) + 256;
}

int moe_expert_ffn(const void* a, int a_rows, const int32_t* a_row_index,
                   const int32_t* group_off, int G, int m_cap, const void* w_gu,
                   const void* w_dn, int d, int f, int dtype, const float* row_scale,
                   int ffn_kind, void* out, void* ws, size_t ws_bytes, moe_stream_t stream) {
  int rc = check_dtype(dtype);
  if (rc) return rc;
  MOE_REQUIRE(ffn_kind == MOE_FFN_SWIGLU || ffn_kind == MOE_FFN_IDENTITY, MOE_ERR_INVALID_ARG,
              "unknown ffn_kind %d", ffn_kind);
  MOE_REQUIRE(G >= 1 && G <= moe::kGemmMaxGroups, MOE_ERR_UNSUPPORTED,
              "G must be in [1, %d] (got %d)", moe::kGemmMaxGroups, G);
  MOE_REQUIRE(m_cap >= 0 && a_rows >= 0, MOE_ERR_INVALID_ARG, "m_cap and a_rows must be >= 0");
  MOE_REQUIRE(a_row_index || a_rows >= m_cap, MOE_ERR_INVALID_ARG,
              "without a row index, a needs at least m_cap rows (a_rows=%d m_cap=%d)", a_rows,
              m_cap);
  MOE_REQUIRE(d >= 64 && d % 64 == 0, MOE_ERR_UNSUPPORTED, "d must be a positive multiple of 64");
  if (m_cap == 0) return MOE_OK;
  MOE_REQUIRE(a && group_off && out && a_rows > 0, MOE_ERR_INVALID_ARG, "null pointer or empty a");
  MOE_REQUIRE(aligned16(a) && aligned16(out), MOE_ERR_INVALID_ARG, "a and out must be 16-byte aligned");
  DeviceInfo* di;
  if ((rc = device_info(&di))) return rc;
  if (ffn_kind == MOE_FFN_IDENTITY) {
    MOE_REQUIRE(a_row_index == nullptr, MOE_ERR_UNSUPPORTED,
                "the identity expert takes its rows in place (no row index)");
    const int grid = di->num_sms * 8;
    if (dtype == MOE_BF16)
      MOE_CUDA(launch_k(moe::identity_expert_kernel<__nv_bfloat16>, grid, moe::kMoverWarps * 32, 0, stream, 
          static_cast<const __nv_bfloat16*>(a), group_off, G, d, row_scale,
          static_cast<__nv_bfloat16*>(out)));
    else
      MOE_CUDA(launch_k(moe::identity_expert_kernel<float>, grid, moe::kMoverWarps * 32, 0, stream, 
          static_cast<const float*>(a), group_off, G, d, row_scale, static_cast<float*>(out)));
    MOE_LAUNCHED("identity_expert_kernel");
    return MOE_OK;
  }
  MOE_REQUIRE(f >= 64 && f % 64 == 0, MOE_ERR_UNSUPPORTED, "f must be a positive multiple of 64");
  MOE_REQUIRE(w_gu && w_dn && ws, MOE_ERR_INVALID_ARG, "null pointer");
  MOE_REQUIRE(ws_bytes >= moe_expert_ffn_workspace_size(m_cap, f, dtype), MOE_ERR_INVALID_ARG,
              "workspace too small: %zu < %zu bytes", ws_bytes,
              moe_expert_ffn_workspace_size(m_cap, f, dtype));
  MOE_REQUIRE(aligned16(w_gu) && aligned16(w_dn) && aligned16(ws), MOE_ERR_INVALID_ARG,
              "weights and workspace must be 16-byte aligned");
  void* h = ws;  // [m_cap, f]
  if (dtype == MOE_BF16) {
    rc = launch_gemm_auto<moe::kEpiSwiGLU, false>(di, a, a_rows, a_row_index, m_cap, d, w_gu, G,
                                                  2 * f, group_off, nullptr, h, f, stream);
    if (rc) return rc;
    rc = launch_gemm_auto<moe::kEpiScale, false>(di, h, m_cap, nullptr, m_cap, f, w_dn, G, d,
                                                 group_off, row_scale, out, d, stream);
  } else {
    rc = launch_gemm_auto<moe::kEpiSwiGLU, true>(di, a, a_rows, a_row_index, m_cap, d, w_gu, G,
                                                 2 * f, group_off, nullptr, h, f, stream);
    if (rc) return rc;
    rc = launch_gemm_auto<moe::kEpiScale, true>(di, h, m_cap, nullptr, m_cap, f, w_dn, G, d,
                                                group_off, row_scale, out, d, stream);
  }
  return rc;
}

// ---------------------------------------------------------------------------
int moe_count_dispatched_rows(const int32_t* topk_idx, int T, int k, const int32_t* slot_of,
                              int E, int R, int32_t* per_rank, int64_t* total, int64_t* remote,
                              moe_stream_t stream) {
  int rc = check_common(T, E, k, R);
  if (rc) return rc;
  MOE_REQUIRE(slot_of && per_rank && total && remote, MOE_ERR_INVALID_ARG, "null pointer");
  DeviceInfo* di;
  if ((rc = device_info(&di))) return rc;
  MOE_CUDA(cudaMemsetAsync(per_rank, 0, sizeof(int32_t) * R, stream));
  MOE_CUDA(cudaMemsetAsync(total, 0, sizeof(int64_t), stream));
  MOE_CUDA(cudaMemsetAsync(remote, 0, sizeof(int64_t), stream));
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(topk_idx, MOE_ERR_INVALID_ARG, "null pointer");
  {
    auto* tot = reinterpret_cast<unsigned long long*>(total);
    auto* rem = reinterpret_cast<unsigned long long*>(remote);
    const int blocks = (T + 255) / 256;
    if (k <= 2)
      MOE_CUDA(launch_k(moe::count_dispatched_kernel<2>, blocks, 256, 0, stream, topk_idx, T, k, slot_of, E, R,
                                                                  per_rank, tot, rem, di->err_flag));
    else if (k <= 4)
      MOE_CUDA(launch_k(moe::count_dispatched_kernel<4>, blocks, 256, 0, stream, topk_idx, T, k, slot_of, E, R,
                                                                  per_rank, tot, rem, di->err_flag));
    else if (k <= 8)
      MOE_CUDA(launch_k(moe::count_dispatched_kernel<8>, blocks, 256, 0, stream, topk_idx, T, k, slot_of, E, R,
                                                                  per_rank, tot, rem, di->err_flag));
    else
      MOE_CUDA(launch_k(moe::count_dispatched_kernel<16>, blocks, 256, 0, stream, topk_idx, T, k, slot_of, E, R,
                                                                   per_rank, tot, rem, di->err_flag));
  }
  MOE_LAUNCHED("count_dispatched_kernel");
  return MOE_OK;
}

int moe_coact_histogram(const int32_t* topk_idx, int T, int k, int E, uint32_t* hist,
                        int accumulate, moe_stream_t stream) {
  int rc = check_common(T, E, k, 1);
  if (rc) return rc;
  MOE_REQUIRE(hist, MOE_ERR_INVALID_ARG, "null pointer");
  DeviceInfo* di;
  if ((rc = device_info(&di))) return rc;
  if (!accumulate) MOE_CUDA(cudaMemsetAsync(hist, 0, sizeof(uint32_t) * E * E, stream));
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(topk_idx, MOE_ERR_INVALID_ARG, "null pointer");
  {
    const int blocks = (T + 255) / 256;
    if (k <= 2)
      MOE_CUDA(launch_k(moe::coact_hist_kernel<2>, blocks, 256, 0, stream, topk_idx, T, k, E, hist, di->err_flag));
    else if (k <= 4)
      MOE_CUDA(launch_k(moe::coact_hist_kernel<4>, blocks, 256, 0, stream, topk_idx, T, k, E, hist, di->err_flag));
    else if (k <= 8)
      MOE_CUDA(launch_k(moe::coact_hist_kernel<8>, blocks, 256, 0, stream, topk_idx, T, k, E, hist, di->err_flag));
    else
      MOE_CUDA(launch_k(moe::coact_hist_kernel<16>, blocks, 256, 0, stream, topk_idx, T, k, E, hist, di->err_flag));
  }
  MOE_LAUNCHED("coact_hist_kernel");
  return MOE_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// The whole layer.  The workspace is carved into the layer's intermediate
// state, every region 256-byte aligned.
__global__ void set_pair_kernel(int32_t* p, int a, int b) {
  moe::pdl_enter();
  p[0] = a;
  p[1] = b;
}

namespace {

struct LayerCarve {
  size_t off = 0;
  char* base = nullptr;
  template <typename T>
  T* take(size_t count) {
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += align256(sizeof(T) * (count ? count : 1));
    return p;
  }
};

struct LayerState {
  float* logits; void* x; void* y;   // host staging (host variant only)
  int32_t* topk_idx; float* topk_w;
  int32_t *brim0, *sfd_token, *sfd_off, *brim1, *epd_off, *epd_sfd; float* epd_gate;
  int32_t* c_t; void* brim_ws; size_t brim_ws_bytes;
  void *x_sfd, *x_epd, *o_epd, *y_sfd, *shared_out;
  void* ffn_ws; size_t ffn_ws_bytes; void* sffn_ws; size_t sffn_ws_bytes;
  int32_t* shared_off;
  int32_t* per_rank; int64_t* total; int64_t* remote; uint32_t* hist;
};

size_t carve_layer(char* base, int T, int d, int f, int E, int k, int R, int S, int fs,
                   int dtype, bool host, LayerState* st) {
  LayerCarve c;
  c.base = base;
  LayerState s{};
  const int es = esize(dtype);
  const size_t cap = (size_t)T * (k < R ? k : R), tk = (size_t)T * k;
  const int L = E / R;
  if (host) {
    s.logits = c.take<float>((size_t)T * E);
    s.x = c.take<char>((size_t)T * d * es);
    s.y = c.take<char>((size_t)T * d * es);
  }
  s.topk_idx = c.take<int32_t>(tk);
  s.topk_w = c.take<float>(tk);
  s.brim0 = c.take<int32_t>((size_t)R * T);
  s.sfd_token = c.take<int32_t>(cap);
  s.sfd_off = c.take<int32_t>(R + 1);
  s.brim1 = c.take<int32_t>((size_t)L * cap);
  s.epd_off = c.take<int32_t>(E + 1);
  s.epd_sfd = c.take<int32_t>(tk);
  s.epd_gate = c.take<float>(tk);
  s.c_t = c.take<int32_t>(1);
  s.brim_ws_bytes = moe_route_brim_workspace_size(T, E, R);
  s.brim_ws = c.take<char>(s.brim_ws_bytes);
  s.x_sfd = c.take<char>(cap * d * es);
  s.x_epd = L > 1 ? c.take<char>(tk * d * es) : nullptr;
  s.o_epd = c.take<char>(tk * d * es);
  s.y_sfd = c.take<char>(cap * d * es);
  s.ffn_ws_bytes = moe_expert_ffn_workspace_size((int)(tk ? tk : 1), f, dtype);
  s.ffn_ws = c.take<char>(s.ffn_ws_bytes);
  if (S > 0) {
    s.shared_out = c.take<char>((size_t)T * d * es);
    s.sffn_ws_bytes = moe_expert_ffn_workspace_size(T ? T : 1, S * fs, dtype);
    s.sffn_ws = c.take<char>(s.sffn_ws_bytes);
    s.shared_off = c.take<int32_t>(2);
  }
  s.per_rank = c.take<int32_t>(R);
  s.total = c.take<int64_t>(1);
  s.remote = c.take<int64_t>(1);
  s.hist = c.take<uint32_t>((size_t)E * E);
  if (!host) {
    s.logits = nullptr;
    s.x = s.y = nullptr;
  }
  if (st) *st = s;
  return c.off + 256;
}

int layer_steps(int T, int d, int f, int E, int k, int R, int renorm, int prune_m, int S, int fs,
                int dtype,
                const float* logits, const void* x, const int32_t* slot_of, const void* w_gu,
                const void* w_dn, const void* sw_gu, const void* sw_dn, void* y, int32_t* c_t_out,
                int32_t* per_rank, int64_t* total, int64_t* remote, uint32_t* hist,
                const LayerState& st, cudaStream_t stream) {
  const int L = E / R;
  const size_t tk = (size_t)T * k;
  const size_t cap = (size_t)T * (k < R ? k : R);
  int rc;
  if ((rc = moe_route_brim(logits, T, E, k, renorm, slot_of, R, prune_m, st.topk_idx, st.topk_w,
                           st.brim0,
                           st.sfd_token, st.sfd_off, st.brim1, st.epd_off, st.epd_sfd,
                           st.epd_gate, c_t_out ? c_t_out : st.c_t,
                           per_rank ? per_rank : st.per_rank, total ? total : st.total,
                           remote ? remote : st.remote, hist ? hist : st.hist, hist ? 1 : 0,
                           st.brim_ws, st.brim_ws_bytes, stream)))
    return rc;
  if ((rc = moe_dispatch_gather(x, T, d, dtype, k, R, L, st.brim0, st.brim1, st.x_sfd, st.x_epd,
                                stream)))
    return rc;
  // with L = 1 the EPD state is the SFD state row for row: run on the payload
  const void* a = L > 1 ? st.x_epd : st.x_sfd;
  const int a_rows = (int)(L > 1 ? (tk ? tk : 1) : (cap ? cap : 1));
  if ((rc = moe_expert_ffn(a, a_rows, nullptr, st.epd_off, E, (int)(tk ? tk : 1), w_gu, w_dn, d,
                           f, dtype, st.epd_gate, MOE_FFN_SWIGLU, st.o_epd, st.ffn_ws,
                           st.ffn_ws_bytes, stream)))
    return rc;
  if (S > 0) {
    MOE_CUDA(launch_k(set_pair_kernel, 1, 1, 0, stream, st.shared_off, 0, T));  // the one shared group: [0, T)
    MOE_LAUNCHED("set_pair_kernel");
    if ((rc = moe_expert_ffn(x, T, nullptr, st.shared_off, 1, T, sw_gu, sw_dn, d, S * fs, dtype,
                             nullptr, MOE_FFN_SWIGLU, st.shared_out, st.sffn_ws,
                             st.sffn_ws_bytes, stream)))
      return rc;
  }
  if ((rc = moe_combine_scatter(st.o_epd, T, d, dtype, k, R, L, st.brim0, st.brim1,
                                S > 0 ? st.shared_out : nullptr, st.y_sfd, y, stream)))
    return rc;
  return MOE_OK;
}

int check_layer_args(int T, int d, int f, int E, int k, int R, int renorm, int S, int fs,
                     int dtype) {
  int rc = check_common(T, E, k, R);
  if (rc) return rc;
  if ((rc = check_dtype(dtype))) return rc;
  MOE_REQUIRE(renorm == 0 || renorm == 1, MOE_ERR_INVALID_ARG, "renorm must be 0 or 1");
  MOE_REQUIRE(d >= 64 && d % 64 == 0 && f >= 64 && f % 64 == 0, MOE_ERR_UNSUPPORTED,
              "d and f must be positive multiples of 64 (d=%d f=%d)", d, f);
  MOE_REQUIRE(S >= 0 && (S == 0 || (fs >= 64 && fs % 64 == 0)), MOE_ERR_UNSUPPORTED,
              "shared experts need fs a positive multiple of 64 (S=%d fs=%d)", S, fs);
  return MOE_OK;
}

}  // namespace

extern "C" {

size_t moe_layer_workspace_size(int T, int d, int f, int E, int k, int R, int S, int fs,
                                int dtype, int host_staging) {
  if (check_layer_args(T, d, f, E, k, R, 0, S, fs, dtype)) return 0;
  return carve_layer(nullptr, T, d, f, E, k, R, S, fs, dtype, host_staging != 0, nullptr);
}

int moe_layer_forward(int T, int d, int f, int E, int k, int R, int renorm, int prune_m, int S,
                      int fs, int dtype, const float* logits, const void* x, const int32_t* slot_of,
                      const void* w_gu, const void* w_dn, const void* sw_gu, const void* sw_dn,
                      void* y, int32_t* c_t, int32_t* per_rank, int64_t* total, int64_t* remote,
                      uint32_t* hist, void* ws, size_t ws_bytes, moe_stream_t stream) {
  int rc = check_layer_args(T, d, f, E, k, R, renorm, S, fs, dtype);
  if (rc) return rc;
  MOE_REQUIRE(ws && aligned16(ws), MOE_ERR_INVALID_ARG, "workspace missing or misaligned");
  const size_t need = carve_layer(nullptr, T, d, f, E, k, R, S, fs, dtype, false, nullptr);
  MOE_REQUIRE(ws_bytes >= need, MOE_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes",
              ws_bytes, need);
  MOE_REQUIRE(S == 0 || (sw_gu && sw_dn), MOE_ERR_INVALID_ARG, "shared weights missing");
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(logits && x && y && slot_of && w_gu && w_dn, MOE_ERR_INVALID_ARG, "null pointer");
  char* base = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~uintptr_t(255));
  LayerState st;
  carve_layer(base, T, d, f, E, k, R, S, fs, dtype, false, &st);
  MOE_REQUIRE(prune_m >= 0, MOE_ERR_INVALID_ARG, "prune_m must be >= 0 (0 = no pruning)");
  return layer_steps(T, d, f, E, k, R, renorm, prune_m, S, fs, dtype, logits, x, slot_of, w_gu,
                     w_dn,
                     sw_gu, sw_dn, y, c_t, per_rank, total, remote, hist, st, stream);
}

namespace {
int layer_forward_host(int T, int d, int f, int E, int k, int R, int renorm, int prune_m, int S,
                       int fs, int dtype, const float* h_logits, const void* h_x,
                       const int32_t* slot_of, const void* w_gu, const void* w_dn,
                       const void* sw_gu, const void* sw_dn, void* h_y, void* ws,
                       size_t ws_bytes, cudaStream_t stream, bool sync) {
  int rc = check_layer_args(T, d, f, E, k, R, renorm, S, fs, dtype);
  if (rc) return rc;
  MOE_REQUIRE(ws && aligned16(ws), MOE_ERR_INVALID_ARG, "workspace missing or misaligned");
  const size_t need = carve_layer(nullptr, T, d, f, E, k, R, S, fs, dtype, true, nullptr);
  MOE_REQUIRE(ws_bytes >= need, MOE_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes",
              ws_bytes, need);
  MOE_REQUIRE(S == 0 || (sw_gu && sw_dn), MOE_ERR_INVALID_ARG, "shared weights missing");
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(h_logits && h_x && h_y && slot_of && w_gu && w_dn, MOE_ERR_INVALID_ARG,
              "null pointer");
  MOE_REQUIRE(prune_m >= 0, MOE_ERR_INVALID_ARG, "prune_m must be >= 0 (0 = no pruning)");
  char* base = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~uintptr_t(255));
  LayerState st;
  carve_layer(base, T, d, f, E, k, R, S, fs, dtype, true, &st);
  const size_t xb = (size_t)T * d * esize(dtype);
  MOE_CUDA(cudaMemcpyAsync(st.logits, h_logits, sizeof(float) * (size_t)T * E,
                           cudaMemcpyHostToDevice, stream));
  MOE_CUDA(cudaMemcpyAsync(st.x, h_x, xb, cudaMemcpyHostToDevice, stream));
  rc = layer_steps(T, d, f, E, k, R, renorm, prune_m, S, fs, dtype, st.logits, st.x, slot_of,
                   w_gu, w_dn, sw_gu, sw_dn, st.y, nullptr, nullptr, nullptr, nullptr, nullptr,
                   st, stream);
  if (rc) return rc;
  MOE_CUDA(cudaMemcpyAsync(h_y, st.y, xb, cudaMemcpyDeviceToHost, stream));
  if (sync) MOE_CUDA(cudaStreamSynchronize(stream));
  return MOE_OK;
}
}  // namespace

int moe_layer_forward_host(int T, int d, int f, int E, int k, int R, int renorm, int prune_m,
                           int S, int fs, int dtype, const float* h_logits, const void* h_x,
                           const int32_t* slot_of, const void* w_gu, const void* w_dn,
                           const void* sw_gu, const void* sw_dn, void* h_y, void* ws,
                           size_t ws_bytes, moe_stream_t stream) {
  return layer_forward_host(T, d, f, E, k, R, renorm, prune_m, S, fs, dtype, h_logits, h_x,
                            slot_of, w_gu, w_dn, sw_gu, sw_dn, h_y, ws, ws_bytes, stream, true);
}

int moe_layer_forward_host_async(int T, int d, int f, int E, int k, int R, int renorm,
                                 int prune_m, int S, int fs, int dtype, const float* h_logits,
                                 const void* h_x, const int32_t* slot_of, const void* w_gu,
                                 const void* w_dn, const void* sw_gu, const void* sw_dn,
                                 void* h_y, void* ws, size_t ws_bytes, moe_stream_t stream) {
  return layer_forward_host(T, d, f, E, k, R, renorm, prune_m, S, fs, dtype, h_logits, h_x,
                            slot_of, w_gu, w_dn, sw_gu, sw_dn, h_y, ws, ws_bytes, stream, false);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Correlated placement (host).
extern "C" int moe_place_greedy(const uint32_t* hist, int E, int R, int32_t* slot_of) {
  MOE_REQUIRE(hist && slot_of, MOE_ERR_INVALID_ARG, "null pointer");
  MOE_REQUIRE(E >= 1 && E <= moe::kMaxE && R >= 1 && E % R == 0, MOE_ERR_UNSUPPORTED,
              "need 1 <= E <= 256 and R dividing E (E=%d R=%d)", E, R);
  const int L = E / R;
  std::vector<char> free_(E, 1);
  // affinity[b] = sum over the current rank's members a of hist[a][b]
  std::vector<uint64_t> affinity(E);
  auto self = [&](int e) { return hist[(size_t)e * E + e]; };
  for (int r = 0; r < R; ++r) {
    std::fill(affinity.begin(), affinity.end(), 0);
    for (int n = 0; n < L; ++n) {
      int pick = -1;
      for (int b = 0; b < E; ++b) {
        if (!free_[b]) continue;
        if (pick < 0) {
          pick = b;
          continue;
        }
        // first member: most-selected expert; then: strongest co-activation,
        // ties by self count, then by lower id (b ascends, so `>` keeps it)
        const bool better =
            n == 0 ? self(b) > self(pick)
                   : (affinity[b] > affinity[pick] ||
                      (affinity[b] == affinity[pick] && self(b) > self(pick)));
        if (better) pick = b;
      }
      free_[pick] = 0;
      slot_of[pick] = r * L + n;
      for (int b = 0; b < E; ++b) affinity[b] += hist[(size_t)pick * E + b];
    }
  }
  return MOE_OK;
}
