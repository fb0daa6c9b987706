// brim.cuh -- BRIM_0 / BRIM_1 construction, the placement-aware dispatched-row
// counter and the expert co-activation histogram.
//
// BRIM_0 is [EP ranks x ORI tokens] and BRIM_1 is [local experts x SFD
// tokens] (Occult paper, Figure 5).  An entry is the row the token occupies in
// the next state (-1 = not sent); the same entry drives the gather into the
// compact state and the scatter back out of it.  A token is sent once to each
// rank holding one of its experts ("Expert Coupling", Abstract), so the SFD
// row count C_T is the all-to-all budget (Occult paper, TL;DR).
//
// Positions are stable (ascending token order inside every rank segment and
// every expert group), which makes them unique.  They come from a three-pass
// deterministic scan over tiles of 256 tokens:
//   1. count   : per tile, how many tokens hit each rank and each slot
//   2. scan    : exclusive scan of the tile counts per column, column totals
//                -> sfd_off, epd_off, C_T, and each tile's global base
//   3. scatter : inside a tile, a token's rank among the tile's tokens that hit
//                the same column is the popcount of a per-warp lane mask plus
//                the counts of the earlier warps; add the tile base, write.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kBrimTile = 256;     // tokens per tile (one per thread)
constexpr int kBrimWarps = kBrimTile / 32;
constexpr int kMaxK = 16;
constexpr int kMaxE = 256;

// Gather one token's experts, slots and distinct ranks.  Returns false (and
// raises the error flag) when an expert id is out of range or repeated.
struct TokenRoute {
  int n_rank;               // distinct ranks hit
  int rank[kMaxK];          // the ranks, in order of first appearance
  int slot[kMaxK];          // slot of each selected expert
};

__device__ __forceinline__ bool load_token_route(const int32_t* __restrict__ topk_idx,
                                                 const int32_t* __restrict__ slot_of, int t,
                                                 int k, int E, int L, TokenRoute& tr,
                                                 unsigned* err) {
  tr.n_rank = 0;
  bool ok = true;
  for (int j = 0; j < k; ++j) {
    int e = topk_idx[(size_t)t * k + j];
    int q = -1;
    if (e >= 0 && e < E) q = slot_of[e];
    if (q < 0 || q >= E) {
      ok = false;
      tr.slot[j] = -1;
      continue;
    }
    for (int i = 0; i < j; ++i)
      if (tr.slot[i] == q) ok = false;  // the same expert twice
    tr.slot[j] = q;
    const int r = q / L;
    bool seen = false;
    for (int i = 0; i < tr.n_rank; ++i) seen |= (tr.rank[i] == r);
    if (!seen) tr.rank[tr.n_rank++] = r;
  }
  if (!ok) raise_error(err, kErrIndex);
  return ok;
}

// ---- pass 1 ---------------------------------------------------------------
// counts[c][tile] (column-major, so a column's tiles are contiguous):
//   c < R      : tokens of the tile that hit rank c
//   c = R + q  : tokens of the tile that selected the expert at slot q
__global__ void __launch_bounds__(kBrimTile) brim_count_kernel(
    const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ slot_of, int T, int k,
    int E, int R, int n_tiles, int32_t* __restrict__ counts, unsigned* err) {
  __shared__ int32_t sc[kMaxE * 2];
  const int ncol = R + E;
  const int L = E / R;
  for (int c = threadIdx.x; c < ncol; c += blockDim.x) sc[c] = 0;
  __syncthreads();
  const int t = blockIdx.x * kBrimTile + threadIdx.x;
  if (t < T) {
    TokenRoute tr;
    if (load_token_route(topk_idx, slot_of, t, k, E, L, tr, err)) {
      for (int i = 0; i < tr.n_rank; ++i) atomicAdd(&sc[tr.rank[i]], 1);
      for (int j = 0; j < k; ++j) atomicAdd(&sc[R + tr.slot[j]], 1);
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < ncol; c += blockDim.x)
    counts[(size_t)c * n_tiles + blockIdx.x] = sc[c];
}

// Inclusive scan of one value per lane across the warp.
__device__ __forceinline__ int warp_inclusive_scan(int x) {
  const unsigned lane = lane_id();
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, off);
    if ((int)lane >= off) x += y;
  }
  return x;
}

// Exclusive scan of n values (smem) by one warp, chunk by chunk; returns the total.
__device__ __forceinline__ int warp_exclusive_scan_smem(const int32_t* in, int32_t* out, int n) {
  const unsigned lane = lane_id();
  int carry = 0;
  for (int i0 = 0; i0 < n; i0 += 32) {
    const int i = i0 + (int)lane;
    const int v = i < n ? in[i] : 0;
    const int inc = warp_inclusive_scan(v);
    if (i < n) out[i] = carry + inc - v;
    carry += __shfl_sync(0xffffffffu, inc, 31);
  }
  return carry;
}

// ---- pass 2 ---------------------------------------------------------------
// One block of 32 warps.  counts[c][tile] becomes the global first row of
// `tile` in column c; sfd_off / epd_off / C_T are written.
__global__ void __launch_bounds__(1024) brim_scan_kernel(int32_t* __restrict__ counts,
                                                        int n_tiles, int E, int R,
                                                        int32_t* __restrict__ sfd_off,
                                                        int32_t* __restrict__ epd_off,
                                                        int32_t* __restrict__ c_t) {
  __shared__ int32_t total[kMaxE * 2];
  __shared__ int32_t colbase[kMaxE * 2];
  const int ncol = R + E;
  const int warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const unsigned lane = lane_id();
  // per column: exclusive scan over its tiles (tile order = token order)
  for (int c = warp; c < ncol; c += nwarps) {
    int32_t* col = counts + (size_t)c * n_tiles;
    int carry = 0;
    for (int b0 = 0; b0 < n_tiles; b0 += 32) {
      const int b = b0 + (int)lane;
      const int n = b < n_tiles ? col[b] : 0;
      const int inc = warp_inclusive_scan(n);
      if (b < n_tiles) col[b] = carry + inc - n;
      carry += __shfl_sync(0xffffffffu, inc, 31);
    }
    if (lane == 0) total[c] = carry;
  }
  __syncthreads();
  // where each rank's SFD segment and each slot's EPD group starts
  if (warp == 0) {
    const int ct = warp_exclusive_scan_smem(total, colbase, R);
    for (int r = lane; r < R; r += 32) sfd_off[r] = colbase[r];
    if (lane == 0) {
      sfd_off[R] = ct;
      *c_t = ct;
    }
  } else if (warp == 1) {
    const int tk = warp_exclusive_scan_smem(total + R, colbase + R, E);
    for (int q = lane; q < E; q += 32) epd_off[q] = colbase[R + q];
    if (lane == 0) epd_off[E] = tk;
  }
  __syncthreads();
  const int n_all = ncol * n_tiles;
  for (int i = threadIdx.x; i < n_all; i += blockDim.x) counts[i] += colbase[i / n_tiles];
}

// ---- pass 3 ---------------------------------------------------------------
__global__ void __launch_bounds__(kBrimTile) brim_scatter_kernel(
    const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_w,
    const int32_t* __restrict__ slot_of, int T, int k, int E, int R, int n_tiles,
    const int32_t* __restrict__ tile_base, int32_t* __restrict__ brim0,
    int32_t* __restrict__ sfd_token, int32_t* __restrict__ brim1,
    int32_t* __restrict__ epd_sfd, float* __restrict__ epd_gate, unsigned* err) {
  __shared__ uint32_t mask[kBrimWarps][kMaxE * 2];  // lanes of warp w that hit column c
  __shared__ int32_t before[kBrimWarps][kMaxE * 2]; // hits in warps < w, plus the tile base
  const int ncol = R + E;
  const int L = E / R;
  const size_t cap = (size_t)T * (k < R ? k : R);
  const int warp = threadIdx.x >> 5;
  const unsigned lane = lane_id();
  for (int i = threadIdx.x; i < kBrimWarps * ncol; i += blockDim.x)
    mask[i / ncol][i % ncol] = 0u;
  __syncthreads();

  const int t = blockIdx.x * kBrimTile + threadIdx.x;
  TokenRoute tr;
  bool ok = false;
  if (t < T) {
    ok = load_token_route(topk_idx, slot_of, t, k, E, L, tr, err);
    if (ok) {
      for (int i = 0; i < tr.n_rank; ++i) atomicOr(&mask[warp][tr.rank[i]], 1u << lane);
      for (int j = 0; j < k; ++j) atomicOr(&mask[warp][R + tr.slot[j]], 1u << lane);
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < ncol; c += blockDim.x) {
    int run = tile_base[(size_t)c * n_tiles + blockIdx.x];
    for (int w = 0; w < kBrimWarps; ++w) {
      before[w][c] = run;
      run += __popc(mask[w][c]);
    }
  }
  __syncthreads();
  if (t >= T) return;

  const uint32_t lt = (1u << lane) - 1u;
  // BRIM_0 column of this token (every rank: a row or -1) and sfd_token
  int s_of_rank[kMaxK];
  for (int r = 0; r < R; ++r) brim0[(size_t)r * T + t] = -1;
  if (!ok) return;
  for (int i = 0; i < tr.n_rank; ++i) {
    const int r = tr.rank[i];
    const int s = before[warp][r] + __popc(mask[warp][r] & lt);
    s_of_rank[i] = s;
    brim0[(size_t)r * T + t] = s;
    sfd_token[s] = t;
    // every local expert of this rank starts as "not selected" for row s
    for (int l = 0; l < L; ++l) brim1[(size_t)l * cap + s] = -1;
  }
  for (int j = 0; j < k; ++j) {
    const int q = tr.slot[j];
    const int r = q / L, l = q - r * L;
    int s = -1;
    for (int i = 0; i < tr.n_rank; ++i)
      if (tr.rank[i] == r) s = s_of_rank[i];
    const int p = before[warp][R + q] + __popc(mask[warp][R + q] & lt);
    brim1[(size_t)l * cap + s] = p;
    epd_sfd[p] = s;
    epd_gate[p] = topk_w[(size_t)t * k + j];
  }
}

// ---- placement-aware dispatched-row counter ------------------------------
__global__ void __launch_bounds__(256) count_dispatched_kernel(
    const int32_t* __restrict__ topk_idx, int T, int k, const int32_t* __restrict__ slot_of,
    int E, int R, int32_t* __restrict__ per_rank, unsigned long long* __restrict__ total,
    unsigned long long* __restrict__ remote, unsigned* err) {
  __shared__ int32_t sc[kMaxE];
  __shared__ unsigned long long s_total, s_remote;
  const int L = E / R;
  for (int r = threadIdx.x; r < R; r += blockDim.x) sc[r] = 0;
  if (threadIdx.x == 0) {
    s_total = 0ull;
    s_remote = 0ull;
  }
  __syncthreads();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t < T) {
    TokenRoute tr;
    if (load_token_route(topk_idx, slot_of, t, k, E, L, tr, err)) {
      const int src = (int)(((long long)t * R) / T);
      int n_remote = 0;
      for (int i = 0; i < tr.n_rank; ++i) {
        atomicAdd(&sc[tr.rank[i]], 1);
        n_remote += (tr.rank[i] != src);
      }
      atomicAdd(&s_total, (unsigned long long)tr.n_rank);
      if (n_remote) atomicAdd(&s_remote, (unsigned long long)n_remote);
    }
  }
  __syncthreads();
  for (int r = threadIdx.x; r < R; r += blockDim.x)
    if (sc[r]) atomicAdd(&per_rank[r], sc[r]);
  if (threadIdx.x == 0) {
    if (s_total) atomicAdd(total, s_total);
    if (s_remote) atomicAdd(remote, s_remote);
  }
}

// ---- expert co-activation histogram --------------------------------------
// Integer atomics, so the result does not depend on the order they land in.
// Small E: a per-block histogram in shared memory flushed once per block.
constexpr int kHistSmemE = 64;
__global__ void __launch_bounds__(256) coact_hist_kernel(const int32_t* __restrict__ topk_idx,
                                                         int T, int k, int E,
                                                         uint32_t* __restrict__ hist,
                                                         unsigned* err) {
  __shared__ uint32_t sh[kHistSmemE * kHistSmemE];
  const bool use_smem = E <= kHistSmemE;
  if (use_smem) {
    for (int i = threadIdx.x; i < E * E; i += blockDim.x) sh[i] = 0u;
    __syncthreads();
  }
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t < T) {
    int ids[kMaxK];
    bool ok = true;
    for (int j = 0; j < k; ++j) {
      ids[j] = topk_idx[(size_t)t * k + j];
      if (ids[j] < 0 || ids[j] >= E) ok = false;
      for (int i = 0; i < j; ++i) ok &= ids[i] != ids[j];
    }
    if (!ok) {
      raise_error(err, kErrIndex);
    } else {
      for (int a = 0; a < k; ++a)
        for (int b = 0; b < k; ++b) {
          const int cell = ids[a] * E + ids[b];
          if (use_smem) atomicAdd(&sh[cell], 1u);
          else atomicAdd(&hist[cell], 1u);
        }
    }
  }
  if (use_smem) {
    __syncthreads();
    for (int i = threadIdx.x; i < E * E; i += blockDim.x)
      if (sh[i]) atomicAdd(&hist[i], sh[i]);
  }
}

}  // namespace moe
