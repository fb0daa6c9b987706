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
// every expert group), which makes them unique.  Tokens are taken in tiles of
// 32, one warp per tile and one lane per token.  A "column" is a rank (c < R)
// or an expert slot (c = R + q).
//   1. mask    : per tile and column, the 32-bit mask of lanes that hit it
//   2. scan    : per column, exclusive scan of popcount(mask) over the tiles;
//                column totals give sfd_off, epd_off and C_T; the masks are
//                replaced in place by each tile's first global row
//   3. scatter : each lane rebuilds its tile's masks and finds its row in
//                column c as base[c][tile] + popcount(mask_c & lanes below it)
// No pass depends on the order in which atomics land.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kBrimTileTokens = 32;  // one warp
constexpr int kMaxK = 16;
constexpr int kMaxE = 256;
constexpr int kMaxCols = 2 * kMaxE;

// One token's experts, as slots, with their ranks; `first[j]` marks the first
// expert of each distinct rank.  KMAX is a compile-time bound on k so that
// every array lives in registers.
template <int KMAX>
struct TokenRoute {
  int slot[KMAX];
  int rank[KMAX];
  bool first[KMAX];
};

// Builds a token's route from its k expert ids.  An id of -1 is an empty slot
// (a pruned assignment): it is sent nowhere and is not an error.  Returns
// false (and raises the error flag) when an id is otherwise out of range or
// repeated; such a token is sent nowhere.
template <int KMAX>
__device__ __forceinline__ bool make_token_route(const int (&ids)[KMAX],
                                                 const int32_t* __restrict__ slot_of, int k,
                                                 int E, int L, TokenRoute<KMAX>& tr,
                                                 unsigned* err) {
  bool ok = true;
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    tr.slot[j] = -1;
    tr.rank[j] = -1;
    if (j < k && ids[j] != -1) {
      const int e = ids[j];
      const int q = (e >= 0 && e < E) ? __ldg(slot_of + e) : -1;
      if (q < 0 || q >= E) ok = false;
      tr.slot[j] = q;
      tr.rank[j] = q >= 0 ? q / L : -1;
    }
  }
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    bool first = j < k && tr.slot[j] >= 0;
#pragma unroll
    for (int i = 0; i < j; ++i) {
      if (j < k && tr.slot[j] >= 0 && tr.slot[i] >= 0) {  // empty slots compare with nothing
        if (tr.slot[i] == tr.slot[j]) ok = false;         // the same expert twice
        if (tr.rank[i] == tr.rank[j]) first = false;
      }
    }
    tr.first[j] = first;
  }
  if (!ok && err) raise_error(err, kErrIndex);
  return ok;
}

// Routing-score-based collaboration pruning of one token (in registers): keep
// the first m distinct ranks met along the descending-score list, empty every
// slot on another rank, and rescale the kept gates to the original sum.
template <int KMAX>
__device__ __forceinline__ void prune_token(int (&ids)[KMAX], float (&gates)[KMAX],
                                            const int32_t* __restrict__ slot_of, int k, int E,
                                            int L, int m) {
  int rank[KMAX];
  bool keep[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    const int e = ids[j];
    rank[j] = (j < k && e >= 0 && e < E) ? __ldg(slot_of + e) / L : -1;
  }
  int n_kept_ranks = 0;
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    keep[j] = false;
    if (rank[j] < 0) continue;
    bool seen = false, seen_kept = false;
#pragma unroll
    for (int i = 0; i < j; ++i)
      if (rank[i] == rank[j]) {
        seen = true;
        seen_kept |= keep[i];
      }
    if (!seen && n_kept_ranks < m) {
      keep[j] = true;
      ++n_kept_ranks;
    } else if (seen) {
      keep[j] = seen_kept;
    }
  }
  float before = 0.f, kept = 0.f;
#pragma unroll
  for (int j = 0; j < KMAX; ++j)
    if (j < k) {
      before += gates[j];
      if (keep[j]) kept += gates[j];
    }
  const float scale = kept > 0.f ? before / kept : 0.f;
#pragma unroll
  for (int j = 0; j < KMAX; ++j)
    if (j < k) {
      if (keep[j]) {
        gates[j] *= scale;
      } else if (rank[j] >= 0) {
        ids[j] = -1;
        gates[j] = 0.f;
      }
    }
}

// Loads token t's k expert ids from topk_idx and builds its route.
template <int KMAX>
__device__ __forceinline__ bool load_token_route(const int32_t* __restrict__ topk_idx,
                                                 const int32_t* __restrict__ slot_of, int t,
                                                 int k, int E, int L, TokenRoute<KMAX>& tr,
                                                 unsigned* err) {
  int ids[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) ids[j] = j < k ? __ldg(topk_idx + (size_t)t * k + j) : -1;
  return make_token_route<KMAX>(ids, slot_of, k, E, L, tr, err);
}

// Build this warp's tile masks in shared memory (mask[c], ncol entries).
template <int KMAX>
__device__ __forceinline__ void tile_masks(uint32_t* mask, int ncol, int R, bool active, int k,
                                           const TokenRoute<KMAX>& tr) {
  const unsigned lane = lane_id();
  for (int c = lane; c < ncol; c += 32) mask[c] = 0u;
  __syncwarp();
  if (active) {
    const uint32_t bit = 1u << lane;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j < k && tr.slot[j] >= 0) {
        atomicOr(&mask[R + tr.slot[j]], bit);
        if (tr.first[j]) atomicOr(&mask[tr.rank[j]], bit);
      }
    }
  }
  __syncwarp();
}

// ---- pass 1 ---------------------------------------------------------------
// masks[c * n_tiles + tile]
template <int KMAX>
__global__ void __launch_bounds__(128) brim_mask_kernel(const int32_t* __restrict__ topk_idx,
                                                        const int32_t* __restrict__ slot_of,
                                                        int T, int k, int E, int R, int n_tiles,
                                                        uint32_t* __restrict__ masks,
                                                        unsigned* err) {
  pdl_enter();
  __shared__ uint32_t sm[4][kMaxCols];
  const int w = threadIdx.x >> 5;
  const int tile = blockIdx.x * 4 + w;
  if (tile >= n_tiles) return;
  const int ncol = R + E, L = E / R;
  const unsigned lane = lane_id();
  const int t = tile * kBrimTileTokens + (int)lane;
  TokenRoute<KMAX> tr;
  const bool active = t < T && load_token_route<KMAX>(topk_idx, slot_of, t, k, E, L, tr, err);
  tile_masks<KMAX>(sm[w], ncol, R, active, k, tr);
  for (int c = lane; c < ncol; c += 32) masks[(size_t)c * n_tiles + tile] = sm[w][c];
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

// Exclusive scan of n values (smem) by one warp; returns the total.
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
// One block of 32 warps.  Each warp scans whole columns: lane i sums a
// contiguous run of tiles, a warp scan orders the runs, each lane writes its
// run's bases.  The mask words are replaced by the tile's first global row.
// Reads go to L2 (ld.cg): the masks may have been written by other blocks of
// the same grid.
__device__ __forceinline__ void scan_columns(uint32_t* __restrict__ masks, int n_tiles, int E,
                                             int R, int32_t* __restrict__ sfd_off,
                                             int32_t* __restrict__ epd_off,
                                             int32_t* __restrict__ c_t, int32_t* total,
                                             int32_t* colbase) {
  const int ncol = R + E;
  const int warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const unsigned lane = lane_id();
  const int run = (n_tiles + 31) / 32;  // tiles per lane
  for (int c = warp; c < ncol; c += nwarps) {
    uint32_t* col = masks + (size_t)c * n_tiles;
    const int b0 = (int)lane * run;
    const int b1 = min(b0 + run, n_tiles);
    int sum = 0;
#pragma unroll 8
    for (int b = b0; b < b1; ++b) sum += __popc(__ldcg(col + b));
    const int inc = warp_inclusive_scan(sum);
    int base = inc - sum;
    for (int b = b0; b < b1; ++b) {
      const int n = __popc(__ldcg(col + b));
      col[b] = (uint32_t)base;
      base += n;
    }
    if (lane == 31) total[c] = inc;
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
  for (int i = threadIdx.x; i < n_all; i += blockDim.x)
    masks[i] = (uint32_t)((int32_t)masks[i] + colbase[i / n_tiles]);
}

__global__ void __launch_bounds__(1024) brim_scan_kernel(uint32_t* __restrict__ masks,
                                                        int n_tiles, int E, int R,
                                                        int32_t* __restrict__ sfd_off,
                                                        int32_t* __restrict__ epd_off,
                                                        int32_t* __restrict__ c_t) {
  pdl_enter();
  __shared__ int32_t total[kMaxCols];
  __shared__ int32_t colbase[kMaxCols];
  scan_columns(masks, n_tiles, E, R, sfd_off, epd_off, c_t, total, colbase);
}

// ---- pass 3 ---------------------------------------------------------------
template <int KMAX>
__global__ void __launch_bounds__(128) brim_scatter_kernel(
    const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_w,
    const int32_t* __restrict__ slot_of, int T, int k, int E, int R, int n_tiles,
    const int32_t* __restrict__ tile_base, int32_t* __restrict__ brim0,
    int32_t* __restrict__ sfd_token, int32_t* __restrict__ brim1,
    int32_t* __restrict__ epd_sfd, float* __restrict__ epd_gate) {
  pdl_enter();
  __shared__ uint32_t sm[4][kMaxCols];
  const int w = threadIdx.x >> 5;
  const int tile = blockIdx.x * 4 + w;
  if (tile >= n_tiles) return;
  const int ncol = R + E, L = E / R;
  const size_t cap = (size_t)T * (k < R ? k : R);
  const unsigned lane = lane_id();
  const int t = tile * kBrimTileTokens + (int)lane;
  TokenRoute<KMAX> tr;
  // the error flag was raised by pass 1 already
  const bool active = t < T && load_token_route<KMAX>(topk_idx, slot_of, t, k, E, L, tr, nullptr);
  tile_masks<KMAX>(sm[w], ncol, R, active, k, tr);
  if (t >= T) return;
  for (int r = 0; r < R; ++r) brim0[(size_t)r * T + t] = -1;
  if (!active) return;
  const uint32_t lt = (1u << lane) - 1u;
  const int32_t* base = tile_base + tile;  // base[c] at base[c * n_tiles]
  int s_of[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    s_of[j] = -1;
    if (j < k && tr.first[j]) {
      const int r = tr.rank[j];
      s_of[j] = __ldg(base + (size_t)r * n_tiles) + __popc(sm[w][r] & lt);
    }
  }
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    if (j < k && tr.first[j]) {
      const int s = s_of[j];
      brim0[(size_t)tr.rank[j] * T + t] = s;
      sfd_token[s] = t;
      // every local expert of this rank starts as "not selected" for row s
      for (int l = 0; l < L; ++l) brim1[(size_t)l * cap + s] = -1;
    }
  }
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    if (j < k && tr.slot[j] >= 0) {
      const int q = tr.slot[j];
      int s = -1;
#pragma unroll
      for (int i = 0; i <= j; ++i)
        if (tr.first[i] && tr.rank[i] == tr.rank[j]) s = s_of[i];
      const int p = __ldg(base + (size_t)(R + q) * n_tiles) + __popc(sm[w][R + q] & lt);
      brim1[(size_t)(q - tr.rank[j] * L) * cap + s] = p;
      epd_sfd[p] = s;
      epd_gate[p] = __ldg(topk_w + (size_t)t * k + j);
    }
  }
}

// ---- placement-aware dispatched-row counter ------------------------------
// Warp-aggregated: lanes holding the same rank are merged with match.any
// before one shared atomic; totals are warp-reduced before one global atomic.
template <int KMAX>
__global__ void __launch_bounds__(256) count_dispatched_kernel(
    const int32_t* __restrict__ topk_idx, int T, int k, const int32_t* __restrict__ slot_of,
    int E, int R, int32_t* __restrict__ per_rank, unsigned long long* __restrict__ total,
    unsigned long long* __restrict__ remote, unsigned* err) {
  pdl_enter();
  __shared__ int32_t sc[kMaxE];
  __shared__ unsigned s_total, s_remote;
  const int L = E / R;
  for (int r = threadIdx.x; r < R; r += blockDim.x) sc[r] = 0;
  if (threadIdx.x == 0) {
    s_total = 0u;
    s_remote = 0u;
  }
  __syncthreads();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  TokenRoute<KMAX> tr;
  const bool active = t < T && load_token_route<KMAX>(topk_idx, slot_of, t, k, E, L, tr, err);
  const int src = (int)(((long long)t * R) / (T > 0 ? T : 1));
  unsigned n_rank = 0, n_remote = 0;
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    const int r = (active && j < k && tr.first[j]) ? tr.rank[j] : -1;
    if (r >= 0) {
      ++n_rank;
      n_remote += (r != src);
    }
    const unsigned same = __match_any_sync(0xffffffffu, r);
    if (r >= 0 && (int)lane_id() == __ffs(same) - 1) atomicAdd(&sc[r], __popc(same));
  }
  n_rank = __reduce_add_sync(0xffffffffu, n_rank);
  n_remote = __reduce_add_sync(0xffffffffu, n_remote);
  if (lane_id() == 0) {
    atomicAdd(&s_total, n_rank);
    atomicAdd(&s_remote, n_remote);
  }
  __syncthreads();
  for (int r = threadIdx.x; r < R; r += blockDim.x)
    if (sc[r]) atomicAdd(&per_rank[r], sc[r]);
  if (threadIdx.x == 0) {
    if (s_total) atomicAdd(total, (unsigned long long)s_total);
    if (s_remote) atomicAdd(remote, (unsigned long long)s_remote);
  }
}

// ---- expert co-activation histogram --------------------------------------
// Integer atomics, so the result does not depend on the order they land in.
// Small E: a per-block histogram in shared memory flushed once per block.
constexpr int kHistSmemE = 64;
template <int KMAX>
__global__ void __launch_bounds__(256) coact_hist_kernel(const int32_t* __restrict__ topk_idx,
                                                         int T, int k, int E,
                                                         uint32_t* __restrict__ hist,
                                                         unsigned* err) {
  pdl_enter();
  __shared__ uint32_t sh[kHistSmemE * kHistSmemE];
  const bool use_smem = E <= kHistSmemE;
  if (use_smem) {
    for (int i = threadIdx.x; i < E * E; i += blockDim.x) sh[i] = 0u;
    __syncthreads();
  }
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t < T) {
    int ids[KMAX];
    bool ok = true;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      ids[j] = 0;
      if (j < k) {
        ids[j] = __ldg(topk_idx + (size_t)t * k + j);
        if (ids[j] != -1 && (ids[j] < 0 || ids[j] >= E)) ok = false;
#pragma unroll
        for (int i = 0; i < j; ++i) ok &= ids[j] == -1 || ids[i] != ids[j];
      }
    }
    if (!ok) {
      raise_error(err, kErrIndex);
    } else {
#pragma unroll
      for (int a = 0; a < KMAX; ++a)
#pragma unroll
        for (int b = 0; b < KMAX; ++b)
          if (a < k && b < k && ids[a] >= 0 && ids[b] >= 0) {
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

// ---- collaboration pruning, in place ----------------------------------------
template <int KMAX>
__global__ void __launch_bounds__(256) prune_kernel(int32_t* __restrict__ topk_idx,
                                                    float* __restrict__ topk_w, int T, int k,
                                                    const int32_t* __restrict__ slot_of, int E,
                                                    int R, int m) {
  pdl_enter();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  int ids[KMAX];
  float gates[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    ids[j] = j < k ? topk_idx[(size_t)t * k + j] : -1;
    gates[j] = j < k ? topk_w[(size_t)t * k + j] : 0.f;
  }
  prune_token<KMAX>(ids, gates, slot_of, k, E, E / R, m);
#pragma unroll
  for (int j = 0; j < KMAX; ++j)
    if (j < k) {
      topk_idx[(size_t)t * k + j] = ids[j];
      topk_w[(size_t)t * k + j] = gates[j];
    }
}

}  // namespace moe
