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
//   2. scan    : one block per column: exclusive scan of popcount(mask) over
//                the tiles, written in place (each tile's first row within
//                the column), and the column's total
//   3. scatter : each warp rebuilds its tile's masks, turns the column totals
//                into column offsets (sfd_off, epd_off, C_T) and finds each
//                lane's row in column c as offset[c] + base[c][tile] +
//                popcount(mask_c & lanes below it)
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

// Builds a token's route from its k expert ids (slot_of in global or shared
// memory; null: the identity placement).  An id of -1 is an empty slot
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
      const int q = (e >= 0 && e < E) ? (slot_of ? slot_of[e] : e) : -1;  // null: identity
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
    rank[j] = (j < k && e >= 0 && e < E) ? slot_of[e] / L : -1;
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

// ---- expert co-activation histogram --------------------------------------
// Integer atomics, so the result does not depend on the order they land in.
// Small E: a per-block histogram in shared memory flushed once per block.
constexpr int kHistSmemE = 64;

// Adds tokens [t0, t1) to the histogram, one thread per token.  With
// E <= kHistSmemE the counts gather in shared memory `sh` first (cleared
// here) and go to global memory once per nonzero cell.  All threads of the
// block must call it.  A token with an out-of-range or repeated id raises the
// index error bit and is skipped; -1 is an empty slot.
template <int KMAX>
__device__ __forceinline__ void coact_hist_range(const int32_t* __restrict__ topk_idx, int t0,
                                                 int t1, int k, int E,
                                                 uint32_t* __restrict__ hist, unsigned* err,
                                                 uint32_t* sh) {
  const bool use_smem = E <= kHistSmemE;
  if (use_smem) {
    for (int i = threadIdx.x; i < E * E; i += blockDim.x) sh[i] = 0u;
    __syncthreads();
  }
  for (int t = t0 + (int)threadIdx.x; t < t1; t += blockDim.x) {
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
      continue;
    }
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
  if (use_smem) {
    __syncthreads();
    for (int i = threadIdx.x; i < E * E; i += blockDim.x)
      if (sh[i]) atomicAdd(&hist[i], sh[i]);
  }
}

// ---- pass 2, parallel ------------------------------------------------------
// Block c scans column c on its own: the popcounts of its n_tiles masks,
// exclusive prefix over the tiles, written to bases[c * n_tiles + tile] (the
// tile's first row WITHIN the column; bases may be the masks themselves) and
// the column total into totals[c].  The scatter (pass 3) adds each column's
// offset among the columns of its kind.  With `own`, each rank column r < R
// also counts its own-rank hits: the tokens t of rank r's own slice of the
// batch, floor(t * R / T) = r, that are sent to rank r.
__device__ __forceinline__ uint32_t lanes_in_range(int tile, long long lo, long long hi) {
  const long long base = (long long)tile * kBrimTileTokens;
  const long long s = lo > base ? lo - base : 0;
  const long long e = hi - base < 32 ? hi - base : 32;
  if (e <= s) return 0u;
  const uint32_t below_e = e == 32 ? 0xffffffffu : ((1u << e) - 1u);
  return below_e & ~((1u << s) - 1u);
}

// Threads per column block: 256 measured 2 us faster than 1024 on the OLMoE-shaped
// index path (T = 4096: one tile per thread against eight) and the same on the
// correlated prefill (T = 32768); 32 was slower on both large batches.
constexpr int kColscanThreads = 256;

__global__ void __launch_bounds__(kColscanThreads) brim_colscan_kernel(
    const uint32_t* masks, uint32_t* bases, int n_tiles, int ncol, int32_t* __restrict__ totals,
    int T, int R, int32_t* __restrict__ own) {
  pdl_enter();
  __shared__ int32_t warp_sums[32];
  __shared__ int32_t s_own;
  const int c = blockIdx.x;
  const uint32_t* col = masks + (size_t)c * n_tiles;
  uint32_t* out = bases + (size_t)c * n_tiles;
  const int per = (n_tiles + blockDim.x - 1) / blockDim.x;  // tiles per thread
  const int b0 = threadIdx.x * per, b1 = min(b0 + per, n_tiles);
  const bool count_own = own != nullptr && c < R;
  long long lo = 0, hi = 0;  // rank c's own tokens: [lo, hi)
  if (count_own) {
    lo = ((long long)c * T + R - 1) / R;
    hi = ((long long)(c + 1) * T + R - 1) / R;
  }
  int sum = 0, mine = 0;
  for (int b = b0; b < b1; ++b) {
    const uint32_t m = col[b];
    sum += __popc(m);
    if (count_own) mine += __popc(m & lanes_in_range(b, lo, hi));
  }
  // block-wide exclusive scan of the per-thread sums
  const int warp = threadIdx.x >> 5, lane = (int)lane_id();
  const int inc = warp_inclusive_scan(sum);
  if (lane == 31) warp_sums[warp] = inc;
  if (threadIdx.x == 0) s_own = 0;
  __syncthreads();
  if (count_own) {
    mine = __reduce_add_sync(0xffffffffu, mine);
    if (lane == 0 && mine) atomicAdd(&s_own, mine);
  }
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    const int v = lane < nw ? warp_sums[lane] : 0;
    const int winc = warp_inclusive_scan(v);
    if (lane < nw) warp_sums[lane] = winc - v;
    if (lane == nw - 1) totals[c] = winc;
  }
  __syncthreads();
  if (count_own && threadIdx.x == 0) own[c] = s_own;
  int base = warp_sums[warp] + inc - sum;
  for (int b = b0; b < b1; ++b) {
    const int n = __popc(col[b]);
    out[b] = (uint32_t)base;
    base += n;
  }
}

// ---- co-activation histogram from the slot masks -----------------------------
// hist[a][b] += the number of tokens routed to both experts a and b: the sum
// over the tiles of popcount(mask(a) & mask(b)), mask(e) being the column of
// e's slot.  The masks hold exactly the tokens with a valid route, without
// their empty (pruned) slots, so this is the count coact_hist_range makes
// from the ids.  One block per chunk of hist_chunk_tiles(E) tiles: it stages
// the chunk's E columns in shared memory, tile-major and by expert id, sums
// every cell over the chunk and adds the nonzero sums to hist, one atomic
// per cell per chunk.
constexpr int kHistMaxChunk = 8;
__host__ __device__ constexpr int hist_chunk_tiles(int E) {
  return E <= 128 ? kHistMaxChunk : kHistMaxChunk / 2;
}
constexpr int kHistStageWords = kHistMaxChunk * 128;  // chunk tiles x E, for every E <= kMaxE

__device__ __forceinline__ void coact_hist_chunk_from_masks(
    const uint32_t* __restrict__ masks, int n_tiles, int R, int E,
    const int32_t* __restrict__ slot_of, int chunk, uint32_t* __restrict__ hist,
    uint32_t* stage) {
  const int ct = hist_chunk_tiles(E);
  const int tile0 = chunk * ct;
  for (int i = threadIdx.x; i < E * ct; i += blockDim.x) {
    const int e = i / ct, t = i % ct;
    const int q = slot_of ? __ldg(slot_of + e) : e;
    stage[t * E + e] = tile0 + t < n_tiles ? masks[(size_t)(R + q) * n_tiles + tile0 + t] : 0u;
  }
  __syncthreads();
  // tpr threads per row a: row a's chunk in registers, the b columns read
  // from shared memory (a warp reads at most tpr distinct words per load)
  const int nt = blockDim.x;
  const int tpr = nt >= E ? nt / E : 1;
  const int rows = nt / tpr;
  const int sub = threadIdx.x % tpr;
  for (int a = threadIdx.x / tpr; a < E; a += rows) {
    uint32_t ra[kHistMaxChunk];
#pragma unroll
    for (int t = 0; t < kHistMaxChunk; ++t) ra[t] = t < ct ? stage[t * E + a] : 0u;
    for (int b = sub; b < E; b += tpr) {
      int n = 0;
#pragma unroll
      for (int t = 0; t < kHistMaxChunk; ++t)
        if (t < ct) n += __popc(ra[t] & stage[t * E + b]);
      if (n) atomicAdd(&hist[(size_t)a * E + b], (uint32_t)n);
    }
  }
}

// ---- pass 3 ---------------------------------------------------------------
// One block of kScatterWarps warps per tile.  Warp 0 rebuilds the tile's
// masks and the tile's first row in every column; then warp w walks the
// ranks r = w, w + kScatterWarps, ... and, inside each, the rank's local
// experts l, so that for one column the lanes that hit it hold consecutive
// rows: every store of a warp lands on consecutive addresses.
//   BRIM_0[r][t] = s (or -1), sfd_token[s] = t
//   BRIM_1[l][s] = p (or -1 for a local expert the token did not pick), for
//                  all l of each rank the token reaches
//   epd_sfd[p] = s, epd_gate[p] = the token's gate weight for that expert
//
// tile_base holds each tile's first row within each column (pass 2); warp 0
// adds the column offsets -- the exclusive scans of the column totals over
// the R rank columns and over the E slot columns -- and tile 0 writes
// sfd_off, epd_off and C_T.  Every global load a block needs before its
// stores is issued first, slot_of staged in shared memory among them, so a
// block waits on one load round trip before it computes.
//
// BrimExtras adds, in the fused index path, the dispatched-row counter and
// the co-activation histogram to the same launch:
//   * tile 0 writes per_rank (the rank columns' totals), total (C_T) and
//     remote (C_T less the own-rank hits that pass 2 counted);
//   * blocks 0 .. n_hist - 1 come before the tiles and each add one chunk of
//     tiles to the histogram from the slot masks, which must then still be
//     intact (pass 2 writing its bases elsewhere).
constexpr int kScatterWarps = 4;

struct BrimExtras {
  int32_t* per_rank;             // [R], or null: no counter
  unsigned long long* total;     // rows sent, C_T
  unsigned long long* remote;    // rows sent to a rank other than the token's source
  const int32_t* own;            // [R] own-rank hits (pass 2)
  uint32_t* hist;                // [E, E], accumulated; or null
  const uint32_t* masks;         // the slot masks (pass 1), for the histogram rows
  int n_hist;                    // tile chunks (hist_chunk_tiles) when hist is given, else 0
};

template <int KMAX>
__global__ void __launch_bounds__(32 * kScatterWarps) brim_scatter_kernel(
    const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_w,
    const int32_t* __restrict__ slot_of, int T, int k, int E, int R, int n_tiles,
    const int32_t* __restrict__ tile_base, const int32_t* __restrict__ totals,
    int32_t* __restrict__ sfd_off, int32_t* __restrict__ epd_off, int32_t* __restrict__ c_t,
    int32_t* __restrict__ brim0, int32_t* __restrict__ sfd_token, int32_t* __restrict__ brim1,
    int32_t* __restrict__ epd_sfd, float* __restrict__ epd_gate, BrimExtras x) {
  pdl_enter();
  // the histogram's staging and the tile's arrays share one buffer
  static_assert(kHistStageWords <= 4 * kMaxCols, "staging fits the scatter's arrays");
  __shared__ uint32_t s_buf[4 * kMaxCols];
  if ((int)blockIdx.x < x.n_hist) {
    coact_hist_chunk_from_masks(x.masks, n_tiles, R, E, slot_of, (int)blockIdx.x, x.hist, s_buf);
    return;
  }
  uint32_t* sm = s_buf;
  int32_t* sb = reinterpret_cast<int32_t*>(s_buf + kMaxCols);
  int32_t* s_tot = reinterpret_cast<int32_t*>(s_buf + 2 * kMaxCols);
  int32_t* s_off = reinterpret_cast<int32_t*>(s_buf + 3 * kMaxCols);
  const int tile = (int)blockIdx.x - x.n_hist;
  const int warp = threadIdx.x >> 5;
  const int ncol = R + E, L = E / R;
  const size_t cap = (size_t)T * (k < R ? k : R);
  const unsigned lane = lane_id();
  const int t = tile * kBrimTileTokens + (int)lane;
  __shared__ int32_t s_slot[kMaxE];
  int ids[KMAX];
  float gw[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    const bool in = t < T && j < k;
    ids[j] = in ? __ldg(topk_idx + (size_t)t * k + j) : -1;
    gw[j] = in && topk_w ? __ldg(topk_w + (size_t)t * k + j) : 1.f;
  }
  if (warp == 0) {
    // the first 128 columns' loads all issue before any of them is stored
    int32_t tot[4], base[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int c = lane + 32 * i;
      tot[i] = c < ncol ? totals[c] : 0;
      base[i] = c < ncol ? tile_base[(size_t)c * n_tiles + tile] : 0;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int c = lane + 32 * i;
      if (c < ncol) {
        s_tot[c] = tot[i];
        sb[c] = base[i];
      }
    }
    for (int c = lane + 128; c < ncol; c += 32) {
      s_tot[c] = totals[c];
      sb[c] = tile_base[(size_t)c * n_tiles + tile];
    }
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_slot[e] = slot_of ? __ldg(slot_of + e) : e;
  __syncthreads();  // s_slot
  TokenRoute<KMAX> tr;
  // the error flag was raised by pass 1 already
  const bool active = t < T && make_token_route<KMAX>(ids, s_slot, k, E, L, tr, nullptr);
  float gate[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) gate[j] = (active && j < k && tr.slot[j] >= 0) ? gw[j] : 0.f;
  if (warp == 0) {
    tile_masks<KMAX>(sm, ncol, R, active, k, tr);
    // the tile's first global row in every column
    const int ct = warp_exclusive_scan_smem(s_tot, s_off, R);
    const int tk = warp_exclusive_scan_smem(s_tot + R, s_off + R, E);
    __syncwarp();
    for (int c = lane; c < ncol; c += 32) sb[c] += s_off[c];
    if (tile == 0) {
      for (int r = lane; r < R; r += 32) sfd_off[r] = s_off[r];
      for (int q = lane; q < E; q += 32) epd_off[q] = s_off[R + q];
      if (lane == 0) {
        sfd_off[R] = ct;
        epd_off[E] = tk;
        *c_t = ct;
      }
      if (x.per_rank) {
        int o = 0;
        for (int r = lane; r < R; r += 32) {
          x.per_rank[r] = s_tot[r];
          o += x.own[r];
        }
        o = __reduce_add_sync(0xffffffffu, o);
        if (lane == 0) {
          *x.total = (unsigned long long)ct;
          *x.remote = (unsigned long long)(ct - o);
        }
      }
    }
  }
  __syncthreads();
  const uint32_t lt = (1u << lane) - 1u;
  for (int r = warp; r < R; r += kScatterWarps) {
    const uint32_t mr = sm[r];
    const int s = ((mr >> lane) & 1u) ? sb[r] + __popc(mr & lt) : -1;
    if (t < T) brim0[(size_t)r * T + t] = s;
    if (mr == 0u) continue;  // no token of the tile reaches rank r (warp-uniform)
    if (s >= 0) sfd_token[s] = t;
    for (int l = 0; l < L; ++l) {
      const int q = r * L + l;
      const uint32_t mq = sm[R + q];
      int p = -1;
      float g = 0.f;
      if ((mq >> lane) & 1u) {
        p = sb[R + q] + __popc(mq & lt);
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
          if (j < k && tr.slot[j] == q) g = gate[j];
      }
      if (s >= 0) brim1[(size_t)l * cap + s] = p;
      if (p >= 0) {
        epd_sfd[p] = s;
        epd_gate[p] = g;
      }
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

template <int KMAX>
__global__ void __launch_bounds__(256) coact_hist_kernel(const int32_t* __restrict__ topk_idx,
                                                         int T, int k, int E,
                                                         uint32_t* __restrict__ hist,
                                                         unsigned* err) {
  pdl_enter();
  __shared__ uint32_t sh[kHistSmemE * kHistSmemE];
  const int t0 = blockIdx.x * blockDim.x;
  coact_hist_range<KMAX>(topk_idx, t0, min(T, t0 + (int)blockDim.x), k, E, hist, err, sh);
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
