// route_brim.cuh -- routing, the BRIM masks and the dispatched-row counter in
// one kernel (pass 1 of the BRIM build fused with routing).
//
// The same computation as moe_route_topk + brim_mask_kernel +
// moe_count_dispatched_rows: one block of kRouteTileWarps warps per 32-token
// tile.  The warps route the tile's tokens (route_token_warp, the very code of
// moe_route_topk), then every warp takes the tile lane-per-token and builds a
// share of its column masks by ballot; warp 0 writes the top-k (pruned, when
// asked) and adds the tile's contribution to the counter.  The column scan with the histogram (brim_colscan_kernel) and
// the scatter (brim_scatter_kernel) follow.
#pragma once
#include "brim.cuh"
#include "route.cuh"

namespace moe {

constexpr int kRouteTileWarps = 32;  // warps per 32-token tile: one token each

template <int KMAX>
__global__ void __launch_bounds__(32 * kRouteTileWarps) route_brim_tile_kernel(
    const float* __restrict__ logits, int T, int E, int k, int renorm,
    const int32_t* __restrict__ slot_of, int R, int prune_m, int n_tiles,
    int32_t* __restrict__ topk_idx,
    float* __restrict__ topk_w, uint32_t* __restrict__ masks, int32_t* __restrict__ per_rank,
    unsigned long long* __restrict__ total, unsigned long long* __restrict__ remote,
    unsigned* err) {
  pdl_enter();
  __shared__ int s_ids[32][KMAX];
  __shared__ float s_gates[32][KMAX];
  const int warp = threadIdx.x >> 5;
  const unsigned lane = lane_id();
  const int tile = blockIdx.x;
  const int L = E / R, ncol = R + E;

  // 1. warp w routes tokens w, w + kRouteTileWarps, ... of the tile
  for (int i = warp; i < kBrimTileTokens; i += kRouteTileWarps) {
    const int t = tile * kBrimTileTokens + i;
    int id = -1;
    float gate = 0.f;
    if (t < T) route_token_warp(logits + (size_t)t * E, E, k, renorm, &id, &gate);
    if ((int)lane < KMAX) {
      s_ids[i][lane] = (t < T && (int)lane < k) ? id : -1;
      s_gates[i][lane] = (t < T && (int)lane < k) ? gate : 0.f;
    }
  }
  __syncthreads();

  // 2. every warp takes the tile lane-per-token (each builds the same routes);
  //    warp w then makes the column masks c = w, w + kRouteTileWarps, ... by
  //    ballot, and warp 0 writes the top-k and adds the tile to the counter
  const int t = tile * kBrimTileTokens + (int)lane;
  int ids[KMAX];
  float gates[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    ids[j] = s_ids[lane][j];
    gates[j] = s_gates[lane][j];
  }
  if (prune_m > 0 && t < T) prune_token<KMAX>(ids, gates, slot_of, k, E, L, prune_m);
  TokenRoute<KMAX> tr;
  const bool active =
      t < T && make_token_route<KMAX>(ids, slot_of, k, E, L, tr, warp == 0 ? err : nullptr);
  for (int c = warp; c < ncol; c += kRouteTileWarps) {
    bool hit = false;
    if (active) {
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (j < k && tr.slot[j] >= 0) hit |= c < R ? tr.rank[j] == c : tr.slot[j] == c - R;
    }
    const uint32_t m = __ballot_sync(0xffffffffu, hit);
    if (lane == 0) {
      masks[(size_t)c * n_tiles + tile] = m;
      if (per_rank && c < R && m) atomicAdd(&per_rank[c], __popc(m));  // tokens per rank
    }
  }
  if (warp == 0) {
    if (t < T)
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (j < k) {
          topk_idx[(size_t)t * k + j] = ids[j];
          topk_w[(size_t)t * k + j] = gates[j];
        }
    if (per_rank) {
      // rows sent, and the remote ones: ranks other than the token's source
      // rank floor(t * R / T)
      const int src = (int)(((long long)t * R) / (T > 0 ? T : 1));
      unsigned n_rank = 0, n_remote = 0;
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (active && j < k && tr.first[j]) {
          ++n_rank;
          n_remote += tr.rank[j] != src;
        }
      n_rank = __reduce_add_sync(0xffffffffu, n_rank);
      n_remote = __reduce_add_sync(0xffffffffu, n_remote);
      if (lane == 0) {
        if (n_rank) atomicAdd(total, (unsigned long long)n_rank);
        if (n_remote) atomicAdd(remote, (unsigned long long)n_remote);
      }
    }
  }
}

}  // namespace moe
