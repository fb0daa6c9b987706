// route_brim.cuh -- routing, the BRIM masks and the dispatched-row counter in
// one kernel (pass 1 of the BRIM build fused with routing).
//
// The same computation as moe_route_topk + brim_mask_kernel +
// moe_count_dispatched_rows: one block of 16 warps per 32-token tile.  Each
// warp routes two tokens (route_token_warp_v, the very code of moe_route_topk);
// warp 0 then takes the tile lane-per-token, prunes (when asked), writes the
// top-k, builds the tile's column masks and adds the tile's contribution to
// the counter.  The column scan with the histogram (brim_colscan_kernel) and
// the scatter (brim_scatter_kernel) follow.
#pragma once
#include "brim.cuh"
#include "route.cuh"

namespace moe {

// Tokens each warp routes (its logits loaded together up front): the block is
// 32 / kRouteTokensPerWarp warps, so two blocks fit on an SM and one block's
// tile work overlaps another's routing.
constexpr int kRouteTokensPerWarp = 2;
constexpr int kRouteTileThreads = 32 * (kBrimTileTokens / kRouteTokensPerWarp);

template <int KMAX>
__global__ void __launch_bounds__(kRouteTileThreads, 2) route_brim_tile_kernel(
    const float* __restrict__ logits, int T, int E, int k, int renorm,
    const int32_t* __restrict__ slot_of, int R, int prune_m, int n_tiles,
    int32_t* __restrict__ topk_idx,
    float* __restrict__ topk_w, uint32_t* __restrict__ masks, int32_t* __restrict__ per_rank,
    unsigned long long* __restrict__ total, unsigned long long* __restrict__ remote,
    unsigned* err) {
  pdl_enter();
  __shared__ int s_ids[32][KMAX];
  __shared__ float s_gates[32][KMAX];
  __shared__ uint32_t s_mask[kMaxCols];
  const int warp = threadIdx.x >> 5;
  const unsigned lane = lane_id();
  const int tile = blockIdx.x;
  const int L = E / R, ncol = R + E;

  // 1. warp w routes tokens w, w + 16 of the tile (both rows' logits loaded first)
  {
    constexpr int kWarps = kRouteTileThreads / 32;
    float v[kRouteTokensPerWarp][kRouteMaxPerLane];
#pragma unroll
    for (int u = 0; u < kRouteTokensPerWarp; ++u) {
      const int t = tile * kBrimTileTokens + warp + u * kWarps;
      if (t < T) load_token_logits(logits + (size_t)t * E, E, v[u]);
    }
#pragma unroll
    for (int u = 0; u < kRouteTokensPerWarp; ++u) {
      const int i = warp + u * kWarps;
      const int t = tile * kBrimTileTokens + i;
      int id = -1;
      float gate = 0.f;
      if (t < T) route_token_warp_v(v[u], E, k, renorm, &id, &gate);
      if ((int)lane < KMAX) {
        s_ids[i][lane] = (t < T && (int)lane < k) ? id : -1;
        s_gates[i][lane] = (t < T && (int)lane < k) ? gate : 0.f;
      }
    }
  }
  __syncthreads();

  // 2. warp 0, one lane per token: pruning, top-k out, masks, counter
  if (warp == 0) {
    const int t = tile * kBrimTileTokens + (int)lane;
    int ids[KMAX];
    float gates[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      ids[j] = s_ids[lane][j];
      gates[j] = s_gates[lane][j];
    }
    if (prune_m > 0 && t < T) prune_token<KMAX>(ids, gates, slot_of, k, E, L, prune_m);
    if (t < T)
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (j < k) {
          topk_idx[(size_t)t * k + j] = ids[j];
          topk_w[(size_t)t * k + j] = gates[j];
        }
    TokenRoute<KMAX> tr;
    const bool active = t < T && make_token_route<KMAX>(ids, slot_of, k, E, L, tr, err);
    tile_masks<KMAX>(s_mask, ncol, R, active, k, tr);
    for (int c = lane; c < ncol; c += 32) masks[(size_t)c * n_tiles + tile] = s_mask[c];
    if (per_rank) {
      // tokens per rank: popcount of the rank columns; remote: ranks other than
      // the token's source rank floor(t * R / T)
      for (int r = lane; r < R; r += 32) {
        const int n = __popc(s_mask[r]);
        if (n) atomicAdd(&per_rank[r], n);
      }
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
