// route_brim.cuh -- routing and the BRIM masks in one kernel (pass 1 of the
// BRIM build fused with routing).
//
// The same computation as moe_route_topk + brim_mask_kernel.  Tokens are
// routed by groups of G lanes (route_token_group, the very code of
// moe_route_topk; G from the batch size, the result does not depend on it).
// Then one warp per 32-token tile, one lane per token, prunes (when asked),
// writes the top-k and builds the tile's column masks.  With G = 1 a lane
// keeps its own token throughout; with G > 1 the routes pass through shared
// memory.  The column scan (brim_colscan_kernel) and the scatter
// (brim_scatter_kernel) follow; the dispatched-row counter and the
// co-activation histogram come out of those two from the masks.
#pragma once
#include "brim.cuh"
#include "route.cuh"

namespace moe {

// threads per block and 32-token tiles per block for G lanes per token: 256
// threads (8 / G tiles) measured 2 us faster than 128 on the correlated prefill
// (T = 32768, G = 2) and the same elsewhere
template <int G>
struct RouteTile {
  static constexpr int kThreads = 256;
  static constexpr int kTiles = kThreads / (32 * G);
};

template <int KMAX>
__device__ __forceinline__ void route_tile_masks(
    int t, int tile, int T, int E, int k, int R, int prune_m, int n_tiles,
    const int32_t* __restrict__ slot_of, int (&ids)[KMAX], float (&gates)[KMAX],
    uint32_t* s_mask, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
    uint32_t* __restrict__ masks, unsigned* err) {
  const unsigned lane = lane_id();
  const int L = E / R, ncol = R + E;
  if (t < T) {
    if (prune_m > 0) prune_token<KMAX>(ids, gates, slot_of, k, E, L, prune_m);
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (j < k) {
        topk_idx[(size_t)t * k + j] = ids[j];
        topk_w[(size_t)t * k + j] = gates[j];
      }
  }
  TokenRoute<KMAX> tr;
  const bool active = t < T && make_token_route<KMAX>(ids, slot_of, k, E, L, tr, err);
  tile_masks<KMAX>(s_mask, ncol, R, active, k, tr);
  for (int c = lane; c < ncol; c += 32) masks[(size_t)c * n_tiles + tile] = s_mask[c];
}

template <int KMAX, int G>
__global__ void __launch_bounds__(RouteTile<G>::kThreads) route_brim_tile_kernel(
    const float* __restrict__ logits, int T, int E, int k, int renorm,
    const int32_t* __restrict__ slot_of, int R, int prune_m, int n_tiles,
    int32_t* __restrict__ topk_idx,
    float* __restrict__ topk_w, uint32_t* __restrict__ masks, unsigned* err) {
  pdl_enter();
  constexpr int kTiles = RouteTile<G>::kTiles;
  __shared__ uint32_t s_mask[kTiles][kMaxCols];
  // With G > 1, slot_of is staged in shared memory while the tokens are
  // routed (the block's barrier follows the routing); with G = 1 the warps
  // never meet, so they read it from global memory.
  __shared__ int32_t s_slot[G > 1 ? kMaxE : 1];
  if constexpr (G > 1)
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_slot[e] = __ldg(slot_of + e);
  const int w = threadIdx.x >> 5;
  const unsigned lane = lane_id();
  int ids[KMAX];
  float gates[KMAX];
  if constexpr (G == 1) {
    // a lane per token from routing to masks
    const int tile = blockIdx.x * kTiles + w;
    if (tile >= n_tiles) return;
    const int t = tile * kBrimTileTokens + (int)lane;
    route_token_group<KMAX, 1>(logits + (size_t)(t < T ? t : 0) * E, t < T, E, k, renorm, ids,
                               gates);
    route_tile_masks<KMAX>(t, tile, T, E, k, R, prune_m, n_tiles, slot_of, ids, gates, s_mask[w],
                           topk_idx, topk_w, masks, err);
  } else {
    __shared__ int s_ids[kTiles * kBrimTileTokens][KMAX];
    __shared__ float s_gates[kTiles * kBrimTileTokens][KMAX];
    const int tok = threadIdx.x / G;  // this group's token within the block
    const int t0 = blockIdx.x * kTiles * kBrimTileTokens;
    const int t = t0 + tok;
    route_token_group<KMAX, G>(logits + (size_t)(t < T ? t : 0) * E, t < T, E, k, renorm, ids,
                               gates);
    if ((threadIdx.x & (G - 1)) == 0) {
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        s_ids[tok][j] = ids[j];
        s_gates[tok][j] = gates[j];
      }
    }
    __syncthreads();
    const int tile = blockIdx.x * kTiles + w;
    if (w < kTiles && tile < n_tiles) {
      const int lt = w * kBrimTileTokens + (int)lane;
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        ids[j] = s_ids[lt][j];
        gates[j] = s_gates[lt][j];
      }
      route_tile_masks<KMAX>(tile * kBrimTileTokens + (int)lane, tile, T, E, k, R, prune_m,
                             n_tiles, s_slot, ids, gates, s_mask[w], topk_idx, topk_w, masks,
                             err);
    }
  }
}

}  // namespace moe
