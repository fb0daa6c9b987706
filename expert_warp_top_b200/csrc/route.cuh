// route.cuh -- top-k routing with softmax gate weights.
//
// Each token is routed to k of the E experts ("Expert Coupling in MoE
// Pretraining", Abstract).  Selection compares logits; of equal logits the
// lower expert id wins; the k ids come out in descending order.  Gate
// weights: softmax over all E logits (renorm = 0) or over the k selected
// ones (renorm = 1), in fp32.
//
// One warp per token.  Lane i holds logits i, i+32, ... (E <= 256, so at
// most 8 per lane).  Each of the k rounds is one warp max-reduction of an
// order-preserving 32-bit key (redux.sync) followed by a min-reduction of the
// ids that hold the maximum, so ties resolve to the lower id exactly.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kRouteMaxPerLane = 8;  // E <= 256

// Order-preserving map float -> uint32 (larger float -> larger key);
// -0.0 is folded onto +0.0 so the two compare equal, like the floats do.
__device__ __forceinline__ uint32_t float_order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u << 1) == 0u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// This lane's logits of one token: lane i holds logits i, i + 32, ... (the
// slots past E hold -inf and are never selected).
__device__ __forceinline__ void load_token_logits(const float* __restrict__ row, int E,
                                                  float (&v)[kRouteMaxPerLane]) {
  const unsigned lane = lane_id();
  const int per_lane = (E + 31) >> 5;
#pragma unroll
  for (int i = 0; i < kRouteMaxPerLane; ++i) {
    const int e = lane + 32 * i;
    v[i] = (i < per_lane && e < E) ? __ldg(row + e) : -INFINITY;
  }
}

// Routes one token with the whole warp, from its logits as load_token_logits
// leaves them.  On return lane j < k holds the j-th selected expert id in
// *sel_id and its gate weight in *gate (other lanes: unspecified).  All lanes
// must call it.
__device__ __forceinline__ void route_token_warp_v(const float (&v)[kRouteMaxPerLane], int E,
                                                   int k, int renorm, int* sel_id_out,
                                                   float* gate_out) {
  const unsigned lane = lane_id();
  uint32_t key[kRouteMaxPerLane];
  const int per_lane = (E + 31) >> 5;
#pragma unroll
  for (int i = 0; i < kRouteMaxPerLane; ++i) {
    const int e = lane + 32 * i;
    // below every real key; never selected (valid[] is false)
    key[i] = (i < per_lane && e < E) ? float_order_key(v[i]) : 0u;
  }
  unsigned valid = 0;  // bit i: slot i of this lane is a live candidate
#pragma unroll
  for (int i = 0; i < kRouteMaxPerLane; ++i)
    if (i < per_lane && (int)(lane + 32 * i) < E) valid |= 1u << i;

  float sel_logit = 0.f;  // lane j < k keeps the j-th selected logit
  int sel_id = 0;
  for (int j = 0; j < k; ++j) {
    // this lane's best live candidate: larger key, then lower id (= lower i)
    uint32_t best_key = 0u;
    int best_i = -1;
#pragma unroll
    for (int i = 0; i < kRouteMaxPerLane; ++i)
      if (((valid >> i) & 1u) && (best_i < 0 || key[i] > best_key)) {
        best_key = key[i];
        best_i = i;
      }
    const uint32_t wmax = __reduce_max_sync(0xffffffffu, best_i >= 0 ? best_key : 0u);
    const uint32_t my_id = (best_i >= 0 && best_key == wmax) ? (lane + 32u * best_i) : 0xffffffffu;
    const uint32_t win = __reduce_min_sync(0xffffffffu, my_id);
    const unsigned owner = win & 31u;
    const int win_i = (int)(win >> 5);
    float win_logit = 0.f;
#pragma unroll
    for (int i = 0; i < kRouteMaxPerLane; ++i)
      if (i == win_i) win_logit = v[i];
    win_logit = __shfl_sync(0xffffffffu, win_logit, owner);
    if (lane == owner) valid &= ~(1u << win_i);
    if ((int)lane == j) {
      sel_logit = win_logit;
      sel_id = (int)win;
    }
  }

  // softmax: m = the largest logit (the first selected one)
  const float m = __shfl_sync(0xffffffffu, sel_logit, 0);
  float denom;
  if (renorm) {
    float part = ((int)lane < k) ? expf(sel_logit - m) : 0.f;
    // fixed-order tree over the lanes: deterministic
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    denom = part;
  } else {
    float part = 0.f;
#pragma unroll
    for (int i = 0; i < kRouteMaxPerLane; ++i)
      if (i < per_lane && (int)(lane + 32 * i) < E) part += expf(v[i] - m);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    denom = part;
  }
  *sel_id_out = sel_id;
  *gate_out = expf(sel_logit - m) / denom;
}

__device__ __forceinline__ void route_token_warp(const float* __restrict__ row, int E, int k,
                                                 int renorm, int* sel_id_out, float* gate_out) {
  float v[kRouteMaxPerLane];
  load_token_logits(row, E, v);
  route_token_warp_v(v, E, k, renorm, sel_id_out, gate_out);
}

__global__ void __launch_bounds__(256) route_topk_kernel(const float* __restrict__ logits,
                                                         int T, int E, int k, int renorm,
                                                         int32_t* __restrict__ topk_idx,
                                                         float* __restrict__ topk_w) {
  pdl_enter();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const unsigned lane = lane_id();
  if (warp >= T) return;
  int id;
  float gate;
  route_token_warp(logits + (size_t)warp * E, E, k, renorm, &id, &gate);
  if ((int)lane < k) {
    topk_idx[(size_t)warp * k + lane] = id;
    topk_w[(size_t)warp * k + lane] = gate;
  }
}

}  // namespace moe
