// backward.cuh -- the small kernels of the layer's backward pass.
//
// The backward pass is the exact derivative of the layer for fixed expert
// choices: top-k selection passes no gradient, the gate weights pass theirs
// through the softmax they came from.  The data movement mirrors the
// forward through the same BRIMs ("bidirectional re-index", Occult, Fig. 4):
// the upstream gradient dY travels ORI -> SFD -> EPD exactly like X did, and
// the input gradient returns EPD -> SFD -> ORI exactly like the output did,
// so the dispatch and combine kernels serve both directions.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kBwdMaxPerLane = 8;  // logits per lane of a routing warp (E <= 256)

// d_row[p] = sum_j partial[p * n_part + j] for the rows the groups cover,
// group_off[0] <= p < group_off[G]; 0 elsewhere.  Fixed order: deterministic.
__global__ void __launch_bounds__(256) row_partial_sum_kernel(const float* __restrict__ partial,
                                                              int n_part, int m_cap,
                                                              const int32_t* __restrict__ group_off,
                                                              int G, float* __restrict__ d_row) {
  pdl_enter();
  const int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= m_cap) return;
  const int lo = group_off[0], hi = group_off[G];
  float s = 0.f;
  if (p >= lo && p < hi)
    for (int j = 0; j < n_part; ++j) s += partial[(size_t)p * n_part + j];
  d_row[p] = s;
}

// Writes two int32 values (the bounds of a single group).
__global__ void set_two_kernel(int32_t* p, int a, int b) {
  pdl_enter();
  p[0] = a;
  p[1] = b;
}

// Routing backward, one warp per token.  With q the softmax of the token's
// logits over all E experts (renorm = 0) or over its k selected experts
// (renorm = 1, q = 0 elsewhere), each gate is w_j = q_{e_j} and
//   dL/dl_e = q_e * (dw(e) - sum_j dw_j w_j),   dw(e) = dw_j if e = e_j, else 0.
// dw_j is the gradient of the gate weight of slot j, read in EPD order at the
// row the BRIMs give for (t, j): p = BRIM_1[loc(e_j)][BRIM_0[rank(e_j)][t]].
template <int KMAX>
__global__ void __launch_bounds__(256) route_backward_kernel(
    const float* __restrict__ logits, int T, int E, int k, int renorm,
    const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ slot_of, int R,
    const int32_t* __restrict__ brim0, const int32_t* __restrict__ brim1, size_t cap,
    const float* __restrict__ d_gate_epd, int n_epd, float* __restrict__ d_logits,
    float* __restrict__ d_topk_w, unsigned* err) {
  pdl_enter();
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const unsigned lane = lane_id();
  if (t >= T) return;
  const int L = E / R;
  const float* row = logits + (size_t)t * E;
  float v[kBwdMaxPerLane];
  const int per_lane = (E + 31) >> 5;
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < kBwdMaxPerLane; ++i) {
    const int e = lane + 32 * i;
    v[i] = (i < per_lane && e < E) ? __ldg(row + e) : -INFINITY;
    mx = fmaxf(mx, v[i]);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));

  // slot j lives in lane j: its expert, its gradient, exp(logit - max)
  int e_j = -1;
  float dw_j = 0.f, x_j = 0.f;
  if ((int)lane < k) {
    e_j = topk_idx[(size_t)t * k + lane];
    if (e_j >= 0 && e_j < E) {
      const int q = slot_of[e_j];
      const int s = brim0[(size_t)(q / L) * T + t];
      const int p = s >= 0 ? brim1[(size_t)(q % L) * cap + s] : -1;
      if (p >= 0 && p < n_epd) dw_j = d_gate_epd[p];
      else raise_error(err, kErrIndex);
      x_j = expf(__ldg(row + e_j) - mx);
    } else {
      if (e_j != -1) raise_error(err, kErrIndex);
      e_j = -1;
    }
  }
  float z = 0.f;
  if (renorm) {
    z = x_j;
  } else {
#pragma unroll
    for (int i = 0; i < kBwdMaxPerLane; ++i)
      if (i < per_lane && (int)(lane + 32 * i) < E) z += expf(v[i] - mx);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
  const float w_j = x_j / z;
  float sdw = dw_j * w_j;  // lanes >= k contribute 0
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sdw += __shfl_xor_sync(0xffffffffu, sdw, off);
  if (d_topk_w && (int)lane < k) d_topk_w[(size_t)t * k + lane] = dw_j;

  float dl[kBwdMaxPerLane];
  bool sel[kBwdMaxPerLane];
#pragma unroll
  for (int i = 0; i < kBwdMaxPerLane; ++i) {
    dl[i] = 0.f;
    sel[i] = false;
  }
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    if (j >= k) break;
    const int ej = __shfl_sync(0xffffffffu, e_j, j);
    const float dwj = __shfl_sync(0xffffffffu, dw_j, j);
    if (ej >= 0 && (ej & 31) == (int)lane) {
      const int i = ej >> 5;
#pragma unroll
      for (int ii = 0; ii < kBwdMaxPerLane; ++ii)
        if (ii == i) {
          dl[ii] = dwj;
          sel[ii] = true;
        }
    }
  }
  float* out = d_logits + (size_t)t * E;
#pragma unroll
  for (int i = 0; i < kBwdMaxPerLane; ++i) {
    const int e = lane + 32 * i;
    if (i < per_lane && e < E) {
      const bool in_set = renorm ? sel[i] : true;
      const float q = in_set ? expf(v[i] - mx) / z : 0.f;
      out[e] = q * (dl[i] - sdw);
    }
  }
}

}  // namespace moe
