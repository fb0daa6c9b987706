// shuffle.cuh -- token shuffling across layers ("Expert Coupling in MoE
// Pretraining", Abstract): the experts a token selects at one layer predict
// the experts it selects at the next, so each token can move to the rank
// predicted to hold its next-layer experts before that layer's dispatch.
//
//   interlayer_hist_kernel  H[a][b] += #tokens with expert a at layer l and
//                           expert b at layer l+1 (calibration statistic)
//   rank_affinity_kernel    A[a][r] = sum of H[a][b] over the experts b that
//                           rank r holds at layer l+1
//   predict_home_kernel     home[t] = argmax_r sum_j A[idx_l[t][j]][r] (ties:
//                           lower r; all-zero scores: floor(t R / T))
//   count_local_kernel      assignments of layer l+1 served on the token's
//                           home rank, and all assignments
//   gather_rows_kernel      x_out[i] = x[perm[i]], inv[perm[i]] = i: the
//                           token rows in home-rank order (the order itself
//                           comes from the BRIM passes, one "expert" per rank)
// Integer atomics only: results do not depend on the order they land in.
#pragma once
#include "brim.cuh"

namespace moe {

// Adds tokens [t0, t1) to the inter-layer histogram, one thread per token;
// in shared memory first when E <= kHistSmemE.  Ids outside [0, E) other than
// -1 (an empty slot) raise the index error bit and count nothing.
template <int KMAX>
__global__ void __launch_bounds__(256) interlayer_hist_kernel(
    const int32_t* __restrict__ idx_a, const int32_t* __restrict__ idx_b, int T, int k, int E,
    uint32_t* __restrict__ hist, unsigned* err) {
  pdl_enter();
  __shared__ uint32_t sh[kHistSmemE * kHistSmemE];
  const bool use_smem = E <= kHistSmemE;
  if (use_smem) {
    for (int i = threadIdx.x; i < E * E; i += blockDim.x) sh[i] = 0u;
    __syncthreads();
  }
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t < T) {
    int a[KMAX], b[KMAX];
    bool bad = false;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      a[j] = j < k ? __ldg(idx_a + (size_t)t * k + j) : -1;
      b[j] = j < k ? __ldg(idx_b + (size_t)t * k + j) : -1;
      if (a[j] >= E || a[j] < -1) { bad = true; a[j] = -1; }
      if (b[j] >= E || b[j] < -1) { bad = true; b[j] = -1; }
    }
    if (bad) raise_error(err, kErrIndex);
#pragma unroll
    for (int i = 0; i < KMAX; ++i)
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (a[i] >= 0 && b[j] >= 0) {
          const int cell = a[i] * E + b[j];
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

// One thread per (a, r): A[a][r] = sum over b with slot_of_b[b] / L == r of H[a][b].
__global__ void __launch_bounds__(256) rank_affinity_kernel(const uint32_t* __restrict__ hist,
                                                            int E, const int32_t* __restrict__ slot_of_b,
                                                            int R, uint32_t* __restrict__ table,
                                                            unsigned* err) {
  pdl_enter();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= E * R) return;
  const int a = i / R, r = i - a * R, L = E / R;
  uint32_t s = 0;
  bool bad = false;
  for (int b = 0; b < E; ++b) {
    const int q = __ldg(slot_of_b + b);
    if (q < 0 || q >= E) bad = true;
    else if (q / L == r) s += __ldg(hist + (size_t)a * E + b);
  }
  if (bad) raise_error(err, kErrIndex);
  table[i] = s;
}

// One warp per token; lane i scores ranks i, i + 32, ...  The warp takes the
// largest score (redux max) and, among the ranks that reach it, the lowest
// (redux min).
template <int KMAX>
__global__ void __launch_bounds__(256) predict_home_kernel(const int32_t* __restrict__ idx_a,
                                                           int T, int k, int E,
                                                           const uint32_t* __restrict__ table,
                                                           int R, int32_t* __restrict__ home) {
  pdl_enter();
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const unsigned lane = lane_id();
  if (t >= T) return;
  int a[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    a[j] = j < k ? __ldg(idx_a + (size_t)t * k + j) : -1;
    if (a[j] >= E) a[j] = -1;
  }
  uint32_t best = 0u;
  int best_r = 0x7fffffff;
  for (int r = lane; r < R; r += 32) {
    uint32_t s = 0u;
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (a[j] >= 0) s += __ldg(table + (size_t)a[j] * R + r);
    if (best_r == 0x7fffffff || s > best) {  // ascending r: ties keep the lower
      best = s;
      best_r = r;
    }
  }
  const uint32_t wmax = __reduce_max_sync(0xffffffffu, best_r == 0x7fffffff ? 0u : best);
  const unsigned cand = (best_r != 0x7fffffff && best == wmax) ? (unsigned)best_r : 0xffffffffu;
  const unsigned win = __reduce_min_sync(0xffffffffu, cand);
  if (lane == 0)
    home[t] = wmax > 0u ? (int32_t)win : (int32_t)(((long long)t * R) / T);
}

// out[0] += assignments on the token's home rank, out[1] += all assignments.
// home == nullptr: the contiguous home floor(t R / T).
template <int KMAX>
__global__ void __launch_bounds__(256) count_local_kernel(
    const int32_t* __restrict__ idx, int T, int k, const int32_t* __restrict__ slot_of, int E,
    int R, const int32_t* __restrict__ home, unsigned long long* __restrict__ out, unsigned* err) {
  pdl_enter();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  const int L = E / R;
  unsigned loc = 0, all = 0;
  bool bad = false;
  if (t < T) {
    const int h = home ? __ldg(home + t) : (int)(((long long)t * R) / T);
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j >= k) break;
      const int e = __ldg(idx + (size_t)t * k + j);
      if (e == -1) continue;
      if (e < 0 || e >= E) {
        bad = true;
        continue;
      }
      ++all;
      loc += __ldg(slot_of + e) / L == h;
    }
  }
  if (bad) raise_error(err, kErrIndex);
  loc = __reduce_add_sync(0xffffffffu, loc);
  all = __reduce_add_sync(0xffffffffu, all);
  if (lane_id() == 0 && all) {
    atomicAdd(&out[0], (unsigned long long)loc);
    atomicAdd(&out[1], (unsigned long long)all);
  }
}

// x_out[i] = x[perm[i]] (rows of row_bytes, 16-byte multiple), one warp per
// row; inv[perm[i]] = i when inv is given.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint8_t* __restrict__ x,
                                                          const int32_t* __restrict__ perm, int T,
                                                          int row_bytes, uint8_t* __restrict__ x_out,
                                                          int32_t* __restrict__ inv, unsigned* err) {
  pdl_enter();
  const int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (i >= T) return;
  const int t = __ldg(perm + i);
  if (t < 0 || t >= T) {
    if (lane_id() == 0) raise_error(err, kErrIndex);
    return;
  }
  if (inv && lane_id() == 0) inv[t] = i;
  const uint8_t* src = x + (size_t)t * row_bytes;
  uint8_t* dst = x_out + (size_t)i * row_bytes;
  for (int off = (int)lane_id() * 16; off < row_bytes; off += 512) st_v4(dst + off, ld_nc_v4(src + off));
}

}  // namespace moe
