// ep.cuh -- the device side of real expert parallelism: what a source rank
// sends with each token row, so that the destination rank can build its own
// expert-partitioned state.
//
// Occult paper, Abstract and Figure 2: under expert parallelism a token is
// sent to the devices that hold its experts; the once-per-device dispatch
// ("Expert Coupling in MoE Pretraining", Abstract: a dispatcher that sends
// each token to each GPU once) ships one row per (token, destination).  The
// destination needs, with each row, which of ITS experts the token selected
// and with what gate weight: the token's top-k list restricted to the
// destination's experts.
#pragma once
#include "brim.cuh"
#include "dispatch.cuh"

namespace moe {

// For every SFD row s < C_T (token t = sfd_token[s], destination q = the
// segment of sfd_off holding s): idx_send[s][j] = topk_idx[t][j] when that
// expert lives on rank q, else -1; w_send[s][j] = its gate weight, else 0.
// One thread per SFD row.  Out-of-range tokens or expert ids raise the index
// error bit and leave an all-empty row.  PEER: row s of destination q is
// written to row peers.row0[q] + s of peers.idx[q] / peers.w[q] (the
// receiving rank's buffers) instead of idx_send / w_send.
template <bool PEER>
__device__ __forceinline__ void ep_pack_routing_body(
    const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_w, int T, int k,
    const int32_t* __restrict__ slot_of, int E, int R, int L,
    const int32_t* __restrict__ sfd_token, const int32_t* __restrict__ sfd_off,
    const int32_t* __restrict__ c_t, long long cap, int32_t* __restrict__ idx_send,
    float* __restrict__ w_send, unsigned* err, const EpPeers* peers) {
  pdl_enter();
  __shared__ int s_off[kMaxE + 1];
  for (int i = threadIdx.x; i <= R; i += blockDim.x) s_off[i] = sfd_off[i];
  __syncthreads();
  const long long n = min((long long)*c_t, cap);
  bool bad = false;
  for (long long s = (long long)blockIdx.x * blockDim.x + threadIdx.x; s < n;
       s += (long long)gridDim.x * blockDim.x) {
    int lo = 0, hi = R;  // the largest q with sfd_off[q] <= s
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_off[mid] <= s) lo = mid;
      else hi = mid;
    }
    const int t = sfd_token[s];
    const bool t_ok = t >= 0 && t < T;
    bad |= !t_ok;
    int32_t* idx_row = idx_send + s * k;
    float* w_row = w_send + s * k;
    if constexpr (PEER) {
      const long long row = peers->row0[lo] + s;
      idx_row = peers->idx[lo] + row * k;
      w_row = peers->w[lo] + row * k;
    }
    for (int j = 0; j < k; ++j) {
      int e = t_ok ? topk_idx[(size_t)t * k + j] : -1;
      float w = 0.f;
      if (e >= E) {
        bad = true;
        e = -1;
      }
      if (e >= 0) {
        const int slot = slot_of[e];
        if (slot < 0 || slot >= E) {
          bad = true;
          e = -1;
        } else if (slot / L != lo) {
          e = -1;
        } else {
          w = topk_w[(size_t)t * k + j];
        }
      }
      idx_row[j] = e;
      w_row[j] = w;
    }
  }
  if (bad) raise_error(err, kErrIndex);
}

__global__ void __launch_bounds__(256) ep_pack_routing_kernel(
    const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_w, int T, int k,
    const int32_t* __restrict__ slot_of, int E, int R, int L,
    const int32_t* __restrict__ sfd_token, const int32_t* __restrict__ sfd_off,
    const int32_t* __restrict__ c_t, long long cap, int32_t* __restrict__ idx_send,
    float* __restrict__ w_send, unsigned* err) {
  ep_pack_routing_body<false>(topk_idx, topk_w, T, k, slot_of, E, R, L, sfd_token, sfd_off, c_t,
                              cap, idx_send, w_send, err, nullptr);
}
__global__ void __launch_bounds__(256) ep_pack_routing_peer_kernel(
    const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_w, int T, int k,
    const int32_t* __restrict__ slot_of, int E, int R, int L,
    const int32_t* __restrict__ sfd_token, const int32_t* __restrict__ sfd_off,
    const int32_t* __restrict__ c_t, long long cap, unsigned* err,
    const __grid_constant__ EpPeers peers) {
  ep_pack_routing_body<true>(topk_idx, topk_w, T, k, slot_of, E, R, L, sfd_token, sfd_off, c_t,
                             cap, nullptr, nullptr, err, &peers);
}

}  // namespace moe
