// route.cuh -- top-k routing with softmax gate weights.
//
// Each token is routed to k of the E experts ("Expert Coupling in MoE
// Pretraining", Abstract).  Selection compares logits; of equal logits the
// lower expert id wins; the k ids come out in descending order.  Gate
// weights: softmax over all E logits (renorm = 0) or over the k selected
// ones (renorm = 1), in fp32.
//
// A group of G lanes per token (route_token_group, G = 1..8 by batch size):
// each lane streams its share of the token's logits, keeping its best on one
// 64-bit rank each (an order-preserving 32-bit key of the logit above, the
// bitwise complement of the expert id below), so a larger rank is a larger
// logit or, at equal logits, a lower id: ties resolve to the lower id
// exactly.  A candidate enters a lane's sorted list only above its lowest
// entry.  The group merges its lists with a butterfly max per selected slot,
// and one lane sums the softmax denominator over the row in expert order.
#pragma once
#include "common.cuh"

namespace moe {

// Order-preserving map float -> uint32 (larger float -> larger key);
// -0.0 is folded onto +0.0 so the two compare equal, like the floats do.
__device__ __forceinline__ uint32_t float_order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u << 1) == 0u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The float a key came from (-0.0 comes back as +0.0).
__device__ __forceinline__ float float_from_order_key(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// Offers expert e with logit x to a thread's best-KMAX list of ranks top[],
// ascending; a rank holds the logit's key, so the list needs no logits beside
// it.  top[0] is the entry threshold.  The k best are top[KMAX - 1],
// top[KMAX - 2], ... (k <= KMAX), so every index is a compile-time constant and
// the list stays in registers.
template <int KMAX>
__device__ __forceinline__ void route_offer(uint64_t (&top)[KMAX], int e, float x) {
  const uint64_t c = (static_cast<uint64_t>(float_order_key(x)) << 32) | static_cast<uint32_t>(~e);
  if (c > top[0]) {
    top[0] = c;
#pragma unroll
    for (int j = 0; j + 1 < KMAX; ++j) {
      const bool sw = top[j] > top[j + 1];
      const uint64_t lo = sw ? top[j + 1] : top[j], hi = sw ? top[j] : top[j + 1];
      top[j] = lo;
      top[j + 1] = hi;
    }
  }
}

// Routes one token with a group of G consecutive lanes (G = 1, 2, 4 or 8;
// every lane of the warp calls it, a token per group; `valid` false for a
// group without a token).  Selection: lane s of the group offers experts
// 4q..4q+3 for q = s, s + G, ... (or e = s, s + G, ... when the row is not
// float4-aligned) to its best-KMAX list; the group then takes k rounds of a
// butterfly max over its lanes' list heads, the owner popping its head.  The
// ranks are unique, so the selection is the same for every G.  The softmax
// denominator is summed by the group's first lane alone, over the row in
// expert order (renorm = 0) or over the selected in selection order
// (renorm = 1): the same code for every G, so the gates do not depend on G.
// On return every lane of the group holds ids[j], gates[j] for j < k (the
// j-th selected expert, descending logit, ties -> lower id, and its gate);
// slots j >= k are -1 and 0.
template <int KMAX, int G>
__device__ __forceinline__ void route_token_group(const float* __restrict__ row, bool valid,
                                                  int E, int k, int renorm, int (&ids)[KMAX],
                                                  float (&gates)[KMAX]) {
  static_assert(G == 1 || G == 2 || G == 4 || G == 8, "G must be 1, 2, 4 or 8");
  const int sub = static_cast<int>(lane_id()) & (G - 1);
  uint64_t top[KMAX];  // this lane's best ranks, ascending; 0 = empty
#pragma unroll
  for (int j = 0; j < KMAX; ++j) top[j] = 0ull;
  const bool vec = (E & 3) == 0 && (reinterpret_cast<uintptr_t>(row) & 15) == 0;
  // With KMAX = 8 and E = 8 G, a lane holds exactly eight logits: it sorts their
  // ranks with a 19-comparator network (Batcher's odd-even merge sort) instead
  // of eight insertions.  The list comes out the same, as the ranks are unique.
  bool sorted8 = false;
  if constexpr (KMAX == 8) {
    if (valid && vec && (E >> 2) == 2 * G) {
      const float4* r4 = reinterpret_cast<const float4*>(row);
      const float4 x0 = __ldg(r4 + sub), x1 = __ldg(r4 + sub + G);
      const float xs[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = 4 * (i < 4 ? sub : sub + G) + (i & 3);
        top[i] = (static_cast<uint64_t>(float_order_key(xs[i])) << 32) |
                 static_cast<uint32_t>(~e);
      }
      constexpr int kNet[19][2] = {{0, 1}, {2, 3}, {4, 5}, {6, 7}, {0, 2}, {1, 3}, {4, 6},
                                   {5, 7}, {1, 2}, {5, 6}, {0, 4}, {1, 5}, {2, 6}, {3, 7},
                                   {2, 4}, {3, 5}, {1, 2}, {3, 4}, {5, 6}};
#pragma unroll
      for (int c = 0; c < 19; ++c) {
        const uint64_t lo = top[kNet[c][0]], hi = top[kNet[c][1]];
        const bool sw = lo > hi;
        top[kNet[c][0]] = sw ? hi : lo;
        top[kNet[c][1]] = sw ? lo : hi;
      }
      sorted8 = true;
    }
  }
  if (valid && !sorted8) {
    if (vec) {
      const float4* r4 = reinterpret_cast<const float4*>(row);
      for (int q = sub; q < (E >> 2); q += G) {
        const float4 x = __ldg(r4 + q);
        route_offer<KMAX>(top, 4 * q, x.x);
        route_offer<KMAX>(top, 4 * q + 1, x.y);
        route_offer<KMAX>(top, 4 * q + 2, x.z);
        route_offer<KMAX>(top, 4 * q + 3, x.w);
      }
    } else {
      for (int e = sub; e < E; e += G) route_offer<KMAX>(top, e, __ldg(row + e));
    }
  }
  uint64_t sel[KMAX];
  if constexpr (G == 1) {
#pragma unroll
    for (int j = 0; j < KMAX; ++j) sel[j] = top[KMAX - 1 - j];
  } else {
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      sel[j] = 0ull;
      if (j < k) {  // k is the same on every lane: the shuffles stay converged
        uint64_t best = top[KMAX - 1];
#pragma unroll
        for (int off = G / 2; off >= 1; off >>= 1) {
          const uint32_t olo = __shfl_xor_sync(0xffffffffu, static_cast<uint32_t>(best), off);
          const uint32_t ohi = __shfl_xor_sync(0xffffffffu, static_cast<uint32_t>(best >> 32), off);
          const uint64_t o = (static_cast<uint64_t>(ohi) << 32) | olo;
          if (o > best) best = o;
        }
        sel[j] = best;
        if (best != 0ull && top[KMAX - 1] == best) {  // this lane held it: pop the head
#pragma unroll
          for (int i = KMAX - 1; i > 0; --i) top[i] = top[i - 1];
          top[0] = 0ull;
        }
      }
    }
  }
  // the selected logits, from their keys
  float selv[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j)
    selv[j] = float_from_order_key(static_cast<uint32_t>(sel[j] >> 32));
  // softmax: m = the largest logit (the first selected one)
  const float m = selv[0];
  float denom = 0.f;
  if (valid && sub == 0) {
    if (renorm) {
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (j < k) denom += expf(selv[j] - m);
    } else if (vec) {
      const float4* r4 = reinterpret_cast<const float4*>(row);
      for (int q = 0; q < (E >> 2); ++q) {
        const float4 x = __ldg(r4 + q);
        denom += expf(x.x - m);
        denom += expf(x.y - m);
        denom += expf(x.z - m);
        denom += expf(x.w - m);
      }
    } else {
      for (int e = 0; e < E; ++e) denom += expf(__ldg(row + e) - m);
    }
  }
  if constexpr (G > 1)
    denom = __shfl_sync(0xffffffffu, denom, static_cast<int>(lane_id()) & ~(G - 1));
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    ids[j] = j < k ? static_cast<int>(~static_cast<uint32_t>(sel[j])) : -1;
    gates[j] = j < k ? expf(selv[j] - m) / denom : 0.f;
  }
}

// Lanes per token for a batch of T tokens: enough groups to give every SM
// about 16 warps of routing, at most 8 lanes per token.
__host__ __device__ constexpr int route_lanes_per_token(long long T, int num_sms) {
  return T * 8 <= 16LL * 32 * num_sms ? 8 : T * 4 <= 16LL * 32 * num_sms ? 4
         : T * 2 <= 16LL * 32 * num_sms ? 2 : 1;
}

template <int KMAX, int G>
__global__ void __launch_bounds__(256) route_topk_kernel(const float* __restrict__ logits,
                                                         int T, int E, int k, int renorm,
                                                         int32_t* __restrict__ topk_idx,
                                                         float* __restrict__ topk_w) {
  pdl_enter();
  const long long g = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) / G;
  if ((g - static_cast<long long>(threadIdx.x % 32) / G) >= T) return;  // whole warp past the end
  const bool valid = g < T;
  const int t = valid ? static_cast<int>(g) : 0;
  int ids[KMAX];
  float gates[KMAX];
  route_token_group<KMAX, G>(logits + (size_t)t * E, valid, E, k, renorm, ids, gates);
  if (valid && (threadIdx.x & (G - 1)) == 0) {
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (j < k) {
        topk_idx[(size_t)t * k + j] = ids[j];
        topk_w[(size_t)t * k + j] = gates[j];
      }
  }
}

}  // namespace moe
