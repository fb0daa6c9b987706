// dispatch.cuh -- the BRIM-guided row movers: dispatch (ORI -> SFD -> EPD),
// combine (per-rank pre-reduce, then back to ORI), the identity expert, and
// the one-time weight repacking.
//
// Occult paper, Figure 4: token tensors move between the ORI, SFD and EPD
// states, compactly stored in HBM and guided by the BRIMs; the re-index is
// bidirectional, so the same BRIM entries drive the gather on the way out and
// the scatter on the way back.  Occult paper, Abstract: experts on the same
// device that a token co-activates ("intra-collaboration") are summed before
// the single return row leaves the device.
//
// The movers split every token row into 512-byte slices (16 bytes per lane,
// fully coalesced 128-bit accesses) and give each warp one slice (or a few), so
// a batch of a few thousand tokens still fills every SM.  A warp first reads
// its token's BRIM entries into a short destination list in shared memory,
// then moves its slice.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kMoverWarps = 8;     // warps per block
constexpr int kMaxDst = 16;        // >= k (and >= min(k, R))

// Destinations of one token, per warp, in shared memory:
//   sfd[i]   SFD rows of the ranks the token is sent to (ascending rank)
//   p[j]     EPD rows of its experts, ascending (rank, local expert), and
//   p_sfd[j] the SFD row each of them hangs off
struct WarpDst {
  int n_sfd;
  int n_p;
  int sfd[kMaxDst];
  int p[kMaxDst];
  int p_sfd[kMaxDst];
};

// Reads token t's BRIM_0 column and, for every (rank, local expert) slot, its
// BRIM_1 entry; ballots keep ascending order.  Out-of-range entries raise the
// error flag and are dropped.  A null brim1 stands for one "expert" per rank
// whose row is the SFD row itself (p = s; L must be 1): the rows a source rank
// gets back from its destinations under real expert parallelism.
__device__ __forceinline__ void collect_dst(const int32_t* __restrict__ brim0,
                                            const int32_t* __restrict__ brim1, int t, int T,
                                            int R, int L, size_t cap, int tk, WarpDst& w,
                                            unsigned* err) {
  const unsigned lane = lane_id();
  const uint32_t lt = (1u << lane) - 1u;
  bool bad = false;
  int n = 0;
  for (int r0 = 0; r0 < R; r0 += 32) {
    const int r = r0 + (int)lane;
    int s = (r < R) ? __ldg(brim0 + (size_t)r * T + t) : -1;
    if (s >= (int)cap) {
      bad = true;
      s = -1;
    }
    const unsigned hit = __ballot_sync(0xffffffffu, s >= 0);
    const int pos = n + __popc(hit & lt);
    if (s >= 0 && pos < kMaxDst) w.sfd[pos] = s;
    n += __popc(hit);
  }
  if (n > kMaxDst) bad = true;
  const int n_sfd = min(n, kMaxDst);
  n = 0;
  const int E = R * L;
  for (int q0 = 0; q0 < E; q0 += 32) {
    const int q = q0 + (int)lane;
    int s = -1, p = -1;
    if (q < E) {
      const int r = q / L, l = q - r * L;
      s = __ldg(brim0 + (size_t)r * T + t);
      if (s >= 0 && s < (int)cap) p = brim1 ? __ldg(brim1 + (size_t)l * cap + s) : s;
      if (p >= tk) {
        bad = true;
        p = -1;
      }
    }
    const unsigned hit = __ballot_sync(0xffffffffu, p >= 0);
    const int pos = n + __popc(hit & lt);
    if (p >= 0 && pos < kMaxDst) {
      w.p[pos] = p;
      w.p_sfd[pos] = s;
    }
    n += __popc(hit);
  }
  if (n > kMaxDst) bad = true;
  if (lane == 0) {
    w.n_sfd = n_sfd;
    w.n_p = min(n, kMaxDst);
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) raise_error(err, kErrIndex);
  __syncwarp();
}

// x_sfd[s] = x[t] and x_epd[p] = x[t] for every destination of token t.
// One warp per token (P > 1: per 1/P of its row, for small batches); the row
// is read CH x 512 bytes at a time, all CH loads in flight before the stores.
template <int CH>
__global__ void __launch_bounds__(kMoverWarps * 32) dispatch_kernel(
    const uint8_t* __restrict__ x, int T, int row_bytes, int P, int R, int L, size_t cap, int tk,
    const int32_t* __restrict__ brim0, const int32_t* __restrict__ brim1,
    uint8_t* __restrict__ x_sfd, uint8_t* __restrict__ x_epd, unsigned* err) {
  pdl_enter();
  __shared__ WarpDst sdst[kMoverWarps];
  const int wib = threadIdx.x >> 5;
  const long long wg = (long long)blockIdx.x * kMoverWarps + wib;
  const int t = (int)(wg / P);
  if (t >= T) return;
  const int part = (int)(wg - (long long)t * P);
  const unsigned lane = lane_id();
  WarpDst& w = sdst[wib];
  collect_dst(brim0, brim1, t, T, R, L, cap, tk, w, err);
  const int span = (row_bytes + P - 1) / P;
  const int lo = part * span, hi = min(row_bytes, lo + span);
  const uint8_t* src = x + (size_t)t * row_bytes;
  const int n_sfd = x_sfd ? w.n_sfd : 0, n_p = x_epd ? w.n_p : 0;
  for (int off0 = lo; off0 < hi; off0 += CH * 512) {
    uint4 v[CH];
#pragma unroll
    for (int u = 0; u < CH; ++u) {
      const int off = off0 + u * 512 + (int)lane * 16;
      if (off < hi) v[u] = ld_nc_v4(src + off);
    }
    for (int i = 0; i < n_sfd; ++i) {
      uint8_t* dst = x_sfd + (size_t)w.sfd[i] * row_bytes;
#pragma unroll
      for (int u = 0; u < CH; ++u) {
        const int off = off0 + u * 512 + (int)lane * 16;
        if (off < hi) st_v4(dst + off, v[u]);
      }
    }
    for (int i = 0; i < n_p; ++i) {
      uint8_t* dst = x_epd + (size_t)w.p[i] * row_bytes;
#pragma unroll
      for (int u = 0; u < CH; ++u) {
        const int off = off0 + u * 512 + (int)lane * 16;
        if (off < hi) st_v4(dst + off, v[u]);
      }
    }
  }
}

// y_sfd[s] = sum_l o_epd[BRIM_1[l][s]] (fp32, rounded to TA); y[t] = sum_r y_sfd[..]
// (+ shared[t]).  y sums the rounded payload rows, exactly as if it had read
// them back.  A null y leaves only the return rows y_sfd (the destination
// side of real expert parallelism); a null brim1 sums rows already reduced
// per rank (see collect_dst).  One warp per token (or 1/P of its row); the k expert rows of the
// next 512-byte slice are loaded while the current slice is summed, so up to
// 2k loads are in flight per warp.  KMAX >= k bounds the register arrays.
template <typename TA, int KMAX>
__global__ void __launch_bounds__(kMoverWarps * 32) combine_kernel(
    const TA* __restrict__ o_epd, int T, int d, int P, int R, int L, size_t cap, int tk,
    const int32_t* __restrict__ brim0, const int32_t* __restrict__ brim1,
    const TA* __restrict__ shared_out, TA* __restrict__ y_sfd, TA* __restrict__ y,
    unsigned* err) {
  pdl_enter();
  constexpr int VN = Vec16<TA>::n;  // elements per 16 bytes
  constexpr int SL = 32 * VN;       // elements per 512-byte slice
  __shared__ WarpDst sdst[kMoverWarps];
  const int wib = threadIdx.x >> 5;
  const long long wg = (long long)blockIdx.x * kMoverWarps + wib;
  const int t = (int)(wg / P);
  if (t >= T) return;
  const int part = (int)(wg - (long long)t * P);
  const unsigned lane = lane_id();
  WarpDst& w = sdst[wib];
  collect_dst(brim0, brim1, t, T, R, L, cap, tk, w, err);
  const int n_slices = (d + SL - 1) / SL;
  const int per = (n_slices + P - 1) / P;
  const int s_lo = part * per, s_hi = min(n_slices, s_lo + per);
  const int n_p = min(w.n_p, KMAX);
  int prow[KMAX], psfd[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    prow[j] = j < n_p ? w.p[j] : 0;
    psfd[j] = j < n_p ? w.p_sfd[j] : -1;
  }
  uint4 cur[KMAX], nxt[KMAX];
  auto load_slice = [&](int sl, uint4 (&v)[KMAX]) {
    const int c = sl * SL + (int)lane * VN;
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (j < n_p && c < d) v[j] = ld_nc_v4(o_epd + (size_t)prow[j] * d + c);
  };
  if (s_lo < s_hi) load_slice(s_lo, cur);
  for (int sl = s_lo; sl < s_hi; ++sl) {
    if (sl + 1 < s_hi) load_slice(sl + 1, nxt);
    const int c = sl * SL + (int)lane * VN;
    if (c < d) {
      float acc[VN], ya[VN];
#pragma unroll
      for (int e = 0; e < VN; ++e) ya[e] = acc[e] = 0.f;
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        if (j < n_p) {
          float f[VN];
          Vec16<TA>::to_f32(cur[j], f);
#pragma unroll
          for (int e = 0; e < VN; ++e) acc[e] += f[e];
          // the last expert of this rank: emit the rank's return row
          if (j + 1 == n_p || psfd[j + 1 < KMAX ? j + 1 : j] != psfd[j]) {
            const uint4 packed = Vec16<TA>::from_f32(acc);
            if (y_sfd) st_v4(y_sfd + (size_t)psfd[j] * d + c, packed);
            float rounded[VN];
            Vec16<TA>::to_f32(packed, rounded);
#pragma unroll
            for (int e = 0; e < VN; ++e) {
              ya[e] += rounded[e];
              acc[e] = 0.f;
            }
          }
        }
      }
      if (y) {
        if (shared_out) {
          float f[VN];
          Vec16<TA>::to_f32(ld_nc_v4(shared_out + (size_t)t * d + c), f);
#pragma unroll
          for (int e = 0; e < VN; ++e) ya[e] += f[e];
        }
        st_v4(y + (size_t)t * d + c, Vec16<TA>::from_f32(ya));
      }
    }
#pragma unroll
    for (int j = 0; j < KMAX; ++j) cur[j] = nxt[j];
  }
}

// Identity expert: out[p] = row_scale[p] * a[p] for the rows of all groups.
template <typename TA>
__global__ void __launch_bounds__(kMoverWarps * 32) identity_expert_kernel(
    const TA* __restrict__ a, const int32_t* __restrict__ group_off, int G, int d,
    const float* __restrict__ row_scale, TA* __restrict__ out) {
  pdl_enter();
  constexpr int VN = Vec16<TA>::n;
  const int lo = group_off[0], hi = group_off[G];
  const int lane = (int)lane_id();
  for (int row = lo + blockIdx.x * kMoverWarps + (threadIdx.x >> 5); row < hi;
       row += gridDim.x * kMoverWarps) {
    const float s = row_scale ? row_scale[row] : 1.0f;
    for (int c = lane * VN; c < d; c += 32 * VN) {
      float f[VN];
      Vec16<TA>::to_f32(ld_nc_v4(a + (size_t)row * d + c), f);
#pragma unroll
      for (int e = 0; e < VN; ++e) f[e] *= s;
      st_v4(out + (size_t)row * d + c, Vec16<TA>::from_f32(f));
    }
  }
}

// ---- weight repacking (one-time, off the layer path) ---------------------
// One warp per destination row; rows are copied 16 bytes per lane.
__device__ __forceinline__ void copy_row(uint8_t* dst, const uint8_t* src, int bytes) {
  for (int off = (int)lane_id() * 16; off < bytes; off += 512) st_v4(dst + off, ld_nc_v4(src + off));
}

// w_gu[slot(e)][128i + j] = (j < 64 ? wg : wu)[e][64i + j % 64]
__global__ void pack_gate_up_kernel(const uint8_t* __restrict__ wg, const uint8_t* __restrict__ wu,
                                    int E, int d, int f, int esz,
                                    const int32_t* __restrict__ slot_of,
                                    uint8_t* __restrict__ w_gu) {
  pdl_enter();
  const long long n_rows = (long long)E * 2 * f;
  const int row_bytes = d * esz;
  for (long long w = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); w < n_rows;
       w += (long long)gridDim.x * (blockDim.x >> 5)) {
    const int e = (int)(w / (2 * f));
    const int r = (int)(w % (2 * f));
    const int blk = r / 128, j = r % 128;
    const uint8_t* src = (j < 64 ? wg : wu) + ((size_t)e * f + (size_t)blk * 64 + (j & 63)) * row_bytes;
    const int q = slot_of ? slot_of[e] : e;
    copy_row(w_gu + ((size_t)q * 2 * f + r) * row_bytes, src, row_bytes);
  }
}

// w_dn[slot(e)] = wd[e]
__global__ void pack_down_kernel(const uint8_t* __restrict__ wd, int E, int d, int f, int esz,
                                 const int32_t* __restrict__ slot_of, uint8_t* __restrict__ w_dn) {
  pdl_enter();
  const long long n_rows = (long long)E * d;
  const int row_bytes = f * esz;
  for (long long w = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); w < n_rows;
       w += (long long)gridDim.x * (blockDim.x >> 5)) {
    const int e = (int)(w / d);
    const int c = (int)(w % d);
    const int q = slot_of ? slot_of[e] : e;
    copy_row(w_dn + ((size_t)q * d + c) * row_bytes, wd + ((size_t)e * d + c) * row_bytes, row_bytes);
  }
}

// S shared experts -> one expert of width F = S*fs.
// gate'/up' row i = row (i % fs) of expert i / fs; then the 64-row interleave.
__global__ void pack_shared_gate_up_kernel(const uint8_t* __restrict__ sg,
                                           const uint8_t* __restrict__ su, int S, int d, int fs,
                                           int esz, uint8_t* __restrict__ w_gu) {
  pdl_enter();
  const int F = S * fs;
  const int row_bytes = d * esz;
  for (long long w = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); w < 2LL * F;
       w += (long long)gridDim.x * (blockDim.x >> 5)) {
    const int r = (int)w;
    const int blk = r / 128, j = r % 128;
    const int i = blk * 64 + (j & 63);  // row of gate' / up'
    const int s = i / fs, ri = i % fs;
    const uint8_t* src = (j < 64 ? sg : su) + ((size_t)s * fs + ri) * row_bytes;
    copy_row(w_gu + (size_t)r * row_bytes, src, row_bytes);
  }
}

// down'[c][s*fs + i] = sd[s][c][i]
__global__ void pack_shared_down_kernel(const uint8_t* __restrict__ sd, int S, int d, int fs,
                                        int esz, uint8_t* __restrict__ w_dn) {
  pdl_enter();
  const int seg_bytes = fs * esz;
  for (long long w = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
       w < (long long)S * d; w += (long long)gridDim.x * (blockDim.x >> 5)) {
    const int s = (int)(w / d), c = (int)(w % d);
    copy_row(w_dn + ((size_t)c * S + s) * seg_bytes, sd + ((size_t)s * d + c) * seg_bytes, seg_bytes);
  }
}

}  // namespace moe
