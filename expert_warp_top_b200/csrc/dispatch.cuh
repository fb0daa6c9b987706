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
// All movers work one warp per token and move 16 bytes per lane per access
// (128-bit, fully coalesced 512-byte warp accesses).  A warp first reads the
// token's BRIM entries into a short destination list, then streams the row.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int kMoverWarps = 8;     // warps per block
constexpr int kMaxDst = 32;        // >= min(k,R) + k for k <= 16

// Collect, for token t, the SFD rows (ascending rank) and for each of them
// its EPD rows (ascending local expert).  n_sfd <= min(k, R); p_start has
// n_sfd + 1 entries into p_list.  Out-of-range entries raise the error flag
// and are dropped.
struct DstList {
  int n_sfd;
  int sfd[16];
  int p_start[17];
  int p_list[16];
};

__device__ __forceinline__ void collect_dst(const int32_t* __restrict__ brim0,
                                            const int32_t* __restrict__ brim1, int t, int T,
                                            int R, int L, size_t cap, int tk, DstList& dl,
                                            unsigned* err) {
  const unsigned lane = lane_id();
  dl.n_sfd = 0;
  int np = 0;
  bool bad = false;
  for (int r0 = 0; r0 < R; r0 += 32) {
    const int r = r0 + (int)lane;
    int s = (r < R) ? brim0[(size_t)r * T + t] : -1;
    if (s >= (int)cap) {
      bad = true;
      s = -1;
    }
    unsigned hit = __ballot_sync(0xffffffffu, s >= 0);
    while (hit) {
      const int src = __ffs(hit) - 1;
      hit &= hit - 1;
      const int sv = __shfl_sync(0xffffffffu, s, src);
      if (dl.n_sfd < 16) {
        dl.sfd[dl.n_sfd] = sv;
        dl.p_start[dl.n_sfd] = np;
        // this SFD row's local experts
        for (int l0 = 0; l0 < L; l0 += 32) {
          const int l = l0 + (int)lane;
          int p = (l < L) ? brim1[(size_t)l * cap + sv] : -1;
          if (p >= tk) {
            bad = true;
            p = -1;
          }
          unsigned ph = __ballot_sync(0xffffffffu, p >= 0);
          while (ph) {
            const int ps = __ffs(ph) - 1;
            ph &= ph - 1;
            const int pv = __shfl_sync(0xffffffffu, p, ps);
            if (np < 16) dl.p_list[np++] = pv;
            else bad = true;
          }
        }
        dl.n_sfd++;
      } else {
        bad = true;
      }
    }
  }
  dl.p_start[dl.n_sfd] = np;
  if (__any_sync(0xffffffffu, bad) && lane == 0) raise_error(err, kErrIndex);
}

// x_sfd[s] = x[t] and x_epd[p] = x[t] for every destination of token t.
__global__ void __launch_bounds__(kMoverWarps * 32) dispatch_kernel(
    const uint8_t* __restrict__ x, int T, int row_bytes, int R, int L, size_t cap, int tk,
    const int32_t* __restrict__ brim0, const int32_t* __restrict__ brim1,
    uint8_t* __restrict__ x_sfd, uint8_t* __restrict__ x_epd, unsigned* err) {
  const int t = blockIdx.x * kMoverWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  const unsigned lane = lane_id();
  DstList dl;
  collect_dst(brim0, brim1, t, T, R, L, cap, tk, dl, err);
  const uint8_t* src = x + (size_t)t * row_bytes;
  const int n_p = dl.p_start[dl.n_sfd];
  // 4 x 512 bytes in flight per warp per step
  for (int off0 = 0; off0 < row_bytes; off0 += 4 * 512) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int off = off0 + u * 512 + (int)lane * 16;
      if (off < row_bytes) v[u] = ld_nc_v4(src + off);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int off = off0 + u * 512 + (int)lane * 16;
      if (off >= row_bytes) continue;
      if (x_sfd)
        for (int i = 0; i < dl.n_sfd; ++i) st_v4(x_sfd + (size_t)dl.sfd[i] * row_bytes + off, v[u]);
      if (x_epd)
        for (int i = 0; i < n_p; ++i) st_v4(x_epd + (size_t)dl.p_list[i] * row_bytes + off, v[u]);
    }
  }
}

// y_sfd[s] = sum_l o_epd[BRIM_1[l][s]] (fp32, rounded to T); y[t] = sum_r y_sfd[..]
// (+ shared[t]).  y sums the rounded payload rows, exactly as if it had read
// them back.
template <typename TA>
__global__ void __launch_bounds__(kMoverWarps * 32) combine_kernel(
    const TA* __restrict__ o_epd, int T, int d, int R, int L, size_t cap, int tk,
    const int32_t* __restrict__ brim0, const int32_t* __restrict__ brim1,
    const TA* __restrict__ shared_out, TA* __restrict__ y_sfd, TA* __restrict__ y,
    unsigned* err) {
  constexpr int VN = Vec16<TA>::n;  // elements per 16 bytes
  const int t = blockIdx.x * kMoverWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  const unsigned lane = lane_id();
  DstList dl;
  collect_dst(brim0, brim1, t, T, R, L, cap, tk, dl, err);
  for (int c0 = 0; c0 < d; c0 += 2 * 32 * VN) {
    float ya[2][VN];
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int i = 0; i < VN; ++i) ya[u][i] = 0.f;
    for (int i = 0; i < dl.n_sfd; ++i) {
      float acc[2][VN];
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int e = 0; e < VN; ++e) acc[u][e] = 0.f;
      for (int j = dl.p_start[i]; j < dl.p_start[i + 1]; ++j) {
        const TA* row = o_epd + (size_t)dl.p_list[j] * d;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int c = c0 + u * 32 * VN + (int)lane * VN;
          if (c < d) {
            float f[VN];
            Vec16<TA>::to_f32(ld_nc_v4(row + c), f);
#pragma unroll
            for (int e = 0; e < VN; ++e) acc[u][e] += f[e];
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int c = c0 + u * 32 * VN + (int)lane * VN;
        if (c < d) {
          const uint4 packed = Vec16<TA>::from_f32(acc[u]);
          if (y_sfd) st_v4(y_sfd + (size_t)dl.sfd[i] * d + c, packed);
          float rounded[VN];
          Vec16<TA>::to_f32(packed, rounded);
#pragma unroll
          for (int e = 0; e < VN; ++e) ya[u][e] += rounded[e];
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int c = c0 + u * 32 * VN + (int)lane * VN;
      if (c < d) {
        if (shared_out) {
          float f[VN];
          Vec16<TA>::to_f32(ld_nc_v4(shared_out + (size_t)t * d + c), f);
#pragma unroll
          for (int e = 0; e < VN; ++e) ya[u][e] += f[e];
        }
        st_v4(y + (size_t)t * d + c, Vec16<TA>::from_f32(ya[u]));
      }
    }
  }
}

// Identity expert: out[p] = row_scale[p] * a[p] for the rows of all groups.
template <typename TA>
__global__ void __launch_bounds__(kMoverWarps * 32) identity_expert_kernel(
    const TA* __restrict__ a, const int32_t* __restrict__ group_off, int G, int d,
    const float* __restrict__ row_scale, TA* __restrict__ out) {
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
  const int seg_bytes = fs * esz;
  for (long long w = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
       w < (long long)S * d; w += (long long)gridDim.x * (blockDim.x >> 5)) {
    const int s = (int)(w / d), c = (int)(w % d);
    copy_row(w_dn + ((size_t)c * S + s) * seg_bytes, sd + ((size_t)s * d + c) * seg_bytes, seg_bytes);
  }
}

}  // namespace moe
