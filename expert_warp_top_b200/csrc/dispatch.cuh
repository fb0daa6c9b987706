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
#include "tc_ptx.cuh"

namespace moe {

constexpr int kMoverWarps = 4;     // warps per block
constexpr int kMaxDst = 16;        // >= k (and >= min(k, R))

// Destination buffers of the other ranks, for the movers that write their rows
// straight into the ranks that receive them (real expert parallelism over
// peer memory).  For rank q: rows[q] its row buffer, idx[q] / w[q] its
// routing-list buffers (k entries per row), and this rank's row i lands at
// row row0[q] + i there.  seg[0..R] splits this rank's own rows by owner when
// the owner is found from the row (the return rows: row i belongs to source q
// when seg[q] <= i < seg[q + 1]).  Passed by value as a kernel parameter.
constexpr int kMaxEpPeers = 64;
struct EpPeers {
  uint8_t* rows[kMaxEpPeers];
  int32_t* idx[kMaxEpPeers];
  float* w[kMaxEpPeers];
  long long row0[kMaxEpPeers];
  int seg[kMaxEpPeers + 1];
};

// The owner q of row i: the largest q < R with seg[q] <= i.
__device__ __forceinline__ int ep_peer_owner(const EpPeers& peers, int R, long long i) {
  int lo = 0, hi = R;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (peers.seg[mid] <= i) lo = mid;
    else hi = mid;
  }
  return lo;
}

// Destinations of one token, per warp, in shared memory:
//   sfd[i]   SFD rows of the ranks the token is sent to (ascending rank), and
//   sfd_r[i] the rank of each
//   p[j]     EPD rows of its experts, ascending (rank, local expert), and
//   p_sfd[j] the SFD row each of them hangs off
struct WarpDst {
  int n_sfd;
  int n_p;
  int sfd[kMaxDst];
  int sfd_r[kMaxDst];
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
    if (s >= 0 && pos < kMaxDst) {
      w.sfd[pos] = s;
      w.sfd_r[pos] = r;
    }
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
// PEER: the SFD row s of rank r goes to peers.rows[r] row peers.row0[r] + s
// instead (the receiving rank's buffer), and x_sfd is unused.
template <int CH, bool PEER>
__device__ __forceinline__ void dispatch_body(
    const uint8_t* __restrict__ x, int T, int row_bytes, int P, int R, int L, size_t cap, int tk,
    const int32_t* __restrict__ brim0, const int32_t* __restrict__ brim1,
    uint8_t* __restrict__ x_sfd, uint8_t* __restrict__ x_epd, unsigned* err,
    const EpPeers* peers) {
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
  const int n_sfd = (x_sfd || PEER) ? w.n_sfd : 0, n_p = x_epd ? w.n_p : 0;
  for (int off0 = lo; off0 < hi; off0 += CH * 512) {
    uint4 v[CH];
#pragma unroll
    for (int u = 0; u < CH; ++u) {
      const int off = off0 + u * 512 + (int)lane * 16;
      if (off < hi) v[u] = ld_nc_v4(src + off);
    }
    for (int i = 0; i < n_sfd; ++i) {
      uint8_t* dst;
      if constexpr (PEER) {
        const int r = w.sfd_r[i];
        dst = peers->rows[r] + (size_t)(peers->row0[r] + w.sfd[i]) * row_bytes;
      } else {
        dst = x_sfd + (size_t)w.sfd[i] * row_bytes;
      }
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

template <int CH>
__global__ void __launch_bounds__(kMoverWarps * 32) dispatch_kernel(
    const uint8_t* __restrict__ x, int T, int row_bytes, int P, int R, int L, size_t cap, int tk,
    const int32_t* __restrict__ brim0, const int32_t* __restrict__ brim1,
    uint8_t* __restrict__ x_sfd, uint8_t* __restrict__ x_epd, unsigned* err) {
  dispatch_body<CH, false>(x, T, row_bytes, P, R, L, cap, tk, brim0, brim1, x_sfd, x_epd, err,
                           nullptr);
}
template <int CH>
__global__ void __launch_bounds__(kMoverWarps * 32) dispatch_peer_kernel(
    const uint8_t* __restrict__ x, int T, int row_bytes, int P, int R, int L, size_t cap, int tk,
    const int32_t* __restrict__ brim0, const int32_t* __restrict__ brim1, uint8_t* __restrict__ x_epd,
    unsigned* err, const __grid_constant__ EpPeers peers) {
  dispatch_body<CH, true>(x, T, row_bytes, P, R, L, cap, tk, brim0, brim1, nullptr, x_epd, err,
                          &peers);
}

// The same dispatch through the copy engine (TMA bulk copies, no multicast):
// a warp's lane 0 loads a piece of a token row (at most kBulkPiece bytes) into
// one of the warp's kBulkBufs shared-memory buffers with one cp.async.bulk,
// then stores it to every destination row with one cp.async.bulk each.  The
// loads of the warp's next pieces are in flight while the current piece is
// stored.  A unit of work is (token, piece): pieces are whole rows when the
// batch fills the GPU, shorter for small batches.  Every mbarrier wait is
// bounded: on expiry the timeout bit is raised, the warp stops issuing, waits
// (bounded) for its loads in flight and lets its stores drain before exit.
constexpr int kBulkWarps = 4;       // warps per block
constexpr int kBulkBufs = 3;        // row buffers per warp
constexpr int kBulkPiece = 8192;    // bytes per buffer
constexpr size_t kBulkSmem = (size_t)kBulkWarps * kBulkBufs * kBulkPiece;

__global__ void __launch_bounds__(kBulkWarps * 32) dispatch_bulk_kernel(
    const uint8_t* __restrict__ x, int T, int row_bytes, int piece, int n_pieces, int R, int L,
    size_t cap, int tk, const int32_t* __restrict__ brim0, const int32_t* __restrict__ brim1,
    uint8_t* __restrict__ x_sfd, uint8_t* __restrict__ x_epd, unsigned* err,
    uint64_t wait_limit_ns) {
  extern __shared__ __align__(128) uint8_t bulk_smem[];
  __shared__ __align__(8) uint64_t bars[kBulkWarps][kBulkBufs];
  __shared__ WarpDst sdst[kBulkWarps];
  __shared__ int abort_flag;
  const int wib = threadIdx.x >> 5;
  const unsigned lane = lane_id();
  if (threadIdx.x == 0) abort_flag = 0;
  if (lane == 0)
    for (int b = 0; b < kBulkBufs; ++b) tc::mbar_init(tc::smem_u32(&bars[wib][b]), 1);
  tc::mbar_init_fence();
  __syncthreads();
  pdl_enter();
  const tc::WaitCtl wctl{&abort_flag, err, wait_limit_ns};
  uint8_t* bufs = bulk_smem + (size_t)wib * kBulkBufs * kBulkPiece;
  const long long n_units = (long long)T * n_pieces;
  const long long stride = (long long)gridDim.x * kBulkWarps;
  const long long first = (long long)blockIdx.x * kBulkWarps + wib;
  const long long mine = first < n_units ? (n_units - first + stride - 1) / stride : 0;
  auto unit_of = [&](long long i, int& t, int& off, int& bytes) {
    const long long u = first + i * stride;
    t = (int)(u / n_pieces);
    off = (int)(u - (long long)t * n_pieces) * piece;
    bytes = min(piece, row_bytes - off);
  };
  auto issue_load = [&](long long i) {  // lane 0
    int t, off, bytes;
    unit_of(i, t, off, bytes);
    const int b = (int)(i % kBulkBufs);
    const uint32_t bar = tc::smem_u32(&bars[wib][b]);
    tc::mbar_arrive_expect_tx(bar, (uint32_t)bytes);
    tc::bulk_load(tc::smem_u32(bufs + (size_t)b * kBulkPiece), x + (size_t)t * row_bytes + off,
                  (uint32_t)bytes, bar);
  };
  long long issued = 0;  // loads issued (lane 0)
  if (lane == 0)
    for (; issued < mine && issued < kBulkBufs - 1; ++issued) issue_load(issued);
  bool ok = true;
  for (long long i = 0; i < mine; ++i) {
    int t, off, bytes;
    unit_of(i, t, off, bytes);
    WarpDst& w = sdst[wib];
    collect_dst(brim0, brim1, t, T, R, L, cap, tk, w, err);
    if (lane == 0) {
      // the buffer of load i + kBulkBufs - 1 was last read by the stores of unit i - 1
      if (issued < mine) {
        tc::bulk_wait_read_all();
        issue_load(issued++);
      }
      const int b = (int)(i % kBulkBufs);
      ok = tc::wait_bounded(tc::smem_u32(&bars[wib][b]), (uint32_t)((i / kBulkBufs) & 1), wctl);
      if (ok) {
        const uint32_t src = tc::smem_u32(bufs + (size_t)b * kBulkPiece);
        if (x_sfd)
          for (int j = 0; j < w.n_sfd; ++j)
            tc::bulk_store(x_sfd + (size_t)w.sfd[j] * row_bytes + off, src, (uint32_t)bytes);
        if (x_epd)
          for (int j = 0; j < w.n_p; ++j)
            tc::bulk_store(x_epd + (size_t)w.p[j] * row_bytes + off, src, (uint32_t)bytes);
        tc::bulk_commit_group();
      }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0) != 0;
    __syncwarp();  // the destination list may be rewritten
    if (!ok) {
      // leave no load in flight into this warp's buffers: wait (bounded) for
      // every load issued and not yet consumed
      if (lane == 0)
        for (long long j = i; j < issued; ++j)
          tc::wait_bounded(tc::smem_u32(&bars[wib][j % kBulkBufs]),
                           (uint32_t)((j / kBulkBufs) & 1), wctl, false);
      break;
    }
  }
  if (lane == 0) tc::bulk_wait_all();  // stores complete before the warp's buffers go away
  __syncwarp();
}

// y_sfd[s] = sum_l o_epd[BRIM_1[l][s]] (fp32, rounded to TA); y[t] = sum_r y_sfd[..]
// (+ shared[t]).  y sums the rounded payload rows, exactly as if it had read
// them back.  A null y leaves only the return rows y_sfd (the destination
// side of real expert parallelism); a null brim1 sums rows already reduced
// per rank (see collect_dst).  One warp per token (or 1/P of its row); the k expert rows of the
// next 512-byte slice are loaded while the current slice is summed, so up to
// 2k loads are in flight per warp.  KMAX >= k bounds the register arrays.
// PEER: the return row of SFD row s goes to its owner q (peers.seg) at row
// peers.row0[q] + s of peers.rows[q] (the source rank's buffer); y_sfd unused.
template <typename TA, int KMAX, bool PEER>
__device__ __forceinline__ void combine_body(
    const TA* __restrict__ o_epd, int T, int d, int P, int R, int L, size_t cap, int tk,
    const int32_t* __restrict__ brim0, const int32_t* __restrict__ brim1,
    const TA* __restrict__ shared_out, TA* __restrict__ y_sfd, TA* __restrict__ y,
    unsigned* err, const EpPeers* peers) {
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
  // PEER: where the return row of psfd[j] goes (an array the plain kernel
  // does not carry: its registers would halve that kernel's occupancy)
  TA* ydst[PEER ? KMAX : 1];
  if constexpr (PEER) {
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      ydst[j] = nullptr;
      if (j < n_p) {
        const int q = ep_peer_owner(*peers, R, psfd[j]);
        ydst[j] = reinterpret_cast<TA*>(peers->rows[q]) + (size_t)(peers->row0[q] + psfd[j]) * d;
      }
    }
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
            if constexpr (PEER) {
              st_v4(ydst[j] + c, packed);
            } else {
              if (y_sfd) st_v4(y_sfd + (size_t)psfd[j] * d + c, packed);
            }
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

template <typename TA, int KMAX>
__global__ void __launch_bounds__(kMoverWarps * 32) combine_kernel(
    const TA* __restrict__ o_epd, int T, int d, int P, int R, int L, size_t cap, int tk,
    const int32_t* __restrict__ brim0, const int32_t* __restrict__ brim1,
    const TA* __restrict__ shared_out, TA* __restrict__ y_sfd, TA* __restrict__ y,
    unsigned* err) {
  combine_body<TA, KMAX, false>(o_epd, T, d, P, R, L, cap, tk, brim0, brim1, shared_out, y_sfd,
                                y, err, nullptr);
}
// Return rows only, each written into its source rank's buffer.
template <typename TA, int KMAX>
__global__ void __launch_bounds__(kMoverWarps * 32) combine_peer_kernel(
    const TA* __restrict__ o_epd, int T, int d, int P, int R, int L, size_t cap, int tk,
    const int32_t* __restrict__ brim0, const int32_t* __restrict__ brim1, unsigned* err,
    const __grid_constant__ EpPeers peers) {
  combine_body<TA, KMAX, true>(o_epd, T, d, P, R, L, cap, tk, brim0, brim1, nullptr, nullptr,
                               nullptr, err, &peers);
}

// The combine through the copy engine.  A unit is (token, piece of its row);
// per unit, lane 0 loads the piece of each of the token's expert rows into the
// warp's input stage with one cp.async.bulk each (the next unit's loads are in
// flight while this one is summed), every lane sums its 16-byte columns in
// fp32 per rank, and the return pieces and the output piece are written to
// the warp's output stage and stored with one cp.async.bulk each.  Per warp:
// two input stages of KMAX x piece bytes and one output stage of
// (KMAX + 1) x piece bytes, carved from dynamic shared memory.
template <typename TA, int KMAX>
__global__ void __launch_bounds__(kBulkWarps * 32) combine_bulk_kernel(
    const TA* __restrict__ o_epd, int T, int d, int piece_elems, int n_pieces, int R, int L,
    size_t cap, int tk, const int32_t* __restrict__ brim0, const int32_t* __restrict__ brim1,
    const TA* __restrict__ shared_out, TA* __restrict__ y_sfd, TA* __restrict__ y,
    unsigned* err, uint64_t wait_limit_ns) {
  constexpr int VN = Vec16<TA>::n;
  extern __shared__ __align__(128) uint8_t bulk_smem[];
  __shared__ __align__(8) uint64_t bars[kBulkWarps][2];
  __shared__ WarpDst sdst[kBulkWarps][2];
  __shared__ int abort_flag;
  const int wib = threadIdx.x >> 5;
  const unsigned lane = lane_id();
  if (threadIdx.x == 0) abort_flag = 0;
  if (lane == 0)
    for (int b = 0; b < 2; ++b) tc::mbar_init(tc::smem_u32(&bars[wib][b]), 1);
  tc::mbar_init_fence();
  __syncthreads();
  pdl_enter();
  const tc::WaitCtl wctl{&abort_flag, err, wait_limit_ns};
  const int piece_bytes = piece_elems * (int)sizeof(TA);
  const size_t warp_bytes = (size_t)(3 * KMAX + 1) * piece_bytes;
  uint8_t* in_stage = bulk_smem + (size_t)wib * warp_bytes;  // [2][KMAX][piece]
  uint8_t* out_stage = in_stage + (size_t)2 * KMAX * piece_bytes;  // [KMAX + 1][piece]
  const long long n_units = (long long)T * n_pieces;
  const long long stride = (long long)gridDim.x * kBulkWarps;
  const long long first = (long long)blockIdx.x * kBulkWarps + wib;
  const long long mine = first < n_units ? (n_units - first + stride - 1) / stride : 0;
  auto unit_of = [&](long long i, int& t, int& c0, int& n) {
    const long long u = first + i * stride;
    t = (int)(u / n_pieces);
    c0 = (int)(u - (long long)t * n_pieces) * piece_elems;
    n = min(piece_elems, d - c0);
  };
  // lane 0: the expert pieces of unit i into input stage i % 2
  auto issue_loads = [&](long long i) {
    int t, c0, n;
    unit_of(i, t, c0, n);
    const WarpDst& w = sdst[wib][i & 1];
    const int n_p = min(w.n_p, KMAX);
    const uint32_t bar = tc::smem_u32(&bars[wib][i & 1]);
    const uint32_t bytes = (uint32_t)(n * (int)sizeof(TA));
    tc::mbar_arrive_expect_tx(bar, bytes * (uint32_t)n_p);
    uint8_t* st = in_stage + (size_t)(i & 1) * KMAX * piece_bytes;
    for (int j = 0; j < n_p; ++j)
      tc::bulk_load(tc::smem_u32(st + (size_t)j * piece_bytes), o_epd + (size_t)w.p[j] * d + c0,
                    bytes, bar);
  };
  if (mine > 0) {
    int t, c0, n;
    unit_of(0, t, c0, n);
    collect_dst(brim0, brim1, t, T, R, L, cap, tk, sdst[wib][0], err);
    if (lane == 0) issue_loads(0);
  }
  bool ok = true;
  long long i = 0;
  for (; i < mine; ++i) {
    int t, c0, n;
    unit_of(i, t, c0, n);
    if (i + 1 < mine) {  // the next unit's destinations and loads (its stage was freed below)
      int t1, c1, n1;
      unit_of(i + 1, t1, c1, n1);
      collect_dst(brim0, brim1, t1, T, R, L, cap, tk, sdst[wib][(i + 1) & 1], err);
      if (lane == 0) issue_loads(i + 1);
    }
    ok = tc::wait_bounded(tc::smem_u32(&bars[wib][i & 1]), (uint32_t)((i >> 1) & 1), wctl);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) break;
    const WarpDst& w = sdst[wib][i & 1];
    const int n_p = min(w.n_p, KMAX);
    const uint8_t* st = in_stage + (size_t)(i & 1) * KMAX * piece_bytes;
    if (lane == 0) tc::bulk_wait_read_all();  // the output stage's last stores have read it
    __syncwarp();
    int n_ret = 0;  // return pieces written to the output stage
    int ret_row[KMAX];
    for (int c = (int)lane * VN; c < n; c += 32 * VN) {
      float acc[VN], ya[VN];
#pragma unroll
      for (int e = 0; e < VN; ++e) ya[e] = acc[e] = 0.f;
      int nr = 0;
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        if (j < n_p) {
          float f[VN];
          Vec16<TA>::to_f32(ld_v4(st + (size_t)j * piece_bytes + c * sizeof(TA)), f);
#pragma unroll
          for (int e = 0; e < VN; ++e) acc[e] += f[e];
          if (j + 1 == n_p || w.p_sfd[j + 1 < KMAX ? j + 1 : j] != w.p_sfd[j]) {
            const uint4 packed = Vec16<TA>::from_f32(acc);
            st_v4(out_stage + (size_t)nr * piece_bytes + c * sizeof(TA), packed);
            ret_row[nr] = w.p_sfd[j];
            ++nr;
            float r[VN];
            Vec16<TA>::to_f32(packed, r);
#pragma unroll
            for (int e = 0; e < VN; ++e) {
              ya[e] += r[e];
              acc[e] = 0.f;
            }
          }
        }
      }
      n_ret = nr;
      if (y) {
        if (shared_out) {
          float f[VN];
          Vec16<TA>::to_f32(ld_nc_v4(shared_out + (size_t)t * d + c0 + c), f);
#pragma unroll
          for (int e = 0; e < VN; ++e) ya[e] += f[e];
        }
        st_v4(out_stage + (size_t)KMAX * piece_bytes + c * sizeof(TA), Vec16<TA>::from_f32(ya));
      }
    }
    tc::fence_proxy_async_smem();  // this lane's stage writes, before the copy engine reads them
    __syncwarp();
    if (lane == 0) {
      // lane 0 always handles column 0 (n >= VN), so its n_ret and ret_row are the warp's
      const uint32_t bytes = (uint32_t)(n * (int)sizeof(TA));
      const uint32_t ob = tc::smem_u32(out_stage);
      if (y_sfd)
        for (int r = 0; r < n_ret; ++r)
          tc::bulk_store(y_sfd + (size_t)ret_row[r] * d + c0, ob + (uint32_t)(r * piece_bytes),
                         bytes);
      if (y)
        tc::bulk_store(y + (size_t)t * d + c0, ob + (uint32_t)(KMAX * piece_bytes), bytes);
      tc::bulk_commit_group();
    }
    __syncwarp();
  }
  if (!ok && lane == 0) {
    // leave no load in flight: units i and i + 1 had their loads issued (bounded waits)
    for (long long j = i; j <= i + 1 && j < mine; ++j)
      tc::wait_bounded(tc::smem_u32(&bars[wib][j & 1]), (uint32_t)((j >> 1) & 1), wctl, false);
  }
  if (lane == 0) tc::bulk_wait_all();
  __syncwarp();
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
