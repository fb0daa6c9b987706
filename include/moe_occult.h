/*
 * moe_occult.h -- C ABI of the Occult-style MoE layer hot path on B200 (sm_100a).
 *
 * One mixture-of-experts layer on one GPU, done the way the Occult paper
 * ("Occult: Optimizing Collaborative Communication across Experts for
 * Accelerated Parallel MoE Training and Inference") lays it out:
 *
 *   route        each token picks its top-k experts       moe_route_topk
 *   BRIM build   BRIM_0 [R x T], BRIM_1 [L x C_T], C_T     moe_brim_build
 *   dispatch     ORI -> SFD (one row per token and rank)   moe_dispatch_gather
 *                SFD -> EPD (one row per token and expert)
 *   experts      grouped SwiGLU FFN on the EPD rows        moe_expert_ffn
 *   combine      per-rank pre-reduce (intra-collaboration) moe_combine_scatter
 *                then scatter back to ORI order
 *
 * plus a placement-aware dispatched-row counter and an expert co-activation
 * histogram for correlated placement ("Expert Coupling in MoE Pretraining",
 * Abstract).  R expert-parallel ranks are simulated: they are partitions of
 * the expert set on this one GPU, and the SFD segments stand for what an
 * all-to-all would carry.  Nothing here moves data between GPUs.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every function returns an int status (moe_status).  On failure,
 *    moe_last_error() gives a message for the calling host thread.
 *  - Pointers are DEVICE pointers unless a parameter says "host".  The caller
 *    owns every buffer; no entry point allocates device memory.  Scratch
 *    space is passed in as a workspace whose size a *_workspace_size query
 *    gives.
 *  - Work is enqueued asynchronously on the caller's stream (NULL = legacy
 *    default stream); no entry point synchronises, except
 *    moe_get_device_status() and moe_layer_forward_host().
 *  - Arguments are validated on the host before anything is launched: a bad
 *    argument returns MOE_ERR_INVALID_ARG, an unsupported shape or dtype
 *    returns MOE_ERR_UNSUPPORTED, and nothing is enqueued in either case.
 *    Index values that live on the device (expert ids, BRIM entries) are
 *    range-checked by the kernels: an invalid one is skipped and raises the
 *    device error flag, which moe_get_device_status() reports.
 *  - Matrices are row-major and densely packed unless a stride is given.
 *  - Supported range: 1 <= E <= 256, 1 <= k <= min(E, 16), 1 <= R <= E,
 *    E % R == 0, d % 64 == 0, f % 64 == 0, T >= 0.
 *
 * Notation: T tokens, d model width, f expert FFN width, E routed experts,
 * k experts per token, R simulated EP ranks, L = E / R local experts per rank,
 * cap = T * min(k, R) (the largest possible C_T), slot_of[E] the placement
 * (a permutation of 0..E-1): expert e lives on rank slot_of[e] / L as local
 * expert slot_of[e] % L.
 */
#ifndef MOE_OCCULT_H
#define MOE_OCCULT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* the same type as cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1,  /* null pointer, negative size, bad enum */
  MOE_ERR_UNSUPPORTED = -2,  /* shape or dtype outside the supported range */
  MOE_ERR_CUDA = -3,         /* a CUDA runtime/driver call or launch failed */
  MOE_ERR_DEVICE_CHECK = -4, /* a kernel met an out-of-range index */
  MOE_ERR_TIMEOUT = -5       /* a bounded device-side wait expired */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;
typedef enum { MOE_FFN_SWIGLU = 0, MOE_FFN_IDENTITY = 1 } moe_ffn_kind;

/* Version of this ABI (incremented on any signature change). */
int moe_abi_version(void);

/* Message describing the last failure on the calling host thread ("" if none).
 * The string stays valid until the next call on the same thread. */
const char* moe_last_error(void);

/* Test-only knobs.  flags bit 0: the expert GEMM's producer skips its first
 * TMA load, so a bounded wait is certain to expire (exercises the timeout
 * path without faulting or hanging the GPU).  The other bits choose among the
 * library's equivalent kernel variants, for tests and measurements:
 *   2 single-CTA GEMMs, 4 CTA-pair GEMMs where the shape allows, 8 pair tiles
 *   with single-CTA tails, 16 the movers through TMA bulk copies, 32 the GEMM
 *   L2 policies and tile order of bits 20..27, 64 / 128 force / forbid the
 *   swapped-operand GEMM, 256 / 512 force / forbid 256 x 512 pair tiles,
 *   65536 pair GEMMs with one K chunk per stage only, 131072 weight-gradient
 *   pairs on 64-row stages only.
 * wait_limit_ms: how long a device-side wait may last before it gives up
 * (default 4000 ms).  Process wide; not for production use. */
int moe_set_debug(int flags, double wait_limit_ms);

/* Reads and clears the device error flag that the kernels raise, in one
 * atomic exchange enqueued on `stream` after its earlier work, then
 * synchronises `stream`.  Kernels still running on other streams may raise the
 * flag at any time; such a bit is never lost, it shows in this reading or in
 * the next one.  Returns MOE_ERR_TIMEOUT if a bounded wait expired,
 * MOE_ERR_DEVICE_CHECK if an index was out of range, else MOE_OK. */
int moe_get_device_status(moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_route_topk -- each token is routed to k of the E experts ("Expert
 * Coupling in MoE Pretraining", Abstract; top-2/4/6/8 in the Occult paper,
 * Figure 3).
 *   logits   [T, E] float32   router logits
 *   topk_idx [T, k] int32     out: expert ids in descending logit order; of
 *                              equal logits the lower id ranks first
 *                              (-0.0 and +0.0 compare equal)
 *   topk_w   [T, k] float32   out: gate weights.  renorm = 0: softmax over all
 *                              E logits, then the k selected entries;
 *                              renorm = 1: softmax over the k selected logits.
 * Logits must be finite; NaN gives unspecified (but in-range) ids.
 * ------------------------------------------------------------------------- */
int moe_route_topk(const float* logits, int T, int E, int k, int renorm,
                   int32_t* topk_idx, float* topk_w, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_prune_topk -- routing-score-based collaboration pruning (Occult paper,
 * TL;DR: two pruning schemes, routing-score-based and similarity-based, that
 * minimise the all-to-all budget C_T; Abstract: collaboration pruning
 * controllably minimises the cost).  In place, per token, on a top-k list in
 * descending score order:
 *   keep the first m distinct ranks met along the list (the ranks of the
 *   token's highest-scoring experts); every assignment on another rank becomes
 *   an empty slot (id -1, weight 0); the kept weights are rescaled so that
 *   their sum equals the sum before pruning.
 *   topk_idx [T, k] int32, topk_w [T, k] float32 (device, in place)
 *   m >= 1; m >= the token's number of distinct ranks leaves it unchanged.
 * An id of -1 is accepted everywhere downstream as an empty slot: the BRIM
 * build, the dispatch, the counter and the histogram skip it, and the EPD
 * state then has epd_off[E] <= T*k rows.
 * ------------------------------------------------------------------------- */
int moe_prune_topk(int32_t* topk_idx, float* topk_w, int T, int k, const int32_t* slot_of,
                   int E, int R, int m, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_brim_build -- the two bidirectional re-index matrices of the Occult
 * paper (Figure 5: BRIM_0 is [EP devices x ORI tokens], BRIM_1 is [local
 * experts per device x SFD tokens]) and the all-to-all budget C_T (TL;DR).
 * A token is sent once to every rank that holds at least one of its experts.
 *   topk_idx [T, k] int32   distinct expert ids per token, or -1 for an empty
 *                           slot (checked on device)
 *   topk_w   [T, k] float32 gate weights
 *   slot_of  [E] int32      placement (device)
 *   brim0    [R, T] int32   out: SFD row of (rank r, token t), or -1
 *   sfd_token[cap] int32    out: ORI token of each SFD row (first C_T used)
 *   sfd_off  [R+1] int32    out: first SFD row of each rank; sfd_off[R] = C_T
 *   brim1    [L, cap] int32 out: EPD row of (local expert l, SFD row s), or
 *                           -1; row stride cap; columns >= C_T are not written
 *   epd_off  [E+1] int32    out: first EPD row of each slot (slot order)
 *   epd_sfd  [T*k] int32    out: SFD row feeding each EPD row
 *   epd_gate [T*k] float32  out: gate weight of each EPD row
 *   c_t      [1] int32      out: C_T, the number of SFD rows
 *   ws, ws_bytes            scratch, at least moe_brim_workspace_size(T, E, R)
 * Inside a rank's SFD segment and inside an expert's EPD group, rows follow
 * ascending token order, so every output is unique and reproducible.
 * ------------------------------------------------------------------------- */
size_t moe_brim_workspace_size(int T, int E, int R);
int moe_brim_build(const int32_t* topk_idx, const float* topk_w, int T, int k,
                   const int32_t* slot_of, int E, int R,
                   int32_t* brim0, int32_t* sfd_token, int32_t* sfd_off,
                   int32_t* brim1, int32_t* epd_off, int32_t* epd_sfd,
                   float* epd_gate, int32_t* c_t,
                   void* ws, size_t ws_bytes, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_brim_build_noalloc -- the same BRIM build as moe_brim_build, for callers
 * that must not allocate device memory at all.  It has no counterpart in the
 * paper; it exists for the host side of this library.
 * Who needs it: code embedded in a host framework that owns every byte of
 * device memory through its own pool (a raw cudaMalloc would bypass that
 * pool's accounting and limits), and code on a latency-critical path where
 * cudaMalloc / cudaFree are off limits because they can synchronise the
 * device and stall unrelated streams.  Such callers may also have no
 * workspace to lend, so this entry point takes none.
 * Scratch: a fixed array of 1 MiB (262144 int32) in this library's device
 * memory, reserved on every GPU that loads the library until the process
 * exits.  A call needs (ceil(T / 32) + 1) * (R + E) entries of it (T <= 116k tokens
 * at E = 64, R = 8); a larger call returns MOE_ERR_UNSUPPORTED and enqueues
 * nothing.  The passes overwrite
 * every scratch entry they read, so nothing has to be cleared between calls.
 * All calls on a device share the one array: calls that may run on the GPU at
 * the same time (e.g. on two streams without ordering) race on it and must be
 * serialised by the caller.
 * Set-up: the first call on each device looks up the array's device address
 * with that device current; make that first call before any stream capture.
 * The call allocates nothing: no cudaMalloc, no cudaFree.
 * Arguments and outputs are those of moe_brim_build, without ws / ws_bytes.
 * ------------------------------------------------------------------------- */
int moe_brim_build_noalloc(const int32_t* topk_idx, const float* topk_w, int T, int k,
                           const int32_t* slot_of, int E, int R,
                           int32_t* brim0, int32_t* sfd_token, int32_t* sfd_off,
                           int32_t* brim1, int32_t* epd_off, int32_t* epd_sfd,
                           float* epd_gate, int32_t* c_t, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_route_brim -- moe_route_topk, moe_brim_build, moe_count_dispatched_rows
 * and moe_coact_histogram in three kernel launches instead of six, with no
 * memset: one block per 32-token tile routes its tokens (the code of
 * moe_route_topk) and builds the tile's BRIM column masks; then one block per
 * column scans that column, the rank columns also counting the tokens their
 * own rank receives; a third kernel scatters BRIM_0 / BRIM_1 and their
 * inverses, writes the counter from the column totals, and has more blocks
 * that add the histogram from the masks, 128 or 256 tokens each (tokens on
 * both experts: the popcount of the AND of their columns).  Every output is bit for bit the one
 * the separate entry points produce.
 *   prune_m > 0 applies moe_prune_topk with m = prune_m between routing and
 *   the BRIMs (0 = no pruning);
 *   other arguments as in those entry points; per_rank / total / remote are given
 *   together or all NULL (counter skipped); hist may be NULL (histogram
 *   skipped), else it is cleared first unless hist_accumulate != 0.
 *   ws  at least moe_route_brim_workspace_size(T, E, R) bytes, 16-byte aligned
 * ------------------------------------------------------------------------- */
size_t moe_route_brim_workspace_size(int T, int E, int R);
int moe_route_brim(const float* logits, int T, int E, int k, int renorm, const int32_t* slot_of,
                   int R, int prune_m, int32_t* topk_idx, float* topk_w, int32_t* brim0, int32_t* sfd_token,
                   int32_t* sfd_off, int32_t* brim1, int32_t* epd_off, int32_t* epd_sfd,
                   float* epd_gate, int32_t* c_t, int32_t* per_rank, int64_t* total,
                   int64_t* remote, uint32_t* hist, int hist_accumulate, void* ws,
                   size_t ws_bytes, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_dispatch_gather -- ORI -> SFD -> EPD (Occult paper, Figure 4), guided by
 * the BRIMs: for every token t and rank r with s = BRIM_0[r][t] >= 0,
 *   x_sfd[s] = x[t]                         (the simulated all-to-all payload)
 * and for every local expert l with p = BRIM_1[l][s] >= 0,
 *   x_epd[p] = x[t]                         (the expert-partitioned rows).
 * Rows are copied bit for bit; each ORI row is read once.
 *   x     [T, d]   dtype
 *   x_sfd [cap, d] dtype  (may be NULL to skip it)
 *   x_epd [T*k, d] dtype  (may be NULL to skip it; not both NULL)
 * ------------------------------------------------------------------------- */
int moe_dispatch_gather(const void* x, int T, int d, int dtype, int k, int R, int L,
                        const int32_t* brim0, const int32_t* brim1,
                        void* x_sfd, void* x_epd, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_prepare_weights -- one-time repacking of routed expert weights for
 * moe_expert_ffn (not on the per-layer path):
 *   wg, wu [E, f, d], wd [E, d, f]  (expert-id order, dtype)
 *   slot_of [E] (device, may be NULL = identity placement)
 *   w_gu  [E, 2f, d] out: slot order; gate and up rows interleaved in blocks
 *                         of 64: rows 128i..128i+63 = gate rows 64i..64i+63,
 *                         rows 128i+64..128i+127 = up rows 64i..64i+63
 *   w_dn  [E, d, f]  out: slot order
 * moe_prepare_shared_weights packs S always-on experts (sg, su [S, fs, d],
 * sd [S, d, fs]) into ONE expert of width S*fs (gate/up rows concatenated over
 * the experts, then interleaved as above; down columns concatenated), whose
 * output is the sum of the S experts' outputs.  Requires (S*fs) % 64 == 0.
 * ------------------------------------------------------------------------- */
int moe_prepare_weights(const void* wg, const void* wu, const void* wd, int E, int d,
                        int f, int dtype, const int32_t* slot_of, void* w_gu, void* w_dn,
                        moe_stream_t stream);
int moe_prepare_shared_weights(const void* sg, const void* su, const void* sd, int S,
                               int d, int fs, int dtype, void* w_gu, void* w_dn,
                               moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_expert_ffn -- the expert computation of the Occult pipeline (TL;DR:
 * "sparse-matrix-multiplication pipeline"), as a grouped GEMM over ragged
 * row groups on the tcgen05 tensor cores:
 *   for every group g (rows group_off[g] .. group_off[g+1]-1, expert g):
 *     h   = silu(A Wg^T) * (A Wu^T)        [rows, f]  (kept in the workspace)
 *     out = row_scale * (h Wd^T)           [rows, d]
 *   a           [a_rows, d] dtype      the source rows
 *   a_row_index [m_cap] int32 or NULL  with it, GEMM row p reads a[a_row_index[p]]
 *                                      (e.g. the SFD payload with epd_sfd: the
 *                                      EPD rows are gathered on the fly by TMA and
 *                                      never stored); without it, row p is a[p]
 *                                      and a_rows must be >= m_cap
 *   group_off   [G+1] int32 (device)   ascending, group_off[0] >= 0,
 *                                      group_off[G] <= m_cap (violations are
 *                                      treated as empty groups and raise the
 *                                      device error flag)
 *   w_gu, w_dn                         packed by moe_prepare_weights (G experts)
 *   row_scale   [m_cap] float32        per-row factor (e.g. epd_gate), or NULL = 1
 *   ffn_kind    MOE_FFN_SWIGLU, or MOE_FFN_IDENTITY (out = row_scale * a; needs
 *               a_row_index == NULL; the weights are not read and may be NULL)
 *   out         [m_cap, d] dtype       rows outside every group are not written
 *   ws          at least moe_expert_ffn_workspace_size(m_cap, f, dtype) bytes
 * bf16 runs bf16 x bf16 -> fp32 MMAs; f32 runs TF32 MMAs (fp32 accumulate).
 * The hidden activation h is rounded to dtype between the two GEMMs.
 * Device-side waits are bounded: a wait that expires raises MOE_ERR_TIMEOUT
 * through moe_get_device_status() and the kernel returns.
 * ------------------------------------------------------------------------- */
size_t moe_expert_ffn_workspace_size(int m_cap, int f, int dtype);
int moe_expert_ffn(const void* a, int a_rows, const int32_t* a_row_index,
                   const int32_t* group_off, int G, int m_cap,
                   const void* w_gu, const void* w_dn, int d, int f, int dtype,
                   const float* row_scale, int ffn_kind, void* out,
                   void* ws, size_t ws_bytes, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_combine_scatter -- the return path (Occult paper, Figure 4, and the
 * intra-collaboration of the Abstract): for every SFD row s, its rank's
 * expert outputs are summed into ONE return row
 *   y_sfd[s] = sum over l ascending with BRIM_1[l][s] >= 0 of o_epd[BRIM_1[l][s]]
 * and every token sums its return rows back in ORI order
 *   y[t] = sum over r ascending with BRIM_0[r][t] >= 0 of y_sfd[BRIM_0[r][t]]
 *          (+ shared_out[t] when shared_out is not NULL).
 * Sums run in fp32; y_sfd is rounded to dtype (it is the payload), and y sums
 * the rounded payload rows.
 *   o_epd [T*k, d] dtype; y_sfd [cap, d] dtype (may be NULL); y [T, d] dtype;
 *   shared_out [T, d] dtype or NULL.
 * ------------------------------------------------------------------------- */
int moe_combine_scatter(const void* o_epd, int T, int d, int dtype, int k, int R, int L,
                        const int32_t* brim0, const int32_t* brim1,
                        const void* shared_out, void* y_sfd, void* y,
                        moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * Real expert parallelism (one process per GPU, R = the number of ranks).
 * Rank r holds the experts at slots r*L .. r*L+L-1 and the tokens of its own
 * batch.  The Occult paper's all-to-all (Abstract; Figure 2) then carries
 * the SFD segments to their ranks and the return rows back, and the count of
 * rows sent is the budget C_T.  The exchanges themselves are collectives of
 * the caller's process group; these are the device steps around them.
 *
 * Source rank, before the exchange: moe_route_brim (or route + brim build) on
 * its own T tokens gives BRIM_0, sfd_token, sfd_off (row counts per
 * destination: sfd_off[q+1] - sfd_off[q]) and C_T; moe_dispatch_gather with
 * x_epd = NULL writes the SFD rows; moe_ep_pack_routing writes, for each SFD
 * row, the token's top-k list restricted to the destination's experts.
 * Destination rank, after receiving n rows (source-major, then ascending
 * token: exactly its SFD segment of the single-GPU layer over the
 * concatenated batches): moe_brim_build over the n received rows with their
 * restricted lists gives its local BRIM_1 and EPD groups; moe_dispatch_gather
 * with x_sfd = NULL writes the EPD rows; moe_expert_ffn runs its L groups
 * (group_off = epd_off + r*L, G = L, its own packed weights);
 * moe_ep_return_rows sums each row's expert outputs into one return row.
 * Source rank, after the return exchange: moe_ep_combine sums every token's
 * returned rows in ORI order (+ the shared experts).
 * ------------------------------------------------------------------------- */

/* moe_ep_pack_routing -- for every SFD row s < C_T, with t = sfd_token[s] and
 * q the destination whose segment [sfd_off[q], sfd_off[q+1]) holds s:
 *   idx_send[s][j] = topk_idx[t][j] if that expert lives on rank q, else -1
 *   w_send[s][j]   = topk_w[t][j]   for the same entries, else 0
 *   topk_idx, topk_w [T, k]; slot_of [E]; sfd_token [cap]; sfd_off [R+1];
 *   c_t [1] (device); idx_send [cap, k] int32, w_send [cap, k] float32 out
 *   (rows >= C_T are not written).  Invalid ids raise the device error flag.
 * ------------------------------------------------------------------------- */
int moe_ep_pack_routing(const int32_t* topk_idx, const float* topk_w, int T, int k,
                        const int32_t* slot_of, int E, int R, const int32_t* sfd_token,
                        const int32_t* sfd_off, const int32_t* c_t, int32_t* idx_send,
                        float* w_send, moe_stream_t stream);

/* moe_ep_return_rows -- the destination's intra-collaboration pre-reduce
 * (Occult paper, Abstract): for every received row s (here the T "tokens"
 * of the local BRIM build are the received rows),
 *   y_ret[s] = sum over l ascending with BRIM_1[l][s] >= 0 of o_epd[BRIM_1[l][s]]
 * in fp32, rounded to dtype.  Arguments as moe_combine_scatter (brim0, brim1
 * of the local build); y_ret [T*min(k,R), d].  Nothing is written in ORI order.
 * ------------------------------------------------------------------------- */
int moe_ep_return_rows(const void* o_epd, int T, int d, int dtype, int k, int R, int L,
                       const int32_t* brim0, const int32_t* brim1, void* y_ret,
                       moe_stream_t stream);

/* moe_ep_combine -- the source's combine of the returned rows: y_ret holds
 * one row per SFD row of the source's build (the return exchange delivers
 * them in the order the SFD rows were sent), and
 *   y[t] = sum over q ascending with BRIM_0[q][t] >= 0 of y_ret[BRIM_0[q][t]]
 *          (+ shared_out[t] when not NULL), fp32 sums rounded to dtype.
 *   y_ret [T*min(k,R), d]; brim0 [R, T]; shared_out [T, d] or NULL; y [T, d].
 * ------------------------------------------------------------------------- */
int moe_ep_combine(const void* y_ret, int T, int d, int dtype, int k, int R,
                   const int32_t* brim0, const void* shared_out, void* y, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * The same exchange without a collective: the movers write every row straight
 * into the buffer of the rank that receives it (peer memory: on a multi-GPU
 * node, the other processes' buffers mapped into this one, reached over
 * NVLink; within one process, plain device buffers).  The caller owns the
 * ordering between ranks: before a send every destination's receive buffers
 * must be free, and a rank may read what it received only once every sender's
 * kernel has completed (a stream synchronisation on each rank and a host
 * barrier between them, or one stream for ranks in one process).
 *
 * moe_ep_peers -- one entry per rank q < R (MOE_EP_MAX_PEERS at most):
 *   rows[q]  the rank's row buffer (dtype rows of d elements)
 *   idx[q]   its routing-list buffer (k int32 per row), or NULL
 *   w[q]     its gate buffer (k float32 per row), or NULL
 *   row0[q]  this rank's row i for q lands at row row0[q] + i there
 *   seg[0..R] (moe_ep_return_peer) the owners of this rank's own rows: row i
 *            belongs to rank q when seg[q] <= i < seg[q+1]
 * Passed by value to the kernels (the struct is read on the host only).
 * ------------------------------------------------------------------------- */
#define MOE_EP_MAX_PEERS 64
typedef struct moe_ep_peers {
  void* rows[MOE_EP_MAX_PEERS];
  int32_t* idx[MOE_EP_MAX_PEERS];
  float* w[MOE_EP_MAX_PEERS];
  int64_t row0[MOE_EP_MAX_PEERS];
  int32_t seg[MOE_EP_MAX_PEERS + 1];
} moe_ep_peers;

/* moe_ep_send_peer -- the source's send: moe_dispatch_gather (SFD rows) and
 * moe_ep_pack_routing fused with the transfer.  Every SFD row s of this rank's
 * build, for destination q (its segment of sfd_off), is written to row
 * peers->row0[q] + s of peers->rows[q], and its restricted routing list to the
 * same row of peers->idx[q] and peers->w[q].  With row0[q] = (the first row of
 * this source's segment in q's receive buffer) - sfd_off[q], each destination
 * gets exactly the rows the all-to-all would deliver.  x [T, d]; topk_idx,
 * topk_w [T, k]; slot_of [E]; brim0 [R, T], brim1 [L, cap], sfd_token, sfd_off,
 * c_t of this rank's build (device).  Bad indices raise the device error flag.
 * ------------------------------------------------------------------------- */
int moe_ep_send_peer(const void* x, int T, int d, int dtype, int k, int R, int L,
                     const int32_t* topk_idx, const float* topk_w, const int32_t* slot_of,
                     const int32_t* brim0, const int32_t* brim1, const int32_t* sfd_token,
                     const int32_t* sfd_off, const int32_t* c_t, const moe_ep_peers* peers,
                     moe_stream_t stream);

/* moe_ep_return_peer -- the destination's pre-reduce (moe_ep_return_rows)
 * fused with the return transfer: the return row of received row s, whose
 * source q is found by peers->seg, is written to row peers->row0[q] + s of
 * peers->rows[q].  With seg = the first received row of each source and
 * row0[q] = (q's sfd_off[this rank]) - seg[q], every source gets its rows at
 * its own SFD positions, ready for moe_ep_combine.  Other arguments as
 * moe_ep_return_rows (T = the received rows; brim0, brim1 of the local build).
 * ------------------------------------------------------------------------- */
int moe_ep_return_peer(const void* o_epd, int T, int d, int dtype, int k, int R, int L,
                       const int32_t* brim0, const int32_t* brim1, const moe_ep_peers* peers,
                       moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_count_dispatched_rows -- rows a once-per-rank dispatcher sends under a
 * placement ("Expert Coupling in MoE Pretraining", Abstract), without
 * building BRIMs:
 *   per_rank [R] int32  out: tokens sent to each rank
 *   total    [1] int64  out: sum of per_rank (= C_T)
 *   remote   [1] int64  out: rows whose rank differs from the token's source
 *                            rank floor(t * R / T)
 * ------------------------------------------------------------------------- */
int moe_count_dispatched_rows(const int32_t* topk_idx, int T, int k,
                              const int32_t* slot_of, int E, int R,
                              int32_t* per_rank, int64_t* total, int64_t* remote,
                              moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_coact_histogram -- expert co-activation counts for correlated placement
 * ("Expert Coupling in MoE Pretraining", Abstract; "collaborated" experts in
 * the Occult paper, Abstract):
 *   hist [E, E] uint32: hist[a][b] (a != b) = tokens that selected both a and
 *   b; hist[a][a] = tokens that selected a.  accumulate = 0 clears it first.
 * ------------------------------------------------------------------------- */
int moe_coact_histogram(const int32_t* topk_idx, int T, int k, int E, uint32_t* hist,
                        int accumulate, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_place_greedy -- correlated expert placement from a co-activation
 * histogram ("Expert Coupling in MoE Pretraining", Abstract: experts that are
 * often selected together go on the same GPU; Occult paper, TL;DR:
 * expert-placement rescheduling).  HOST function (no GPU work):
 *   hist    [E, E] uint32, HOST memory (e.g. moe_coact_histogram of a
 *           calibration batch, copied back)
 *   slot_of [E] int32, HOST memory, out: the placement
 * Ranks are filled one after another: a rank is seeded with the unplaced
 * expert selected by the most tokens (hist[a][a]; ties -> lower id), then
 * grows by the unplaced expert with the largest co-activation count with the
 * rank's members (ties -> larger hist[b][b], then lower id) until it holds L
 * experts; slots inside a rank follow that order.
 * ------------------------------------------------------------------------- */
int moe_place_greedy(const uint32_t* hist, int E, int R, int32_t* slot_of);

/* ---------------------------------------------------------------------------
 * moe_layer_forward -- the whole layer in one call, every step of the hot
 * path in order on `stream`: moe_route_topk, moe_brim_build,
 * moe_dispatch_gather, moe_expert_ffn (routed experts over the EPD groups,
 * then the S shared experts over the ORI rows), moe_combine_scatter,
 * moe_count_dispatched_rows and moe_coact_histogram.
 *   logits [T, E] f32, x [T, d] dtype, y [T, d] dtype  (device)
 *   slot_of [E] int32 (device) placement used to pack w_gu / w_dn
 *   w_gu, w_dn   routed weights packed by moe_prepare_weights with slot_of
 *   sw_gu, sw_dn shared weights packed by moe_prepare_shared_weights
 *                (S shared experts of width fs; NULL when S = 0)
 *   stats        optional device outputs, each may be NULL:
 *                c_t [1] int32; per_rank [R] int32, total [1] int64,
 *                remote [1] int64 (the dispatched-row counter);
 *                hist [E, E] uint32 (the co-activation histogram is ADDED
 *                to it).  Outputs left NULL are still computed, into the
 *                workspace.
 *   ws           at least moe_layer_workspace_size(...) bytes, 256-byte aligned;
 *                it holds every intermediate state (top-k, BRIMs, SFD / EPD
 *                rows, return rows) for the duration of the call
 * prune_m > 0 prunes each token to its first prune_m ranks (moe_prune_topk)
 * before the BRIMs are built; 0 keeps every assignment.
 * With one expert per rank (E == R) the GEMM reads the SFD payload in place
 * (the EPD state equals it row for row); otherwise the dispatch stores the
 * EPD rows.
 * moe_layer_forward_host -- the same, with logits, x and y in HOST memory
 * (pinned memory makes the copies asynchronous DMA): copies logits and x to
 * device staging in the workspace, runs the layer, copies y back and
 * synchronises `stream` before returning (one cudaMemcpyAsync per buffer).
 * ------------------------------------------------------------------------- */
size_t moe_layer_workspace_size(int T, int d, int f, int E, int k, int R, int S, int fs,
                                int dtype, int host_staging);
int moe_layer_forward(int T, int d, int f, int E, int k, int R, int renorm, int prune_m, int S,
                      int fs, int dtype, const float* logits, const void* x, const int32_t* slot_of,
                      const void* w_gu, const void* w_dn, const void* sw_gu, const void* sw_dn,
                      void* y, int32_t* c_t, int32_t* per_rank, int64_t* total, int64_t* remote,
                      uint32_t* hist, void* ws, size_t ws_bytes, moe_stream_t stream);
int moe_layer_forward_host(int T, int d, int f, int E, int k, int R, int renorm, int prune_m,
                           int S, int fs, int dtype, const float* h_logits, const void* h_x,
                           const int32_t* slot_of, const void* w_gu, const void* w_dn,
                           const void* sw_gu, const void* sw_dn, void* h_y,
                           void* ws, size_t ws_bytes, moe_stream_t stream);
/* moe_layer_forward_host_async -- moe_layer_forward_host without the final
 * synchronisation: everything (both copies in, the layer, the copy out) is
 * enqueued on `stream` and the call returns.  The host buffers (pinned) and
 * the workspace must stay untouched until the stream has passed this work.
 * With two workspaces on two streams, one batch's copies overlap another
 * batch's layer. */
int moe_layer_forward_host_async(int T, int d, int f, int E, int k, int R, int renorm,
                                 int prune_m, int S, int fs, int dtype, const float* h_logits,
                                 const void* h_x, const int32_t* slot_of, const void* w_gu,
                                 const void* w_dn, const void* sw_gu, const void* sw_dn,
                                 void* h_y, void* ws, size_t ws_bytes, moe_stream_t stream);

/* ===========================================================================
 * Token shuffling across layers ("Expert Coupling in MoE Pretraining",
 * Abstract): the experts a token selects at one layer predict the experts it
 * selects at the next, so each token can be moved to the rank predicted to
 * hold its next-layer experts (in a real system during the reduce-scatter
 * after attention).  On one GPU the statistics, the prediction, the new token
 * order and the row movement are computed; the share of next-layer
 * assignments served on the token's home rank measures the effect.
 * ========================================================================= */

/* moe_interlayer_histogram -- hist [E, E] uint32 (device):
 *   hist[a][b] += #tokens t with a in idx_l[t] and b in idx_next[t]
 * (both [T, k] int32; -1 = empty slot, counts nothing; other ids outside
 * [0, E) raise MOE_ERR_DEVICE_CHECK).  accumulate = 0 clears hist first.  A
 * calibration statistic, like the co-activation histogram. */
int moe_interlayer_histogram(const int32_t* idx_l, const int32_t* idx_next, int T, int k, int E,
                             uint32_t* hist, int accumulate, moe_stream_t stream);

/* moe_rank_affinity -- table [E, R] uint32 (device):
 *   table[a][r] = sum of hist[a][b] over the experts b that rank r holds at
 *                 the next layer (slot_of_next[b] / (E / R) == r).
 * Sums are 32-bit: the histogram's total must stay below 2^32. */
int moe_rank_affinity(const uint32_t* hist, int E, const int32_t* slot_of_next, int R,
                      uint32_t* table, moe_stream_t stream);

/* moe_predict_home -- home [T] int32 (device): the rank r maximising
 * sum_j table[idx_l[t][j]][r] (ties: the lower r); a token whose scores are all
 * zero keeps its contiguous home floor(t * R / T).  One warp per token. */
int moe_predict_home(const int32_t* idx_l, int T, int k, int E, const uint32_t* table, int R,
                     int32_t* home, moe_stream_t stream);

/* moe_count_local -- out [2] int64 (device): out[0] = assignments in idx [T, k]
 * whose expert sits on the token's home rank (home [T], or NULL for the
 * contiguous home floor(t * R / T)); out[1] = all assignments (-1 slots
 * excluded).  The share out[0] / out[1] is what token shuffling raises. */
int moe_count_local(const int32_t* idx, int T, int k, const int32_t* slot_of, int E, int R,
                    const int32_t* home, int64_t* out, moe_stream_t stream);

/* moe_token_shuffle -- the tokens in home-rank order:
 *   perm [T] int32       perm[i] = the token at position i (ascending token
 *                        order within each rank's segment)
 *   rank_off [R+1] int32 where each rank's segment starts; rank_off[R] = T
 *   inv [T] int32        (may be NULL) inv[t] = the position of token t
 *   x_out [T, d]         (x may be NULL to skip) x_out[i] = x[perm[i]], rows of
 *                        dtype, bit for bit
 * home values must lie in [0, R).  The order is a BRIM_0 over one "expert" per
 * rank (the BRIM passes with k = 1, E = R); the rows move one warp per row.
 *   ws  at least moe_token_shuffle_workspace_size(T, R) bytes, 16-byte aligned */
size_t moe_token_shuffle_workspace_size(int T, int R);
int moe_token_shuffle(const int32_t* home, int T, int R, const void* x, int d, int dtype,
                      void* x_out, int32_t* perm, int32_t* rank_off, int32_t* inv, void* ws,
                      size_t ws_bytes, moe_stream_t stream);

/* ===========================================================================
 * Training: forward that keeps what the backward needs, and the backward.
 *
 * The backward is the exact derivative of the layer for fixed expert choices:
 * the top-k selection passes no gradient, and each gate weight passes its
 * gradient through the softmax it came from (renorm 0: over all E logits;
 * renorm 1: over the k selected ones).  Data moves through the same BRIMs as
 * in the forward ("bidirectional re-index", Occult paper, Figure 4): the
 * upstream gradient travels ORI -> SFD -> EPD like x did (moe_dispatch_gather)
 * and the input gradient returns EPD -> SFD -> ORI like y did
 * (moe_combine_scatter).  Training is bf16 only (MOE_BF16 activations and
 * weights) and defined for unpruned routing; d must be a multiple of 128.
 * ========================================================================= */

/* ---------------------------------------------------------------------------
 * moe_expert_ffn_train -- moe_expert_ffn (SwiGLU) that also returns
 *   z  [m_cap, 2f] bf16  the gate/up pre-activations A W_gu^T, rounded to bf16,
 *                        in w_gu's packed column order (64-wide gate and up
 *                        blocks interleaved)
 *   h  [m_cap, f]  bf16  silu(z_gate) * z_up of those rounded values
 *   out [m_cap, d] bf16  row_scale * (h W_down^T)
 * Rows outside the groups are not written.  No workspace.  Arguments otherwise
 * as moe_expert_ffn (no row index: a's rows are the groups' rows).
 * ------------------------------------------------------------------------- */
int moe_expert_ffn_train(const void* a, int a_rows, const int32_t* group_off, int G, int m_cap,
                         const void* w_gu, const void* w_dn, int d, int f,
                         const float* row_scale, void* z, void* h, void* out,
                         moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_expert_ffn_backward -- gradients of moe_expert_ffn_train for the upstream
 * gradient dout [a_rows, d] (bf16, the same rows as a):
 *   dx          [m_cap, d] bf16   d/da                   (rows of the groups)
 *   d_row_scale [m_cap] f32       d/d row_scale, 0 on rows past the groups
 *                                 (may be NULL; requires row_scale)
 *   dw_gu       [G, 2f, d]        d/d w_gu, packed like w_gu   (may be NULL)
 *   dw_dn       [G, d, f]         d/d w_dn                     (may be NULL)
 * dw_dtype (MOE_F32 or MOE_BF16) is the type of dw_gu / dw_dn; accumulate = 1
 * adds to them instead of overwriting (an expert with no rows then leaves
 * them as they are; with accumulate = 0 it gets zeros).  z is the
 * moe_expert_ffn_train output.  Kernels: the input-gradient GEMM of the down
 * projection with the SwiGLU and gate backward fused into its epilogue, the
 * input-gradient GEMM of gate/up, and two weight-gradient GEMMs (tcgen05).
 *   ws  at least moe_expert_ffn_backward_workspace_size(m_cap, f) bytes,
 *       16-byte aligned
 * ------------------------------------------------------------------------- */
size_t moe_expert_ffn_backward_workspace_size(int m_cap, int f);
int moe_expert_ffn_backward(const void* dout, const void* a, int a_rows, const void* z,
                            const int32_t* group_off, int G, int m_cap, const void* w_gu,
                            const void* w_dn, int d, int f, const float* row_scale, void* dx,
                            float* d_row_scale, void* dw_gu, void* dw_dn, int dw_dtype,
                            int accumulate, void* ws, size_t ws_bytes, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_route_backward -- gradient of the router logits.  d_gate_epd [T*k] f32
 * holds the gradient of each gate weight in EPD order (moe_expert_ffn_backward's
 * d_row_scale); the row of token t's slot j is found through the BRIMs,
 * p = BRIM_1[loc(e)][BRIM_0[rank(e)][t]] with e = topk_idx[t][j].  With q the
 * softmax of the token's logits over the normalisation set of `renorm`,
 *   d_logits[t][e] = q_e * (dw(e) - sum_j dw_j w_j),   q_e = 0 off the set,
 * where dw(e) is the gradient of e's gate (0 if e was not selected).
 *   d_logits [T, E] f32 out;  d_topk_w [T, k] f32 out (may be NULL): dw_j
 * ------------------------------------------------------------------------- */
int moe_route_backward(const float* logits, int T, int E, int k, int renorm,
                       const int32_t* topk_idx, const int32_t* slot_of, int R,
                       const int32_t* brim0, const int32_t* brim1, const float* d_gate_epd,
                       float* d_logits, float* d_topk_w, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_layer_forward_train / moe_layer_backward -- the whole layer for
 * training.  moe_layer_forward_train is moe_layer_forward (no pruning, no
 * statistics outputs) that keeps in `ws` what moe_layer_backward needs: the
 * top-k, the BRIMs, the EPD rows and the expert pre-activations.
 * moe_layer_backward then takes the upstream gradient dy [T, d] and writes
 *   dx        [T, d] bf16     d/dx (routed experts + shared experts)
 *   d_logits  [T, E] f32      d/d logits
 *   d_topk_w  [T, k] f32      d/d the gate weights (may be NULL)
 *   dw_gu, dw_dn              d/d the routed weights, packed like w_gu / w_dn
 *                             (slot order), dw_dtype
 *   dsw_gu, dsw_dn            d/d the shared weights (packed), dw_dtype
 *                             (NULL when S = 0)
 * with the same arguments and the same `ws` as the forward call before it
 * (nothing else may use ws in between).  accumulate as in
 * moe_expert_ffn_backward.
 *   ws  at least moe_layer_train_workspace_size(...) bytes, 256-byte aligned
 * ------------------------------------------------------------------------- */
size_t moe_layer_train_workspace_size(int T, int d, int f, int E, int k, int R, int S, int fs);
int moe_layer_forward_train(int T, int d, int f, int E, int k, int R, int renorm, int S, int fs,
                            const float* logits, const void* x, const int32_t* slot_of,
                            const void* w_gu, const void* w_dn, const void* sw_gu,
                            const void* sw_dn, void* y, void* ws, size_t ws_bytes,
                            moe_stream_t stream);
int moe_layer_backward(int T, int d, int f, int E, int k, int R, int renorm, int S, int fs,
                       const float* logits, const void* x, const int32_t* slot_of,
                       const void* w_gu, const void* w_dn, const void* sw_gu, const void* sw_dn,
                       const void* dy, void* dx, float* d_logits, float* d_topk_w, void* dw_gu,
                       void* dw_dn, void* dsw_gu, void* dsw_dn, int dw_dtype, int accumulate,
                       void* ws, size_t ws_bytes, moe_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_OCCULT_H */
