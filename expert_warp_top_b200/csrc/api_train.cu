// api_train.cu -- the training entry points of the C ABI
// (include/moe_occult.h): the forward that keeps what the backward needs, the
// expert backward (input- and weight-gradient GEMMs), the routing backward
// and the whole-layer backward.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/moe_occult.h"
#include "backward.cuh"
#include "host.h"

using namespace moe_host;

namespace {

int check_train_ffn(int G, int m_cap, int a_rows, int d, int f) {
  MOE_REQUIRE(G >= 1 && G <= moe::kGemmMaxGroups, MOE_ERR_UNSUPPORTED,
              "G must be in [1, %d] (got %d)", moe::kGemmMaxGroups, G);
  MOE_REQUIRE(m_cap >= 0 && a_rows >= m_cap, MOE_ERR_INVALID_ARG,
              "a needs at least m_cap rows (a_rows=%d m_cap=%d)", a_rows, m_cap);
  MOE_REQUIRE(d >= 128 && d % 128 == 0, MOE_ERR_UNSUPPORTED,
              "training needs d a positive multiple of 128 (got %d)", d);
  MOE_REQUIRE(f >= 64 && f % 64 == 0, MOE_ERR_UNSUPPORTED, "f must be a positive multiple of 64");
  return MOE_OK;
}

// Gate-gradient partials per row: one per N block of the down-projection's
// input-gradient GEMM (N = f; BN as the launcher picks it).
int n_partials(int f) { return f / pick_bn(f); }

}  // namespace

extern "C" {

// ---------------------------------------------------------------------------
int moe_expert_ffn_train(const void* a, int a_rows, const int32_t* group_off, int G, int m_cap,
                         const void* w_gu, const void* w_dn, int d, int f,
                         const float* row_scale, void* z, void* h, void* out,
                         moe_stream_t stream) {
  int rc = check_train_ffn(G, m_cap, a_rows, d, f);
  if (rc) return rc;
  if (m_cap == 0) return MOE_OK;
  MOE_REQUIRE(a && group_off && w_gu && w_dn && z && h && out, MOE_ERR_INVALID_ARG,
              "null pointer");
  MOE_REQUIRE(aligned16(a) && aligned16(w_gu) && aligned16(w_dn) && aligned16(z) &&
                  aligned16(h) && aligned16(out),
              MOE_ERR_INVALID_ARG, "buffers must be 16-byte aligned");
  DeviceInfo* di;
  if ((rc = device_info(&di))) return rc;
  GemmExtra ex;
  ex.aux_out = z;
  ex.ld_aux = 2 * f;
  if ((rc = launch_gemm_auto<moe::kEpiSwiGLUSave, false>(di, a, a_rows, nullptr, m_cap, d, w_gu,
                                                         G, 2 * f, group_off, nullptr, h, f,
                                                         stream, ex)))
    return rc;
  return launch_gemm_auto<moe::kEpiScale, false>(di, h, m_cap, nullptr, m_cap, f, w_dn, G, d,
                                                 group_off, row_scale, out, d, stream);
}

// ---------------------------------------------------------------------------
size_t moe_expert_ffn_backward_workspace_size(int m_cap, int f) {
  if (m_cap < 0 || f < 64 || f % 64) return 0;
  const size_t m = (size_t)m_cap;
  return align256(m * 2 * f * 2) + align256(m * f * 2) +
         align256(m * (size_t)n_partials(f) * sizeof(float)) + 256;
}

int moe_expert_ffn_backward(const void* dout, const void* a, int a_rows, const void* z,
                            const int32_t* group_off, int G, int m_cap, const void* w_gu,
                            const void* w_dn, int d, int f, const float* row_scale, void* dx,
                            float* d_row_scale, void* dw_gu, void* dw_dn, int dw_dtype,
                            int accumulate, void* ws, size_t ws_bytes, moe_stream_t stream) {
  int rc = check_train_ffn(G, m_cap, a_rows, d, f);
  if (rc) return rc;
  MOE_REQUIRE(dw_dtype == MOE_F32 || dw_dtype == MOE_BF16, MOE_ERR_INVALID_ARG,
              "dw_dtype must be MOE_F32 or MOE_BF16");
  MOE_REQUIRE(accumulate == 0 || accumulate == 1, MOE_ERR_INVALID_ARG, "accumulate must be 0 or 1");
  MOE_REQUIRE(!d_row_scale || row_scale, MOE_ERR_INVALID_ARG,
              "d_row_scale needs the row_scale of the forward");
  MOE_REQUIRE(group_off && w_gu && w_dn, MOE_ERR_INVALID_ARG, "null pointer");
  const size_t wbytes = dw_dtype == MOE_F32 ? 4 : 2;
  if (m_cap == 0) {
    // every group is empty: the weight gradients are zero
    if (!accumulate) {
      if (dw_gu) MOE_CUDA(cudaMemsetAsync(dw_gu, 0, (size_t)G * 2 * f * d * wbytes, stream));
      if (dw_dn) MOE_CUDA(cudaMemsetAsync(dw_dn, 0, (size_t)G * d * f * wbytes, stream));
    }
    return MOE_OK;
  }
  MOE_REQUIRE(dout && a && z && dx && ws, MOE_ERR_INVALID_ARG, "null pointer");
  MOE_REQUIRE(aligned16(dout) && aligned16(a) && aligned16(z) && aligned16(dx) &&
                  aligned16(w_gu) && aligned16(w_dn) && aligned16(ws) &&
                  (!dw_gu || aligned16(dw_gu)) && (!dw_dn || aligned16(dw_dn)),
              MOE_ERR_INVALID_ARG, "buffers must be 16-byte aligned");
  const size_t need = moe_expert_ffn_backward_workspace_size(m_cap, f);
  MOE_REQUIRE(ws_bytes >= need, MOE_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes",
              ws_bytes, need);
  DeviceInfo* di;
  if ((rc = device_info(&di))) return rc;

  char* base = static_cast<char*>(ws);
  const size_t m = (size_t)m_cap;
  void* dz = base;                                         // [m_cap, 2f] bf16
  void* hg = base + align256(m * 2 * f * 2);               // [m_cap, f]  bf16: w * h
  float* partial = reinterpret_cast<float*>(static_cast<char*>(hg) + align256(m * f * 2));
  const int n_part = n_partials(f);

  // 1. dH' = dout W_down (B = W_down read MN-major), SwiGLU + gate backward fused
  GemmExtra ex;
  ex.aux_in = z;
  ex.aux_out = dz;
  ex.ld_aux = 2 * f;
  ex.partial = d_row_scale ? partial : nullptr;
  ex.n_part = n_part;
  if ((rc = launch_gemm_auto<moe::kEpiSwiGLUBwd, false, true>(di, dout, a_rows, nullptr, m_cap, d,
                                                              w_dn, G, f, group_off, row_scale,
                                                              hg, f, stream, ex)))
    return rc;
  // 2. dx = dZ W_gu (B = W_gu read MN-major)
  if ((rc = launch_gemm_auto<moe::kEpiScale, false, true>(di, dz, m_cap, nullptr, m_cap, 2 * f,
                                                          w_gu, G, d, group_off, nullptr, dx, d,
                                                          stream)))
    return rc;
  // 3. gate gradient: the partials of step 1 summed per row
  if (d_row_scale) {
    MOE_CUDA(launch_k(moe::row_partial_sum_kernel, dim3((m_cap + 255) / 256), dim3(256), 0,
                      stream, static_cast<const float*>(partial), n_part, m_cap, group_off, G,
                      d_row_scale));
    MOE_LAUNCHED("row_partial_sum_kernel");
  }
  // 4. weight gradients: dW_down[g] = dout_g^T (w h)_g, dW_gu[g] = dZ_g^T a_g
  if (dw_dn) {
    rc = dw_dtype == MOE_F32
             ? launch_wgrad<float>(di, dout, hg, m_cap, d, f, group_off, G, dw_dn, accumulate, stream)
             : launch_wgrad<__nv_bfloat16>(di, dout, hg, m_cap, d, f, group_off, G, dw_dn,
                                           accumulate, stream);
    if (rc) return rc;
  }
  if (dw_gu) {
    rc = dw_dtype == MOE_F32
             ? launch_wgrad<float>(di, dz, a, m_cap, 2 * f, d, group_off, G, dw_gu, accumulate,
                                   stream)
             : launch_wgrad<__nv_bfloat16>(di, dz, a, m_cap, 2 * f, d, group_off, G, dw_gu,
                                           accumulate, stream);
    if (rc) return rc;
  }
  return MOE_OK;
}

// ---------------------------------------------------------------------------
int moe_route_backward(const float* logits, int T, int E, int k, int renorm,
                       const int32_t* topk_idx, const int32_t* slot_of, int R,
                       const int32_t* brim0, const int32_t* brim1, const float* d_gate_epd,
                       float* d_logits, float* d_topk_w, moe_stream_t stream) {
  int rc = check_common(T, E, k, R);
  if (rc) return rc;
  MOE_REQUIRE(renorm == 0 || renorm == 1, MOE_ERR_INVALID_ARG, "renorm must be 0 or 1");
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(logits && topk_idx && slot_of && brim0 && brim1 && d_gate_epd && d_logits,
              MOE_ERR_INVALID_ARG, "null pointer");
  DeviceInfo* di;
  if ((rc = device_info(&di))) return rc;
  const size_t cap = (size_t)T * (k < R ? k : R);
  const long long n_epd = (long long)T * k;
  MOE_REQUIRE(n_epd <= INT32_MAX, MOE_ERR_UNSUPPORTED, "T * k too large");
  const dim3 grid((unsigned)(((long long)T * 32 + 255) / 256));
#define MOE_ROUTE_BWD(KM)                                                                    \
  MOE_CUDA(launch_k(moe::route_backward_kernel<KM>, grid, dim3(256), 0, stream, logits, T, E, \
                    k, renorm, topk_idx, slot_of, R, brim0, brim1, cap, d_gate_epd,          \
                    (int)n_epd, d_logits, d_topk_w, di->err_flag))
  if (k <= 2) MOE_ROUTE_BWD(2);
  else if (k <= 4) MOE_ROUTE_BWD(4);
  else if (k <= 8) MOE_ROUTE_BWD(8);
  else MOE_ROUTE_BWD(16);
#undef MOE_ROUTE_BWD
  MOE_LAUNCHED("route_backward_kernel");
  return MOE_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// The whole layer for training.  One workspace holds the forward's state and
// the backward's temporaries, each region 256-byte aligned.
namespace {

struct Carve {
  size_t off = 0;
  char* base = nullptr;
  template <typename T>
  T* take(size_t count) {
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += align256(sizeof(T) * (count ? count : 1));
    return p;
  }
};

struct TrainState {
  int32_t* topk_idx; float* topk_w;
  int32_t *brim0, *sfd_token, *sfd_off, *brim1, *epd_off, *epd_sfd; float* epd_gate;
  int32_t* c_t; void* brim_ws; size_t brim_ws_bytes;
  void *x_sfd, *x_epd, *o_epd, *y_sfd;   // o_epd / y_sfd carry dx_epd / dx_sfd in the backward
  void *z, *h;                           // routed experts' pre-activations and h
  void *shared_out, *zs, *hs; int32_t* shared_off;
  void *dy_sfd, *dy_epd, *dx_s; float* d_gate;
  void* bwd_ws; size_t bwd_ws_bytes; void* sbwd_ws; size_t sbwd_ws_bytes;
};

size_t carve_train(char* base, int T, int d, int f, int E, int k, int R, int S, int fs,
                   TrainState* out) {
  Carve c;
  c.base = base;
  TrainState s{};
  const size_t es = 2;
  const size_t cap = (size_t)T * (k < R ? k : R), tk = (size_t)T * k;
  const int L = E / R;
  s.topk_idx = c.take<int32_t>(tk);
  s.topk_w = c.take<float>(tk);
  s.brim0 = c.take<int32_t>((size_t)R * T);
  s.sfd_token = c.take<int32_t>(cap);
  s.sfd_off = c.take<int32_t>(R + 1);
  s.brim1 = c.take<int32_t>((size_t)L * cap);
  s.epd_off = c.take<int32_t>(E + 1);
  s.epd_sfd = c.take<int32_t>(tk);
  s.epd_gate = c.take<float>(tk);
  s.c_t = c.take<int32_t>(1);
  s.brim_ws_bytes = moe_route_brim_workspace_size(T, E, R);
  s.brim_ws = c.take<char>(s.brim_ws_bytes);
  s.x_sfd = c.take<char>(cap * d * es);
  s.x_epd = L > 1 ? c.take<char>(tk * d * es) : nullptr;
  s.o_epd = c.take<char>(tk * d * es);
  s.y_sfd = c.take<char>(cap * d * es);
  s.z = c.take<char>(tk * 2 * f * es);
  s.h = c.take<char>(tk * f * es);
  if (S > 0) {
    s.shared_out = c.take<char>((size_t)T * d * es);
    s.zs = c.take<char>((size_t)T * 2 * S * fs * es);
    s.hs = c.take<char>((size_t)T * S * fs * es);
    s.shared_off = c.take<int32_t>(2);
    s.dx_s = c.take<char>((size_t)T * d * es);
    s.sbwd_ws_bytes = moe_expert_ffn_backward_workspace_size(T, S * fs);
    s.sbwd_ws = c.take<char>(s.sbwd_ws_bytes);
  }
  s.dy_sfd = c.take<char>(cap * d * es);
  s.dy_epd = L > 1 ? c.take<char>(tk * d * es) : nullptr;
  s.d_gate = c.take<float>(tk);
  s.bwd_ws_bytes = moe_expert_ffn_backward_workspace_size((int)tk, f);
  s.bwd_ws = c.take<char>(s.bwd_ws_bytes);
  if (out) *out = s;
  return c.off + 256;
}

int check_train_layer(int T, int d, int f, int E, int k, int R, int renorm, int S, int fs) {
  int rc = check_common(T, E, k, R);
  if (rc) return rc;
  MOE_REQUIRE(renorm == 0 || renorm == 1, MOE_ERR_INVALID_ARG, "renorm must be 0 or 1");
  MOE_REQUIRE(d >= 128 && d % 128 == 0 && f >= 64 && f % 64 == 0, MOE_ERR_UNSUPPORTED,
              "training needs d a positive multiple of 128 and f of 64 (d=%d f=%d)", d, f);
  MOE_REQUIRE(S >= 0 && (S == 0 || (fs >= 64 && fs % 64 == 0)), MOE_ERR_UNSUPPORTED,
              "shared experts need fs a positive multiple of 64 (S=%d fs=%d)", S, fs);
  MOE_REQUIRE((long long)T * k <= INT32_MAX / 2, MOE_ERR_UNSUPPORTED, "T * k too large");
  return MOE_OK;
}

int train_state(int T, int d, int f, int E, int k, int R, int S, int fs, void* ws,
                size_t ws_bytes, TrainState* st) {
  MOE_REQUIRE(ws && aligned16(ws), MOE_ERR_INVALID_ARG, "workspace missing or misaligned");
  const size_t need = carve_train(nullptr, T, d, f, E, k, R, S, fs, nullptr);
  MOE_REQUIRE(ws_bytes >= need, MOE_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes",
              ws_bytes, need);
  char* base = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~uintptr_t(255));
  carve_train(base, T, d, f, E, k, R, S, fs, st);
  return MOE_OK;
}

}  // namespace

extern "C" {

size_t moe_layer_train_workspace_size(int T, int d, int f, int E, int k, int R, int S, int fs) {
  if (check_train_layer(T, d, f, E, k, R, 0, S, fs)) return 0;
  return carve_train(nullptr, T, d, f, E, k, R, S, fs, nullptr);
}

int moe_layer_forward_train(int T, int d, int f, int E, int k, int R, int renorm, int S, int fs,
                            const float* logits, const void* x, const int32_t* slot_of,
                            const void* w_gu, const void* w_dn, const void* sw_gu,
                            const void* sw_dn, void* y, void* ws, size_t ws_bytes,
                            moe_stream_t stream) {
  int rc = check_train_layer(T, d, f, E, k, R, renorm, S, fs);
  if (rc) return rc;
  TrainState st;
  if ((rc = train_state(T, d, f, E, k, R, S, fs, ws, ws_bytes, &st))) return rc;
  MOE_REQUIRE(S == 0 || (sw_gu && sw_dn), MOE_ERR_INVALID_ARG, "shared weights missing");
  if (T == 0) return MOE_OK;
  MOE_REQUIRE(logits && x && y && slot_of && w_gu && w_dn, MOE_ERR_INVALID_ARG, "null pointer");
  const int L = E / R;
  const int tk = T * k;
  if ((rc = moe_route_brim(logits, T, E, k, renorm, slot_of, R, 0, st.topk_idx, st.topk_w,
                           st.brim0, st.sfd_token, st.sfd_off, st.brim1, st.epd_off, st.epd_sfd,
                           st.epd_gate, st.c_t, nullptr, nullptr, nullptr, nullptr, 0,
                           st.brim_ws, st.brim_ws_bytes, stream)))
    return rc;
  if ((rc = moe_dispatch_gather(x, T, d, MOE_BF16, k, R, L, st.brim0, st.brim1, st.x_sfd,
                                st.x_epd, stream)))
    return rc;
  // with L = 1 the EPD state is the SFD state row for row: run on the payload
  const void* a = L > 1 ? st.x_epd : st.x_sfd;
  if ((rc = moe_expert_ffn_train(a, tk, st.epd_off, E, tk, w_gu, w_dn, d, f, st.epd_gate, st.z,
                                 st.h, st.o_epd, stream)))
    return rc;
  if (S > 0) {
    DeviceInfo* di;
    if ((rc = device_info(&di))) return rc;
    MOE_CUDA(launch_k(moe::set_two_kernel, 1, 1, 0, stream, st.shared_off, 0, T));
    MOE_LAUNCHED("set_two_kernel");
    if ((rc = moe_expert_ffn_train(x, T, st.shared_off, 1, T, sw_gu, sw_dn, d, S * fs, nullptr,
                                   st.zs, st.hs, st.shared_out, stream)))
      return rc;
  }
  return moe_combine_scatter(st.o_epd, T, d, MOE_BF16, k, R, L, st.brim0, st.brim1,
                             S > 0 ? st.shared_out : nullptr, st.y_sfd, y, stream);
}

int moe_layer_backward(int T, int d, int f, int E, int k, int R, int renorm, int S, int fs,
                       const float* logits, const void* x, const int32_t* slot_of,
                       const void* w_gu, const void* w_dn, const void* sw_gu, const void* sw_dn,
                       const void* dy, void* dx, float* d_logits, float* d_topk_w, void* dw_gu,
                       void* dw_dn, void* dsw_gu, void* dsw_dn, int dw_dtype, int accumulate,
                       void* ws, size_t ws_bytes, moe_stream_t stream) {
  int rc = check_train_layer(T, d, f, E, k, R, renorm, S, fs);
  if (rc) return rc;
  TrainState st;
  if ((rc = train_state(T, d, f, E, k, R, S, fs, ws, ws_bytes, &st))) return rc;
  MOE_REQUIRE(S == 0 || (sw_gu && sw_dn), MOE_ERR_INVALID_ARG, "shared weights missing");
  MOE_REQUIRE(w_gu && w_dn && slot_of, MOE_ERR_INVALID_ARG, "null pointer");
  const int L = E / R;
  const int tk = T * k;
  if (T == 0) {
    // no rows at all: zero weight gradients (unless accumulating)
    if ((rc = moe_expert_ffn_backward(nullptr, nullptr, 0, nullptr, st.epd_off, E, 0, w_gu, w_dn,
                                      d, f, nullptr, nullptr, nullptr, dw_gu, dw_dn, dw_dtype,
                                      accumulate, nullptr, 0, stream)))
      return rc;
    if (S > 0)
      return moe_expert_ffn_backward(nullptr, nullptr, 0, nullptr, st.shared_off, 1, 0, sw_gu,
                                     sw_dn, d, S * fs, nullptr, nullptr, nullptr, dsw_gu, dsw_dn,
                                     dw_dtype, accumulate, nullptr, 0, stream);
    return MOE_OK;
  }
  MOE_REQUIRE(logits && x && dy && dx && d_logits, MOE_ERR_INVALID_ARG, "null pointer");
  // dY: ORI -> SFD -> EPD through the forward's BRIMs
  if ((rc = moe_dispatch_gather(dy, T, d, MOE_BF16, k, R, L, st.brim0, st.brim1, st.dy_sfd,
                                st.dy_epd, stream)))
    return rc;
  const void* a = L > 1 ? st.x_epd : st.x_sfd;
  const void* dout = L > 1 ? st.dy_epd : st.dy_sfd;
  if ((rc = moe_expert_ffn_backward(dout, a, tk, st.z, st.epd_off, E, tk, w_gu, w_dn, d, f,
                                    st.epd_gate, st.o_epd, st.d_gate, dw_gu, dw_dn, dw_dtype,
                                    accumulate, st.bwd_ws, st.bwd_ws_bytes, stream)))
    return rc;
  if (S > 0 &&
      (rc = moe_expert_ffn_backward(dy, x, T, st.zs, st.shared_off, 1, T, sw_gu, sw_dn, d, S * fs,
                                    nullptr, st.dx_s, nullptr, dsw_gu, dsw_dn, dw_dtype,
                                    accumulate, st.sbwd_ws, st.sbwd_ws_bytes, stream)))
    return rc;
  // dX: EPD -> SFD -> ORI (pre-reduce per rank, then combine), plus the shared experts'
  if ((rc = moe_combine_scatter(st.o_epd, T, d, MOE_BF16, k, R, L, st.brim0, st.brim1,
                                S > 0 ? st.dx_s : nullptr, st.y_sfd, dx, stream)))
    return rc;
  return moe_route_backward(logits, T, E, k, renorm, st.topk_idx, slot_of, R, st.brim0, st.brim1,
                            st.d_gate, d_logits, d_topk_w, stream);
}

}  // extern "C"
