// C ABI of libengram_b200.so: argument checks, workspace carving, launches.
// Declarations and their contracts: include/engram.h.
#include <cstring>
#include <mutex>

#include "internal.cuh"

namespace engram {

namespace {

__device__ unsigned int g_status;  // one status word per device

constexpr int kMaxDevices = 64;
unsigned int* g_status_addr[kMaxDevices] = {nullptr};
std::mutex g_status_mu;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_cfg(const engram_cfg_t* c) {
  if (c == nullptr) return ENGRAM_ERR_INVALID_ARG;
  if (c->K < 1 || 2 * c->K > ENGRAM_MAX_HEADS) return ENGRAM_ERR_INVALID_ARG;
  if (c->D_h < 1 || c->d_model < 1 || c->n_branch < 1) return ENGRAM_ERR_INVALID_ARG;
  if (c->V_raw < 1 || c->V_c < 1 || c->V_c > c->V_raw) return ENGRAM_ERR_INVALID_ARG;
  if (c->dtype != ENGRAM_F32 && c->dtype != ENGRAM_BF16) return ENGRAM_ERR_INVALID_ARG;
  if ((c->flags & ~(ENGRAM_SAVE_KV | ENGRAM_VARIANT_FLAGS | ENGRAM_TEST_STALL)) != 0)
    return ENGRAM_ERR_INVALID_ARG;
  const int es = c->dtype == ENGRAM_F32 ? 4 : 2;
  if ((c->D_h * es) % 16 != 0) return ENGRAM_ERR_MISALIGNED;
  for (int j = 0; j < 2 * c->K; ++j) {
    const int64_t P = c->rows[j];
    // slots must fit int32 and a prime row count is odd and > 2
    if (P < 3 || P > 0x7fffffffLL || (P & 1) == 0) return ENGRAM_ERR_INVALID_ARG;
  }
  return ENGRAM_OK;
}

inline int elem_bytes(const engram_cfg_t* c) { return c->dtype == ENGRAM_F32 ? 4 : 2; }

// variants the bf16 path implements: learnable norm scales, the dilated
// conv, the pre-conv norm, and per-branch conv weights (with one branch, the
// same as shared ones)
constexpr int kBf16Variants = ENGRAM_NORM_SCALES | ENGRAM_CONV_PER_BRANCH | ENGRAM_CONV_DILATED |
                              ENGRAM_CONV_PRENORM;
inline bool bf16_variant_ok(const engram_cfg_t* c) {
  return (c->flags & ENGRAM_VARIANT_FLAGS & ~kBf16Variants) == 0;
}
inline bool bf16_scaled(const engram_cfg_t* c) {
  return c->dtype == ENGRAM_BF16 && (c->flags & ENGRAM_NORM_SCALES) != 0;
}

// bf16 layers with ENGRAM_SAVE_KV keep k and v after alpha in `saved`
inline bool saves_kv(const engram_cfg_t* c) {
  return c->dtype == ENGRAM_BF16 && (c->flags & ENGRAM_SAVE_KV) != 0;
}
inline size_t alpha_bytes_padded(int64_t n_tok) { return ((size_t)n_tok * 4 + 255) & ~(size_t)255; }
inline bool bf16_prenorm(const engram_cfg_t* c) {
  return c->dtype == ENGRAM_BF16 && (c->flags & ENGRAM_CONV_PRENORM) != 0;
}
inline size_t up256(size_t b) { return (b + 255) & ~(size_t)255; }

// bf16 forward workspace: the passes' buffers, then g_h g_k (norm scales),
// then with the pre-conv norm v [N, d] fp32 and rc [N]
struct Bf16FwdWs {
  size_t gg, vbuf, rc, ctr, total;
};
inline Bf16FwdWs bf16_fwd_ws(const engram_cfg_t* c, int64_t n) {
  const int d = c->d_model, E = 2 * c->K * c->D_h;
  Bf16FwdWs w;
  w.gg = tc_forward_ws_bytes(n, d, E);
  w.vbuf = w.gg + (bf16_scaled(c) ? up256((size_t)d * 4) : 0);
  const bool pn = bf16_prenorm(c);
  w.rc = w.vbuf + (pn ? up256((size_t)n * d * 4) : 0);
  w.ctr = w.rc + (pn ? up256((size_t)n * 4) : 0);  // two counters of the decode kernel
  w.total = w.ctr + 256;
  return w;
}

}  // namespace

unsigned int* status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_status_mu);
  if (g_status_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
    g_status_addr[dev] = static_cast<unsigned int*>(p);
  }
  return g_status_addr[dev];
}

HeadParams make_head_params(const engram_cfg_t* cfg) {
  HeadParams hp;
  std::memset(&hp, 0, sizeof(hp));
  hp.K = cfg->K;
  hp.J = 2 * cfg->K;
  hp.D_h = cfg->D_h;
  hp.E = hp.J * cfg->D_h;
  hp.V_raw = cfg->V_raw;
  hp.V_c = cfg->V_c;
  int64_t base = 0;
  for (int j = 0; j < hp.J; ++j) {
    for (int i = 0; i < 3; ++i) hp.mult[j][i] = cfg->mult[j][i];
    hp.P[j] = (uint64_t)cfg->rows[j];
    hp.mu[j] = ~0ull / hp.P[j];
    hp.row_base[j] = base;
    base += cfg->rows[j];
  }
  return hp;
}

// The layer after the gather (gate, value, conv, residual), for engram_forward
// and engram_decode_step; `chained`: a gather kernel of this call runs just
// before, so the first pass may start as it ends (programmatic launch).
int forward_from_e(const engram_cfg_t* cfg, const HeadParams& hp, void* e, const void* h,
                   const void* Wk, const void* Wv, const float* conv_w, float* conv_state,
                   void* out, float* saved, int64_t N, int32_t T, void* ws, size_t ws_bytes,
                   bool chained, cudaStream_t s, bool counters_zeroed = false) {
  const int M = cfg->n_branch, d = cfg->d_model, E = hp.E;
  int rc;
  if (cfg->dtype == ENGRAM_F32)
    return launch_forward_f32(static_cast<const float*>(e), static_cast<const float*>(h),
                              static_cast<const float*>(Wk), static_cast<const float*>(Wv), conv_w,
                              cfg->flags, conv_state, static_cast<float*>(out), saved, N, T, M, d,
                              E, ws, s);
  float* kv_save = saved != nullptr && conv_state == nullptr && saves_kv(cfg)
                       ? reinterpret_cast<float*>(reinterpret_cast<char*>(saved) +
                                                  alpha_bytes_padded(N))
                       : nullptr;
  const Bf16FwdWs wl = bf16_fwd_ws(cfg, N);
  char* wsb = static_cast<char*>(ws);
  float* gg = nullptr;  // g_h g_k, after the passes' workspace
  if (bf16_scaled(cfg)) {
    gg = reinterpret_cast<float*>(wsb + wl.gg);
    if ((rc = launch_scale_product(conv_w + 4 * d, conv_w + 5 * d, d, gg, s))) return rc;
  }
  // a decode step: both passes, the gate, the conv and the residual in one
  // persistent launch
  const int dil = (cfg->flags & ENGRAM_CONV_DILATED) ? 3 : 1;
  const bool stall = (cfg->flags & ENGRAM_TEST_STALL) != 0;
  if (conv_state != nullptr && !bf16_prenorm(cfg) && decode_fused_ok(N, d, E)) {
    float4* part = reinterpret_cast<float4*>(wsb);
    float* alpha = reinterpret_cast<float*>(wsb + (size_t)N * (d / 32) * sizeof(float4));
    return launch_decode_fused(static_cast<const __nv_bfloat16*>(e),
                               static_cast<const __nv_bfloat16*>(h),
                               static_cast<const __nv_bfloat16*>(Wk),
                               static_cast<const __nv_bfloat16*>(Wv), conv_w, conv_state,
                               static_cast<__nv_bfloat16*>(out), saved, gg, dil, N, d, E, part,
                               alpha, reinterpret_cast<int*>(wsb + wl.ctr), counters_zeroed,
                               chained, stall, s);
  }
  // the pre-conv norm: v into the kept [k | v] rows when there are any
  PrenormFwd pn{bf16_scaled(cfg) ? conv_w + 6 * d : nullptr,
                kv_save != nullptr ? kv_save + d : reinterpret_cast<float*>(wsb + wl.vbuf),
                kv_save != nullptr ? 2 * d : d, reinterpret_cast<float*>(wsb + wl.rc)};
  return launch_forward_tc(static_cast<const __nv_bfloat16*>(e), static_cast<const __nv_bfloat16*>(h),
                           static_cast<const __nv_bfloat16*>(Wk),
                           static_cast<const __nv_bfloat16*>(Wv), conv_w, conv_state,
                           static_cast<__nv_bfloat16*>(out), saved, kv_save, gg,
                           (cfg->flags & ENGRAM_CONV_DILATED) ? 3 : 1, N, T, d, E, ws, ws_bytes,
                           chained, bf16_prenorm(cfg) ? &pn : nullptr,
                           (cfg->flags & ENGRAM_TEST_STALL) != 0, s);
}

}  // namespace engram

using namespace engram;


extern "C" {

size_t engram_workspace_size(const engram_cfg_t* cfg, int32_t call, int64_t n) {
  if (n < 0) return 0;
  if (call == ENGRAM_WS_VOCAB) return vocab_ws_bytes(n);
  if (check_cfg(cfg) != ENGRAM_OK) return 0;
  const int M = cfg->n_branch, d = cfg->d_model, E = 2 * cfg->K * cfg->D_h;
  switch (call) {
    case ENGRAM_WS_FORWARD:
      if (cfg->dtype == ENGRAM_F32) return f32_forward_ws_bytes(n, M, d);
      return bf16_fwd_ws(cfg, n).total;
    case ENGRAM_WS_BACKWARD:
      if (cfg->dtype == ENGRAM_BF16)
        return backward_bf16_ws_bytes(n, d, E, 2 * cfg->K, saves_kv(cfg), bf16_scaled(cfg),
                                      bf16_prenorm(cfg));
      return backward_f32_ws_bytes(n, M, d, E) + table_grad_ws_bytes(n * 2 * cfg->K);
    case ENGRAM_WS_TABLE_GRAD:
      return table_grad_ws_bytes(n * 2 * cfg->K);
    case ENGRAM_WS_HOSTCACHE_RANK:
      return hot_rows_ws_bytes(n * 2 * cfg->K);
    case ENGRAM_WS_HOSTCACHE_GATHER:
      return cached_gather_ws_bytes(n, 2 * cfg->K);
    default:
      return 0;
  }
}

size_t engram_saved_size(const engram_cfg_t* cfg, int64_t n_tok) {
  if (check_cfg(cfg) != ENGRAM_OK || n_tok < 0) return 0;
  if (cfg->dtype == ENGRAM_F32) return f32_saved_bytes(n_tok, cfg->n_branch, cfg->d_model);
  if (saves_kv(cfg))  // alpha, then k and v from the 256-byte boundary on
    return alpha_bytes_padded(n_tok) + (size_t)n_tok * 2 * cfg->d_model * sizeof(float);
  return (size_t)n_tok * cfg->n_branch * sizeof(float);  // alpha
}

int engram_build_vocab_proj(const int64_t* keys, int32_t V, int32_t* proj, int32_t* V_c_out,
                            void* ws, size_t ws_bytes, void* stream) {
  const NvtxRange nvtx("engram_build_vocab_proj");
  if (V < 1 || keys == nullptr || proj == nullptr || V_c_out == nullptr || ws == nullptr)
    return ENGRAM_ERR_INVALID_ARG;
  if (!aligned16(keys) || !aligned16(proj) || !aligned16(ws)) return ENGRAM_ERR_MISALIGNED;
  if (status_ptr() == nullptr) return ENGRAM_ERR_CUDA;
  return launch_vocab_proj(keys, V, proj, V_c_out, ws, ws_bytes, (cudaStream_t)stream);
}

int engram_hash_indices(const engram_cfg_t* cfg, const int32_t* proj, const int32_t* ids,
                        int32_t B, int32_t T, int32_t* ngram_state, int32_t* idx, void* stream) {
  const NvtxRange nvtx("engram_hash_indices");
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (B < 0 || T < 0 || proj == nullptr || idx == nullptr || (B * (int64_t)T > 0 && ids == nullptr))
    return ENGRAM_ERR_INVALID_ARG;
  if (ngram_state != nullptr && T != 1) return ENGRAM_ERR_INVALID_ARG;
  if (!aligned16(proj) || !aligned16(ids) || !aligned16(idx) ||
      (ngram_state && !aligned16(ngram_state)))
    return ENGRAM_ERR_MISALIGNED;
  if (status_ptr() == nullptr) return ENGRAM_ERR_CUDA;
  return launch_hash(make_head_params(cfg), proj, ids, B, T, ngram_state, idx,
                     (cudaStream_t)stream);
}

int engram_gather(const engram_cfg_t* cfg, const int32_t* idx, const void* table, int64_t n_tok,
                  void* e, void* stream) {
  const NvtxRange nvtx("engram_gather");
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (n_tok < 0 || (n_tok > 0 && (idx == nullptr || table == nullptr || e == nullptr)))
    return ENGRAM_ERR_INVALID_ARG;
  if (!aligned16(idx) || !aligned16(table) || !aligned16(e)) return ENGRAM_ERR_MISALIGNED;
  if (status_ptr() == nullptr) return ENGRAM_ERR_CUDA;
  return launch_gather(make_head_params(cfg), idx, table, n_tok, elem_bytes(cfg), e,
                       (cudaStream_t)stream);
}

int engram_forward(const engram_cfg_t* cfg, const int32_t* idx, const void* table, void* e,
                   const void* h, const void* Wk, const void* Wv, const float* conv_w,
                   float* conv_state, void* out, float* saved, int32_t B, int32_t T, void* ws,
                   size_t ws_bytes, void* stream) {
  const NvtxRange nvtx("engram_forward");
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (B < 0 || T < 0) return ENGRAM_ERR_INVALID_ARG;
  const int64_t N = (int64_t)B * T;
  if (conv_state != nullptr && T != 1) return ENGRAM_ERR_INVALID_ARG;
  if (N == 0) return ENGRAM_OK;
  if (e == nullptr || h == nullptr || Wk == nullptr || Wv == nullptr || conv_w == nullptr ||
      out == nullptr || (table != nullptr && idx == nullptr))
    return ENGRAM_ERR_INVALID_ARG;
  if (!aligned16(idx) || !aligned16(table) || !aligned16(e) || !aligned16(h) || !aligned16(Wk) ||
      !aligned16(Wv) || !aligned16(conv_w) || !aligned16(conv_state) || !aligned16(out) ||
      !aligned16(saved) || !aligned16(ws))
    return ENGRAM_ERR_MISALIGNED;
  if (ws_bytes < engram_workspace_size(cfg, ENGRAM_WS_FORWARD, N)) return ENGRAM_ERR_WORKSPACE;
  if (status_ptr() == nullptr) return ENGRAM_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  const HeadParams hp = make_head_params(cfg);
  if (cfg->dtype == ENGRAM_BF16 &&
      (!tc_supported(cfg->d_model, hp.E, cfg->n_branch) || !bf16_variant_ok(cfg)))
    return ENGRAM_ERR_UNSUPPORTED;
  // a bf16 decode step: the gather zeroes the decode kernel's counters, so
  // that the two stay one launch chain
  const bool zero_first = table != nullptr && conv_state != nullptr && cfg->dtype == ENGRAM_BF16;
  if (table != nullptr) {
    int* ctr = zero_first ? reinterpret_cast<int*>(static_cast<char*>(ws) + bf16_fwd_ws(cfg, N).ctr)
                          : nullptr;
    rc = launch_gather(hp, idx, table, N, elem_bytes(cfg), e, s, ctr);
    if (rc) return rc;
  }
  return forward_from_e(cfg, hp, e, h, Wk, Wv, conv_w, conv_state, out, saved, N, T, ws, ws_bytes,
                        table != nullptr, s, zero_first);
}

int engram_decode_step(const engram_cfg_t* cfg, const int32_t* proj, const int32_t* ids,
                       int32_t* ngram_state, int32_t* idx, const void* table, void* e,
                       const void* h, const void* Wk, const void* Wv, const float* conv_w,
                       float* conv_state, void* out, int32_t B, void* ws, size_t ws_bytes,
                       void* stream) {
  const NvtxRange nvtx("engram_decode_step");
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (B < 0) return ENGRAM_ERR_INVALID_ARG;
  if (B == 0) return ENGRAM_OK;
  if (proj == nullptr || ids == nullptr || ngram_state == nullptr || table == nullptr ||
      e == nullptr || h == nullptr || Wk == nullptr || Wv == nullptr || conv_w == nullptr ||
      conv_state == nullptr || out == nullptr)
    return ENGRAM_ERR_INVALID_ARG;
  if (!aligned16(proj) || !aligned16(ids) || !aligned16(ngram_state) || !aligned16(idx) ||
      !aligned16(table) || !aligned16(e) || !aligned16(h) || !aligned16(Wk) || !aligned16(Wv) ||
      !aligned16(conv_w) || !aligned16(conv_state) || !aligned16(out) || !aligned16(ws))
    return ENGRAM_ERR_MISALIGNED;
  if (ws_bytes < engram_workspace_size(cfg, ENGRAM_WS_FORWARD, B)) return ENGRAM_ERR_WORKSPACE;
  if (status_ptr() == nullptr) return ENGRAM_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  const HeadParams hp = make_head_params(cfg);
  if (cfg->dtype == ENGRAM_BF16 &&
      (!tc_supported(cfg->d_model, hp.E, cfg->n_branch) || !bf16_variant_ok(cfg)))
    return ENGRAM_ERR_UNSUPPORTED;
  // bf16 decode: the gather also zeroes the counters of the decode kernel
  int* ctr = cfg->dtype == ENGRAM_BF16
                 ? reinterpret_cast<int*>(static_cast<char*>(ws) + bf16_fwd_ws(cfg, B).ctr)
                 : nullptr;
  if ((rc = launch_hash_gather_decode(hp, proj, ids, B, ngram_state, idx, table, elem_bytes(cfg),
                                      e, ctr, s)))
    return rc;
  return forward_from_e(cfg, hp, e, h, Wk, Wv, conv_w, conv_state, out, nullptr, B, 1, ws,
                        ws_bytes, true, s, ctr != nullptr);
}

int engram_backward(const engram_cfg_t* cfg, const int32_t* idx, const void* e, const void* h,
                    const void* Wk, const void* Wv, const float* conv_w, const float* saved,
                    const float* dout, float* dh, float* dWk, float* dWv, float* dconv_w, float* de,
                    int64_t* dtab_keys, float* dtab_rows, int32_t* n_unique, int32_t B, int32_t T,
                    void* ws, size_t ws_bytes, void* stream) {
  const NvtxRange nvtx("engram_backward");
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (cfg->dtype == ENGRAM_BF16 && (cfg->n_branch != 1 || !bf16_variant_ok(cfg)))
    return ENGRAM_ERR_UNSUPPORTED;
  if (cfg->dtype == ENGRAM_BF16 && saved == nullptr) return ENGRAM_ERR_INVALID_ARG;
  if (B < 0 || T < 0) return ENGRAM_ERR_INVALID_ARG;
  const int64_t N = (int64_t)B * T;
  if (idx == nullptr || e == nullptr || h == nullptr || Wk == nullptr || Wv == nullptr ||
      conv_w == nullptr || dout == nullptr || dh == nullptr || dWk == nullptr ||
      dWv == nullptr || dconv_w == nullptr || dtab_keys == nullptr || dtab_rows == nullptr ||
      n_unique == nullptr || ws == nullptr)
    return ENGRAM_ERR_INVALID_ARG;
  if (!aligned16(idx) || !aligned16(e) || !aligned16(h) || !aligned16(Wk) || !aligned16(Wv) ||
      !aligned16(conv_w) || !aligned16(saved) || !aligned16(dout) || !aligned16(dh) ||
      !aligned16(dWk) || !aligned16(dWv) || !aligned16(dconv_w) || !aligned16(de) ||
      !aligned16(dtab_keys) || !aligned16(dtab_rows) || !aligned16(ws))
    return ENGRAM_ERR_MISALIGNED;
  if (ws_bytes < engram_workspace_size(cfg, ENGRAM_WS_BACKWARD, N)) return ENGRAM_ERR_WORKSPACE;
  if (status_ptr() == nullptr) return ENGRAM_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  const HeadParams hp = make_head_params(cfg);
  const int M = cfg->n_branch, d = cfg->d_model, E = hp.E;
  if (cfg->dtype == ENGRAM_BF16) {
    if (N == 0) {  // no tokens: zero weight gradients, no rows
      if ((rc = ck(cudaMemsetAsync(dWk, 0, (size_t)d * E * 4, s)))) return rc;
      if ((rc = ck(cudaMemsetAsync(dWv, 0, (size_t)d * E * 4, s)))) return rc;
      if ((rc = ck(cudaMemsetAsync(dconv_w, 0, (size_t)engram_param_floats(cfg) * 4, s))))
        return rc;
      return ck(cudaMemsetAsync(n_unique, 0, sizeof(int32_t), s));
    }
    using bf = __nv_bfloat16;
    const float* kv_saved =
        saves_kv(cfg) ? reinterpret_cast<const float*>(reinterpret_cast<const char*>(saved) +
                                                       alpha_bytes_padded(N))
                      : nullptr;
    return launch_backward_bf16(hp, idx, static_cast<const bf*>(e), static_cast<const bf*>(h),
                                static_cast<const bf*>(Wk), static_cast<const bf*>(Wv), conv_w,
                                bf16_scaled(cfg) ? conv_w + 4 * d : nullptr, saved, kv_saved,
                                dout, dh, dWk, dWv, dconv_w, de, dtab_keys, dtab_rows, n_unique,
                                N, T, d, (cfg->flags & ENGRAM_CONV_DILATED) ? 3 : 1,
                                bf16_prenorm(cfg),
                                bf16_scaled(cfg) && bf16_prenorm(cfg) ? conv_w + 6 * d : nullptr,
                                ws, ws_bytes, (cfg->flags & ENGRAM_TEST_STALL) != 0, s);
  }
  const size_t bw = backward_f32_ws_bytes(N, M, d, E);
  // de lives in the dense-backward workspace unless the caller wants it
  float* de_buf = de != nullptr ? de : backward_f32_de_slot(ws, N, M, d, E);
  F32Saved sv = f32_saved_layout(saved != nullptr ? const_cast<float*>(saved) : ws, N, M, d);
  rc = launch_backward_f32(static_cast<const float*>(e), static_cast<const float*>(h),
                           static_cast<const float*>(Wk), static_cast<const float*>(Wv), conv_w,
                           cfg->flags, sv, dout, dh, dWk, dWv, dconv_w, de_buf, N, T, M, d, E, ws,
                           s);
  if (rc) return rc;
  return launch_table_grad(hp, idx, de_buf, N, dtab_keys, dtab_rows, n_unique,
                           static_cast<char*>(ws) + bw, ws_bytes - bw, s);
}

int engram_table_grad(const engram_cfg_t* cfg, const int32_t* idx, const float* de, int64_t n_tok,
                      int64_t* dtab_keys, float* dtab_rows, int32_t* n_unique, void* ws,
                      size_t ws_bytes, void* stream) {
  const NvtxRange nvtx("engram_table_grad");
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (n_tok < 0 || n_unique == nullptr) return ENGRAM_ERR_INVALID_ARG;
  if (n_tok > 0 && (idx == nullptr || de == nullptr || dtab_keys == nullptr ||
                    dtab_rows == nullptr || ws == nullptr))
    return ENGRAM_ERR_INVALID_ARG;
  if (n_tok >= 0x7fffffffLL / (2 * cfg->K)) return ENGRAM_ERR_UNSUPPORTED;
  if (!aligned16(idx) || !aligned16(de) || !aligned16(dtab_keys) || !aligned16(dtab_rows) ||
      !aligned16(ws))
    return ENGRAM_ERR_MISALIGNED;
  if (status_ptr() == nullptr) return ENGRAM_ERR_CUDA;
  return launch_table_grad(make_head_params(cfg), idx, de, n_tok, dtab_keys, dtab_rows, n_unique,
                           ws, ws_bytes, (cudaStream_t)stream);
}

int engram_table_grad_noalloc(const engram_cfg_t* cfg, const int32_t* idx, const float* de,
                              int64_t n_tok, int64_t* dtab_keys, float* dtab_rows,
                              int32_t* n_unique, void* stream) {
  const NvtxRange nvtx("engram_table_grad_noalloc");
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (n_tok < 0 || n_unique == nullptr) return ENGRAM_ERR_INVALID_ARG;
  if (n_tok > 0 && (idx == nullptr || de == nullptr || dtab_keys == nullptr || dtab_rows == nullptr))
    return ENGRAM_ERR_INVALID_ARG;
  if (!aligned16(idx) || !aligned16(de) || !aligned16(dtab_keys) || !aligned16(dtab_rows))
    return ENGRAM_ERR_MISALIGNED;
  // compared before multiplying, so that no n_tok can overflow the product
  if (n_tok > ENGRAM_NOALLOC_MAX_ITEMS / (2 * cfg->K)) return ENGRAM_ERR_TOO_LARGE;
  if (status_ptr() == nullptr) return ENGRAM_ERR_CUDA;
  return launch_table_grad_noalloc(make_head_params(cfg), idx, de, n_tok, dtab_keys, dtab_rows,
                                   n_unique, (cudaStream_t)stream);
}

int engram_forward_hosttable(const engram_cfg_t* cfg, const int32_t* idx, const void* host_table,
                             int64_t n_tok, void* e, void* side_stream, void* done_event) {
  const NvtxRange nvtx("engram_forward_hosttable");
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (n_tok < 0 || (n_tok > 0 && (idx == nullptr || host_table == nullptr || e == nullptr)))
    return ENGRAM_ERR_INVALID_ARG;
  if (!aligned16(idx) || !aligned16(host_table) || !aligned16(e)) return ENGRAM_ERR_MISALIGNED;
  if (status_ptr() == nullptr) return ENGRAM_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)side_stream;
  if (n_tok > 0) {
    // the device-side address of the pinned host range (equal to the host
    // address under unified addressing; fails if the memory is not mapped)
    void* dev_ptr = nullptr;
    if (cudaHostGetDevicePointer(&dev_ptr, const_cast<void*>(host_table), 0) != cudaSuccess) {
      cudaGetLastError();
      return ENGRAM_ERR_INVALID_ARG;
    }
    rc = launch_gather_host(make_head_params(cfg), idx, dev_ptr, n_tok, elem_bytes(cfg), e, s);
    if (rc) return rc;
  }
  if (done_event != nullptr) return ck(cudaEventRecord((cudaEvent_t)done_event, s));
  return ENGRAM_OK;
}

int64_t engram_param_floats(const engram_cfg_t* cfg) {
  if (check_cfg(cfg) != ENGRAM_OK) return 0;
  if (cfg->dtype == ENGRAM_BF16)  // conv weights, then g_h, g_k (and g_v with the pre-conv norm)
    return (int64_t)cfg->d_model *
           (4 + ((cfg->flags & ENGRAM_NORM_SCALES) ? ((cfg->flags & ENGRAM_CONV_PRENORM) ? 3 : 2) : 0));
  return f32_param_floats(cfg->flags, cfg->n_branch, cfg->d_model);
}

int64_t engram_table_rows(const engram_cfg_t* cfg) {
  if (check_cfg(cfg) != ENGRAM_OK) return 0;
  int64_t t = 0;
  for (int j = 0; j < 2 * cfg->K; ++j) t += cfg->rows[j];
  return t;
}

int engram_hostcache_rank(const engram_cfg_t* cfg, const int32_t* idx, int64_t n_tok, int64_t C,
                          int64_t* rows_out, int32_t* n_out, void* ws, size_t ws_bytes,
                          void* stream) {
  const NvtxRange nvtx("engram_hostcache_rank");
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (n_tok < 0 || C < 0 || n_out == nullptr || (C > 0 && rows_out == nullptr) ||
      (n_tok > 0 && (idx == nullptr || ws == nullptr)))
    return ENGRAM_ERR_INVALID_ARG;
  if (n_tok >= 0x7fffffffLL / (2 * cfg->K) || C >= 0x7fffffffLL) return ENGRAM_ERR_UNSUPPORTED;
  if (!aligned16(idx) || !aligned16(rows_out) || !aligned16(ws)) return ENGRAM_ERR_MISALIGNED;
  if (ws_bytes < engram_workspace_size(cfg, ENGRAM_WS_HOSTCACHE_RANK, n_tok))
    return ENGRAM_ERR_WORKSPACE;
  if (status_ptr() == nullptr) return ENGRAM_ERR_CUDA;
  return launch_hot_rows(make_head_params(cfg), idx, n_tok, C, rows_out, n_out, ws, ws_bytes,
                         (cudaStream_t)stream);
}

namespace {
// the device-side address of a pinned host range (equal to the host address
// under unified addressing; fails if the memory is not mapped)
int mapped_host(const void* host, void** dev) {
  if (cudaHostGetDevicePointer(dev, const_cast<void*>(host), 0) != cudaSuccess) {
    cudaGetLastError();
    return ENGRAM_ERR_INVALID_ARG;
  }
  return ENGRAM_OK;
}
}  // namespace

int engram_hostcache_fill(const engram_cfg_t* cfg, const void* host_table, const int64_t* rows,
                          int64_t C, void* cache, int32_t* map, void* stream) {
  const NvtxRange nvtx("engram_hostcache_fill");
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (C < 0 || host_table == nullptr || map == nullptr ||
      (C > 0 && (rows == nullptr || cache == nullptr)))
    return ENGRAM_ERR_INVALID_ARG;
  if (C >= 0x7fffffffLL) return ENGRAM_ERR_UNSUPPORTED;
  if (!aligned16(host_table) || !aligned16(rows) || !aligned16(cache) || !aligned16(map))
    return ENGRAM_ERR_MISALIGNED;
  if (status_ptr() == nullptr) return ENGRAM_ERR_CUDA;
  void* dev_ptr = nullptr;
  if ((rc = mapped_host(host_table, &dev_ptr))) return rc;
  return launch_cache_fill(make_head_params(cfg), dev_ptr, rows, C, elem_bytes(cfg), cache, map,
                           (cudaStream_t)stream);
}

int engram_forward_hostcache(const engram_cfg_t* cfg, const int32_t* idx, const void* host_table,
                             const void* cache, const int32_t* map, int64_t n_tok, void* e,
                             int32_t* n_miss, void* ws, size_t ws_bytes, void* side_stream,
                             void* done_event) {
  const NvtxRange nvtx("engram_forward_hostcache");
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (n_tok < 0 || host_table == nullptr || map == nullptr || ws == nullptr ||
      (n_tok > 0 && (idx == nullptr || e == nullptr)))
    return ENGRAM_ERR_INVALID_ARG;
  if (n_tok >= 0x7fffffffLL / (2 * cfg->K)) return ENGRAM_ERR_UNSUPPORTED;
  if (!aligned16(idx) || !aligned16(host_table) || !aligned16(cache) || !aligned16(map) ||
      !aligned16(e) || !aligned16(ws))
    return ENGRAM_ERR_MISALIGNED;
  if (ws_bytes < engram_workspace_size(cfg, ENGRAM_WS_HOSTCACHE_GATHER, n_tok))
    return ENGRAM_ERR_WORKSPACE;
  if (status_ptr() == nullptr) return ENGRAM_ERR_CUDA;
  void* dev_ptr = nullptr;
  if ((rc = mapped_host(host_table, &dev_ptr))) return rc;
  cudaStream_t s = (cudaStream_t)side_stream;
  rc = launch_gather_cached(make_head_params(cfg), idx, dev_ptr, cache, map, n_tok,
                            elem_bytes(cfg), e, n_miss, ws, s);
  if (rc) return rc;
  if (done_event != nullptr) return ck(cudaEventRecord((cudaEvent_t)done_event, s));
  return ENGRAM_OK;
}

int engram_get_status(void* stream) {
  const NvtxRange nvtx("engram_get_status");
  unsigned int* p = status_ptr();
  if (p == nullptr) return ENGRAM_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  unsigned int v = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ENGRAM_ERR_CUDA;
  if (cudaMemcpyAsync(&v, p, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return ENGRAM_ERR_CUDA;
  if (cudaMemsetAsync(p, 0, sizeof(v), s) != cudaSuccess) return ENGRAM_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ENGRAM_ERR_CUDA;
  return (int)(v & 0x7fffffffu);
}

int engram_device_sm_count(void) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ENGRAM_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return ENGRAM_ERR_CUDA;
  return sms;
}

}  // extern "C"
