// fp32 CUDA-core path of the fusion stage and its backward, for small layers
// (d and E in the tens to hundreds, a few hundred tokens, several branches).
// These shapes are launch-latency bound; the tensor-core path handles the
// large bf16 layers.
//
// Method: discuss.deepseek.club 二.1 (2) (h as query, e as key and value; the
// gate factor; 1-D conv; residual), 二.2 (branches share table and value
// projection, own key projection); sechub.in answer (short depthwise causal
// conv); gitcode.csdn.net blog 第三步 / 第四步 and end-to-end training.
#include "internal.cuh"

namespace engram {

namespace {

constexpr float RMS_EPS = 1e-6f;

// The formulation variants of the layer's flags, and where their parameters
// sit in the small-parameter block: conv weights ([M or 1][d][4]), then with
// ENGRAM_NORM_SCALES g_h [M][d], g_k [M][d] and, with ENGRAM_CONV_PRENORM,
// g_v [M][d].
struct F32Var {
  int dil;         // conv dilation: 1, or 3 with ENGRAM_CONV_DILATED
  int prenorm;     // the conv reads RMSNorm(vt) (times g_v)
  int per_branch;  // conv weights per branch
  const float* w;
  const float *gh, *gk, *gv;  // NULL when absent (scale 1)
  __device__ const float* taps(int m, int d, int c) const {
    return w + ((int64_t)(per_branch ? m : 0) * d + c) * 4;
  }
  // g_h g_k of branch m, feature c
  __device__ double gg(int m, int d, int c) const {
    return gh != nullptr ? (double)gh[m * d + c] * (double)gk[m * d + c] : 1.0;
  }
  // the conv input of token n, branch m, feature c
  __device__ double conv_in(const double* alpha, const double* v, const double* rc, int64_t n,
                            int m, int M, int d, int c) const {
    const double vt = alpha[n * M + m] * v[n * d + c];
    if (!prenorm) return vt;
    return vt * rc[n * M + m] * (gv != nullptr ? (double)gv[m * d + c] : 1.0);
  }
};

// The forward keeps every product and sum in fp64 and rounds each stored
// value (out, and alpha, k, v, y in `saved`) to fp32 once.

__device__ __forceinline__ double warp_sum_fd(double x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// k[n,m,c] = <Wk[m,c,:], e[n,:]> (m < M) and v[n,c] = <Wv[c,:], e[n,:]> (m == M):
// one warp per output, lanes stride the contraction axis.
__global__ void proj_f32_kernel(const float* __restrict__ e, const float* __restrict__ Wk,
                                const float* __restrict__ Wv, double* __restrict__ k,
                                double* __restrict__ v, float* __restrict__ k32,
                                float* __restrict__ v32, int64_t N, int M, int d, int E) {
  const int lane = threadIdx.x & 31;
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t total = N * (M + 1) * d;
  if (w >= total) return;
  const int c = (int)(w % d);
  const int m = (int)((w / d) % (M + 1));
  const int64_t n = w / ((int64_t)d * (M + 1));
  const float* wrow = (m < M) ? Wk + ((int64_t)m * d + c) * E : Wv + (int64_t)c * E;
  const float* erow = e + n * E;
  double acc = 0.0;
  for (int i = lane; i < E; i += 32) acc = fma((double)__ldg(wrow + i), (double)__ldg(erow + i), acc);
  acc = warp_sum_fd(acc);
  if (lane == 0) {
    if (m < M) {
      k[(n * M + m) * d + c] = acc;
      k32[(n * M + m) * d + c] = (float)acc;
    } else {
      v[n * d + c] = acc;
      v32[n * d + c] = (float)acc;
    }
  }
}

// alpha[n,m] = sigmoid(<RMSNorm(h) g_h, RMSNorm(k) g_k> / sqrt(d)): one warp
// per (n, m).  With the pre-conv norm it also keeps
// r_c[n,m] = (mean(vt^2) + eps)^(-1/2), vt = alpha v.
__global__ void gate_f32_kernel(const float* __restrict__ h, const double* __restrict__ k,
                                const double* __restrict__ v, const F32Var var,
                                double* __restrict__ alpha, float* __restrict__ alpha32,
                                double* __restrict__ rc, int64_t NM, int M, int d) {
  const int lane = threadIdx.x & 31;
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (w >= NM) return;
  const int m = (int)(w % M);
  const float* hr = h + w * d;
  const double* kr = k + w * d;
  const double* vr = v + (w / M) * d;
  double hh = 0.0, kk = 0.0, hk = 0.0, vv = 0.0;
  for (int c = lane; c < d; c += 32) {
    const double a = hr[c], b = kr[c];
    hh = fma(a, a, hh);
    kk = fma(b, b, kk);
    hk = fma(a * b, var.gg(m, d, c), hk);
    if (var.prenorm) vv = fma(vr[c], vr[c], vv);
  }
  hh = warp_sum_fd(hh);
  kk = warp_sum_fd(kk);
  hk = warp_sum_fd(hk);
  vv = warp_sum_fd(vv);
  if (lane == 0) {
    const double rh = 1.0 / sqrt(hh / d + (double)RMS_EPS);
    const double rk = 1.0 / sqrt(kk / d + (double)RMS_EPS);
    const double a = 1.0 / (1.0 + exp(-(hk * rh * rk / sqrt((double)d))));
    alpha[w] = a;
    alpha32[w] = (float)a;
    if (var.prenorm) rc[w] = 1.0 / sqrt(a * a * vv / d + (double)RMS_EPS);
  }
}

// y = sum_i w[c,i] c_{t-(3-i) dil}, out = h + vt + SiLU(y): one thread per
// (n, m, c); the conv input c is vt, or RMSNorm(vt) g_v with the pre-conv
// norm.  With conv_state (decode, T == 1) the earlier inputs come from the
// state ([3 dil][d] per (n, m), oldest first), which is then shifted by one
// step.  h and out may be the same buffer (each element is read before it
// is written, by the same thread), so neither is declared __restrict__.
__global__ void conv_f32_kernel(const float* h, const double* __restrict__ v,
                                const double* __restrict__ alpha, const double* __restrict__ rc,
                                const F32Var var, float* __restrict__ conv_state,
                                float* __restrict__ y_out, float* out, int64_t N, int T, int M,
                                int d) {
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= N * M * d) return;
  const int c = (int)(g % d);
  const int m = (int)((g / d) % M);
  const int64_t n = g / ((int64_t)d * M);
  const float* wp = var.taps(m, d, c);
  const double taps[4] = {wp[0], wp[1], wp[2], wp[3]};
  const double vt = alpha[n * M + m] * v[n * d + c];
  const double cin = var.conv_in(alpha, v, rc, n, m, M, d, c);
  double y = taps[3] * cin;
  const int dil = var.dil;
  if (conv_state != nullptr) {
    float* st = conv_state + ((n * M + m) * 3 * dil) * d + c;  // [3 dil][d] oldest first
    for (int L = 3; L >= 1; --L) y = fma(taps[3 - L], (double)st[(3 * dil - L * dil) * d], y);
    for (int q = 0; q + 1 < 3 * dil; ++q) st[q * d] = st[(q + 1) * d];
    st[(3 * dil - 1) * d] = (float)cin;
  } else {
    const int t = (int)(n % T);
    for (int L = 1; L <= 3; ++L) {
      const int lag = L * dil;
      if (t >= lag) y = fma(taps[3 - L], var.conv_in(alpha, v, rc, n - lag, m, M, d, c), y);
    }
  }
  y_out[g] = (float)y;
  out[g] = (float)((double)h[g] + vt + y / (1.0 + exp(-y)));
}

// ------------------------------------------------------------------ backward
//
// The backward recomputes the forward intermediates (k, v, alpha, y) in fp64
// from e, h and the weights, and carries every product and sum in fp64; each
// gradient is rounded to fp32 once when stored.

__device__ __forceinline__ double warp_sum_d(double x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ double sigmoid_d(double z) { return 1.0 / (1.0 + exp(-z)); }

// k64[n,m,c], v64[n,c] in fp64: one warp per output
__global__ void rec_proj_kernel(const float* __restrict__ e, const float* __restrict__ Wk,
                                const float* __restrict__ Wv, double* __restrict__ k,
                                double* __restrict__ v, int64_t N, int M, int d, int E) {
  const int lane = threadIdx.x & 31;
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (w >= N * (M + 1) * d) return;
  const int c = (int)(w % d);
  const int m = (int)((w / d) % (M + 1));
  const int64_t n = w / ((int64_t)d * (M + 1));
  const float* wrow = (m < M) ? Wk + ((int64_t)m * d + c) * E : Wv + (int64_t)c * E;
  const float* erow = e + n * E;
  double acc = 0.0;
  for (int i = lane; i < E; i += 32) acc = fma((double)wrow[i], (double)erow[i], acc);
  acc = warp_sum_d(acc);
  if (lane == 0) {
    if (m < M) k[(n * M + m) * d + c] = acc;
    else v[n * d + c] = acc;
  }
}

// alpha64[n,m] and the row sums the gate backward needs (r_h, r_k,
// <h g_h g_k, k>; r_c of the pre-conv norm in rc): one warp per (n, m)
__global__ void rec_gate_kernel(const float* __restrict__ h, const double* __restrict__ k,
                                const double* __restrict__ v, const F32Var var,
                                double* __restrict__ alpha, double* __restrict__ sums,
                                double* __restrict__ rc, int64_t NM, int M, int d) {
  const int lane = threadIdx.x & 31;
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (w >= NM) return;
  const int m = (int)(w % M);
  const double* vr = v + (w / M) * d;
  double hh = 0.0, kk = 0.0, hk = 0.0, vv = 0.0;
  for (int c = lane; c < d; c += 32) {
    const double a = h[w * d + c], b = k[w * d + c];
    hh = fma(a, a, hh);
    kk = fma(b, b, kk);
    hk = fma(a * b, var.gg(m, d, c), hk);
    if (var.prenorm) vv = fma(vr[c], vr[c], vv);
  }
  hh = warp_sum_d(hh);
  kk = warp_sum_d(kk);
  hk = warp_sum_d(hk);
  vv = warp_sum_d(vv);
  if (lane == 0) {
    const double rh = 1.0 / sqrt(hh / d + (double)RMS_EPS);
    const double rk = 1.0 / sqrt(kk / d + (double)RMS_EPS);
    const double a = sigmoid_d(hk * rh * rk / sqrt((double)d));
    alpha[w] = a;
    sums[3 * w + 0] = rh;
    sums[3 * w + 1] = rk;
    sums[3 * w + 2] = hk;
    if (var.prenorm) rc[w] = 1.0 / sqrt(a * a * vv / d + (double)RMS_EPS);
  }
}

// y64 and dy64 = dout * SiLU'(y): one thread per (n, m, c)
__global__ void rec_conv_dsilu_kernel(const double* __restrict__ v, const double* __restrict__ alpha,
                                      const double* __restrict__ rc, const F32Var var,
                                      const float* __restrict__ dout, double* __restrict__ dy,
                                      int64_t N, int T, int M, int d) {
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= N * M * d) return;
  const int c = (int)(g % d);
  const int m = (int)((g / d) % M);
  const int64_t n = g / ((int64_t)d * M);
  const int t = (int)(n % T);
  const float* wp = var.taps(m, d, c);
  double y = 0.0;
  for (int L = 0; L <= 3; ++L) {
    const int lag = L * var.dil;
    if (t >= lag) y = fma((double)wp[3 - L], var.conv_in(alpha, v, rc, n - lag, m, M, d, c), y);
  }
  const double s = sigmoid_d(y);
  dy[g] = (double)dout[g] * s * (1.0 + y * (1.0 - s));
}

// One warp per (n, m).  dc = sum_i w[:,i] dy_{t+(3-i) dil} (the gradient of
// the conv input); dvt = dout + dc, or with the pre-conv norm
// dout + r_c dc^ - r_c^3 vt <dc^, vt> / d with dc^ = dc g_v; dalpha =
// <dvt, v>; dz = dalpha a (1 - a); the gate's RMSNorm backwards:
//   dx = r dxh - r^3 x <dxh, x> / d, with dh^ = dz g_h g_k k^ / sqrt(d) and
//   dk^ = dz g_h g_k h^ / sqrt(d).
// dc (for g_v's gradient) and dz (for g_h's and g_k's) are kept when asked.
struct GateBwdArgs {
  const float* dout;
  const double *dy, *k, *v, *alpha, *sums, *rc;
  const float* h;
  double *dvt, *dc_keep, *dz_keep, *dk;
  float* dh;
  int64_t N;
  int T, M, d;
};

// the gate backward of row wid = n M + m, by one warp
template <int MAXC>
__device__ __forceinline__ void gate_bwd_row(const GateBwdArgs& ga, const F32Var& var,
                                             int64_t wid, int lane) {
  const float* __restrict__ dout = ga.dout;
  const double* __restrict__ dy = ga.dy;
  const float* __restrict__ h = ga.h;
  const double* __restrict__ k = ga.k;
  const double* __restrict__ v = ga.v;
  const double* __restrict__ alpha = ga.alpha;
  const double* __restrict__ sums = ga.sums;
  const double* __restrict__ rc = ga.rc;
  double* __restrict__ dvt = ga.dvt;
  double* __restrict__ dc_keep = ga.dc_keep;
  double* __restrict__ dz_keep = ga.dz_keep;
  float* __restrict__ dh = ga.dh;
  double* __restrict__ dk = ga.dk;
  const int T = ga.T, M = ga.M, d = ga.d;
  const int m = (int)(wid % M);
  const int64_t n = wid / M;
  const int t = (int)(n % T);
  const double al = alpha[wid];
  // MAXC > 0 (d <= 32 MAXC): this lane's features c = lane + 32 j are held in
  // registers, their loads all issued up front; MAXC = 0: read where used
  constexpr int R = MAXC > 0 ? MAXC : 1;
  constexpr int JMAX = MAXC > 0 ? MAXC : 1 << 20;
  double dout_r[R], v_r[R], g_r[R], h_r[R], k_r[R];
  if constexpr (MAXC > 0) {
#pragma unroll
    for (int j = 0; j < MAXC; ++j) {
      const int c = lane + 32 * j;
      dout_r[j] = c < d ? (double)dout[wid * d + c] : 0.0;
      v_r[j] = c < d ? v[n * d + c] : 0.0;
      h_r[j] = c < d ? (double)h[wid * d + c] : 0.0;
      k_r[j] = c < d ? k[wid * d + c] : 0.0;
    }
  }
  // dc into dvt; with the pre-conv norm also <dc^, vt>
  double cv = 0.0;
#pragma unroll
  for (int j = 0; j < JMAX; ++j) {
    const int c = lane + 32 * j;
    if (c >= d) break;
    const float* wp = var.taps(m, d, c);
    double g = 0.0;
    for (int L = 0; L <= 3; ++L) {
      const int lag = L * var.dil;
      if (t + lag < T) g = fma((double)wp[3 - L], dy[((n + lag) * M + m) * d + c], g);
    }
    if constexpr (MAXC > 0) g_r[j] = g; else dvt[wid * d + c] = g;
    if (dc_keep != nullptr) dc_keep[wid * d + c] = g;
    if (var.prenorm) {
      const double gvc = var.gv != nullptr ? (double)var.gv[m * d + c] : 1.0;
      const double vc = MAXC > 0 ? v_r[MAXC > 0 ? j : 0] : v[n * d + c];
      cv = fma(g * gvc, al * vc, cv);
    }
  }
  cv = warp_sum_d(cv);
  const double r = var.prenorm ? rc[wid] : 0.0;
  double da = 0.0;
#pragma unroll
  for (int j = 0; j < JMAX; ++j) {
    const int c = lane + 32 * j;
    if (c >= d) break;
    double g = MAXC > 0 ? g_r[MAXC > 0 ? j : 0] : dvt[wid * d + c];
    const double vc = MAXC > 0 ? v_r[MAXC > 0 ? j : 0] : v[n * d + c];
    if (var.prenorm) {
      const double gvc = var.gv != nullptr ? (double)var.gv[m * d + c] : 1.0;
      g = r * (g * gvc) - r * r * r * (al * vc) * cv / d;
    }
    g += MAXC > 0 ? dout_r[MAXC > 0 ? j : 0] : (double)dout[wid * d + c];
    dvt[wid * d + c] = g;
    da = fma(g, vc, da);
  }
  da = warp_sum_d(da);
  const double dz = da * al * (1.0 - al);
  if (dz_keep != nullptr && lane == 0) dz_keep[wid] = dz;
  const double rh = sums[3 * wid], rk = sums[3 * wid + 1], hk = sums[3 * wid + 2];
  const double isd = 1.0 / sqrt((double)d);
  // <dh^, h> = dz/sqrt(d) * rk * <h g g, k>, <dk^, k> = dz/sqrt(d) * rh * <h g g, k>
  const double dot_hh = dz * isd * rk * hk;
  const double dot_kk = dz * isd * rh * hk;
#pragma unroll
  for (int j = 0; j < JMAX; ++j) {
    const int c = lane + 32 * j;
    if (c >= d) break;
    const double a = MAXC > 0 ? h_r[MAXC > 0 ? j : 0] : (double)h[wid * d + c];
    const double b = MAXC > 0 ? k_r[MAXC > 0 ? j : 0] : k[wid * d + c];
    const double gg = var.gg(m, d, c);
    const double dhh = dz * isd * rk * gg * b;
    const double dkh = dz * isd * rh * gg * a;
    const double dov = MAXC > 0 ? dout_r[MAXC > 0 ? j : 0] : (double)dout[wid * d + c];
    dh[wid * d + c] = (float)(dov + rh * dhh - rh * rh * rh * a * dot_hh / d);
    dk[wid * d + c] = rk * dkh - rk * rk * rk * b * dot_kk / d;
  }
}

// A block per token: its warps take the token's M rows of the gate
// backward, then the block forms dv[n,c] = sum_m alpha[n,m] dvt[n,m,c]
// (branches in ascending order) from the rows just written.
constexpr int GB_THREADS = 256;
template <int MAXC>
__global__ void __launch_bounds__(GB_THREADS) gate_bwd_dv_kernel(const GateBwdArgs ga,
                                                                 const F32Var var,
                                                                 double* __restrict__ dv) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t n = blockIdx.x;
  const int M = ga.M, d = ga.d;
  for (int m = warp; m < M; m += GB_THREADS / 32) gate_bwd_row<MAXC>(ga, var, n * M + m, lane);
  __syncthreads();  // the rows' dvt are written (global memory, this block)
  for (int c = threadIdx.x; c < d; c += GB_THREADS) {
    double acc = 0.0;
    for (int m = 0; m < M; ++m) acc = fma(ga.alpha[n * M + m], ga.dvt[(n * M + m) * d + c], acc);
    dv[n * d + c] = acc;
  }
}

// dconv_w[mc,c,i] = sum_n sum_m dy[n,m,c] c_{n-(3-i) dil}[m,c] over the
// branches m that conv mc serves (all of them for a shared conv).  One warp
// per weight: lane l takes the (token, branch) terms l, l + 32, ... (tokens
// outer, branches inner, ascending), then a fixed butterfly, so the sum has
// the same bits on every run.
__device__ __forceinline__ void dconv_out(const double* __restrict__ dy,
                                          const double* __restrict__ v,
                                          const double* __restrict__ alpha,
                                          const double* __restrict__ rc, const F32Var& var,
                                          float* __restrict__ dw, int64_t N, int T, int M, int d,
                                          int64_t g, int lane) {
  const int i = (int)(g & 3), c = (int)((g >> 2) % d), mc = (int)((g >> 2) / d);
  const int lag = (3 - i) * var.dil;
  const int m0 = var.per_branch ? mc : 0, nm = var.per_branch ? 1 : M;
  double acc = 0.0;
  for (int64_t q = lane; q < N * nm; q += 32) {
    const int64_t n = q / nm;
    const int m = m0 + (int)(q - n * nm);
    if ((int)(n % T) < lag) continue;
    acc = fma(dy[(n * M + m) * d + c], var.conv_in(alpha, v, rc, n - lag, m, M, d, c), acc);
  }
  acc = warp_sum_d(acc);
  if (lane == 0) dw[g] = (float)acc;
}

// The learnable norm scales' gradients, one warp per (m, c), lanes taking
// the tokens l, l + 32, ... in ascending order, then a fixed butterfly:
//   dg_h = sum_n dz h^ k^ g_k / sqrt(d),  dg_k = sum_n dz h^ k^ g_h / sqrt(d),
//   dg_v = sum_n dc c^ (c^ = RMSNorm(vt), with the pre-conv norm).
__device__ __forceinline__ void dscale_out(const float* __restrict__ h,
                                           const double* __restrict__ k,
                                           const double* __restrict__ v,
                                           const double* __restrict__ alpha,
                                           const double* __restrict__ sums,
                                           const double* __restrict__ rc,
                                           const double* __restrict__ dz,
                                           const double* __restrict__ dc, const F32Var& var,
                                           float* __restrict__ dgh, float* __restrict__ dgk,
                                           float* __restrict__ dgv, int64_t N, int M, int d,
                                           int64_t gw, int lane) {
  const int g = (int)gw;
  const int m = g / d, c = g % d;
  const double isd = 1.0 / sqrt((double)d);
  double ah = 0.0, ak = 0.0, avv = 0.0;
  for (int64_t n = lane; n < N; n += 32) {
    const int64_t w = n * M + m;
    const double hk = (double)h[w * d + c] * sums[3 * w] * k[w * d + c] * sums[3 * w + 1];
    ah = fma(dz[w] * hk, (double)var.gk[g] * isd, ah);
    ak = fma(dz[w] * hk, (double)var.gh[g] * isd, ak);
    if (var.prenorm) avv = fma(dc[w * d + c], alpha[w] * v[n * d + c] * rc[w], avv);
  }
  ah = warp_sum_d(ah);
  ak = warp_sum_d(ak);
  avv = warp_sum_d(avv);
  if (lane != 0) return;
  dgh[g] = (float)ah;
  dgk[g] = (float)ak;
  if (var.prenorm) dgv[g] = (float)avv;
}

// dWk[m,c,i] = sum_n dk[n,m,c] e[n,i]; dWv[c,i] = sum_n dv[n,c] e[n,i]: one
// warp per weight, lanes taking the tokens l, l + 32, ..., then a fixed
// butterfly
__device__ __forceinline__ void dweight_out(const double* __restrict__ dk,
                                            const double* __restrict__ dv,
                                            const float* __restrict__ e, float* __restrict__ dWk,
                                            float* __restrict__ dWv, int64_t N, int M, int d, int E,
                                            int64_t g, int lane) {
  const int i = (int)(g % E);
  const int c = (int)((g / E) % d);
  const int m = (int)(g / ((int64_t)E * d));
  double acc = 0.0;
  if (m < M) {
    for (int64_t n = lane; n < N; n += 32)
      acc = fma(dk[(n * M + m) * d + c], (double)e[n * E + i], acc);
  } else {
    for (int64_t n = lane; n < N; n += 32) acc = fma(dv[n * d + c], (double)e[n * E + i], acc);
  }
  acc = warp_sum_d(acc);
  if (lane != 0) return;
  if (m < M)
    dWk[g] = (float)acc;
  else
    dWv[(int64_t)c * E + i] = (float)acc;
}

// de[n,i] = sum_m sum_c Wk[m,c,i] dk[n,m,c] + sum_c Wv[c,i] dv[n,c]: one warp
// per element, lanes taking the terms l, l + 32, ... of the (m, c) then c
// sequence, then a fixed butterfly
__device__ __forceinline__ void de_out(const double* __restrict__ dk,
                                       const double* __restrict__ dv, const float* __restrict__ Wk,
                                       const float* __restrict__ Wv, float* __restrict__ de,
                                       int64_t N, int M, int d, int E, int64_t g, int lane) {
  const int i = (int)(g % E);
  const int64_t n = g / E;
  const int Md = M * d;
  double acc = 0.0;
  for (int q = lane; q < Md + d; q += 32) {
    if (q < Md)  // q = m d + c
      acc = fma((double)Wk[(int64_t)q * E + i], dk[n * Md + q], acc);
    else
      acc = fma((double)Wv[(int64_t)(q - Md) * E + i], dv[n * d + (q - Md)], acc);
  }
  acc = warp_sum_d(acc);
  if (lane == 0) de[g] = (float)acc;
}

// The backward's sums over tokens or features in one launch, one warp per
// output: warps [0, n_conv) the conv weights, then n_scale norm scales,
// n_w weights of W_k and W_v, n_de elements of de.
struct SumsArgs {
  const double *dy, *v, *alpha, *rc, *k, *sums, *dz, *dc, *dk, *dv;
  const float *h, *e, *Wk, *Wv;
  float *dw, *dgh, *dgk, *dgv, *dWk, *dWv, *de;
  int64_t N, n_conv, n_scale, n_w, n_de;
  int T, M, d, E;
};
__global__ void bwd_sums_kernel(const SumsArgs a, const F32Var var) {
  const int lane = threadIdx.x & 31;
  int64_t g = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (g < a.n_conv) {
    dconv_out(a.dy, a.v, a.alpha, a.rc, var, a.dw, a.N, a.T, a.M, a.d, g, lane);
    return;
  }
  g -= a.n_conv;
  if (g < a.n_scale) {
    dscale_out(a.h, a.k, a.v, a.alpha, a.sums, a.rc, a.dz, a.dc, var, a.dgh, a.dgk, a.dgv, a.N,
               a.M, a.d, g, lane);
    return;
  }
  g -= a.n_scale;
  if (g < a.n_w) {
    dweight_out(a.dk, a.dv, a.e, a.dWk, a.dWv, a.N, a.M, a.d, a.E, g, lane);
    return;
  }
  g -= a.n_w;
  if (g < a.n_de) de_out(a.dk, a.dv, a.Wk, a.Wv, a.de, a.N, a.M, a.d, a.E, g, lane);
}

inline unsigned blocks_for(int64_t threads_total, int per_block) {
  return (unsigned)((threads_total + per_block - 1) / per_block);
}

// the variants of `flags` over a small-parameter block (or its gradient)
F32Var make_var(int flags, const float* block, int M, int d) {
  F32Var v;
  v.dil = (flags & ENGRAM_CONV_DILATED) ? 3 : 1;
  v.prenorm = (flags & ENGRAM_CONV_PRENORM) ? 1 : 0;
  v.per_branch = (flags & ENGRAM_CONV_PER_BRANCH) ? 1 : 0;
  v.w = block;
  v.gh = v.gk = v.gv = nullptr;
  if (flags & ENGRAM_NORM_SCALES) {
    v.gh = block + (int64_t)(v.per_branch ? M : 1) * d * 4;
    v.gk = v.gh + (int64_t)M * d;
    if (v.prenorm) v.gv = v.gk + (int64_t)M * d;
  }
  return v;
}

}  // namespace

size_t f32_saved_bytes(int64_t N, int M, int d) {
  auto up = [](size_t b) { return (b + 255) & ~(size_t)255; };
  return up(N * M * 4) + up(N * M * d * 4) + up(N * d * 4) + up(N * M * d * 4);
}

F32Saved f32_saved_layout(void* base, int64_t N, int M, int d) {
  auto up = [](size_t b) { return (b + 255) & ~(size_t)255; };
  char* p = static_cast<char*>(base);
  F32Saved s;
  s.alpha = reinterpret_cast<float*>(p);
  p += up(N * M * 4);
  s.k = reinterpret_cast<float*>(p);
  p += up(N * M * d * 4);
  s.v = reinterpret_cast<float*>(p);
  p += up(N * d * 4);
  s.y = reinterpret_cast<float*>(p);
  return s;
}

size_t f32_forward_ws_bytes(int64_t N, int M, int d) {
  auto up = [](size_t b) { return (b + 255) & ~(size_t)255; };
  return up((size_t)N * M * d * 8) + up((size_t)N * d * 8) + 2 * up((size_t)N * M * 8) +
         f32_saved_bytes(N, M, d);
}

int64_t f32_param_floats(int flags, int M, int d) {
  int64_t n = (int64_t)((flags & ENGRAM_CONV_PER_BRANCH) ? M : 1) * d * 4;
  if (flags & ENGRAM_NORM_SCALES) n += (int64_t)((flags & ENGRAM_CONV_PRENORM) ? 3 : 2) * M * d;
  return n;
}

int launch_forward_f32(const float* e, const float* h, const float* Wk, const float* Wv,
                       const float* params, int flags, float* conv_state, float* out,
                       float* saved, int64_t N, int T, int M, int d, int E, void* ws,
                       cudaStream_t s) {
  if (N == 0) return ENGRAM_OK;
  auto up = [](size_t b) { return (b + 255) & ~(size_t)255; };
  char* p = static_cast<char*>(ws);
  double* k64 = reinterpret_cast<double*>(p);
  p += up((size_t)N * M * d * 8);
  double* v64 = reinterpret_cast<double*>(p);
  p += up((size_t)N * d * 8);
  double* a64 = reinterpret_cast<double*>(p);
  p += up((size_t)N * M * 8);
  double* rc64 = reinterpret_cast<double*>(p);
  p += up((size_t)N * M * 8);
  F32Saved sv = f32_saved_layout(saved != nullptr ? static_cast<void*>(saved) : p, N, M, d);
  const F32Var var = make_var(flags, params, M, d);
  const int tb = 256;
  // (a block per token computing its projections and then its gate measured
  // alike for one branch and 7% slower for four: the warp-per-output
  // projections keep more loads in flight)
  proj_f32_kernel<<<blocks_for(N * (M + 1) * d * 32, tb), tb, 0, s>>>(e, Wk, Wv, k64, v64, sv.k,
                                                                      sv.v, N, M, d, E);
  gate_f32_kernel<<<blocks_for(N * M * 32, tb), tb, 0, s>>>(h, k64, v64, var, a64, sv.alpha,
                                                            rc64, N * M, M, d);
  conv_f32_kernel<<<blocks_for(N * M * d, tb), tb, 0, s>>>(h, v64, a64, rc64, var, conv_state,
                                                           sv.y, out, N, T, M, d);
  return ck(cudaGetLastError());
}

namespace {
struct BwdWs {
  double *k, *v, *alpha, *sums, *rc, *dz, *dy, *dvt, *dc, *dk, *dv;
  float* de;
};
size_t bwd_layout(void* base, int64_t N, int M, int d, int E, BwdWs* out) {
  auto up = [](size_t b) { return (b + 255) & ~(size_t)255; };
  const size_t NMd = (size_t)N * M * d, Nd = (size_t)N * d, NM = (size_t)N * M;
  char* p = static_cast<char*>(base);
  size_t off = 0;
  BwdWs w;
  w.k = reinterpret_cast<double*>(p + off); off += up(NMd * 8);
  w.v = reinterpret_cast<double*>(p + off); off += up(Nd * 8);
  w.alpha = reinterpret_cast<double*>(p + off); off += up(NM * 8);
  w.sums = reinterpret_cast<double*>(p + off); off += up(NM * 3 * 8);
  w.rc = reinterpret_cast<double*>(p + off); off += up(NM * 8);
  w.dz = reinterpret_cast<double*>(p + off); off += up(NM * 8);
  w.dy = reinterpret_cast<double*>(p + off); off += up(NMd * 8);
  w.dvt = reinterpret_cast<double*>(p + off); off += up(NMd * 8);
  w.dc = reinterpret_cast<double*>(p + off); off += up(NMd * 8);
  w.dk = reinterpret_cast<double*>(p + off); off += up(NMd * 8);
  w.dv = reinterpret_cast<double*>(p + off); off += up(Nd * 8);
  w.de = reinterpret_cast<float*>(p + off); off += up((size_t)N * E * 4);
  if (out) *out = w;
  return off;
}
}  // namespace

size_t backward_f32_ws_bytes(int64_t N, int M, int d, int E) {
  return bwd_layout(nullptr, N, M, d, E, nullptr);
}

float* backward_f32_de_slot(void* ws, int64_t N, int M, int d, int E) {
  BwdWs w;
  bwd_layout(ws, N, M, d, E, &w);
  return w.de;
}

int launch_backward_f32(const float* e, const float* h, const float* Wk, const float* Wv,
                        const float* params, int flags, F32Saved sv, const float* dout, float* dh,
                        float* dWk, float* dWv, float* dparams, float* de, int64_t N, int T, int M,
                        int d, int E, void* ws, cudaStream_t s) {
  (void)sv;
  BwdWs w;
  bwd_layout(ws, N, M, d, E, &w);
  const F32Var var = make_var(flags, params, M, d);
  const F32Var dvar = make_var(flags, dparams, M, d);  // where each gradient goes
  const bool scales = (flags & ENGRAM_NORM_SCALES) != 0;
  const int tb = 256;
  if (N > 0) {
    rec_proj_kernel<<<blocks_for(N * (M + 1) * d * 32, tb), tb, 0, s>>>(e, Wk, Wv, w.k, w.v, N, M,
                                                                        d, E);
    rec_gate_kernel<<<blocks_for(N * M * 32, tb), tb, 0, s>>>(h, w.k, w.v, var, w.alpha, w.sums,
                                                              w.rc, N * M, M, d);
    rec_conv_dsilu_kernel<<<blocks_for(N * M * d, tb), tb, 0, s>>>(w.v, w.alpha, w.rc, var, dout,
                                                                   w.dy, N, T, M, d);
    // a block per token: its rows of the gate backward, then dv; small d:
    // each lane's features in registers, their loads issued together
    const GateBwdArgs ga = {dout, w.dy, w.k, w.v, w.alpha, w.sums, w.rc, h, w.dvt,
                            scales ? w.dc : nullptr, scales ? w.dz : nullptr, w.dk, dh, N, T, M, d};
    if (d <= 128)
      gate_bwd_dv_kernel<4><<<(unsigned)N, GB_THREADS, 0, s>>>(ga, var, w.dv);
    else
      gate_bwd_dv_kernel<0><<<(unsigned)N, GB_THREADS, 0, s>>>(ga, var, w.dv);
  }
  const int Mc = var.per_branch ? M : 1;
  if (scales && N == 0) {  // no tokens: zero scale gradients
    const size_t nb = (size_t)(f32_param_floats(flags, M, d) - (int64_t)Mc * d * 4) * 4;
    const int rc = ck(cudaMemsetAsync(const_cast<float*>(dvar.gh), 0, nb, s));
    if (rc) return rc;
  }
  // conv weights, norm scales, W_k and W_v, de: one warp per output, one launch
  SumsArgs sa;
  sa.dy = w.dy; sa.v = w.v; sa.alpha = w.alpha; sa.rc = w.rc; sa.k = w.k; sa.sums = w.sums;
  sa.dz = w.dz; sa.dc = w.dc; sa.dk = w.dk; sa.dv = w.dv;
  sa.h = h; sa.e = e; sa.Wk = Wk; sa.Wv = Wv;
  sa.dw = dparams;
  sa.dgh = const_cast<float*>(dvar.gh);
  sa.dgk = const_cast<float*>(dvar.gk);
  sa.dgv = const_cast<float*>(dvar.gv);
  sa.dWk = dWk; sa.dWv = dWv; sa.de = de;
  sa.N = N; sa.T = T; sa.M = M; sa.d = d; sa.E = E;
  sa.n_conv = (int64_t)Mc * d * 4;
  sa.n_scale = (scales && N > 0) ? (int64_t)M * d : 0;
  sa.n_w = (int64_t)(M + 1) * d * E;
  sa.n_de = N * E;
  const int64_t warps = sa.n_conv + sa.n_scale + sa.n_w + sa.n_de;
  bwd_sums_kernel<<<blocks_for(warps * 32, tb), tb, 0, s>>>(sa, var);
  return ck(cudaGetLastError());
}

}  // namespace engram
