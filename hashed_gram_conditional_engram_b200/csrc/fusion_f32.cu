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

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float sigmoidf_(float z) { return 1.0f / (1.0f + expf(-z)); }

// k[n,m,c] = <Wk[m,c,:], e[n,:]> (m < M) and v[n,c] = <Wv[c,:], e[n,:]> (m == M):
// one warp per output, lanes stride the contraction axis.
__global__ void proj_f32_kernel(const float* __restrict__ e, const float* __restrict__ Wk,
                                const float* __restrict__ Wv, float* __restrict__ k,
                                float* __restrict__ v, int64_t N, int M, int d, int E) {
  const int lane = threadIdx.x & 31;
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t total = N * (M + 1) * d;
  if (w >= total) return;
  const int c = (int)(w % d);
  const int m = (int)((w / d) % (M + 1));
  const int64_t n = w / ((int64_t)d * (M + 1));
  const float* wrow = (m < M) ? Wk + ((int64_t)m * d + c) * E : Wv + (int64_t)c * E;
  const float* erow = e + n * E;
  float acc = 0.f;
  for (int i = lane; i < E; i += 32) acc = fmaf(__ldg(wrow + i), __ldg(erow + i), acc);
  acc = warp_sum(acc);
  if (lane == 0) {
    if (m < M) k[(n * M + m) * d + c] = acc;
    else v[n * d + c] = acc;
  }
}

// alpha[n,m] = sigmoid(<RMSNorm(h), RMSNorm(k)> / sqrt(d)): one warp per (n, m).
__global__ void gate_f32_kernel(const float* __restrict__ h, const float* __restrict__ k,
                                float* __restrict__ alpha, int64_t NM, int d) {
  const int lane = threadIdx.x & 31;
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (w >= NM) return;
  const float* hr = h + w * d;
  const float* kr = k + w * d;
  float hh = 0.f, kk = 0.f, hk = 0.f;
  for (int c = lane; c < d; c += 32) {
    const float a = hr[c], b = kr[c];
    hh = fmaf(a, a, hh);
    kk = fmaf(b, b, kk);
    hk = fmaf(a, b, hk);
  }
  hh = warp_sum(hh);
  kk = warp_sum(kk);
  hk = warp_sum(hk);
  if (lane == 0) {
    const float rh = rsqrtf(hh / d + RMS_EPS), rk = rsqrtf(kk / d + RMS_EPS);
    alpha[w] = sigmoidf_(hk * rh * rk * rsqrtf((float)d));
  }
}

// y = sum_i w[c,i] vt_{t-3+i}, out = h + vt + SiLU(y): one thread per (n, m, c).
// With conv_state (decode, T == 1) the three earlier vt come from the state,
// which is then shifted by one step.
__global__ void conv_f32_kernel(const float* __restrict__ h, const float* __restrict__ v,
                                const float* __restrict__ alpha, const float* __restrict__ w,
                                float* __restrict__ conv_state, float* __restrict__ y_out,
                                float* __restrict__ out, int64_t N, int T, int M, int d) {
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= N * M * d) return;
  const int c = (int)(g % d);
  const int m = (int)((g / d) % M);
  const int64_t n = g / ((int64_t)d * M);
  const float4 wc = *reinterpret_cast<const float4*>(w + 4 * c);
  const float taps[4] = {wc.x, wc.y, wc.z, wc.w};
  const float vt = alpha[n * M + m] * v[n * d + c];
  float y = taps[3] * vt;
  if (conv_state != nullptr) {
    float* st = conv_state + ((n * M + m) * 3) * d + c;  // [3][d] oldest first
    const float s0 = st[0], s1 = st[d], s2 = st[2 * d];
    y = fmaf(taps[0], s0, fmaf(taps[1], s1, fmaf(taps[2], s2, y)));
    st[0] = s1;
    st[d] = s2;
    st[2 * d] = vt;
  } else {
    const int t = (int)(n % T);
    for (int lag = 1; lag <= 3; ++lag) {
      if (t >= lag) {
        const int64_t p = n - lag;
        y = fmaf(taps[3 - lag], alpha[p * M + m] * v[p * d + c], y);
      }
    }
  }
  y_out[g] = y;
  out[g] = h[g] + vt + y * sigmoidf_(y);
}

// ------------------------------------------------------------------ backward

// dy = dout * SiLU'(y), SiLU'(y) = s (1 + y (1 - s)), s = sigmoid(y)
__global__ void dsilu_kernel(const float* __restrict__ dout, const float* __restrict__ y,
                             float* __restrict__ dy, int64_t total) {
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= total) return;
  const float yy = y[g];
  const float s = sigmoidf_(yy);
  dy[g] = dout[g] * s * (1.f + yy * (1.f - s));
}

// One warp per (n, m): dvt = dout + sum_i w[:,i] dy_{t+3-i}; dalpha = <dvt, v>;
// dz = dalpha a (1 - a); RMSNorm backward for h and k:
//   dx = r dxh - r^3 x <dxh, x> / d, with dh^ = dz k^ / sqrt(d), dk^ = dz h^ / sqrt(d).
__global__ void gate_bwd_kernel(const float* __restrict__ dout, const float* __restrict__ dy,
                                const float* __restrict__ h, const float* __restrict__ k,
                                const float* __restrict__ v, const float* __restrict__ alpha,
                                const float* __restrict__ w, float* __restrict__ dvt,
                                float* __restrict__ dh, float* __restrict__ dk, int64_t N, int T,
                                int M, int d) {
  const int lane = threadIdx.x & 31;
  const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (wid >= N * M) return;
  const int m = (int)(wid % M);
  const int64_t n = wid / M;
  const int t = (int)(n % T);
  const float* hr = h + wid * d;
  const float* kr = k + wid * d;
  const float* vr = v + n * d;
  float hh = 0.f, kk = 0.f, hk = 0.f, da = 0.f;
  for (int c = lane; c < d; c += 32) {
    float g = dout[wid * d + c];
    for (int lag = 1; lag <= 3; ++lag) {
      if (t + lag < T) g = fmaf(w[4 * c + 3 - lag], dy[((n + lag) * M + m) * d + c], g);
    }
    g = fmaf(w[4 * c + 3], dy[wid * d + c], g);
    dvt[wid * d + c] = g;
    da = fmaf(g, vr[c], da);
    const float a = hr[c], b = kr[c];
    hh = fmaf(a, a, hh);
    kk = fmaf(b, b, kk);
    hk = fmaf(a, b, hk);
  }
  hh = warp_sum(hh);
  kk = warp_sum(kk);
  hk = warp_sum(hk);
  da = warp_sum(da);
  const float al = alpha[wid];
  const float dz = da * al * (1.f - al);
  const float rh = rsqrtf(hh / d + RMS_EPS), rk = rsqrtf(kk / d + RMS_EPS);
  const float isd = rsqrtf((float)d);
  // <dh^, h> = dz/sqrt(d) * rk * <k, h>, <dk^, k> = dz/sqrt(d) * rh * <h, k>
  const float dot_hh = dz * isd * rk * hk;
  const float dot_kk = dz * isd * rh * hk;
  for (int c = lane; c < d; c += 32) {
    const float a = hr[c], b = kr[c];
    const float dhh = dz * isd * rk * b;
    const float dkh = dz * isd * rh * a;
    dh[wid * d + c] = dout[wid * d + c] + rh * dhh - rh * rh * rh * a * dot_hh / d;
    dk[wid * d + c] = rk * dkh - rk * rk * rk * b * dot_kk / d;
  }
}

// dv[n,c] = sum_m alpha[n,m] dvt[n,m,c], branches in ascending order
__global__ void dv_kernel(const float* __restrict__ dvt, const float* __restrict__ alpha,
                          float* __restrict__ dv, int64_t N, int M, int d) {
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= N * d) return;
  const int c = (int)(g % d);
  const int64_t n = g / d;
  float acc = 0.f;
  for (int m = 0; m < M; ++m) acc = fmaf(alpha[n * M + m], dvt[(n * M + m) * d + c], acc);
  dv[g] = acc;
}

// dconv_w[c,i] = sum_n sum_m dy[n,m,c] vt_{n-3+i}[m,c] (tokens, then branches, ascending)
__global__ void dconv_kernel(const float* __restrict__ dy, const float* __restrict__ v,
                             const float* __restrict__ alpha, float* __restrict__ dw, int64_t N,
                             int T, int M, int d) {
  const int g = blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= d * 4) return;
  const int c = g >> 2, i = g & 3, lag = 3 - i;
  float acc = 0.f;
  for (int64_t n = 0; n < N; ++n) {
    if ((int)(n % T) < lag) continue;
    const int64_t p = n - lag;
    for (int m = 0; m < M; ++m)
      acc = fmaf(dy[(n * M + m) * d + c], alpha[p * M + m] * v[p * d + c], acc);
  }
  dw[g] = acc;
}

// dWk[m,c,i] = sum_n dk[n,m,c] e[n,i]; dWv[c,i] = sum_n dv[n,c] e[n,i]
__global__ void dweight_kernel(const float* __restrict__ dk, const float* __restrict__ dv,
                               const float* __restrict__ e, float* __restrict__ dWk,
                               float* __restrict__ dWv, int64_t N, int M, int d, int E) {
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t total = (int64_t)(M + 1) * d * E;
  if (g >= total) return;
  const int i = (int)(g % E);
  const int c = (int)((g / E) % d);
  const int m = (int)(g / ((int64_t)E * d));
  float acc = 0.f;
  if (m < M) {
    for (int64_t n = 0; n < N; ++n) acc = fmaf(dk[(n * M + m) * d + c], e[n * E + i], acc);
    dWk[g] = acc;
  } else {
    for (int64_t n = 0; n < N; ++n) acc = fmaf(dv[n * d + c], e[n * E + i], acc);
    dWv[(int64_t)c * E + i] = acc;
  }
}

// de[n,i] = sum_m sum_c Wk[m,c,i] dk[n,m,c] + sum_c Wv[c,i] dv[n,c]
__global__ void de_kernel(const float* __restrict__ dk, const float* __restrict__ dv,
                          const float* __restrict__ Wk, const float* __restrict__ Wv,
                          float* __restrict__ de, int64_t N, int M, int d, int E) {
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= N * E) return;
  const int i = (int)(g % E);
  const int64_t n = g / E;
  float acc = 0.f;
  for (int m = 0; m < M; ++m)
    for (int c = 0; c < d; ++c)
      acc = fmaf(Wk[((int64_t)m * d + c) * E + i], dk[(n * M + m) * d + c], acc);
  for (int c = 0; c < d; ++c) acc = fmaf(Wv[(int64_t)c * E + i], dv[n * d + c], acc);
  de[g] = acc;
}

inline unsigned blocks_for(int64_t threads_total, int per_block) {
  return (unsigned)((threads_total + per_block - 1) / per_block);
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

int launch_forward_f32(const float* e, const float* h, const float* Wk, const float* Wv,
                       const float* conv_w, float* conv_state, float* out, F32Saved sv, int64_t N,
                       int T, int M, int d, int E, cudaStream_t s) {
  if (N == 0) return ENGRAM_OK;
  const int tb = 256;
  proj_f32_kernel<<<blocks_for(N * (M + 1) * d * 32, tb), tb, 0, s>>>(e, Wk, Wv, sv.k, sv.v, N, M,
                                                                      d, E);
  gate_f32_kernel<<<blocks_for(N * M * 32, tb), tb, 0, s>>>(h, sv.k, sv.alpha, N * M, d);
  conv_f32_kernel<<<blocks_for(N * M * d, tb), tb, 0, s>>>(h, sv.v, sv.alpha, conv_w, conv_state,
                                                           sv.y, out, N, T, M, d);
  return ck(cudaGetLastError());
}

size_t backward_f32_ws_bytes(int64_t N, int M, int d, int E) {
  auto up = [](size_t b) { return (b + 255) & ~(size_t)255; };
  // dy, dvt, dk [N,M,d]; dv [N,d]; de [N,E]
  return 3 * up((size_t)N * M * d * 4) + up((size_t)N * d * 4) + up((size_t)N * E * 4);
}

int launch_backward_f32(const float* e, const float* h, const float* Wk, const float* Wv,
                        const float* conv_w, F32Saved sv, const float* dout, float* dh, float* dWk,
                        float* dWv, float* dconv_w, float* de, int64_t N, int T, int M, int d,
                        int E, void* ws, cudaStream_t s) {
  auto up = [](size_t b) { return (b + 255) & ~(size_t)255; };
  char* p = static_cast<char*>(ws);
  float* dy = reinterpret_cast<float*>(p);
  p += up((size_t)N * M * d * 4);
  float* dvt = reinterpret_cast<float*>(p);
  p += up((size_t)N * M * d * 4);
  float* dk = reinterpret_cast<float*>(p);
  p += up((size_t)N * M * d * 4);
  float* dv = reinterpret_cast<float*>(p);
  p += up((size_t)N * d * 4);
  (void)p;
  const int tb = 256;
  if (N > 0) {
    dsilu_kernel<<<blocks_for(N * M * d, tb), tb, 0, s>>>(dout, sv.y, dy, N * M * d);
    gate_bwd_kernel<<<blocks_for(N * M * 32, tb), tb, 0, s>>>(dout, dy, h, sv.k, sv.v, sv.alpha,
                                                              conv_w, dvt, dh, dk, N, T, M, d);
    dv_kernel<<<blocks_for(N * d, tb), tb, 0, s>>>(dvt, sv.alpha, dv, N, M, d);
  }
  dconv_kernel<<<blocks_for((int64_t)d * 4, tb), tb, 0, s>>>(dy, sv.v, sv.alpha, dconv_w, N, T, M,
                                                             d);
  dweight_kernel<<<blocks_for((int64_t)(M + 1) * d * E, tb), tb, 0, s>>>(dk, dv, e, dWk, dWv, N,
                                                                         M, d, E);
  if (N > 0)
    de_kernel<<<blocks_for(N * E, tb), tb, 0, s>>>(dk, dv, Wk, Wv, de, N, M, d, E);
  return ck(cudaGetLastError());
}

}  // namespace engram
