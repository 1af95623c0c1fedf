// The pre-conv RMSNorm variant of the bf16 layer (ENGRAM_CONV_PRENORM):
// the conv reads c = RMSNorm(vt) g_v, vt = alpha v, instead of vt.
//
// The norm needs, per token, the sum of squares over all d features of vt,
// while the tensor-core pass V spreads a token's features over the CTAs of
// its tile.  So with this variant the layer runs pass K and the gate as
// usual, then v = e W_v^T as a plain tensor-core GEMM (fp32 out), one warp per
// token for rc = (alpha^2 <v, v> / d + eps)^(-1/2) (RMSNorm(vt) = rc vt),
// and a walk along each feature over the tokens for the conv, SiLU and
// residual: out = h + vt + SiLU(y), y_t = sum_i w_i c_{t-(3-i) dil}.
//
// Method: discuss.deepseek.club 二.1 (2) (1-D conv over the gated value,
// residual); the norm before the conv and its learnable scale g_v are one of
// the formulations the pages leave open.
#include "internal.cuh"

namespace engram {

namespace {

constexpr float PN_EPS = 1e-6f;  // the RMSNorm epsilon of the layer
constexpr int PN_TOK = 128;       // tokens per thread of the conv walk
constexpr int PN_THREADS = 128;   // feature pairs per block of the conv walk

// rc[t] = (alpha_t^2 <v_t, v_t> / d + eps)^(-1/2): one warp per token, the
// lanes' sums of squares added in a fixed butterfly order
__global__ void prenorm_rc_kernel(const float* __restrict__ v, int ldv,
                                  const float* __restrict__ alpha, int64_t N, int d,
                                  float* __restrict__ rc) {
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (t >= N) return;
  const float4* row = reinterpret_cast<const float4*>(v + t * ldv);
  float s = 0.f;
  for (int i = lane; i < d / 4; i += 32) {
    const float4 x = row[i];
    s = fmaf(x.x, x.x, fmaf(x.y, x.y, fmaf(x.z, x.z, fmaf(x.w, x.w, s))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) {
    const float a = alpha[t];
    rc[t] = rsqrtf(a * a * s / (float)d + PN_EPS);
  }
}

__device__ __forceinline__ float silu(float y) { return __fdividef(y, 1.0f + __expf(-y)); }

// Whole sequences: thread = (feature pair, chunk of PN_TOK tokens); it first
// rebuilds the conv inputs of the 3 dil tokens before its chunk (within the
// sequence), then walks the chunk keeping them in a register ring.
template <int DIL>
__global__ void __launch_bounds__(PN_THREADS) prenorm_conv_kernel(
    const float* __restrict__ v, int ldv, const float* __restrict__ alpha,
    const float* __restrict__ rc, const float4* __restrict__ conv_w,
    const float* __restrict__ gv, const __nv_bfloat16* __restrict__ h,
    __nv_bfloat16* __restrict__ out, int64_t N, int T, int d) {
  constexpr int NH = 3 * DIL;
  const int f = (blockIdx.x * PN_THREADS + threadIdx.x) * 2;
  if (f >= d) return;
  const int64_t t0 = (int64_t)blockIdx.y * PN_TOK;
  const int64_t t1 = t0 + PN_TOK < N ? t0 + PN_TOK : N;
  const float4 wx = __ldg(conv_w + f), wy = __ldg(conv_w + f + 1);
  const float2 g = gv != nullptr ? *reinterpret_cast<const float2*>(gv + f) : make_float2(1.f, 1.f);
  float2 hist[NH];  // hist[k]: conv input of token t-1-k (zero before the sequence)
  int pos = (int)(t0 % T);
#pragma unroll
  for (int k = 0; k < NH; ++k) {
    hist[k] = make_float2(0.f, 0.f);
    if (pos >= k + 1) {
      const int64_t tt = t0 - 1 - k;
      const float q = alpha[tt] * rc[tt];
      const float2 x = *reinterpret_cast<const float2*>(v + tt * ldv + f);
      hist[k] = make_float2(q * g.x * x.x, q * g.y * x.y);
    }
  }
#pragma unroll 4
  for (int64_t t = t0; t < t1; ++t) {
    if (pos == 0) {
#pragma unroll
      for (int k = 0; k < NH; ++k) hist[k] = make_float2(0.f, 0.f);
    }
    const float a = alpha[t], q = a * rc[t];
    const float2 x = *reinterpret_cast<const float2*>(v + t * ldv + f);
    const float2 c = make_float2(q * g.x * x.x, q * g.y * x.y);
    // taps: w.x reads c_{t-3 dil}, w.y c_{t-2 dil}, w.z c_{t-dil}, w.w c_t
    const float yx = fmaf(wx.x, hist[NH - 1].x,
                          fmaf(wx.y, hist[2 * DIL - 1].x, fmaf(wx.z, hist[DIL - 1].x, wx.w * c.x)));
    const float yy = fmaf(wy.x, hist[NH - 1].y,
                          fmaf(wy.y, hist[2 * DIL - 1].y, fmaf(wy.z, hist[DIL - 1].y, wy.w * c.y)));
    const __nv_bfloat162 hv = *reinterpret_cast<const __nv_bfloat162*>(h + t * d + f);
    const float2 hf = __bfloat1622float2(hv);
    *reinterpret_cast<__nv_bfloat162*>(out + t * d + f) =
        __floats2bfloat162_rn(hf.x + a * x.x + silu(yx), hf.y + a * x.y + silu(yy));
#pragma unroll
    for (int k = NH - 1; k > 0; --k) hist[k] = hist[k - 1];
    hist[0] = c;
    pos = pos + 1 == T ? 0 : pos + 1;
  }
}

// Decode (one token per sequence): state [B, 3 dil, d] holds the conv inputs
// of the 3 dil previous steps, oldest first; it is shifted and this step's c
// appended.
template <int DIL>
__global__ void prenorm_decode_kernel(const float* __restrict__ v, int ldv,
                                      const float* __restrict__ alpha,
                                      const float* __restrict__ rc,
                                      const float4* __restrict__ conv_w,
                                      const float* __restrict__ gv,
                                      const __nv_bfloat16* __restrict__ h,
                                      __nv_bfloat16* __restrict__ out, float* __restrict__ state,
                                      int64_t B, int d) {
  constexpr int NH = 3 * DIL;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= B * d) return;
  const int64_t b = i / d;
  const int f = (int)(i - b * d);
  const float a = alpha[b], q = a * rc[b];
  const float x = v[b * ldv + f];
  const float c = q * (gv != nullptr ? gv[f] : 1.f) * x;
  const float4 w = __ldg(conv_w + f);
  float* st = state + b * NH * d + f;  // st[j d]: input of step -(NH - j)
  const float y = fmaf(w.x, st[0], fmaf(w.y, st[(NH - 2 * DIL) * d],
                                        fmaf(w.z, st[(NH - DIL) * d], w.w * c)));
  const float hv = __bfloat162float(h[b * d + f]);
  out[b * d + f] = __float2bfloat16_rn(hv + a * x + silu(y));
#pragma unroll
  for (int j = 0; j < NH - 1; ++j) st[j * d] = st[(j + 1) * d];
  st[(NH - 1) * d] = c;
}

}  // namespace

int launch_prenorm_rc(const float* v, int ldv, const float* alpha, int64_t N, int d, float* rc,
                      cudaStream_t s) {
  if (N == 0) return ENGRAM_OK;
  prenorm_rc_kernel<<<(unsigned)((N + 7) / 8), 256, 0, s>>>(v, ldv, alpha, N, d, rc);
  return ck(cudaGetLastError());
}

int launch_prenorm_tail(const PrenormFwd& p, const __nv_bfloat16* e, const __nv_bfloat16* Wv,
                        const __nv_bfloat16* h, const float* conv_w, const float* alpha,
                        float* conv_state, __nv_bfloat16* out, int dil, int64_t N, int T, int d,
                        int E, bool stall, cudaStream_t s) {
  // v = e W_v^T, fp32, rows ldv apart
  int rc = launch_gemm_kv(e, nullptr, Wv, N, d, E, p.vbuf, p.ldv, s, stall);
  if (rc) return rc;
  if ((rc = launch_prenorm_rc(p.vbuf, p.ldv, alpha, N, d, p.rc, s))) return rc;
  const float4* w = reinterpret_cast<const float4*>(conv_w);
  if (conv_state != nullptr) {
    const unsigned grid = (unsigned)((N * d + 255) / 256);
    if (dil == 3)
      prenorm_decode_kernel<3><<<grid, 256, 0, s>>>(p.vbuf, p.ldv, alpha, p.rc, w, p.gv, h, out,
                                                    conv_state, N, d);
    else
      prenorm_decode_kernel<1><<<grid, 256, 0, s>>>(p.vbuf, p.ldv, alpha, p.rc, w, p.gv, h, out,
                                                    conv_state, N, d);
  } else {
    if ((N + PN_TOK - 1) / PN_TOK > 65535) return ENGRAM_ERR_UNSUPPORTED;
    const dim3 grid((unsigned)((d / 2 + PN_THREADS - 1) / PN_THREADS),
                    (unsigned)((N + PN_TOK - 1) / PN_TOK));
    if (dil == 3)
      prenorm_conv_kernel<3><<<grid, PN_THREADS, 0, s>>>(p.vbuf, p.ldv, alpha, p.rc, w, p.gv, h,
                                                         out, N, T, d);
    else
      prenorm_conv_kernel<1><<<grid, PN_THREADS, 0, s>>>(p.vbuf, p.ldv, alpha, p.rc, w, p.gv, h,
                                                         out, N, T, d);
  }
  return ck(cudaGetLastError());
}

}  // namespace engram
