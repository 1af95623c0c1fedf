// Backward of the bf16 layer (one branch) at full scale.
//
// The four dense contractions of the backward are plain GEMMs with no work
// to fuse into them: k and v are recomputed as e W_k^T and e W_v^T, the
// weight gradients are contractions over tokens (dW = d{k,v}^T e) and the
// row gradient is de = dk W_k + dv W_v.  They run in cuBLAS (bf16 operands,
// fp32 accumulation), loaded with dlopen on first use so that the library
// itself has no load-time dependency on it.  Everything between them -- the
// conv and SiLU backward, the gate, both RMSNorm backwards -- is in the
// kernels below, and the table rows' gradient goes through the same
// deterministic sort-and-segment-sum as the fp32 path.
//
// Method: discuss.deepseek.club 二.1 (2) (gate with h as query, e as key and
// value; 1-D conv; residual); gitcode.csdn.net blog, end-to-end training
// paragraph (deterministic lookups give consistent gradients to the slots).
#include <cublas_v2.h>
#include <dlfcn.h>

#include <mutex>

#include "internal.cuh"

namespace engram {

namespace {

// ------------------------------------------------------------ cuBLAS, loaded late

struct Blas {
  bool ok = false;
  cublasStatus_t (*create)(cublasHandle_t*) = nullptr;
  cublasStatus_t (*set_stream)(cublasHandle_t, cudaStream_t) = nullptr;
  cublasStatus_t (*set_workspace)(cublasHandle_t, void*, size_t) = nullptr;
  cublasStatus_t (*gemm_ex)(cublasHandle_t, cublasOperation_t, cublasOperation_t, int, int, int,
                            const void*, const void*, cudaDataType, int, const void*, cudaDataType,
                            int, const void*, void*, cudaDataType, int, cublasComputeType_t,
                            cublasGemmAlgo_t) = nullptr;
};

Blas& blas() {
  static Blas b;
  static std::once_flag once;
  std::call_once(once, [] {
    void* h = dlopen("libcublas.so.12", RTLD_NOW | RTLD_LOCAL);
    if (h == nullptr) return;
    b.create = reinterpret_cast<decltype(b.create)>(dlsym(h, "cublasCreate_v2"));
    b.set_stream = reinterpret_cast<decltype(b.set_stream)>(dlsym(h, "cublasSetStream_v2"));
    b.set_workspace =
        reinterpret_cast<decltype(b.set_workspace)>(dlsym(h, "cublasSetWorkspace_v2"));
    b.gemm_ex = reinterpret_cast<decltype(b.gemm_ex)>(dlsym(h, "cublasGemmEx"));
    b.ok = b.create && b.set_stream && b.set_workspace && b.gemm_ex;
  });
  return b;
}

constexpr int kMaxDevices = 64;
constexpr size_t kBlasWorkspace = 32u << 20;  // from the caller's workspace

// One handle per device, created on first use and kept for the process.
int blas_handle(cudaStream_t s, void* workspace, cublasHandle_t* out) {
  static cublasHandle_t handles[kMaxDevices] = {};
  static std::mutex mu;
  Blas& b = blas();
  if (!b.ok) return ENGRAM_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ENGRAM_ERR_CUDA;
  std::lock_guard<std::mutex> lk(mu);
  if (handles[dev] == nullptr && b.create(&handles[dev]) != CUBLAS_STATUS_SUCCESS) {
    handles[dev] = nullptr;
    return ENGRAM_ERR_CUDA;
  }
  if (b.set_stream(handles[dev], s) != CUBLAS_STATUS_SUCCESS ||
      b.set_workspace(handles[dev], workspace, kBlasWorkspace) != CUBLAS_STATUS_SUCCESS)
    return ENGRAM_ERR_CUDA;
  *out = handles[dev];
  return ENGRAM_OK;
}

// C[m x n] (row-major, fp32, row stride ldc) = op(A)[m x k] . op(B)[k x n]
// + beta * C with A, B bf16 row-major: op(A) = A (a_t = false, A is [m x k])
// or A^T (A is [k x m]), rows lda apart; likewise B.  Row-major C = A.B is
// column-major C^T = B^T.A^T, which is what cuBLAS is asked for.
int gemm_rm(cublasHandle_t hd, bool a_t, bool b_t, int m, int n, int k, const void* A, int lda,
            const void* B, int ldb, float* C, int ldc, float beta) {
  const float alpha = 1.0f;
  const cublasOperation_t opB = b_t ? CUBLAS_OP_T : CUBLAS_OP_N;
  const cublasOperation_t opA = a_t ? CUBLAS_OP_T : CUBLAS_OP_N;
  const cublasStatus_t st =
      blas().gemm_ex(hd, opB, opA, n, m, k, &alpha, B, CUDA_R_16BF, ldb, A, CUDA_R_16BF, lda,
                     &beta, C, CUDA_R_32F, ldc, CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT);
  return st == CUBLAS_STATUS_SUCCESS ? ENGRAM_OK : ENGRAM_ERR_CUDA;
}

// ------------------------------------------------------------ elementwise backward
//
// Notation per token t and feature f (u = dout):
//   vt = alpha v, y_t = sum_i w_i vt_{t-3+i} (zero before the sequence start),
//   out = h + vt + SiLU(y)
//   dy_t = u_t SiLU'(y_t),  SiLU'(y) = s (1 + y (1 - s)), s = sigmoid(y)
//   dvt_t = u_t + sum_{s = t..t+3, same sequence} w_{3-(s-t)} dy_s
//   dalpha = <dvt, v>, dv = alpha dvt, dz = dalpha alpha (1 - alpha)
//   dh^ = dz k^ / sqrt(d), dk^ = dz h^ / sqrt(d)   (h^ = r_h h, k^ = r_k k)
//   RMSNorm backward: dx = r dx^ - r^3 x <dx^, x> / d, where
//   <dh^, h> = dz r_k <k, h> / sqrt(d) and <dk^, k> = dz r_h <h, k> / sqrt(d)
//   dh = u + r_h dh^ - r_h^3 h <dh^, h> / d,  dk = r_k dk^ - r_k^3 k <dk^, k> / d
//   dw_i = sum_t dy_t vt_{t-3+i}

__device__ __forceinline__ float silu_grad(float y) {
  const float sg = __fdividef(1.0f, 1.0f + __expf(-y));
  return sg * (1.0f + y * (1.0f - sg));
}

constexpr int ROW_THREADS = 256;
constexpr float BW_RMS_EPS = 1e-6f;  // the forward's RMSNorm epsilon

// Sum of a value over the block, the same order on every run.
__device__ __forceinline__ float block_sum(float x, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();  // red is reused
  if (lane == 0) red[warp] = x;
  __syncthreads();
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < ROW_THREADS / 32; ++i) s += red[i];
  return s;
}

constexpr int COL_TOK = 128;      // tokens per column chunk
constexpr int COL_THREADS = 128;  // features per block

// One thread per (feature, chunk of COL_TOK tokens), walking the chunk in
// token order with the three previous tokens' vt, v, alpha, dy and dout in
// registers.  At token t it forms y_t and dy_t.  dvt of token t-3 is complete
// then (its vt enters y_{t-3} .. y_t), or earlier when its sequence ends; the
// walk runs 3 tokens past the chunk for those dy.  `live` counts the ring's
// tokens that belong to t's sequence and lie in this chunk's walk.  For each
// completed token the walk writes dv = alpha dvt (bf16, for the GEMMs) and
// the warp's partial of dalpha = <dvt, v> over its 32 features (fixed
// butterfly order), dalpha_part[token][f / 32]; and at the end the chunk's
// partial conv-weight gradient part[chunk][f] = sum over its tokens of
// dy_t * (vt_{t-3}, vt_{t-2}, vt_{t-1}, vt_t).  All lanes of a warp walk the
// same tokens, so the warp-wide sums run on uniform branches.
// j: the token's index within the walk (token t0 + j); dvb, pab point at
// token t0's dv element and dalpha partial of this thread / warp.
__device__ __forceinline__ void col_emit(float r, float v_tok, float a_tok, int j, int d, int ld,
                                         __nv_bfloat16* __restrict__ dvb,
                                         float* __restrict__ pab) {
  dvb[j * ld] = __float2bfloat16_rn(a_tok * r);
  float p = r * v_tok;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
  if ((threadIdx.x & 31) == 0) pab[j * (d / 32)] = p;
}

__global__ void __launch_bounds__(COL_THREADS, 8) bw_col_kernel(
    const float* __restrict__ v, const float* __restrict__ alpha,
    const float4* __restrict__ conv_w, const float* __restrict__ dout, int64_t N, int T, int d,
    int ld, __nv_bfloat16* __restrict__ dv, float* __restrict__ dalpha_part,
    float4* __restrict__ part) {
  // v and dv rows are ld apart (they share rows with k and dk), dout rows d
  const int f = blockIdx.y * COL_THREADS + threadIdx.x;  // d is a multiple of COL_THREADS
  const int64_t t0 = (int64_t)blockIdx.x * COL_TOK;
  const int64_t t1 = t0 + COL_TOK < N ? t0 + COL_TOK : N;
  const int64_t t_stop = t1 + 3 < N ? t1 + 3 : N;
  // the gates of the walk's tokens (and the 3 before it), staged once
  __shared__ float al_s[COL_TOK + 6];
  for (int i = threadIdx.x; i < COL_TOK + 6; i += COL_THREADS) {
    const int64_t tt = t0 - 3 + i;
    al_s[i] = (tt >= 0 && tt < t_stop) ? alpha[tt] : 0.f;
  }
  __syncthreads();
  auto al = [&](int64_t tt) { return al_s[(int)(tt - t0) + 3]; };  // t0 - 3 <= tt < t_stop
  const float4 w = __ldg(conv_w + f);
  int pos = (int)(t0 % T);
  float s1 = 0.f, s2 = 0.f, s3 = 0.f;  // vt of t-1, t-2, t-3 (zero before the sequence start)
  if (pos >= 1) s1 = al(t0 - 1) * v[(t0 - 1) * ld + f];
  if (pos >= 2) s2 = al(t0 - 2) * v[(t0 - 2) * ld + f];
  if (pos >= 3) s3 = al(t0 - 3) * v[(t0 - 3) * ld + f];
  float g1 = 0.f, g2 = 0.f, g3 = 0.f;  // dy of t-1, t-2, t-3
  float u1 = 0.f, u2 = 0.f, u3 = 0.f;  // dout
  float v1 = 0.f, v2 = 0.f, v3 = 0.f;  // v
  float al1 = 0.f, al2 = 0.f, al3 = 0.f;  // alpha
  int live = 0;
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  __nv_bfloat16* dvb = dv + t0 * ld + f;
  float* pab = dalpha_part + t0 * (d / 32) + f / 32;
  const int n_chunk = (int)(t1 - t0);
  // the next PF tokens' v and dout, loaded ahead of the walk; row pointers
  // advance by d per token (no 64-bit index products in the loop)
  constexpr int PF = 4;
  float pv[PF], pu[PF];
  const float* vp = v + t0 * ld + f;
  const float* up = dout + t0 * d + f;
  const int n_walk = (int)(t_stop - t0);
#pragma unroll
  for (int q = 0; q < PF; ++q) {
    pv[q] = q < n_walk ? vp[(int64_t)q * ld] : 0.f;
    pu[q] = q < n_walk ? up[(int64_t)q * d] : 0.f;
  }
  vp += (int64_t)PF * ld;
  up += (int64_t)PF * d;
#pragma unroll 4
  for (int i = 0; i < n_walk; ++i) {
    const float vr = pv[0], at = al_s[i + 3], ut = pu[0];
#pragma unroll
    for (int q = 0; q < PF - 1; ++q) {
      pv[q] = pv[q + 1];
      pu[q] = pu[q + 1];
    }
    const bool more = i + PF < n_walk;
    pv[PF - 1] = more ? *vp : 0.f;
    pu[PF - 1] = more ? *up : 0.f;
    vp += ld;
    up += d;
    if (pos == 0) {  // a sequence starts at t
      s1 = s2 = s3 = 0.f;
      live = 0;
    }
    const float vt = at * vr;
    const float y = fmaf(w.x, s3, fmaf(w.y, s2, fmaf(w.z, s1, w.w * vt)));
    const float gt = ut * silu_grad(y);
    if (i < n_chunk) {
      a0 = fmaf(gt, s3, a0);
      a1 = fmaf(gt, s2, a1);
      a2 = fmaf(gt, s1, a2);
      a3 = fmaf(gt, vt, a3);
    }
    if (live == 3 && i >= 3)
      col_emit(u3 + w.w * g3 + w.z * g2 + w.y * g1 + w.x * gt, v3, al3, i - 3, d, ld, dvb, pab);
    if (pos == T - 1) {  // the sequence ends at token i: its last tokens are complete
      if (live >= 2 && i >= 2 && i - 2 < n_chunk)
        col_emit(u2 + w.w * g2 + w.z * g1 + w.y * gt, v2, al2, i - 2, d, ld, dvb, pab);
      if (live >= 1 && i >= 1 && i - 1 < n_chunk)
        col_emit(u1 + w.w * g1 + w.z * gt, v1, al1, i - 1, d, ld, dvb, pab);
      if (i < n_chunk) col_emit(ut + w.w * gt, vr, at, i, d, ld, dvb, pab);
    }
    s3 = s2;
    s2 = s1;
    s1 = vt;
    g3 = g2;
    g2 = g1;
    g1 = gt;
    u3 = u2;
    u2 = u1;
    u1 = ut;
    v3 = v2;
    v2 = v1;
    v1 = vr;
    al3 = al2;
    al2 = al1;
    al1 = at;
    live = live < 3 ? live + 1 : 3;
    pos = pos + 1 == T ? 0 : pos + 1;
  }
  if (t1 > t0) part[(int64_t)blockIdx.x * d + f] = make_float4(a0, a1, a2, a3);
}

constexpr int ROW_MAX_ITEMS = 16;  // d <= ROW_THREADS * ROW_MAX_ITEMS = 4,096

// One block per token: the gate and both RMSNorm backwards need whole-row
// sums; the row's h and k are read once into registers, dalpha is the sum of
// the column walk's d/32 partials (in order), then dk (bf16, for the GEMMs)
// and dh are written.
__global__ void __launch_bounds__(ROW_THREADS) bw_row_kernel(
    const __nv_bfloat16* __restrict__ h, const float* __restrict__ k,
    const float* __restrict__ alpha, const float* __restrict__ dout,
    const float* __restrict__ dalpha_part, int64_t N, int d, int ld, float* __restrict__ dh,
    __nv_bfloat16* __restrict__ dk_out) {
  // k and dk rows are ld apart (they share rows with v and dv)
  __shared__ float red[ROW_THREADS / 32];
  const int64_t t = blockIdx.x;
  if (t >= N) return;
  const int64_t r0 = t * d;
  float hv[ROW_MAX_ITEMS], kv[ROW_MAX_ITEMS];
  float shh = 0.f, skk = 0.f, shk = 0.f;
#pragma unroll
  for (int q = 0; q < ROW_MAX_ITEMS; ++q) {
    const int f = threadIdx.x + q * ROW_THREADS;
    hv[q] = kv[q] = 0.f;
    if (f < d) {
      hv[q] = __bfloat162float(h[r0 + f]);
      kv[q] = k[t * ld + f];
      shh = fmaf(hv[q], hv[q], shh);
      skk = fmaf(kv[q], kv[q], skk);
      shk = fmaf(hv[q], kv[q], shk);
    }
  }
  // dalpha: the d/32 warp partials of the column walk, added in order by
  // the first warp then broadcast
  float sgv = 0.f;
  if (threadIdx.x < 32) {
    const float* pp = dalpha_part + t * (d / 32);
    for (int i = threadIdx.x; i < d / 32; i += 32) sgv += pp[i];
  }
  shh = block_sum(shh, red);
  skk = block_sum(skk, red);
  shk = block_sum(shk, red);
  sgv = block_sum(sgv, red);
  const float invd = 1.0f / (float)d, isd = rsqrtf((float)d);
  const float rh = rsqrtf(shh * invd + BW_RMS_EPS), rk = rsqrtf(skk * invd + BW_RMS_EPS);
  const float a = alpha[t];
  const float c = sgv * a * (1.0f - a) * isd;  // dz / sqrt(d): dh^ = c k^, dk^ = c h^
  const float ch = rh * rh * rh * (c * rk * shk) * invd;   // r_h^3 <dh^, h> / d
  const float ck = rk * rk * rk * (c * rh * shk) * invd;   // r_k^3 <dk^, k> / d
#pragma unroll
  for (int q = 0; q < ROW_MAX_ITEMS; ++q) {
    const int f = threadIdx.x + q * ROW_THREADS;
    if (f < d) {
      dk_out[t * ld + f] = __float2bfloat16_rn(rk * (c * rh * hv[q]) - ck * kv[q]);
      dh[r0 + f] = dout[r0 + f] + rh * (c * rk * kv[q]) - ch * hv[q];
    }
  }
}

// dconv_w[f] = sum over chunks in order.
__global__ void bw_dconv_reduce_kernel(const float4* __restrict__ part, int chunks, int d,
                                       float4* __restrict__ dw) {
  const int f = blockIdx.x * blockDim.x + threadIdx.x;
  if (f >= d) return;
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int c = 0; c < chunks; ++c) {
    const float4 p = part[(int64_t)c * d + f];
    s.x += p.x;
    s.y += p.y;
    s.z += p.z;
    s.w += p.w;
  }
  dw[f] = s;
}

// Workspace: k, v fp32 [N, d], dalpha partials (sized [N, d] for simplicity); dk, dv bf16 [N, d]; de fp32 [N, E] when
// the caller passes none; conv partials; cuBLAS's workspace; the table
// gradient's sort buffers.
struct BwdBf16Ws {
  // k and v stay fp32: dh and dalpha are sums whose terms can cancel, so a
  // bf16 rounding of k or v would show at full size in a small result.
  // They share rows (kv [N, 2d] = [k | v]), as do dk and dv, and W_k, W_v
  // are stacked (Wkv [2d, E]), so that each pair of GEMMs is one.
  float* kv;
  __nv_bfloat16* dkv;
  __nv_bfloat16* Wkv;
  float* dWkv;          // [2d, E], copied out to dWk and dWv
  float *dalpha_part, *de;  // [N, d/32] partials of <dvt, v>
  float4* part;
  void* blas_ws;
  void* tg_ws;
  size_t tg_bytes;
};

constexpr size_t up256b(size_t b) { return (b + 255) & ~(size_t)255; }

size_t bwd_bf16_layout(void* base, int64_t N, int d, int E, int J, BwdBf16Ws* w) {
  const int64_t chunks = (N + COL_TOK - 1) / COL_TOK;
  const size_t KV = up256b((size_t)N * 2 * d * 4), DKV = up256b((size_t)N * 2 * d * 2);
  const size_t WKV = up256b((size_t)2 * d * E * 2), DW = up256b((size_t)2 * d * E * 4);
  const size_t DA = up256b((size_t)N * (d / 32) * 4);
  const size_t NE4 = up256b((size_t)N * E * 4), P = up256b((size_t)chunks * d * 16);
  const size_t tg = table_grad_ws_bytes(N * J);
  size_t off[9];
  const size_t sz[9] = {KV, DKV, WKV, DW, DA, NE4, P, kBlasWorkspace, tg};
  size_t o = 0;
  for (int i = 0; i < 9; ++i) {
    off[i] = o;
    o += sz[i];
  }
  if (w != nullptr) {
    char* p = static_cast<char*>(base);
    w->kv = reinterpret_cast<float*>(p + off[0]);
    w->dkv = reinterpret_cast<__nv_bfloat16*>(p + off[1]);
    w->Wkv = reinterpret_cast<__nv_bfloat16*>(p + off[2]);
    w->dWkv = reinterpret_cast<float*>(p + off[3]);
    w->dalpha_part = reinterpret_cast<float*>(p + off[4]);
    w->de = reinterpret_cast<float*>(p + off[5]);
    w->part = reinterpret_cast<float4*>(p + off[6]);
    w->blas_ws = p + off[7];
    w->tg_ws = p + off[8];
    w->tg_bytes = tg;
  }
  return o;
}

}  // namespace

size_t backward_bf16_ws_bytes(int64_t N, int d, int E, int J) {
  return bwd_bf16_layout(nullptr, N, d, E, J, nullptr);
}

int launch_backward_bf16(const HeadParams& hp, const int32_t* idx, const __nv_bfloat16* e,
                         const __nv_bfloat16* h, const __nv_bfloat16* Wk,
                         const __nv_bfloat16* Wv, const float* conv_w, const float* alpha,
                         const float* dout, float* dh, float* dWk, float* dWv, float* dconv_w,
                         float* de, int64_t* dtab_keys, float* dtab_rows, int32_t* n_unique,
                         int64_t N, int T, int d, void* ws, size_t ws_bytes, cudaStream_t s) {
  const int E = hp.E;
  if (ws_bytes < backward_bf16_ws_bytes(N, d, E, hp.J)) return ENGRAM_ERR_WORKSPACE;
  if (N > 0x7fffffffLL / 8) return ENGRAM_ERR_UNSUPPORTED;  // cuBLAS takes int sizes
  if (d > ROW_THREADS * ROW_MAX_ITEMS || d % COL_THREADS != 0)
    return ENGRAM_ERR_UNSUPPORTED;  // a row in registers; whole column blocks
  BwdBf16Ws w;
  bwd_bf16_layout(ws, N, d, E, hp.J, &w);
  if (de == nullptr) de = w.de;
  cublasHandle_t hd;
  int rc = blas_handle(s, w.blas_ws, &hd);
  if (rc) return rc;
  const int n = (int)N;
  // W_k and W_v stacked, then [k | v] = e [W_k; W_v]^T (fp32)
  const size_t wbytes = (size_t)d * E * 2;
  if ((rc = ck(cudaMemcpyAsync(w.Wkv, Wk, wbytes, cudaMemcpyDeviceToDevice, s)))) return rc;
  if ((rc = ck(cudaMemcpyAsync(w.Wkv + (size_t)d * E, Wv, wbytes, cudaMemcpyDeviceToDevice, s))))
    return rc;
  if ((rc = gemm_rm(hd, false, true, n, 2 * d, E, e, E, w.Wkv, E, w.kv, 2 * d, 0.f))) return rc;
  const int chunks = (int)((N + COL_TOK - 1) / COL_TOK);
  bw_col_kernel<<<dim3((unsigned)chunks, (unsigned)(d / COL_THREADS)), COL_THREADS, 0, s>>>(
      w.kv + d, alpha, reinterpret_cast<const float4*>(conv_w), dout, N, T, d, 2 * d, w.dkv + d,
      w.dalpha_part, w.part);
  bw_row_kernel<<<(unsigned)N, ROW_THREADS, 0, s>>>(h, w.kv, alpha, dout, w.dalpha_part, N, d,
                                                    2 * d, dh, w.dkv);
  bw_dconv_reduce_kernel<<<(unsigned)((d + 255) / 256), 256, 0, s>>>(
      w.part, chunks, d, reinterpret_cast<float4*>(dconv_w));
  if ((rc = ck(cudaGetLastError()))) return rc;
  // [dW_k; dW_v] = [dk | dv]^T e (a contraction over tokens), then split;
  // de = [dk | dv] [W_k; W_v]
  if ((rc = gemm_rm(hd, true, false, 2 * d, E, n, w.dkv, 2 * d, e, E, w.dWkv, E, 0.f))) return rc;
  const size_t gbytes = (size_t)d * E * 4;
  if ((rc = ck(cudaMemcpyAsync(dWk, w.dWkv, gbytes, cudaMemcpyDeviceToDevice, s)))) return rc;
  if ((rc = ck(cudaMemcpyAsync(dWv, w.dWkv + (size_t)d * E, gbytes, cudaMemcpyDeviceToDevice, s))))
    return rc;
  if ((rc = gemm_rm(hd, false, false, n, E, 2 * d, w.dkv, 2 * d, w.Wkv, E, de, E, 0.f))) return rc;
  // the table rows' gradient from de, in the deterministic order
  return launch_table_grad(hp, idx, de, N, dtab_keys, dtab_rows, n_unique, w.tg_ws, w.tg_bytes, s);
}

}  // namespace engram
