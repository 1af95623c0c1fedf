// Backward of the bf16 layer (one branch) at full scale.
//
// The dense contractions of the backward are plain GEMMs with no work to
// fuse into them: k and v are recomputed as e W_k^T and e W_v^T (unless the
// forward kept them), the weight gradients are contractions over tokens
// (dW = d{k,v}^T e) and the row gradient is de = dk W_k + dv W_v.  They run
// on the tensor cores (gemm_tc.cu: tcgen05, bf16 operands, fp32
// accumulation).  Everything between them -- the conv and SiLU backward, the
// gate, both RMSNorm backwards -- is in the kernels below, and the table
// rows' gradient goes through the same deterministic sort-and-segment-sum as
// the fp32 path.
//
// Method: discuss.deepseek.club 二.1 (2) (gate with h as query, e as key and
// value; 1-D conv; residual); gitcode.csdn.net blog, end-to-end training
// paragraph (deterministic lookups give consistent gradients to the slots).
#include <algorithm>
#include <mutex>

#include "internal.cuh"

namespace engram {

namespace {

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

// SiLU'(y) = s (1 + y (1 - s)), s = sigmoid(y), for two features at once:
// the arithmetic around the two exponentials and reciprocals runs on packed
// fp32 pairs.
__device__ __forceinline__ float2 silu_grad2(float2 y) {
  const float2 one = make_float2(1.0f, 1.0f);
  const float2 den = __fadd2_rn(one, make_float2(__expf(-y.x), __expf(-y.y)));
  const float2 sg = make_float2(__fdividef(1.0f, den.x), __fdividef(1.0f, den.y));
  const float2 om = __ffma2_rn(make_float2(-1.0f, -1.0f), sg, one);  // 1 - s
  return __fmul2_rn(sg, __ffma2_rn(y, om, one));
}

constexpr int COL_TOK = 128;   // tokens per column chunk; one warp walks one chunk
constexpr int COL_WARPS = 4;   // chunks per block
// tokens per warp in a shared-memory ring (all but one in flight): 12, or 8
// with four pairs per lane, whose slots are twice as large
template <int NP>
__host__ __device__ constexpr int col_ring() {
  return NP >= 4 ? 8 : 12;
}

// Features per warp of the walk: NP pairs per lane
__host__ __device__ constexpr int col_feat(int np_lane) { return 64 * np_lane; }
// dalpha partials per token, padded to 16 bytes for the row kernel's copies
__host__ __device__ constexpr int col_partials(int d, int np_lane) {
  return ((d / col_feat(np_lane)) + 3) & ~3;
}

// A lane's features: NP pairs of adjacent ones.
template <int NP>
struct FPairs {
  float2 p[NP];
};

template <int NP>
__device__ __forceinline__ FPairs<NP> ld_pairs(const float* q) {
  FPairs<NP> r;
  if constexpr (NP >= 2) {
#pragma unroll
    for (int h = 0; h < NP / 2; ++h) {
      const float4 t = *reinterpret_cast<const float4*>(q + 4 * h);
      r.p[2 * h] = make_float2(t.x, t.y);
      r.p[2 * h + 1] = make_float2(t.z, t.w);
    }
  } else {
    r.p[0] = *reinterpret_cast<const float2*>(q);
  }
  return r;
}

// Asynchronous copy of a lane's features (8 NP bytes), global -> its own
// shared-memory slot.
template <int NP>
__device__ __forceinline__ void cp_async_pairs(void* dst, const void* src) {
  if constexpr (NP >= 2) {
#pragma unroll
    for (int h = 0; h < NP / 2; ++h)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                       (uint32_t)__cvta_generic_to_shared(dst) + 16u * h),
                   "l"(static_cast<const float*>(src) + 4 * h)
                   : "memory");
  } else {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(
                     (uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
  }
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N_PENDING>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N_PENDING) : "memory");
}

// The warp's dalpha partials, 32 emitted tokens at a time: lane L's share of
// the warp's e-th emitted token sits at [e % 32][L] (rows padded to 33 so
// that both the writes and the row sums below are free of bank conflicts).
struct ColPartials {
  float p[32][33];
};

// Sum rows 0 .. cnt-1 of the buffer across the 32 lanes, lane r adding row r
// in lane order, and store row r as token jbase + r * stride; warp-uniform.
__device__ __forceinline__ void col_flush(ColPartials& pb, int jbase, int stride, int cnt, int np,
                                          float* __restrict__ pab) {
  __syncwarp();
  const int lane = threadIdx.x & 31;
  if (lane < cnt) {
    float sum = 0.f;
#pragma unroll 8
    for (int c = 0; c < 32; ++c) sum += pb.p[lane][c];
    pab[(jbase + lane * stride) * np] = sum;
  }
  __syncwarp();
}

// Emit the warp's e-th token, token j = r + e S of its chunk (a walk emits
// the tokens r, r + S, r + 2 S, ... of its chunk, each once and in order):
// dv = alpha dvt (the lane's features, bf16), and the lane's share of
// dalpha = <dvt, v>; every 32nd token flushes the warp's partials.
template <int NP>
__device__ __forceinline__ void col_emit(const FPairs<NP>& r, const FPairs<NP>& vv, float a,
                                         int j, int e, int S, int ld, int np,
                                         __nv_bfloat16* __restrict__ dvb, ColPartials& pb,
                                         float* __restrict__ pab) {
  __nv_bfloat162 o[NP];
  float dot = 0.f;
#pragma unroll
  for (int q = 0; q < NP; ++q) {
    const float2 dvr = __fmul2_rn(make_float2(a, a), r.p[q]);
    o[q] = __floats2bfloat162_rn(dvr.x, dvr.y);
    dot = fmaf(r.p[q].x, vv.p[q].x, fmaf(r.p[q].y, vv.p[q].y, dot));
  }
  if constexpr (NP == 4) {
    uint4 w;
    w.x = *reinterpret_cast<const uint32_t*>(&o[0]);
    w.y = *reinterpret_cast<const uint32_t*>(&o[1 % NP]);
    w.z = *reinterpret_cast<const uint32_t*>(&o[2 % NP]);
    w.w = *reinterpret_cast<const uint32_t*>(&o[3 % NP]);
    *reinterpret_cast<uint4*>(dvb + j * ld) = w;
  } else if constexpr (NP == 2) {
    uint2 w;
    w.x = *reinterpret_cast<const uint32_t*>(&o[0]);
    w.y = *reinterpret_cast<const uint32_t*>(&o[NP - 1]);
    *reinterpret_cast<uint2*>(dvb + j * ld) = w;
  } else {
    *reinterpret_cast<__nv_bfloat162*>(dvb + j * ld) = o[0];
  }
  pb.p[e & 31][threadIdx.x & 31] = dot;
  if ((e & 31) == 31) col_flush(pb, j - 31 * S, S, 32, np, pab);
}

// With the pre-conv norm the walk's result for token j is dc (the conv
// input's gradient, fp32, the lane's features at dcb + j d) instead of dv:
// the lane's share of <g_v dc, vt> (vt = alpha v) goes to the partials, which
// the pre-norm row kernel adds up for the norm's backward, and dc rc vt
// (= dc q v, q = alpha rc) is added to gacc for g_v's gradient.
template <int NP>
__device__ __forceinline__ void col_emit_pre(const FPairs<NP>& r, const FPairs<NP>& vv, float a,
                                             float qa, const FPairs<NP>& gv, FPairs<NP>& gacc,
                                             int j, int e, int S, int d, int np,
                                             float* __restrict__ dcb, ColPartials& pb,
                                             float* __restrict__ pab) {
  float dot = 0.f;
#pragma unroll
  for (int q = 0; q < NP; ++q) {
    const float2 gr = __fmul2_rn(gv.p[q], r.p[q]);
    dot = fmaf(gr.x, a * vv.p[q].x, fmaf(gr.y, a * vv.p[q].y, dot));
    gacc.p[q] = __ffma2_rn(r.p[q], __fmul2_rn(make_float2(qa, qa), vv.p[q]), gacc.p[q]);
  }
  if constexpr (NP >= 2) {
#pragma unroll
    for (int h = 0; h < NP / 2; ++h)
      *reinterpret_cast<float4*>(dcb + (int64_t)j * d + 4 * h) =
          make_float4(r.p[2 * h].x, r.p[2 * h].y, r.p[2 * h + 1].x, r.p[2 * h + 1].y);
  } else {
    *reinterpret_cast<float2*>(dcb + (int64_t)j * d) = r.p[0];
  }
  pb.p[e & 31][threadIdx.x & 31] = dot;
  if ((e & 31) == 31) col_flush(pb, j - 31 * S, S, 32, np, pab);
}

// The pre-conv norm's inputs and outputs of the walk (unused without it):
// rc[t] = (alpha_t^2 <v_t, v_t> / d + eps)^(-1/2), g_v (NULL: ones), dc
// [N, d] fp32 and the walks' partial sums of dc rc vt, gvpart [units, d].
struct ColPre {
  const float* rc;
  const float* gv;
  float* dc;
  float* gvpart;
};

// dynamic shared memory of the column walk: per warp the copy ring, the
// dalpha partials and the chunk's gates (with DIL * 3 tokens on each side),
// and with the pre-conv norm the tokens' alpha rc likewise
template <int DIL, int NP, bool PRE>
constexpr int col_smem_bytes() {
  return COL_WARPS * (col_ring<NP>() * 2 * 32 * (int)sizeof(FPairs<NP>) + (int)sizeof(ColPartials) +
                      (PRE ? 2 : 1) * (COL_TOK + 6 * DIL) * 4);
}

// One warp per (chunk of COL_TOK tokens, chain, 64 NP features), each lane
// holding NP pairs of adjacent features.  The conv reads
// y_t = sum_i w_i vt_{t-(3-i) DIL}, so the tokens of a chunk fall into DIL
// chains (token index mod DIL, S = DIL apart), each an independent conv of
// dilation 1 along the chain; a warp walks one chain in token order.  The
// warp keeps, for the chain's three previous tokens, vt and v, and the
// partial sums of their dvt:
// dvt_s = u_s + w_3 dy_s + w_2 dy_{s+S} + w_1 dy_{s+2 S} + w_0 dy_{s+3 S}
// (terms past the sequence end absent), to which each new dy_t adds its
// share.  At token t it forms y_t and dy_t; dvt of token t-3S is then
// complete, and at a sequence end so are the chain's later ones.  The walk
// runs three chain steps past the chunk for the last tokens' dy.  v and dout
// of the next col_ring - 1 chain tokens are in flight into a per-warp
// shared-memory ring (asynchronous copies, each lane its own bytes).  `live`
// counts the history's tokens that belong to t's sequence and to this
// walk (tokens before the chunk are emitted by the previous chunk's walks).
// For each completed token it writes dv (bf16, for the GEMMs) and the warp's
// partial of dalpha, dalpha_part[token][f / (64 NP)] (the lanes' shares
// summed per 32 tokens, from shared memory, in lane order); at the end the
// walk's partial conv-weight gradient, part[unit][f] = sum over its chain's
// tokens in the chunk of dy_t * (vt_{t-3 S}, vt_{t-2 S}, vt_{t-S}, vt_t).
// The arithmetic runs on packed fp32 pairs.  Warps are independent (all
// lanes of one walk the same tokens, so the branches are uniform); the block
// only groups COL_WARPS walks for scheduling.
// With the pre-conv norm (PRE) the conv reads c = alpha rc g_v v instead of
// vt, the running sums are those of dc (dvt without u and without the norm's
// backward, which needs whole rows and is left to the pre-norm row kernel),
// and each completed token's dc goes out as col_emit_pre describes; part then
// holds the sums of dy_t * (c_{t-3 S}, ..., c_t).
template <int DIL, int NP, bool PRE>
__global__ void __launch_bounds__(32 * COL_WARPS) bw_col_kernel(
    const float* __restrict__ v, const float* __restrict__ alpha,
    const float4* __restrict__ conv_w, const float* __restrict__ dout, int64_t N, int T, int d,
    int ld, int units, __nv_bfloat16* __restrict__ dv, float* __restrict__ dalpha_part,
    float4* __restrict__ part, ColPre pre) {
  // v and dv rows are ld apart (they share rows with k and dk), dout rows d
  using FP = FPairs<NP>;
  constexpr int S = DIL;       // token stride of a chain
  constexpr int HT = 3 * DIL;  // tokens of conv history
  extern __shared__ __align__(16) unsigned char col_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int COL_RING = col_ring<NP>();
  constexpr int RING_BYTES = COL_RING * 2 * 32 * (int)sizeof(FP);
  auto* ring_all = reinterpret_cast<FP(*)[COL_RING][2][32]>(col_smem);  // [slot][v, dout][lane]
  auto* pb_all = reinterpret_cast<ColPartials*>(col_smem + COL_WARPS * RING_BYTES);
  auto* al_all = reinterpret_cast<float(*)[COL_TOK + 2 * HT]>(col_smem + COL_WARPS * RING_BYTES +
                                                               COL_WARPS * sizeof(ColPartials));
  ColPartials& pb = pb_all[warp];
  // PRE: q_s[i] = alpha rc of the token al_s[i] belongs to
  float* q_s = PRE ? al_all[COL_WARPS + warp] : nullptr;
  const int unit = blockIdx.x * COL_WARPS + warp;
  if (unit >= units) return;  // no block-wide barrier follows
  const int chunk = unit / S, r0 = unit - chunk * S;  // the chain: tokens r0, r0 + S, ...
  const int f = blockIdx.y * col_feat(NP) + lane * 2 * NP;
  const int np = col_partials(d, NP);
  const int64_t t0 = (int64_t)chunk * COL_TOK;
  const int64_t t1 = t0 + COL_TOK < N ? t0 + COL_TOK : N;
  const int64_t t_stop = t1 + HT < N ? t1 + HT : N;
  // the gates of the chunk's tokens and the HT on each side: al_s[tt - t0 + HT]
  float* al_s = al_all[warp];
  for (int i = lane; i < COL_TOK + 2 * HT; i += 32) {
    const int64_t tt = t0 - HT + i;
    al_s[i] = (tt >= 0 && tt < t_stop) ? alpha[tt] : 0.f;
    if constexpr (PRE) q_s[i] = (tt >= 0 && tt < t_stop) ? alpha[tt] * pre.rc[tt] : 0.f;
  }
  __syncwarp();
  // PRE: g_v of the lane's features, and its gradient's running sum
  FPairs<NP> Gv, Gacc;
#pragma unroll
  for (int q = 0; q < NP; ++q) {
    Gv.p[q] = make_float2(1.f, 1.f);
    Gacc.p[q] = make_float2(0.f, 0.f);
  }
  if (PRE && pre.gv != nullptr) Gv = ld_pairs<NP>(pre.gv + f);
  // the weights as (feature x, feature y) pairs: W0 multiplies vt_{t-3S}, W3 vt_t
  FP W0, W1, W2, W3;
#pragma unroll
  for (int q = 0; q < NP; ++q) {
    const float4 wx = __ldg(conv_w + f + 2 * q), wy = __ldg(conv_w + f + 2 * q + 1);
    W0.p[q] = make_float2(wx.x, wy.x);
    W1.p[q] = make_float2(wx.y, wy.y);
    W2.p[q] = make_float2(wx.z, wy.z);
    W3.p[q] = make_float2(wx.w, wy.w);
  }
  const FP zero = {};
  // chain steps: step i is token r0 + S i of the chunk
  const int span = (int)(t1 - t0), wspan = (int)(t_stop - t0);
  const int n_chunk = span > r0 ? (span - r0 + S - 1) / S : 0;
  const int n_walk = wspan > r0 ? (wspan - r0 + S - 1) / S : 0;
  int pos = (int)((t0 + r0) % T);
  // rings over the three previous chain tokens: index k holds token t-(k+1)S
  FP sr[3], ar[3], vr_[3];  // vt, partial dvt, v
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    sr[k] = ar[k] = vr_[k] = zero;
    if (pos >= S * (k + 1)) {  // the token lies in this sequence
      const int jk = r0 - S * (k + 1);
      FP q = ld_pairs<NP>(v + (t0 + jk) * ld + f);
      const float a = PRE ? q_s[jk + HT] : al_s[jk + HT];
#pragma unroll
      for (int j = 0; j < NP; ++j) {
        q.p[j] = __fmul2_rn(make_float2(a, a), q.p[j]);
        if constexpr (PRE) q.p[j] = __fmul2_rn(Gv.p[j], q.p[j]);
      }
      sr[k] = q;
    }
  }
  FP C0 = zero, C1 = zero, C2 = zero, C3 = zero;  // conv-weight partials for w_0 .. w_3
  int live = 0;
  __nv_bfloat16* dvb = dv + t0 * ld + f;
  float* dcb = PRE ? pre.dc + t0 * d + f : nullptr;
  float* pab = dalpha_part + t0 * np + blockIdx.y;
  // emit the chain's e-th token
  auto emit = [&](const FP& rr, const FP& vv, int e) {
    const int j = r0 + S * e;
    if constexpr (PRE)
      col_emit_pre<NP>(rr, vv, al_s[j + HT], q_s[j + HT], Gv, Gacc, j, e, S, d, np, dcb, pb, pab);
    else
      col_emit<NP>(rr, vv, al_s[j + HT], j, e, S, ld, np, dvb, pb, pab);
  };
  // step q's v and dout go to ring slot q % COL_RING; the slot refilled at
  // step i held step i - 1, whose values step i - 1 has already used
  FP (*ring)[2][32] = ring_all[warp];
  const float* vp = v + (t0 + r0) * ld + f;
  const float* up = dout + (t0 + r0) * d + f;
#pragma unroll
  for (int q = 0; q < COL_RING - 1; ++q) {
    if (q < n_walk) {
      cp_async_pairs<NP>(&ring[q][0][lane], vp);
      cp_async_pairs<NP>(&ring[q][1][lane], up);
    }
    cp_async_commit();
    vp += S * ld;
    up += S * d;
  }
#pragma unroll 4
  for (int i = 0; i < n_walk; ++i) {
    cp_async_wait<COL_RING - 2>();  // step i's copies have landed
    const int slot = i % COL_RING;
    const FP vr = ring[slot][0][lane], ut = ring[slot][1][lane];
    const int ia = r0 + S * i + HT;  // the token's gate at al_s[ia]
    const float at = al_s[ia];
    if (i + COL_RING - 1 < n_walk) {
      const int refill = (i + COL_RING - 1) % COL_RING;
      cp_async_pairs<NP>(&ring[refill][0][lane], vp);
      cp_async_pairs<NP>(&ring[refill][1][lane], up);
    }
    cp_async_commit();
    vp += S * ld;
    up += S * d;
    if (pos < S) {  // the chain's previous token lies in an earlier sequence
#pragma unroll
      for (int k = 0; k < 3; ++k) sr[k] = zero;
      live = 0;
    }
    FP vt, g, E, A0;  // vt: the conv's input at t (c with PRE)
    const float ct = PRE ? q_s[ia] : at;
#pragma unroll
    for (int q = 0; q < NP; ++q) {
      vt.p[q] = __fmul2_rn(make_float2(ct, ct), vr.p[q]);
      if constexpr (PRE) vt.p[q] = __fmul2_rn(Gv.p[q], vt.p[q]);
      const float2 y = __ffma2_rn(
          W0.p[q], sr[2].p[q],
          __ffma2_rn(W1.p[q], sr[1].p[q], __ffma2_rn(W2.p[q], sr[0].p[q], __fmul2_rn(W3.p[q], vt.p[q]))));
      g.p[q] = __fmul2_rn(ut.p[q], silu_grad2(y));
      E.p[q] = __ffma2_rn(W0.p[q], g.p[q], ar[2].p[q]);  // dvt of t-3S, complete
      ar[1].p[q] = __ffma2_rn(W1.p[q], g.p[q], ar[1].p[q]);
      ar[0].p[q] = __ffma2_rn(W2.p[q], g.p[q], ar[0].p[q]);
      A0.p[q] = PRE ? __fmul2_rn(W3.p[q], g.p[q]) : __ffma2_rn(W3.p[q], g.p[q], ut.p[q]);
    }
    if (i < n_chunk) {
#pragma unroll
      for (int q = 0; q < NP; ++q) {
        C0.p[q] = __ffma2_rn(g.p[q], sr[2].p[q], C0.p[q]);
        C1.p[q] = __ffma2_rn(g.p[q], sr[1].p[q], C1.p[q]);
        C2.p[q] = __ffma2_rn(g.p[q], sr[0].p[q], C2.p[q]);
        C3.p[q] = __ffma2_rn(g.p[q], vt.p[q], C3.p[q]);
      }
    }
    if (live == 3) emit(E, vr_[2], i - 3);
    if (pos + S >= T) {  // the chain's sequence ends at t: its later tokens are complete
#pragma unroll
      for (int k = 2; k >= 1; --k)  // steps i-k, oldest first
        if (live >= k && i - k < n_chunk) emit(ar[k - 1], vr_[k - 1], i - k);
      if (i < n_chunk) emit(A0, vr, i);
    }
#pragma unroll
    for (int k = 2; k > 0; --k) {
      ar[k] = ar[k - 1];
      sr[k] = sr[k - 1];
      vr_[k] = vr_[k - 1];
    }
    ar[0] = A0;
    sr[0] = vt;
    vr_[0] = vr;
    live = live < 3 ? live + 1 : 3;
    pos += S;
    while (pos >= T) pos -= T;  // at most S / T + 1 times
  }
  if (n_chunk & 31) col_flush(pb, r0 + S * (n_chunk & ~31), S, n_chunk & 31, np, pab);
#pragma unroll
  for (int q = 0; q < NP; ++q) {
    part[(int64_t)unit * d + f + 2 * q] =
        make_float4(C0.p[q].x, C1.p[q].x, C2.p[q].x, C3.p[q].x);
    part[(int64_t)unit * d + f + 2 * q + 1] =
        make_float4(C0.p[q].y, C1.p[q].y, C2.p[q].y, C3.p[q].y);
  }
  if constexpr (PRE) {
#pragma unroll
    for (int q = 0; q < NP; ++q)
      *reinterpret_cast<float2*>(pre.gvpart + (int64_t)unit * d + f + 2 * q) = Gacc.p[q];
  }
}

constexpr int ROW_THREADS = 256;
constexpr int ROW_VEC = 4;        // features per load
constexpr int ROW_MAX_ITEMS = 4;  // d <= ROW_THREADS * ROW_VEC * ROW_MAX_ITEMS = 4,096
constexpr float BW_RMS_EPS = 1e-6f;  // the forward's RMSNorm epsilon

__device__ __forceinline__ float4 bf16x4_to_f4(uint2 u) {
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}

constexpr int ROW_STAGES = 2;
constexpr uint64_t ROW_WAIT_NS = 2000000000ull;  // 2 s: a copy that has not landed by then never will

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// Bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned)
// from global to this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

constexpr uint64_t ROW_TEST_WAIT_NS = 1000000ull;  // 1 ms, with ENGRAM_TEST_STALL

// Wait for the phase of `bar` with the given parity; false after limit_ns.
__device__ __forceinline__ bool row_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  uint64_t t0 = 0;
  for (int spin = 0;; ++spin) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(20000u)
        : "memory");
    if (ok) return true;
    uint64_t now;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
    if (spin == 0) t0 = now;
    else if (now - t0 > limit_ns) return false;
  }
}

// Shared memory of one stage of the row kernel: the token's h (bf16), k and
// dout (fp32) rows and its np_pad dalpha partials (a multiple of 4); all
// offsets are multiples of 16 bytes because d is a multiple of 256.
__host__ __device__ constexpr size_t row_stage_bytes(int d, int np_pad) {
  return (size_t)d * 2 + (size_t)d * 4 + (size_t)d * 4 + (size_t)np_pad * 4;
}

// The gate and both RMSNorm backwards need whole-row sums, so each token is
// one step of one block: a persistent block walks tokens blockIdx.x,
// + gridDim.x, ..., with the next token's rows already in flight into the
// other shared-memory stage (bulk copies issued by one thread, completing on
// an mbarrier).  Each thread takes 4 features per item from shared memory
// into registers; <h,h>, <k,k>, <h,k> and dalpha (the column walk's np
// partials per token, rows np_pad apart, added by the first warp) are reduced together in one
// fixed-order pass, whose barrier also frees the stage for the token after
// next; then dk (bf16, for the GEMMs) and dh are written.  A copy that never
// lands sets ENGRAM_STATUS_TIMEOUT and the block stops.
// With learnable norm scales (SCALED) the gate reads <RMSNorm(h) g_h,
// RMSNorm(k) g_k>: h k is weighted by gg = g_h g_k in the sums and in dk, dh,
// and each thread adds up, over the block's tokens, c (r_h h)(r_k k) for its
// features (c = dz / sqrt(d)); the block's sums go to spart[block][f] for
// the scales' gradients (dg_h = S g_k, dg_k = S g_h).
template <int ITEMS, bool SCALED>  // ITEMS = ceil(d / (ROW_THREADS * ROW_VEC)) <= ROW_MAX_ITEMS
__global__ void __launch_bounds__(ROW_THREADS) bw_row_kernel(
    const __nv_bfloat16* __restrict__ h, const float* __restrict__ k,
    const float* __restrict__ alpha, const float* __restrict__ dout,
    const float* __restrict__ dalpha_part, int np, int np_pad, const float* __restrict__ gscale,
    int64_t N, int d, int ld, float* __restrict__ dh, __nv_bfloat16* __restrict__ dk_out,
    float* __restrict__ spart, unsigned int* status, uint64_t wait_ns, int stall) {
  // k and dk rows are ld apart (they share rows with v and dv)
  extern __shared__ __align__(128) unsigned char row_smem[];
  __shared__ uint64_t full[ROW_STAGES];
  __shared__ float4 red[2][ROW_THREADS / 32];
  __shared__ int abort_flag;
  const size_t SB = row_stage_bytes(d, np_pad);
  const uint32_t hb_bytes = (uint32_t)d * 2, f_bytes = (uint32_t)d * 4,
                 p_bytes = (uint32_t)np_pad * 4;
  const int64_t G = gridDim.x;
  unsigned pend = 0;  // thread 0: stages with a copy issued and not yet seen landed
  auto issue = [&](int64_t t, int st) {  // thread 0
    pend |= 1u << st;
    unsigned char* base = row_smem + st * SB;
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(&full[st])),
                 "r"(hb_bytes + 2 * f_bytes + p_bytes)
                 : "memory");
    if (stall) return;  // ENGRAM_TEST_STALL: the stage is armed, its copies never issued
    bulk_load(base, h + t * d, hb_bytes, &full[st]);
    bulk_load(base + hb_bytes, k + t * ld, f_bytes, &full[st]);
    bulk_load(base + hb_bytes + f_bytes, dout + t * d, f_bytes, &full[st]);
    bulk_load(base + hb_bytes + 2 * f_bytes, dalpha_part + t * np_pad, p_bytes, &full[st]);
  };
  if (threadIdx.x == 0) {
    for (int st = 0; st < ROW_STAGES; ++st)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(&full[st])));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    abort_flag = 0;
    for (int st = 0; st < ROW_STAGES; ++st)
      if (blockIdx.x + st * G < N) issue(blockIdx.x + st * G, st);
  }
  __syncthreads();
  const int nv = d / ROW_VEC;
  const float invd = 1.0f / (float)d, isd = rsqrtf((float)d);
  // SCALED: g_h g_k of the thread's features, and its running sums
  float4 ggv[SCALED ? ITEMS : 1], sacc[SCALED ? ITEMS : 1];
  if constexpr (SCALED) {
#pragma unroll
    for (int q = 0; q < ITEMS; ++q) {
      const int c4 = threadIdx.x + q * ROW_THREADS;
      ggv[q] = sacc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c4 < nv) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(gscale) + c4);
        const float4 b = __ldg(reinterpret_cast<const float4*>(gscale + d) + c4);
        ggv[q] = make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w);
      }
    }
  }
  int it = 0;
  for (int64_t t = blockIdx.x; t < N; t += G, ++it) {
    const int st = it % ROW_STAGES;
    const unsigned char* base = row_smem + st * SB;
    if (row_wait(&full[st], (uint32_t)(it / ROW_STAGES) & 1u, wait_ns)) {
      pend &= ~(1u << st);
    } else {
      abort_flag = 1;  // every thread reaches the barrier below, then all stop
      atomicOr(status, ENGRAM_STATUS_TIMEOUT);
    }
    const __nv_bfloat16* hs = reinterpret_cast<const __nv_bfloat16*>(base);
    const float* ks = reinterpret_cast<const float*>(base + hb_bytes);
    const float* us = reinterpret_cast<const float*>(base + hb_bytes + f_bytes);
    const float* ps = reinterpret_cast<const float*>(base + hb_bytes + 2 * f_bytes);
    uint2 hb[ITEMS];  // h kept as bf16 (4 per item) until used
    float4 kv[ITEMS], uv[ITEMS];
    float shh = 0.f, skk = 0.f, shk = 0.f;
#pragma unroll
    for (int q = 0; q < ITEMS; ++q) {
      const int c = threadIdx.x + q * ROW_THREADS;
      hb[q] = make_uint2(0u, 0u);
      kv[q] = uv[q] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c < nv) {
        hb[q] = *reinterpret_cast<const uint2*>(hs + c * ROW_VEC);
        kv[q] = *reinterpret_cast<const float4*>(ks + c * ROW_VEC);
        uv[q] = *reinterpret_cast<const float4*>(us + c * ROW_VEC);
      }
      const float4 hq = bf16x4_to_f4(hb[q]), kq = kv[q];
      shh = fmaf(hq.x, hq.x, fmaf(hq.y, hq.y, fmaf(hq.z, hq.z, fmaf(hq.w, hq.w, shh))));
      skk = fmaf(kq.x, kq.x, fmaf(kq.y, kq.y, fmaf(kq.z, kq.z, fmaf(kq.w, kq.w, skk))));
      if constexpr (SCALED) {
        const float4 g = ggv[q];
        shk = fmaf(hq.x * g.x, kq.x,
                   fmaf(hq.y * g.y, kq.y, fmaf(hq.z * g.z, kq.z, fmaf(hq.w * g.w, kq.w, shk))));
      } else {
        shk = fmaf(hq.x, kq.x, fmaf(hq.y, kq.y, fmaf(hq.z, kq.z, fmaf(hq.w, kq.w, shk))));
      }
    }
    float sgv = 0.f;
    if (threadIdx.x < 32)
      for (int i = threadIdx.x; i < np; i += 32) sgv += ps[i];
    float4 r = make_float4(shh, skk, shk, sgv);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      r.x += __shfl_xor_sync(0xffffffffu, r.x, o);
      r.y += __shfl_xor_sync(0xffffffffu, r.y, o);
      r.z += __shfl_xor_sync(0xffffffffu, r.z, o);
      r.w += __shfl_xor_sync(0xffffffffu, r.w, o);
    }
    float4* rb = red[it & 1];  // two buffers: a fast thread's next write never meets a slow read
    if ((threadIdx.x & 31) == 0) rb[threadIdx.x >> 5] = r;
    __syncthreads();  // all reads of this stage are done: it can be refilled
    if (abort_flag) break;
    if (threadIdx.x == 0 && t + ROW_STAGES * G < N) issue(t + ROW_STAGES * G, st);
    r = rb[0];
#pragma unroll
    for (int i = 1; i < ROW_THREADS / 32; ++i) {
      r.x += rb[i].x;
      r.y += rb[i].y;
      r.z += rb[i].z;
      r.w += rb[i].w;
    }
    const float rh = rsqrtf(r.x * invd + BW_RMS_EPS), rk = rsqrtf(r.y * invd + BW_RMS_EPS);
    const float shk_all = r.z;
    const float a = __ldg(alpha + t);
    const float c = r.w * a * (1.0f - a) * isd;  // dz / sqrt(d): dh^ = c k^, dk^ = c h^
    const float ch = rh * rh * rh * (c * rk * shk_all) * invd;  // r_h^3 <dh^, h> / d
    const float ck = rk * rk * rk * (c * rh * shk_all) * invd;  // r_k^3 <dk^, k> / d
    const float crh = c * rh, crk = c * rk;
    __nv_bfloat16* dkr = dk_out + t * ld;
    float* dhr = dh + t * d;
#pragma unroll
    for (int q = 0; q < ITEMS; ++q) {
      const int c4 = threadIdx.x + q * ROW_THREADS;
      if (c4 < nv) {
        const float4 hq = bf16x4_to_f4(hb[q]), kq0 = kv[q], uq = uv[q];
        float4 hg = hq, kg = kq0;  // h, k weighted by g_h g_k where they cross
        if constexpr (SCALED) {
          const float4 g = ggv[q];
          hg = make_float4(hq.x * g.x, hq.y * g.y, hq.z * g.z, hq.w * g.w);
          kg = make_float4(kq0.x * g.x, kq0.y * g.y, kq0.z * g.z, kq0.w * g.w);
          const float cr = c * rh * rk;
          sacc[q].x = fmaf(cr * hq.x, kq0.x, sacc[q].x);
          sacc[q].y = fmaf(cr * hq.y, kq0.y, sacc[q].y);
          sacc[q].z = fmaf(cr * hq.z, kq0.z, sacc[q].z);
          sacc[q].w = fmaf(cr * hq.w, kq0.w, sacc[q].w);
        }
        const float4 kq = kq0;
        const __nv_bfloat162 k01 = __floats2bfloat162_rn(rk * (crh * hg.x) - ck * kq.x,
                                                        rk * (crh * hg.y) - ck * kq.y);
        const __nv_bfloat162 k23 = __floats2bfloat162_rn(rk * (crh * hg.z) - ck * kq.z,
                                                        rk * (crh * hg.w) - ck * kq.w);
        uint2 pk;
        pk.x = *reinterpret_cast<const uint32_t*>(&k01);
        pk.y = *reinterpret_cast<const uint32_t*>(&k23);
        *reinterpret_cast<uint2*>(dkr + c4 * ROW_VEC) = pk;
        float4 o;
        o.x = uq.x + rh * (crk * kg.x) - ch * hq.x;
        o.y = uq.y + rh * (crk * kg.y) - ch * hq.y;
        o.z = uq.z + rh * (crk * kg.z) - ch * hq.z;
        o.w = uq.w + rh * (crk * kg.w) - ch * hq.w;
        __stcs(reinterpret_cast<float4*>(dhr + c4 * ROW_VEC), o);
      }
    }
  }
  if constexpr (SCALED) {
#pragma unroll
    for (int q = 0; q < ITEMS; ++q) {
      const int c4 = threadIdx.x + q * ROW_THREADS;
      if (c4 < nv) reinterpret_cast<float4*>(spart + (int64_t)blockIdx.x * d)[c4] = sacc[q];
    }
  }
  // on a timeout, let copies still in flight land (bounded) before the
  // block's shared memory is released; a stage holds at most one, of the
  // phase after the last one waited for
  if (threadIdx.x == 0 && pend != 0) {
    const int done = it;  // uses waited for: stage s had uses j < done with j % ROW_STAGES == s
    for (int st = 0; st < ROW_STAGES; ++st) {
      if (!(pend & (1u << st))) continue;
      const int use = done / ROW_STAGES + (st < done % ROW_STAGES ? 1 : 0);
      row_wait(&full[st], (uint32_t)use & 1u, wait_ns);
    }
  }
}

// dg_h[f] = S[f] g_k[f], dg_k[f] = S[f] g_h[f], S[f] = the row blocks' sums
// added in block order
__global__ void bw_scale_reduce_kernel(const float* __restrict__ spart, int blocks, int d,
                                       const float* __restrict__ gscale,
                                       float* __restrict__ dgscale) {
  const int f = blockIdx.x * blockDim.x + threadIdx.x;
  if (f >= d) return;
  float S = 0.f;
#pragma unroll 8
  for (int b = 0; b < blocks; ++b) S += spart[(int64_t)b * d + f];
  dgscale[f] = S * gscale[d + f];      // d/dg_h
  dgscale[d + f] = S * gscale[f];      // d/dg_k
}

// The pre-conv norm's backward, one token per block step (persistent blocks,
// 256 threads): S = <g_v dc, vt> from the column walk's partials (added in
// order by the first warp), then per feature
//   dvt = u + rc g_v dc - rc^3 vt S / d   (vt = alpha v; RMSNorm backward)
// dv = alpha dvt (bf16, for the GEMMs) and dalpha = <dvt, v> (a fixed-order
// block reduction), written as the one dalpha partial of the token's row of
// da (rows 4 floats apart) for the gate's row kernel.
constexpr int PN_ROW_THREADS = 256;
__global__ void __launch_bounds__(PN_ROW_THREADS) bw_prenorm_row_kernel(
    const float* __restrict__ dc, const float* __restrict__ v, int ld,
    const float* __restrict__ dout, const float* __restrict__ alpha,
    const float* __restrict__ rc, const float* __restrict__ gv, const float* __restrict__ ppart,
    int np, int np_pad, int64_t N, int d, __nv_bfloat16* __restrict__ dv,
    float* __restrict__ da) {
  __shared__ float Ssh;
  __shared__ float red[2][PN_ROW_THREADS / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nv = d / 4;
  const float invd = 1.0f / (float)d;
  int it = 0;
  for (int64_t t = blockIdx.x; t < N; t += gridDim.x, ++it) {
    if (warp == 0) {
      float S = 0.f;
      for (int i = lane; i < np; i += 32) S += ppart[t * np_pad + i];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);
      if (lane == 0) Ssh = S;
    }
    __syncthreads();
    const float S = Ssh;
    const float a = alpha[t], r = rc[t];
    const float cS = r * r * r * a * S * invd;  // rc^3 S / d, times alpha for vt = alpha v
    const float4* dcr = reinterpret_cast<const float4*>(dc + t * d);
    const float4* vr = reinterpret_cast<const float4*>(v + t * ld);
    const float4* ur = reinterpret_cast<const float4*>(dout + t * d);
    const float4* gr = reinterpret_cast<const float4*>(gv);
    float dot = 0.f;
    for (int c4 = threadIdx.x; c4 < nv; c4 += PN_ROW_THREADS) {
      const float4 x = dcr[c4], vv = vr[c4], u = ur[c4];
      const float4 g = gv != nullptr ? gr[c4] : make_float4(1.f, 1.f, 1.f, 1.f);
      float4 o;
      o.x = u.x + r * g.x * x.x - cS * vv.x;
      o.y = u.y + r * g.y * x.y - cS * vv.y;
      o.z = u.z + r * g.z * x.z - cS * vv.z;
      o.w = u.w + r * g.w * x.w - cS * vv.w;
      dot = fmaf(o.x, vv.x, fmaf(o.y, vv.y, fmaf(o.z, vv.z, fmaf(o.w, vv.w, dot))));
      const __nv_bfloat162 p01 = __floats2bfloat162_rn(a * o.x, a * o.y);
      const __nv_bfloat162 p23 = __floats2bfloat162_rn(a * o.z, a * o.w);
      uint2 pk;
      pk.x = *reinterpret_cast<const uint32_t*>(&p01);
      pk.y = *reinterpret_cast<const uint32_t*>(&p23);
      *reinterpret_cast<uint2*>(dv + t * ld + c4 * 4) = pk;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    float* rb = red[it & 1];  // two buffers: a fast warp's next write never meets a slow read
    if (lane == 0) rb[warp] = dot;
    __syncthreads();  // also: every thread has read Ssh before the next token's write
    if (threadIdx.x == 0) {
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < PN_ROW_THREADS / 32; ++w) sum += rb[w];
      *reinterpret_cast<float4*>(da + t * 4) = make_float4(sum, 0.f, 0.f, 0.f);
    }
  }
}

// dg_v[f] = sum over the walks, in order, of gvpart[unit][f]
__global__ void bw_gv_reduce_kernel(const float* __restrict__ gvpart, int units, int d,
                                    float* __restrict__ dgv) {
  const int f = blockIdx.x * blockDim.x + threadIdx.x;
  if (f >= d) return;
  float S = 0.f;
#pragma unroll 8
  for (int c = 0; c < units; ++c) S += gvpart[(int64_t)c * d + f];
  dgv[f] = S;
}

constexpr int DCONV_WARPS = 32;

// dconv_w[f] = sum over the walks of part[unit][f]: warp w adds units w,
// w + 32, ... in order (its loads all in flight at once for up to 256
// units), then the 32 warp sums are added in warp order.
__global__ void __launch_bounds__(32 * DCONV_WARPS) bw_dconv_reduce_kernel(
    const float4* __restrict__ part, int units, int d, float4* __restrict__ dw) {
  __shared__ float4 red[DCONV_WARPS][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int f = blockIdx.x * 32 + lane;
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
  if (f < d) {
#pragma unroll 8
    for (int c = warp; c < units; c += DCONV_WARPS) {
      const float4 p = part[(int64_t)c * d + f];
      s.x += p.x;
      s.y += p.y;
      s.z += p.z;
      s.w += p.w;
    }
  }
  red[warp][lane] = s;
  __syncthreads();
  if (warp == 0 && f < d) {
    float4 o = red[0][lane];
#pragma unroll
    for (int w = 1; w < DCONV_WARPS; ++w) {
      o.x += red[w][lane].x;
      o.y += red[w][lane].y;
      o.z += red[w][lane].z;
      o.w += red[w][lane].w;
    }
    dw[f] = o;
  }
}

// Workspace: [k | v] fp32 [N, 2d]; [dk | dv] bf16 [N, 2d]; dalpha partials
// [N, up to d/64 padded to 4]; de fp32 [N, E] when the caller passes none;
// conv partials; the weight-gradient GEMM's tile counters; the table
// gradient's sort buffers.
struct BwdBf16Ws {
  // k and v stay fp32: dh and dalpha are sums whose terms can cancel, so a
  // bf16 rounding of k or v would show at full size in a small result.
  // They share rows (kv [N, 2d] = [k | v]), as do dk and dv, and W_k, W_v
  // are read as one stacked operand, so that each pair of GEMMs is one.
  float* kv;  // recomputed here, or NULL when the forward saved them
  __nv_bfloat16* dkv;
  float *dalpha_part, *de;  // partials of <dvt, v>, padded rows
  float4* part;
  float* spart;  // with norm scales: [kMaxRowBlocks][d] sums of the row blocks
  // with the pre-conv norm: rc [N], dc [N, d], dalpha rows [N, 4], the
  // chunks' g_v sums [chunks, d]
  float *rc, *dc, *da, *gvpart;
  void* gemm_ws;
  void* tg_ws;
  size_t tg_bytes;
};

constexpr size_t up256b(size_t b) { return (b + 255) & ~(size_t)255; }

constexpr int kMaxRowBlocks = 1024;  // row-kernel blocks when the scales' sums are kept

size_t bwd_bf16_layout(void* base, int64_t N, int d, int E, int J, bool kv_saved, bool scaled,
                       bool prenorm, BwdBf16Ws* w) {
  const int64_t chunks = (N + COL_TOK - 1) / COL_TOK;
  const size_t KV = kv_saved ? 0 : up256b((size_t)N * 2 * d * 4);
  const size_t DKV = up256b((size_t)N * 2 * d * 2);
  const size_t DA = up256b((size_t)N * col_partials(d, 1) * 4);  // the most partials
  // conv partials of up to three walks (chains) per chunk
  const size_t NE4 = up256b((size_t)N * E * 4), P = up256b((size_t)chunks * 3 * d * 16);
  const size_t tg = table_grad_ws_bytes(N * J);
  const size_t SP = scaled ? up256b((size_t)kMaxRowBlocks * d * 4) : 0;
  const size_t RC = prenorm ? up256b((size_t)N * 4) : 0;
  const size_t DC = prenorm ? up256b((size_t)N * d * 4) : 0;
  const size_t DA1 = prenorm ? up256b((size_t)N * 16) : 0;
  const size_t GVP = prenorm ? up256b((size_t)chunks * 3 * d * 4) : 0;
  const size_t GF = gemm_dw_ws_bytes(d, E);
  size_t off[12];
  const size_t sz[12] = {KV, DKV, DA, NE4, P, GF, tg, SP, RC, DC, DA1, GVP};
  size_t o = 0;
  for (int i = 0; i < 12; ++i) {
    off[i] = o;
    o += sz[i];
  }
  if (w != nullptr) {
    char* p = static_cast<char*>(base);
    w->kv = kv_saved ? nullptr : reinterpret_cast<float*>(p + off[0]);
    w->dkv = reinterpret_cast<__nv_bfloat16*>(p + off[1]);
    w->dalpha_part = reinterpret_cast<float*>(p + off[2]);
    w->de = reinterpret_cast<float*>(p + off[3]);
    w->part = reinterpret_cast<float4*>(p + off[4]);
    w->gemm_ws = p + off[5];
    w->tg_ws = p + off[6];
    w->tg_bytes = tg;
    w->spart = scaled ? reinterpret_cast<float*>(p + off[7]) : nullptr;
    w->rc = prenorm ? reinterpret_cast<float*>(p + off[8]) : nullptr;
    w->dc = prenorm ? reinterpret_cast<float*>(p + off[9]) : nullptr;
    w->da = prenorm ? reinterpret_cast<float*>(p + off[10]) : nullptr;
    w->gvpart = prenorm ? reinterpret_cast<float*>(p + off[11]) : nullptr;
  }
  return o;
}

}  // namespace

size_t backward_bf16_ws_bytes(int64_t N, int d, int E, int J, bool kv_saved, bool scaled,
                              bool prenorm) {
  return bwd_bf16_layout(nullptr, N, d, E, J, kv_saved, scaled, prenorm, nullptr);
}

int launch_backward_bf16(const HeadParams& hp, const int32_t* idx, const __nv_bfloat16* e,
                         const __nv_bfloat16* h, const __nv_bfloat16* Wk,
                         const __nv_bfloat16* Wv, const float* conv_w, const float* gscale,
                         const float* alpha, const float* kv_saved, const float* dout, float* dh,
                         float* dWk,
                         float* dWv, float* dconv_w, float* de, int64_t* dtab_keys,
                         float* dtab_rows, int32_t* n_unique, int64_t N, int T, int d, int dil,
                         bool prenorm, const float* gv, void* ws, size_t ws_bytes, bool stall,
                         cudaStream_t s) {
  const int E = hp.E;
  const bool have_kv = kv_saved != nullptr;
  const bool scaled = gscale != nullptr;
  if (ws_bytes < backward_bf16_ws_bytes(N, d, E, hp.J, have_kv, scaled, prenorm))
    return ENGRAM_ERR_WORKSPACE;
  if (!gemm_supported(N, d, E)) return ENGRAM_ERR_UNSUPPORTED;
  // a row in registers; whole column blocks; 16-byte multiples for the row copies
  if (d > ROW_THREADS * ROW_VEC * ROW_MAX_ITEMS || d % 256 != 0 || (dil != 1 && dil != 3))
    return ENGRAM_ERR_UNSUPPORTED;
  BwdBf16Ws w;
  bwd_bf16_layout(ws, N, d, E, hp.J, have_kv, scaled, prenorm, &w);
  if (de == nullptr) de = w.de;
  int rc;
  // unless the forward saved them, [k | v] = e [W_k; W_v]^T (fp32)
  if (!have_kv && (rc = launch_gemm_kv(e, Wk, Wv, N, d, E, w.kv, 2 * d, s, stall))) return rc;
  const float* kv = have_kv ? kv_saved : w.kv;
  const int chunks = (int)((N + COL_TOK - 1) / COL_TOK);
  // one walk per (chunk, chain): the dilated conv's chunks hold three chains
  const int units = chunks * dil;
  constexpr int CP = 2;  // feature pairs per lane of the walk
  const int np = d / col_feat(CP), np_pad = col_partials(d, CP);
  const ColPre pre{w.rc, gv, w.dc, w.gvpart};
  // with the pre-conv norm: rc of every token first (the walk's conv input
  // is alpha rc g_v v)
  if (prenorm && (rc = launch_prenorm_rc(kv + d, 2 * d, alpha, N, d, w.rc, s))) return rc;
  {
    auto col = dil == 1 ? (prenorm ? bw_col_kernel<1, CP, true> : bw_col_kernel<1, CP, false>)
                        : (prenorm ? bw_col_kernel<3, CP, true> : bw_col_kernel<3, CP, false>);
    const int smem = dil == 1 ? (prenorm ? col_smem_bytes<1, CP, true>() : col_smem_bytes<1, CP, false>())
                              : (prenorm ? col_smem_bytes<3, CP, true>() : col_smem_bytes<3, CP, false>());
    if ((rc = ck(cudaFuncSetAttribute(col, cudaFuncAttributeMaxDynamicSharedMemorySize, smem))))
      return rc;
    col<<<dim3((unsigned)((units + COL_WARPS - 1) / COL_WARPS), (unsigned)np), 32 * COL_WARPS,
          smem, s>>>(kv + d, alpha, reinterpret_cast<const float4*>(conv_w), dout, N, T, d, 2 * d,
                     units, w.dkv + d, w.dalpha_part, w.part, pre);
  }
  // the pre-conv norm's backward per token: dv and dalpha (one partial per row)
  const float* da_rows = w.dalpha_part;
  int da_np = np, da_np_pad = np_pad;
  if (prenorm) {
    int dev = 0, sms = 0;
    if ((rc = ck(cudaGetDevice(&dev))) ||
        (rc = ck(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev))))
      return rc;
    const int64_t grid = std::min<int64_t>(N, (int64_t)sms * 8);
    bw_prenorm_row_kernel<<<(unsigned)grid, PN_ROW_THREADS, 0, s>>>(
        w.dc, kv + d, 2 * d, dout, alpha, w.rc, gv, w.dalpha_part, np, np_pad, N, d, w.dkv + d,
        w.da);
    if (scaled)  // dg_v after dg_h, dg_k
      bw_gv_reduce_kernel<<<(unsigned)((d + 255) / 256), 256, 0, s>>>(w.gvpart, units, d,
                                                                      dconv_w + 6 * (int64_t)d);
    da_rows = w.da;
    da_np = 1;
    da_np_pad = 4;
  }
  {
    const int items = (d / ROW_VEC + ROW_THREADS - 1) / ROW_THREADS;
    auto row = scaled ? (items == 1 ? bw_row_kernel<1, true>
                         : items == 2 ? bw_row_kernel<2, true>
                         : items == 3 ? bw_row_kernel<3, true> : bw_row_kernel<4, true>)
                      : (items == 1 ? bw_row_kernel<1, false>
                         : items == 2 ? bw_row_kernel<2, false>
                         : items == 3 ? bw_row_kernel<3, false> : bw_row_kernel<4, false>);
    const int smem = (int)(ROW_STAGES * row_stage_bytes(d, da_np_pad));
    int dev = 0, sms = 0, per_sm = 0;
    if ((rc = ck(cudaFuncSetAttribute(row, cudaFuncAttributeMaxDynamicSharedMemorySize, smem))) ||
        (rc = ck(cudaGetDevice(&dev))) ||
        (rc = ck(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev))) ||
        (rc = ck(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, row, ROW_THREADS, smem))))
      return rc;
    int64_t grid = std::min<int64_t>(N, (int64_t)sms * std::max(per_sm, 1));
    if (scaled) grid = std::min<int64_t>(grid, kMaxRowBlocks);
    row<<<(unsigned)grid, ROW_THREADS, smem, s>>>(h, kv, alpha, dout, da_rows, da_np, da_np_pad,
                                                  gscale, N, d, 2 * d, dh, w.dkv, w.spart,
                                                  status_ptr(),
                                                  stall ? ROW_TEST_WAIT_NS : ROW_WAIT_NS,
                                                  stall ? 1 : 0);
    if (scaled)
      bw_scale_reduce_kernel<<<(unsigned)((d + 255) / 256), 256, 0, s>>>(
          w.spart, (int)grid, d, gscale, dconv_w + 4 * (int64_t)d);
  }
  bw_dconv_reduce_kernel<<<(unsigned)((d + 31) / 32), 32 * DCONV_WARPS, 0, s>>>(
      w.part, units, d, reinterpret_cast<float4*>(dconv_w));
  if ((rc = ck(cudaGetLastError()))) return rc;
  // [dW_k; dW_v] = [dk | dv]^T e (a contraction over tokens, rows d.. into
  // dW_v); de = [dk | dv] [W_k; W_v]
  if ((rc = launch_gemm_dw(w.dkv, e, N, d, E, dWk, dWv, w.gemm_ws, s, stall))) return rc;
  if ((rc = launch_gemm_de(w.dkv, Wk, Wv, N, d, E, de, s, stall))) return rc;
  // the table rows' gradient from de, in the deterministic order
  return launch_table_grad(hp, idx, de, N, dtab_keys, dtab_rows, n_unique, w.tg_ws, w.tg_bytes, s);
}

}  // namespace engram
