// One decode step's projections, gate, conv and residual in one persistent
// launch (bf16 layers, one token per sequence).
//
// Method: discuss.deepseek.club 二.1 (2) (h as query, e as key and value;
// the gate sigma(<RMSNorm(h), RMSNorm(W_k e)>/sqrt(d)); a 1-D causal conv;
// the residual) and 三.4 (per-token inference); sechub.in answer (short
// depthwise causal conv).
//
// The two passes of a decode step stream weight rows with little reuse, so a
// step is bound by how fast each SM takes operand bytes in.  As two launches
// (pass K, the gate kernel, pass V) every CTA pair ends pass K, exits, and
// pass V's CTAs start over: set-up, the first stage's latency, an idle SM
// port in between.  Here each CTA pair walks its pass-K tiles and then its
// pass-V tiles in one launch: the producers run on from the last K stage into
// the first V stage, and the MMAs of the V tiles overlap the K epilogues.
// The gate needs every pass-K tile: after its K tiles each CTA adds one to a
// counter, waits (bounded) until every CTA has, forms alpha for its share of
// the tokens from the partials (the same fixed-order sums as
// gate_from_partials_kernel) and adds one to a second counter, which the V
// epilogues wait for before they read alpha.  Those waits need every CTA of
// the grid resident at once: one CTA per SM, at most one per SM of the GPU.
// Partials, alpha and outputs come out bit for bit as from the two passes.
#include <cuda.h>
#include <cuda_bf16.h>

#include "internal.cuh"
#include "tc_ptx.cuh"

namespace engram {
namespace {

using namespace tc;

constexpr float DEC_RMS_EPS = 1e-6f;
constexpr int DBN = 64;                    // pass K: features per pair tile; pass V: tokens
constexpr int DKCH = 2;                    // 64-element K chunks per copy
constexpr int DSTAGES = 4;
constexpr int DEPI = 8;                    // epilogue warps: 2 per TMEM lane quadrant
constexpr int DPARTS = 2;                  // column parts of a tile, one per warp of a quadrant
constexpr int DPART = DBN / DPARTS;        // 32 columns: one chunk per warp
constexpr int DA_CHUNK = BM * BK * 2;
constexpr int DB_CHUNK = (DBN / 2) * BK * 2;
constexpr int DA_BYTES = DA_CHUNK * DKCH;  // 32 KB
constexpr int DB_BYTES = DB_CHUNK * DKCH;  // 8 KB
constexpr int DHBOX = 32 * BM * 2;         // 32 tokens x 128 features of h (bf16)
constexpr int DHSLOT = DPARTS * DHBOX;
constexpr int DHSLOTS = 2;
constexpr int DTMEM_COLS = 2 * DBN;
constexpr int D_HP_WARP = 2 + DEPI;
constexpr int D_BP_WARP = 3 + DEPI;
constexpr int D_THREADS = 64 + DEPI * 32 + 64;
constexpr size_t D_SMEM = (size_t)DSTAGES * (DA_BYTES + DB_BYTES) + (size_t)DHSLOTS * DHSLOT + 256 +
                          2 * DBN * 4;
static_assert(D_SMEM <= 232448, "shared memory");
static_assert(2 * DSTAGES + 13 <= 30, "barrier area");

struct DecArgs {
  int tiles_k, tiles_v;   // pass K: (token blocks of 256) x (feature blocks of 64)
  int nn_k, nn_v;         // feature blocks per token block: d / 64, d / 256
  int num_k_tiles;        // K steps of DKCH chunks
  int64_t N;
  int d;
  int n_part;             // gate partials per token: 2 (d / 64)
  const __nv_bfloat16* h;
  float4* part;
  const float* gg;        // optional g_h g_k
  const float4* conv_w;
  float* conv_state;
  float* alpha;           // [N]
  float* alpha_out;       // optional copy for the caller
  int* counters;          // [2], zero at launch: CTAs past their K tiles, CTAs past their gates
  unsigned int* status;
  uint64_t wait_ns;
  int stall;
};

__device__ __forceinline__ float dec_silu(float y) {  // y/2 (1 + tanh(y/2)), one hardware tanh
  const float hy = 0.5f * y;
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(hy));
  return fmaf(hy, t, hy);
}

__device__ __forceinline__ void dec_unpack32(const uint4 (&w4)[4], float (&x)[32]) {
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const uint32_t ws[4] = {w4[v].x, w4[v].y, w4[v].z, w4[v].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[v * 8 + 2 * i] = __uint_as_float(ws[i] << 16);
      x[v * 8 + 2 * i + 1] = __uint_as_float(ws[i] & 0xffff0000u);
    }
  }
}

// one thread of each CTA waits until counter >= target (bounded; on expiry
// the CTA aborts and flags the status word)
__device__ __forceinline__ bool dec_wait_count(const int* counter, int target,
                                               volatile int* abort_flag, unsigned int* status,
                                               uint64_t limit_ns) {
  const uint64_t t0 = global_ns();
  for (;;) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
    if (v >= target) return true;
    if (*abort_flag || global_ns() - t0 > limit_ns) {
      if (!*abort_flag) atomicOr(status, ENGRAM_STATUS_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
    __nanosleep(64);
  }
}

template <int DIL, bool SCALED>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(D_THREADS, 1)
    tc_decode_kernel(const __grid_constant__ CUtensorMap tmAK,  // e, 128-row boxes
                     const __grid_constant__ CUtensorMap tmBK,  // W_k, 32-row boxes
                     const __grid_constant__ CUtensorMap tmAV,  // W_v, 128-row boxes
                     const __grid_constant__ CUtensorMap tmBV,  // e, 32-row boxes
                     const __grid_constant__ CUtensorMap tmH,   // h, 128 features x 32 tokens
                     const __grid_constant__ CUtensorMap tmO,   // out, the same boxes
                     const __grid_constant__ DecArgs args) {
  constexpr uint32_t STAGE_TX = DA_BYTES + DB_BYTES;
  constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(DBN >> 3) << 17) |
                             ((uint32_t)((2 * BM) >> 4) << 24);
  constexpr int HT = 3 * DIL;  // steps of conv history per feature
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicOr(args.status, ENGRAM_STATUS_TIMEOUT);
    return;
  }
  uint8_t* sA = smem;
  uint8_t* sB = smem + DSTAGES * DA_BYTES;
  uint8_t* hring = sB + DSTAGES * DB_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(hring + DHSLOTS * DHSLOT);
  uint64_t* full = bars;
  uint64_t* empty = bars + DSTAGES;
  uint64_t* tfull = bars + 2 * DSTAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* hfull = drain + 1;
  uint64_t* hempty = hfull + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 30);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 31);
  volatile int* gate_ok = reinterpret_cast<volatile int*>(bars + 29);
  float* alpha_s = reinterpret_cast<float*>(bars + 32);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = (int)(blockIdx.x >> 1), num_pairs = (int)(gridDim.x >> 1);
  // units: the pass-K tiles, then the pass-V tiles
  const int num_units = args.tiles_k + args.tiles_v;
  const int KT = args.num_k_tiles;

  // Pass K tile t: 256 tokens (A = e) x 64 features (B = W_k); pass V tile t:
  // 256 features (A = W_v) x 64 tokens (B = e).  This CTA loads its 128 rows
  // of A and its 32 rows of B.
  auto operand_rows = [&](int unit, int& arow, int& brow) {
    if (unit < args.tiles_k) {
      const int mi = unit / args.nn_k, ni = unit - mi * args.nn_k;
      arow = mi * (2 * BM) + (int)rank * BM;
      brow = ni * DBN + (int)rank * (DBN / 2);
    } else {
      const int t = unit - args.tiles_k;
      const int mi = t / args.nn_v, ni = t - mi * args.nn_v;
      arow = ni * (2 * BM) + (int)rank * BM;
      brow = mi * DBN + (int)rank * (DBN / 2);
    }
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < DSTAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * DEPI);  // epilogue warps of both CTAs
    }
    mbar_init(drain, 1);
    for (int b = 0; b < DHSLOTS; ++b) {
      mbar_init(&hfull[b], 1);
      mbar_init(&hempty[b], DPARTS);  // one release per part, after its output box is stored
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    prefetch_tmap(&tmAK);
    prefetch_tmap(&tmBK);
    prefetch_tmap(&tmAV);
    prefetch_tmap(&tmBV);
    prefetch_tmap(&tmH);
    prefetch_tmap(&tmO);
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc_pair(tmem_slot, DTMEM_COLS);
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // e comes from the gather launched just before this kernel
  wait_prior_grid();
  allow_dependents();

  if (warp == 0 || warp == D_BP_WARP) {
    // -------------------------------------------------- operand producers (A: warp 0, B)
    // The B producer's bytes count on the leader's full barrier, whose
    // expected total the A producer posts.  With ENGRAM_TEST_STALL the B
    // producer issues nothing, so the stages never fill and the waits run out.
    const bool is_a = warp == 0;
    if (lane == 0 && (is_a || !args.stall)) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0;
      for (int unit = pair; unit < num_units; unit += num_pairs) {
        int arow, brow;
        operand_rows(unit, arow, brow);
        const bool vp = unit >= args.tiles_k;
        bool ok = true;
        for (int kt = 0; kt < KT; ++kt) {
          if (!wait_bounded(&empty[stage], phase ^ 1u, abort_flag, args.status, args.wait_ns)) {
            ok = false;
            break;
          }
          const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
          if (is_a) {
            if (leader) mbar_expect_tx(&full[stage], 2 * STAGE_TX);
            tma_load_3d_pair(sA + stage * DA_BYTES, vp ? &tmAV : &tmAK, fb, 0, arow, kt * DKCH);
          } else {
            tma_load_3d_pair(sB + stage * DB_BYTES, vp ? &tmBV : &tmBK, fb, 0, brow, kt * DKCH);
          }
          ++issued;
          if (++stage == DSTAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      // every issued copy of the pair lands before the leader leaves
      if (is_a && leader) {
        for (int s = 0; s < DSTAGES; ++s) {
          const uint32_t n_s = issued > (uint32_t)s ? (issued - 1 - s) / DSTAGES + 1 : 0;
          if (n_s > 0) wait_drain(&full[s], (n_s - 1) & 1u, args.wait_ns);
        }
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------- MMA issuer (leader)
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int unit = pair; unit < num_units && ok; unit += num_pairs) {
        if (!wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, args.status, args.wait_ns)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * DBN);
        for (int kt = 0; kt < KT; ++kt) {
          if (!wait_bounded(&full[stage], phase, abort_flag, args.status, args.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * DA_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * DB_BYTES);
#pragma unroll
          for (int c = 0; c < DKCH; ++c) {
#pragma unroll
            for (int k = 0; k < BK / UMMA_K; ++k) {
              umma_bf16_pair(d_tmem, sw128_desc(a0 + c * DA_CHUNK + k * UMMA_K * 2),
                             sw128_desc(b0 + c * DB_CHUNK + k * UMMA_K * 2), IDESC,
                             (kt | c | k) != 0 ? 1u : 0u);
            }
          }
          umma_commit_pair_both(&empty[stage]);
          if (++stage == DSTAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair_both(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      umma_commit_pair_self(drain);
      wait_drain(drain, 0, args.wait_ns);
    }
  } else if (warp == D_HP_WARP) {
    // -------------------------------------------------- h producer (pass-V tiles)
    if (lane == 0) {
      int slot = 0;
      uint32_t ph = 0;
      uint32_t issued = 0;
      for (int unit = pair; unit < num_units; unit += num_pairs) {
        if (unit < args.tiles_k) continue;
        const int t = unit - args.tiles_k;
        const int mi = t / args.nn_v, ni = t - mi * args.nn_v;
        const int tok0 = mi * DBN;
        const int f0 = ni * (2 * BM) + (int)rank * BM;
        if (!wait_bounded(&hempty[slot], ph ^ 1u, abort_flag, args.status, args.wait_ns)) break;
        mbar_expect_tx(&hfull[slot], DHSLOT);
        uint8_t* dst = hring + slot * DHSLOT;
#pragma unroll
        for (int pt = 0; pt < DPARTS; ++pt)
          tma_load_2d(dst + pt * DHBOX, &tmH, &hfull[slot], f0, tok0 + pt * DPART);
        ++issued;
        if (++slot == DHSLOTS) {
          slot = 0;
          ph ^= 1u;
        }
      }
      for (int b = 0; b < DHSLOTS; ++b) {
        const uint32_t n_b = issued > (uint32_t)b ? (issued - 1 - b) / DHSLOTS + 1 : 0;
        if (n_b > 0) wait_drain(&hfull[b], (n_b - 1) & 1u, args.wait_ns);
      }
    }
  } else {
    // -------------------------------------------------- epilogue
    const int ew = warp - 2;
    const int quad = warp & 3;  // TMEM lanes this warp may read: 32 * quad ..
    const int part = ew >> 2;   // which 32 columns of the tile
    const int etid = ew * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t hslot = 0, hphase = 0;
    int pending_slot = -1;  // storing thread: slot whose output store may still read it
    bool gate_done = false;
    int viter = 0;
    const int G = (int)gridDim.x;
    int* kdone = args.counters;
    int* adone = args.counters + 1;
    // After this CTA's pass-K tiles: count it, wait for every CTA, form the
    // gates of this CTA's tokens (a warp per token), count that, and wait
    // for every CTA's gates.
    auto gate_step = [&]() {
      named_bar_sync(1, DEPI * 32);  // every warp's partials are written
      if (etid == 0) {
        __threadfence();
        atomicAdd(kdone, 1);
        *gate_ok = dec_wait_count(kdone, G, abort_flag, args.status, args.wait_ns) ? 1 : 0;
      }
      named_bar_sync(1, DEPI * 32);
      if (*gate_ok) {
        for (int64_t n = (int64_t)blockIdx.x * DEPI + ew; n < args.N; n += (int64_t)G * DEPI) {
          float kk = 0.f, hk = 0.f, hh = 0.f;
          const float4* pr = args.part + n * args.n_part;
          for (int i = lane; i < args.n_part; i += 32) {
            const float4 q = __ldcg(pr + i);  // written by other CTAs of this grid
            kk += q.x;
            hk += q.y;
            hh += q.z;
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            kk += __shfl_xor_sync(FULL, kk, o);
            hk += __shfl_xor_sync(FULL, hk, o);
            hh += __shfl_xor_sync(FULL, hh, o);
          }
          if (lane == 0) {
            const float invd = 1.0f / (float)args.d;
            const float rh = rsqrtf(hh * invd + DEC_RMS_EPS), rk = rsqrtf(kk * invd + DEC_RMS_EPS);
            const float a = 1.0f / (1.0f + expf(-(hk * rh * rk * rsqrtf((float)args.d))));
            args.alpha[n] = a;
            if (args.alpha_out != nullptr) args.alpha_out[n] = a;
          }
        }
      }
      named_bar_sync(1, DEPI * 32);  // this CTA's gates are written
      if (etid == 0) {
        __threadfence();
        atomicAdd(adone, 1);
        dec_wait_count(adone, G, abort_flag, args.status, args.wait_ns);
      }
      named_bar_sync(1, DEPI * 32);
      gate_done = true;
    };

    for (int unit = pair; unit < num_units; unit += num_pairs) {
      const bool vp = unit >= args.tiles_k;
      if (vp && !gate_done) gate_step();
      const uint32_t t_acc = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * DBN);
      auto wait_acc = [&]() {
        int ok = 0;
        if (lane == 0)
          ok = wait_bounded(&tfull[acc], acc_phase, abort_flag, args.status, args.wait_ns) ? 1 : 0;
        ok = __shfl_sync(FULL, ok, 0);
        tc_fence_after();
        return ok;
      };
      if (!vp) {
        // ---- pass K: this lane's token, 32 features of the tile
        const int mi = unit / args.nn_k, ni = unit - mi * args.nn_k;
        const int64_t n = (int64_t)mi * (2 * BM) + (int)rank * BM + quad * 32 + lane;
        const bool valid = n < args.N;
        const int col_base = ni * DBN + part * DPART;
        uint4 h0[4];
        if (valid) {
          const uint4* q = reinterpret_cast<const uint4*>(args.h + n * args.d + col_base);
#pragma unroll
          for (int v = 0; v < 4; ++v) h0[v] = __ldg(q + v);
        }
        const int got = wait_acc();
        float v[32];
        __syncwarp();
        if (got) {
          tmem_ld32(t_acc + (uint32_t)(part * DPART), v);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0.f;
        }
        if (valid) {
          float hv[32];
          dec_unpack32(h0, hv);
          float kk = 0.f, hk = 0.f, hh = 0.f;
          if constexpr (SCALED) {
            const float4* gq = reinterpret_cast<const float4*>(args.gg + col_base);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 g4 = __ldg(gq + q);
              const float gw[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
              for (int r = 0; r < 4; ++r) {
                const int i = 4 * q + r;
                kk = fmaf(v[i], v[i], kk);
                hk = fmaf(hv[i] * gw[r], v[i], hk);
                hh = fmaf(hv[i], hv[i], hh);
              }
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              kk = fmaf(v[i], v[i], kk);
              hk = fmaf(hv[i], v[i], hk);
              hh = fmaf(hv[i], hv[i], hh);
            }
          }
          args.part[n * args.n_part + ni * DPARTS + part] = make_float4(kk, hk, hh, 0.f);
        }
      } else {
        // ---- pass V (decode): this lane's feature, 32 tokens of the tile;
        // the conv state of each token, its gate, the conv, the residual
        const int t = unit - args.tiles_k;
        const int mi = t / args.nn_v, ni = t - mi * args.nn_v;
        const int64_t tok0 = (int64_t)mi * DBN;
        const int f0 = ni * (2 * BM) + (int)rank * BM;
        const int feat = f0 + quad * 32 + lane;
        const float4 w = __ldg(args.conv_w + feat);  // taps: w.x for t-3 dil .. w.w for t
        float* al = alpha_s + (viter & 1) * DBN;
        for (int i = etid; i < DBN; i += DEPI * 32) {
          const int64_t nn = tok0 + i;
          al[i] = nn < args.N ? __ldcg(args.alpha + nn) : 0.f;  // written during this grid
        }
        const int j0 = part * DPART;
        const int64_t nb = tok0 + j0;
        // tokens in groups of GT, each group's states loaded before any is
        // written back; with dilation 1 the first group's are fetched while
        // the MMAs finish
        constexpr int GT = DIL == 1 ? 16 : 4;
        float pre[DIL == 1 ? GT : 1][HT];
        if constexpr (DIL == 1) {
#pragma unroll
          for (int i = 0; i < GT; ++i) {
            const int64_t nn = nb + i;
#pragma unroll
            for (int k = 0; k < HT; ++k) pre[i][k] = 0.f;
            if (nn < args.N) {
              const float* st = args.conv_state + nn * HT * args.d + feat;
#pragma unroll
              for (int k = 0; k < HT; ++k) pre[i][k] = st[(int64_t)k * args.d];
            }
          }
        }
        named_bar_sync(1, DEPI * 32);  // the gates are staged
        const int got = wait_acc();
        int hgot = 0;
        if (lane == 0)
          hgot = wait_bounded(&hfull[hslot], hphase, abort_flag, args.status, args.wait_ns) ? 1 : 0;
        hgot = __shfl_sync(FULL, hgot, 0);
        uint8_t* box = hring + hslot * DHSLOT + part * DHBOX;
        uint16_t* hs = reinterpret_cast<uint16_t*>(box) + quad * 32 + lane;
        uint32_t u[16], un[16];
        __syncwarp();
        if (got) {
          tmem_ld16(t_acc + (uint32_t)j0, u);
          tmem_ld16(t_acc + (uint32_t)(j0 + 16), un);
          tmem_wait16(u);
          tmem_wait16(un);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) u[i] = un[i] = 0u;
        }
#pragma unroll
        for (int g = 0; g < 32 / GT; ++g) {
          float sq[GT][HT];
          if (DIL == 1 && g == 0) {
#pragma unroll
            for (int i = 0; i < GT; ++i)
#pragma unroll
              for (int k = 0; k < HT; ++k) sq[i][k] = pre[DIL == 1 ? i : 0][k];
          } else {
#pragma unroll
            for (int i = 0; i < GT; ++i) {
              const int64_t nn = nb + g * GT + i;
#pragma unroll
              for (int k = 0; k < HT; ++k) sq[i][k] = 0.f;
              if (nn < args.N) {
                const float* st = args.conv_state + nn * HT * args.d + feat;
#pragma unroll
                for (int k = 0; k < HT; ++k) sq[i][k] = st[(int64_t)k * args.d];
              }
            }
          }
#pragma unroll
          for (int i = 0; i < GT; ++i) {
            const int jj = g * GT + i;
            const int64_t nn = nb + jj;
            const float vt = al[j0 + jj] * __uint_as_float(jj < 16 ? u[jj] : un[jj - 16]);
            if (nn < args.N) {
              float* st = args.conv_state + nn * HT * args.d + feat;
#pragma unroll
              for (int k = 0; k + 1 < HT; ++k) st[(int64_t)k * args.d] = sq[i][k + 1];
              st[(int64_t)(HT - 1) * args.d] = vt;
            }
            const float y =
                fmaf(w.x, sq[i][0], fmaf(w.y, sq[i][DIL], fmaf(w.z, sq[i][2 * DIL], w.w * vt)));
            const float hv = __uint_as_float(((uint32_t)hs[jj * BM]) << 16);
            hs[jj * BM] = __bfloat16_as_ushort(__float2bfloat16_rn(hv + vt + dec_silu(y)));
          }
        }
        // the part's four warps have written the box: one thread stores it
        fence_async_shared();
        named_bar_sync(2 + part, 128);
        if (ew == part * 4 && lane == 0) {
          if (hgot && got)
            tma_store_2d(&tmO, box, f0, (int)nb);
          else
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");  // one group per tile
          asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
          if (pending_slot >= 0) mbar_arrive(&hempty[pending_slot]);
          pending_slot = (int)hslot;
        }
        if (++hslot == (uint32_t)DHSLOTS) {
          hslot = 0;
          hphase ^= 1u;
        }
        ++viter;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    // a CTA without pass-V tiles still counts its K tiles and its gates
    if (!gate_done) gate_step();
    if (ew == part * 4 && lane == 0) {
      asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
      if (pending_slot >= 0) mbar_arrive(&hempty[pending_slot]);
    }
  }

  tc_fence_before();
  __syncwarp();
  cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, DTMEM_COLS);
  }
}

}  // namespace

// N <= 4096: the gate partials' room in the forward workspace is that of
// the narrow tiles (d / 32 per token) up to there
bool decode_fused_ok(int64_t N, int d, int E) {
  return N > 0 && N <= 4096 && d % (2 * BM) == 0 && E % (DKCH * BK) == 0 && E > 0;
}

int launch_decode_fused(const __nv_bfloat16* e, const __nv_bfloat16* h, const __nv_bfloat16* Wk,
                        const __nv_bfloat16* Wv, const float* conv_w, float* conv_state,
                        __nv_bfloat16* out, float* alpha_saved, const float* gg, int dil,
                        int64_t N, int d, int E, float4* part, float* alpha, int* counters,
                        bool counters_zeroed, bool chained, bool stall, cudaStream_t s) {
  CUtensorMap tak, tbk, tav, tbv, th, to;
  if (!make_tmap_k(&tak, e, (uint64_t)E, (uint64_t)N, BM, DKCH) ||
      !make_tmap_k(&tbk, Wk, (uint64_t)E, (uint64_t)d, DBN / 2, DKCH) ||
      !make_tmap_k(&tav, Wv, (uint64_t)E, (uint64_t)d, BM, DKCH) ||
      !make_tmap_k(&tbv, e, (uint64_t)E, (uint64_t)N, DBN / 2, DKCH) ||
      !make_tmap(&th, h, (uint64_t)d, (uint64_t)N, BM, 32, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tmap(&to, out, (uint64_t)d, (uint64_t)N, BM, 32, CU_TENSOR_MAP_SWIZZLE_NONE))
    return ENGRAM_ERR_CUDA;
  int rc;
  if (!counters_zeroed && (rc = ck(cudaMemsetAsync(counters, 0, 2 * sizeof(int), s)))) return rc;
  DecArgs a = {};
  a.nn_k = d / DBN;
  a.nn_v = d / (2 * BM);
  a.tiles_k = (int)((N + 2 * BM - 1) / (2 * BM)) * a.nn_k;
  a.tiles_v = (int)((N + DBN - 1) / DBN) * a.nn_v;
  a.num_k_tiles = E / (BK * DKCH);
  a.N = N;
  a.d = d;
  a.n_part = 2 * (d / DBN);
  a.h = h;
  a.part = part;
  a.gg = gg;
  a.conv_w = reinterpret_cast<const float4*>(conv_w);
  a.conv_state = conv_state;
  a.alpha = alpha;
  a.alpha_out = alpha_saved;
  a.counters = counters;
  a.status = status_ptr();
  a.wait_ns = stall ? TEST_WAIT_LIMIT_NS : WAIT_LIMIT_NS;
  a.stall = stall ? 1 : 0;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ENGRAM_ERR_CUDA;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int units = a.tiles_k > a.tiles_v ? a.tiles_k : a.tiles_v;
  auto run = [&](auto kern) -> int {
    static bool configured[64][4] = {};
    static int max_pairs[64][4] = {};
    const int key = (dil == 3 ? 2 : 0) + (gg != nullptr ? 1 : 0);
    if (!configured[dev][key]) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)D_SMEM) !=
          cudaSuccess)
        return (int)ENGRAM_ERR_CUDA;
      // the CTA pairs that fit on the GPU at once (one CTA per SM; a pair
      // needs two SMs of one cluster-capable group): the waits at the gate
      // need every CTA of the grid resident
      cudaLaunchConfig_t q = {};
      q.gridDim = dim3((unsigned)(sms & ~1));
      q.blockDim = dim3(D_THREADS);
      q.dynamicSmemBytes = D_SMEM;
      cudaLaunchAttribute qa[1];
      qa[0].id = cudaLaunchAttributeClusterDimension;
      qa[0].val.clusterDim.x = 2;
      qa[0].val.clusterDim.y = 1;
      qa[0].val.clusterDim.z = 1;
      q.attrs = qa;
      q.numAttrs = 1;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, kern, &q) != cudaSuccess || clusters <= 0) {
        cudaGetLastError();
        clusters = sms / 2;
      }
      max_pairs[dev][key] = clusters < sms / 2 ? clusters : sms / 2;
      configured[dev][key] = true;
    }
    const int pairs = units < max_pairs[dev][key] ? units : max_pairs[dev][key];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(D_THREADS);
    cfg.dynamicSmemBytes = D_SMEM;
    cfg.stream = s;
    // cooperative: the CTAs start together or not at all, so work on other
    // streams cannot hold back part of the grid while the rest waits at the
    // gate
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = chained ? 2 : 1;
    return ck(cudaLaunchKernelEx(&cfg, kern, tak, tbk, tav, tbv, th, to, a));
  };
  if (dil == 3)
    return gg != nullptr ? run(tc_decode_kernel<3, true>) : run(tc_decode_kernel<3, false>);
  return gg != nullptr ? run(tc_decode_kernel<1, true>) : run(tc_decode_kernel<1, false>);
}

}  // namespace engram
