// bf16 fusion stage on the sm_100a tensor cores.
//
// The two projections k = W_k e and v = W_v e are the layer's only dense
// contractions (discuss.deepseek.club 二.1 (2): h is the query, e the key and
// value, combined by matrix products).  Each runs as one persistent tcgen05
// GEMM pass with the rest of the layer fused into its epilogue:
//
//   pass K:  C = e * W_k^T (tokens on TMEM lanes); the epilogue reduces each
//            token's row of the tile to (sum k^2, sum h*k, sum h^2) partials --
//            k never reaches HBM.  A small kernel then forms
//            alpha = sigmoid(<h, k> r_h r_k / sqrt(d)) per token.
//   pass V:  C = W_v * e^T (features on TMEM lanes, tokens on columns); each
//            epilogue thread owns one feature and walks consecutive tokens:
//            vt = alpha * v, the width-4 depthwise causal conv with the three
//            previous vt in registers, SiLU, and h + vt + SiLU(y) (sechub.in
//            answer: short depthwise causal conv; discuss.deepseek.club
//            二.1 (2): 1-D conv, residual).  h comes in and out goes back in
//            32-token boxes by TMA.
//
// The conv needs vt of the three tokens before each one.  Pass V's token
// tiles of 256 overlap by 3: the first three tokens of a tile are a
// recomputed halo and are not stored.  In decode (one token per sequence) the
// three earlier vt come from the conv state.
//
// Pipeline per CTA (one CTA per SM):
//   warp 0      one lane issues TMA loads of the A and B tiles into a ring of
//               shared-memory stages (128-byte swizzle, K-major);
//   warp 1      allocates TMEM; one lane issues tcgen05.mma (M=128, N=BN,
//               K=16 per instruction) into one of two TMEM accumulators;
//   epilogue    8 warps: warp w reads TMEM lanes 32*(w%4).. and half of the
//               tile's columns;
//   last warp   pass V: one lane streams h into a ring of shared-memory boxes.
// mbarriers link the roles; every wait is bounded in time and, when it runs
// out, sets ENGRAM_STATUS_TIMEOUT and winds the CTA down without hanging.
#include "tc_ptx.cuh"

namespace engram {

namespace {

using namespace tc;

constexpr float RMS_EPS = 1e-6f;

// pass K; pass V over whole sequences (conv history from the rows above);
// pass V in decode (one token per sequence, conv history from the state)
// Kernel modes, as bits: pass K (MODE_GATE_SCALED: with learnable norm
// scales) or pass V (MODE_V_PASS) with its options: decode steps, v also
// stored for the backward, the conv dilated by 3.
enum {
  MODE_GATE_PARTIAL = 0,
  MODE_GATE_SCALED = 1,
  MODE_V_PASS = 16,
  MODE_V_DECODE = 2,
  MODE_V_KEEP = 4,
  MODE_V_DILATED = 8,
  MODE_VALUE_CONV = MODE_V_PASS,
  MODE_VALUE_DECODE = MODE_V_PASS | MODE_V_DECODE,
  MODE_VALUE_CONV_KV = MODE_V_PASS | MODE_V_KEEP
};

struct TcArgs {
  int num_m_tiles, num_n_tiles, num_k_tiles;
  int m_stride, m_offset;
  int64_t N;
  int T;
  int d;
  int n_part;
  const __nv_bfloat16* h;
  __nv_bfloat16* out;
  float4* part;
  const float4* conv_w;
  float* conv_state;
  float* alpha_out;     // pass V: optional copy of alpha for the caller
  const float* alpha;   // pass V: gate of every token, from the gate kernel
  float* kv_save;       // optional fp32 [N, 2d]: k (pass K) then v (pass V) of each token
  const float* gg;      // optional [d]: g_h * g_k, the learnable norm scales' product (pass K)
  unsigned int* status;
  uint64_t wait_ns;     // limit of every bounded wait
  int stall;            // ENGRAM_TEST_STALL: the B producer issues nothing
};


// 32 bf16 held in 4 x 16 bytes -> fp32
__device__ __forceinline__ void unpack_bf16x32(const uint4 (&w4)[4], float (&x)[32]) {
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

// 32 bf16 (64 bytes) -> fp32
__device__ __forceinline__ void load_bf16x32(const __nv_bfloat16* p, float (&x)[32]) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const uint4 w = __ldg(q + v);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[v * 8 + 2 * i] = __uint_as_float(ws[i] << 16);
      x[v * 8 + 2 * i + 1] = __uint_as_float(ws[i] & 0xffff0000u);
    }
  }
}

// Pass V, 16 consecutive tokens of one feature: vt = alpha * v, the width-4
// causal conv over (s3, s2, s1, vt), out = h + vt + SiLU(y), written over h in
// place.  CHECK = true when a sequence may start inside the group: the conv
// history is cleared at position 0.
//
// SiLU(y) = y * sigmoid(y) = y/2 * (1 + tanh(y/2)): one hardware tanh
// (tanh.approx.f32, relative error about 2^-11) instead of an exponential and
// a reciprocal; the error stays below the bf16 rounding of the output (2^-9).
__device__ __forceinline__ float silu_tanh(float y) {
  const float hy = 0.5f * y;
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(hy));
  return fmaf(hy, t, hy);
}

// sh[q] holds vt of token t-1-q (the conv's 3 * DIL tokens of history).
template <bool CHECK, int DIL>
__device__ __forceinline__ void conv_group16(const uint32_t (&u)[16], const float4* al4,
                                             uint16_t* hs, const float4 w, float (&sh)[3 * DIL],
                                             int& pos, const int T) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float4 a4 = al4[q];
    const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int jj = q * 4 + r;
      const float vt = av[r] * __uint_as_float(u[jj]);
      if (CHECK) {
        if (pos == 0) {  // a sequence starts at this token
#pragma unroll
          for (int k = 0; k < 3 * DIL; ++k) sh[k] = 0.f;
        }
        pos = (pos + 1 == T) ? 0 : pos + 1;
      }
      const float y =
          fmaf(w.x, sh[3 * DIL - 1], fmaf(w.y, sh[2 * DIL - 1], fmaf(w.z, sh[DIL - 1], w.w * vt)));
#pragma unroll
      for (int k = 3 * DIL - 1; k > 0; --k) sh[k] = sh[k - 1];
      sh[0] = vt;
      const float hv = __uint_as_float(((uint32_t)hs[jj * BM]) << 16);
      const float o = hv + vt + silu_tanh(y);  // h + vt + SiLU(y)
      hs[jj * BM] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
    }
  }
}

// ------------------------------------------------------------------ kernel

template <int BN, int STAGES, int MODE, int KCH>
struct TcShape {
  static constexpr bool VPASS = (MODE & MODE_V_PASS) != 0;
  static constexpr bool DECODE = VPASS && (MODE & MODE_V_DECODE) != 0;
  static constexpr bool KEEP_V = VPASS && (MODE & MODE_V_KEEP) != 0;
  static constexpr bool SCALED = !VPASS && (MODE & MODE_GATE_SCALED) != 0;
  static constexpr int DIL = (VPASS && (MODE & MODE_V_DILATED) != 0) ? 3 : 1;  // conv dilation
  static constexpr int HALO_T = 3 * DIL;  // tokens of conv history a token needs
  // epilogue warps: 2 per TMEM lane quadrant
  static constexpr int EPI = 8;
  static constexpr int PARTS = EPI / 4;        // column parts of a tile, one per warp of a quadrant
  static constexpr int HP_WARP = 2 + EPI;      // pass V: warp that streams h in by TMA
  // B-operand producer: a second issuing thread, since one thread issues
  // tiled copies at only about one per 150 ns (measured on B200), which would
  // bound a stage of two boxes at ~300 ns
  static constexpr int BP_WARP = 3 + EPI;
  static constexpr int NUM_THREADS = 64 + EPI * 32 + 64;
  // a CTA pair computes a (2 * BM) x BN tile: each CTA loads its BM rows of
  // A and half of the BN rows of B, and holds its BM rows of the accumulator
  // a stage holds KCH chunks of 64 K elements (128 bytes) of each operand,
  // each chunk a 128-byte-swizzled tile of its rows
  static constexpr int A_CHUNK = BM * BK * 2;
  static constexpr int B_CHUNK = (BN / 2) * BK * 2;
  static constexpr int A_BYTES = A_CHUNK * KCH;
  static constexpr int B_BYTES = B_CHUNK * KCH;
  static constexpr int TMEM_COLS = 2 * BN;
  // pass K (tokens on TMEM lanes, features on columns): each epilogue warp
  // takes one part of the tile's columns, 32 at a time
  static constexpr int PART_COLS = BN / PARTS;
  static constexpr int NCHUNK = PART_COLS / 32;
  // pass V (features on TMEM lanes, tokens on columns): each epilogue warp
  // takes one part of the tile's tokens, 32 at a time; h arrives by TMA in
  // slots of PARTS boxes (one per part) of 32 tokens x 128 features
  static constexpr int HBOX_BYTES = 32 * BM * 2;
  static constexpr int HSLOT_BYTES = PARTS * HBOX_BYTES;
  static constexpr int ALPHA_BYTES = VPASS ? 2 * BN * 4 : 0;  // gates of a tile, two tiles
  // pass K, when k is kept: each epilogue warp stages its 32 tokens x 32
  // features (fp32, 128-byte swizzled) for one tiled store; pass V keeping v
  // stages its 32 tokens x 32 features (token rows) the same way
  static constexpr int KVBUF_BYTES = (VPASS && !KEEP_V) ? 0 : EPI * 32 * 32 * 4;
  // as many h slots (up to 4) as the shared memory left by the operand stages holds
  static constexpr int HSLOTS_FIT =
      (232448 - STAGES * (A_BYTES + B_BYTES) - KVBUF_BYTES - 256 - ALPHA_BYTES) / HSLOT_BYTES;
  static constexpr int HSLOTS = VPASS ? (HSLOTS_FIT < 4 ? HSLOTS_FIT : 4) : 0;
  static constexpr size_t SMEM = (size_t)STAGES * (A_BYTES + B_BYTES) +
                                 (size_t)HSLOTS * HSLOT_BYTES + KVBUF_BYTES + 256 + ALPHA_BYTES;
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "N tile");
  static_assert(2 * STAGES + 13 <= 30, "barrier area");
  static_assert(SMEM <= 232448, "shared memory");
  static_assert(!VPASS || HSLOTS >= 2, "h ring");
  static_assert(PART_COLS % 32 == 0, "parts of whole 32-column chunks");
};

template <int BN, int STAGES, int MODE, int KCH>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(TcShape<BN, STAGES, MODE, KCH>::NUM_THREADS, 1)
    tc_fused_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmO,
                    const __grid_constant__ CUtensorMap tmO29, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmV29, const __grid_constant__ TcArgs args) {
  using S = TcShape<BN, STAGES, MODE, KCH>;
  constexpr bool VPASS = S::VPASS;
  constexpr int NUM_EPI_WARPS = S::EPI;
  constexpr int HP_WARP = S::HP_WARP;
  constexpr int PARTS = S::PARTS;
  constexpr uint32_t STAGE_TX = S::A_BYTES + S::B_BYTES;
  // instruction descriptor: fp32 accumulate, bf16 A and B, both K-major,
  // N >> 3 at bit 17, M >> 4 at bit 24 (M = 256 over the CTA pair)
  constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                             ((uint32_t)((2 * BM) >> 4) << 24);

  // The kernel declares no static shared memory, so the dynamic block starts
  // at the base of the CTA's window.  Addressing everything from the
  // __shared__ array keeps every access a shared-memory instruction.
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {  // 128-byte swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicOr(args.status, ENGRAM_STATUS_TIMEOUT);
    return;
  }
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * S::A_BYTES;
  uint8_t* hring = sB + STAGES * S::B_BYTES;
  uint8_t* kvbuf = hring + S::HSLOTS * S::HSLOT_BYTES;  // pass K, and pass V keeping v
  uint64_t* bars = reinterpret_cast<uint64_t*>(kvbuf + S::KVBUF_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* hfull = drain + 1;
  uint64_t* hempty = hfull + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 30);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 31);
  float* alpha_s = reinterpret_cast<float*>(bars + 32);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_tiles = args.num_m_tiles * args.num_n_tiles;
  // CTA pair: rank 0 (the leader) issues the MMAs for both
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = (int)(blockIdx.x >> 1), num_pairs = (int)(gridDim.x >> 1);

  // Tile t covers token block t / num_n_tiles and feature block
  // t % num_n_tiles.  Pass K multiplies e (256 tokens, A) by W_k (BN
  // features, B); pass V multiplies W_v (256 features, A) by e (BN tokens,
  // B).  This CTA loads its 128 rows of A and its half of B.
  auto operand_rows = [&](int tile, int& arow, int& brow) {
    const int mi = tile / args.num_n_tiles, ni = tile - mi * args.num_n_tiles;
    const int tok0 = mi * args.m_stride + args.m_offset;
    if (VPASS) {
      arow = ni * (2 * BM) + (int)rank * BM;
      brow = tok0 + (int)rank * (BN / 2);
    } else {
      arow = tok0 + (int)rank * BM;
      brow = ni * BN + (int)rank * (BN / 2);
    }
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * NUM_EPI_WARPS);  // epilogue warps of both CTAs
    }
    mbar_init(drain, 1);
    for (int b = 0; b < S::HSLOTS; ++b) {
      mbar_init(&hfull[b], 1);
      mbar_init(&hempty[b], PARTS);  // one release per part, after its output box is stored
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    if (VPASS) {
      prefetch_tmap(&tmH);
      prefetch_tmap(&tmO);
      prefetch_tmap(&tmO29);
      if constexpr (S::KEEP_V) {
        prefetch_tmap(&tmV);
        prefetch_tmap(&tmV29);
      }
    }
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc_pair(tmem_slot, S::TMEM_COLS);
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync();  // both CTAs' barriers exist before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Pass K reads e, written by the gather launched just before it: wait for
  // it after the set-up above, then let the gate and pass V launch.  Pass V
  // starts its operand loads and MMAs at once (e is complete by then) and
  // waits for the gate only where its epilogue first reads alpha.
  if (!VPASS) wait_prior_grid();
  allow_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ operand producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0;
      for (int tile = pair; tile < num_tiles; tile += num_pairs) {
        int arow, brow;
        operand_rows(tile, arow, brow);
        bool ok = true;
        for (int kt = 0; kt < args.num_k_tiles; ++kt) {
          if (!wait_bounded(&empty[stage], phase ^ 1u, abort_flag, args.status, args.wait_ns)) {
            ok = false;
            break;
          }
          // the leader's full barrier counts the bytes of both CTAs' A and B
          // boxes (B comes from the B producer below)
          if (leader) mbar_expect_tx(&full[stage], 2 * STAGE_TX);
          const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
          tma_load_3d_pair(sA + stage * S::A_BYTES, &tmA, fb, 0, arow, kt * KCH);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      // every issued copy of the pair lands before the leader leaves (the
      // peer waits for the leader at the closing cluster barrier)
      if (leader) {
        for (int s = 0; s < STAGES; ++s) {
          const uint32_t n_s = issued > (uint32_t)s ? (issued - 1 - s) / STAGES + 1 : 0;
          if (n_s > 0) wait_drain(&full[s], (n_s - 1) & 1u, args.wait_ns);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
        if (!wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, args.status, args.wait_ns)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kt = 0; kt < args.num_k_tiles; ++kt) {
          if (!wait_bounded(&full[stage], phase, abort_flag, args.status, args.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * S::A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * S::B_BYTES);
#pragma unroll
          for (int c = 0; c < KCH; ++c) {
#pragma unroll
            for (int k = 0; k < BK / UMMA_K; ++k) {
              umma_bf16_pair(d_tmem, sw128_desc(a0 + c * S::A_CHUNK + k * UMMA_K * 2),
                             sw128_desc(b0 + c * S::B_CHUNK + k * UMMA_K * 2), IDESC,
                             (kt | c | k) != 0 ? 1u : 0u);
            }
          }
          umma_commit_pair_both(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair_both(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      // all issued MMAs complete before TMEM is released
      umma_commit_pair_self(drain);
      wait_drain(drain, 0, args.wait_ns);
    }
  } else if (warp == S::BP_WARP) {
    // ------------------------------------------------------------ B-operand producer
    // Same stages and order as the A producer; its bytes count on the
    // leader's full barrier, whose expected total the A producer posts (a
    // phase cannot complete before that arrival).  With ENGRAM_TEST_STALL it
    // issues nothing, so the stages never fill and the waits run out.
    if (lane == 0 && !args.stall) {
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = pair; tile < num_tiles; tile += num_pairs) {
        int arow, brow;
        operand_rows(tile, arow, brow);
        bool ok = true;
        for (int kt = 0; kt < args.num_k_tiles; ++kt) {
          if (!wait_bounded(&empty[stage], phase ^ 1u, abort_flag, args.status, args.wait_ns)) {
            ok = false;
            break;
          }
          const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
          tma_load_3d_pair(sB + stage * S::B_BYTES, &tmB, fb, 0, brow, kt * KCH);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
    }
  } else if (warp == HP_WARP) {
    // ------------------------------------------------------------ h producer (pass V)
    if (VPASS && lane == 0) {
      constexpr int NCH = S::NCHUNK;
      int slot = 0;
      uint32_t ph = 0;
      uint32_t issued = 0;
      for (int tile = pair; tile < num_tiles; tile += num_pairs) {
        const int mi = tile / args.num_n_tiles, ni = tile - mi * args.num_n_tiles;
        const int tok0 = mi * args.m_stride + args.m_offset;
        const int f0 = ni * (2 * BM) + (int)rank * BM;  // this CTA's features
        bool ok = true;
        for (int c = 0; c < NCH; ++c) {
          if (!wait_bounded(&hempty[slot], ph ^ 1u, abort_flag, args.status, args.wait_ns)) {
            ok = false;
            break;
          }
          mbar_expect_tx(&hfull[slot], S::HSLOT_BYTES);
          uint8_t* dst = hring + slot * S::HSLOT_BYTES;
#pragma unroll
          for (int pt = 0; pt < PARTS; ++pt)
            tma_load_2d(dst + pt * S::HBOX_BYTES, &tmH, &hfull[slot], f0,
                        tok0 + pt * S::PART_COLS + c * 32);
          ++issued;
          if (++slot == S::HSLOTS) {
            slot = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
      }
      for (int b = 0; b < S::HSLOTS; ++b) {
        const uint32_t n_b = issued > (uint32_t)b ? (issued - 1 - b) / (S::HSLOTS > 0 ? S::HSLOTS : 1) + 1 : 0;
        if (n_b > 0) wait_drain(&hfull[b], (n_b - 1) & 1u, args.wait_ns);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;
    const int quad = warp & 3;  // TMEM lanes this warp may read: 32 * quad ..
    const int part = ew >> 2;   // which part of the tile's columns
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t hslot = 0, hphase = 0;  // pass V: next h ring slot and its phase parity
    int pending_slot = -1;  // pass V, storing thread: slot whose output store may still read it
    int iter = 0;
    for (int tile = pair; tile < num_tiles; tile += num_pairs, ++iter) {
      const int mi = tile / args.num_n_tiles, ni = tile - mi * args.num_n_tiles;
      const int64_t tok0 = (int64_t)mi * args.m_stride + args.m_offset;
      // while the MMAs of this tile run: pull what the epilogue will read
      // into L2 (pass K: the first tile's h; decode: the conv state)
      if constexpr (!VPASS) {
        if (iter == 0) {
          const int64_t n0 = tok0 + (int)rank * BM + quad * 32 + lane;
          if (n0 >= 0 && n0 < args.N) {
            const __nv_bfloat16* hp0 = args.h + n0 * args.d + ni * BN + part * S::PART_COLS;
            for (int b = 0; b < S::PART_COLS * 2; b += 128) prefetch_l2(hp0 + b / 2);
          }
        }
      } else if constexpr (S::DECODE) {
        const int64_t n0 = tok0 + part * S::PART_COLS + lane;
        if (lane < S::PART_COLS && n0 < args.N) {
          const float* st = args.conv_state + n0 * 3 * args.d + ni * (2 * BM) + (int)rank * BM +
                            quad * 32;
          prefetch_l2(st);
          prefetch_l2(st + args.d);
          prefetch_l2(st + 2 * args.d);
        }
      }
      const uint32_t t_acc = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * BN);
      // the tile's accumulator is complete (each branch first issues the
      // loads that do not depend on it)
      auto wait_acc = [&]() {
        int ok = 0;
        if (lane == 0) ok = wait_bounded(&tfull[acc], acc_phase, abort_flag, args.status, args.wait_ns) ? 1 : 0;
        ok = __shfl_sync(FULL, ok, 0);
        tc_fence_after();
        return ok;
      };

      if constexpr (!VPASS) {
        // pass K: this lane's token, one part of the tile's features
        const int64_t n = tok0 + (int)rank * BM + quad * 32 + lane;
        const bool valid = n >= 0 && n < args.N;
        const int col_base = ni * BN + part * S::PART_COLS;
        // h of the first 32 features, fetched while the MMAs finish
        uint4 h0[4];
        if (valid) {
          const uint4* q = reinterpret_cast<const uint4*>(args.h + n * args.d + col_base);
#pragma unroll
          for (int v = 0; v < 4; ++v) h0[v] = __ldg(q + v);
        }
        const int got = wait_acc();
        const uint32_t t_row = t_acc + (uint32_t)(part * S::PART_COLS);
        {  // pull the next tile's rows of h into L2 while this one is reduced
          const int nxt = tile + num_pairs;
          if (nxt < num_tiles) {
            const int mi2 = nxt / args.num_n_tiles, ni2 = nxt - mi2 * args.num_n_tiles;
            const int64_t n2 = (int64_t)mi2 * args.m_stride + args.m_offset + (int)rank * BM +
                               quad * 32 + lane;
            if (n2 >= 0 && n2 < args.N) {
              const __nv_bfloat16* hp2 = args.h + n2 * args.d + ni2 * BN + part * S::PART_COLS;
              for (int b = 0; b < S::PART_COLS * 2; b += 128) prefetch_l2(hp2 + b / 2);
            }
          }
        }
        float kk = 0.f, hk = 0.f, hh = 0.f;
#pragma unroll 1
        for (int c = 0; c < S::NCHUNK; ++c) {
          float v[32];
          __syncwarp();
          if (got) {
            tmem_ld32(t_row + c * 32, v);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0.f;
          }
          if (args.kv_save != nullptr && got) {
            // k itself, for the backward: the warp's 32 x 32 block goes
            // through its staging buffer (row = token, 16-byte chunks
            // swizzled by the row) and out in one tiled store; rows past N
            // are not written
            uint8_t* kb = kvbuf + ew * (32 * 32 * 4);
            if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
            __syncwarp();  // the previous store has read the buffer
#pragma unroll
            for (int q = 0; q < 8; ++q)
              *reinterpret_cast<float4*>(kb + lane * 128 + ((q ^ (lane & 7)) * 16)) =
                  make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            fence_async_shared();
            __syncwarp();
            if (lane == 0)
              tma_store_2d(&tmO, kb, col_base + c * 32, (int)(tok0 + (int)rank * BM + quad * 32));
          }
          if (valid) {
            float hv[32];
            if (c == 0)
              unpack_bf16x32(h0, hv);
            else
              load_bf16x32(args.h + n * args.d + col_base + c * 32, hv);
            if constexpr (S::SCALED) {
              // <RMSNorm(h) g_h, RMSNorm(k) g_k>: weight h k by g_h g_k
              const float4* gq = reinterpret_cast<const float4*>(args.gg + col_base + c * 32);
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
          }
        }
        if (valid) args.part[n * args.n_part + ni * PARTS + part] = make_float4(kk, hk, hh, 0.f);
        if (args.kv_save != nullptr && tile + num_pairs >= num_tiles && lane == 0)
          asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");  // before the CTA exits
      } else {
        // pass V: this lane's feature, one part of the tile's tokens.  The causal
        // conv walks the tokens in order with vt of the three previous tokens
        // of the same sequence in registers.
        constexpr bool DECODE = S::DECODE;
        constexpr int NCH = S::NCHUNK;
        const int f0 = ni * (2 * BM) + (int)rank * BM;  // this CTA's features
        const int feat = f0 + quad * 32 + lane;
        const int T = args.T;
        const float4 w = __ldg(args.conv_w + feat);  // taps: w.x for t-3 .. w.w for t
        if (iter == 0) wait_prior_grid();  // alpha comes from the gate kernel
        // gates of the tile's tokens, staged once by all epilogue warps
        float* al = alpha_s + (iter & 1) * BN;
        for (int i = ew * 32 + lane; i < BN; i += NUM_EPI_WARPS * 32) {
          const int64_t n = tok0 + i;
          // written by the gate kernel while this grid may already run:
          // read through L2, not the read-only cache
          al[i] = (n >= 0 && n < args.N) ? __ldcg(args.alpha + n) : 0.f;
        }
        const int j0 = part * S::PART_COLS;          // first tile column of this warp
        // decode, one chunk per part: the conv states of the first 16 tokens,
        // fetched while the MMAs finish
        constexpr bool PRELOAD = DECODE && NCH == 1 && S::DIL == 1;
        float pre1[PRELOAD ? 16 : 1], pre2[PRELOAD ? 16 : 1], pre3[PRELOAD ? 16 : 1];
        if constexpr (PRELOAD) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int64_t n = tok0 + j0 + i;
            pre1[i] = pre2[i] = pre3[i] = 0.f;
            if (n < args.N) {
              const float* st = args.conv_state + n * 3 * args.d + feat;
              pre3[i] = st[0];
              pre2[i] = st[args.d];
              pre1[i] = st[2 * args.d];
            }
          }
        }
        named_bar_sync(1, NUM_EPI_WARPS * 32);
        const int got = wait_acc();
        const int first_out = -args.m_offset;        // halo columns produce no output
        int pos = (int)((((tok0 + j0) % T) + T) % T);  // sequence position of column j0
        constexpr int NH = S::HALO_T;                 // tokens of conv history
        float sh[NH];                                 // sh[q]: vt of token t-1-q
#pragma unroll
        for (int k = 0; k < NH; ++k) sh[k] = 0.f;
        if (!DECODE && j0 > 0) {
          // the NH columns before this part, recomputed from TMEM
          uint32_t u4[16];
          __syncwarp();
          if (got) {
            tmem_ld16(t_acc + (uint32_t)(j0 - 16), u4);
            tmem_wait16(u4);
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) u4[i] = 0u;
          }
#pragma unroll
          for (int i = 16 - NH; i < 16; ++i) {
            const int pq = (((pos - (16 - i)) % T) + T) % T;
            const float vt = al[j0 - 16 + i] * __uint_as_float(u4[i]);
            if (pq == 0) {
#pragma unroll
              for (int k = 0; k < NH; ++k) sh[k] = 0.f;
            }
#pragma unroll
            for (int k = NH - 1; k > 0; --k) sh[k] = sh[k - 1];
            sh[0] = vt;
          }
        }
#pragma unroll 1
        for (int c = 0; c < NCH; ++c) {
          int hgot = 0;
          if (lane == 0) hgot = wait_bounded(&hfull[hslot], hphase, abort_flag, args.status, args.wait_ns) ? 1 : 0;
          hgot = __shfl_sync(FULL, hgot, 0);
          // h of token jj and feature f of this box: box[jj * BM + f]; the
          // output of the same element replaces it in place
          uint8_t* box = hring + hslot * S::HSLOT_BYTES + part * S::HBOX_BYTES;
          uint16_t* hs = reinterpret_cast<uint16_t*>(box) + quad * 32 + lane;
          uint32_t u[16], un[16];
          __syncwarp();
          if (got) {
            tmem_ld16(t_acc + (uint32_t)(j0 + c * 32), u);
            tmem_ld16(t_acc + (uint32_t)(j0 + c * 32 + 16), un);
            tmem_wait16(u);
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) u[i] = un[i] = 0u;
          }
          const int jb = j0 + c * 32;
          const int64_t nb = tok0 + jb;
          const float4* al4 = reinterpret_cast<const float4*>(al + jb);
          if constexpr (DECODE && S::DIL > 1) {
            // dilated conv: the state holds vt of the 3 dil previous steps
            // (oldest first); 4 tokens' states are loaded before any of them
            // is written back
            constexpr int NS = S::HALO_T;
#pragma unroll
            for (int g4 = 0; g4 < 8; ++g4) {
              if (g4 == 4 && got) tmem_wait16(un);
              float sq[4][NS];
#pragma unroll
              for (int r = 0; r < 4; ++r) {
                const int64_t n = nb + g4 * 4 + r;
#pragma unroll
                for (int k = 0; k < NS; ++k) sq[r][k] = 0.f;
                if (n < args.N) {
                  const float* st = args.conv_state + n * NS * args.d + feat;
#pragma unroll
                  for (int k = 0; k < NS; ++k) sq[r][k] = st[k * args.d];
                }
              }
              const float4 a4 = al4[g4];
              const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
              for (int r = 0; r < 4; ++r) {
                const int jj = g4 * 4 + r;
                const int64_t n = nb + jj;
                const float vt = av[r] * __uint_as_float(jj < 16 ? u[jj] : un[jj - 16]);
                if (n < args.N) {
                  float* st = args.conv_state + n * NS * args.d + feat;
#pragma unroll
                  for (int k = 0; k + 1 < NS; ++k) st[k * args.d] = sq[r][k + 1];
                  st[(NS - 1) * args.d] = vt;
                }
                const float y = fmaf(w.x, sq[r][0], fmaf(w.y, sq[r][S::DIL],
                                                         fmaf(w.z, sq[r][2 * S::DIL], w.w * vt)));
                const float hv = __uint_as_float(((uint32_t)hs[jj * BM]) << 16);
                const float o = hv + vt + silu_tanh(y);
                hs[jj * BM] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
              }
            }
          } else if (DECODE) {
#pragma unroll
            for (int g = 0; g < 2; ++g) {
              // the conv states of 16 tokens, loaded before any of them is
              // written back, so the loads overlap instead of each waiting
              // behind the previous token's stores
              float sa1[16], sa2[16], sa3[16];
              if (PRELOAD && g == 0) {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                  sa1[i] = pre1[PRELOAD ? i : 0];
                  sa2[i] = pre2[PRELOAD ? i : 0];
                  sa3[i] = pre3[PRELOAD ? i : 0];
                }
              } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                  const int64_t n = nb + g * 16 + i;
                  sa1[i] = sa2[i] = sa3[i] = 0.f;
                  if (n < args.N) {
                    const float* st = args.conv_state + n * 3 * args.d + feat;
                    sa3[i] = st[0];
                    sa2[i] = st[args.d];
                    sa1[i] = st[2 * args.d];
                  }
                }
              }
              if (g == 1 && got) tmem_wait16(un);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const float4 a4 = al4[g * 4 + q];
                const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                  const int jj = g * 16 + q * 4 + r;
                  const int64_t n = nb + jj;
                  const float vt = av[r] * __uint_as_float(g == 0 ? u[q * 4 + r] : un[q * 4 + r]);
                  const float a1 = sa1[q * 4 + r], a2 = sa2[q * 4 + r], a3 = sa3[q * 4 + r];
                  if (n < args.N) {
                    float* st = args.conv_state + n * 3 * args.d + feat;
                    st[0] = a2;
                    st[args.d] = a1;
                    st[2 * args.d] = vt;
                  }
                  const float y = fmaf(w.x, a3, fmaf(w.y, a2, fmaf(w.z, a1, w.w * vt)));
                  const float hv = __uint_as_float(((uint32_t)hs[jj * BM]) << 16);
                  const float o = hv + vt + silu_tanh(y);
                  hs[jj * BM] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
                }
              }
            }
          } else if (pos + 32 <= T && pos != 0) {
            // no sequence starts inside the chunk: no per-token checks
            conv_group16<false, S::DIL>(u, al4, hs, w, sh, pos, T);
            if (got) tmem_wait16(un);
            conv_group16<false, S::DIL>(un, al4 + 4, hs + 16 * BM, w, sh, pos, T);
            pos += 32;
            if (pos == T) pos = 0;
          } else {
            conv_group16<true, S::DIL>(u, al4, hs, w, sh, pos, T);
            if (got) tmem_wait16(un);
            conv_group16<true, S::DIL>(un, al4 + 4, hs + 16 * BM, w, sh, pos, T);
          }
          if constexpr (S::KEEP_V) {
            // v itself, for the backward: the warp's 32 tokens x 32 features
            // go through its staging buffer (row = token) and out in one
            // tiled store by lane 1 (its own bulk groups); the halo tokens of
            // a tile are stored by the tile that owns them
            uint8_t* vb = kvbuf + ew * (32 * 32 * 4);
            if (lane == 1) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
            __syncwarp();  // the previous store has read the buffer
            float* vrow = reinterpret_cast<float*>(vb) + lane;
#pragma unroll
            for (int i = 0; i < 32; ++i) vrow[i * 32] = __uint_as_float(i < 16 ? u[i] : un[i - 16]);
            fence_async_shared();
            __syncwarp();
            if (lane == 1 && got) {
              const int vx = args.d + f0 + quad * 32;
              if (jb < first_out)
                tma_store_2d(&tmV29, vb + first_out * 128, vx, (int)(nb + first_out));
              else
                tma_store_2d(&tmV, vb, vx, (int)nb);
            }
          }
          // the part's four warps have written the box: one thread stores it
          fence_async_shared();
          named_bar_sync(2 + part, 128);
          if (ew == part * 4 && lane == 0) {
            if (hgot && got) {
              if (jb < first_out) {
                // the first tokens of the tile are the conv halo of the
                // previous tile: store from the first output token on
                tma_store_2d(&tmO29, box + first_out * BM * 2, f0, (int)(nb + first_out));
              } else {
                tma_store_2d(&tmO, box, f0, (int)nb);
              }
            } else {
              asm volatile("cp.async.bulk.commit_group;" ::: "memory");  // keep one group per chunk
            }
            // the previous chunk's store has read its box: release that slot
            // (this one is released after the next chunk, off the critical path)
            asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
            if (pending_slot >= 0) mbar_arrive(&hempty[pending_slot]);
            pending_slot = (int)hslot;
          }
          if (++hslot == (uint32_t)S::HSLOTS) {
            hslot = 0;
            hphase ^= 1u;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      // this CTA's accumulator rows are read: release them to the leader's MMA
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if constexpr (S::KEEP_V) {  // v's staging buffers read before the CTA exits
      if (lane == 1) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
    }
    // output boxes of pass V fully written before the CTA exits
    if (VPASS && ew == part * 4 && lane == 0) {
      // the stores have read their boxes; their writes complete with the grid
      asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
      if (pending_slot >= 0) mbar_arrive(&hempty[pending_slot]);
    }
  }

  tc_fence_before();
  __syncwarp();
  cluster_sync();  // the pair's MMAs, loads and reads are all done
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, S::TMEM_COLS);
  }
}

// alpha of every token from the gate partials of pass K, TPT lanes per token
// (a fixed order: lane-strided sums, then a butterfly over the TPT lanes):
// alpha = sigmoid(<h, k> r_h r_k / sqrt(d)), r_x = (mean(x^2) + eps)^(-1/2).
// Few tokens (decode) take a warp each; many take a thread each, which keeps
// more tokens' loads in flight.
constexpr int GATE_THREADS = 256;
template <int TPT>
__global__ void __launch_bounds__(GATE_THREADS) gate_from_partials_kernel(
    const float4* __restrict__ part, int n_part, int64_t N, int d, float* __restrict__ alpha,
    float* __restrict__ alpha_copy) {
  allow_dependents();
  wait_prior_grid();  // the partials of pass K
  const int sub = threadIdx.x % TPT;
  const int64_t n = (int64_t)blockIdx.x * (GATE_THREADS / TPT) + threadIdx.x / TPT;
  float kk = 0.f, hk = 0.f, hh = 0.f;
  if (n < N) {
    const float4* pr = part + n * n_part;
    for (int i = sub; i < n_part; i += TPT) {
      const float4 q = __ldcg(pr + i);  // written by pass K during this grid's lifetime
      kk += q.x;
      hk += q.y;
      hh += q.z;
    }
  }
#pragma unroll
  for (int o = TPT / 2; o > 0; o >>= 1) {  // every lane takes part in the shuffles
    kk += __shfl_xor_sync(0xffffffffu, kk, o);
    hk += __shfl_xor_sync(0xffffffffu, hk, o);
    hh += __shfl_xor_sync(0xffffffffu, hh, o);
  }
  if (n >= N || sub != 0) return;
  const float invd = 1.0f / (float)d;
  const float rh = rsqrtf(hh * invd + RMS_EPS), rk = rsqrtf(kk * invd + RMS_EPS);
  const float a = 1.0f / (1.0f + expf(-(hk * rh * rk * rsqrtf((float)d))));
  alpha[n] = a;
  if (alpha_copy != nullptr) alpha_copy[n] = a;
}


template <int BN, int STAGES, int MODE, int KCH>
int launch_pass(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& th,
                const CUtensorMap& to, const CUtensorMap& to29, const CUtensorMap& tv,
                const CUtensorMap& tv29, const TcArgs& a, cudaStream_t s, bool pdl) {
  using S = TcShape<BN, STAGES, MODE, KCH>;
  auto kern = tc_fused_kernel<BN, STAGES, MODE, KCH>;
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return ENGRAM_ERR_CUDA;
  if (!configured[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)S::SMEM) !=
        cudaSuccess)
      return ENGRAM_ERR_CUDA;
    configured[dev] = true;
  }
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // one CTA pair per two SMs, each pair walking its tiles
  const int tiles = a.num_m_tiles * a.num_n_tiles;
  const int pairs = tiles < sms / 2 ? tiles : sms / 2;
  if (pairs <= 0) return ENGRAM_OK;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(S::NUM_THREADS);
  cfg.dynamicSmemBytes = S::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return ck(cudaLaunchKernelEx(&cfg, kern, ta, tb, th, to, to29, tv, tv29, a));
}

// STAGES_VKV: operand stages of pass V when it also keeps v (its staging
// buffers take the room of one stage on the wide tiles)
template <int BN, int STAGES_K, int STAGES_V, int STAGES_VKV, int KCH>
int run_layer(const __nv_bfloat16* e, const __nv_bfloat16* h, const __nv_bfloat16* Wk,
              const __nv_bfloat16* Wv, const float* conv_w, float* conv_state, __nv_bfloat16* out,
              float* alpha_saved, float* kv_save, const float* gg, int dil, int64_t N, int T,
              int d, int E, float4* part, float* alpha, bool chained, bool gate_only, bool stall,
              cudaStream_t s) {
  // Each CTA of a pair loads 128 rows of A and BN/2 rows of B per stage.
  // pass K: A = e (256 tokens per pair tile), B = W_k (BN features)
  CUtensorMap ta_k, tb_k, ta_v, tb_v, th, to, to29;
  if (!make_tmap_k(&ta_k, e, (uint64_t)E, (uint64_t)N, BM, KCH)) return ENGRAM_ERR_CUDA;
  if (!make_tmap_k(&tb_k, Wk, (uint64_t)E, (uint64_t)d, BN / 2, KCH)) return ENGRAM_ERR_CUDA;
  // pass V: A = W_v (256 features per pair tile), B = e (BN tokens);
  // h in boxes of 32 tokens x 128 features
  if (!make_tmap_k(&ta_v, Wv, (uint64_t)E, (uint64_t)d, BM, KCH)) return ENGRAM_ERR_CUDA;
  if (!make_tmap_k(&tb_v, e, (uint64_t)E, (uint64_t)N, BN / 2, KCH)) return ENGRAM_ERR_CUDA;
  if (!make_tmap(&th, h, (uint64_t)d, (uint64_t)N, BM, 32, CU_TENSOR_MAP_SWIZZLE_NONE))
    return ENGRAM_ERR_CUDA;
  // out in the same boxes; a shorter box skips the halo tokens of a tile
  // (3 dil: the conv's history)
  const int halo = 3 * dil;
  if (!make_tmap(&to, out, (uint64_t)d, (uint64_t)N, BM, 32, CU_TENSOR_MAP_SWIZZLE_NONE))
    return ENGRAM_ERR_CUDA;
  if (!make_tmap(&to29, out, (uint64_t)d, (uint64_t)N, BM, 32 - halo, CU_TENSOR_MAP_SWIZZLE_NONE))
    return ENGRAM_ERR_CUDA;
  TcArgs a;
  a.num_k_tiles = E / (BK * KCH);
  a.N = N;
  a.T = T;
  a.d = d;
  a.n_part = TcShape<BN, STAGES_K, MODE_GATE_PARTIAL, KCH>::PARTS * (d / BN);
  a.h = h;
  a.out = out;
  a.part = part;
  a.conv_w = reinterpret_cast<const float4*>(conv_w);
  a.conv_state = conv_state;
  a.alpha_out = alpha_saved;
  a.alpha = nullptr;
  a.kv_save = conv_state == nullptr ? kv_save : nullptr;
  a.gg = gg;
  a.status = status_ptr();
  a.wait_ns = stall ? TEST_WAIT_LIMIT_NS : WAIT_LIMIT_NS;
  a.stall = stall ? 1 : 0;
  // pass K: gate partials, pair tiles of 256 tokens x BN features
  a.num_n_tiles = d / BN;
  a.m_stride = 2 * BM;
  a.m_offset = 0;
  a.num_m_tiles = (int)((N + 2 * BM - 1) / (2 * BM));
  // pass K starts early only behind this call's own gather; as the call's
  // first kernel it keeps plain stream order with the caller's work
  // pass K writes no output; when k is kept, the output-map slot carries the
  // map of the saved k (fp32 [N, 2d], boxes of 32 x 32, 128-byte swizzled)
  CUtensorMap tkv = to;
  if (a.kv_save != nullptr &&
      !make_tmap_f32(&tkv, a.kv_save, (uint64_t)(2 * d), (uint64_t)N, 32, 32,
                     CU_TENSOR_MAP_SWIZZLE_128B))
    return ENGRAM_ERR_CUDA;
  int rc = gg != nullptr
               ? launch_pass<BN, STAGES_K, MODE_GATE_SCALED, KCH>(ta_k, tb_k, th, tkv, to29, to,
                                                                  to29, a, s, chained)
               : launch_pass<BN, STAGES_K, MODE_GATE_PARTIAL, KCH>(ta_k, tb_k, th, tkv, to29, to,
                                                                   to29, a, s, chained);
  if (rc) return rc;
  {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const bool warp_per_token = N * 32 <= (int64_t)sms * 2048;  // one wave of the GPU
    const int tok_per_block = warp_per_token ? GATE_THREADS / 32 : GATE_THREADS;
    const dim3 grid((unsigned)((N + tok_per_block - 1) / tok_per_block));
    rc = warp_per_token
             ? launch_pdl(gate_from_partials_kernel<32>, grid, dim3(GATE_THREADS), 0, s,
                          (const float4*)part, a.n_part, N, d, alpha, alpha_saved)
             : launch_pdl(gate_from_partials_kernel<1>, grid, dim3(GATE_THREADS), 0, s,
                          (const float4*)part, a.n_part, N, d, alpha, alpha_saved);
    if (rc) return rc;
  }
  if (gate_only) return ENGRAM_OK;  // the pre-conv norm's path takes over from alpha
  a.alpha = alpha;
  // pass V: pair tiles of 256 features x BN tokens.  Whole sequences: the
  // token tiles overlap by the conv's history (recomputed); decode: plain
  // tiles.
  a.num_n_tiles = d / (2 * BM);
  if (conv_state != nullptr) {
    a.m_stride = BN;
    a.m_offset = 0;
  } else {
    a.m_stride = BN - halo;
    a.m_offset = -halo;
  }
  a.num_m_tiles = (int)((N + a.m_stride - 1) / a.m_stride);
  constexpr int D3 = MODE_V_DILATED;
  if (conv_state != nullptr)
    return dil == 3 ? launch_pass<BN, STAGES_V, MODE_VALUE_DECODE | D3, KCH>(
                          ta_v, tb_v, th, to, to29, to, to29, a, s, true)
                    : launch_pass<BN, STAGES_V, MODE_VALUE_DECODE, KCH>(ta_v, tb_v, th, to, to29, to,
                                                                        to29, a, s, true);
  if (a.kv_save != nullptr) {
    // v into the saved [k | v] rows: boxes of 32 features x 32 tokens, and a
    // shorter box that skips a tile's conv halo
    CUtensorMap tv, tv29;
    if (!make_tmap_f32(&tv, a.kv_save, (uint64_t)(2 * d), (uint64_t)N, 32, 32,
                       CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_tmap_f32(&tv29, a.kv_save, (uint64_t)(2 * d), (uint64_t)N, 32, 32 - halo,
                       CU_TENSOR_MAP_SWIZZLE_NONE))
      return ENGRAM_ERR_CUDA;
    return dil == 3 ? launch_pass<BN, STAGES_VKV, MODE_VALUE_CONV_KV | D3, KCH>(
                          ta_v, tb_v, th, to, to29, tv, tv29, a, s, true)
                    : launch_pass<BN, STAGES_VKV, MODE_VALUE_CONV_KV, KCH>(ta_v, tb_v, th, to, to29,
                                                                           tv, tv29, a, s, true);
  }
  return dil == 3 ? launch_pass<BN, STAGES_V, MODE_VALUE_CONV | D3, KCH>(ta_v, tb_v, th, to, to29,
                                                                         to, to29, a, s, true)
                  : launch_pass<BN, STAGES_V, MODE_VALUE_CONV, KCH>(ta_v, tb_v, th, to, to29, to,
                                                                    to29, a, s, true);
}

inline bool use_wide(int64_t N, int d) { return d % 256 == 0 && N > 4096; }

}  // namespace

namespace {
__global__ void scale_product_kernel(const float* __restrict__ gh, const float* __restrict__ gk,
                                     int d, float* __restrict__ gg) {
  const int f = blockIdx.x * blockDim.x + threadIdx.x;
  if (f < d) gg[f] = gh[f] * gk[f];
}
}  // namespace

int launch_scale_product(const float* gh, const float* gk, int d, float* gg, cudaStream_t s) {
  scale_product_kernel<<<(unsigned)((d + 255) / 256), 256, 0, s>>>(gh, gk, d, gg);
  return ck(cudaGetLastError());
}

int tc_supported(int d, int E, int M) {
  return M == 1 && E % BK == 0 && E >= BK && d % (2 * BM) == 0 && d >= 2 * BM;
}

size_t tc_forward_ws_bytes(int64_t N, int d, int E) {
  (void)E;
  const int BN = use_wide(N, d) ? 256 : 64;
  const size_t part = (size_t)N * 2 * (d / BN) * sizeof(float4);
  return part + (((size_t)N * sizeof(float) + 255) & ~(size_t)255);
}

int launch_forward_tc(const __nv_bfloat16* e, const __nv_bfloat16* h, const __nv_bfloat16* Wk,
                      const __nv_bfloat16* Wv, const float* conv_w, float* conv_state,
                      __nv_bfloat16* out, float* alpha_saved, float* kv_save, const float* gg,
                      int dil, int64_t N, int T, int d, int E, void* ws, size_t ws_bytes,
                      bool chained, const PrenormFwd* pn, bool stall, cudaStream_t s) {
  if (ws_bytes < tc_forward_ws_bytes(N, d, E) || ws == nullptr) return ENGRAM_ERR_WORKSPACE;
  if (N > 0x7fffffffLL - 256) return ENGRAM_ERR_UNSUPPORTED;
  const bool wide = use_wide(N, d);
  const int BN = wide ? 256 : 64;
  float4* part = static_cast<float4*>(ws);
  float* alpha = reinterpret_cast<float*>(static_cast<char*>(ws) +
                                          (size_t)N * 2 * (d / BN) * sizeof(float4));
  // with the pre-conv norm the passes stop at the gate (pass K and alpha)
  const bool gate_only = pn != nullptr;
  int rc;
  if (wide)
    rc = run_layer<256, 6, 5, 4, 1>(e, h, Wk, Wv, conv_w, conv_state, out, alpha_saved, kv_save,
                                    gg, dil, N, T, d, E, part, alpha, chained, gate_only, stall, s);
  // few tokens: each CTA streams long operand rows at a rate set by how many
  // bytes one copy instruction brings, so two K chunks go in each box
  else if (E % (2 * BK) == 0)
    rc = run_layer<64, 4, 3, 3, 2>(e, h, Wk, Wv, conv_w, conv_state, out, alpha_saved, kv_save,
                                   gg, dil, N, T, d, E, part, alpha, chained, gate_only, stall, s);
  else
    rc = run_layer<64, 8, 6, 6, 1>(e, h, Wk, Wv, conv_w, conv_state, out, alpha_saved, kv_save,
                                   gg, dil, N, T, d, E, part, alpha, chained, gate_only, stall, s);
  if (rc || pn == nullptr) return rc;
  return launch_prenorm_tail(*pn, e, Wv, h, conv_w, alpha, conv_state, out, dil, N, T, d, E,
                             stall, s);
}

}  // namespace engram
