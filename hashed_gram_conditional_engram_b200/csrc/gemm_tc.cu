// Plain bf16 GEMMs on the sm_100a tensor cores: C [M x N] fp32 = A . B with
// bf16 operands and fp32 accumulation in TMEM.
//
// The backward of the bf16 layer has three dense contractions with nothing
// around them to fuse (gitcode.csdn.net blog, end-to-end training paragraph:
// the table rows, W_k and W_v all train by backpropagation):
//   [k | v]          = e [W_k; W_v]^T     A = e (K-major), B = W (K-major)
//   [dW_k; dW_v]     = [dk | dv]^T e      A, B MN-major (K = tokens)
//   de               = [dk | dv] [W_k; W_v]  A K-major, B MN-major
// and the pre-conv-norm forward needs v = e W_v^T alone.  The layouts in
// memory are the layer's own (token rows for e, k, v, dk, dv; W [d, E]), so
// the operands reach the tensor cores either K-major or MN-major; the
// instruction descriptor says which, and TMA lands both as 128-byte swizzled
// tiles.  Stacked operands are not materialised: B switches from one tensor
// map to a second one at a row (W_k then W_v), and C switches output blocks
// at a row (dW_k then dW_v).
//
// Pipeline per CTA of a pair (cluster of 2, tcgen05.mma.cta_group::2, a
// 256 x 256 pair tile, K in steps of 64):
//   warp 0      A producer: one lane issues the TMA loads of this CTA's 128
//               rows of A into a ring of stages;
//   warp 1      allocates TMEM (two 256-column accumulators); on the leader
//               one lane issues the MMAs;
//   warps 2-9   epilogue: TMEM -> registers -> a swizzled staging block ->
//               TMA store (fp32), or plain stores for split tiles (below);
//   warp 10     B producer: this CTA's half of the tile's 256 columns.
//
// Scheduling.  Each pair takes units p, p + P, ... of the output's pair
// tiles.  The weight gradient has few output tiles (2d/256 x E/256 = 100 at
// the 27B shape) and a long K (one row per token), so there the k steps of
// every tile are cut into S parts and unit u is part u / tiles of tile
// u % tiles: the pairs at work at any moment all read the same stretch of
// tokens, which stays in L2 while every tile takes its turn on it.  A tile's
// parts are summed in a fixed order: part 0 stores its sum, then part s,
// once the tile's counter shows that all 16 epilogue warps of part s - 1
// have stored, loads the sum so far, adds its own and stores (part s - 1
// ran about one round of units earlier, so the wait is rarely felt).  The
// result therefore does not depend on timing.  Every wait is bounded in
// time; one that runs out sets ENGRAM_STATUS_TIMEOUT and the CTA winds down.
#include "tc_ptx.cuh"

namespace engram {

namespace {

using namespace tc;

constexpr int GN = 256;                       // columns of a pair tile (N of one MMA)
constexpr int G_EPI = 8;                      // epilogue warps
constexpr int G_BP_WARP = 2 + G_EPI;          // B-operand producer
constexpr int G_THREADS = (3 + G_EPI) * 32;
constexpr int G_STAGES = 6;
constexpr int G_A_BYTES = BM * BK * 2;        // 128 rows x 64 k
constexpr int G_B_BYTES = (GN / 2) * BK * 2;  // this CTA's 128 of the tile's columns x 64 k
constexpr int G_STG = 32 * 32 * 4;            // a warp's 32 x 32 fp32 staging block
constexpr int G_BUFS = 1;                     // staging blocks per warp (a seventh operand
                                              // stage would not fit; six stages and one
                                              // block measured faster than five and two)
constexpr int G_MN_LBO = BK * 128;            // MN-major tiles: next 64 M/N elements
constexpr size_t G_SMEM =
    (size_t)G_STAGES * (G_A_BYTES + G_B_BYTES) + (size_t)G_EPI * G_BUFS * G_STG + 256;
static_assert(G_SMEM <= 232448, "shared memory");

struct GemmArgs {
  int m_tiles, n_tiles;  // pair tiles of 256 x 256
  int k_iters;           // K in steps of 64
  int b_split;           // B map row (K-major: n; MN-major: k) where the second map takes over
  int c_split;           // output row where the second output block takes over
  int splits;            // parts S of each tile's k steps (1: whole tiles)
  float* c0;             // output blocks (row-major, ldc floats per row) for the plain stores
  float* c1;
  int64_t ldc;
  int64_t c_rows;        // output rows over both blocks
  int c_cols;            // output columns (a multiple of 32)
  int* flags;            // S > 1: a counter per tile, zero at launch
  unsigned int* status;
  uint64_t wait_ns;      // limit of every bounded wait
  int stall;             // ENGRAM_TEST_STALL: the B producer issues nothing
};

// One unit of a pair's work: part `split` of a tile, k steps [kb, ke).
struct GUnit {
  int tile, split, kb, ke;
};

// The pair's units in order, the same walk in every role.
struct GWalk {
  int cur, end, step, tiles, KT, S;
  __device__ GWalk(const GemmArgs& a, int pair, int npairs) {
    tiles = a.m_tiles * a.n_tiles;
    KT = a.k_iters;
    S = a.splits;
    cur = pair;
    end = tiles * S;
    step = npairs;
  }
  __device__ bool next(GUnit& u) {
    if (cur >= end) return false;
    u.split = cur / tiles;
    u.tile = cur - u.split * tiles;
    u.kb = (int)((int64_t)u.split * KT / S);
    u.ke = (int)((int64_t)(u.split + 1) * KT / S);
    cur += step;
    return true;
  }
};

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

template <bool A_MN, bool B_MN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(G_THREADS, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                   const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmC0,
                   const __grid_constant__ CUtensorMap tmC1, const __grid_constant__ GemmArgs a) {
  constexpr uint32_t STAGE_TX = G_A_BYTES + G_B_BYTES;
  // fp32 accumulate, bf16 A and B, A / B major-ness, N >> 3 at bit 17,
  // M >> 4 at bit 24 (M = 256 over the pair)
  constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((A_MN ? 1u : 0u) << 15) |
                             ((B_MN ? 1u : 0u) << 16) | ((uint32_t)(GN >> 3) << 17) |
                             ((uint32_t)((2 * BM) >> 4) << 24);
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {  // swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) atomicOr(a.status, ENGRAM_STATUS_TIMEOUT);
    return;
  }
  uint8_t* sA = smem;
  uint8_t* sB = smem + G_STAGES * G_A_BYTES;
  uint8_t* stg = sB + G_STAGES * G_B_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(stg + G_EPI * G_BUFS * G_STG);
  uint64_t* full = bars;
  uint64_t* empty = bars + G_STAGES;
  uint64_t* tfull = bars + 2 * G_STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(drain + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = (int)(blockIdx.x >> 1), npairs = (int)(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < G_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int c = 0; c < 2; ++c) {
      mbar_init(&tfull[c], 1);
      mbar_init(&tempty[c], 2 * G_EPI);  // epilogue warps of both CTAs
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB0);
    prefetch_tmap(&tmB1);
    prefetch_tmap(&tmC0);
    prefetch_tmap(&tmC1);
  }
  if (warp == 1) {
    __syncwarp();
    tmem_alloc_pair(tmem_slot, 2 * GN);
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync();  // both CTAs' barriers exist before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 || warp == G_BP_WARP) {
    // ------------------------------------------------------------ operand producers
    // Warp 0 loads A and posts the stage's expected bytes (both CTAs' A and
    // B boxes count on the leader's barrier); warp 10 loads B into the same
    // stages in the same order (with ENGRAM_TEST_STALL it issues nothing, so
    // the stages never fill and the waits run out).
    if (lane == 0 && !(warp == G_BP_WARP && a.stall)) {
      const bool isA = warp == 0;
      GWalk w(a, pair, npairs);
      GUnit u;
      int stage = 0;
      uint32_t phase = 0, issued = 0;
      bool ok = true;
      while (ok && w.next(u)) {
        const int mi = u.tile / a.n_tiles, ni = u.tile - mi * a.n_tiles;
        const int m0 = mi * (2 * BM) + (int)rank * BM;      // this CTA's rows of A
        const int n0 = ni * GN + (int)rank * (GN / 2);      // this CTA's columns of B
        for (int kt = u.kb; kt < u.ke; ++kt) {
          if (!wait_bounded(&empty[stage], phase ^ 1u, abort_flag, a.status, a.wait_ns)) {
            ok = false;
            break;
          }
          const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
          if (isA) {
            if (leader) mbar_expect_tx(&full[stage], 2 * STAGE_TX);
            if (A_MN)
              tma_load_3d_pair(sA + stage * G_A_BYTES, &tmA, fb, 0, kt * BK, m0 / BK);
            else
              tma_load_3d_pair(sA + stage * G_A_BYTES, &tmA, fb, 0, m0, kt);
          } else {
            int c1 = B_MN ? kt * BK : n0;
            const CUtensorMap* mb = &tmB0;
            if (c1 >= a.b_split) {
              c1 -= a.b_split;
              mb = &tmB1;
            }
            if (B_MN)
              tma_load_3d_pair(sB + stage * G_B_BYTES, mb, fb, 0, c1, n0 / BK);
            else
              tma_load_3d_pair(sB + stage * G_B_BYTES, mb, fb, 0, c1, kt);
          }
          ++issued;
          if (++stage == G_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // every copy issued for the pair lands before the leader leaves (the
      // peer waits for the leader at the closing cluster barrier)
      if (isA && leader) {
        for (int s = 0; s < G_STAGES; ++s) {
          const uint32_t n_s = issued > (uint32_t)s ? (issued - 1 - s) / G_STAGES + 1 : 0;
          if (n_s > 0) wait_drain(&full[s], (n_s - 1) & 1u, a.wait_ns);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (leader && lane == 0) {
      GWalk w(a, pair, npairs);
      GUnit u;
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      while (ok && w.next(u)) {
        if (!wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, a.status, a.wait_ns)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * GN);
        for (int kt = u.kb; kt < u.ke; ++kt) {
          if (!wait_bounded(&full[stage], phase, abort_flag, a.status, a.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * G_A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * G_B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / UMMA_K; ++k) {
            // K-major: the next 16 k are 32 bytes along the row; MN-major:
            // 16 rows of 128 bytes further
            const uint64_t da = A_MN ? sw128_mn_desc(a0 + k * UMMA_K * 128, G_MN_LBO)
                                     : sw128_desc(a0 + k * UMMA_K * 2);
            const uint64_t db = B_MN ? sw128_mn_desc(b0 + k * UMMA_K * 128, G_MN_LBO)
                                     : sw128_desc(b0 + k * UMMA_K * 2);
            umma_bf16_pair(d_tmem, da, db, IDESC, (kt > u.kb || k > 0) ? 1u : 0u);
          }
          umma_commit_pair_both(&empty[stage]);
          if (++stage == G_STAGES) {
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
      wait_drain(drain, 0, a.wait_ns);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;
    const int quad = warp & 3;  // TMEM lanes 32 quad .. of this warp
    const int part = ew >> 2;   // which 128 of the tile's 256 columns
    uint8_t* my_stg = stg + ew * G_BUFS * G_STG;
    GWalk w(a, pair, npairs);
    GUnit u;
    int acc = 0;
    uint32_t acc_phase = 0, nstore = 0;
    while (w.next(u)) {
      const int mi = u.tile / a.n_tiles, ni = u.tile - mi * a.n_tiles;
      const int r0 = mi * (2 * BM) + (int)rank * BM + quad * 32;  // the warp's first row
      const int col0 = ni * GN + part * (GN / 2);
      int ok = 0;
      if (lane == 0) ok = wait_bounded(&tfull[acc], acc_phase, abort_flag, a.status, a.wait_ns) ? 1 : 0;
      ok = __shfl_sync(FULL, ok, 0);
      tc_fence_after();
      if (!ok) break;
      const uint32_t t_row =
          tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * GN + part * (GN / 2));
      if (a.splits == 1) {
        // the whole tile: 32 x 32 blocks through the staging buffers, one
        // tiled store each (rows and columns outside C are not written)
        int rr = r0;
        const CUtensorMap* mc = &tmC0;
        if (rr >= a.c_split) {
          rr -= a.c_split;
          mc = &tmC1;
        }
#pragma unroll 1
        for (int c = 0; c < GN / 2 / 32; ++c) {
          float v[32];
          tmem_ld32(t_row + c * 32, v);
          uint8_t* buf = my_stg + (nstore % G_BUFS) * G_STG;
          // the store issued G_BUFS blocks ago has read this buffer
          if (lane == 0) asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(G_BUFS - 1) : "memory");
          __syncwarp();
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4*>(buf + lane * 128 + ((q ^ (lane & 7)) * 16)) =
                make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          fence_async_shared();
          __syncwarp();
          if (lane == 0) tma_store_2d(mc, buf, col0 + c * 32, rr);
          ++nstore;
        }
      } else {
        // part s of a split tile: wait for part s - 1 of this tile, then for
        // each 32 x 32 block, stage it (the same swizzled layout as above)
        // and move it in 16-byte pieces, four 128-byte rows per instruction:
        // loaded (the sum so far), added to, stored
        int good = 1;
        if (u.split > 0) {
          if (lane == 0) {
            const int want = 2 * G_EPI * u.split;
            const uint64_t t0 = global_ns();
            while (ld_acquire_gpu(a.flags + u.tile) < want) {
              if (*abort_flag) {
                good = 0;
                break;
              }
              if (global_ns() - t0 > a.wait_ns) {
                *abort_flag = 1;
                atomicOr(a.status, ENGRAM_STATUS_TIMEOUT);
                good = 0;
                break;
              }
              __nanosleep(200);
            }
          }
          good = __shfl_sync(FULL, good, 0);
        }
        uint8_t* buf = my_stg;
#pragma unroll 1
        for (int c = 0; c < GN / 2 / 32; ++c) {
          float v[32];
          tmem_ld32(t_row + c * 32, v);
          __syncwarp();  // the previous block's reads of buf are done
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4*>(buf + lane * 128 + ((q ^ (lane & 7)) * 16)) =
                make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          __syncwarp();
          // lane: 4 columns (16-byte chunk cg) of rows rg, rg + 4, ..., rg + 28
          const int cg = lane & 7, rg = lane >> 3;
          const int col = col0 + c * 32 + cg * 4;
          if (good && col < a.c_cols) {
            float4* gp[8];
            float4 x[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int r = 4 * i + rg;
              const int64_t row = (int64_t)r0 + r;
              gp[i] = row < a.c_rows
                          ? reinterpret_cast<float4*>(
                                (row < a.c_split ? a.c0 + row * a.ldc
                                                 : a.c1 + (row - a.c_split) * a.ldc) + col)
                          : nullptr;
              x[i] = *reinterpret_cast<const float4*>(buf + r * 128 + ((cg ^ (r & 7)) << 4));
            }
            if (u.split > 0) {
              // the sum of parts 0 .. s-1: all eight loads in flight, then the adds
              float4 o[8];
#pragma unroll
              for (int i = 0; i < 8; ++i)
                o[i] = gp[i] != nullptr ? __ldcg(gp[i]) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                x[i].x = o[i].x + x[i].x;
                x[i].y = o[i].y + x[i].y;
                x[i].z = o[i].z + x[i].z;
                x[i].w = o[i].w + x[i].w;
              }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i)
              if (gp[i] != nullptr) __stcg(gp[i], x[i]);
          }
        }
        // publish: all lanes' stores, then one count for this warp
        __syncwarp();
        if (lane == 0 && good) {
          __threadfence();
          atomicAdd(a.flags + u.tile, 1);
        }
      }
      tc_fence_before();
      __syncwarp();
      // this CTA's accumulator rows are read: release them to the leader's MMA
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    // the staging buffers are read before the CTA exits
    if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
  }

  tc_fence_before();
  __syncwarp();
  cluster_sync();  // the pair's MMAs, loads and reads are all done
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 2 * GN);
  }
}

template <bool A_MN, bool B_MN>
int run_gemm(const CUtensorMap& ta, const CUtensorMap& tb0, const CUtensorMap& tb1,
             const CUtensorMap& tc0, const CUtensorMap& tc1, GemmArgs a, cudaStream_t s) {
  auto kern = tc_gemm_kernel<A_MN, B_MN>;
  static bool configured[64] = {false};
  static int max_pairs[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ENGRAM_ERR_CUDA;
  if (!configured[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)G_SMEM) !=
        cudaSuccess)
      return ENGRAM_ERR_CUDA;
    // pairs that fit on the GPU at once: split tiles wait between pairs, so
    // all of them must be resident
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return ENGRAM_ERR_CUDA;
    cudaLaunchConfig_t q = {};
    q.gridDim = dim3((unsigned)(sms & ~1));
    q.blockDim = dim3(G_THREADS);
    q.dynamicSmemBytes = G_SMEM;
    cudaLaunchAttribute qa[1];
    qa[0].id = cudaLaunchAttributeClusterDimension;
    qa[0].val.clusterDim.x = 2;
    qa[0].val.clusterDim.y = 1;
    qa[0].val.clusterDim.z = 1;
    q.attrs = qa;
    q.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kern, &q) != cudaSuccess || clusters <= 0)
      clusters = sms / 2;
    max_pairs[dev] = clusters < sms / 2 ? clusters : sms / 2;
    configured[dev] = true;
  }
  const int tiles = a.m_tiles * a.n_tiles;
  const int P = max_pairs[dev];
  if (a.splits == 0) {
    // parts per tile: the fewest rounds of units per part of the work
    // (rounds / S), each part charged 2% for the extra partial sums it
    // moves through L2 (measured at the 27B shape: S = 5 and 8 equal, 4 and
    // 6 slower, 11 slower still), with at least 8 k steps in a part
    int best = 1;
    double best_cost = (double)((tiles + P - 1) / P) * 1.02;
    const int s_max = a.k_iters / 8 < 32 ? a.k_iters / 8 : 32;
    for (int S = 2; S <= s_max; ++S) {
      const double cost = (double)(((int64_t)S * tiles + P - 1) / P) / S * (1.0 + 0.02 * S);
      if (cost < best_cost - 1e-9) {
        best_cost = cost;
        best = S;
      }
    }
    a.splits = best;
  }
  if (a.splits > 1 &&
      cudaMemsetAsync(a.flags, 0, (size_t)tiles * sizeof(int), s) != cudaSuccess)
    return ENGRAM_ERR_CUDA;
  const int64_t units = (int64_t)tiles * a.splits;
  const int pairs = (int)(units < P ? units : P);
  if (pairs <= 0) return ENGRAM_OK;
  if (a.splits == 1) {
    kern<<<dim3(2 * pairs), dim3(G_THREADS), G_SMEM, s>>>(ta, tb0, tb1, tc0, tc1, a);
    return ck(cudaGetLastError());
  }
  // split tiles: a part waits for the part before it, run by another pair,
  // so every pair must be resident together: a cooperative launch starts
  // them together or not at all
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(G_THREADS);
  cfg.dynamicSmemBytes = G_SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return ck(cudaLaunchKernelEx(&cfg, kern, ta, tb0, tb1, tc0, tc1, a));
}

GemmArgs gemm_args(int64_t M, int64_t Nc, int64_t K, bool stall) {
  GemmArgs a = {};
  a.m_tiles = (int)((M + 2 * BM - 1) / (2 * BM));
  a.n_tiles = (int)((Nc + GN - 1) / GN);
  a.k_iters = (int)((K + BK - 1) / BK);
  a.b_split = 0x7fffffff;
  a.c_split = 0x7fffffff;
  a.splits = 1;
  a.status = status_ptr();
  a.wait_ns = stall ? TEST_WAIT_LIMIT_NS : WAIT_LIMIT_NS;
  a.stall = stall ? 1 : 0;
  return a;
}

}  // namespace

int gemm_supported(int64_t N, int d, int E) {
  return d % (2 * BM) == 0 && d > 0 && E % BK == 0 && E > 0 && N >= 0 && N <= 0x7fffffffLL - 2 * BM;
}

int launch_gemm_kv(const __nv_bfloat16* e, const __nv_bfloat16* Wk, const __nv_bfloat16* Wv,
                   int64_t N, int d, int E, float* C, int64_t ldc, cudaStream_t s, bool stall) {
  if (!gemm_supported(N, d, E) || ldc % 4 != 0) return ENGRAM_ERR_UNSUPPORTED;
  if (N == 0) return ENGRAM_OK;
  const bool both = Wk != nullptr;
  const int cols = both ? 2 * d : d;
  CUtensorMap ta, tb0, tb1, tc0;
  if (!make_tmap_k(&ta, e, (uint64_t)E, (uint64_t)N, BM, 1) ||
      !make_tmap_k(&tb0, both ? Wk : Wv, (uint64_t)E, (uint64_t)d, GN / 2, 1) ||
      !make_tmap_k(&tb1, Wv, (uint64_t)E, (uint64_t)d, GN / 2, 1) ||
      !make_tmap_f32_ld(&tc0, C, (uint64_t)cols, (uint64_t)N, (uint64_t)ldc, 32, 32,
                        CU_TENSOR_MAP_SWIZZLE_128B))
    return ENGRAM_ERR_CUDA;
  GemmArgs a = gemm_args(N, cols, E, stall);
  if (both) a.b_split = d;  // columns d.. of C come from W_v
  a.c0 = C;
  a.ldc = ldc;
  a.c_rows = N;
  a.c_cols = cols;
  return run_gemm<false, false>(ta, tb0, tb1, tc0, tc0, a, s);
}

size_t gemm_dw_ws_bytes(int d, int E) {
  const int tiles = ((2 * d + 2 * BM - 1) / (2 * BM)) * ((E + GN - 1) / GN);
  return ((size_t)tiles * sizeof(int) + 255) & ~(size_t)255;
}

int launch_gemm_dw(const __nv_bfloat16* dkv, const __nv_bfloat16* e, int64_t N, int d, int E,
                   float* dWk, float* dWv, void* ws, cudaStream_t s, bool stall) {
  if (!gemm_supported(N, d, E)) return ENGRAM_ERR_UNSUPPORTED;
  if (N == 0) {  // no tokens: the gradients are zero
    if (cudaMemsetAsync(dWk, 0, (size_t)d * E * 4, s) != cudaSuccess ||
        cudaMemsetAsync(dWv, 0, (size_t)d * E * 4, s) != cudaSuccess)
      return ENGRAM_ERR_CUDA;
    return ENGRAM_OK;
  }
  // A = [dk | dv]^T: element (token, f) at token * 2d + f; B = e: (token, c)
  // at token * E + c; both MN-major over K = tokens
  CUtensorMap ta, tb, tc0, tc1;
  if (!make_tmap_mn(&ta, dkv, (uint64_t)(2 * d), (uint64_t)N, (uint64_t)(2 * d), BK, BM / BK) ||
      !make_tmap_mn(&tb, e, (uint64_t)E, (uint64_t)N, (uint64_t)E, BK, GN / 2 / BK) ||
      !make_tmap_f32(&tc0, dWk, (uint64_t)E, (uint64_t)d, 32, 32, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_f32(&tc1, dWv, (uint64_t)E, (uint64_t)d, 32, 32, CU_TENSOR_MAP_SWIZZLE_128B))
    return ENGRAM_ERR_CUDA;
  GemmArgs a = gemm_args(2 * d, E, N, stall);
  a.c_split = d;  // rows d.. are dW_v
  a.splits = 0;   // chosen at launch
  a.c0 = dWk;
  a.c1 = dWv;
  a.ldc = E;
  a.c_rows = 2 * (int64_t)d;
  a.c_cols = E;
  a.flags = static_cast<int*>(ws);
  return run_gemm<true, true>(ta, tb, tb, tc0, tc1, a, s);
}

int launch_gemm_de(const __nv_bfloat16* dkv, const __nv_bfloat16* Wk, const __nv_bfloat16* Wv,
                   int64_t N, int d, int E, float* de, cudaStream_t s, bool stall) {
  if (!gemm_supported(N, d, E)) return ENGRAM_ERR_UNSUPPORTED;
  if (N == 0) return ENGRAM_OK;
  // A = [dk | dv] (K-major over K = 2d); B = [W_k; W_v]: (f, c) at f * E + c,
  // MN-major, W_v from k = d on
  CUtensorMap ta, tb0, tb1, tc0;
  if (!make_tmap_k(&ta, dkv, (uint64_t)(2 * d), (uint64_t)N, BM, 1) ||
      !make_tmap_mn(&tb0, Wk, (uint64_t)E, (uint64_t)d, (uint64_t)E, BK, GN / 2 / BK) ||
      !make_tmap_mn(&tb1, Wv, (uint64_t)E, (uint64_t)d, (uint64_t)E, BK, GN / 2 / BK) ||
      !make_tmap_f32(&tc0, de, (uint64_t)E, (uint64_t)N, 32, 32, CU_TENSOR_MAP_SWIZZLE_128B))
    return ENGRAM_ERR_CUDA;
  GemmArgs a = gemm_args(N, E, 2 * d, stall);
  a.b_split = d;
  a.c0 = de;
  a.ldc = E;
  a.c_rows = N;
  a.c_cols = E;
  return run_gemm<false, true>(ta, tb0, tb1, tc0, tc0, a, s);
}

}  // namespace engram
