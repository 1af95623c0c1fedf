// Retrieval kernels: fused compress + suffix n-gram + multi-head hash, and the
// row gather that builds e_t.
//
// Method: discuss.deepseek.club 二.1 (1) (vocabulary projection, multi-head
// hashing into per-head tables, concatenation of the retrieved rows);
// gitcode.csdn.net blog "Engram 到底怎么工作的", 第一步 / 第二步 (the last two and
// last three tokens address several slots of a large table).
#include "internal.cuh"

namespace engram {

namespace {

constexpr unsigned FULL = 0xffffffffu;

// x mod P for P < 2^63 odd, by Barrett reduction (P. Barrett, CRYPTO '86):
// with mu = floor((2^64-1)/P) = floor(2^64/P) (P does not divide 2^64),
// q = floor(x*mu / 2^64) is floor(x/P) or one less, so one conditional
// subtraction finishes the remainder.
__device__ __forceinline__ uint64_t mod_prime(uint64_t x, uint64_t P, uint64_t mu) {
  uint64_t q = __umul64hi(x, mu);
  uint64_t r = x - q * P;
  return r >= P ? r - P : r;
}

// One 16-byte piece of a table row.  Rows are read once and 160 or 256 bytes
// long at 32-byte alignment: no L1 allocation, and the L2 asked to fetch
// 64-byte sector pairs on a miss instead of whole 128-byte lines (a 160-byte
// row spans two lines: 256 bytes from DRAM at line granularity, 192 at 64).
__device__ __forceinline__ uint4 ld_row_piece(const uint4* p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.L2::64B.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
  return v;
}

// Compressed id of flat token m, PAD for m < 0; -1 for a raw id out of range.
__device__ __forceinline__ int32_t token_cid(const int32_t* __restrict__ proj,
                                             const int32_t* __restrict__ ids, int64_t m,
                                             int32_t V_raw, int32_t pad) {
  if (m < 0) return pad;
  int32_t x = __ldg(ids + m);
  if (x < 0 || x >= V_raw) return -1;
  return __ldg(proj + x);
}

// TPT threads per token (J / HPT rounded up to a power of two), HPT heads
// each: four (one 16-byte store) when J is a multiple of 4, else two (an
// 8-byte store; J = 2K is even); a warp covers 32 / TPT consecutive tokens
// in flat order.  c_{t-1} and c_{t-2} travel from the lanes of the previous
// tokens by warp shuffles; the lanes of a warp's first two tokens fetch the
// tokens before the warp themselves.
template <int HPT>
__global__ void __launch_bounds__(256) hash_kernel(const __grid_constant__ HeadParams hp,
                                                   const int32_t* __restrict__ proj,
                                                   const int32_t* __restrict__ ids, int64_t N,
                                                   int T, int tpt,
                                                   int32_t* __restrict__ ngram_state,
                                                   int32_t* __restrict__ idx,
                                                   unsigned int* status) {
  allow_dependents();  // a programmatically launched successor waits for this grid anyway
  const int64_t gt = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int lane = threadIdx.x & 31;
  const int q = lane % tpt;             // which HPT heads
  const int64_t n = gt / tpt;           // token
  const int32_t pad = hp.V_c;
  const bool live = n < N;

  int32_t c0 = live ? token_cid(proj, ids, n, hp.V_raw, pad) : pad;
  int32_t c1 = __shfl_up_sync(FULL, c0, tpt);
  int32_t c2 = __shfl_up_sync(FULL, c0, 2 * tpt);
  if (!live) return;
  const int tk = lane / tpt;            // token index within the warp
  if (tk == 0) c1 = token_cid(proj, ids, n - 1, hp.V_raw, pad);
  if (tk <= 1) c2 = token_cid(proj, ids, n - 2, hp.V_raw, pad);

  if (ngram_state != nullptr) {
    // decode: one token per sequence, history from the rolling state
    c1 = ngram_state[2 * n + 0];
    c2 = ngram_state[2 * n + 1];
    __syncwarp(__activemask());
    if (q == 0) {
      ngram_state[2 * n + 0] = c0;
      ngram_state[2 * n + 1] = c1;
    }
  } else {
    const int t = (int)(n % T);
    if (t < 1) c1 = pad;
    if (t < 2) c2 = pad;
  }
  if (c0 < 0 && q == 0) atomicOr(status, ENGRAM_STATUS_BAD_ID);
  const bool bad2 = (c0 < 0) | (c1 < 0);
  const bool bad3 = bad2 | (c2 < 0);

  const uint64_t g0 = (uint64_t)(uint32_t)c0, g1 = (uint64_t)(uint32_t)c1,
                 g2 = (uint64_t)(uint32_t)c2;
  const int j0 = HPT * q;
  if (j0 >= hp.J) return;  // padding lane of a token (J / HPT not a power of two)
  int32_t s[HPT];
#pragma unroll
  for (int u = 0; u < HPT; ++u) {
    const int j = j0 + u;
    uint64_t x = g0 * hp.mult[j][0];
    x ^= g1 * hp.mult[j][1];
    const bool tri = j >= hp.K;
    if (tri) x ^= g2 * hp.mult[j][2];
    const bool bad = tri ? bad3 : bad2;
    s[u] = bad ? -1 : (int32_t)mod_prime(x, hp.P[j], hp.mu[j]);
  }
  if constexpr (HPT == 4)
    *reinterpret_cast<int4*>(idx + n * hp.J + j0) = make_int4(s[0], s[1], s[2], s[3]);
  else
    *reinterpret_cast<int2*>(idx + n * hp.J + j0) = make_int2(s[0], s[1]);
}

// Row gather with 16-byte vectors, generic shape.  The e row of a token is
// J*CR chunks of 16 bytes (CR per head row); consecutive threads take
// consecutive chunks, so the stores are fully coalesced.  Every thread keeps
// UNROLL loads in flight before storing.
template <int UNROLL>
__global__ void __launch_bounds__(256) gather_kernel(const __grid_constant__ HeadParams hp,
                                                     const int32_t* __restrict__ idx,
                                                     const uint4* __restrict__ table,
                                                     int64_t n_tok, int CR,
                                                     uint4* __restrict__ e,
                                                     unsigned int* status) {
  allow_dependents();
  const int per_tok = hp.J * CR;
  const int64_t total = n_tok * per_tok;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t base = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; base < total;
       base += stride * UNROLL) {
    uint4 v[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int64_t g = base + u * stride;
      v[u] = make_uint4(0, 0, 0, 0);
      if (g < total) {
        const int64_t n = g / per_tok;
        const int r = (int)(g - n * per_tok);
        const int j = r / CR;
        const int c = r - j * CR;
        const int32_t s = __ldg(idx + n * hp.J + j);
        if (s >= 0 && (uint64_t)s < hp.P[j]) {
          v[u] = ld_row_piece(table + (hp.row_base[j] + s) * CR + c);
        } else if (s != -1) {
          atomicOr(status, ENGRAM_STATUS_BAD_INDEX);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int64_t g = base + u * stride;
      if (g < total) e[g] = v[u];
    }
  }
}

// Row gather for head count JH and head-row width CR (16-byte pieces) fixed
// at compile time.  One warp takes TPW tokens at a time: lanes 0..JH-1 read
// the tokens' slots (one coalesced read per token) and pass them by
// shuffles; then every lane loads its pieces of all TPW tokens' rows
// (TPW * JH * CR / 32 loads in flight per lane) before storing them,
// consecutive lanes on consecutive pieces of e.
template <int JH, int CR, int TPW>
__global__ void __launch_bounds__(256) gather_rows_kernel(const __grid_constant__ HeadParams hp,
                                                          const int32_t* __restrict__ idx,
                                                          const uint4* __restrict__ table,
                                                          int64_t n_tok,
                                                          uint4* __restrict__ e,
                                                          unsigned int* status) {
  allow_dependents();
  constexpr int PER_TOK = JH * CR;             // pieces per token
  constexpr int PER_LANE = (PER_TOK + 31) / 32;
  const int lane = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t t0 = warp * TPW; t0 < n_tok; t0 += nwarps * TPW) {
    int32_t slot[TPW];
#pragma unroll
    for (int k = 0; k < TPW; ++k) {
      const int64_t n = t0 + k;
      slot[k] = (lane < JH && n < n_tok) ? __ldg(idx + n * JH + lane) : -1;
    }
    uint4 v[TPW][PER_LANE];
#pragma unroll
    for (int k = 0; k < TPW; ++k) {
#pragma unroll
      for (int p = 0; p < PER_LANE; ++p) {
        const int piece = p * 32 + lane;
        const int j = piece / CR;  // head of this piece (>= JH past the row's end)
        const int c = piece - j * CR;
        const int32_t s = __shfl_sync(FULL, slot[k], j < JH ? j : 0);
        v[k][p] = make_uint4(0, 0, 0, 0);
        if (piece < PER_TOK) {
          if (s >= 0 && (uint64_t)s < hp.P[j]) {
            v[k][p] = ld_row_piece(table + (hp.row_base[j] + s) * CR + c);
          } else if (s != -1) {
            atomicOr(status, ENGRAM_STATUS_BAD_INDEX);
          }
        }
      }
    }
#pragma unroll
    for (int k = 0; k < TPW; ++k) {
      const int64_t n = t0 + k;
      if (n < n_tok) {
#pragma unroll
        for (int p = 0; p < PER_LANE; ++p) {
          const int piece = p * 32 + lane;
          if (piece < PER_TOK) e[n * PER_TOK + piece] = v[k][p];
        }
      }
    }
  }
}

}  // namespace

int launch_hash(const HeadParams& hp, const int32_t* proj, const int32_t* ids, int B, int T,
                int32_t* ngram_state, int32_t* idx, cudaStream_t s) {
  const int64_t N = (int64_t)B * T;
  if (N == 0) return ENGRAM_OK;
  // threads per token: J / HPT (HPT heads each) rounded up to a power of two
  const int hpt = hp.J % 4 == 0 ? 4 : 2;
  int tpt = 1;
  while (tpt < hp.J / hpt) tpt *= 2;
  const int threads = 256;
  const int64_t total = N * tpt;
  const int64_t blocks = (total + threads - 1) / threads;
  if (hpt == 4)
    hash_kernel<4><<<(unsigned)blocks, threads, 0, s>>>(hp, proj, ids, N, T, tpt, ngram_state,
                                                        idx, status_ptr());
  else
    hash_kernel<2><<<(unsigned)blocks, threads, 0, s>>>(hp, proj, ids, N, T, tpt, ngram_state,
                                                        idx, status_ptr());
  return ck(cudaGetLastError());
}

int launch_gather(const HeadParams& hp, const int32_t* idx, const void* table, int64_t n_tok,
                  int elem_bytes, void* e, cudaStream_t s) {
  if (n_tok == 0) return ENGRAM_OK;
  const int CR = hp.D_h * elem_bytes / 16;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const uint4* tb = static_cast<const uint4*>(table);
  uint4* eo = static_cast<uint4*>(e);
  unsigned int* st = status_ptr();
  const int threads = 256;
  auto rows = [&](auto kern, int tpw) {
    const int64_t warps = (n_tok + tpw - 1) / tpw;
    int64_t blocks = (warps * 32 + threads - 1) / threads;
    const int64_t cap = (int64_t)sms * 8;  // 8 resident blocks of 256 threads per SM
    if (blocks > cap) blocks = cap;
    kern<<<(unsigned)blocks, threads, 0, s>>>(hp, idx, tb, n_tok, eo, st);
    return ck(cudaGetLastError());
  };
  const int64_t total = n_tok * hp.J * CR;
  if (n_tok * 32 < (int64_t)sms * threads * 4) {
    // few tokens (a decode step): warps of tokens would leave most SMs idle;
    // one 16-byte piece per thread instead, a single round trip each
    constexpr int UNROLL_SMALL = 2;
    const int64_t blocks =
        (total + (int64_t)threads * UNROLL_SMALL - 1) / ((int64_t)threads * UNROLL_SMALL);
    gather_kernel<UNROLL_SMALL><<<(unsigned)blocks, threads, 0, s>>>(hp, idx, tb, n_tok, CR, eo,
                                                                     st);
    return ck(cudaGetLastError());
  }
  const int key = hp.J * 100 + CR;
  switch (key) {
    case 4 * 100 + 4: return rows(gather_rows_kernel<4, 4, 8>, 8);     // fp32 rows of 16, 4 heads
    case 16 * 100 + 10: return rows(gather_rows_kernel<16, 10, 2>, 2);  // bf16 rows of 80
    case 16 * 100 + 16: return rows(gather_rows_kernel<16, 16, 2>, 2);  // bf16 rows of 128
    case 16 * 100 + 20: return rows(gather_rows_kernel<16, 20, 2>, 2);  // bf16 rows of 160
    default: break;
  }
  constexpr int UNROLL = 8;
  int64_t blocks = (total + (int64_t)threads * UNROLL - 1) / ((int64_t)threads * UNROLL);
  const int64_t cap = (int64_t)sms * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  gather_kernel<UNROLL><<<(unsigned)blocks, threads, 0, s>>>(hp, idx, tb, n_tok, CR, eo, st);
  return ck(cudaGetLastError());
}

// Gather from a table in pinned, mapped host memory.  Reads cross PCIe, so
// the time goes to latency, not to the SMs: a few small CTAs with many loads
// in flight each (128 threads x 8 x 16 B) leave the rest of the GPU to the
// work on the compute stream.  Measured on B200 with a bf16 GEMM
// [8,192 x 2,560] x [2,560 x 10,240] on the compute stream: 16 CTAs keep the
// GEMM within 9% of its time alone at 17 GB/s of rows; 32 CTAs reach 21 GB/s
// but slow the GEMM by 46%; a full grid reaches 30 GB/s and serialises it.
#ifndef ENGRAM_HOST_GATHER_CTAS
#define ENGRAM_HOST_GATHER_CTAS 16
#endif

int launch_gather_host(const HeadParams& hp, const int32_t* idx, const void* table, int64_t n_tok,
                       int elem_bytes, void* e, cudaStream_t s) {
  if (n_tok == 0) return ENGRAM_OK;
  const int CR = hp.D_h * elem_bytes / 16;
  constexpr int UNROLL = 8;
  constexpr int threads = 128;
  const int64_t total = n_tok * hp.J * CR;
  int64_t blocks = (total + (int64_t)threads * UNROLL - 1) / ((int64_t)threads * UNROLL);
  if (blocks > ENGRAM_HOST_GATHER_CTAS) blocks = ENGRAM_HOST_GATHER_CTAS;
  gather_kernel<UNROLL><<<(unsigned)blocks, threads, 0, s>>>(
      hp, idx, static_cast<const uint4*>(table), n_tok, CR, static_cast<uint4*>(e), status_ptr());
  return ck(cudaGetLastError());
}

// ------------------------------------------------------- HBM cache of host rows
//
// The pages' multi-level cache: the rows of frequent n-grams (Zipfian
// frequencies) stay in HBM, the long tail in host memory.  A dense map gives
// each packed-table row its cache slot (-1: not cached), so a lookup is one
// 4-byte read.

namespace {

// Cache slot i <- host row rows[i] (rows[i] < 0 leaves the slot empty), and
// map[rows[i]] = i.  A warp per slot, lanes over the row's 16-byte pieces.
__global__ void cache_fill_kernel(const uint4* __restrict__ host, const int64_t* __restrict__ rows,
                                  int64_t C, int CR, int64_t total_rows, uint4* __restrict__ cache,
                                  int32_t* __restrict__ map, unsigned int* status) {
  const int64_t slot = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (slot >= C) return;
  const int64_t r = rows[slot];
  if (r < 0) return;
  if (r >= total_rows) {
    if (lane == 0) atomicOr(status, ENGRAM_STATUS_BAD_INDEX);
    return;
  }
  for (int c = lane; c < CR; c += 32) cache[slot * CR + c] = ld_row_piece(host + r * CR + c);
  if (lane == 0) map[r] = (int32_t)slot;
}

// Pass 1 of a cached gather: one thread per (token, head) looks its row up.
// item_slot = the cache slot, -1 for a row left in host memory (appended to
// the miss list, one atomic per warp), -2 for an invalid slot (zeros).
__global__ void cache_probe_kernel(const __grid_constant__ HeadParams hp,
                                   const int32_t* __restrict__ idx,
                                   const int32_t* __restrict__ map, int64_t n_items,
                                   int32_t* __restrict__ item_slot, int32_t* __restrict__ miss_list,
                                   int32_t* __restrict__ n_miss, unsigned int* status) {
  const int64_t item = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int lane = threadIdx.x & 31;
  bool miss = false;
  if (item < n_items) {
    const int j = (int)(item % hp.J);
    const int32_t s = __ldg(idx + item);
    int32_t slot = -2;
    if (s >= 0 && (uint64_t)s < hp.P[j]) {
      slot = __ldg(map + hp.row_base[j] + s);
      miss = slot < 0;
      if (miss) slot = -1;
    } else if (s != -1) {
      atomicOr(status, ENGRAM_STATUS_BAD_INDEX);
    }
    item_slot[item] = slot;
  }
  const unsigned ballot = __ballot_sync(FULL, miss);
  if (ballot == 0) return;
  int32_t base = 0;
  if (lane == __ffs(ballot) - 1) base = atomicAdd(n_miss, __popc(ballot));
  base = __shfl_sync(FULL, base, __ffs(ballot) - 1);
  if (miss) miss_list[base + __popc(ballot & ((1u << lane) - 1u))] = (int32_t)item;
}

// Pass 2, on the whole GPU: the pieces of cached rows from HBM, zeros for
// invalid slots; rows left in host memory are pass 3's.
template <int UNROLL>
__global__ void __launch_bounds__(256) gather_hits_kernel(
    int J, const int32_t* __restrict__ item_slot, const uint4* __restrict__ cache, int64_t n_tok,
    int CR, uint4* __restrict__ e) {
  const int per_tok = J * CR;
  const int64_t total = n_tok * per_tok;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t base = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; base < total;
       base += stride * UNROLL) {
    uint4 v[UNROLL];
    bool own[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int64_t g = base + u * stride;
      v[u] = make_uint4(0, 0, 0, 0);
      own[u] = false;
      if (g < total) {
        const int64_t item = g / CR;
        const int c = (int)(g - item * CR);
        const int32_t slot = __ldg(item_slot + item);
        own[u] = slot != -1;
        if (slot >= 0) v[u] = ld_row_piece(cache + (int64_t)slot * CR + c);
      }
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u)
      if (own[u]) e[base + u * stride] = v[u];
  }
}

// Pass 3, on a few CTAs (the reads cross PCIe): the listed (token, head)
// rows from host memory.
template <int UNROLL>
__global__ void __launch_bounds__(128) gather_misses_kernel(
    const __grid_constant__ HeadParams hp, const int32_t* __restrict__ idx,
    const uint4* __restrict__ host, const int32_t* __restrict__ miss_list,
    const int32_t* __restrict__ n_miss, int CR, uint4* __restrict__ e) {
  const int64_t total = (int64_t)(*n_miss) * CR;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t base = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; base < total;
       base += stride * UNROLL) {
    uint4 v[UNROLL];
    int64_t dst[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int64_t g = base + u * stride;
      dst[u] = -1;
      if (g < total) {
        const int64_t m = g / CR;
        const int c = (int)(g - m * CR);
        const int32_t item = miss_list[m];  // n * J + j
        const int j = item % hp.J;
        const int32_t s = __ldg(idx + item);  // valid: the probe checked it
        v[u] = ld_row_piece(host + (hp.row_base[j] + s) * CR + c);
        dst[u] = (int64_t)item * CR + c;
      }
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u)
      if (dst[u] >= 0) e[dst[u]] = v[u];
  }
}

}  // namespace

int launch_cache_fill(const HeadParams& hp, const void* host, const int64_t* rows, int64_t C,
                      int elem_bytes, void* cache, int32_t* map, cudaStream_t s) {
  const int64_t total_rows = hp.row_base[hp.J - 1] + (int64_t)hp.P[hp.J - 1];
  int rc = ck(cudaMemsetAsync(map, 0xff, (size_t)total_rows * sizeof(int32_t), s));  // all -1
  if (rc || C == 0) return rc;
  const int CR = hp.D_h * elem_bytes / 16;
  const int64_t threads = 256;
  const int64_t blocks = (C * 32 + threads - 1) / threads;
  cache_fill_kernel<<<(unsigned)blocks, (unsigned)threads, 0, s>>>(
      static_cast<const uint4*>(host), rows, C, CR, total_rows, static_cast<uint4*>(cache), map,
      status_ptr());
  return ck(cudaGetLastError());
}

size_t cached_gather_ws_bytes(int64_t n_tok, int J) {
  const size_t list = ((size_t)n_tok * J * 4 + 255) & ~(size_t)255;
  return 2 * list + 256;  // item slots, miss list, miss count
}

int launch_gather_cached(const HeadParams& hp, const int32_t* idx, const void* host,
                         const void* cache, const int32_t* map, int64_t n_tok, int elem_bytes,
                         void* e, int32_t* n_miss_out, void* ws, cudaStream_t s) {
  const size_t list = ((size_t)n_tok * hp.J * 4 + 255) & ~(size_t)255;
  int32_t* item_slot = static_cast<int32_t*>(ws);
  int32_t* miss_list = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + list);
  int32_t* n_miss = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + 2 * list);
  int rc = ck(cudaMemsetAsync(n_miss, 0, sizeof(int32_t), s));
  if (rc) return rc;
  if (n_tok > 0) {
    const int CR = hp.D_h * elem_bytes / 16;
    const int64_t n_items = n_tok * hp.J;
    cache_probe_kernel<<<(unsigned)((n_items + 255) / 256), 256, 0, s>>>(
        hp, idx, map, n_items, item_slot, miss_list, n_miss, status_ptr());
    // the cached rows come from HBM on the whole GPU, briefly (measured with
    // a GEMM on the compute stream: 32 CTAs here ran longer and delayed the
    // GEMM more than a full grid)
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    constexpr int UNROLL = 4;
    const int64_t total = n_items * CR;
    int64_t blocks = (total + 256 * UNROLL - 1) / (256 * UNROLL);
    if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
    gather_hits_kernel<UNROLL><<<(unsigned)blocks, 256, 0, s>>>(
        hp.J, item_slot, static_cast<const uint4*>(cache), n_tok, CR, static_cast<uint4*>(e));
    gather_misses_kernel<8><<<ENGRAM_HOST_GATHER_CTAS, 128, 0, s>>>(
        hp, idx, static_cast<const uint4*>(host), miss_list, n_miss, CR, static_cast<uint4*>(e));
    if ((rc = ck(cudaGetLastError()))) return rc;
  }
  if (n_miss_out != nullptr)
    return ck(cudaMemcpyAsync(n_miss_out, n_miss, sizeof(int32_t), cudaMemcpyDeviceToDevice, s));
  return ENGRAM_OK;
}

}  // namespace engram
