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

// One decode step's hash and gather in one launch (one token per sequence,
// the n-gram history from the rolling state): a block per token.  Thread 0
// reads the token's compressed id and state; threads 0..J-1 hash one head
// each; then the block copies the token's J rows in 16-byte pieces, and
// thread 0 writes the new state (c_t, c_{t-1}) -- only thread 0 reads or
// writes the state, so no other thread can see it half-updated.
__global__ void __launch_bounds__(256) hash_gather_decode_kernel(
    const __grid_constant__ HeadParams hp, const int32_t* __restrict__ proj,
    const int32_t* __restrict__ ids, int32_t* __restrict__ ngram_state,
    int32_t* __restrict__ idx, const uint4* __restrict__ table, int CR,
    uint4* __restrict__ e, int* __restrict__ zero_counters, unsigned int* status) {
  allow_dependents();
  if (zero_counters != nullptr && blockIdx.x == 0 && threadIdx.x < 2) zero_counters[threadIdx.x] = 0;
  __shared__ int32_t cid[3];
  __shared__ int32_t slot[ENGRAM_MAX_HEADS];
  const int64_t n = blockIdx.x;
  const int J = hp.J;
  if (threadIdx.x == 0) {
    const int32_t c0 = token_cid(proj, ids, n, hp.V_raw, hp.V_c);
    const int32_t c1 = ngram_state[2 * n + 0], c2 = ngram_state[2 * n + 1];
    if (c0 < 0) atomicOr(status, ENGRAM_STATUS_BAD_ID);
    cid[0] = c0;
    cid[1] = c1;
    cid[2] = c2;
  }
  __syncthreads();
  const int32_t c0 = cid[0], c1 = cid[1], c2 = cid[2];
  if (threadIdx.x < J) {
    const int j = threadIdx.x;
    const bool bad2 = (c0 < 0) | (c1 < 0);
    const bool bad3 = bad2 | (c2 < 0);
    uint64_t x = (uint64_t)(uint32_t)c0 * hp.mult[j][0];
    x ^= (uint64_t)(uint32_t)c1 * hp.mult[j][1];
    const bool tri = j >= hp.K;
    if (tri) x ^= (uint64_t)(uint32_t)c2 * hp.mult[j][2];
    const int32_t sl = (tri ? bad3 : bad2) ? -1 : (int32_t)mod_prime(x, hp.P[j], hp.mu[j]);
    slot[j] = sl;
    if (idx != nullptr) idx[n * J + j] = sl;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    ngram_state[2 * n + 0] = c0;
    ngram_state[2 * n + 1] = c1;
  }
  const int per_tok = J * CR;
  for (int p = threadIdx.x; p < per_tok; p += blockDim.x) {
    const int j = p / CR, c = p - j * CR;
    const int32_t sl = slot[j];
    e[n * per_tok + p] =
        sl >= 0 ? ld_row_piece(table + (hp.row_base[j] + sl) * CR + c) : make_uint4(0, 0, 0, 0);
  }
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
                                                     int* __restrict__ zero_counters,
                                                     unsigned int* status) {
  allow_dependents();
  if (zero_counters != nullptr && blockIdx.x == 0 && threadIdx.x < 2) zero_counters[threadIdx.x] = 0;
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
                  int elem_bytes, void* e, cudaStream_t s, int* zero_counters) {
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
                                                                     zero_counters, st);
    return ck(cudaGetLastError());
  }
  if (zero_counters != nullptr) {
    const int rc = ck(cudaMemsetAsync(zero_counters, 0, 2 * sizeof(int), s));
    if (rc) return rc;
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
  gather_kernel<UNROLL><<<(unsigned)blocks, threads, 0, s>>>(hp, idx, tb, n_tok, CR, eo, nullptr,
                                                             st);
  return ck(cudaGetLastError());
}

int launch_hash_gather_decode(const HeadParams& hp, const int32_t* proj, const int32_t* ids,
                              int64_t B, int32_t* ngram_state, int32_t* idx, const void* table,
                              int elem_bytes, void* e, int* zero_counters, cudaStream_t s) {
  if (B == 0) return ENGRAM_OK;
  const int CR = hp.D_h * elem_bytes / 16;
  const int per_tok = hp.J * CR;
  // at least a warp (threads 0..J-1 hash, J <= 32), at most 256 pieces at a time
  int threads = ((per_tok + 31) / 32) * 32;
  if (threads > 256) threads = 256;
  hash_gather_decode_kernel<<<(unsigned)B, (unsigned)threads, 0, s>>>(
      hp, proj, ids, ngram_state, idx, static_cast<const uint4*>(table), CR,
      static_cast<uint4*>(e), zero_counters, status_ptr());
  return ck(cudaGetLastError());
}

// Gather from a table in pinned, mapped host memory.  Reads cross PCIe, so
// the time goes to latency and to the size of the link's read requests, not
// to the SMs: a few CTAs, each with many rows in flight, leave the rest of
// the GPU to the work on the compute stream.  Each warp walks its own tokens;
// for a token, lanes 0..J-1 each copy one table row (D_h elements, a multiple
// of 16 bytes) from host memory into a shared-memory slot with one
// cp.async.bulk, all completing on the slot's mbarrier, so a row crosses the
// link as one request stream instead of 16-byte loads.  The warp then writes
// the slot to e with coalesced 16-byte stores.  HG_SLOTS slots per warp keep
// that many tokens' rows in flight.  Slots of -1 read nothing and give zero
// rows; slots outside [0, P_j) also set ENGRAM_STATUS_BAD_INDEX.  A slot
// whose copies do not land within the wait limit sets
// ENGRAM_STATUS_TIMEOUT; the warp then stops and lets its copies in flight
// land (bounded) before the block exits.
namespace {

#ifndef ENGRAM_HOST_GATHER_CTAS
#define ENGRAM_HOST_GATHER_CTAS 16
#endif
constexpr int HG_WARPS = 8;
constexpr int HG_SLOTS = 2;  // 1, 2 and 3 slots measured alike (16 CTAs)
constexpr uint64_t HG_WAIT_NS = 2000000000ull;  // 2 s

__device__ __forceinline__ uint32_t hg_smem(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ bool hg_wait(uint64_t* bar, uint32_t parity) {
  uint64_t t0 = 0;
  for (int spin = 0;; ++spin) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(hg_smem(bar)), "r"(parity), "r"(20000u)
        : "memory");
    if (ok) return true;
    uint64_t now;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
    if (spin == 0) t0 = now;
    else if (now - t0 > HG_WAIT_NS) return false;
  }
}

__global__ void __launch_bounds__(HG_WARPS * 32) gather_host_rows_kernel(
    const __grid_constant__ HeadParams hp, const int32_t* __restrict__ idx,
    const uint8_t* __restrict__ table, int64_t n_tok, int row_bytes, int slots,
    uint4* __restrict__ e, unsigned int* status) {
  extern __shared__ __align__(128) uint8_t hg_ring[];
  __shared__ uint64_t bars[HG_WARPS][HG_SLOTS];
  __shared__ uint32_t masks[HG_WARPS][HG_SLOTS];  // rows of the slot's token that were copied
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int J = hp.J;
  const int tok_bytes = J * row_bytes;
  const int pieces = tok_bytes / 16, row_pieces = row_bytes / 16;
  uint8_t* ring = hg_ring + (size_t)warp * slots * tok_bytes;
  const int64_t first = (int64_t)blockIdx.x * HG_WARPS + warp;
  const int64_t stride = (int64_t)gridDim.x * HG_WARPS;
  if (lane < slots) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(hg_smem(&bars[warp][lane])));
  }
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  __syncwarp();
  unsigned pend = 0;  // lane 0: slots with copies issued and not yet seen landed
  // Copies of token t's rows into `slot`: lane 0 posts the bytes to expect,
  // then lanes 0..J-1 issue one row each.
  auto issue = [&](int64_t t, int slot) {
    int32_t sl = -1;
    bool ok = false;
    if (lane < J) {
      sl = __ldg(idx + t * J + lane);
      ok = sl >= 0 && (uint64_t)sl < hp.P[lane];
      if (!ok && sl != -1) atomicOr(status, ENGRAM_STATUS_BAD_INDEX);
    }
    const uint32_t mask = __ballot_sync(0xffffffffu, ok);
    if (lane == 0) {
      masks[warp][slot] = mask;
      pend |= 1u << slot;
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
                       hg_smem(&bars[warp][slot])),
                   "r"((uint32_t)__popc(mask) * (uint32_t)row_bytes)
                   : "memory");
    }
    __syncwarp();
    if (ok) {
      const uint8_t* src = table + (uint64_t)(hp.row_base[lane] + sl) * (uint64_t)row_bytes;
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
          ::"r"(hg_smem(ring + (size_t)slot * tok_bytes + (size_t)lane * row_bytes)),
          "l"(src), "r"((uint32_t)row_bytes), "r"(hg_smem(&bars[warp][slot]))
          : "memory");
    }
  };
  for (int k = 0; k < slots; ++k) {
    const int64_t t = first + k * stride;
    if (t < n_tok) issue(t, k);
  }
  int k = 0;
  for (int64_t t = first; t < n_tok; t += stride, ++k) {
    const int slot = k % slots;
    int ok = 1;
    if (lane == 0) ok = hg_wait(&bars[warp][slot], (uint32_t)(k / slots) & 1u) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) {
      if (lane == 0) atomicOr(status, ENGRAM_STATUS_TIMEOUT);
      break;
    }
    if (lane == 0) pend &= ~(1u << slot);
    const uint32_t mask = masks[warp][slot];
    const uint4* src = reinterpret_cast<const uint4*>(ring + (size_t)slot * tok_bytes);
    uint4* dst = e + t * pieces;
    for (int p = lane; p < pieces; p += 32) {
      const int r = p / row_pieces;
      dst[p] = ((mask >> r) & 1u) ? src[p] : make_uint4(0u, 0u, 0u, 0u);
    }
    __syncwarp();  // every lane has read the slot before it is refilled
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    const int64_t nt = t + (int64_t)slots * stride;
    if (nt < n_tok) issue(nt, slot);
  }
  // after a timeout: let the copies still in flight land (bounded) before the
  // block's shared memory is released; a slot holds at most one use, the one
  // after the last waited for
  if (lane == 0 && pend != 0) {
    for (int sl = 0; sl < slots; ++sl) {
      if (!(pend & (1u << sl))) continue;
      const int use = k / slots + (sl < k % slots ? 1 : 0);
      hg_wait(&bars[warp][sl], (uint32_t)use & 1u);
    }
  }
}

}  // namespace

int launch_gather_host(const HeadParams& hp, const int32_t* idx, const void* table, int64_t n_tok,
                       int elem_bytes, void* e, cudaStream_t s) {
  if (n_tok == 0) return ENGRAM_OK;
  const int row_bytes = hp.D_h * elem_bytes;
  constexpr size_t kRing = 160 * 1024;  // shared memory for the warps' slots
  const size_t tok_bytes = (size_t)hp.J * row_bytes;
  int slots = (int)(kRing / (HG_WARPS * tok_bytes));
  if (slots > HG_SLOTS) slots = HG_SLOTS;
  if (slots < 1) {
    // a token's rows exceed a slot: 16-byte loads, eight in flight per thread
    constexpr int UNROLL = 8;
    const int CR = row_bytes / 16;
    const int64_t total = n_tok * hp.J * CR;
    int64_t blocks = (total + 128 * UNROLL - 1) / (128 * UNROLL);
    if (blocks > ENGRAM_HOST_GATHER_CTAS) blocks = ENGRAM_HOST_GATHER_CTAS;
    gather_kernel<UNROLL><<<(unsigned)blocks, 128, 0, s>>>(
        hp, idx, static_cast<const uint4*>(table), n_tok, CR, static_cast<uint4*>(e), nullptr,
        status_ptr());
    return ck(cudaGetLastError());
  }
  const size_t smem = (size_t)HG_WARPS * slots * tok_bytes;
  static bool configured[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ENGRAM_ERR_CUDA;
  if (!configured[dev]) {
    if (cudaFuncSetAttribute(gather_host_rows_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRing) !=
        cudaSuccess)
      return ENGRAM_ERR_CUDA;
    configured[dev] = true;
  }
  // one warp per token at most; ENGRAM_HOST_GATHER_CTAS blocks at most
  int64_t blocks = (n_tok + HG_WARPS - 1) / HG_WARPS;
  if (blocks > ENGRAM_HOST_GATHER_CTAS) blocks = ENGRAM_HOST_GATHER_CTAS;
  gather_host_rows_kernel<<<(unsigned)blocks, HG_WARPS * 32, smem, s>>>(
      hp, idx, static_cast<const uint8_t*>(table), n_tok, row_bytes, slots,
      static_cast<uint4*>(e), status_ptr());
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
// rows from host memory, by bulk copies as in gather_host_rows_kernel: a
// warp takes grp (up to 32) listed rows at a time, each lane copying one row
// into the warp's shared-memory slot; the warp then writes the rows to their
// places in e.  `slots` groups per warp are in flight.
__global__ void __launch_bounds__(HG_WARPS * 32) gather_misses_kernel(
    const __grid_constant__ HeadParams hp, const int32_t* __restrict__ idx,
    const uint8_t* __restrict__ host, const int32_t* __restrict__ miss_list,
    const int32_t* __restrict__ n_miss, int row_bytes, int grp, int slots,
    uint8_t* __restrict__ e, unsigned int* status) {
  extern __shared__ __align__(128) uint8_t hg_ring[];
  __shared__ uint64_t bars[HG_WARPS][HG_SLOTS];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int J = hp.J;
  const int grp_bytes = grp * row_bytes, row_pieces = row_bytes / 16;
  uint8_t* ring = hg_ring + (size_t)warp * slots * grp_bytes;
  const int64_t n = *n_miss;
  const int64_t groups = (n + grp - 1) / grp;
  const int64_t first = (int64_t)blockIdx.x * HG_WARPS + warp;
  const int64_t stride = (int64_t)gridDim.x * HG_WARPS;
  if (lane < slots) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(hg_smem(&bars[warp][lane])));
  }
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  __syncwarp();
  unsigned pend = 0;
  auto issue = [&](int64_t gi, int slot) {
    const int64_t m = gi * grp + lane;
    const bool ok = lane < grp && m < n;
    const uint32_t cnt = __popc(__ballot_sync(0xffffffffu, ok));
    if (lane == 0) {
      pend |= 1u << slot;
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
                       hg_smem(&bars[warp][slot])),
                   "r"(cnt * (uint32_t)row_bytes)
                   : "memory");
    }
    __syncwarp();
    if (ok) {
      const int32_t item = miss_list[m];  // n * J + j
      const int j = item % J;
      const int32_t sl = __ldg(idx + item);  // valid: the probe checked it
      const uint8_t* src = host + (uint64_t)(hp.row_base[j] + sl) * (uint64_t)row_bytes;
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
          ::"r"(hg_smem(ring + (size_t)slot * grp_bytes + (size_t)lane * row_bytes)),
          "l"(src), "r"((uint32_t)row_bytes), "r"(hg_smem(&bars[warp][slot]))
          : "memory");
    }
  };
  for (int k = 0; k < slots; ++k) {
    const int64_t gi = first + k * stride;
    if (gi < groups) issue(gi, k);
  }
  int k = 0;
  for (int64_t gi = first; gi < groups; gi += stride, ++k) {
    const int slot = k % slots;
    int ok = 1;
    if (lane == 0) ok = hg_wait(&bars[warp][slot], (uint32_t)(k / slots) & 1u) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) {
      if (lane == 0) atomicOr(status, ENGRAM_STATUS_TIMEOUT);
      break;
    }
    if (lane == 0) pend &= ~(1u << slot);
    const int64_t m0 = gi * grp;
    const int cnt = (int)(n - m0 < grp ? n - m0 : grp);
    const uint4* src = reinterpret_cast<const uint4*>(ring + (size_t)slot * grp_bytes);
    for (int p = lane; p < cnt * row_pieces; p += 32) {
      const int r = p / row_pieces;
      const int c = p - r * row_pieces;
      uint4* dst = reinterpret_cast<uint4*>(e + (int64_t)miss_list[m0 + r] * row_bytes) + c;
      *dst = src[p];
    }
    __syncwarp();
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    const int64_t ng = gi + (int64_t)slots * stride;
    if (ng < groups) issue(ng, slot);
  }
  if (lane == 0 && pend != 0) {
    for (int sl = 0; sl < slots; ++sl) {
      if (!(pend & (1u << sl))) continue;
      const int use = k / slots + (sl < k % slots ? 1 : 0);
      hg_wait(&bars[warp][sl], (uint32_t)use & 1u);
    }
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
    // groups of up to 32 rows per warp slot, as many slots (up to
    // HG_SLOTS) as kRing bytes of shared memory hold
    const int row_bytes = CR * 16;
    constexpr size_t kRing = 160 * 1024;
    int grp = (int)(kRing / ((size_t)HG_WARPS * row_bytes));
    if (grp > 32) grp = 32;
    if (grp < 1) return ENGRAM_ERR_UNSUPPORTED;  // a row over 20 KB
    int slots = (int)(kRing / ((size_t)HG_WARPS * grp * row_bytes));
    if (slots > HG_SLOTS) slots = HG_SLOTS;
    static bool configured[64] = {false};
    if (dev < 0 || dev >= 64) return ENGRAM_ERR_CUDA;
    if (!configured[dev]) {
      if ((rc = ck(cudaFuncSetAttribute(gather_misses_kernel,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRing))))
        return rc;
      configured[dev] = true;
    }
    gather_misses_kernel<<<ENGRAM_HOST_GATHER_CTAS, HG_WARPS * 32,
                           (size_t)HG_WARPS * slots * grp * row_bytes, s>>>(
        hp, idx, static_cast<const uint8_t*>(host), miss_list, n_miss, row_bytes, grp, slots,
        static_cast<uint8_t*>(e), status_ptr());
    if ((rc = ck(cudaGetLastError()))) return rc;
  }
  if (n_miss_out != nullptr)
    return ck(cudaMemcpyAsync(n_miss_out, n_miss, sizeof(int32_t), cudaMemcpyDeviceToDevice, s));
  return ENGRAM_OK;
}

}  // namespace engram
