// Stable LSD radix sort of (64-bit key, 32-bit value) pairs, an exclusive
// scan, and the two users built on them:
//  * the sparse table gradient: every (token, head) pair becomes (packed row
//    id, item index); a stable sort by row id lines up each row's tokens in
//    ascending order, and one thread per (row, dimension) adds their de
//    segments in that order in fp32 -- the same sum, bit for bit, on every run
//    (gitcode.csdn.net blog: lookups are deterministic, so a slot receives
//    consistent gradient updates during end-to-end training);
//  * the vocabulary projection: a stable sort by key groups the raw ids of one
//    key with the smallest id first; compressed ids number the groups in order
//    of that first id (discuss.deepseek.club 二.1 (1) 词汇投影).
#include <mutex>

#include "internal.cuh"

namespace engram {

namespace {

// digits of up to RADIX_MAX_BITS bits: a sort of b key bits takes
// ceil(b / 10) passes, the bits spread evenly over them (27-bit row ids: 3
// passes of 9 bits)
constexpr int RADIX_MAX_BITS = 10;
constexpr int RADIX_MAX = 1 << RADIX_MAX_BITS;
constexpr int SORT_THREADS = 256;
constexpr int SORT_WARPS = SORT_THREADS / 32;
constexpr int CHUNKS_PER_WARP = 8;                       // 8 x 32 items per warp
constexpr int TILE = SORT_THREADS * CHUNKS_PER_WARP;     // 2048 items per block
constexpr unsigned FULL = 0xffffffffu;

constexpr size_t up256(size_t b) { return (b + 255) & ~(size_t)255; }

__device__ __forceinline__ int digit_of(uint64_t key, int shift, int radix) {
  return (int)((key >> shift) & (uint64_t)(radix - 1));
}

// Counts of each of the radix digits in this block's tile ->
// hist[digit * nblocks + block].
__global__ void __launch_bounds__(SORT_THREADS) radix_hist_kernel(const uint64_t* __restrict__ keys,
                                                                  int64_t n, int shift, int radix,
                                                                  int32_t* __restrict__ hist) {
  __shared__ int32_t cnt[RADIX_MAX];
  for (int i = threadIdx.x; i < radix; i += SORT_THREADS) cnt[i] = 0;
  __syncthreads();
  const int64_t base = (int64_t)blockIdx.x * TILE;
  for (int i = threadIdx.x; i < TILE; i += SORT_THREADS) {
    const int64_t p = base + i;
    if (p < n) atomicAdd(&cnt[digit_of(keys[p], shift, radix)], 1);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < radix; i += SORT_THREADS)
    hist[(int64_t)i * gridDim.x + blockIdx.x] = cnt[i];
}

__device__ __forceinline__ int32_t block_scan(int32_t t, int32_t* excl);

// Stable scatter: item order inside the tile is (warp, chunk, lane); each
// item's destination = start of its digit (the exclusive scan of the digit
// totals dtot, formed here) + the digit's items in earlier blocks (offsets,
// per digit) + items of the same digit before it in that order.
__global__ void __launch_bounds__(SORT_THREADS) radix_scatter_kernel(
    const uint64_t* __restrict__ keys_in, const uint32_t* __restrict__ vals_in, int64_t n,
    int shift, int radix, const int32_t* __restrict__ offsets, const int32_t* __restrict__ dtot,
    uint64_t* __restrict__ keys_out, uint32_t* __restrict__ vals_out) {
  __shared__ int32_t wcnt[SORT_WARPS][RADIX_MAX];
  __shared__ int32_t boff[RADIX_MAX];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int w = 0; w < SORT_WARPS; ++w)
    for (int i = threadIdx.x; i < radix; i += SORT_THREADS) wcnt[w][i] = 0;
  {
    // digits 4 t .. 4 t + 3 of this thread (radix <= 4 * SORT_THREADS)
    constexpr int PD = RADIX_MAX / SORT_THREADS;
    int32_t tv[PD], sum = 0;
#pragma unroll
    for (int q = 0; q < PD; ++q) {
      const int dq = threadIdx.x * PD + q;
      tv[q] = dq < radix ? dtot[dq] : 0;
      sum += tv[q];
    }
    int32_t run;
    block_scan(sum, &run);
#pragma unroll
    for (int q = 0; q < PD; ++q) {
      const int dq = threadIdx.x * PD + q;
      if (dq < radix) boff[dq] = run + offsets[(int64_t)dq * gridDim.x + blockIdx.x];
      run += tv[q];
    }
  }
  __syncthreads();

  const int64_t wbase = (int64_t)blockIdx.x * TILE + (int64_t)warp * 32 * CHUNKS_PER_WARP;
  const unsigned lt_mask = (1u << lane) - 1u;
  uint64_t k[CHUNKS_PER_WARP];
  uint32_t v[CHUNKS_PER_WARP];
  int dg[CHUNKS_PER_WARP], rk[CHUNKS_PER_WARP];
#pragma unroll
  for (int c = 0; c < CHUNKS_PER_WARP; ++c) {
    const int64_t p = wbase + c * 32 + lane;
    const bool ok = p < n;
    k[c] = ok ? keys_in[p] : 0;
    v[c] = ok ? vals_in[p] : 0;
    const int d = ok ? digit_of(k[c], shift, radix) : radix;  // radix marks "no item"
    dg[c] = d;
    const unsigned peers = __match_any_sync(FULL, d);
    const int before = (d < radix) ? wcnt[warp][d] : 0;
    rk[c] = before + __popc(peers & lt_mask);
    __syncwarp();
    if (d < radix && (peers & lt_mask) == 0) wcnt[warp][d] = before + __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // exclusive prefix over warps, per digit
  for (int d = threadIdx.x; d < radix; d += SORT_THREADS) {
    int run = 0;
    for (int w = 0; w < SORT_WARPS; ++w) {
      const int t = wcnt[w][d];
      wcnt[w][d] = run;
      run += t;
    }
  }
  __syncthreads();
#pragma unroll
  for (int c = 0; c < CHUNKS_PER_WARP; ++c) {
    if (dg[c] < radix) {
      const int64_t dst = (int64_t)boff[dg[c]] + wcnt[warp][dg[c]] + rk[c];
      keys_out[dst] = k[c];
      vals_out[dst] = v[c];
    }
  }
}

// Exclusive scan of int32 x[0..n) into y (may alias x), total into *total
// (if non-null), in three passes over at most SCAN_MAX_BLOCKS chunks: each
// block sums its chunk, one block scans the chunk sums, each block scans its
// chunk from its offset.  Loads and stores are 16-byte vectors of a thread's
// SCAN_ITEMS consecutive elements.
constexpr int SCAN_THREADS = 256;
constexpr int SCAN_ITEMS = 16;
constexpr int SCAN_TILE = SCAN_THREADS * SCAN_ITEMS;  // 4096 elements
constexpr int SCAN_MAX_BLOCKS = 1024;

constexpr int64_t scan_chunk(int64_t n) {
  const int64_t tiles = (n + SCAN_TILE - 1) / SCAN_TILE;
  const int64_t per_block = (tiles + SCAN_MAX_BLOCKS - 1) / SCAN_MAX_BLOCKS;
  return (per_block > 0 ? per_block : 1) * SCAN_TILE;
}

__device__ __forceinline__ void scan_load(const int32_t* x, int64_t n, int64_t base,
                                          int32_t (&v)[SCAN_ITEMS]) {
  if (base + SCAN_ITEMS <= n) {
    const int4* q = reinterpret_cast<const int4*>(x + base);
#pragma unroll
    for (int u = 0; u < SCAN_ITEMS / 4; ++u) {
      const int4 t = q[u];
      v[4 * u] = t.x;
      v[4 * u + 1] = t.y;
      v[4 * u + 2] = t.z;
      v[4 * u + 3] = t.w;
    }
  } else {
#pragma unroll
    for (int u = 0; u < SCAN_ITEMS; ++u) v[u] = base + u < n ? x[base + u] : 0;
  }
}

// Sum of the block's SCAN_THREADS values `t`, returned to every thread, and
// the exclusive prefix of `t` within the block in *excl.
__device__ __forceinline__ int32_t block_scan(int32_t t, int32_t* excl) {
  __shared__ int32_t wsum[SCAN_THREADS / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t incl = t;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t u = __shfl_up_sync(FULL, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int32_t before = 0, all = 0;
#pragma unroll
  for (int w = 0; w < SCAN_THREADS / 32; ++w) {
    const int32_t s = wsum[w];
    if (w < warp) before += s;
    all += s;
  }
  __syncthreads();  // wsum is reused by the next call
  *excl = before + incl - t;
  return all;
}

// The per-block counts of one digit (hist[d * nblocks + b], b ascending)
// replaced by their exclusive prefix, one block per digit; the digit's total
// into dtot[d].  Each thread takes a run of consecutive blocks.
__global__ void __launch_bounds__(SCAN_THREADS) radix_digit_scan_kernel(int32_t* hist, int nblocks,
                                                                        int32_t* dtot) {
  int32_t* h = hist + (int64_t)blockIdx.x * nblocks;
  const int per = (nblocks + SCAN_THREADS - 1) / SCAN_THREADS;
  const int lo = threadIdx.x * per, hi = lo + per < nblocks ? lo + per : nblocks;
  int32_t s = 0;
  for (int b = lo; b < hi; ++b) s += h[b];
  int32_t run;
  const int32_t all = block_scan(s, &run);
  for (int b = lo; b < hi; ++b) {
    const int32_t t = h[b];
    h[b] = run;
    run += t;
  }
  if (threadIdx.x == 0) dtot[blockIdx.x] = all;
}

__global__ void __launch_bounds__(SCAN_THREADS) scan_reduce_kernel(const int32_t* x, int64_t n,
                                                                   int64_t chunk,
                                                                   int32_t* bsum) {
  const int64_t lo = (int64_t)blockIdx.x * chunk;
  const int64_t hi = lo + chunk < n ? lo + chunk : n;
  int32_t s = 0;
  for (int64_t t0 = lo; t0 < hi; t0 += SCAN_TILE) {
    int32_t v[SCAN_ITEMS];
    scan_load(x, hi, t0 + (int64_t)threadIdx.x * SCAN_ITEMS, v);
#pragma unroll
    for (int u = 0; u < SCAN_ITEMS; ++u) s += v[u];
  }
  int32_t ex;
  const int32_t all = block_scan(s, &ex);
  if (threadIdx.x == 0) bsum[blockIdx.x] = all;
}

// Exclusive scan of the nblk chunk sums in place (nblk <= SCAN_MAX_BLOCKS);
// the grand total into *total.
__global__ void __launch_bounds__(SCAN_MAX_BLOCKS) scan_sums_kernel(int32_t* bsum, int nblk,
                                                                    int32_t* total) {
  __shared__ int32_t wsum[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int32_t v = tid < nblk ? bsum[tid] : 0;
  int32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t u = __shfl_up_sync(FULL, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int32_t w = wsum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t u = __shfl_up_sync(FULL, w, o);
      if (lane >= o) w += u;
    }
    wsum[lane] = w;
  }
  __syncthreads();
  const int32_t ex = incl - v + (warp > 0 ? wsum[warp - 1] : 0);
  if (tid < nblk) bsum[tid] = ex;
  if (total != nullptr && tid == SCAN_MAX_BLOCKS - 1) *total = ex + v;
}

__global__ void __launch_bounds__(SCAN_THREADS) scan_apply_kernel(const int32_t* x, int32_t* y,
                                                                  int64_t n, int64_t chunk,
                                                                  const int32_t* bsum) {
  const int64_t lo = (int64_t)blockIdx.x * chunk;
  const int64_t hi = lo + chunk < n ? lo + chunk : n;
  int32_t carry = bsum[blockIdx.x];
  for (int64_t t0 = lo; t0 < hi; t0 += SCAN_TILE) {
    const int64_t base = t0 + (int64_t)threadIdx.x * SCAN_ITEMS;
    int32_t v[SCAN_ITEMS];
    scan_load(x, hi, base, v);
    int32_t s = 0;
#pragma unroll
    for (int u = 0; u < SCAN_ITEMS; ++u) s += v[u];
    int32_t ex;
    const int32_t all = block_scan(s, &ex);
    int32_t run = carry + ex;
#pragma unroll
    for (int u = 0; u < SCAN_ITEMS; ++u) {
      const int32_t t = v[u];
      v[u] = run;
      run += t;
    }
    if (base + SCAN_ITEMS <= hi) {
      int4* q = reinterpret_cast<int4*>(y + base);
#pragma unroll
      for (int u = 0; u < SCAN_ITEMS / 4; ++u)
        q[u] = make_int4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
    } else {
#pragma unroll
      for (int u = 0; u < SCAN_ITEMS; ++u)
        if (base + u < hi) y[base + u] = v[u];
    }
    carry += all;
  }
}

constexpr size_t scan_ws_bytes() { return up256((SCAN_MAX_BLOCKS + 1) * 4); }
static_assert(SCAN_THREADS == SORT_THREADS, "the scatter kernel uses block_scan");
static_assert(RADIX_MAX <= SCAN_MAX_BLOCKS, "digit totals fit the scan scratch");

// x and y 16-byte aligned; bsum: scan_ws_bytes() of workspace.
int launch_scan(const int32_t* x, int32_t* y, int64_t n, int32_t* total, int32_t* bsum,
                cudaStream_t s) {
  if (n <= 0) return total != nullptr ? ck(cudaMemsetAsync(total, 0, sizeof(int32_t), s)) : 0;
  const int64_t chunk = scan_chunk(n);
  const int nblk = (int)((n + chunk - 1) / chunk);
  scan_reduce_kernel<<<nblk, SCAN_THREADS, 0, s>>>(x, n, chunk, bsum);
  scan_sums_kernel<<<1, SCAN_MAX_BLOCKS, 0, s>>>(bsum, nblk, total);
  scan_apply_kernel<<<nblk, SCAN_THREADS, 0, s>>>(x, y, n, chunk, bsum);
  return ck(cudaGetLastError());
}

int radix_sort_pairs(uint64_t*& keys, uint32_t*& vals, uint64_t* keys_alt, uint32_t* vals_alt,
                     int64_t n, int key_bits, int32_t* hist, int32_t* bsum, cudaStream_t s) {
  if (n == 0) return ENGRAM_OK;
  const int64_t nblocks = (n + TILE - 1) / TILE;
  const int passes = (key_bits + RADIX_MAX_BITS - 1) / RADIX_MAX_BITS;
  const int bits = (key_bits + passes - 1) / passes;
  const int radix = 1 << bits;
  // bsum holds the digit totals (radix <= SCAN_MAX_BLOCKS ints)
  for (int shift = 0; shift < key_bits; shift += bits) {
    radix_hist_kernel<<<(unsigned)nblocks, SORT_THREADS, 0, s>>>(keys, n, shift, radix, hist);
    radix_digit_scan_kernel<<<(unsigned)radix, SCAN_THREADS, 0, s>>>(hist, (int)nblocks, bsum);
    radix_scatter_kernel<<<(unsigned)nblocks, SORT_THREADS, 0, s>>>(
        keys, vals, n, shift, radix, hist, bsum, keys_alt, vals_alt);
    uint64_t* tk = keys;
    keys = keys_alt;
    keys_alt = tk;
    uint32_t* tv = vals;
    vals = vals_alt;
    vals_alt = tv;
  }
  return ck(cudaGetLastError());
}

int bits_for(uint64_t max_value) {
  int b = 1;
  while (b < 64 && (max_value >> b) != 0) ++b;
  return b;
}

// ---------------------------------------------------------------- table grad

// item i = n*J + j -> key = packed row id of head j's slot (or `sentinel` for
// an invalid slot), value = i
__global__ void tg_items_kernel(const __grid_constant__ HeadParams hp,
                                const int32_t* __restrict__ idx, int64_t n_items,
                                uint64_t sentinel, uint64_t* __restrict__ keys,
                                uint32_t* __restrict__ vals) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_items) return;
  const int j = (int)(i % hp.J);
  const int32_t s = idx[i];
  keys[i] = (s >= 0 && (uint64_t)s < hp.P[j]) ? (uint64_t)(hp.row_base[j] + s) : sentinel;
  vals[i] = (uint32_t)i;
}

__global__ void tg_flags_kernel(const uint64_t* __restrict__ keys, int64_t n, uint64_t sentinel,
                                int32_t* __restrict__ flags) {
  const int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= n) return;
  const uint64_t k = keys[p];
  flags[p] = (k != sentinel && (p == 0 || keys[p - 1] != k)) ? 1 : 0;
}

// segment starts, unique keys; seg_start[n_unique] = number of valid items
__global__ void tg_heads_kernel(const uint64_t* __restrict__ keys, int64_t n, uint64_t sentinel,
                                const int32_t* __restrict__ ex, int32_t* __restrict__ seg_start,
                                int64_t* __restrict__ out_keys) {
  const int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= n) return;
  const uint64_t k = keys[p];
  if (k == sentinel) return;
  const bool head = (p == 0 || keys[p - 1] != k);
  if (head) {
    seg_start[ex[p]] = (int32_t)p;
    out_keys[ex[p]] = (int64_t)k;
  }
  const bool last_valid = (p + 1 == n) || keys[p + 1] == sentinel;
  if (last_valid) seg_start[ex[p] + (head ? 1 : 0)] = (int32_t)(p + 1);
}

// de of item i = n*J + j starts at i * D_h because E = J * D_h.
//
// One thread per (unique row, group of 4 dimensions): the row's de segments
// added in sorted (= ascending token) order, from +0, in fp32, each of the 4
// dimensions on its own (16-byte loads; D_h is a multiple of 4).  The order
// of the adds is fixed; the loads are not: a thread takes TG_U items at once
// so that their first loads overlap, and walks a long segment (a frequent
// n-gram) with TG_PF loads issued ahead of the adds.
constexpr int TG_U = 4;
constexpr int TG_PF = 8;
constexpr int TG_LONG = 64;  // longer segments go to tg_long_reduce_kernel
__device__ __forceinline__ void add4(float4& a, const float4 x) {
  a.x = a.x + x.x;
  a.y = a.y + x.y;
  a.z = a.z + x.z;
  a.w = a.w + x.w;
}
__global__ void tg_reduce_kernel(const int32_t* __restrict__ seg_start,
                                 const uint32_t* __restrict__ vals, const float4* __restrict__ de,
                                 const int32_t* __restrict__ n_unique, int D4,
                                 float4* __restrict__ rows) {
  const int64_t total = (int64_t)(*n_unique) * D4;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t g0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g0 < total;
       g0 += stride * TG_U) {
    int64_t gg[TG_U];
    int cc[TG_U];
    int32_t bb[TG_U], ee[TG_U];
#pragma unroll
    for (int k = 0; k < TG_U; ++k) {
      gg[k] = g0 + k * stride;
      bb[k] = ee[k] = 0;
      cc[k] = 0;
      if (gg[k] < total) {
        const int64_t u = gg[k] / D4;
        cc[k] = (int)(gg[k] - u * D4);
        bb[k] = seg_start[u];
        ee[k] = seg_start[u + 1];
      }
    }
    uint32_t it[TG_U];
#pragma unroll
    for (int k = 0; k < TG_U; ++k) it[k] = bb[k] < ee[k] ? __ldg(vals + bb[k]) : 0u;
    float4 x[TG_U];
#pragma unroll
    for (int k = 0; k < TG_U; ++k)
      x[k] = bb[k] < ee[k] ? __ldg(de + (int64_t)it[k] * D4 + cc[k]) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < TG_U; ++k) {
      if (gg[k] >= total || ee[k] - bb[k] > TG_LONG) continue;  // long rows: below
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      if (bb[k] < ee[k]) add4(acc, x[k]);
      int32_t p = bb[k] + 1;
      for (; p + TG_PF <= ee[k]; p += TG_PF) {
        uint32_t iq[TG_PF];
#pragma unroll
        for (int q = 0; q < TG_PF; ++q) iq[q] = __ldg(vals + p + q);
        float4 xq[TG_PF];
#pragma unroll
        for (int q = 0; q < TG_PF; ++q) xq[q] = __ldg(de + (int64_t)iq[q] * D4 + cc[k]);
#pragma unroll
        for (int q = 0; q < TG_PF; ++q) add4(acc, xq[q]);
      }
      for (; p < ee[k]; ++p) add4(acc, __ldg(de + (int64_t)vals[p] * D4 + cc[k]));
      rows[gg[k]] = acc;
    }
  }
}

// ---------------------------------------------------------------- vocab build

__global__ void vb_items_kernel(const int64_t* __restrict__ keys_in, int64_t V,
                                uint64_t* __restrict__ keys, uint32_t* __restrict__ vals) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= V) return;
  keys[i] = (uint64_t)keys_in[i];
  vals[i] = (uint32_t)i;
}

__global__ void vb_first_kernel(const uint64_t* __restrict__ keys, const uint32_t* __restrict__ vals,
                                int64_t V, const int32_t* __restrict__ flags,
                                const int32_t* __restrict__ ex, int32_t* __restrict__ first_id) {
  const int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= V) return;
  if (flags[p]) first_id[ex[p]] = (int32_t)vals[p];
}

__global__ void vb_rep_kernel(const uint32_t* __restrict__ vals, int64_t V,
                              const int32_t* __restrict__ flags, const int32_t* __restrict__ ex,
                              const int32_t* __restrict__ first_id, int32_t* __restrict__ rep) {
  const int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= V) return;
  rep[vals[p]] = first_id[ex[p] + flags[p] - 1];
}

__global__ void vb_isfirst_kernel(const int32_t* __restrict__ rep, int64_t V,
                                  int32_t* __restrict__ isfirst) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= V) return;
  isfirst[i] = rep[i] == (int32_t)i ? 1 : 0;
}

__global__ void vb_proj_kernel(const int32_t* __restrict__ rep, const int32_t* __restrict__ cid,
                               int64_t V, int32_t* __restrict__ proj) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= V) return;
  proj[i] = cid[rep[i]];
}

__global__ void vb_flags_kernel(const uint64_t* __restrict__ keys, int64_t n,
                                int32_t* __restrict__ flags) {
  const int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= n) return;
  flags[p] = (p == 0 || keys[p - 1] != keys[p]) ? 1 : 0;
}

inline unsigned nb(int64_t n, int t = 256) { return (unsigned)((n + t - 1) / t); }

struct SortWs {
  uint64_t *k0, *k1;
  uint32_t *v0, *v1;
  int32_t* hist;
  int32_t* a;   // n int32
  int32_t* b;   // n int32
  int32_t* c;   // n + 1 int32
  int32_t* bsum;  // chunk sums of the scans
  int32_t* scal;  // 4 int32
};

constexpr size_t sort_ws_bytes(int64_t n) {
  const int64_t nblocks = (n + TILE - 1) / TILE;
  return 2 * up256(n * 8) + 2 * up256(n * 4) + up256(RADIX_MAX * nblocks * 4 + 4) +
         2 * up256(n * 4 + 4) + up256((n + 1) * 4) + scan_ws_bytes() + 256;
}

SortWs carve(void* ws, int64_t n) {
  const int64_t nblocks = (n + TILE - 1) / TILE;
  char* p = static_cast<char*>(ws);
  SortWs w;
  w.k0 = reinterpret_cast<uint64_t*>(p); p += up256(n * 8);
  w.k1 = reinterpret_cast<uint64_t*>(p); p += up256(n * 8);
  w.v0 = reinterpret_cast<uint32_t*>(p); p += up256(n * 4);
  w.v1 = reinterpret_cast<uint32_t*>(p); p += up256(n * 4);
  w.hist = reinterpret_cast<int32_t*>(p); p += up256(RADIX_MAX * nblocks * 4 + 4);
  w.a = reinterpret_cast<int32_t*>(p); p += up256(n * 4 + 4);
  w.b = reinterpret_cast<int32_t*>(p); p += up256(n * 4 + 4);
  w.c = reinterpret_cast<int32_t*>(p); p += up256((n + 1) * 4);
  w.bsum = reinterpret_cast<int32_t*>(p); p += scan_ws_bytes();
  w.scal = reinterpret_cast<int32_t*>(p);
  return w;
}

}  // namespace

// Rows whose segment is longer than TG_LONG (frequent n-grams; under
// Zipf-distributed tokens a few run to hundreds of tokens), listed by one
// thread per row (the list's order is free: each row has its own output slot).
__global__ void tg_long_list_kernel(const int32_t* __restrict__ seg_start,
                                    const int32_t* __restrict__ n_unique, int32_t* __restrict__ list,
                                    int32_t* __restrict__ count) {
  const int32_t u = blockIdx.x * blockDim.x + threadIdx.x;
  if (u >= *n_unique) return;
  if (seg_start[u + 1] - seg_start[u] > TG_LONG) list[atomicAdd(count, 1)] = u;
}

// One block per long row at a time, its segment in chunks of TG_LONG items:
// the block copies a chunk's rows of de into shared memory (cp.async, 16
// bytes a thread at a time), BUFS chunks in flight, then one thread per 4
// dimensions adds the chunk's rows in order while the next chunks land.  A
// chunk's item ids are read one chunk further ahead, so no copy waits on an
// id load.  The same fp32 sums as tg_reduce_kernel, bit for bit.
constexpr int TG_LONG_THREADS = 256;
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(smem)),
               "l"(gmem)
               : "memory");
}
template <int BUFS>
__global__ void __launch_bounds__(TG_LONG_THREADS) tg_long_reduce_kernel(
    const int32_t* __restrict__ seg_start, const uint32_t* __restrict__ vals,
    const float4* __restrict__ de, const int32_t* __restrict__ list,
    const int32_t* __restrict__ count, int D4, float4* __restrict__ rows) {
  extern __shared__ float4 chunk[];               // [BUFS][TG_LONG * D4]
  __shared__ uint32_t ids[BUFS + 1][TG_LONG];     // item ids of the chunks ahead
  const int n = *count;
  const int tid = threadIdx.x;
  const int CH = TG_LONG * D4;
  for (int li = blockIdx.x; li < n; li += gridDim.x) {
    const int32_t u = list[li];
    const int32_t b = seg_start[u], e = seg_start[u + 1];
    const int nch = (int)((e - b + TG_LONG - 1) / TG_LONG);
    auto load_ids = [&](int q) {  // chunk q's item ids -> ids[q % (BUFS + 1)]
      const int32_t p = b + q * TG_LONG + tid;
      if (q < nch && tid < TG_LONG && p < e) ids[q % (BUFS + 1)][tid] = __ldg(vals + p);
    };
    auto issue = [&](int q) {  // chunk q's rows -> buffer q % BUFS; one group per chunk
      if (q < nch) {
        const int32_t p0 = b + q * TG_LONG;
        const int m = e - p0 < TG_LONG ? (int)(e - p0) : TG_LONG;
        float4* buf = chunk + (q % BUFS) * CH;
        const uint32_t* id = ids[q % (BUFS + 1)];
        for (int i = tid; i < m * D4; i += TG_LONG_THREADS) {
          const int it = i / D4, c = i - it * D4;
          cp_async16(buf + i, de + (int64_t)id[it] * D4 + c);
        }
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
    for (int q = 0; q < BUFS; ++q) load_ids(q);
    __syncthreads();
    for (int q = 0; q < BUFS - 1; ++q) issue(q);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int q = 0; q < nch; ++q) {
      // buffer (q - 1) % BUFS was released at the end of the previous chunk;
      // ids of chunk q + BUFS - 1 were made visible by that barrier too
      issue(q + BUFS - 1);
      load_ids(q + BUFS);  // the slot of chunk q - 1's ids, issued already
      asm volatile("cp.async.wait_group %0;" ::"n"(BUFS - 1) : "memory");
      __syncthreads();  // chunk q has landed for every thread
      if (tid < D4) {
        const int32_t p0 = b + q * TG_LONG;
        const int m = e - p0 < TG_LONG ? (int)(e - p0) : TG_LONG;
        const float4* buf = chunk + (q % BUFS) * CH + tid;
        for (int it = 0; it < m; ++it) add4(acc, buf[it * D4]);
      }
      __syncthreads();  // buffer q % BUFS is free
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    if (tid < D4) rows[(int64_t)u * D4 + tid] = acc;
  }
}

// The whole table gradient in one block for up to TG_SMALL_MAX items (a
// short sequence, a training step on a small batch): the items' (row id,
// item) keys are sorted in shared memory (by rank counting up to TG_RANK_MAX
// items, else by a bitonic network; the item index
// in the low bits keeps equal rows in ascending token order, as the stable
// radix sort does), segment heads are counted by a block scan, and each
// (row, 4 dimensions) sums its segment in that order from +0.  The same sums
// as the multi-kernel path, bit for bit, in one launch instead of ~27.
constexpr int TG_SMALL_MAX = 2048;   // 24 KB of static shared memory
constexpr int TG_SMALL_THREADS = 1024;
constexpr int TG_ITEM_BITS = 12;  // item index < 2^12
constexpr int TG_RANK_MAX = 512;  // up to here, ranks by counting instead of the sorting network

__global__ void __launch_bounds__(TG_SMALL_THREADS) tg_small_kernel(
    const __grid_constant__ HeadParams hp, const int32_t* __restrict__ idx, int n,
    uint64_t sentinel, const float4* __restrict__ de, int D4, int64_t* __restrict__ keys_out,
    float4* __restrict__ rows_out, int32_t* __restrict__ n_unique) {
  __shared__ uint64_t sk[TG_SMALL_MAX];
  __shared__ int32_t seg[TG_SMALL_MAX + 1];
  __shared__ int32_t wsum[TG_SMALL_THREADS / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int np2 = 1;
  while (np2 < n) np2 <<= 1;
  for (int i = tid; i < np2; i += TG_SMALL_THREADS) {
    uint64_t key = ~0ull;  // padding sorts last
    if (i < n) {
      const int j = i % hp.J;
      const int32_t sl = idx[i];
      const uint64_t row = (sl >= 0 && (uint64_t)sl < hp.P[j]) ? (uint64_t)(hp.row_base[j] + sl)
                                                                : sentinel;
      key = (row << TG_ITEM_BITS) | (uint64_t)i;
    }
    sk[i] = key;
  }
  __syncthreads();
  if (n <= TG_RANK_MAX) {
    // few items: each key's sorted position is the number of smaller keys
    // (keys are distinct: the item index is in their low bits); one pass
    // instead of the network's log2(n) (log2(n) + 1) / 2 barrier stages
    uint64_t key = 0;
    int rank = 0;
    if (tid < n) {
      key = sk[tid];
      for (int j = 0; j < n; ++j) rank += sk[j] < key ? 1 : 0;
    }
    __syncthreads();
    if (tid < n) sk[rank] = key;
    __syncthreads();
  } else {
    for (int k = 2; k <= np2; k <<= 1) {
      for (int jj = k >> 1; jj > 0; jj >>= 1) {
        for (int i = tid; i < np2; i += TG_SMALL_THREADS) {
          const int ixj = i ^ jj;
          if (ixj > i) {
            const uint64_t a = sk[i], b = sk[ixj];
            const bool up = (i & k) == 0;
            if ((a > b) == up) {
              sk[i] = b;
              sk[ixj] = a;
            }
          }
        }
        __syncthreads();
      }
    }
  }
  // segment heads over sorted positions, 4 consecutive positions per thread
  constexpr int PER = TG_SMALL_MAX / TG_SMALL_THREADS;
  int heads = 0, valid = 0;
  bool hd[PER];
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    const int p = tid * PER + q;
    hd[q] = false;
    if (p < n) {
      const uint64_t row = sk[p] >> TG_ITEM_BITS;
      if (row != sentinel) {
        ++valid;
        hd[q] = p == 0 || (sk[p - 1] >> TG_ITEM_BITS) != row;
        heads += hd[q] ? 1 : 0;
      }
    }
  }
  int incl = heads, vincl = valid;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(FULL, incl, o), b = __shfl_up_sync(FULL, vincl, o);
    if (lane >= o) {
      incl += a;
      vincl += b;
    }
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int before = 0, all = 0;
  for (int w = 0; w < TG_SMALL_THREADS / 32; ++w) {
    if (w < warp) before += wsum[w];
    all += wsum[w];
  }
  __syncthreads();
  if (lane == 31) wsum[warp] = vincl;
  __syncthreads();
  int n_valid = 0;
  for (int w = 0; w < TG_SMALL_THREADS / 32; ++w) n_valid += wsum[w];
  int h = before + incl - heads;  // exclusive count of heads before this thread's run
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    if (hd[q]) {
      const int p = tid * PER + q;
      seg[h] = p;
      keys_out[h] = (int64_t)(sk[p] >> TG_ITEM_BITS);
      ++h;
    }
  }
  if (tid == 0) {
    seg[all] = n_valid;  // valid items sort first: they end where the sentinel rows begin
    *n_unique = all;
  }
  __syncthreads();
  constexpr uint64_t ITEM_MASK = (1ull << TG_ITEM_BITS) - 1;
  for (int g = tid; g < all * D4; g += TG_SMALL_THREADS) {
    const int u = g / D4, c = g - u * D4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const int pe = seg[u + 1];
    // up to 8 of the segment's rows are loaded before any is added, then
    // added in ascending order (the same sums, without a round trip each)
    for (int p = seg[u]; p < pe; p += 8) {
      float4 a[8];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (p + q < pe) a[q] = __ldg(de + (int64_t)(sk[p + q] & ITEM_MASK) * D4 + c);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (p + q < pe) add4(acc, a[q]);
    }
    rows_out[g] = acc;
  }
}

size_t table_grad_ws_bytes(int64_t n_items) { return sort_ws_bytes(n_items); }

int launch_table_grad(const HeadParams& hp, const int32_t* idx, const float* de, int64_t n_tok,
                      int64_t* keys_out, float* rows_out, int32_t* n_unique, void* ws,
                      size_t ws_bytes, cudaStream_t s) {
  const int64_t n = n_tok * hp.J;
  if (ws_bytes < sort_ws_bytes(n)) return ENGRAM_ERR_WORKSPACE;
  if (n == 0) return ck(cudaMemsetAsync(n_unique, 0, sizeof(int32_t), s));
  const uint64_t sentinel = (uint64_t)(hp.row_base[hp.J - 1] + (int64_t)hp.P[hp.J - 1]);
  if (n <= TG_SMALL_MAX) {
    tg_small_kernel<<<1, TG_SMALL_THREADS, 0, s>>>(
        hp, idx, (int)n, sentinel, reinterpret_cast<const float4*>(de), hp.D_h / 4, keys_out,
        reinterpret_cast<float4*>(rows_out), n_unique);
    return ck(cudaGetLastError());
  }
  SortWs w = carve(ws, n);
  tg_items_kernel<<<nb(n), 256, 0, s>>>(hp, idx, n, sentinel, w.k0, w.v0);
  uint64_t* k = w.k0;
  uint32_t* v = w.v0;
  int rc = radix_sort_pairs(k, v, w.k1, w.v1, n, bits_for(sentinel), w.hist, w.bsum, s);
  if (rc) return rc;
  tg_flags_kernel<<<nb(n), 256, 0, s>>>(k, n, sentinel, w.a);
  rc = launch_scan(w.a, w.b, n, n_unique, w.bsum, s);
  if (rc) return rc;
  // seg_start needs n_unique + 1 entries; with no valid item it stays empty
  tg_heads_kernel<<<nb(n), 256, 0, s>>>(k, n, sentinel, w.b, w.c, keys_out);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int D4 = hp.D_h / 4;  // D_h * 4 bytes is a multiple of 16 (checked with the config)
  int64_t blocks = nb(n * D4);
  if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
  tg_reduce_kernel<<<(unsigned)blocks, 256, 0, s>>>(w.c, v, reinterpret_cast<const float4*>(de),
                                                    n_unique, D4,
                                                    reinterpret_cast<float4*>(rows_out));
  // long segments: w.a (the flags, free after the heads) holds their list,
  // w.scal[2] its length
  int32_t* long_count = w.scal + 2;
  if ((rc = ck(cudaMemsetAsync(long_count, 0, sizeof(int32_t), s)))) return rc;
  tg_long_list_kernel<<<nb(n), 256, 0, s>>>(w.c, n_unique, w.a, long_count);
  // as many chunk buffers (4, 2 or 1) as 220 KB of shared memory holds
  const size_t chunk_bytes = (size_t)TG_LONG * D4 * sizeof(float4);
  if (D4 > TG_LONG_THREADS || chunk_bytes > 220 * 1024) return ENGRAM_ERR_UNSUPPORTED;
  const int bufs = 4 * chunk_bytes <= 220 * 1024 ? 4 : 2 * chunk_bytes <= 220 * 1024 ? 2 : 1;
  const size_t long_smem = bufs * chunk_bytes;
  const float4* de4 = reinterpret_cast<const float4*>(de);
  float4* rows4 = reinterpret_cast<float4*>(rows_out);
  auto run_long = [&](auto kern) -> int {
    if (long_smem > 48 * 1024 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)long_smem) != cudaSuccess)
      return (int)ENGRAM_ERR_CUDA;
    kern<<<(unsigned)sms, TG_LONG_THREADS, long_smem, s>>>(w.c, v, de4, w.a, long_count, D4,
                                                           rows4);
    return ck(cudaGetLastError());
  };
  return bufs == 4   ? run_long(tg_long_reduce_kernel<4>)
         : bufs == 2 ? run_long(tg_long_reduce_kernel<2>)
                     : run_long(tg_long_reduce_kernel<1>);
}

size_t vocab_ws_bytes(int64_t V) { return sort_ws_bytes(V); }

// ------------------------------------------------------- hot rows of a sample
//
// The rows a sample of hash indices addresses most often: the candidates for
// an HBM cache in front of a host-memory table (the pages' multi-level cache
// keeps the frequent n-grams' rows near the GPU, relying on their Zipfian
// frequencies).  Rows are ranked by how many (token, head) pairs address
// them, ties by ascending row id, so the ranking is a pure function of the
// sample.  The same sort as the table gradient finds each distinct row and
// its count; a second stable sort by descending count keeps ascending row
// order among equal counts.

namespace {

// key of distinct row u: a count-descending order; past n_unique: last
__global__ void hot_count_kernel(const int32_t* __restrict__ seg_start,
                                 const int32_t* __restrict__ n_unique, int64_t n,
                                 uint64_t* __restrict__ keys, uint32_t* __restrict__ vals) {
  const int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (u >= n) return;
  const int32_t U = *n_unique;
  const uint32_t cnt = u < U ? (uint32_t)(seg_start[u + 1] - seg_start[u]) : 0u;
  keys[u] = 0xffffffffull - cnt;  // cnt >= 1 for every distinct row
  vals[u] = (uint32_t)u;
}

__global__ void hot_out_kernel(const int64_t* __restrict__ ukeys, const uint32_t* __restrict__ order,
                               const int32_t* __restrict__ n_unique, int64_t C,
                               int64_t* __restrict__ rows_out, int32_t* __restrict__ n_out) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int32_t U = *n_unique;
  if (i == 0) *n_out = (int32_t)(C < U ? C : U);
  if (i >= C) return;
  rows_out[i] = i < U ? ukeys[order[i]] : -1;
}

}  // namespace

size_t hot_rows_ws_bytes(int64_t n_items) { return sort_ws_bytes(n_items) + up256(n_items * 8); }

int launch_hot_rows(const HeadParams& hp, const int32_t* idx, int64_t n_tok, int64_t C,
                    int64_t* rows_out, int32_t* n_out, void* ws, size_t ws_bytes, cudaStream_t s) {
  const int64_t n = n_tok * hp.J;
  if (ws_bytes < hot_rows_ws_bytes(n)) return ENGRAM_ERR_WORKSPACE;
  if (n == 0 || C == 0) {
    int rc = ck(cudaMemsetAsync(n_out, 0, sizeof(int32_t), s));
    if (rc || C == 0) return rc;
    return ck(cudaMemsetAsync(rows_out, 0xff, (size_t)C * sizeof(int64_t), s));  // all -1
  }
  const uint64_t sentinel = (uint64_t)(hp.row_base[hp.J - 1] + (int64_t)hp.P[hp.J - 1]);
  SortWs w = carve(ws, n);
  int64_t* ukeys = reinterpret_cast<int64_t*>(static_cast<char*>(ws) + sort_ws_bytes(n));
  int32_t* n_unique = w.scal + 3;
  tg_items_kernel<<<nb(n), 256, 0, s>>>(hp, idx, n, sentinel, w.k0, w.v0);
  uint64_t* k = w.k0;
  uint32_t* v = w.v0;
  uint64_t* k_alt = w.k1;
  uint32_t* v_alt = w.v1;
  int rc = radix_sort_pairs(k, v, k_alt, v_alt, n, bits_for(sentinel), w.hist, w.bsum, s);
  if (rc) return rc;
  tg_flags_kernel<<<nb(n), 256, 0, s>>>(k, n, sentinel, w.a);
  if ((rc = launch_scan(w.a, w.b, n, n_unique, w.bsum, s))) return rc;
  tg_heads_kernel<<<nb(n), 256, 0, s>>>(k, n, sentinel, w.b, w.c, ukeys);
  // the sorted items are no longer needed: their buffers take the second sort
  uint64_t* k2 = w.k0;
  uint32_t* v2 = w.v0;
  uint64_t* k2_alt = w.k1;
  uint32_t* v2_alt = w.v1;
  hot_count_kernel<<<nb(n), 256, 0, s>>>(w.c, n_unique, n, k2, v2);
  if ((rc = radix_sort_pairs(k2, v2, k2_alt, v2_alt, n, 32, w.hist, w.bsum, s))) return rc;
  hot_out_kernel<<<nb(C > 0 ? C : 1), 256, 0, s>>>(ukeys, v2, n_unique, C, rows_out, n_out);
  return ck(cudaGetLastError());
}


// ------------------------------------------------- table gradient without allocation
//
// For callers that cannot allocate device memory themselves (a host that
// hands this library a fixed pool, or a plugin whose host framework owns
// every allocation), the sparse table gradient can run on a scratch
// array that is part of the library image: the GPU reserves it when the
// library's device code is loaded and keeps it until the process exits.  It
// holds the sort buffers for up to ENGRAM_NOALLOC_MAX_ITEMS (token, head)
// pairs.  Every call reuses the same array: calls that overlap on the GPU
// (different streams, or different host threads on one device) race and
// must be serialised by the caller.  No word of the array has to start at
// zero: each pass writes everything it reads.

namespace {

constexpr size_t kNoAllocScratchBytes = sort_ws_bytes(ENGRAM_NOALLOC_MAX_ITEMS);
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {nullptr};
std::mutex g_noalloc_mu;

// Device address of the scratch array on the current device.  Host code only
// sees a host-side stand-in under the array's name, so the address is taken
// once per device with that device current.
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices)
    return ENGRAM_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
      cudaGetLastError();
      return ENGRAM_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return ENGRAM_OK;
}

}  // namespace

int launch_table_grad_noalloc(const HeadParams& hp, const int32_t* idx, const float* de,
                              int64_t n_tok, int64_t* keys, float* rows, int32_t* n_unique,
                              cudaStream_t s) {
  if (n_tok < 0 || n_tok > ENGRAM_NOALLOC_MAX_ITEMS / hp.J) return ENGRAM_ERR_TOO_LARGE;
  void* scratch = nullptr;
  const int rc = noalloc_scratch(&scratch);
  if (rc) return rc;
  return launch_table_grad(hp, idx, de, n_tok, keys, rows, n_unique, scratch, kNoAllocScratchBytes,
                           s);
}

int launch_vocab_proj(const int64_t* keys, int32_t V, int32_t* proj, int32_t* V_c_out, void* ws,
                      size_t ws_bytes, cudaStream_t s) {
  if (ws_bytes < sort_ws_bytes(V)) return ENGRAM_ERR_WORKSPACE;
  SortWs w = carve(ws, V);
  vb_items_kernel<<<nb(V), 256, 0, s>>>(keys, V, w.k0, w.v0);
  uint64_t* k = w.k0;
  uint32_t* v = w.v0;
  int rc = radix_sort_pairs(k, v, w.k1, w.v1, V, 64, w.hist, w.bsum, s);
  if (rc) return rc;
  vb_flags_kernel<<<nb(V), 256, 0, s>>>(k, V, w.a);
  rc = launch_scan(w.a, w.b, V, w.scal, w.bsum, s);
  if (rc) return rc;
  // w.c: first raw id of each group, then reused below
  vb_first_kernel<<<nb(V), 256, 0, s>>>(k, v, V, w.a, w.b, w.c);
  int32_t* rep = reinterpret_cast<int32_t*>(k == w.k0 ? w.k1 : w.k0);  // free after the sort
  vb_rep_kernel<<<nb(V), 256, 0, s>>>(v, V, w.a, w.b, w.c, rep);
  vb_isfirst_kernel<<<nb(V), 256, 0, s>>>(rep, V, w.a);
  rc = launch_scan(w.a, w.b, V, w.scal + 1, w.bsum, s);
  if (rc) return rc;
  vb_proj_kernel<<<nb(V), 256, 0, s>>>(rep, w.b, V, proj);
  int32_t vc = 0;
  int e = ck(cudaMemcpyAsync(&vc, w.scal + 1, sizeof(int32_t), cudaMemcpyDeviceToHost, s));
  if (e) return e;
  e = ck(cudaStreamSynchronize(s));
  if (e) return e;
  *V_c_out = vc;
  return ck(cudaGetLastError());
}

}  // namespace engram
