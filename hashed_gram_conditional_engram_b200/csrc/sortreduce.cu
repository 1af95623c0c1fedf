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

constexpr int RADIX_BITS = 8;
constexpr int RADIX = 1 << RADIX_BITS;
constexpr int SORT_THREADS = 256;
constexpr int SORT_WARPS = SORT_THREADS / 32;
constexpr int CHUNKS_PER_WARP = 8;                       // 8 x 32 items per warp
constexpr int TILE = SORT_THREADS * CHUNKS_PER_WARP;     // 2048 items per block
constexpr unsigned FULL = 0xffffffffu;

constexpr size_t up256(size_t b) { return (b + 255) & ~(size_t)255; }

__device__ __forceinline__ int digit_of(uint64_t key, int shift) {
  return (int)((key >> shift) & (RADIX - 1));
}

// Counts of each digit in this block's tile -> hist[digit * nblocks + block].
__global__ void __launch_bounds__(SORT_THREADS) radix_hist_kernel(const uint64_t* __restrict__ keys,
                                                                  int64_t n, int shift,
                                                                  int32_t* __restrict__ hist) {
  __shared__ int32_t cnt[RADIX];
  for (int i = threadIdx.x; i < RADIX; i += SORT_THREADS) cnt[i] = 0;
  __syncthreads();
  const int64_t base = (int64_t)blockIdx.x * TILE;
  for (int i = threadIdx.x; i < TILE; i += SORT_THREADS) {
    const int64_t p = base + i;
    if (p < n) atomicAdd(&cnt[digit_of(keys[p], shift)], 1);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < RADIX; i += SORT_THREADS)
    hist[(int64_t)i * gridDim.x + blockIdx.x] = cnt[i];
}

// Stable scatter: item order inside the tile is (warp, chunk, lane); each
// item's destination = start of its digit for this block + items of the same
// digit before it in that order.
__global__ void __launch_bounds__(SORT_THREADS) radix_scatter_kernel(
    const uint64_t* __restrict__ keys_in, const uint32_t* __restrict__ vals_in, int64_t n,
    int shift, const int32_t* __restrict__ offsets, uint64_t* __restrict__ keys_out,
    uint32_t* __restrict__ vals_out) {
  __shared__ int32_t wcnt[SORT_WARPS][RADIX];
  __shared__ int32_t boff[RADIX];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < SORT_WARPS * RADIX; i += SORT_THREADS) (&wcnt[0][0])[i] = 0;
  for (int i = threadIdx.x; i < RADIX; i += SORT_THREADS)
    boff[i] = offsets[(int64_t)i * gridDim.x + blockIdx.x];
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
    const int d = ok ? digit_of(k[c], shift) : RADIX;  // RADIX marks "no item"
    dg[c] = d;
    const unsigned peers = __match_any_sync(FULL, d);
    const int before = (d < RADIX) ? wcnt[warp][d] : 0;
    rk[c] = before + __popc(peers & lt_mask);
    __syncwarp();
    if (d < RADIX && (peers & lt_mask) == 0) wcnt[warp][d] = before + __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // exclusive prefix over warps, per digit
  for (int d = threadIdx.x; d < RADIX; d += SORT_THREADS) {
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
    if (dg[c] < RADIX) {
      const int64_t dst = (int64_t)boff[dg[c]] + wcnt[warp][dg[c]] + rk[c];
      keys_out[dst] = k[c];
      vals_out[dst] = v[c];
    }
  }
}

// Exclusive scan of int32 x[0..n) into y (may alias x), total into *total
// (if non-null).  One block of 1024 threads: each thread owns a contiguous
// run, the run sums are scanned across the block.
__global__ void __launch_bounds__(1024) scan_kernel(const int32_t* x, int32_t* y, int64_t n,
                                                    int32_t* total) {
  __shared__ int32_t wsum[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t per = (n + 1023) / 1024;
  const int64_t lo = tid * per;
  const int64_t hi = lo + per < n ? lo + per : n;
  int32_t s = 0;
  for (int64_t i = lo; i < hi; ++i) s += x[i];
  // inclusive scan of s over the block
  int32_t incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t t = __shfl_up_sync(FULL, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int32_t w = wsum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t t = __shfl_up_sync(FULL, w, o);
      if (lane >= o) w += t;
    }
    wsum[lane] = w;
  }
  __syncthreads();
  int32_t run = incl - s + (warp > 0 ? wsum[warp - 1] : 0);
  for (int64_t i = lo; i < hi; ++i) {
    const int32_t t = x[i];
    y[i] = run;
    run += t;
  }
  if (total != nullptr && tid == 1023) *total = run;
}

int radix_sort_pairs(uint64_t*& keys, uint32_t*& vals, uint64_t* keys_alt, uint32_t* vals_alt,
                     int64_t n, int key_bits, int32_t* hist, cudaStream_t s) {
  if (n == 0) return ENGRAM_OK;
  const int64_t nblocks = (n + TILE - 1) / TILE;
  for (int shift = 0; shift < key_bits; shift += RADIX_BITS) {
    radix_hist_kernel<<<(unsigned)nblocks, SORT_THREADS, 0, s>>>(keys, n, shift, hist);
    scan_kernel<<<1, 1024, 0, s>>>(hist, hist, (int64_t)RADIX * nblocks, nullptr);
    radix_scatter_kernel<<<(unsigned)nblocks, SORT_THREADS, 0, s>>>(keys, vals, n, shift, hist,
                                                                    keys_alt, vals_alt);
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

// One thread per (row, dimension): fp32 sum from +0 over the row's items in
// sorted (= ascending token) order.  de of item i = n*J + j starts at
// i * D_h because E = J * D_h.
__global__ void tg_reduce_kernel(const int32_t* __restrict__ seg_start,
                                 const uint32_t* __restrict__ vals, const float* __restrict__ de,
                                 const int32_t* __restrict__ n_unique, int D_h,
                                 float* __restrict__ rows) {
  const int64_t total = (int64_t)(*n_unique) * D_h;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < total; g += stride) {
    const int64_t u = g / D_h;
    const int c = (int)(g - u * D_h);
    const int32_t b = seg_start[u], e = seg_start[u + 1];
    float acc = 0.0f;
    for (int32_t p = b; p < e; ++p) acc = acc + __ldg(de + (int64_t)vals[p] * D_h + c);
    rows[g] = acc;
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
  int32_t* scal;  // 4 int32
};

constexpr size_t sort_ws_bytes(int64_t n) {
  const int64_t nblocks = (n + TILE - 1) / TILE;
  return 2 * up256(n * 8) + 2 * up256(n * 4) + up256(RADIX * nblocks * 4 + 4) +
         2 * up256(n * 4 + 4) + up256((n + 1) * 4) + 256;
}

SortWs carve(void* ws, int64_t n) {
  const int64_t nblocks = (n + TILE - 1) / TILE;
  char* p = static_cast<char*>(ws);
  SortWs w;
  w.k0 = reinterpret_cast<uint64_t*>(p); p += up256(n * 8);
  w.k1 = reinterpret_cast<uint64_t*>(p); p += up256(n * 8);
  w.v0 = reinterpret_cast<uint32_t*>(p); p += up256(n * 4);
  w.v1 = reinterpret_cast<uint32_t*>(p); p += up256(n * 4);
  w.hist = reinterpret_cast<int32_t*>(p); p += up256(RADIX * nblocks * 4 + 4);
  w.a = reinterpret_cast<int32_t*>(p); p += up256(n * 4 + 4);
  w.b = reinterpret_cast<int32_t*>(p); p += up256(n * 4 + 4);
  w.c = reinterpret_cast<int32_t*>(p); p += up256((n + 1) * 4);
  w.scal = reinterpret_cast<int32_t*>(p);
  return w;
}

}  // namespace

size_t table_grad_ws_bytes(int64_t n_items) { return sort_ws_bytes(n_items); }

int launch_table_grad(const HeadParams& hp, const int32_t* idx, const float* de, int64_t n_tok,
                      int64_t* keys_out, float* rows_out, int32_t* n_unique, void* ws,
                      size_t ws_bytes, cudaStream_t s) {
  const int64_t n = n_tok * hp.J;
  if (ws_bytes < sort_ws_bytes(n)) return ENGRAM_ERR_WORKSPACE;
  if (n == 0) return ck(cudaMemsetAsync(n_unique, 0, sizeof(int32_t), s));
  SortWs w = carve(ws, n);
  const uint64_t sentinel = (uint64_t)(hp.row_base[hp.J - 1] + (int64_t)hp.P[hp.J - 1]);
  tg_items_kernel<<<nb(n), 256, 0, s>>>(hp, idx, n, sentinel, w.k0, w.v0);
  uint64_t* k = w.k0;
  uint32_t* v = w.v0;
  int rc = radix_sort_pairs(k, v, w.k1, w.v1, n, bits_for(sentinel), w.hist, s);
  if (rc) return rc;
  tg_flags_kernel<<<nb(n), 256, 0, s>>>(k, n, sentinel, w.a);
  scan_kernel<<<1, 1024, 0, s>>>(w.a, w.b, n, n_unique);
  // seg_start needs n_unique + 1 entries; with no valid item it stays empty
  tg_heads_kernel<<<nb(n), 256, 0, s>>>(k, n, sentinel, w.b, w.c, keys_out);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = nb(n * hp.D_h);
  if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
  tg_reduce_kernel<<<(unsigned)blocks, 256, 0, s>>>(w.c, v, de, n_unique, hp.D_h, rows_out);
  return ck(cudaGetLastError());
}

size_t vocab_ws_bytes(int64_t V) { return sort_ws_bytes(V); }

// ------------------------------------------------- table gradient without allocation
//
// For callers that cannot allocate device memory themselves (a host that
// hands this library a fixed pool, code running inside a CUDA graph capture
// where allocation calls are not allowed, or a plugin whose host framework
// owns every allocation), the sparse table gradient can run on a scratch
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
  if (n_tok * hp.J > ENGRAM_NOALLOC_MAX_ITEMS) return ENGRAM_ERR_TOO_LARGE;
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
  int rc = radix_sort_pairs(k, v, w.k1, w.v1, V, 64, w.hist, s);
  if (rc) return rc;
  vb_flags_kernel<<<nb(V), 256, 0, s>>>(k, V, w.a);
  scan_kernel<<<1, 1024, 0, s>>>(w.a, w.b, V, w.scal);
  // w.c: first raw id of each group, then reused below
  vb_first_kernel<<<nb(V), 256, 0, s>>>(k, v, V, w.a, w.b, w.c);
  int32_t* rep = reinterpret_cast<int32_t*>(k == w.k0 ? w.k1 : w.k0);  // free after the sort
  vb_rep_kernel<<<nb(V), 256, 0, s>>>(v, V, w.a, w.b, w.c, rep);
  vb_isfirst_kernel<<<nb(V), 256, 0, s>>>(rep, V, w.a);
  scan_kernel<<<1, 1024, 0, s>>>(w.a, w.b, V, w.scal + 1);
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
