// Internal declarations shared by the translation units of libengram_b200.so.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <nvtx3/nvToolsExt.h>

#include "../../include/engram.h"

namespace engram {

// An NVTX range named after the entry point around each call of the C ABI,
// so a timeline (Nsight Systems, Nsight Compute's NVTX filters) shows which
// call issued which kernels.  The NVTX header does nothing unless a tool is
// attached to the process.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Per-head constants handed to kernels by value.
struct HeadParams {
  int J, K, D_h, E;
  int32_t V_raw, V_c;
  uint64_t mult[ENGRAM_MAX_HEADS][3];
  uint64_t P[ENGRAM_MAX_HEADS];
  uint64_t mu[ENGRAM_MAX_HEADS];        // floor((2^64 - 1) / P_j), Barrett reciprocal
  int64_t row_base[ENGRAM_MAX_HEADS];   // first packed-table row of head j
};

HeadParams make_head_params(const engram_cfg_t* cfg);

// The device status word of the current device (a __device__ variable).
unsigned int* status_ptr();

inline int ck(cudaError_t e) { return e == cudaSuccess ? ENGRAM_OK : ENGRAM_ERR_CUDA; }

__device__ __forceinline__ float bf2f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float bfbits2f(uint16_t b) {
  return __uint_as_float(((uint32_t)b) << 16);
}

// ---------------------------------------------------------------- stream order
// Programmatic dependent launch.  Every kernel of the library calls
// wait_prior_grid() before it reads anything that an earlier kernel on its
// stream wrote: it blocks until the kernel launched before this one has
// completed and its writes are visible (a no-op for a kernel launched
// without the attribute).  Since every kernel waits so, completion is
// transitive along the stream, and allow_dependents() may let the next
// kernel start its prologue while this one still runs.
__device__ __forceinline__ void allow_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void wait_prior_grid() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Launch with programmatic stream serialisation allowed (see above).
template <typename... KArgs, typename... Args>
int launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
               Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return ck(cudaLaunchKernelEx(&cfg, kern, args...));
}

// ---------------------------------------------------------------- launches
int launch_hash(const HeadParams& hp, const int32_t* proj, const int32_t* ids, int B, int T,
                int32_t* ngram_state, int32_t* idx, cudaStream_t s);
// zero_counters (may be NULL): two ints set to zero before the gather ends
// (the counters of the decode kernel launched after it)
int launch_gather(const HeadParams& hp, const int32_t* idx, const void* table, int64_t n_tok,
                  int elem_bytes, void* e, cudaStream_t s, int* zero_counters = nullptr);
// one decode step's hash (rolling n-gram state, idx optional) and gather in
// one launch, B sequences of one token
// zero_counters (may be NULL): two ints set to zero by the kernel (the
// counters of the decode kernel launched after it)
int launch_hash_gather_decode(const HeadParams& hp, const int32_t* proj, const int32_t* ids,
                              int64_t B, int32_t* ngram_state, int32_t* idx, const void* table,
                              int elem_bytes, void* e, int* zero_counters, cudaStream_t s);
// the same gather from pinned host memory: a small fixed grid, deep per-thread
// load queues (PCIe latency), the GPU's other SMs left free
int launch_gather_host(const HeadParams& hp, const int32_t* idx, const void* table, int64_t n_tok,
                       int elem_bytes, void* e, cudaStream_t s);

// fp32 CUDA-core path (small layers)
struct F32Saved {
  float* alpha;   // [N, M]
  float* k;       // [N, M, d]
  float* v;       // [N, d]
  float* y;       // [N, M, d]
};
F32Saved f32_saved_layout(void* base, int64_t N, int M, int d);
size_t f32_saved_bytes(int64_t N, int M, int d);
size_t f32_forward_ws_bytes(int64_t N, int M, int d);
// params: the small-parameter block of the layer's flags (conv weights,
// then the norm scales); dparams its gradient in the same layout
int64_t f32_param_floats(int flags, int M, int d);
int launch_forward_f32(const float* e, const float* h, const float* Wk, const float* Wv,
                       const float* params, int flags, float* conv_state, float* out,
                       float* saved, int64_t N, int T, int M, int d, int E, void* ws,
                       cudaStream_t s);
size_t backward_f32_ws_bytes(int64_t N, int M, int d, int E);
float* backward_f32_de_slot(void* ws, int64_t N, int M, int d, int E);
int launch_backward_f32(const float* e, const float* h, const float* Wk, const float* Wv,
                        const float* params, int flags, F32Saved sv, const float* dout, float* dh,
                        float* dWk, float* dWv, float* dparams, float* de, int64_t N, int T, int M,
                        int d, int E, void* ws, cudaStream_t s);

// sort / scan / segmented reduce
size_t table_grad_ws_bytes(int64_t n_items);
int launch_table_grad(const HeadParams& hp, const int32_t* idx, const float* de, int64_t n_tok,
                      int64_t* keys, float* rows, int32_t* n_unique, void* ws, size_t ws_bytes,
                      cudaStream_t s);
size_t vocab_ws_bytes(int64_t V);
// HBM cache of host-table rows: fill the cache and its row -> slot map; gather
// e from the cache (hits) and host memory (the listed misses)
int launch_cache_fill(const HeadParams& hp, const void* host, const int64_t* rows, int64_t C,
                      int elem_bytes, void* cache, int32_t* map, cudaStream_t s);
size_t cached_gather_ws_bytes(int64_t n_tok, int J);
int launch_gather_cached(const HeadParams& hp, const int32_t* idx, const void* host,
                         const void* cache, const int32_t* map, int64_t n_tok, int elem_bytes,
                         void* e, int32_t* n_miss_out, void* ws, cudaStream_t s);
// the C rows a sample of indices addresses most often (ties: lower row id)
size_t hot_rows_ws_bytes(int64_t n_items);
int launch_hot_rows(const HeadParams& hp, const int32_t* idx, int64_t n_tok, int64_t C,
                    int64_t* rows_out, int32_t* n_out, void* ws, size_t ws_bytes, cudaStream_t s);
int launch_table_grad_noalloc(const HeadParams& hp, const int32_t* idx, const float* de,
                              int64_t n_tok, int64_t* keys, float* rows, int32_t* n_unique,
                              cudaStream_t s);
int launch_vocab_proj(const int64_t* keys, int32_t V, int32_t* proj, int32_t* V_c_out, void* ws,
                      size_t ws_bytes, cudaStream_t s);

// bf16 tensor-core GEMMs with fp32 output (gemm_tc.cu); shapes: d a
// multiple of 256, E of 64, W_k and W_v [d, E], token rows for the rest.
int gemm_supported(int64_t N, int d, int E);
// C [N, 2d] (rows ldc floats apart) = e [W_k; W_v]^T, or C [N, d] = e W_v^T
// when Wk is NULL
// stall: ENGRAM_TEST_STALL (the B producer issues nothing, 1 ms waits)
int launch_gemm_kv(const __nv_bfloat16* e, const __nv_bfloat16* Wk, const __nv_bfloat16* Wv,
                   int64_t N, int d, int E, float* C, int64_t ldc, cudaStream_t s,
                   bool stall = false);
// dW_k [d, E] and dW_v [d, E] = [dk | dv]^T e over the N tokens (dkv bf16
// [N, 2d]); ws: gemm_dw_ws_bytes of tile counters
size_t gemm_dw_ws_bytes(int d, int E);
int launch_gemm_dw(const __nv_bfloat16* dkv, const __nv_bfloat16* e, int64_t N, int d, int E,
                   float* dWk, float* dWv, void* ws, cudaStream_t s, bool stall = false);
// de [N, E] = [dk | dv] [W_k; W_v]
int launch_gemm_de(const __nv_bfloat16* dkv, const __nv_bfloat16* Wk, const __nv_bfloat16* Wv,
                   int64_t N, int d, int E, float* de, cudaStream_t s, bool stall = false);

// pre-conv RMSNorm of bf16 layers: rc[t] = (alpha_t^2 <v_t, v_t> / d + eps)^(-1/2)
int launch_prenorm_rc(const float* v, int ldv, const float* alpha, int64_t N, int d, float* rc,
                      cudaStream_t s);
// after the gate: v = e W_v^T into vbuf (fp32, rows ldv apart), rc, then the
// conv over c = alpha rc g_v v with out = h + alpha v + SiLU(y) (decode when
// conv_state is given)
struct PrenormFwd {
  const float* gv;  // g_v [d], or NULL (ones)
  float* vbuf;
  int ldv;
  float* rc;        // [N]
};
int launch_prenorm_tail(const PrenormFwd& p, const __nv_bfloat16* e, const __nv_bfloat16* Wv,
                        const __nv_bfloat16* h, const float* conv_w, const float* alpha,
                        float* conv_state, __nv_bfloat16* out, int dil, int64_t N, int T, int d,
                        int E, bool stall, cudaStream_t s);

// bf16 backward (one branch): elementwise kernels and the tensor-core GEMMs
// kv_saved: the forward's fp32 [N, 2d] k and v, or NULL to recompute them
size_t backward_bf16_ws_bytes(int64_t N, int d, int E, int J, bool kv_saved, bool scaled,
                              bool prenorm);
// gscale: the learnable norm scales g_h [d], g_k [d] (NULL: none); their
// gradients go to dconv_w + 4 d.  dil: the conv's dilation, 1 or 3.
// prenorm: the conv reads RMSNorm(vt) g_v (gv = g_v, or NULL for ones; its
// gradient goes to dconv_w + 6 d when gscale is given)
int launch_backward_bf16(const HeadParams& hp, const int32_t* idx, const __nv_bfloat16* e,
                         const __nv_bfloat16* h, const __nv_bfloat16* Wk,
                         const __nv_bfloat16* Wv, const float* conv_w, const float* gscale,
                         const float* alpha, const float* kv_saved, const float* dout, float* dh,
                         float* dWk, float* dWv, float* dconv_w, float* de, int64_t* dtab_keys,
                         float* dtab_rows, int32_t* n_unique, int64_t N, int T, int d, int dil,
                         bool prenorm, const float* gv, void* ws, size_t ws_bytes, bool stall,
                         cudaStream_t s);

// bf16 tensor-core path (sm_100a tcgen05)
size_t tc_forward_ws_bytes(int64_t N, int d, int E);
// one decode step's passes, gate, conv and residual in one persistent launch
// (bf16; part and alpha: the layout of tc_forward_ws_bytes for N <= 4096)
bool decode_fused_ok(int64_t N, int d, int E);
int launch_decode_fused(const __nv_bfloat16* e, const __nv_bfloat16* h, const __nv_bfloat16* Wk,
                        const __nv_bfloat16* Wv, const float* conv_w, float* conv_state,
                        __nv_bfloat16* out, float* alpha_saved, const float* gg, int dil,
                        int64_t N, int d, int E, float4* part, float* alpha, int* counters,
                        bool counters_zeroed, bool chained, bool stall, cudaStream_t s);
int tc_supported(int d, int E, int M);
// gg[f] = gh[f] * gk[f] (the learnable norm scales' product the gate uses)
int launch_scale_product(const float* gh, const float* gk, int d, float* gg, cudaStream_t s);
int launch_forward_tc(const __nv_bfloat16* e, const __nv_bfloat16* h, const __nv_bfloat16* Wk,
                      const __nv_bfloat16* Wv, const float* conv_w, float* conv_state,
                      __nv_bfloat16* out, float* alpha_saved, float* kv_save, const float* gg,
                      int dil, int64_t N, int T, int d, int E, void* ws, size_t ws_bytes,
                      bool chained, const PrenormFwd* pn, bool stall, cudaStream_t s);

}  // namespace engram
