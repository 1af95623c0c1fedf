/*
 * engram.h -- C ABI of libengram_b200.so, the Engram conditional-memory layer
 * on B200 (sm_100a).
 *
 * The layer ("Conditional Memory via Scalable Lookup: A New Axis of Sparsity
 * for Large Language Models", as summarised by the pages cited below) does,
 * for every token position t of every sequence:
 *   1. compress the raw id through a vocabulary projection,
 *   2. form the suffix 2-gram and 3-gram of compressed ids,
 *   3. hash each n-gram through K independent heads into per-head tables,
 *   4. gather and concatenate the J = 2K head rows into e_t,
 *   5. gate a value projection by alpha_t = sigmoid(<RMSNorm(h_t), RMSNorm(W_k e_t)>/sqrt(d)),
 *   6. pass alpha_t * W_v e_t through a width-4 depthwise causal conv with SiLU
 *      and add both onto the residual stream:
 *        out_t = h_t + vt_t + SiLU(sum_i w[:, i] * vt_{t-3+i}),  vt = alpha * W_v e.
 *
 * Page citations used below:
 *   [p1] reportify.cn tag page 条件记忆, digests 技术方案 / 技术创新与架构 / 关键技术
 *   [p2] sechub.in answer: 2-/3-gram suffixes, gate, short depthwise causal conv,
 *        indices known before the forward pass, host-memory prefetch
 *   [p4] gitcode.csdn.net blog, "Engram 到底怎么工作的": 第一步 .. 第四步,
 *        end-to-end training with consistent slot gradients, offload to DRAM
 *   [p5] discuss.deepseek.club, 二.1 (1) hash retrieval, 二.1 (2) gate and conv,
 *        二.2 multi-branch integration and host prefetch
 *
 * Conventions for every call:
 *   - All device pointers are raw CUDA device addresses, 16-byte aligned.
 *     Host pointers are named so.  The caller owns every buffer; the library
 *     allocates no device memory and keeps no state besides one device status
 *     word per device (and the built-in scratch array that
 *     engram_table_grad_noalloc sorts in).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are asynchronous and never synchronise, except
 *     engram_build_vocab_proj (returns V_c on the host) and engram_get_status.
 *   - Return value: ENGRAM_OK (0) or a negative ENGRAM_ERR_* code.  Host-side
 *     argument errors launch nothing.  Data errors found on the device (a raw
 *     id outside [0, V_raw), a row index outside its table) never trap: the
 *     kernel writes idx = -1 / a zero row and sets a bit of the status word,
 *     read and cleared by engram_get_status.
 *   - Layouts are row-major, the last index fastest.  Token order is flat:
 *     token n = b*T + t.
 */
#ifndef ENGRAM_B200_H
#define ENGRAM_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ENGRAM_MAX_HEADS 32 /* J = 2K <= 32 */
#define ENGRAM_CONV_K 4     /* causal conv width */

enum { ENGRAM_F32 = 0, ENGRAM_BF16 = 1 };

/* engram_cfg_t.flags */
#define ENGRAM_SAVE_KV 1
/* formulation variants: the pages fix neither the conv's dilation, nor a
 * norm before it, nor whether branches share it, nor learnable norm scales
 * ([p2] short depthwise causal conv; [p5 二.1 (2)] 一维卷积; [p5 二.2]).  fp32
 * layers take any combination; bf16 layers (one branch) too, where
 * ENGRAM_CONV_PER_BRANCH is the same as a shared conv.  With
 * ENGRAM_CONV_PRENORM a bf16 layer computes v = e W_v^T as a tensor-core
 * GEMM (fp32 out) after the gate, and its forward workspace holds v and a
 * per-token scale. */
#define ENGRAM_CONV_DILATED 2     /* taps at t, t-3, t-6, t-9 (dilation 3 = the largest order) */
#define ENGRAM_CONV_PRENORM 4     /* the conv reads RMSNorm(vt) (times g_v with NORM_SCALES) */
#define ENGRAM_CONV_PER_BRANCH 8  /* conv weights per branch */
#define ENGRAM_NORM_SCALES 16     /* learnable RMSNorm scales g_h, g_k (and g_v) */
#define ENGRAM_VARIANT_FLAGS \
  (ENGRAM_CONV_DILATED | ENGRAM_CONV_PRENORM | ENGRAM_CONV_PER_BRANCH | ENGRAM_NORM_SCALES)
/* Test only (the pages have no counterpart): makes a bf16 call run the
 * wind-down path of its bounded device-side waits.  The producers of the
 * second operand of every tensor-core kernel (the fused passes of
 * engram_forward, the GEMMs of engram_backward) issue no copies, and the
 * backward's row kernel arms its copy ring without issuing the copies, so
 * the first wait on them cannot complete.  Every bounded wait of the call
 * gives up after about 1 ms instead of 2 s; the kernels set
 * ENGRAM_STATUS_TIMEOUT, let what they issued land, release their tensor
 * memory and return.  The call returns ENGRAM_OK and its outputs are
 * undefined; later calls without the flag are unaffected.  fp32 layers
 * (no such waits) ignore it. */
#define ENGRAM_TEST_STALL (1 << 30)

enum {
  ENGRAM_OK = 0,
  ENGRAM_ERR_INVALID_ARG = -1, /* null pointer, bad size or bad config */
  ENGRAM_ERR_MISALIGNED = -2,  /* a pointer is not 16-byte aligned */
  ENGRAM_ERR_WORKSPACE = -3,   /* ws_bytes below engram_workspace_size */
  ENGRAM_ERR_UNSUPPORTED = -4, /* shape/dtype combination not built */
  ENGRAM_ERR_CUDA = -5,        /* a CUDA runtime call failed */
  ENGRAM_ERR_TIMEOUT = -6,     /* status word reports a pipeline wait that ran out */
  ENGRAM_ERR_TOO_LARGE = -7    /* input larger than a fixed, built-in scratch area */
};

/* bits of the device status word */
#define ENGRAM_STATUS_BAD_ID 1u    /* raw token id outside [0, V_raw) */
#define ENGRAM_STATUS_BAD_INDEX 2u /* gathered row index outside [0, P_j) */
#define ENGRAM_STATUS_TIMEOUT 4u   /* a bounded wait inside a kernel gave up */

/*
 * Layer configuration (host memory, read during the call only).
 *   K        hash heads per n-gram order; J = 2K heads: heads 0..K-1 hash the
 *            2-gram, heads K..2K-1 the 3-gram ([p5 二.1 (1)] 多头哈希).
 *   D_h      dims of one table row; E = J * D_h is the width of e_t.
 *   d_model  width d of h and out.
 *   n_branch M hidden-state branches; each has its own W_k and gate, the
 *            table, W_v and conv weights are shared ([p5 二.2] 多分支架构集成).
 *   V_raw    raw vocabulary size; V_c compressed size; PAD id = V_c.
 *   dtype    ENGRAM_F32 or ENGRAM_BF16: storage of table, e, h, W_k, W_v, out.
 *   flags    0, or ENGRAM_SAVE_KV (bf16 layers; fp32 layers ignore it): a
 *            forward with whole sequences and a `saved` buffer also stores
 *            k = W_k e and v = W_v e there (fp32 [n_tok, 2 d_model], each
 *            token's k then its v, after alpha from the next 256-byte
 *            boundary), and the backward reads them instead of recomputing
 *            them: 8 * n_tok * d_model more bytes of `saved` for one GEMM
 *            less in the backward.
 *            ENGRAM_CONV_DILATED, ENGRAM_CONV_PRENORM, ENGRAM_CONV_PER_BRANCH,
 *            ENGRAM_NORM_SCALES: formulation variants, in any combination,
 *            on fp32 and on bf16 layers.
 *            z = <RMSNorm(h) g_h, RMSNorm(k) g_k> / sqrt(d),
 *            vt = alpha v, c = RMSNorm(vt) g_v (PRENORM) or vt,
 *            y_t = sum_i w[:, i] c_{t-(3-i) dil} (dil 3 with DILATED, else 1),
 *            out = h + vt + SiLU(y); each branch m has its own w (PER_BRANCH)
 *            and its own g_h, g_k, g_v (NORM_SCALES).  Their parameters form
 *            the conv_w block (engram_param_floats floats).
 *            ENGRAM_TEST_STALL: see above (tests only).
 *            Any other bit is ENGRAM_ERR_INVALID_ARG.
 *   rows[j]  P_j, row count (a prime) of head j's table.  Head j's rows sit
 *            in one packed table after those of heads 0..j-1.
 *   mult[j]  odd 64-bit multipliers of head j for n-gram positions 0, 1, 2
 *            (position i holds c_{t-i}).  Slot of head j:
 *              (XOR_i c_{t-i} * mult[j][i]  mod 2^64)  mod P_j.
 */
typedef struct engram_cfg {
  int32_t K;
  int32_t D_h;
  int32_t d_model;
  int32_t n_branch;
  int32_t V_raw;
  int32_t V_c;
  int32_t dtype;
  int32_t flags; /* ENGRAM_SAVE_KV, the variant flags, ENGRAM_TEST_STALL */
  int64_t rows[ENGRAM_MAX_HEADS];
  uint64_t mult[ENGRAM_MAX_HEADS][3];
} engram_cfg_t;

/* which call engram_workspace_size sizes */
enum {
  ENGRAM_WS_VOCAB = 0,     /* engram_build_vocab_proj, n = V */
  ENGRAM_WS_FORWARD = 1,   /* engram_forward, n = tokens */
  ENGRAM_WS_BACKWARD = 2,  /* engram_backward, n = tokens */
  ENGRAM_WS_TABLE_GRAD = 3, /* engram_table_grad, n = tokens */
  ENGRAM_WS_HOSTCACHE_RANK = 4,  /* engram_hostcache_rank, n = tokens of the sample */
  ENGRAM_WS_HOSTCACHE_GATHER = 5 /* engram_forward_hostcache, n = tokens */
};

/* Bytes of device workspace the call needs for n items (0 = none).  Returns
 * 0 as well for an invalid configuration (the call itself then reports it). */
size_t engram_workspace_size(const engram_cfg_t* cfg, int32_t call, int64_t n);

/* Bytes of the `saved` buffer engram_forward fills for engram_backward
 * (bf16: alpha, fp32 [n_tok], and with ENGRAM_SAVE_KV k and v as well). */
size_t engram_saved_size(const engram_cfg_t* cfg, int64_t n_tok);

/*
 * Vocabulary projection ([p5 二.1 (1)] 词汇投影; [p1] 分词器压缩: ids of one
 * meaning but different surface form share one compressed id, ~23% fewer ids).
 *   keys  device int64 [V]: canonical key of each raw id (ids with equal keys
 *         merge).
 *   proj  device int32 [V], out: compressed id of each raw id.  Compressed ids
 *         number the distinct keys in order of first occurrence by raw id.
 *   V_c_out host int32, out: number of distinct keys.
 *   ws    device workspace of engram_workspace_size(NULL-ok, ENGRAM_WS_VOCAB, V).
 * One-time set-up: synchronises `stream` to return V_c.
 */
int engram_build_vocab_proj(const int64_t* keys, int32_t V, int32_t* proj, int32_t* V_c_out,
                            void* ws, size_t ws_bytes, void* stream);

/*
 * Steps 1-3: compress, suffix n-grams, multi-head hash ([p4 第一步, 第二步];
 * [p2] 2-gram / 3-gram suffixes; [p5 二.1 (1)]).
 *   proj  device int32 [V_raw].      ids  device int32 [B, T] raw ids.
 *   idx   device int32 [B, T, J], out: slot of each head (-1 for a token whose
 *         n-gram holds an invalid raw id; the status word then has BAD_ID).
 *   ngram_state  NULL for whole sequences (positions before t = 0 are PAD).
 *         Non-NULL selects decode: T must be 1; device int32 [B, 2] holds
 *         (c_{t-1}, c_{t-2}) of each sequence, PAD at the start, and is
 *         updated in place.
 * The indices depend on the ids alone, so they can be computed ahead of the
 * layer ([p2]: known before the forward pass; [p4] prefetch).
 */
int engram_hash_indices(const engram_cfg_t* cfg, const int32_t* proj, const int32_t* ids,
                        int32_t B, int32_t T, int32_t* ngram_state, int32_t* idx, void* stream);

/*
 * Step 4: e[n, j*D_h:(j+1)*D_h] = table[rowbase_j + idx[n, j]] ([p5 二.1 (1)]
 * 拼接检索结果).  table: device, packed heads, dtype cfg->dtype.
 * e: device [n_tok, E], out.  An exact copy.
 */
int engram_gather(const engram_cfg_t* cfg, const int32_t* idx, const void* table, int64_t n_tok,
                  void* e, void* stream);

/*
 * Steps 4-6: the whole layer for B sequences of T tokens.
 *   idx     device int32 [B, T, J] from engram_hash_indices.
 *   table   device packed table, or NULL when `e` already holds the gathered
 *           rows (host-resident tables: see engram_forward_hosttable).
 *   e       device [B*T, E] (cfg->dtype): written by the gather when table is
 *           non-NULL, read by the projections.
 *   h       device [B, T, M, d] hidden state (cfg->dtype).
 *   Wk      device [M, d, E] key projections, Wv device [d, E] value
 *           projection (cfg->dtype; k = W_k e, v = W_v e: the contraction runs
 *           along the contiguous axis).
 *   conv_w  device fp32 [d, 4]: y_t = sum_i conv_w[:, i] * vt_{t-3+i}; with
 *           variant flags the small-parameter block (engram_param_floats).
 *   conv_state NULL for whole sequences.  Non-NULL selects decode (T == 1):
 *           device fp32 [B, M, 3 dil, d], the conv inputs (vt, or the
 *           normalised vt with ENGRAM_CONV_PRENORM) of the 3 dil previous
 *           steps, oldest first, zeros at the start; updated in place.
 *           A bf16 decode call (B <= 4,096, d a multiple of 256, E of 128,
 *           no ENGRAM_CONV_PRENORM) runs both projections, the gate and the
 *           conv as one cooperative launch of at most one CTA per SM, whose
 *           CTAs wait for one another at the gate (each wait bounded by 2 s,
 *           then ENGRAM_STATUS_TIMEOUT in the status word).
 *   out     device [B, T, M, d] (cfg->dtype); may be h itself (the residual
 *           applied in place): every read of h precedes the write of the same
 *           element.  engram_backward needs the original h, so a forward that
 *           will be differentiated keeps them apart.
 *   saved   device, engram_saved_size bytes, or NULL: what engram_backward needs.
 *   ws      device workspace of engram_workspace_size(cfg, ENGRAM_WS_FORWARD, B*T).
 * bf16: tables, e, h, W, out in bf16; products, gate, conv in fp32; the output
 * is rounded once.  f32: tables, e, h, W, out in fp32; the arithmetic runs in
 * fp64 and every stored value is rounded to fp32 once.
 * ([p5 二.1 (2)] gate with h as query and e as key/value, 1-D conv, residual;
 * [p4 第三步, 第四步]; [p2] short depthwise causal conv.)
 */
int engram_forward(const engram_cfg_t* cfg, const int32_t* idx, const void* table, void* e,
                   const void* h, const void* Wk, const void* Wv, const float* conv_w,
                   float* conv_state, void* out, float* saved, int32_t B, int32_t T, void* ws,
                   size_t ws_bytes, void* stream);

/*
 * One decode step in one call: for B sequences of one new token each,
 * steps 1-3 with the n-gram history from the rolling state and step 4 run
 * as one kernel (a block per token), then steps 5-6 as engram_forward with
 * a conv state.  The same results, bit for bit, as engram_hash_indices
 * (T = 1, with ngram_state) followed by engram_forward (table non-NULL,
 * conv_state non-NULL), with one kernel launch fewer per step ([p4]
 * indices depend only on the tokens; [p5 三.4] per-token inference).
 *   proj, ids        as engram_hash_indices: ids device int32 [B].
 *   ngram_state      device int32 [B, 2], in/out: (c_{t-1}, c_{t-2}).
 *   idx              device int32 [B, J] out (the step's slots), or NULL.
 *   table, e, h, Wk, Wv, conv_w, conv_state, out, ws
 *                    as engram_forward with T = 1 (conv_state required;
 *                    nothing is saved for a backward).
 */
int engram_decode_step(const engram_cfg_t* cfg, const int32_t* proj, const int32_t* ids,
                       int32_t* ngram_state, int32_t* idx, const void* table, void* e,
                       const void* h, const void* Wk, const void* Wv, const float* conv_w,
                       float* conv_state, void* out, int32_t B, void* ws, size_t ws_bytes,
                       void* stream);

/*
 * Backward of engram_forward for L = sum(dout * out) ([p4]: end-to-end
 * training; lookups are deterministic, so a slot gets consistent gradients).
 * Inputs as in engram_forward (e as the forward left it; saved may be NULL:
 * the fp32 backward recomputes the forward's intermediates in fp64 from e, h
 * and the weights and keeps every product and sum in fp64, so each gradient
 * carries one fp32 rounding) and
 *   dout     device fp32 [B, T, M, d].
 * Outputs (device fp32, overwritten):
 *   dh [B, T, M, d], dWk [M, d, E], dWv [d, E], dconv_w [d, 4] (the
 *   gradient of the whole small-parameter block with variant flags),
 *   de       [B*T, E] or NULL,
 *   dtab_keys int64 [<= B*T*J]: packed-table row ids, ascending, unique,
 *   dtab_rows [<= B*T*J, D_h]: gradient of those rows,
 *   n_unique device int32 [1]: number of rows written.
 * Each table row's gradient is summed in fp32 over its tokens in ascending
 * token order (see engram_table_grad), so it is reproducible bit for bit.
 * ENGRAM_F32: any branch count; the arithmetic runs in fp64.
 * ENGRAM_BF16: one branch, d_model a multiple of 256 and <= 4,096 (else
 * ENGRAM_ERR_UNSUPPORTED); e, h, Wk, Wv bf16 as in the forward, `saved`
 * (the forward's alpha) required; dout and every gradient fp32.  The
 * elementwise part runs in fp32; the plain GEMMs (k and v recomputed in fp32
 * as one GEMM against [W_k; W_v], [dW_k; dW_v] as one, de as one with
 * K = 2 d_model) run on the tensor cores with bf16 operands (dk and dv
 * rounded to bf16 once) and fp32 accumulation.  The weight gradients are
 * summed over the tokens in an order fixed by the launch configuration, so
 * they are reproducible from call to call.  A device-side wait that runs out
 * sets ENGRAM_STATUS_TIMEOUT.
 */
int engram_backward(const engram_cfg_t* cfg, const int32_t* idx, const void* e, const void* h,
                    const void* Wk, const void* Wv, const float* conv_w, const float* saved,
                    const float* dout, float* dh, float* dWk, float* dWv, float* dconv_w, float* de,
                    int64_t* dtab_keys, float* dtab_rows, int32_t* n_unique, int32_t B, int32_t T,
                    void* ws, size_t ws_bytes, void* stream);

/*
 * Sparse table gradient alone: a stable sort of the (row id, token) pairs by
 * row id, then one fp32 sum per row and dimension over its tokens in
 * ascending order, each starting from +0.
 *   idx device int32 [n_tok, J]; de device fp32 [n_tok, E].
 *   Outputs as in engram_backward.
 */
int engram_table_grad(const engram_cfg_t* cfg, const int32_t* idx, const float* de, int64_t n_tok,
                      int64_t* dtab_keys, float* dtab_rows, int32_t* n_unique, void* ws,
                      size_t ws_bytes, void* stream);

/*
 * engram_table_grad without a workspace argument, for callers that cannot
 * allocate device memory: a host framework that owns every allocation and
 * hands out none for scratch, or a runtime with a fixed memory pool.  (The pages
 * have no counterpart: this is an interface variant, not part of the method.)
 *   Same arguments, outputs and results as engram_table_grad, minus ws.
 *   The sort buffers live in a device array built into the library, sized
 *   for n_tok * J <= ENGRAM_NOALLOC_MAX_ITEMS (token, head) pairs (about
 *   4.8 MB, held on every GPU that loads the library until the process
 *   exits).  Larger inputs return ENGRAM_ERR_TOO_LARGE and launch nothing.
 *   The call allocates nothing.  Its first call on a device looks up the
 *   array's device address (cudaGetSymbolAddress).
 *   All calls share the array: calls that overlap on the GPU (other streams,
 *   other host threads) race and must be serialised by the caller.
 *   The looked-up address is kept for the life of the process: after a
 *   cudaDeviceReset the array moves, so the library must not be used on
 *   that device again (the same holds for the status word of every call).
 */
#define ENGRAM_NOALLOC_MAX_ITEMS 131072
int engram_table_grad_noalloc(const engram_cfg_t* cfg, const int32_t* idx, const float* de,
                              int64_t n_tok, int64_t* dtab_keys, float* dtab_rows,
                              int32_t* n_unique, void* stream);

/*
 * Gather from a table in pinned, mapped host memory over PCIe ([p5 二.2]
 * the host fetches memory rows while the GPU runs earlier layers; [p4]
 * a 100B-parameter table kept in DRAM; [p2] prefetch over PCIe).
 *   host_table  pinned host memory (cudaHostAlloc / cudaHostRegister with
 *               mapping), packed as the device table.
 *   e           device [n_tok, E], out.
 *   side_stream the stream to run on; done_event (cudaEvent_t as void*, may
 *               be NULL) is recorded after the gather so the compute stream can
 *               wait on it before engram_forward(table = NULL, e).
 */
int engram_forward_hosttable(const engram_cfg_t* cfg, const int32_t* idx, const void* host_table,
                             int64_t n_tok, void* e, void* side_stream, void* done_event);

/*
 * HBM cache of hot host-table rows ([p1 系统效率优化] / [p2] 多级缓存设计: the
 * n-grams' Zipfian frequencies let the rows of frequent n-grams stay in GPU
 * memory and the long tail in host memory).  Three calls:
 *   engram_hostcache_rank  the C rows a sample of hash indices addresses most
 *                          often (the cache's contents);
 *   engram_hostcache_fill  copies them from the host table into the cache and
 *                          builds the row -> slot map;
 *   engram_forward_hostcache  gathers e like engram_forward_hosttable, the
 *                          cached rows from HBM and only the others over PCIe.
 * The gathered e is identical to engram_forward_hosttable's whatever the
 * cache holds; the cache changes where rows are read from, never what.
 */

/* Floats of the small-parameter block `conv_w` (and of its gradient
 * `dconv_w`): the conv weights, [d, 4], or [M, d, 4] with
 * ENGRAM_CONV_PER_BRANCH; then, with ENGRAM_NORM_SCALES, g_h [M, d], g_k
 * [M, d] and, with ENGRAM_CONV_PRENORM as well, g_v [M, d].  0 for an
 * invalid configuration. */
int64_t engram_param_floats(const engram_cfg_t* cfg);

/* Packed-table rows of the configuration: sum of rows[j] over the J heads
 * (the entries of the hostcache map); 0 for an invalid configuration. */
int64_t engram_table_rows(const engram_cfg_t* cfg);

/*
 *   idx      device int32 [n_tok, J]: a sample of hash indices (e.g. earlier
 *            batches); invalid slots (-1) count for no row.
 *   C        rows wanted (>= 0).
 *   rows_out device int64 [C], out: packed-table row ids (row_base_j + slot),
 *            most addressed first, ties by ascending row id; -1 past n_out.
 *   n_out    device int32, out: min(C, distinct rows addressed).
 *   ws       engram_workspace_size(cfg, ENGRAM_WS_HOSTCACHE_RANK, n_tok) bytes.
 * n_tok * J must stay below 2^31.  Asynchronous on `stream`.
 */
int engram_hostcache_rank(const engram_cfg_t* cfg, const int32_t* idx, int64_t n_tok, int64_t C,
                          int64_t* rows_out, int32_t* n_out, void* ws, size_t ws_bytes,
                          void* stream);

/*
 *   host_table pinned, mapped host memory as in engram_forward_hosttable.
 *   rows       device int64 [C]: packed-table rows to cache (-1: slot unused);
 *              a row out of range sets ENGRAM_STATUS_BAD_INDEX.
 *   cache      device [C, D_h] (cfg->dtype), out: cache slot i = rows[i].
 *   map        device int32 [engram_table_rows(cfg)], out: the cache slot of
 *              each packed-table row, -1 for rows not cached.
 * Asynchronous on `stream` (reads C rows over PCIe).
 */
int engram_hostcache_fill(const engram_cfg_t* cfg, const void* host_table, const int64_t* rows,
                          int64_t C, void* cache, int32_t* map, void* stream);

/*
 *   idx, host_table, n_tok, e, side_stream, done_event as in
 *   engram_forward_hosttable; cache and map from engram_hostcache_fill.
 *   n_miss   device int32, out (may be NULL): (token, head) pairs whose row
 *            came from host memory.
 *   ws       engram_workspace_size(cfg, ENGRAM_WS_HOSTCACHE_GATHER, n_tok).
 * Three kernels on side_stream: a probe (one thread per (token, head):
 * the row's slot, misses appended to a list), the cached rows' pieces from
 * HBM on the whole GPU, then the listed rows from host memory on a few CTAs.
 * n_tok * J must stay below 2^31.
 */
int engram_forward_hostcache(const engram_cfg_t* cfg, const int32_t* idx, const void* host_table,
                             const void* cache, const int32_t* map, int64_t n_tok, void* e,
                             int32_t* n_miss, void* ws, size_t ws_bytes, void* side_stream,
                             void* done_event);

/* Synchronises `stream`, then returns the device status word of the current
 * device (bits ENGRAM_STATUS_*) and clears it; a negative value is an
 * ENGRAM_ERR_* code. */
int engram_get_status(void* stream);

/* Multiprocessor count of the current device, or a negative ENGRAM_ERR_*. */
int engram_device_sm_count(void);

#ifdef __cplusplus
}
#endif

#endif /* ENGRAM_B200_H */
