/*
 * gqe.h - C ABI of the GQE (Grouped Query Experts) library: causal prefill
 * and incremental decode.
 *
 * Grouped Query Experts puts a per-group router on grouped-query attention:
 * N query heads form G groups of M = N/G "query-head experts" that share one
 * KV head.  For every token i and group g the router scores the group's M
 * experts, p_{i,g} = softmax(r_g(x_i)), keeps the top k, and only those query
 * heads attend (against the group's dense, never repeated, KV head).  The
 * layer output feeds W_O with Concat(O_i, o_bar_i, s(x_i)): the selected
 * heads' outputs, their renormalised weighted sum, and an always-on shared
 * head.  Sources: the review "论文综述：分组查询专家——在 GQA 自注意力上引入
 * 混合专家" §二 (路由器; 输出怎么拼起来：三个关键部件) and the summary page
 * "Grouped Query Experts: Mixture-of-Experts on GQA Self-Attention" (01 In
 * brief).  GQA head mapping and the causal rule follow "AI 大模型之 GQA"
 * (技术深化 分组查询的张量映射; 工程实操 非方形因果遮罩).
 *
 * Conventions for every entry point
 * ---------------------------------
 *  - Pointers marked "device" are CUDA device pointers owned by the caller;
 *    the library never allocates, frees or retains them.  All work is queued
 *    asynchronously on `stream` (a cudaStream_t; NULL = legacy default).
 *  - Every device pointer must be 16-byte aligned.  Tensors are dense,
 *    row-major, in the layouts stated per argument (B batch, S tokens).
 *  - `ws` is a caller-owned device workspace of at least
 *    gqe_workspace_size(dims) bytes (gqe_decode_workspace_size for the
 *    decode call), zero-filled once before its first use
 *    (it holds a latched device status word; the library keeps the rest
 *    consistent itself).  Calls that share one workspace must be ordered
 *    (same stream or explicit events).
 *  - Arguments are validated before anything is launched; on any error the
 *    call returns a non-zero gqe_status and launches nothing.  Unsupported
 *    shapes are rejected, never silently remapped ("AI 大模型之 GQA",
 *    工程实操: unsupported H/G combinations must be refused explicitly).
 *  - Errors found on the device (a bounded wait that ran out, an expert index
 *    or a decode position out of range, non-finite router logits, V outside
 *    the fp16 range) are latched into the workspace status word; read them
 *    with gqe_get_device_status().  Nothing is thrown across the ABI.
 *
 * Supported shapes: N % G == 0, M = N/G <= 32, 1 <= k <= M,
 * d in {64, 128}; for the router G*M in {4, 8, 16, 32} and d_model % 8 == 0;
 * B*S*G*max(k,M) < 2^31.
 */
#ifndef GQE_H
#define GQE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gqe_status {
  GQE_OK = 0,
  GQE_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size, k > M ... */
  GQE_ERR_UNSUPPORTED = 2,  /* a valid GQE shape this build does not run   */
  GQE_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed         */
  GQE_ERR_TIMEOUT = 4,      /* a bounded device-side wait ran out           */
  GQE_ERR_WORKSPACE = 5,    /* workspace missing or smaller than required   */
  GQE_ERR_BAD_INDEX = 6,    /* a top-k index outside [0, M) reached a kernel */
  GQE_ERR_NONFINITE = 7,    /* non-finite logit, or |V| above the fp16 range */
  GQE_ERR_BAD_POSITION = 8  /* a decode position outside [0, T) reached a kernel */
} gqe_status;

/* Problem size.  M = N / G is derived.  `out_fp32` selects the element type
 * of every output written by the attention calls: 1 = float32, 0 = bf16. */
typedef struct gqe_dims {
  int32_t B, S, N, G, k, d, d_model;
  int32_t out_fp32;
} gqe_dims;

/* Bytes of workspace the calls below need for `dims` (0 if dims invalid). */
size_t gqe_workspace_size(const gqe_dims* dims);

/*
 * gqe_route - the per-group router.
 * Review §二 路由器: p_{i,g} = softmax(r_g(x_i)) over the group's M experts,
 * K_g(x_i) = TopK_m(p_{i,g,m}, k); 三个关键部件: w = p / sum_{m' in K_g} p.
 * r_g is linear: l_{i,g,m} = x_i . W_r[g,:,m] (+ bias[g,m]).
 *
 *  x        device bf16 [B, S, d_model]
 *  W_r      device bf16 [G, d_model, M]
 *  bias     device fp32 [G, M] or NULL (an additive logit offset)
 *  topk_idx device int32 [B, S, G, k]  out: expert indices in rank order
 *  p        device fp32  [B, S, G, M]  out: router probabilities
 *  w        device fp32  [B, S, G, k]  out: renormalised weights (k=1 -> 1)
 *
 * Selection is decided on the exact real-valued logits; exact ties go to the
 * lower expert index.  The fast path certifies each decision with a rigorous
 * float32 error bound; undecided (token, group) pairs are recomputed with an
 * exact fixed-point dot product, so topk_idx is deterministic and exact.
 */
gqe_status gqe_route(const gqe_dims* dims, const void* x, const void* W_r, const float* bias,
                     int32_t* topk_idx, float* p, float* w, void* ws, size_t ws_bytes,
                     void* stream);

/*
 * gqe_bucket - stable per-(batch, group, expert) token lists.
 * For b, g, m in that order, the tokens i (ascending) with m in K_g(x_i).
 *  topk_idx   device int32 [B, S, G, k]   (as written by gqe_route)
 *  bucket_off device int32 [B*G*M + 1]    out: exclusive scan of bucket sizes;
 *             bucket (b,g,m) occupies [off[(b*G+g)*M+m], off[...+1]) and the
 *             (b,g) block starts at (b*G+g)*S*k.
 *  bucket_tok device int32 [B*G*S*k]      out: token positions
 * gqe_attention_prefill runs the same bucketing internally (into `ws`); this
 * entry exists so callers and tests can inspect it.
 */
gqe_status gqe_bucket(const gqe_dims* dims, const int32_t* topk_idx, int32_t* bucket_off,
                      int32_t* bucket_tok, void* ws, size_t ws_bytes, void* stream);

/*
 * gqe_attention_prefill - routed causal attention, shared head and combine.
 * Review §二 三个关键部件: only the selected heads attend; each selected head
 * h = g*M + m uses query Q[:, :, h] against KV head g with scale 1/sqrt(d) and
 * the causal rule key position <= query position.
 *
 *  Q        device bf16 [B, S, N, d]
 *  Qs       device bf16 [B, S, d]      query of the always-on shared head
 *  K, V     device bf16 [B, S, G, d]   one KV head per group, not repeated
 *  topk_idx device int32 [B, S, G, k]; w device fp32 [B, S, G, k] (gqe_route)
 *  O_sel    out: row (b,i) + (g*k + j)*d -> output of the head in slot j
 *  o_bar    out: row (b,i) + g*d         -> sum_j w_j * O_sel[g, j]
 *  s_out    out: row (b,i)               -> shared-head output (attends KV 0)
 *  out_row_stride  elements between consecutive tokens (b,i) in all three
 *           outputs (multiple of 8).  With one concat buffer of row length
 *           (G*k + G + 1)*d, pass O_sel = buf, o_bar = buf + G*k*d,
 *           s_out = buf + (G*k + G)*d and stride (G*k + G + 1)*d.
 * Output element type: float32 if dims->out_fp32 else bf16.
 * The shared head's KV source is not given by the sources; this library
 * fixes it to KV head 0.
 */
gqe_status gqe_attention_prefill(const gqe_dims* dims, const void* Q, const void* Qs,
                                 const void* K, const void* V, const int32_t* topk_idx,
                                 const float* w, void* O_sel, void* o_bar, void* s_out,
                                 int64_t out_row_stride, void* ws, size_t ws_bytes,
                                 void* stream);

/*
 * gqe_attention_prefill_static - gqe_attention_prefill for callers that
 * cannot allocate device memory.  (Not a step of the method: the sources
 * have no counterpart; it only changes where the scratch memory lives.)
 *
 * Some callers cannot give the library a workspace: for instance a plugin
 * whose host framework owns every device allocation, or a loop that must
 * not pay the device-wide synchronisation of cudaMalloc.  This call takes
 * the same arguments as gqe_attention_prefill minus `ws`/`ws_bytes`, writes
 * the same outputs, and allocates nothing: its scratch is one 64 MiB device
 * array compiled into the library, present on every GPU that loads it until
 * the process exits.
 *  - Every call looks up that array's device address with the device current
 *    (host code cannot use the array's name as an address); the first call
 *    on a device, and the first after its context was rebuilt, also zeroes
 *    the array's header with a synchronous cudaMemset.  Make that first call
 *    before any stream capture.
 *  - Shapes whose scratch (V in fp16, token lists, work list) exceeds
 *    64 MiB return GQE_ERR_WORKSPACE without launching anything.
 *  - All calls on a device share the one array and it keeps the previous
 *    call's contents (each call clears the counters that must start at
 *    zero).  Calls that overlap on the GPU - different streams, or different
 *    host threads - race on it and give wrong results; order them.
 *  - Device-side errors (an expert index outside [0, M), V outside the fp16
 *    range, a bounded wait that ran out) are latched into a status word at
 *    the start of the array, as the workspace calls latch them into theirs.
 *    The word keeps the first error until gqe_static_device_status clears it.
 */
gqe_status gqe_attention_prefill_static(const gqe_dims* dims, const void* Q, const void* Qs,
                                        const void* K, const void* V, const int32_t* topk_idx,
                                        const float* w, void* O_sel, void* o_bar, void* s_out,
                                        int64_t out_row_stride, void* stream);

/*
 * gqe_static_device_status - read (and with clear != 0 reset) the status
 * word that gqe_attention_prefill_static latches device-side errors into, on
 * the current device.  Like gqe_attention_prefill_static it has no
 * counterpart in the sources.  Synchronises `stream` first, so the value
 * covers every static call queued on it; returns GQE_OK or the latched
 * gqe_status, and GQE_ERR_CUDA if the read itself failed.
 */
gqe_status gqe_static_device_status(int32_t clear, void* stream);

/* Bytes of workspace gqe_attention_prefill_chunk needs for `dims` (S = the
 * chunk's query count) over caches of T >= S slots (0 if invalid). */
size_t gqe_prefill_chunk_workspace_size(const gqe_dims* dims, int32_t T);

/*
 * gqe_attention_prefill_chunk - gqe_attention_prefill for a chunk of S new
 * tokens per sequence over KV caches of T slots (chunked prefill), with
 * optional left padding.  "AI 大模型之 GQA", 工程实操 非方形因果遮罩: Sq
 * queries at the end of Sk keys, the mask taken on absolute positions; step
 * 4: the causal condition intersected with key validity.  Query row i of
 * sequence b sits at absolute position q_off[b] + i and sees cache slots
 * kv_start[b]..q_off[b] + i (the chunk's own K/V must already be in the
 * caches).  Rows whose position lies before kv_start[b] are padding: they
 * see no key and their outputs are written as zeros.
 *  Q, Qs    device bf16 [B, S, N, d], [B, S, d]   (the chunk's queries)
 *  Kc, Vc   device bf16 [B, T, G, d]
 *  q_off    device int32 [B] or NULL (= 0): 0 <= q_off[b] <= T - S
 *  kv_start device int32 [B] or NULL (= 0): 0 <= kv_start[b] < T
 *  topk_idx, w, outputs, out_row_stride as for gqe_attention_prefill (one
 *  output row per chunk token); ws of gqe_prefill_chunk_workspace_size bytes.
 * Positions are read on the device (so a chunk loop can be captured in a CUDA
 * graph); a value outside its range latches GQE_ERR_BAD_POSITION and is
 * taken as 0.  Always runs the one-tile attention kernel.
 */
gqe_status gqe_attention_prefill_chunk(const gqe_dims* dims, int32_t T, const void* Q,
                                       const void* Qs, const void* Kc, const void* Vc,
                                       const int32_t* q_off, const int32_t* kv_start,
                                       const int32_t* topk_idx, const float* w, void* O_sel,
                                       void* o_bar, void* s_out, int64_t out_row_stride,
                                       void* ws, size_t ws_bytes, void* stream);

/*
 * gqe_dense_gqa_prefill - the all-active GQA baseline ("16 heads all
 * active", review §四): every query head h attends KV head floor(h/M).
 *  Q device bf16 [B, S, N, d]; K, V device bf16 [B, S, G, d]
 *  O device [B, S, N, d], float32 if dims->out_fp32 else bf16.
 * dims->k is ignored.
 */
gqe_status gqe_dense_gqa_prefill(const gqe_dims* dims, const void* Q, const void* K,
                                 const void* V, void* O, void* ws, size_t ws_bytes,
                                 void* stream);

/* Bytes of workspace gqe_attention_decode needs for `dims` (0 if invalid).
 * Its status word sits at offset 0 and its scratch starts at byte 512, after
 * the region gqe_route keeps its counters in; so one zero-filled buffer of
 * max(gqe_workspace_size(route dims), gqe_decode_workspace_size(dims)) bytes
 * serves a decode step's gqe_route and gqe_attention_decode in stream order. */
size_t gqe_decode_workspace_size(const gqe_dims* dims);

/*
 * gqe_attention_decode - one incremental decode step of GQE.
 * "AI 大模型之 GQA", 工程实操 非方形因果遮罩: at a decode step the query length
 * is 1 and the key length is the whole history; the causal mask is taken on
 * the query's absolute position.  The new token of sequence b sits at
 * position pos[b] and sees cache slots 0..pos[b].  As in prefill (review §二),
 * slot j of group g is the head h = g*M + topk_idx[b,g,j] against KV head g,
 * o_bar is the w-weighted sum of the group's slots, and the shared head
 * attends KV head 0.
 *
 *  dims     B sequences, S = T (capacity of the caches' time axis), N, G, k,
 *           d as for prefill; d_model is not used.
 *  Q        device bf16 [B, N, d]     queries of the new tokens
 *  Qs       device bf16 [B, d]        shared-head queries
 *  Kc, Vc   device bf16 [B, T, G, d]  caches; slot pos[b] must already hold
 *           the new token's K and V (the append is the caller's copy)
 *  pos      device int32 [B]          0 <= pos[b] < T, may differ per b
 *  kv_start device int32 [B] or NULL: first valid cache slot of sequence b
 *           (left padding; 工程实操 step 4: the causal condition is
 *           intersected with key validity), 0 <= kv_start[b] <= pos[b];
 *           sequence b then sees slots kv_start[b]..pos[b].  NULL = all 0.
 *  topk_idx device int32 [B, G, k]; w device fp32 [B, G, k]: gqe_route with
 *           dims S = 1 on the new tokens' x
 *  O_sel, o_bar, s_out, out_row_stride: as for gqe_attention_prefill, one
 *           output row per sequence b.
 * Output element type: float32 if dims->out_fp32 else bf16.  A position or
 * first slot out of range latches GQE_ERR_BAD_POSITION and that sequence's
 * outputs are NaN; an expert index out of range latches GQE_ERR_BAD_INDEX
 * and its slot and o_bar are NaN.  The cache is read once per step: each
 * CTA serves every selected head of its KV head (and the shared head for KV
 * head 0) over one chunk of keys, and a second kernel merges the chunks.
 * Errors: GQE_ERR_INVALID_ARG / GQE_ERR_UNSUPPORTED for bad dims, null or
 * misaligned pointers or a stride below d or not a multiple of 8;
 * GQE_ERR_WORKSPACE when ws_bytes < gqe_decode_workspace_size(dims).
 */
gqe_status gqe_attention_decode(const gqe_dims* dims, const void* Q, const void* Qs,
                                const void* Kc, const void* Vc, const int32_t* pos,
                                const int32_t* kv_start, const int32_t* topk_idx,
                                const float* w, void* O_sel, void* o_bar, void* s_out,
                                int64_t out_row_stride, void* ws, size_t ws_bytes,
                                void* stream);

/*
 * gqe_attention_append - n_new new tokens per sequence over the caches: a
 * short chunked prefill, or checking n_new drafted tokens at once.
 * "AI 大模型之 GQA", 工程实操 非方形因果遮罩: Sq queries at the end of Sk keys,
 * masked on absolute positions.  New token r of sequence b sits at cache
 * slot pos[b] + r and sees slots kv_start[b]..pos[b] + r; slots pos[b] ..
 * pos[b] + n_new - 1 must already hold the new tokens' K and V.  Everything
 * else is gqe_attention_decode with an n_new axis after B:
 *  Q bf16 [B, n_new, N, d]; Qs bf16 [B, n_new, d];
 *  topk_idx int32 / w fp32 [B, n_new, G, k] (gqe_route with dims S = n_new);
 *  output row b * n_new + r of O_sel / o_bar / s_out (stride as before).
 * 1 <= n_new <= 64 and n_new <= T (longer chunks belong to the prefill
 * kernels); pos[b] + n_new - 1 < T is checked on the device
 * (GQE_ERR_BAD_POSITION).  gqe_attention_decode is the n_new = 1 case.
 */
size_t gqe_append_workspace_size(const gqe_dims* dims, int32_t n_new);
gqe_status gqe_attention_append(const gqe_dims* dims, int32_t n_new, const void* Q,
                                const void* Qs, const void* Kc, const void* Vc,
                                const int32_t* pos, const int32_t* kv_start,
                                const int32_t* topk_idx, const float* w, void* O_sel,
                                void* o_bar, void* s_out, int64_t out_row_stride, void* ws,
                                size_t ws_bytes, void* stream);

/* Synchronises `stream`, then returns the status word latched in `ws`
 * (GQE_OK if no device-side error was recorded).  If `clear` is non-zero the
 * word is reset to GQE_OK afterwards. */
gqe_status gqe_get_device_status(void* ws, int32_t clear, void* stream);

/* "AI 大模型之 GQA" §4.1: KV-cache bytes = 2 * L * G * d * S * b, times B
 * sequences (L layers, G KV heads, b bytes per element).  Host-only. */
uint64_t gqe_kv_cache_bytes(int32_t L, int32_t G, int64_t S, int32_t d,
                            int32_t bytes_per_elem, int32_t B);

/* Static, human-readable name of a status code. */
const char* gqe_status_string(gqe_status s);

/* Failure-detection self test: launches one kernel whose mbarrier wait can
 * never complete, bounded by `limit_us` microseconds; the kernel gives up,
 * latches GQE_ERR_TIMEOUT into `ws` and exits cleanly.  Returns the launch
 * status (the latched code is read with gqe_get_device_status). */
gqe_status gqe_selftest_bounded_wait(void* ws, size_t ws_bytes, int32_t limit_us,
                                     void* stream);

/* Profiling hook.  When both handles are non-NULL, every later
 * gqe_attention_prefill / gqe_dense_gqa_prefill call records `begin`
 * (a cudaEvent_t) on its stream immediately before its attention kernel and
 * `end` immediately after it, so the caller can time that kernel alone with
 * cudaEventElapsedTime.  Pass NULLs to switch it off.  Process-wide setting,
 * not thread-safe: meant for benchmarks. */
void gqe_set_profile_events(void* begin, void* end);

/* Kernel choice for d = 64 (tuning; no counterpart on the pages).  The
 * attention calls use a pair kernel - two 128-row query tiles of one KV head
 * per CTA, sharing every K/V tile load - once the KV working set of the call,
 * B*S*G*d*4 bytes (K bf16 + V fp16), reaches `kv_bytes`; below it they use one
 * tile per CTA and two CTAs per SM, which is faster while K and V stay in L2.
 * Default 96 MiB.  0 selects the pair kernel always, a negative value never.
 * Results agree within rounding either way.  Process-wide setting, read at
 * each call; returns the previous value. */
int64_t gqe_set_pair_threshold(int64_t kv_bytes);

/* Router kernel choice (tuning; no counterpart on the pages).  gqe_route keeps
 * W_r in shared memory (float32, one CTA of 16 warps per SM over 64-token
 * tiles) when d_model * G * M <= 16384, d_model is a multiple of 128 (of 64
 * when G*M = 32) and the call has at least 3 such tiles per SM; otherwise it
 * streams W_r from a float32 copy.  Both take the same certified decisions
 * (top-k identical; p and w within float32 rounding of each other).
 * on = 1 takes the resident kernel whenever W_r fits, whatever the token
 * count; 0 restores the default; a negative value only reads the setting.
 * Process-wide, read at each call; returns the previous setting (0 or 1). */
int32_t gqe_set_router_resident(int32_t on);

/* ------------------------------------------------------------------------
 * Training: the forward call that also keeps each row's log-sum-exp, and the
 * backward pass of the path.
 * ------------------------------------------------------------------------ */

/*
 * gqe_attention_prefill_train - gqe_attention_prefill (float32 outputs:
 * dims->out_fp32 must be 1) that also writes, per routed slot and per
 * shared-head row, the base-2 log-sum-exp of that row's scaled scores
 * (log2 sum_t 2^(q.k_t log2(e)/sqrt(d))): what the backward pass needs to
 * rebuild the softmax without a second forward.
 *  lse_sel  device float32 [B, S, G, k] (slot order);  lse_s float32 [B, S]
 */
gqe_status gqe_attention_prefill_train(const gqe_dims* dims, const void* Q, const void* Qs,
                                       const void* K, const void* V, const int32_t* topk_idx,
                                       const float* w, void* O_sel, void* o_bar, void* s_out,
                                       int64_t out_row_stride, float* lse_sel, float* lse_s,
                                       void* ws, size_t ws_bytes, void* stream);

/* Bytes of workspace gqe_prefill_backward needs for `dims` (0 if invalid). */
size_t gqe_prefill_backward_workspace_size(const gqe_dims* dims);

/*
 * gqe_prefill_backward - gradients of the path's outputs (O_sel, o_bar, s)
 * with respect to Q, Qs, K, V and the weights w, for upstream gradients in
 * the concat layout.  "AI 大模型之 GQA", 训练与部署 共享键值的梯度归约: each
 * query head's attention backward is computed on its own and the gradients
 * of a KV head are the SUM over every head that reads it (the routed experts
 * of the group that a token selected, and the shared head for KV head 0);
 * review §二 三个关键部件: o_bar = sum_j w_j o_j, so slot j receives
 * dO_sel_j + w_j d(o_bar), and dw_j = <d(o_bar), o_j> (the gradient the
 * weighted-sum slot gives the router; at k = 1, w = 1 and the caller may
 * drop it).  The selection itself is held fixed.
 *  Q, Qs, K, V, topk_idx, w  the forward's inputs (bf16 / int32 / float32)
 *  O_sel, s_out  the forward's float32 outputs, rows at out_row_stride
 *                (the concat buffer of gqe_attention_prefill_train)
 *  lse_sel, lse_s  from gqe_attention_prefill_train
 *  dO_sel, do_bar, ds  float32 upstream gradients, rows at dout_row_stride
 *                (the concat layout: slot j of group g at (g*k + j)*d)
 *  dQ   float32 [B, S, N, d]: rows of heads a token did not select are 0
 *  dQs  float32 [B, S, d];  dK, dV float32 [B, S, G, d];  dw float32 [B, S, G, k]
 *  ws   gqe_prefill_backward_workspace_size(dims) bytes
 * The tensor-core products take bf16 operands: the effective dO, P and dS
 * are rounded to bf16 (float32 accumulation).
 */
gqe_status gqe_prefill_backward(const gqe_dims* dims, const void* Q, const void* Qs,
                                const void* K, const void* V, const int32_t* topk_idx,
                                const float* w, const float* O_sel, const float* s_out,
                                int64_t out_row_stride, const float* lse_sel, const float* lse_s,
                                const float* dO_sel, const float* do_bar, const float* ds,
                                int64_t dout_row_stride, float* dQ, float* dQs, float* dK,
                                float* dV, float* dw, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * The attention layer around the path: projections and W_O.
 * Review §二 路由器: only the query heads the router selected are computed at
 * all, so their query projection runs for the selected (token, head) pairs
 * only; 三个关键部件: y_i = Concat(O_i, o_bar_i, s(x_i)) W_O.  The other
 * projections are plain linear maps (K_{i,g} = x_i W_K[g], V likewise, the
 * shared head's query x_i W_s).  All run on the tensor cores with bf16
 * operands and float32 accumulation.
 * ------------------------------------------------------------------------ */

/*
 * gqe_linear - C[r, n] = sum_k A[r, k] * W[n / nc][k, n % nc] for r < rows,
 * n < nb*nc: A times a stack of nb matrices [K, nc] read as one [K, nb*nc]
 * operand, so x . W_K for all G KV heads is one call whose output is K in its
 * [B, S, G, d] layout (rows = B*S, nb = G, nc = d, ldc = G*d).
 *  A   device bf16, rows x K at row stride lda elements (lda >= K, lda % 8 == 0)
 *  W   device bf16 [nb, K, nc] (row-major)
 *  C   device, rows x nb*nc at row stride ldc elements; float32 if c_fp32
 *      else bf16 (round to nearest even); ldc*element size a multiple of 16 B
 * K and nc must be multiples of 64 (GQE_ERR_UNSUPPORTED otherwise).
 */
gqe_status gqe_linear(int32_t rows, int32_t K, int32_t nb, int32_t nc, const void* A, int64_t lda,
                      const void* W, void* C, int64_t ldc, int32_t c_fp32, void* stream);

/*
 * gqe_routed_q_project - the query projection of the selected heads only:
 * Q[b, i, h, :] = x[b, i, :] . W_Q[h] for every (b, i, g, j) with
 * h = g*M + topk_idx[b, i, g, j].  Rows of heads a token did not select are
 * not written.  Each CTA takes one tile of a (batch, group, expert) bucket
 * (the lists gqe_attention_prefill builds), gathers its x rows and multiplies
 * them by that expert's W_Q[h].
 *  x        device bf16 [B, S, d_model] (d_model % 64 == 0)
 *  W_Q      device bf16 [N, d_model, d]
 *  topk_idx device int32 [B, S, G, k]
 *  Q        device bf16 [B, S, N, d]
 *  ws       workspace of gqe_workspace_size(dims) bytes
 */
gqe_status gqe_routed_q_project(const gqe_dims* dims, const void* x, const void* W_Q,
                                const int32_t* topk_idx, void* Q, void* ws, size_t ws_bytes,
                                void* stream);

/*
 * gqe_layer_prefill - the whole GQE attention layer, causal prefill, x -> y:
 * gqe_route, then K, V and Qs by gqe_linear, Q of the selected heads by
 * gqe_routed_q_project, gqe_attention_prefill into a bf16 concat buffer
 * (whatever dims->out_fp32 says: the buffer feeds W_O in bf16), then
 * y = concat . W_O by gqe_linear.  The caller owns every buffer:
 *  W_K, W_V  device bf16 [G, d_model, d];  W_s bf16 [d_model, d]
 *  W_r, bias as for gqe_route;  W_O bf16 [(G*k + G + 1)*d, d_model], rows
 *            in concat order
 *  topk_idx, p, w as for gqe_route;  Q bf16 [B, S, N, d] (selected rows);
 *  Qs bf16 [B, S, d];  K, V bf16 [B, S, G, d];
 *  concat    bf16 [B*S, (G*k + G + 1)*d];  y float32 [B, S, d_model]
 * K, V and Qs do not depend on the routing, so they are computed on a second
 * stream the library keeps per device (created on first use), ordered after
 * the work already in `stream` and joined back into `stream` before the
 * attention call by events; everything the call writes is complete when
 * `stream` reaches the end of the call, as with the other entry points.
 * Several host threads calling this on one device share that stream (their
 * projections then run in turn).
 */
gqe_status gqe_layer_prefill(const gqe_dims* dims, const void* x, const void* W_Q,
                             const void* W_K, const void* W_V, const void* W_s, const void* W_r,
                             const float* bias, const void* W_O, int32_t* topk_idx, float* p,
                             float* w, void* Q, void* Qs, void* K, void* V, void* concat,
                             float* y, void* ws, size_t ws_bytes, void* stream);

/*
 * gqe_dense_layer_prefill - the all-active GQA layer baseline (review §四):
 * Q of all N heads, K, V, dense GQA attention into O bf16 [B, S, N, d], then
 * y = O . W_O with W_O bf16 [N*d, d_model].
 */
gqe_status gqe_dense_layer_prefill(const gqe_dims* dims, const void* x, const void* W_Q,
                                   const void* W_K, const void* W_V, const void* W_O, void* Q,
                                   void* K, void* V, void* O, float* y, void* ws,
                                   size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GQE_H */
