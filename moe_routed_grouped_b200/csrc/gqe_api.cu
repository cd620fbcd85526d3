// C-ABI entry points of the GQE prefill library (declared in include/gqe.h).
// Argument validation happens here, before any launch; the kernels live in
// gqe_route.cu, gqe_bucket.cu, gqe_attn.cu and gqe_decode.cu.
#include <cmath>
#include <cstring>

#include <cuda.h>
#include <cuda_runtime.h>

#include "gqe_decode.h"
#include "gqe_internal.h"

using namespace gqe;

namespace {

gqe_status from_cuda(cudaError_t e) { return e == cudaSuccess ? GQE_OK : GQE_ERR_CUDA; }

}  // namespace

extern "C" {

size_t gqe_workspace_size(const gqe_dims* dims) {
  if (check_dims(dims, false) != GQE_OK) return 0;
  return make_ws_layout(*dims).total;
}

gqe_status gqe_route(const gqe_dims* dims, const void* x, const void* W_r, const float* bias,
                     int32_t* topk_idx, float* p, float* w, void* ws, size_t ws_bytes,
                     void* stream) {
  gqe_status st = check_dims(dims, true);
  if (st != GQE_OK) return st;
  if (!aligned16(x) || !aligned16(W_r) || !aligned16(topk_idx) || !aligned16(p) ||
      !aligned16(w) || (bias && !aligned16(bias)))
    return GQE_ERR_INVALID_ARG;
  const WsLayout L = make_ws_layout(*dims);
  if (!aligned16(ws) || ws_bytes < L.total) return GQE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* wb = static_cast<uint8_t*>(ws);
  RouteArgs a{};
  a.x = static_cast<const uint16_t*>(x);
  a.Wr = static_cast<const uint16_t*>(W_r);
  a.bias = bias;
  a.topk_idx = topk_idx;
  a.p = p;
  a.w = w;
  a.fix_list = reinterpret_cast<int32_t*>(wb + L.fix_list);
  a.wt = reinterpret_cast<float*>(wb + L.wt);
  a.wsq = reinterpret_cast<float*>(wb + L.wsq);
  a.fix_count = reinterpret_cast<int32_t*>(wb + L.counters);
  a.status = reinterpret_cast<int*>(wb + L.status);
  a.T = dims->B * dims->S;
  a.dm = dims->d_model;
  a.G = dims->G;
  a.M = dims->N / dims->G;
  a.k = dims->k;
  return from_cuda(launch_route(a, s));
}

static BucketArgs bucket_args(const gqe_dims* dims, const int32_t* topk_idx, int32_t* off,
                              int32_t* tok, uint8_t* wb, const WsLayout& L) {
  BucketArgs a{};
  a.topk_idx = topk_idx;
  a.bucket_off = off;
  a.bucket_tok = tok;
  a.tiles_raw = reinterpret_cast<TileDesc*>(wb + L.tiles_raw);
  a.tiles = reinterpret_cast<TileDesc*>(wb + L.tiles);
  a.tile_count = reinterpret_cast<int32_t*>(wb + L.counters) + 1;
  a.done = reinterpret_cast<int32_t*>(wb + L.counters) + 2;
  a.status = reinterpret_cast<int*>(wb + L.status);
  a.B = dims->B;
  a.S = dims->S;
  a.G = dims->G;
  a.M = dims->N / dims->G;
  a.k = dims->k;
  a.cap_bg = L.cap_bg;
  a.n_raw_tiles = L.n_raw_tiles;
  a.T = dims->S;
  return a;
}

gqe_status gqe_bucket(const gqe_dims* dims, const int32_t* topk_idx, int32_t* bucket_off,
                      int32_t* bucket_tok, void* ws, size_t ws_bytes, void* stream) {
  gqe_status st = check_dims(dims, false);
  if (st != GQE_OK) return st;
  if (!aligned16(topk_idx) || !aligned16(bucket_off) || !aligned16(bucket_tok))
    return GQE_ERR_INVALID_ARG;
  const WsLayout L = make_ws_layout(*dims);
  if (!aligned16(ws) || ws_bytes < L.total) return GQE_ERR_WORKSPACE;
  uint8_t* wb = static_cast<uint8_t*>(ws);
  const BucketArgs a = bucket_args(dims, topk_idx, bucket_off, bucket_tok, wb, L);
  return from_cuda(launch_prep(a, nullptr, false, static_cast<cudaStream_t>(stream)));
}

static AttnArgs attn_common(const gqe_dims* dims, uint8_t* wb, const WsLayout& L) {
  AttnArgs a;
  std::memset(&a, 0, sizeof(a));
  a.status = reinterpret_cast<int*>(wb + L.status);
  a.B = dims->B;
  a.S = dims->S;
  a.N = dims->N;
  a.G = dims->G;
  a.M = dims->N / dims->G;
  a.k = dims->k;
  a.d = dims->d;
  a.out_fp32 = dims->out_fp32;
  a.T = dims->S;
  a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(dims->d)));
  a.wait_limit_ns = kWaitLimitNs;
  return a;
}

}  // extern "C"

namespace {

// The routed prefill over a KV sequence of T slots (T = S and null offsets:
// plain prefill; otherwise a chunk of S queries at absolute positions
// q_off[b] + i over a cache, with the first valid slot kv_start[b]).
gqe_status attention_prefill_impl(const gqe_dims* dims, int32_t T, const void* Q, const void* Qs,
                                  const void* K, const void* V, const int32_t* q_off,
                                  const int32_t* kv_start, const int32_t* topk_idx,
                                  const float* w, void* O_sel, void* o_bar, void* s_out,
                                  int64_t out_row_stride, void* ws, size_t ws_bytes,
                                  void* stream, float* lse_sel = nullptr,
                                  float* lse_s = nullptr, bool list_built = false,
                                  bool v16_built = false) {
  gqe_status st = check_dims(dims, false);
  if (st != GQE_OK) return st;
  if (T < dims->S) return GQE_ERR_INVALID_ARG;
  if (static_cast<int64_t>(dims->B) * T * dims->G * dims->d >= (int64_t(1) << 40) ||
      (static_cast<int64_t>(T) / kTileN + 3) * 4 > 200 * 1024)
    return GQE_ERR_UNSUPPORTED;
  if (!aligned16(Q) || !aligned16(Qs) || !aligned16(K) || !aligned16(V) ||
      !aligned16(topk_idx) || !aligned16(w) || !aligned16(O_sel) || !aligned16(o_bar) ||
      !aligned16(s_out) || (q_off && !aligned16(q_off)) || (kv_start && !aligned16(kv_start)))
    return GQE_ERR_INVALID_ARG;
  if (out_row_stride < dims->d || out_row_stride % 8 != 0) return GQE_ERR_INVALID_ARG;
  const WsLayout L = make_ws_layout(*dims, T);
  if (!aligned16(ws) || ws_bytes < L.total) return GQE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* wb = static_cast<uint8_t*>(ws);
  const int64_t B = dims->B, G = dims->G, d = dims->d;
  const bool chunked = q_off || kv_start || T != dims->S;

  ConvertArgs cv{static_cast<const uint16_t*>(V), reinterpret_cast<uint16_t*>(wb + L.v16),
                 B * T * G * d, reinterpret_cast<int*>(wb + L.status)};
  // one decision for the call: the work-list format and the kernel follow it
  // (chunked calls always take the one-tile kernel)
  const bool pair = !chunked && pair_kernel_for(*dims);
  BucketArgs ba = bucket_args(dims, topk_idx, reinterpret_cast<int32_t*>(wb + L.bucket_off),
                              reinterpret_cast<int32_t*>(wb + L.bucket_tok), wb, L);
  ba.pairs = pair ? 1 : 0;
  ba.q_off = q_off;
  ba.kv_start = kv_start;
  ba.T = T;
  // list_built: the buckets and the one-tile work list for these top-k are
  // already in the workspace (the layer's routed Q projection built them);
  // v16_built: so is the fp16 copy of V (the layer converts it on its side
  // stream); what is left of the preparation runs here
  cudaError_t e = cudaSuccess;
  if (!(list_built && !pair))
    e = launch_prep(ba, &cv, true, s);
  else if (!v16_built)
    e = launch_convert_v(cv, s);
  if (e != cudaSuccess) return GQE_ERR_CUDA;

  AttnArgs a = attn_common(dims, wb, L);
  if (!map_bshd(&a.tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, dims->B, T, dims->G, dims->d) ||
      !map_bshd(&a.tmV, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, wb + L.v16, dims->B, T, dims->G,
                dims->d) ||
      !map_bshd(&a.tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Q, dims->B, dims->S, dims->N, dims->d) ||
      !map_bsd(&a.tmQs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Qs, dims->B, dims->S, dims->d))
    return GQE_ERR_CUDA;
  a.Q = static_cast<const uint16_t*>(Q);
  a.bucket_off = reinterpret_cast<const int32_t*>(wb + L.bucket_off);
  a.bucket_tok = reinterpret_cast<const int32_t*>(wb + L.bucket_tok);
  a.topk_idx = topk_idx;
  a.tiles = reinterpret_cast<const TileDesc*>(wb + L.tiles);
  a.tile_count = reinterpret_cast<const int32_t*>(wb + L.counters) + 1;
  a.O_sel = O_sel;
  a.o_bar = o_bar;
  a.s_out = s_out;
  a.out_row_stride = out_row_stride;
  a.q_off = q_off;
  a.kv_start = kv_start;
  a.T = T;
  a.lse_sel = lse_sel;
  a.lse_s = lse_s;
  a.dense = 0;
  a.pair = pair ? 1 : 0;
  e = timed_attention(a, L.n_raw_tiles, s);
  if (e != cudaSuccess) return GQE_ERR_CUDA;

  if (dims->k > 1) {
    CombineArgs c{O_sel, o_bar, w, out_row_stride, dims->B * dims->S, dims->G, dims->k, dims->d,
                  dims->out_fp32};
    e = launch_combine(c, s);
    if (e != cudaSuccess) return GQE_ERR_CUDA;
  }
  return GQE_OK;
}

}  // namespace

extern "C" {

gqe_status gqe_attention_prefill(const gqe_dims* dims, const void* Q, const void* Qs,
                                 const void* K, const void* V, const int32_t* topk_idx,
                                 const float* w, void* O_sel, void* o_bar, void* s_out,
                                 int64_t out_row_stride, void* ws, size_t ws_bytes,
                                 void* stream) {
  if (!dims) return GQE_ERR_INVALID_ARG;
  return attention_prefill_impl(dims, dims->S, Q, Qs, K, V, nullptr, nullptr, topk_idx, w, O_sel,
                                o_bar, s_out, out_row_stride, ws, ws_bytes, stream);
}

size_t gqe_prefill_chunk_workspace_size(const gqe_dims* dims, int32_t T) {
  if (check_dims(dims, false) != GQE_OK || T < dims->S) return 0;
  return make_ws_layout(*dims, T).total;
}

gqe_status gqe_attention_prefill_train(const gqe_dims* dims, const void* Q, const void* Qs,
                                       const void* K, const void* V, const int32_t* topk_idx,
                                       const float* w, void* O_sel, void* o_bar, void* s_out,
                                       int64_t out_row_stride, float* lse_sel, float* lse_s,
                                       void* ws, size_t ws_bytes, void* stream) {
  if (!dims) return GQE_ERR_INVALID_ARG;
  if (dims->out_fp32 != 1 || !aligned16(lse_sel) || !aligned16(lse_s))
    return GQE_ERR_INVALID_ARG;
  return attention_prefill_impl(dims, dims->S, Q, Qs, K, V, nullptr, nullptr, topk_idx, w, O_sel,
                                o_bar, s_out, out_row_stride, ws, ws_bytes, stream, lse_sel,
                                lse_s);
}

gqe_status gqe_attention_prefill_chunk(const gqe_dims* dims, int32_t T, const void* Q,
                                       const void* Qs, const void* Kc, const void* Vc,
                                       const int32_t* q_off, const int32_t* kv_start,
                                       const int32_t* topk_idx, const float* w, void* O_sel,
                                       void* o_bar, void* s_out, int64_t out_row_stride,
                                       void* ws, size_t ws_bytes, void* stream) {
  if (!dims) return GQE_ERR_INVALID_ARG;
  return attention_prefill_impl(dims, T, Q, Qs, Kc, Vc, q_off, kv_start, topk_idx, w, O_sel,
                                o_bar, s_out, out_row_stride, ws, ws_bytes, stream);
}

gqe_status gqe_dense_gqa_prefill(const gqe_dims* dims, const void* Q, const void* K,
                                 const void* V, void* O, void* ws, size_t ws_bytes,
                                 void* stream) {
  gqe_status st = check_dims(dims, false);
  if (st != GQE_OK) return st;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return GQE_ERR_INVALID_ARG;
  const WsLayout L = make_ws_layout(*dims);
  if (!aligned16(ws) || ws_bytes < L.total) return GQE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* wb = static_cast<uint8_t*>(ws);
  const int64_t B = dims->B, S = dims->S, G = dims->G, d = dims->d;
  ConvertArgs cv{static_cast<const uint16_t*>(V), reinterpret_cast<uint16_t*>(wb + L.v16),
                 B * S * G * d, reinterpret_cast<int*>(wb + L.status)};
  if (launch_convert_v(cv, s) != cudaSuccess) return GQE_ERR_CUDA;
  AttnArgs a = attn_common(dims, wb, L);
  if (!map_bshd(&a.tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, dims->B, dims->S, dims->G, dims->d) ||
      !map_bshd(&a.tmV, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, wb + L.v16, dims->B, dims->S, dims->G,
                dims->d) ||
      !map_bshd(&a.tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Q, dims->B, dims->S, dims->N, dims->d))
    return GQE_ERR_CUDA;
  a.tmQs = a.tmQ;  // unused by dense tiles
  a.Q = static_cast<const uint16_t*>(Q);
  a.O_dense = O;
  a.dense = 1;
  return from_cuda(timed_attention(a, 0, s));
}

int64_t gqe_set_pair_threshold(int64_t kv_bytes) { return set_pair_threshold(kv_bytes); }

int32_t gqe_set_router_resident(int32_t on) { return set_route_force_resident(on); }

// ------------------------------------------------------------ backward

namespace {
struct BwdLayout {
  size_t dO_r, D_r, dO_s, D_s, total;
};
BwdLayout bwd_layout(const gqe_dims& d) {
  BwdLayout L{};
  const WsLayout W = make_ws_layout(d);
  const int64_t T = static_cast<int64_t>(d.B) * d.S, R = T * d.G * d.k;
  size_t off = W.total;
  L.dO_r = off; off = align_up(off + sizeof(uint16_t) * R * d.d, 256);
  L.D_r = off;  off = align_up(off + sizeof(float) * R, 256);
  L.dO_s = off; off = align_up(off + sizeof(uint16_t) * T * d.d, 256);
  L.D_s = off;  off = align_up(off + sizeof(float) * T, 256);
  L.total = off;
  return L;
}
}  // namespace

size_t gqe_prefill_backward_workspace_size(const gqe_dims* dims) {
  if (check_dims(dims, false) != GQE_OK) return 0;
  return bwd_layout(*dims).total;
}

gqe_status gqe_prefill_backward(const gqe_dims* dims, const void* Q, const void* Qs,
                                const void* K, const void* V, const int32_t* topk_idx,
                                const float* w, const float* O_sel, const float* s_out,
                                int64_t out_row_stride, const float* lse_sel, const float* lse_s,
                                const float* dO_sel, const float* do_bar, const float* ds,
                                int64_t dout_row_stride, float* dQ, float* dQs, float* dK,
                                float* dV, float* dw, void* ws, size_t ws_bytes, void* stream) {
  gqe_status st = check_dims(dims, false);
  if (st != GQE_OK) return st;
  const void* ptrs[] = {Q, Qs, K, V, topk_idx, w, O_sel, s_out, lse_sel, lse_s, dO_sel, do_bar,
                        ds, dQ, dQs, dK, dV, dw};
  for (const void* q : ptrs)
    if (!aligned16(q)) return GQE_ERR_INVALID_ARG;
  if (out_row_stride < dims->d || out_row_stride % 4 != 0 || dout_row_stride < dims->d ||
      dout_row_stride % 4 != 0)
    return GQE_ERR_INVALID_ARG;
  const WsLayout L = make_ws_layout(*dims);
  const BwdLayout BL = bwd_layout(*dims);
  if (!aligned16(ws) || ws_bytes < BL.total) return GQE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* wb = static_cast<uint8_t*>(ws);
  BucketArgs ba = bucket_args(dims, topk_idx, reinterpret_cast<int32_t*>(wb + L.bucket_off),
                              reinterpret_cast<int32_t*>(wb + L.bucket_tok), wb, L);
  if (launch_prep(ba, nullptr, false, s) != cudaSuccess) return GQE_ERR_CUDA;
  const int64_t T = static_cast<int64_t>(dims->B) * dims->S;
  if (cudaMemsetAsync(dQ, 0, sizeof(float) * T * dims->N * dims->d, s) != cudaSuccess ||
      cudaMemsetAsync(dQs, 0, sizeof(float) * T * dims->d, s) != cudaSuccess)
    return GQE_ERR_CUDA;
  BwdArgs a;
  std::memset(&a, 0, sizeof(a));
  if (!map_bshd(&a.tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, dims->B, dims->S, dims->G, dims->d) ||
      !map_bshd(&a.tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, V, dims->B, dims->S, dims->G, dims->d))
    return GQE_ERR_CUDA;
  a.Q = static_cast<const uint16_t*>(Q);
  a.Qs = static_cast<const uint16_t*>(Qs);
  a.topk_idx = topk_idx;
  a.w = w;
  a.bucket_off = reinterpret_cast<const int32_t*>(wb + L.bucket_off);
  a.bucket_tok = reinterpret_cast<const int32_t*>(wb + L.bucket_tok);
  a.O_sel = O_sel;
  a.s_out = s_out;
  a.out_row_stride = out_row_stride;
  a.lse_sel = lse_sel;
  a.lse_s = lse_s;
  a.dO_sel = dO_sel;
  a.do_bar = do_bar;
  a.ds = ds;
  a.dout_row_stride = dout_row_stride;
  a.dO_r_out = reinterpret_cast<uint16_t*>(wb + BL.dO_r);
  a.dO_r = a.dO_r_out;
  a.D_r_out = reinterpret_cast<float*>(wb + BL.D_r);
  a.D_r = a.D_r_out;
  a.dO_s_out = reinterpret_cast<uint16_t*>(wb + BL.dO_s);
  a.dO_s = a.dO_s_out;
  a.D_s_out = reinterpret_cast<float*>(wb + BL.D_s);
  a.D_s = a.D_s_out;
  a.dQ = dQ;
  a.dQs = dQs;
  a.dK = dK;
  a.dV = dV;
  a.dw = dw;
  a.status = reinterpret_cast<int*>(wb + L.status);
  a.B = dims->B;
  a.S = dims->S;
  a.N = dims->N;
  a.G = dims->G;
  a.M = dims->N / dims->G;
  a.k = dims->k;
  a.d = dims->d;
  a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(dims->d)));
  a.inv_sqrt_d = static_cast<float>(1.0 / std::sqrt(static_cast<double>(dims->d)));
  a.wait_limit_ns = kWaitLimitNs;
  return from_cuda(launch_bwd(a, s));
}

// ------------------------------------------------------------ projections

gqe_status gqe_linear(int32_t rows, int32_t K, int32_t nb, int32_t nc, const void* A, int64_t lda,
                      const void* W, void* C, int64_t ldc, int32_t c_fp32, void* stream) {
  if (rows < 1 || K < 64 || K % 64 != 0 || nb < 1 || nc < 64 || nc % 64 != 0)
    return GQE_ERR_UNSUPPORTED;
  if (c_fp32 != 0 && c_fp32 != 1) return GQE_ERR_INVALID_ARG;
  const int64_t n_total = static_cast<int64_t>(nb) * nc;
  if (lda < K || lda % 8 != 0 || ldc < n_total || ldc % (c_fp32 ? 4 : 8) != 0)
    return GQE_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(W) || !aligned16(C)) return GQE_ERR_INVALID_ARG;
  if (n_total > (int64_t(1) << 30) || static_cast<int64_t>(rows) * ldc >= (int64_t(1) << 40))
    return GQE_ERR_UNSUPPORTED;
  GemmArgs g;
  std::memset(&g, 0, sizeof(g));
  const uint64_t adims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(rows)};
  const uint64_t astr[1] = {static_cast<uint64_t>(lda) * 2};
  const uint32_t abox[2] = {64, static_cast<uint32_t>(kTileM)};
  const uint64_t bdims[3] = {static_cast<uint64_t>(nc), static_cast<uint64_t>(K),
                             static_cast<uint64_t>(nb)};
  const uint64_t bstr[2] = {static_cast<uint64_t>(nc) * 2, static_cast<uint64_t>(K) * nc * 2};
  const uint32_t bbox[3] = {64, 64, 1};
  if (!encode_map(&g.tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, A, adims, astr, abox) ||
      !encode_map(&g.tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, W, bdims, bstr, bbox))
    return GQE_ERR_CUDA;
  g.C = C;
  g.ldc = ldc;
  g.c_fp32 = c_fp32;
  g.K = K;
  g.nc = nc;
  g.n_total = static_cast<int>(n_total);
  g.rows = rows;
  g.wait_limit_ns = kWaitLimitNs;
  g.status = nullptr;
  // column tile: 256 when that still gives two tiles per SM, else 128 or 64
  const int64_t mt = (rows + kTileM - 1) / kTileM;
  int bn = 64;
  if (n_total % 256 == 0 && mt * (n_total / 256) >= 296) bn = 256;
  else if (n_total % 128 == 0) bn = 128;
  return from_cuda(launch_gemm_dense(g, bn, static_cast<cudaStream_t>(stream)));
}

gqe_status gqe_routed_q_project(const gqe_dims* dims, const void* x, const void* W_Q,
                                const int32_t* topk_idx, void* Q, void* ws, size_t ws_bytes,
                                void* stream) {
  gqe_status st = check_dims(dims, false);
  if (st != GQE_OK) return st;
  if (dims->d_model < 64 || dims->d_model % 64 != 0) return GQE_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(W_Q) || !aligned16(topk_idx) || !aligned16(Q))
    return GQE_ERR_INVALID_ARG;
  const WsLayout L = make_ws_layout(*dims);
  if (!aligned16(ws) || ws_bytes < L.total) return GQE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* wb = static_cast<uint8_t*>(ws);
  // the bucket lists and the work list the attention call builds too
  BucketArgs ba = bucket_args(dims, topk_idx, reinterpret_cast<int32_t*>(wb + L.bucket_off),
                              reinterpret_cast<int32_t*>(wb + L.bucket_tok), wb, L);
  ba.pairs = 0;
  if (launch_prep(ba, nullptr, true, s) != cudaSuccess) return GQE_ERR_CUDA;
  GemmArgs g;
  std::memset(&g, 0, sizeof(g));
  const uint64_t bdims[3] = {static_cast<uint64_t>(dims->d), static_cast<uint64_t>(dims->d_model),
                             static_cast<uint64_t>(dims->N)};
  const uint64_t bstr[2] = {static_cast<uint64_t>(dims->d) * 2,
                            static_cast<uint64_t>(dims->d_model) * dims->d * 2};
  const uint32_t bbox[3] = {64, 64, 1};
  if (!encode_map(&g.tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, W_Q, bdims, bstr, bbox))
    return GQE_ERR_CUDA;
  g.A = static_cast<const uint16_t*>(x);
  g.lda = dims->d_model;
  g.C = Q;
  g.K = dims->d_model;
  g.nc = dims->d;
  g.bucket_off = reinterpret_cast<const int32_t*>(wb + L.bucket_off);
  g.bucket_tok = reinterpret_cast<const int32_t*>(wb + L.bucket_tok);
  g.tiles = reinterpret_cast<const TileDesc*>(wb + L.tiles);
  g.tile_count = reinterpret_cast<const int32_t*>(wb + L.counters) + 1;
  g.B = dims->B;
  g.S = dims->S;
  g.N = dims->N;
  g.G = dims->G;
  g.M = dims->N / dims->G;
  g.d = dims->d;
  g.status = reinterpret_cast<int*>(wb + L.status);
  g.wait_limit_ns = kWaitLimitNs;
  return from_cuda(launch_gemm_routed(g, L.n_raw_tiles, s));
}

gqe_status gqe_layer_prefill(const gqe_dims* dims, const void* x, const void* W_Q,
                             const void* W_K, const void* W_V, const void* W_s, const void* W_r,
                             const float* bias, const void* W_O, int32_t* topk_idx, float* p,
                             float* w, void* Q, void* Qs, void* K, void* V, void* concat,
                             float* y, void* ws, size_t ws_bytes, void* stream) {
  gqe_status st = check_dims(dims, true);
  if (st != GQE_OK) return st;
  if (dims->d_model % 64 != 0) return GQE_ERR_UNSUPPORTED;
  gqe_dims db = *dims;
  db.out_fp32 = 0;  // the concat buffer feeds W_O as bf16
  const int32_t T = dims->B * dims->S, dm = dims->d_model, d = dims->d, G = dims->G;
  const int64_t row = static_cast<int64_t>(G * dims->k + G + 1) * d;
  if (!aligned16(concat) || !aligned16(y)) return GQE_ERR_INVALID_ARG;
  // K, V and Qs do not depend on the routing: they run on the side stream
  // while this stream routes and projects the selected query heads; the
  // attention call waits for both.
  cudaStream_t s = static_cast<cudaStream_t>(stream), side = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  if (side_stream(&side) != cudaSuccess ||
      cudaEventCreateWithFlags(&fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&join, cudaEventDisableTiming) != cudaSuccess) {
    if (fork) cudaEventDestroy(fork);
    return GQE_ERR_CUDA;
  }
  // destroying an event whose record is still pending is allowed
  struct Events {
    cudaEvent_t a, b;
    ~Events() {
      cudaEventDestroy(a);
      cudaEventDestroy(b);
    }
  } guard{fork, join};
  if (cudaEventRecord(fork, s) != cudaSuccess || cudaStreamWaitEvent(side, fork, 0) != cudaSuccess)
    return GQE_ERR_CUDA;
  if ((st = gqe_linear(T, dm, G, d, x, dm, W_K, K, int64_t(G) * d, 0, side)) != GQE_OK) return st;
  if ((st = gqe_linear(T, dm, G, d, x, dm, W_V, V, int64_t(G) * d, 0, side)) != GQE_OK) return st;
  // V to fp16 for the attention's P.V (into the workspace), off the critical path
  const bool pair = pair_kernel_for(db);
  const WsLayout L = make_ws_layout(db);
  if (!aligned16(ws) || ws_bytes < L.total) return GQE_ERR_WORKSPACE;
  uint8_t* wb = static_cast<uint8_t*>(ws);
  ConvertArgs cv{static_cast<const uint16_t*>(V), reinterpret_cast<uint16_t*>(wb + L.v16),
                 int64_t(T) * G * d, reinterpret_cast<int*>(wb + L.status)};
  if (!pair && launch_convert_v(cv, side) != cudaSuccess) return GQE_ERR_CUDA;
  if ((st = gqe_linear(T, dm, 1, d, x, dm, W_s, Qs, d, 0, side)) != GQE_OK) return st;
  if (cudaEventRecord(join, side) != cudaSuccess) return GQE_ERR_CUDA;
  if ((st = gqe_route(&db, x, W_r, bias, topk_idx, p, w, ws, ws_bytes, stream)) != GQE_OK)
    return st;
  if ((st = gqe_routed_q_project(&db, x, W_Q, topk_idx, Q, ws, ws_bytes, stream)) != GQE_OK)
    return st;
  if (cudaStreamWaitEvent(s, join, 0) != cudaSuccess) return GQE_ERR_CUDA;
  uint16_t* cb = static_cast<uint16_t*>(concat);
  const int64_t a = int64_t(G) * dims->k * d;
  // the routed Q projection left this call's buckets and work list in ws, the
  // side stream its fp16 V
  if ((st = attention_prefill_impl(&db, db.S, Q, Qs, K, V, nullptr, nullptr, topk_idx, w, cb,
                                   cb + a, cb + a + G * d, row, ws, ws_bytes, stream, nullptr,
                                   nullptr, true, true)) != GQE_OK)
    return st;
  return gqe_linear(T, static_cast<int32_t>(row), 1, dm, concat, row, W_O, y, dm, 1, stream);
}

gqe_status gqe_dense_layer_prefill(const gqe_dims* dims, const void* x, const void* W_Q,
                                   const void* W_K, const void* W_V, const void* W_O, void* Q,
                                   void* K, void* V, void* O, float* y, void* ws,
                                   size_t ws_bytes, void* stream) {
  gqe_status st = check_dims(dims, false);
  if (st != GQE_OK) return st;
  if (dims->d_model < 64 || dims->d_model % 64 != 0) return GQE_ERR_UNSUPPORTED;
  gqe_dims db = *dims;
  db.out_fp32 = 0;  // O feeds W_O as bf16
  const int32_t T = dims->B * dims->S, dm = dims->d_model, d = dims->d, G = dims->G,
                N = dims->N;
  if ((st = gqe_linear(T, dm, N, d, x, dm, W_Q, Q, int64_t(N) * d, 0, stream)) != GQE_OK)
    return st;
  if ((st = gqe_linear(T, dm, G, d, x, dm, W_K, K, int64_t(G) * d, 0, stream)) != GQE_OK)
    return st;
  if ((st = gqe_linear(T, dm, G, d, x, dm, W_V, V, int64_t(G) * d, 0, stream)) != GQE_OK)
    return st;
  if ((st = gqe_dense_gqa_prefill(&db, Q, K, V, O, ws, ws_bytes, stream)) != GQE_OK) return st;
  return gqe_linear(T, N * d, 1, dm, O, int64_t(N) * d, W_O, y, dm, 1, stream);
}

size_t gqe_decode_workspace_size(const gqe_dims* dims) {
  if (check_dims(dims, false) != GQE_OK) return 0;
  return make_decode_plan(*dims).total;
}

size_t gqe_append_workspace_size(const gqe_dims* dims, int32_t n_new) {
  if (check_dims(dims, false) != GQE_OK || n_new < 1 || n_new > kMaxAppend ||
      n_new > dims->S)
    return 0;
  return make_decode_plan(*dims, n_new).total;
}

gqe_status gqe_attention_append(const gqe_dims* dims, int32_t n_new, const void* Q,
                                const void* Qs, const void* Kc, const void* Vc,
                                const int32_t* pos, const int32_t* kv_start,
                                const int32_t* topk_idx, const float* w, void* O_sel,
                                void* o_bar, void* s_out, int64_t out_row_stride, void* ws,
                                size_t ws_bytes, void* stream) {
  gqe_status st = check_dims(dims, false);
  if (st != GQE_OK) return st;
  if (n_new < 1 || n_new > kMaxAppend || n_new > dims->S) return GQE_ERR_INVALID_ARG;
  if (static_cast<int64_t>(dims->B) * n_new * dims->N >= (int64_t(1) << 31))
    return GQE_ERR_UNSUPPORTED;
  if (!aligned16(Q) || !aligned16(Qs) || !aligned16(Kc) || !aligned16(Vc) || !aligned16(pos) ||
      !aligned16(topk_idx) || !aligned16(w) || !aligned16(O_sel) || !aligned16(o_bar) ||
      !aligned16(s_out) || (kv_start && !aligned16(kv_start)))
    return GQE_ERR_INVALID_ARG;
  if (out_row_stride < dims->d || out_row_stride % 8 != 0) return GQE_ERR_INVALID_ARG;
  const DecodePlan P = make_decode_plan(*dims, n_new);
  if (!aligned16(ws) || ws_bytes < P.total) return GQE_ERR_WORKSPACE;
  uint8_t* wb = static_cast<uint8_t*>(ws);
  DecodeArgs a{};
  a.Q = static_cast<const uint16_t*>(Q);
  a.Qs = static_cast<const uint16_t*>(Qs);
  a.Kc = static_cast<const uint16_t*>(Kc);
  a.Vc = static_cast<const uint16_t*>(Vc);
  a.pos = pos;
  a.kv_start = kv_start;
  a.topk_idx = topk_idx;
  a.w = w;
  a.part_m = reinterpret_cast<float*>(wb + P.part_m);
  a.part_l = reinterpret_cast<float*>(wb + P.part_l);
  a.part_o = reinterpret_cast<float*>(wb + P.part_o);
  a.O_sel = O_sel;
  a.o_bar = o_bar;
  a.s_out = s_out;
  a.out_row_stride = out_row_stride;
  a.status = reinterpret_cast<int*>(wb + P.status);
  a.B = dims->B;
  a.T = dims->S;
  a.N = dims->N;
  a.G = dims->G;
  a.M = dims->N / dims->G;
  a.k = dims->k;
  a.d = dims->d;
  a.n_new = n_new;
  a.heads = static_cast<int>(P.heads);
  a.passes = static_cast<int>(P.passes);
  a.nchunks = static_cast<int>(P.nchunks);
  a.chunk = static_cast<int>(P.chunk);
  a.out_fp32 = dims->out_fp32;
  a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(dims->d)));
  return from_cuda(launch_decode(a, static_cast<cudaStream_t>(stream)));
}

gqe_status gqe_attention_decode(const gqe_dims* dims, const void* Q, const void* Qs,
                                const void* Kc, const void* Vc, const int32_t* pos,
                                const int32_t* kv_start, const int32_t* topk_idx,
                                const float* w, void* O_sel, void* o_bar, void* s_out,
                                int64_t out_row_stride, void* ws, size_t ws_bytes,
                                void* stream) {
  return gqe_attention_append(dims, 1, Q, Qs, Kc, Vc, pos, kv_start, topk_idx, w, O_sel, o_bar,
                              s_out, out_row_stride, ws, ws_bytes, stream);
}

gqe_status gqe_get_device_status(void* ws, int32_t clear, void* stream) {
  if (!aligned16(ws)) return GQE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return GQE_ERR_CUDA;
  int32_t code = 0;
  if (cudaMemcpy(&code, ws, sizeof(code), cudaMemcpyDeviceToHost) != cudaSuccess)
    return GQE_ERR_CUDA;
  if (clear && cudaMemset(ws, 0, sizeof(int32_t)) != cudaSuccess) return GQE_ERR_CUDA;
  if (code < GQE_OK || code > GQE_ERR_BAD_POSITION) return GQE_ERR_CUDA;
  return static_cast<gqe_status>(code);
}

uint64_t gqe_kv_cache_bytes(int32_t L, int32_t G, int64_t S, int32_t d, int32_t bytes_per_elem,
                            int32_t B) {
  if (L < 0 || G < 0 || S < 0 || d < 0 || bytes_per_elem < 0 || B < 0) return 0;
  return 2ull * static_cast<uint64_t>(L) * static_cast<uint64_t>(G) * static_cast<uint64_t>(d) *
         static_cast<uint64_t>(S) * static_cast<uint64_t>(bytes_per_elem) *
         static_cast<uint64_t>(B);
}

const char* gqe_status_string(gqe_status s) {
  switch (s) {
    case GQE_OK: return "ok";
    case GQE_ERR_INVALID_ARG: return "invalid argument";
    case GQE_ERR_UNSUPPORTED: return "unsupported shape";
    case GQE_ERR_CUDA: return "CUDA error";
    case GQE_ERR_TIMEOUT: return "device wait timed out";
    case GQE_ERR_WORKSPACE: return "workspace missing or too small";
    case GQE_ERR_BAD_INDEX: return "expert index out of range";
    case GQE_ERR_NONFINITE: return "non-finite value or value outside the fp16 range";
    case GQE_ERR_BAD_POSITION: return "decode position out of range";
  }
  return "unknown status";
}

void gqe_set_profile_events(void* begin, void* end) {
  set_profile_events(static_cast<cudaEvent_t>(begin), static_cast<cudaEvent_t>(end));
}

gqe_status gqe_selftest_bounded_wait(void* ws, size_t ws_bytes, int32_t limit_us, void* stream) {
  if (!aligned16(ws) || ws_bytes < 256) return GQE_ERR_WORKSPACE;
  if (limit_us < 1 || limit_us > 10000000) return GQE_ERR_INVALID_ARG;
  return from_cuda(launch_selftest_wait(static_cast<int*>(ws),
                                        static_cast<uint64_t>(limit_us) * 1000ull,
                                        static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
