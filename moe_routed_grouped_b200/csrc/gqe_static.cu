// gqe_attention_prefill_static: the routed attention call for callers that
// cannot hand the library a workspace.
//
// Some callers cannot allocate device memory when they call the library: a
// plugin running inside a host framework that owns every device allocation,
// or a serving loop that must not pay the device-wide synchronisation that
// cudaMalloc implies.  This entry point needs no workspace: its scratch (V
// converted to fp16, the per-expert token lists and the attention work list)
// lives in one file-scope device array of fixed size, which every GPU that
// loads this library keeps until the process exits.
#include <cmath>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "gqe_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;  // 64 MiB per device
constexpr int kMaxDevices = 64;

__device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

// Regions of the static scratch: status word, counters, then the same
// attention regions as a caller workspace (the router regions are unused).
struct StaticLayout {
  size_t status, counters, v16, bucket_off, bucket_tok, tiles_raw, tiles, total;
  int64_t cap_bg, n_raw_tiles;
};

StaticLayout static_layout(const gqe_dims& d) {
  StaticLayout L{};
  const int64_t B = d.B, S = d.S, G = d.G, M = d.N / d.G, k = d.k, hd = d.d;
  gqe::tile_list_dims(B, S, G, M, k, &L.cap_bg, &L.n_raw_tiles);
  size_t off = 0;
  L.status = off;     off += 256;
  L.counters = off;   off += 256;
  L.v16 = off;        off = gqe::align_up(off + sizeof(uint16_t) * B * S * G * hd, 256);
  L.bucket_off = off; off = gqe::align_up(off + sizeof(int32_t) * (B * G * M + 1), 256);
  L.bucket_tok = off; off = gqe::align_up(off + sizeof(int32_t) * B * G * S * k, 256);
  L.tiles_raw = off;  off = gqe::align_up(off + sizeof(gqe::TileDesc) * L.n_raw_tiles, 256);
  L.tiles = off;      off = gqe::align_up(off + sizeof(gqe::TileDesc) * L.n_raw_tiles, 256);
  L.total = off;
  return L;
}

// The last device address of g_static_scratch seen on each device.  In host
// code the array's name is only a host-side stand-in, so the address is
// looked up with the device current on every call (a cheap host-side
// lookup): if the context was torn down and rebuilt, the module is reloaded
// and the array may move.  A new address means a freshly loaded module; its
// header (status word and counters) is zeroed before first use.
void* g_seen[kMaxDevices] = {};
std::mutex g_seen_mu;

cudaError_t scratch_for_current_device(uint8_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_static_scratch);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_seen_mu);
  if (g_seen[dev] != p) {
    e = cudaMemset(p, 0, 512);
    if (e != cudaSuccess) return e;
    g_seen[dev] = p;
  }
  *out = static_cast<uint8_t*>(p);
  return cudaSuccess;
}

}  // namespace

extern "C" gqe_status gqe_attention_prefill_static(
    const gqe_dims* dims, const void* Q, const void* Qs, const void* K, const void* V,
    const int32_t* topk_idx, const float* w, void* O_sel, void* o_bar, void* s_out,
    int64_t out_row_stride, void* stream) {
  const gqe_status st = gqe::check_dims(dims, false);  // the checks of gqe_attention_prefill
  if (st != GQE_OK) return st;
  if (!gqe::aligned16(Q) || !gqe::aligned16(Qs) || !gqe::aligned16(K) || !gqe::aligned16(V) ||
      !gqe::aligned16(topk_idx) || !gqe::aligned16(w) || !gqe::aligned16(O_sel) ||
      !gqe::aligned16(o_bar) || !gqe::aligned16(s_out))
    return GQE_ERR_INVALID_ARG;
  if (out_row_stride < dims->d || out_row_stride % 8 != 0) return GQE_ERR_INVALID_ARG;
  const StaticLayout L = static_layout(*dims);
  if (L.total > kStaticScratchBytes) return GQE_ERR_WORKSPACE;  // shape needs more scratch

  uint8_t* sb = nullptr;
  if (scratch_for_current_device(&sb) != cudaSuccess) return GQE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the array keeps the previous call's contents: the counters start at 0;
  // the status word keeps latching until gqe_static_device_status clears it
  if (cudaMemsetAsync(sb + L.counters, 0, 256, s) != cudaSuccess) return GQE_ERR_CUDA;

  const int64_t B = dims->B, S = dims->S, G = dims->G, d = dims->d;
  int* status = reinterpret_cast<int*>(sb + L.status);
  int32_t* counters = reinterpret_cast<int32_t*>(sb + L.counters);
  gqe::ConvertArgs cv{static_cast<const uint16_t*>(V), reinterpret_cast<uint16_t*>(sb + L.v16),
                      B * S * G * d, status};
  gqe::BucketArgs ba{};
  ba.topk_idx = topk_idx;
  ba.bucket_off = reinterpret_cast<int32_t*>(sb + L.bucket_off);
  ba.bucket_tok = reinterpret_cast<int32_t*>(sb + L.bucket_tok);
  ba.tiles_raw = reinterpret_cast<gqe::TileDesc*>(sb + L.tiles_raw);
  ba.tiles = reinterpret_cast<gqe::TileDesc*>(sb + L.tiles);
  ba.tile_count = counters + 1;
  ba.done = counters + 2;
  ba.status = status;
  ba.B = dims->B;
  ba.S = dims->S;
  ba.G = dims->G;
  ba.M = dims->N / dims->G;
  ba.k = dims->k;
  ba.cap_bg = L.cap_bg;
  ba.n_raw_tiles = L.n_raw_tiles;
  ba.T = dims->S;
  const bool pair = gqe::pair_kernel_for(*dims);  // one decision: list format and kernel
  ba.pairs = pair ? 1 : 0;
  if (gqe::launch_prep(ba, &cv, true, s) != cudaSuccess) return GQE_ERR_CUDA;

  gqe::AttnArgs a;
  std::memset(&a, 0, sizeof(a));
  if (!gqe::map_bshd(&a.tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, dims->B, dims->S, dims->G,
                     dims->d) ||
      !gqe::map_bshd(&a.tmV, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, sb + L.v16, dims->B, dims->S,
                     dims->G, dims->d) ||
      !gqe::map_bshd(&a.tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Q, dims->B, dims->S, dims->N,
                     dims->d) ||
      !gqe::map_bsd(&a.tmQs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Qs, dims->B, dims->S, dims->d))
    return GQE_ERR_CUDA;
  a.Q = static_cast<const uint16_t*>(Q);
  a.bucket_off = ba.bucket_off;
  a.bucket_tok = ba.bucket_tok;
  a.topk_idx = topk_idx;
  a.tiles = ba.tiles;
  a.tile_count = ba.tile_count;
  a.O_sel = O_sel;
  a.o_bar = o_bar;
  a.s_out = s_out;
  a.out_row_stride = out_row_stride;
  a.status = status;
  a.B = dims->B;
  a.S = dims->S;
  a.N = dims->N;
  a.G = dims->G;
  a.M = dims->N / dims->G;
  a.k = dims->k;
  a.d = dims->d;
  a.out_fp32 = dims->out_fp32;
  a.T = dims->S;
  a.dense = 0;
  a.pair = pair ? 1 : 0;
  a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(d)));
  a.wait_limit_ns = gqe::kWaitLimitNs;
  if (gqe::timed_attention(a, L.n_raw_tiles, s) != cudaSuccess) return GQE_ERR_CUDA;
  if (dims->k > 1) {
    gqe::CombineArgs c{O_sel, o_bar, w, out_row_stride, dims->B * dims->S, dims->G, dims->k,
                       dims->d, dims->out_fp32};
    if (gqe::launch_combine(c, s) != cudaSuccess) return GQE_ERR_CUDA;
  }
  return GQE_OK;
}

extern "C" gqe_status gqe_static_device_status(int32_t clear, void* stream) {
  uint8_t* sb = nullptr;
  if (scratch_for_current_device(&sb) != cudaSuccess) return GQE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return GQE_ERR_CUDA;
  int32_t code = 0;
  if (cudaMemcpy(&code, sb, sizeof(code), cudaMemcpyDeviceToHost) != cudaSuccess)
    return GQE_ERR_CUDA;
  if (clear && cudaMemset(sb, 0, sizeof(int32_t)) != cudaSuccess) return GQE_ERR_CUDA;
  if (code < GQE_OK || code > GQE_ERR_BAD_POSITION) return GQE_ERR_CUDA;
  return static_cast<gqe_status>(code);
}
