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

// Device address of g_static_scratch on each device, looked up once.
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

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

// Once per device, with that device current: the device address of the
// static array (host code only sees a host-side stand-in for its name), and
// a zeroed header.
cudaError_t scratch_for_current_device(uint8_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return e;
    e = cudaMemset(p, 0, 512);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = static_cast<uint8_t*>(g_scratch_ptr[dev]);
  return cudaSuccess;
}

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Tiled TMA map, 128-byte swizzle, box of 64 elements x 128 rows; dims
// innermost first, byte strides for dims 1..rank-1.
bool encode(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base,
            const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box) {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return fn(m, dt, static_cast<cuuint32_t>(rank), const_cast<void*>(base), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool map_bshd(CUtensorMap* m, CUtensorMapDataType dt, const void* base, int B, int S, int H,
              int d) {
  const cuuint64_t dims[4] = {cuuint64_t(d), cuuint64_t(H), cuuint64_t(S), cuuint64_t(B)};
  const cuuint64_t strides[3] = {cuuint64_t(d) * 2, cuuint64_t(H) * d * 2,
                                 cuuint64_t(S) * H * d * 2};
  const cuuint32_t box[4] = {64, 1, gqe::kTileM, 1};
  return encode(m, dt, 4, base, dims, strides, box);
}

bool map_bsd(CUtensorMap* m, CUtensorMapDataType dt, const void* base, int B, int S, int d) {
  const cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(S), cuuint64_t(B)};
  const cuuint64_t strides[2] = {cuuint64_t(d) * 2, cuuint64_t(S) * d * 2};
  const cuuint32_t box[3] = {64, gqe::kTileM, 1};
  return encode(m, dt, 3, base, dims, strides, box);
}

}  // namespace

extern "C" gqe_status gqe_attention_prefill_static(
    const gqe_dims* dims, const void* Q, const void* Qs, const void* K, const void* V,
    const int32_t* topk_idx, const float* w, void* O_sel, void* o_bar, void* s_out,
    int64_t out_row_stride, void* stream) {
  // the shape checks of gqe_attention_prefill
  if (gqe_workspace_size(dims) == 0) {
    if (!dims || dims->B < 1 || dims->S < 1 || dims->N < 1 || dims->G < 1 || dims->k < 1 ||
        dims->d < 1 || dims->N % dims->G != 0 || dims->k > dims->N / dims->G ||
        (dims->out_fp32 != 0 && dims->out_fp32 != 1))
      return GQE_ERR_INVALID_ARG;
    return GQE_ERR_UNSUPPORTED;
  }
  if (!aligned16(Q) || !aligned16(Qs) || !aligned16(K) || !aligned16(V) ||
      !aligned16(topk_idx) || !aligned16(w) || !aligned16(O_sel) || !aligned16(o_bar) ||
      !aligned16(s_out))
    return GQE_ERR_INVALID_ARG;
  if (out_row_stride < dims->d || out_row_stride % 8 != 0) return GQE_ERR_INVALID_ARG;
  const StaticLayout L = static_layout(*dims);
  if (L.total > kStaticScratchBytes) return GQE_ERR_WORKSPACE;  // shape needs more scratch

  uint8_t* sb = nullptr;
  if (scratch_for_current_device(&sb) != cudaSuccess) return GQE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the array keeps the previous call's contents: status and counters start at 0
  if (cudaMemsetAsync(sb, 0, 512, s) != cudaSuccess) return GQE_ERR_CUDA;

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
  const bool pair = gqe::pair_kernel_for(*dims);  // one decision: list format and kernel
  ba.pairs = pair ? 1 : 0;
  if (gqe::launch_prep(ba, &cv, true, s) != cudaSuccess) return GQE_ERR_CUDA;

  gqe::AttnArgs a;
  std::memset(&a, 0, sizeof(a));
  if (!map_bshd(&a.tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, dims->B, dims->S, dims->G,
                     dims->d) ||
      !map_bshd(&a.tmV, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, sb + L.v16, dims->B, dims->S,
                     dims->G, dims->d) ||
      !map_bshd(&a.tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Q, dims->B, dims->S, dims->N,
                     dims->d) ||
      !map_bsd(&a.tmQs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Qs, dims->B, dims->S, dims->d))
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
  a.dense = 0;
  a.pair = pair ? 1 : 0;
  a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(d)));
  a.wait_limit_ns = gqe::kWaitLimitNs;
  if (gqe::launch_attention(a, L.n_raw_tiles, s) != cudaSuccess) return GQE_ERR_CUDA;
  if (dims->k > 1) {
    gqe::CombineArgs c{O_sel, o_bar, w, out_row_stride, dims->B * dims->S, dims->G, dims->k,
                       dims->d, dims->out_fp32};
    if (gqe::launch_combine(c, s) != cudaSuccess) return GQE_ERR_CUDA;
  }
  return GQE_OK;
}
