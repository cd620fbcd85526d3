// Host-side helpers shared by the C-ABI entry points (gqe_api.cu and
// gqe_static.cu): shape checks, pointer checks, TMA tensor maps and the
// optional profiling events around the attention launch.
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "gqe_internal.h"

namespace gqe {
namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point (looked up
// once; std::call_once makes the lookup safe from several host threads).
EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

std::mutex g_prof_mu;
cudaEvent_t g_prof_begin = nullptr, g_prof_end = nullptr;

}  // namespace

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

gqe_status check_dims(const gqe_dims* d, bool router) {
  if (!d) return GQE_ERR_INVALID_ARG;
  if (d->B < 1 || d->S < 1 || d->N < 1 || d->G < 1 || d->k < 1 || d->d < 1)
    return GQE_ERR_INVALID_ARG;
  if (d->N % d->G != 0) return GQE_ERR_INVALID_ARG;
  const int64_t M = d->N / d->G;
  if (d->k > M) return GQE_ERR_INVALID_ARG;
  if (d->out_fp32 != 0 && d->out_fp32 != 1) return GQE_ERR_INVALID_ARG;
  if (M > kMaxM) return GQE_ERR_UNSUPPORTED;
  if (d->d != 64 && d->d != 128) return GQE_ERR_UNSUPPORTED;
  const int64_t B = d->B, S = d->S, G = d->G, k = d->k;
  const int64_t wide = k > M ? k : M;
  if (B * S * G * wide >= (int64_t(1) << 31)) return GQE_ERR_UNSUPPORTED;
  if (B * S * d->N >= (int64_t(1) << 31)) return GQE_ERR_UNSUPPORTED;
  if (B * G * M >= (int64_t(1) << 24) || B >= (int64_t(1) << 24)) return GQE_ERR_UNSUPPORTED;
  const int64_t nq = (S + kTileM - 1) / kTileM;
  if ((nq + 2) * 4 > 200 * 1024) return GQE_ERR_UNSUPPORTED;  // scheduler histogram
  if (router) {
    if (d->d_model < 8 || d->d_model % 8 != 0) return GQE_ERR_UNSUPPORTED;
    const int64_t gm = G * M;
    if (gm != 4 && gm != 8 && gm != 16 && gm != 32) return GQE_ERR_UNSUPPORTED;
  }
  return GQE_OK;
}

bool encode_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base,
                const uint64_t* dims, const uint64_t* strides, const uint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rank < 1 || rank > 5) return false;
  cuuint64_t gd[5], gs[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides[i];
  return fn(m, dt, static_cast<cuuint32_t>(rank), const_cast<void*>(base), gd, gs, bx, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool map_bshd(CUtensorMap* m, CUtensorMapDataType dt, const void* base, int B, int S, int H,
              int d) {
  const uint64_t dims[4] = {static_cast<uint64_t>(d), static_cast<uint64_t>(H),
                            static_cast<uint64_t>(S), static_cast<uint64_t>(B)};
  const uint64_t strides[3] = {static_cast<uint64_t>(d) * 2, static_cast<uint64_t>(H) * d * 2,
                               static_cast<uint64_t>(S) * H * d * 2};
  const uint32_t box[4] = {64, 1, static_cast<uint32_t>(kTileM), 1};
  return encode_map(m, dt, 4, base, dims, strides, box);
}

bool map_bsd(CUtensorMap* m, CUtensorMapDataType dt, const void* base, int B, int S, int d) {
  const uint64_t dims[3] = {static_cast<uint64_t>(d), static_cast<uint64_t>(S),
                            static_cast<uint64_t>(B)};
  const uint64_t strides[2] = {static_cast<uint64_t>(d) * 2, static_cast<uint64_t>(S) * d * 2};
  const uint32_t box[3] = {64, static_cast<uint32_t>(kTileM), 1};
  return encode_map(m, dt, 3, base, dims, strides, box);
}

cudaError_t side_stream(cudaStream_t* out) {
  static std::mutex mu;
  static cudaStream_t streams[kMaxSideDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxSideDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!streams[dev]) {
    e = cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking);
    if (e != cudaSuccess) return e;
  }
  *out = streams[dev];
  return cudaSuccess;
}

void set_profile_events(cudaEvent_t begin, cudaEvent_t end) {
  std::lock_guard<std::mutex> lock(g_prof_mu);
  g_prof_begin = begin;
  g_prof_end = end;
}

cudaError_t timed_attention(const AttnArgs& a, int64_t n_list, cudaStream_t s) {
  cudaEvent_t b = nullptr, e = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_prof_mu);
    b = g_prof_begin;
    e = g_prof_end;
  }
  const bool prof = b && e;
  if (prof && cudaEventRecord(b, s) != cudaSuccess) return cudaErrorUnknown;
  cudaError_t r = launch_attention(a, n_list, s);
  if (r == cudaSuccess && prof) r = cudaEventRecord(e, s);
  return r;
}

}  // namespace gqe
