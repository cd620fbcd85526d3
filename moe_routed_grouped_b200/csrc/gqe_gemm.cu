// The projections around the attention path, on the sm_100a tensor cores.
//
// "论文综述：分组查询专家" §二 路由器: only the query heads the router selected
// are computed at all, so the query projection runs for the selected (token,
// head) pairs only; 三个关键部件: the layer output is
// y_i = Concat(O_i, o_bar_i, s(x_i)) W_O.  The other projections are plain
// linear maps: K_{i,g} = x_i W_K[g], V_{i,g} = x_i W_V[g], and the shared
// head's query x_i W_s.
//
// Two kernels share one pipeline (bf16 operands in shared memory, fp32
// accumulators in TMEM, 128 output rows per CTA):
//   gemm_dense_kernel<BN>   C[rows, n] = A[rows, :] . B[n / nc][:, n % nc]: A
//                           rows contiguous (TMA), B a stack of nb [K, nc]
//                           matrices seen as one [K, nb*nc] operand (TMA), so
//                           x . W_K for all G KV heads is one GEMM whose
//                           output is K in its [B, S, G, d] layout; W_O is
//                           the nb = 1 case.
//   gemm_routed_kernel<D>   one CTA per routed tile of the attention work
//                           list: it gathers the x rows of one (batch, group,
//                           expert) bucket and multiplies them by
//                           W_Q[g*M + m], writing Q[b, i, h] at the tokens'
//                           own rows (the shared head's Qs = x W_s is a
//                           dense projection).
// Warp roles (192 threads): warps 0-3 epilogue (thread r owns output row r,
// TMEM lane r; in the routed kernel they also gather the A rows with
// cp.async), warp 4 TMA producer, warp 5 TMEM owner and tcgen05.mma issuer.
#include <cuda_bf16.h>

#include "gqe_device.cuh"

namespace gqe {
namespace {

constexpr int kGemmThreads = 192;
constexpr int kKc = 64;                    // K columns per stage (128 B of bf16)
constexpr int kABytes = kTileM * kKc * 2;  // 16 KB: 128 rows x 64 bf16
constexpr int kBAtom = kKc * 128;          // 8 KB: 64 K rows x 64 columns

template <int BN>
struct GemmCfg {
  static constexpr int kBBytes = (BN / 64) * kBAtom;
  static constexpr int kStageBytes = kABytes + kBBytes;
  // d = 64 tiles keep two CTAs per SM (4 stages, 96 KB); wider tiles one
  static constexpr int kStages = BN == 128 ? 6 : 4;
  static constexpr int kMinBlocks = BN == 64 ? 2 : 1;
  static constexpr int kSmemBar = kStages * kStageBytes;
  static constexpr int kSmemBytes = kSmemBar + 256 + 1024;
  static constexpr uint32_t kTmemCols = BN;
  // kind::f16 with bf16 A (K-major) and bf16 B (MN-major), fp32 accumulate
  static constexpr uint32_t kIdesc = make_idesc_f16(kTileM, BN, /*bf16*/ 1, 0, /*MN*/ 1);
};

// barrier slots (stage s: full = kGbFull + s, empty = kGbEmpty + s, ...)
enum : int { kGbFull = 0, kGbEmpty = 8, kGbAFull = 16, kGbDFull = 24, kGbSpare = 25, kGbNum = 26 };

struct GWaiter {
  volatile int* abort;
  int* status;
  uint64_t limit;
  __device__ bool operator()(uint64_t* bar, uint32_t parity) const {
    return mbar_wait(bar, parity, abort, status, limit);
  }
};

// The UMMAs of one K stage: 4 steps of K = 16.
template <int BN>
__device__ __forceinline__ void mma_stage(uint32_t tD, uint32_t aaddr, uint32_t baddr,
                                          bool first) {
#pragma unroll
  for (int kk = 0; kk < kKc / 16; ++kk)
    umma_ss(tD, make_sdesc_sw128(aaddr + kk * 32, 16, 1024),
            make_sdesc_sw128(baddr + kk * 2048, kBAtom, 1024), GemmCfg<BN>::kIdesc,
            (!first || kk > 0) ? 1u : 0u);
}

// Epilogue of one warp: its 32 rows x BN columns of the accumulator, in
// chunks of 64 columns staged in shared memory (32 rows x 68 floats) and then
// written row by row with consecutive lanes on consecutive 16-byte pieces.
// dst(row) is this lane's output row start (null: row not stored); element
// type float32 or bf16.
template <int BN>
__device__ __forceinline__ void store_tile_rows(float* stage, uint32_t taddr, uint8_t* dst,
                                                bool fp32) {
  constexpr int kStr = 68;
  const int lane = threadIdx.x & 31;
  const unsigned long long d1 = reinterpret_cast<unsigned long long>(dst);
#pragma unroll 1
  for (int c0 = 0; c0 < BN; c0 += 64) {
    __syncwarp();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t v[32];
      tmem_ld32(taddr + c0 + 32 * h, v);
      tmem_ld_wait(v);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        reinterpret_cast<float4*>(stage + lane * kStr + 32 * h)[q] =
            make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                        __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
    }
    __syncwarp();
    if (fp32) {  // 16 lanes per row (256 B), 2 rows per instruction
      const int sub = lane >> 4, piece = lane & 15;
#pragma unroll 4
      for (int r0 = 0; r0 < 32; r0 += 2) {
        const int row = r0 + sub;
        float* o = reinterpret_cast<float*>(__shfl_sync(0xFFFFFFFFu, d1, row));
        const float4 v = reinterpret_cast<const float4*>(stage + row * kStr)[piece];
        if (o) reinterpret_cast<float4*>(o + c0)[piece] = v;
      }
    } else {  // 8 lanes per row (128 B), 4 rows per instruction
      const int sub = lane >> 3, piece = lane & 7;
#pragma unroll 4
      for (int r0 = 0; r0 < 32; r0 += 4) {
        const int row = r0 + sub;
        uint16_t* o = reinterpret_cast<uint16_t*>(__shfl_sync(0xFFFFFFFFu, d1, row));
        const float4* src = reinterpret_cast<const float4*>(stage + row * kStr + 8 * piece);
        const float4 x0 = src[0], x1 = src[1];
        __nv_bfloat162 h0 = __floats2bfloat162_rn(x0.x, x0.y), h1 = __floats2bfloat162_rn(x0.z, x0.w),
                       h2 = __floats2bfloat162_rn(x1.x, x1.y), h3 = __floats2bfloat162_rn(x1.z, x1.w);
        const uint4 w = make_uint4(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1),
                                   *reinterpret_cast<uint32_t*>(&h2), *reinterpret_cast<uint32_t*>(&h3));
        if (o) reinterpret_cast<uint4*>(o + c0)[piece] = w;
      }
    }
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------
template <int BN>
__global__ void __launch_bounds__(kGemmThreads, GemmCfg<BN>::kMinBlocks)
    gemm_dense_kernel(const __grid_constant__ GemmArgs a) {
  grid_dep_wait();  // launched with launch_pdl
  using C = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kTileM;
  const int n0 = blockIdx.y * BN;
  const int nk = a.K / kKc;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kSmemBar);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + kGbNum);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + kGbNum + 1);
  const GWaiter wait{abort_flag, a.status, a.wait_limit_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&bars[kGbFull + s], 1);
      mbar_init(&bars[kGbEmpty + s], 1);
    }
    mbar_init(&bars[kGbDFull], 1);
    mbar_init(&bars[kGbSpare], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&a.tmA);
    tma_prefetch_desc(&a.tmB);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tD = *tmem_holder;

  if (warp == 4) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int kc = 0; kc < nk; ++kc) {
        const int s = kc % C::kStages;
        const uint32_t round = static_cast<uint32_t>(kc / C::kStages);
        if (round > 0 && !wait(&bars[kGbEmpty + s], (round - 1) & 1)) break;
        uint8_t* sa = smem + s * C::kStageBytes;
        mbar_arrive_expect_tx(&bars[kGbFull + s], C::kStageBytes);
        tma_load_2d(sa, &a.tmA, &bars[kGbFull + s], kc * kKc, m0);
#pragma unroll
        for (int at = 0; at < BN / 64; ++at) {
          const int n = n0 + 64 * at;
          tma_load_3d(sa + kABytes + at * kBAtom, &a.tmB, &bars[kGbFull + s], n % a.nc,
                      kc * kKc, n / a.nc);
        }
        issued = kc + 1;
      }
      if (*abort_flag)  // let the copies in flight land before the CTA exits
        for (int q = max(0, issued - C::kStages); q < issued; ++q)
          mbar_wait(&bars[kGbFull + q % C::kStages], (q / C::kStages) & 1, nullptr, a.status,
                    a.wait_limit_ns);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      for (int kc = 0; kc < nk; ++kc) {
        const int s = kc % C::kStages;
        if (!wait(&bars[kGbFull + s], (kc / C::kStages) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t aaddr = smem_u32(smem + s * C::kStageBytes);
        mma_stage<BN>(tD, aaddr, aaddr + kABytes, kc == 0);
        tc_commit(&bars[kGbEmpty + s]);
      }
      if (ok) {
        tc_commit(&bars[kGbDFull]);
      } else {  // drain whatever was issued before giving up
        tc_commit(&bars[kGbSpare]);
        mbar_wait(&bars[kGbSpare], 0, nullptr, a.status, a.wait_limit_ns);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------ epilogue
    const int r = warp * 32 + lane;
    const bool ok = __all_sync(0xFFFFFFFFu, wait(&bars[kGbDFull], 0));
    if (ok) {
      tc_fence_after();
      const size_t esz = a.c_fp32 ? 4 : 2;
      uint8_t* dst = (m0 + r < a.rows)
                         ? static_cast<uint8_t*>(a.C) +
                               (static_cast<int64_t>(m0 + r) * a.ldc + n0) * esz
                         : nullptr;
      // all K stages are consumed once the accumulator is final: stage rows there
      float* stage = reinterpret_cast<float*>(smem) + warp * 32 * 68;
      store_tile_rows<BN>(stage, tD + (static_cast<uint32_t>(warp * 32) << 16), dst,
                          a.c_fp32 != 0);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tD, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Routed query projection: one CTA per work-list tile (the list the
// attention kernel runs on).  BN = d.
template <int D>
__global__ void __launch_bounds__(kGemmThreads, GemmCfg<D>::kMinBlocks)
    gemm_routed_kernel(const __grid_constant__ GemmArgs a) {
  grid_dep_wait();  // launched with launch_pdl
  using C = GemmCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (static_cast<int>(blockIdx.x) >= *a.tile_count) return;
  const TileDesc td = a.tiles[blockIdx.x];
  if (td.nkv == 0) return;  // empty slot of the list (CTA-uniform)
  const int kind = td.code >> 24, id = td.code & 0xFFFFFF;
  if (kind != kRouted) return;  // shared-head tiles: Qs is a dense projection
  const int b = id / (a.G * a.M);
  const int h = ((id / a.M) % a.G) * a.M + id % a.M;
  const int bstart = a.bucket_off[id];
  const int nk = a.K / kKc;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kSmemBar);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + kGbNum);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + kGbNum + 1);
  const GWaiter wait{abort_flag, a.status, a.wait_limit_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&bars[kGbFull + s], 1);   // B (TMA)
      mbar_init(&bars[kGbAFull + s], 4);  // A (one arrival per gathering warp)
      mbar_init(&bars[kGbEmpty + s], 1);
    }
    mbar_init(&bars[kGbDFull], 1);
    mbar_init(&bars[kGbSpare], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) tma_prefetch_desc(&a.tmB);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tD = *tmem_holder;

  if (warp == 4) {
    // ------------------------------------------------------ W producer (TMA)
    if (lane == 0) {
      int issued = 0;
      for (int kc = 0; kc < nk; ++kc) {
        const int s = kc % C::kStages;
        const uint32_t round = static_cast<uint32_t>(kc / C::kStages);
        if (round > 0 && !wait(&bars[kGbEmpty + s], (round - 1) & 1)) break;
        uint8_t* sb = smem + s * C::kStageBytes + kABytes;
        mbar_arrive_expect_tx(&bars[kGbFull + s], C::kBBytes);
#pragma unroll
        for (int at = 0; at < D / 64; ++at)
          tma_load_3d(sb + at * kBAtom, &a.tmB, &bars[kGbFull + s], 64 * at, kc * kKc, h);
        issued = kc + 1;
      }
      if (*abort_flag)
        for (int q = max(0, issued - C::kStages); q < issued; ++q)
          mbar_wait(&bars[kGbFull + q % C::kStages], (q / C::kStages) & 1, nullptr, a.status,
                    a.wait_limit_ns);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      for (int kc = 0; kc < nk; ++kc) {
        const int s = kc % C::kStages;
        const uint32_t par = (kc / C::kStages) & 1;
        if (!wait(&bars[kGbAFull + s], par) || !wait(&bars[kGbFull + s], par)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t aaddr = smem_u32(smem + s * C::kStageBytes);
        mma_stage<D>(tD, aaddr, aaddr + kABytes, kc == 0);
        tc_commit(&bars[kGbEmpty + s]);
      }
      if (ok) {
        tc_commit(&bars[kGbDFull]);
      } else {
        tc_commit(&bars[kGbSpare]);
        mbar_wait(&bars[kGbSpare], 0, nullptr, a.status, a.wait_limit_ns);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------ gather + epilogue
    const int r = warp * 32 + lane;
    const bool valid = r < td.nrows;
    const int rv = valid ? r : td.nrows - 1;
    const int pos = a.bucket_tok[bstart + td.row0 + rv];
    const uint16_t* xrow = a.A + (static_cast<int64_t>(b) * a.S + pos) * a.lda;
    // stage kc's copies are issued, then stage kc - kLook (landed) is published
    constexpr int kLook = 2;
    auto publish = [&](int kp) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kGbAFull + kp % C::kStages]);
    };
    bool ok = true;
    int kc = 0;
    for (; kc < nk; ++kc) {
      const int s = kc % C::kStages;
      const uint32_t round = static_cast<uint32_t>(kc / C::kStages);
      if (round > 0 && !__all_sync(0xFFFFFFFFu, wait(&bars[kGbEmpty + s], (round - 1) & 1))) {
        ok = false;
        break;
      }
      uint8_t* sa = smem + s * C::kStageBytes;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch)
        cp_async_16(sa + r * 128 + ((ch ^ (r & 7)) << 4), xrow + kc * kKc + ch * 8,
                    valid ? 16u : 0u);
      asm volatile("cp.async.commit_group;" ::: "memory");
      if (kc >= kLook) {
        asm volatile("cp.async.wait_group %0;" ::"n"(kLook) : "memory");
        publish(kc - kLook);
      }
    }
    cp_async_wait_all();
    if (ok)
      for (int kp = nk > kLook ? nk - kLook : 0; kp < nk; ++kp) publish(kp);
    ok = __all_sync(0xFFFFFFFFu, ok && wait(&bars[kGbDFull], 0));
    if (ok) {
      tc_fence_after();
      uint8_t* dst = valid ? reinterpret_cast<uint8_t*>(
                                 static_cast<uint16_t*>(a.C) +
                                 ((static_cast<int64_t>(b) * a.S + pos) * a.N + h) * D)
                           : nullptr;
      float* stage = reinterpret_cast<float*>(smem) + warp * 32 * 68;
      store_tile_rows<D>(stage, tD + (static_cast<uint32_t>(warp * 32) << 16), dst, false);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tD, C::kTmemCols);
  }
}

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

}  // namespace

cudaError_t launch_gemm_dense(const GemmArgs& a, int bn, cudaStream_t st) {
  const unsigned gm = static_cast<unsigned>((a.rows + kTileM - 1) / kTileM);
  cudaError_t e;
  switch (bn) {
    case 64:
      if ((e = set_smem(gemm_dense_kernel<64>, GemmCfg<64>::kSmemBytes)) != cudaSuccess) return e;
      return launch_pdl(gemm_dense_kernel<64>, dim3(gm, a.n_total / 64), dim3(kGemmThreads),
                        GemmCfg<64>::kSmemBytes, st, a);
    case 128:
      if ((e = set_smem(gemm_dense_kernel<128>, GemmCfg<128>::kSmemBytes)) != cudaSuccess) return e;
      return launch_pdl(gemm_dense_kernel<128>, dim3(gm, a.n_total / 128), dim3(kGemmThreads),
                        GemmCfg<128>::kSmemBytes, st, a);
    case 256:
      if ((e = set_smem(gemm_dense_kernel<256>, GemmCfg<256>::kSmemBytes)) != cudaSuccess) return e;
      return launch_pdl(gemm_dense_kernel<256>, dim3(gm, a.n_total / 256), dim3(kGemmThreads),
                        GemmCfg<256>::kSmemBytes, st, a);
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_gemm_routed(const GemmArgs& a, int64_t n_list, cudaStream_t st) {
  if (n_list <= 0) return cudaSuccess;
  cudaError_t e;
  if (a.d == 64) {
    if ((e = set_smem(gemm_routed_kernel<64>, GemmCfg<64>::kSmemBytes)) != cudaSuccess) return e;
    return launch_pdl(gemm_routed_kernel<64>, dim3(static_cast<unsigned>(n_list)), dim3(kGemmThreads),
                      GemmCfg<64>::kSmemBytes, st, a);
  } else if (a.d == 128) {
    if ((e = set_smem(gemm_routed_kernel<128>, GemmCfg<128>::kSmemBytes)) != cudaSuccess) return e;
    return launch_pdl(gemm_routed_kernel<128>, dim3(static_cast<unsigned>(n_list)), dim3(kGemmThreads),
                      GemmCfg<128>::kSmemBytes, st, a);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace gqe
