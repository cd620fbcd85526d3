// GQE router: per-group linear scores, softmax over the group's M experts,
// top-k with an exact decision, and the renormalised weights.
//
// Review "论文综述：分组查询专家" §二 路由器: p_{i,g} = softmax(r_g(x_i)),
// K_g(x_i) = TopK_m(p_{i,g,m}, k); §二 三个关键部件: w = p / sum_{K_g} p.
//
// Exactness.  Top-k is defined on the exact logits (ties -> lower index).
// route_kernel computes each logit with a sequential float32 FMA chain over
// d_model exact bf16*bf16 products, so |l_hat - l| <= (d_model+1) u sum|x_j w_j|
// (+ the bias rounding), with u = 2^-24; sum|x_j w_j| is bounded by
// ||x||_2 ||w||_2.  A decision is kept only if every selected logit beats every
// later one by more than the two bounds; otherwise the (token, group) pair is
// queued and route_fixup_kernel decides it with an exact fixed-point
// (Kulisch-style) accumulation of the products.
#include <cuda_bf16.h>

#include "gqe_device.cuh"

namespace gqe {
namespace {

constexpr int kRouteThreads = 128;  // one token per thread
constexpr int kRouteChunk = 64;     // d_model rows of W_r staged per step

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) {
  return __uint_as_float(b << 16);
}

template <int GM>
__global__ void __launch_bounds__(kRouteThreads) route_kernel(const RouteArgs a) {
  __shared__ __align__(16) float Ws[kRouteChunk][GM];
  __shared__ float wsq[GM];
  __shared__ float lg[kRouteThreads][GM + 1];

  const int tid = threadIdx.x;
  const int t = blockIdx.x * kRouteThreads + tid;
  const bool valid = t < a.T;
  const int dm = a.dm, M = a.M, G = a.G, k = a.k;

  if (tid < GM) wsq[tid] = 0.f;
  float acc[GM];
#pragma unroll
  for (int c = 0; c < GM; ++c) acc[c] = 0.f;
  float xsq = 0.f, wpart = 0.f;
  const uint16_t* xrow = a.x + static_cast<int64_t>(valid ? t : 0) * dm;

  for (int c0 = 0; c0 < dm; c0 += kRouteChunk) {
    const int rows = min(kRouteChunk, dm - c0);
    __syncthreads();
    // stage W_r[g, c0 + j, m] as Ws[j][g*M + m] (fp32); column of this thread
    // is tid % GM because GM divides the block size.
    for (int e = tid; e < kRouteChunk * GM; e += kRouteThreads) {
      const int j = e / GM, col = e % GM;
      float v = 0.f;
      if (j < rows) {
        const int g = col / M, m = col % M;
        v = bf16_bits_to_float(a.Wr[(static_cast<int64_t>(g) * dm + c0 + j) * M + m]);
      }
      Ws[j][col] = v;
      wpart = fmaf(v, v, wpart);
    }
    __syncthreads();
    if (valid) {
      for (int jj = 0; jj < rows; jj += 8) {
        const uint4 xv = __ldg(reinterpret_cast<const uint4*>(xrow + c0 + jj));
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float xf = bf16_bits_to_float((xw[e >> 1] >> ((e & 1) * 16)) & 0xFFFFu);
          xsq = fmaf(xf, xf, xsq);
          const float4* wr = reinterpret_cast<const float4*>(&Ws[jj + e][0]);
#pragma unroll
          for (int c4 = 0; c4 < GM / 4; ++c4) {
            const float4 w4 = wr[c4];
            acc[4 * c4 + 0] = fmaf(xf, w4.x, acc[4 * c4 + 0]);
            acc[4 * c4 + 1] = fmaf(xf, w4.y, acc[4 * c4 + 1]);
            acc[4 * c4 + 2] = fmaf(xf, w4.z, acc[4 * c4 + 2]);
            acc[4 * c4 + 3] = fmaf(xf, w4.w, acc[4 * c4 + 3]);
          }
        }
      }
    }
  }
  atomicAdd(&wsq[tid % GM], wpart);
#pragma unroll
  for (int c = 0; c < GM; ++c) lg[tid][c] = acc[c];
  __syncthreads();
  if (!valid) return;

  const float xn = sqrtf(xsq);
  // bound factor: (dm + 3) u, inflated by 1% for the rounding of the norms
  const float cerr = static_cast<float>(dm + 3) * 5.9604645e-8f * 1.01f;
  const int64_t tG = static_cast<int64_t>(t) * G;
  bool nonfinite = false;

  for (int g = 0; g < G; ++g) {
    float l[kMaxM], e[kMaxM];
    for (int m = 0; m < M; ++m) {
      const int col = g * M + m;
      const float b = a.bias ? a.bias[col] : 0.f;
      l[m] = lg[tid][col] + b;
      e[m] = cerr * fmaf(xn, sqrtf(wsq[col]), fabsf(b)) + 1e-36f;
      nonfinite |= !isfinite(l[m]);
    }
    // provisional top-k from the float32 logits (ties -> lower index)
    uint32_t taken = 0;
    int sel[kMaxM];
    for (int r = 0; r < k; ++r) {
      int best = -1;
      for (int m = 0; m < M; ++m) {
        if (taken & (1u << m)) continue;
        if (best < 0 || l[m] > l[best]) best = m;
      }
      sel[r] = best;
      taken |= 1u << best;
    }
    // certify: every rank r < min(k, M-1) beats every later candidate
    bool certain = true;
    uint32_t above = 0;
    for (int r = 0; r < k && r < M - 1 && certain; ++r) {
      const int am = sel[r];
      above |= 1u << am;
      for (int m = 0; m < M; ++m) {
        if (above & (1u << m)) continue;
        if (!(l[am] - l[m] > (e[am] + e[m]) * 1.001f)) {
          certain = false;
          break;
        }
      }
    }
    if (!certain) {
      const int slot = atomicAdd(a.fix_count, 1);
      a.fix_list[slot] = static_cast<int32_t>(tG + g);
    }
    // softmax over the group's M experts
    float mx = l[0];
    for (int m = 1; m < M; ++m) mx = fmaxf(mx, l[m]);
    float pe[kMaxM], s = 0.f;
    for (int m = 0; m < M; ++m) {
      pe[m] = expf(l[m] - mx);
      s += pe[m];
    }
    float* prow = a.p + (tG + g) * M;
    for (int m = 0; m < M; ++m) prow[m] = pe[m] / s;
    int32_t* irow = a.topk_idx + (tG + g) * k;
    float* wrow = a.w + (tG + g) * k;
    float den = 0.f;
    for (int j = 0; j < k; ++j) den += pe[sel[j]] / s;
    for (int j = 0; j < k; ++j) {
      irow[j] = sel[j];
      wrow[j] = (k == 1) ? 1.0f : (pe[sel[j]] / s) / den;
    }
  }
  if (nonfinite) latch_status(a.status, GQE_ERR_NONFINITE);
}

// ------------------------------------------------------------------------
// Exact logits.  A bf16 value is +-mant * 2^e with an 8-bit mantissa, so a
// product is a 16-bit integer times 2^(ex+ey), ex+ey in [-266, 240]; a fp32
// bias is a 24-bit integer times 2^e, e in [-149, 104].  Shifting every term
// by 2^266 turns the logit into an integer below 2^540, held as 18 signed
// 64-bit limbs of 32 bits each (limb L weighs 2^(32L)).  Adding a term never
// overflows a limb, and after a carry pass the representation is unique:
// limbs 0..16 in [0, 2^32), limb 17 signed.
constexpr int kLimbs = 18;
constexpr int kExpBias = 266;

struct Exact {
  long long v[kLimbs];
};

__device__ __forceinline__ void bf16_decompose(uint32_t b, int& sign, int& mant, int& ex) {
  sign = (b >> 15) & 1;
  const int E = (b >> 7) & 0xFF, F = b & 0x7F;
  if (E == 0) {
    mant = F;
    ex = -133;
  } else {
    mant = F | 0x80;
    ex = E - 134;
  }
}

__device__ __forceinline__ void limbs_add(long long* acc, long long mant, int pos) {
  const int L = pos >> 5, o = pos & 31;
  const long long v = mant * (1ll << o);  // |mant| < 2^25, o < 32: fits in 57 bits
  acc[L] += v & 0xFFFFFFFFll;
  acc[L + 1] += v >> 32;
}

__device__ void exact_logit(const RouteArgs& a, int t, int g, int m, Exact& out, bool& bad) {
  const int lane = threadIdx.x & 31;
  long long acc[kLimbs];
#pragma unroll
  for (int i = 0; i < kLimbs; ++i) acc[i] = 0;
  const uint16_t* xr = a.x + static_cast<int64_t>(t) * a.dm;
  for (int j = lane; j < a.dm; j += 32) {
    const uint32_t xb = xr[j];
    const uint32_t wb = a.Wr[(static_cast<int64_t>(g) * a.dm + j) * a.M + m];
    if (((xb >> 7) & 0xFF) == 0xFF || ((wb >> 7) & 0xFF) == 0xFF) {
      bad = true;
      continue;
    }
    int sx, mx, ex, sw, mw, ew;
    bf16_decompose(xb, sx, mx, ex);
    bf16_decompose(wb, sw, mw, ew);
    long long prod = static_cast<long long>(mx) * mw;
    if (sx ^ sw) prod = -prod;
    if (prod != 0) limbs_add(acc, prod, ex + ew + kExpBias);
  }
  if (lane == 0 && a.bias) {
    const uint32_t bb = __float_as_uint(a.bias[g * a.M + m]);
    const int E = (bb >> 23) & 0xFF;
    if (E == 0xFF) {
      bad = true;
    } else {
      long long mant = (E == 0) ? (bb & 0x7FFFFF) : ((bb & 0x7FFFFF) | 0x800000);
      const int e = (E == 0) ? -149 : E - 150;
      if (bb >> 31) mant = -mant;
      if (mant != 0) limbs_add(acc, mant, e + kExpBias);
    }
  }
#pragma unroll
  for (int i = 0; i < kLimbs; ++i) {
    long long v = acc[i];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
    acc[i] = v;
  }
  // carry pass: limbs 0..16 into [0, 2^32), the top limb keeps the sign
#pragma unroll
  for (int i = 0; i < kLimbs - 1; ++i) {
    const long long c = acc[i] >> 32;  // floor division by 2^32
    acc[i] -= c * 4294967296ll;
    acc[i + 1] += c;
  }
#pragma unroll
  for (int i = 0; i < kLimbs; ++i) out.v[i] = acc[i];
}

// -1, 0, +1 for a < b, a == b, a > b
__device__ __forceinline__ int exact_cmp(const Exact& a, const Exact& b) {
  if (a.v[kLimbs - 1] != b.v[kLimbs - 1]) return a.v[kLimbs - 1] < b.v[kLimbs - 1] ? -1 : 1;
  for (int i = kLimbs - 2; i >= 0; --i)
    if (a.v[i] != b.v[i]) return a.v[i] < b.v[i] ? -1 : 1;
  return 0;
}

constexpr int kFixWarps = 4;

__global__ void __launch_bounds__(32 * kFixWarps) route_fixup_kernel(const RouteArgs a) {
  __shared__ Exact ex[kFixWarps][kMaxM];
  __shared__ int sel[kFixWarps][kMaxM];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * kFixWarps;
  const int count = *reinterpret_cast<volatile int32_t*>(a.fix_count);
  const int M = a.M, k = a.k;
  for (int f = blockIdx.x * kFixWarps + warp; f < count; f += nwarps) {
    const int pair = a.fix_list[f];
    const int t = pair / a.G, g = pair % a.G;
    bool bad = false;
    for (int m = 0; m < M; ++m) {
      Exact e;
      exact_logit(a, t, g, m, e, bad);
      if (lane == 0) ex[warp][m] = e;
    }
    bad = __any_sync(0xFFFFFFFFu, bad);
    __syncwarp();
    if (lane < M) {
      int rank = 0;
      for (int b = 0; b < M; ++b) {
        if (b == lane) continue;
        const int c = exact_cmp(ex[warp][b], ex[warp][lane]);
        if (c > 0 || (c == 0 && b < lane)) ++rank;
      }
      if (rank < k) sel[warp][rank] = lane;
    }
    __syncwarp();
    if (lane == 0) {
      if (bad) latch_status(a.status, GQE_ERR_NONFINITE);
      const int64_t row = static_cast<int64_t>(t) * a.G + g;
      const float* prow = a.p + row * M;
      float den = 0.f;
      for (int j = 0; j < k; ++j) den += prow[sel[warp][j]];
      for (int j = 0; j < k; ++j) {
        a.topk_idx[row * k + j] = sel[warp][j];
        a.w[row * k + j] = (k == 1) ? 1.0f : prow[sel[warp][j]] / den;
      }
    }
    __syncwarp();
  }
}

}  // namespace

cudaError_t launch_route(const RouteArgs& a, cudaStream_t st) {
  const int GM = a.G * a.M;
  const dim3 grid((a.T + kRouteThreads - 1) / kRouteThreads);
  switch (GM) {
    case 4: route_kernel<4><<<grid, kRouteThreads, 0, st>>>(a); break;
    case 8: route_kernel<8><<<grid, kRouteThreads, 0, st>>>(a); break;
    case 16: route_kernel<16><<<grid, kRouteThreads, 0, st>>>(a); break;
    case 32: route_kernel<32><<<grid, kRouteThreads, 0, st>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  route_fixup_kernel<<<148, 32 * kFixWarps, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace gqe
