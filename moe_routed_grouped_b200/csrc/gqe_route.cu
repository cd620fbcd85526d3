// GQE router: per-group linear scores, softmax over the group's M experts,
// top-k with an exact decision, and the renormalised weights.
//
// Review "论文综述：分组查询专家" §二 路由器: p_{i,g} = softmax(r_g(x_i)),
// K_g(x_i) = TopK_m(p_{i,g,m}, k); §二 三个关键部件: w = p / sum_{K_g} p.
//
// Exactness.  Top-k is defined on the exact logits (ties -> lower index).
// route_kernel sums the exact bf16*bf16 products in float32 with a longest
// rounding chain of D = 32 + n_chunks + 3 operations, so
// |l_hat - l| <= D u sum|x_j w_j| (u = 2^-24), and sum|x_j w_j| <= ||x|| ||w||.
// A decision is kept only if every selected logit beats every later one by
// more than the two bounds; otherwise the same CTA recomputes that (token,
// group) pair with an exact fixed-point (Kulisch-style) accumulation of the
// products.
#include <atomic>

#include <cuda_bf16.h>

#include "gqe_device.cuh"

namespace gqe {
namespace {

constexpr int kRouteWarps = 4;
constexpr int kRouteThreads = 32 * kRouteWarps;
constexpr int kRouteChunk = 32;     // d_model rows per chunk; warp w owns chunks w, w+4, ...
constexpr int kRouteMaxWarps = 4;   // warps that take exact ranks (sizes their shared arrays)

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) {
  return __uint_as_float(b << 16);
}

__device__ void exact_rank_pair(const RouteArgs& a, int t, int g, int* sel_smem);

// W_r [G][dm][M] (bf16) -> wt [dm][G*M] (float32) and partial column sums of
// squares wsq[b][G*M] over rows 32b .. 32b+31 (block b; thread (j, col)),
// added by route_kernel in block order.
template <int GM>
__global__ void __launch_bounds__(32 * GM) route_prep_kernel(const RouteArgs a) {
  grid_dep_wait();  // launched with launch_pdl
  const int col = threadIdx.x % GM, jj = threadIdx.x / GM;
  const int j = blockIdx.x * 32 + jj;
  const int g = col / a.M, m = col % a.M;
  float v = 0.f;
  if (j < a.dm) {
    v = bf16_bits_to_float(a.Wr[(static_cast<int64_t>(g) * a.dm + j) * a.M + m]);
    a.wt[static_cast<int64_t>(j) * GM + col] = v;
  }
  __shared__ float part[32][GM + 1];
  part[jj][col] = v * v;
  __syncthreads();
  if (threadIdx.x < GM) {
    float s2 = 0.f;
    for (int r = 0; r < 32; ++r) s2 += part[r][threadIdx.x];
    a.wsq[blockIdx.x * GM + threadIdx.x] = s2;
  }
}

// Tokens per lane: 2 while the accumulators fit in registers, else 1.
template <int GM>
struct RouteShape {
  static constexpr int kTPL = GM <= 16 ? 2 : 1;
  static constexpr int kTok = 32 * kTPL;   // most tokens per tile (RouteArgs::tok)
};

template <int GM>
struct RouteSmem {
  using Sh = RouteShape<GM>;
  float ws[kRouteWarps][kRouteChunk][GM];           // this warp's W_r chunk, [j][col]
  float red[kRouteWarps][Sh::kTok][GM + 1];         // per-warp partial logits
  float lgt[Sh::kTok][GM + 1];                      // logits (+ bias)
  float err[Sh::kTok][GM + 1];                      // their rounding-error bounds
  float xsq[kRouteWarps][Sh::kTok];
  int nflag;
  int flags[Sh::kTok * 32];
  float wnorm[GM];                                  // ||W_r[:, col]||
  float bias[GM];
  int sel[kRouteWarps][kMaxM];
};

// x values of one chunk for one token: 32 bf16 in 4 x 16 bytes
__device__ __forceinline__ void load_x_chunk(const uint16_t* xrow, bool ok, int c0, int rows,
                                             uint4 (&v)[4]) {
#pragma unroll
  for (int q = 0; q < 4; ++q)
    v[q] = (ok && 8 * q < rows) ? __ldg(reinterpret_cast<const uint4*>(xrow + c0 + 8 * q))
                                : make_uint4(0u, 0u, 0u, 0u);
}

__device__ __forceinline__ float xval(const uint4 (&v)[4], int j) {
  const uint4 q = v[j >> 3];
  const uint32_t w = ((j & 7) >> 1) == 0 ? q.x : ((j & 7) >> 1) == 1 ? q.y : ((j & 7) >> 1) == 2 ? q.z : q.w;
  return bf16_bits_to_float((w >> ((j & 1) * 16)) & 0xFFFFu);
}

// Chunk rows [c0, c0 + 32) of the transposed W_r: 32 * GM contiguous floats,
// GM / 4 16-byte pieces per lane (rows past d_model read as zero).
template <int GM>
__device__ __forceinline__ void load_wt_chunk(const float* wt, int c0, int rows,
                                              float4 (&v)[GM / 4]) {
  const int lane = threadIdx.x & 31;
  const float4* src = reinterpret_cast<const float4*>(wt + static_cast<int64_t>(c0) * GM);
#pragma unroll
  for (int i = 0; i < GM / 4; ++i) {
    const int piece = lane + 32 * i;  // rows of 4*... : piece / (GM/4) is the row
    v[i] = (piece / (GM / 4) < rows) ? __ldg(src + piece) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// Softmax, provisional top-k and certification of one (token, group) pair
// with at most MM experts, every per-expert value in registers (loops over
// MM with compile-time indices).  p = e^(l - max) / s is formed as
// e^(l - max) * (1/s); w renormalises the selected p.  Returns whether every
// rank beats every later candidate by more than the two error bounds.
template <int MM>
__device__ __noinline__ bool decide_pair_small(const float* l, const float* e, int M, int k,
                                                  float* prow, int32_t* irow, float* wrow) {
  float lv[MM], ev[MM], xv[MM];
#pragma unroll
  for (int m = 0; m < MM; ++m) {
    lv[m] = m < M ? l[m] : -INFINITY;
    ev[m] = m < M ? e[m] : 0.f;
  }
  float mx = lv[0];
#pragma unroll
  for (int m = 1; m < MM; ++m)
    if (m < M) mx = fmaxf(mx, lv[m]);
  float s = 0.f;
#pragma unroll
  for (int m = 0; m < MM; ++m)
    if (m < M) {
      xv[m] = expf(lv[m] - mx);
      s += xv[m];
    }
  const float inv = 1.0f / s;
#pragma unroll
  for (int m = 0; m < MM; ++m)
    if (m < M) {
      xv[m] *= inv;
      prow[m] = xv[m];
    }
  uint32_t taken = 0;
  bool certain = true;
  float den = 0.f, pr[MM];
#pragma unroll
  for (int r = 0; r < MM; ++r) {
    if (r >= k) break;
    int best = -1;
    float bl = 0.f, be = 0.f, bp = 0.f;
#pragma unroll
    for (int m = 0; m < MM; ++m)
      if (m < M && !(taken & (1u << m)) && (best < 0 || lv[m] > bl)) {
        best = m;
        bl = lv[m];
        be = ev[m];
        bp = xv[m];
      }
    taken |= 1u << best;
    irow[r] = best;
    pr[r] = bp;
    den += bp;
    // rank r must beat every later candidate by more than both bounds
#pragma unroll
    for (int m = 0; m < MM; ++m)
      if (m < M && !(taken & (1u << m)) && !(bl - lv[m] > (be + ev[m]) * 1.001f)) certain = false;
  }
#pragma unroll
  for (int r = 0; r < MM; ++r)
    if (r < k) wrow[r] = (k == 1) ? 1.0f : pr[r] / den;
  return certain;
}

// The same for any M <= kMaxM, reading the values from shared memory.
__device__ __noinline__ bool decide_pair_any(const float* l, const float* e, int M, int k,
                                                float* prow, int32_t* irow, float* wrow) {
  float mx = l[0];
  for (int m = 1; m < M; ++m) mx = fmaxf(mx, l[m]);
  float s = 0.f;
  for (int m = 0; m < M; ++m) s += expf(l[m] - mx);
  const float inv = 1.0f / s;
  for (int m = 0; m < M; ++m) prow[m] = expf(l[m] - mx) * inv;
  uint32_t taken = 0;
  bool certain = true;
  float den = 0.f;
  for (int r = 0; r < k; ++r) {
    int best = -1;
    for (int m = 0; m < M; ++m) {
      if (taken & (1u << m)) continue;
      if (best < 0 || l[m] > l[best]) best = m;
    }
    taken |= 1u << best;
    irow[r] = best;
    den += expf(l[best] - mx) * inv;
    if (r < M - 1)
      for (int m = 0; m < M; ++m)
        if (!(taken & (1u << m)) && !(l[best] - l[m] > (e[best] + e[m]) * 1.001f))
          certain = false;
  }
  for (int r = 0; r < k; ++r)
    wrow[r] = (k == 1) ? 1.0f : (expf(l[irow[r]] - mx) * inv) / den;
  return certain;
}

// The steps after the logits, for one tile of ntok tokens starting at t0:
// per (token, group) the softmax, the provisional top-k and its certification
// against the bounds err, then the exact ranks of the undecided pairs (one
// warp per pair).  lgt and err have row stride GM + 1; every thread of the
// CTA calls this.
template <int GM>
__device__ __forceinline__ void route_tile_epilogue(const RouteArgs& a, const float* lgt,
                                                    const float* err, int t0, int ntok,
                                                    int* nflag, int* flags, int (*sel)[kMaxM]) {
  const int tid = threadIdx.x, warp = tid >> 5, nthreads = blockDim.x;
  const int M = a.M, G = a.G, k = a.k;
  for (int q = tid; q < ntok * G; q += nthreads) {
    const int ql = q / G, g = q % G;
    const float* l = lgt + ql * (GM + 1) + g * M;
    const float* e = err + ql * (GM + 1) + g * M;
    const int64_t row = static_cast<int64_t>(t0 + ql) * G + g;
    float* prow = a.p + row * M;
    int32_t* irow = a.topk_idx + row * k;
    float* wrow = a.w + row * k;
    const bool certain = M <= 8 ? decide_pair_small<(GM < 8 ? GM : 8)>(l, e, M, k, prow, irow, wrow)
                                : decide_pair_any(l, e, M, k, prow, irow, wrow);
    if (!certain) flags[atomicAdd(nflag, 1)] = q;
  }
  __syncthreads();
  const int nf = *nflag;
  if (nf > 0) {  // undecided pairs: exact ranks, one warp per pair (at most kRouteMaxWarps)
    if (tid == 0) atomicAdd(a.fix_count, nf);
    const int nw = min(nthreads / 32, kRouteMaxWarps);
    for (int f = warp; warp < nw && f < nf; f += nw) {
      const int q = flags[f];
      exact_rank_pair(a, t0 + q / G, q % G, sel[warp]);
    }
  }
}

// Persistent CTAs of 4 warps; a tile is a.tok <= kTok tokens (sized so the
// tiles fill the SMs evenly; lane l takes tokens l and l + 32).  Warp w sums the
// products of the d_model chunks w, w+4, ... ; lane l keeps its tokens' x
// values in registers and reads each W_r row as a broadcast from the warp's
// shared-memory copy of the chunk (copied from the float32 transpose made by
// route_prep_kernel).  Each
// chunk's 32 products are summed in fresh accumulators, chunk sums are added
// per warp and the four warp sums are added in warp order, so the longest
// rounding chain is 32 + ceil(n_chunks/4) + 4 (with the bias): that is the D
// of the bound |l_hat - l| <= D u ||x|| ||w_c||, u = 2^-24.
template <int GM>
__global__ void __launch_bounds__(kRouteThreads, 3) route_kernel(const RouteArgs a) {
  grid_dep_wait();  // launched with launch_pdl
  using Sh = RouteShape<GM>;
  constexpr int TPL = Sh::kTPL;
  const int TOK = a.tok;
  extern __shared__ __align__(16) uint8_t route_smem_raw[];
  RouteSmem<GM>& sm = *reinterpret_cast<RouteSmem<GM>*>(route_smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int dm = a.dm;
  const int nchunks = (dm + kRouteChunk - 1) / kRouteChunk;
  const int ntiles = (a.T + TOK - 1) / TOK;
  const float cerr =
      static_cast<float>(32 + (nchunks + kRouteWarps - 1) / kRouteWarps + 4) * 5.9604645e-8f *
      1.01f;

  for (int c = tid; c < GM; c += kRouteThreads) {
    float s2 = 0.f;
    for (int b = 0; b < (dm + 31) / 32; ++b) s2 += a.wsq[b * GM + c];
    sm.wnorm[c] = sqrtf(s2);
    sm.bias[c] = a.bias ? a.bias[c] : 0.f;
  }
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const int t0 = tile * TOK;
    const int ntok = min(TOK, a.T - t0);
    if (tid == 0) sm.nflag = 0;
    const uint16_t* xrow[TPL];
    bool xok[TPL];
#pragma unroll
    for (int r = 0; r < TPL; ++r) {
      const int tl = lane + 32 * r;
      xok[r] = tl < ntok;
      xrow[r] = a.x + static_cast<int64_t>(t0 + (xok[r] ? tl : 0)) * dm;
    }
    float acc[TPL][GM];
    float xsq[TPL];
#pragma unroll
    for (int r = 0; r < TPL; ++r) {
      xsq[r] = 0.f;
#pragma unroll
      for (int c = 0; c < GM; ++c) acc[r][c] = 0.f;
    }
    uint4 xv[TPL][4];
    float4 wv[GM / 4];
    int ci = warp;
    if (ci < nchunks) {
      const int rows = min(kRouteChunk, dm - ci * kRouteChunk);
#pragma unroll
      for (int r = 0; r < TPL; ++r) load_x_chunk(xrow[r], xok[r], ci * kRouteChunk, rows, xv[r]);
      load_wt_chunk<GM>(a.wt, ci * kRouteChunk, rows, wv);
    }
    for (; ci < nchunks; ci += kRouteWarps) {
      const int c0 = ci * kRouteChunk;
      const int rows = min(kRouteChunk, dm - c0);
      __syncwarp();
#pragma unroll
      for (int i = 0; i < GM / 4; ++i)
        reinterpret_cast<float4*>(&sm.ws[warp][0][0])[lane + 32 * i] = wv[i];
      __syncwarp();
      uint4 xc[TPL][4];
#pragma unroll
      for (int r = 0; r < TPL; ++r)
#pragma unroll
        for (int q = 0; q < 4; ++q) xc[r][q] = xv[r][q];
      const int cn = ci + kRouteWarps;  // prefetch this warp's next chunk
      if (cn < nchunks) {
        const int rows_n = min(kRouteChunk, dm - cn * kRouteChunk);
#pragma unroll
        for (int r = 0; r < TPL; ++r)
          load_x_chunk(xrow[r], xok[r], cn * kRouteChunk, rows_n, xv[r]);
        load_wt_chunk<GM>(a.wt, cn * kRouteChunk, rows_n, wv);
      }
      float cacc[TPL][GM];
#pragma unroll
      for (int r = 0; r < TPL; ++r)
#pragma unroll
        for (int c = 0; c < GM; ++c) cacc[r][c] = 0.f;
#pragma unroll
      for (int j = 0; j < kRouteChunk; ++j) {
        float xr[TPL];
#pragma unroll
        for (int r = 0; r < TPL; ++r) {
          xr[r] = xval(xc[r], j);
          xsq[r] = fmaf(xr[r], xr[r], xsq[r]);
        }
        const float4* wrow = reinterpret_cast<const float4*>(&sm.ws[warp][j][0]);
#pragma unroll
        for (int c4 = 0; c4 < GM / 4; ++c4) {
          const float4 w4 = wrow[c4];
#pragma unroll
          for (int r = 0; r < TPL; ++r) {
            cacc[r][4 * c4 + 0] = fmaf(xr[r], w4.x, cacc[r][4 * c4 + 0]);
            cacc[r][4 * c4 + 1] = fmaf(xr[r], w4.y, cacc[r][4 * c4 + 1]);
            cacc[r][4 * c4 + 2] = fmaf(xr[r], w4.z, cacc[r][4 * c4 + 2]);
            cacc[r][4 * c4 + 3] = fmaf(xr[r], w4.w, cacc[r][4 * c4 + 3]);
          }
        }
      }
      (void)rows;
#pragma unroll
      for (int r = 0; r < TPL; ++r)
#pragma unroll
        for (int c = 0; c < GM; ++c) acc[r][c] += cacc[r][c];
    }
#pragma unroll
    for (int r = 0; r < TPL; ++r) {
      sm.xsq[warp][lane + 32 * r] = xsq[r];
#pragma unroll
      for (int c = 0; c < GM; ++c) sm.red[warp][lane + 32 * r][c] = acc[r][c];
    }
    __syncthreads();

    // logits and their bounds, one (token, column) per thread
    bool nonfinite = false;
    for (int q = tid; q < ntok * GM; q += kRouteThreads) {
      const int ql = q / GM, col = q % GM;
      const float b = sm.bias[col];
      const float l = (((sm.red[0][ql][col] + sm.red[1][ql][col]) + sm.red[2][ql][col]) +
                       sm.red[3][ql][col]) + b;
      const float xn = sqrtf(((sm.xsq[0][ql] + sm.xsq[1][ql]) + sm.xsq[2][ql]) + sm.xsq[3][ql]);
      sm.lgt[ql][col] = l;
      sm.err[ql][col] = cerr * fmaf(xn, sm.wnorm[col], fabsf(b)) + 1e-36f;
      nonfinite |= !isfinite(l);
    }
    if (nonfinite) latch_status(a.status, GQE_ERR_NONFINITE);
    __syncthreads();

    route_tile_epilogue<GM>(a, &sm.lgt[0][0], &sm.err[0][0], t0, ntok, &sm.nflag, sm.flags,
                            sm.sel);
    __syncthreads();
  }
}

// ------------------------------------------------------------------------
// Router with W_r resident in shared memory (d_model * G * M float32 within
// kWresMaxW): one persistent CTA of 16 warps per SM over tiles of 64
// consecutive tokens.  Lane l of warp (cg, ks) takes tokens l and l + 32 of
// the tile, the CPW columns of column group cg and rows [ks*dm/KS,
// (ks+1)*dm/KS) of d_model (a K slice): every W_r load of a warp is one
// broadcast address, and each loaded W_r value serves two tokens (a 16-byte
// shared-memory load per 32 lanes returns 512 bytes, so the loads, not the
// FMAs, would bound a one-token lane).
//
// x streams per warp: each warp copies its own slice of the coming tiles into
// a ring of kWresRing groups of 8 values x 64 tokens with cp.async, waiting
// only for its own copies, so the copies run ahead across tile boundaries.
//
// Each step takes a pair of rows (2p, 2p+1): one f32x2 FMA per column and
// token adds x[2p] w[2p][c] to the even half and x[2p+1] w[2p+1][c] to the
// odd half of the accumulator, with W_r stored as (w[2p][c], w[2p+1][c])
// pairs (one 16-byte load gives two columns; laid out by route_pairs_kernel).
// The halves are added, the K slices are added in slice order, then the
// bias: the longest rounding chain is D = dm/(2 KS) + 1 + (KS - 1) + 1, the
// D of the bound |l_hat - l| <= D u ||x|| ||w_c|| used to certify each
// decision, as in route_kernel; the steps after the logits are
// route_tile_epilogue's.
// Tests set this to take the resident kernel at any token count (a host
// setting read at each call; atomic, as calls may come from several threads).
std::atomic<int> g_route_force_resident{0};

constexpr int kWresWarps = 16;
constexpr int kWresThreads = 32 * kWresWarps;
constexpr int kWresTok = 64;                   // tokens per tile (two per lane)
constexpr int kWresRing = 4;                   // x groups in flight per warp
constexpr int kWresMaxW = 64 << 10;            // most bytes of float32 W_r
constexpr int kWresMaxSmem = 215 << 10;        // most dynamic shared memory

template <int GM>
struct WresShape {
  static constexpr int CPW = GM < 16 ? GM : 16;  // columns per warp
  static constexpr int CGW = GM / CPW;           // column groups
  static constexpr int KS = kWresWarps / CGW;    // K slices
};

template <int GM>
struct WresFixed {
  using Sh = WresShape<GM>;
  uint16_t ring[kWresWarps][kWresRing][kWresTok * 8];  // x groups: [token][8 values]
  float xsqp[Sh::KS][kWresTok];                        // per-slice sums of x^2
  float lgt[kWresTok][GM + 1];
  float err[kWresTok][GM + 1];
  float wsqp[kWresWarps][GM];                          // per-warp column sums of squares
  float wnorm[GM];
  float bias[GM];
  uint64_t wbar;                                       // the W_r copy
  int nflag;
  int flags[kWresTok * GM];
  int sel[kRouteMaxWarps][kMaxM];
};

__host__ __device__ constexpr size_t align128(size_t x) { return (x + 127) / 128 * 128; }

// Dynamic shared memory: W_r as [dm/2][GM] float pairs, the per-slice
// partial logits part[KS][64][GM+1], then the fixed part.
template <int GM>
struct WresLayout {
  size_t part, fixed, total;
  __host__ __device__ explicit WresLayout(int dm) {
    part = align128(static_cast<size_t>(dm) * GM * 4);
    fixed = align128(part + sizeof(float) * WresShape<GM>::KS * kWresTok * (GM + 1));
    total = fixed + sizeof(WresFixed<GM>);
  }
};

// W_r [G][dm][M] bf16 -> float32 pairs: 16-byte unit d holds rows 2p, 2p+1
// of columns c, c+1 (p = d / (GM/2), c = 2 (d % (GM/2))).
template <int GM>
__global__ void __launch_bounds__(256) route_pairs_kernel(const RouteArgs a) {
  grid_dep_wait();  // launched with launch_pdl
  const int d = blockIdx.x * 256 + threadIdx.x;
  if (d >= a.dm * GM / 4) return;
  const int dm = a.dm, M = a.M;
  const int p = d / (GM / 2), c = 2 * (d % (GM / 2));
  const int g0 = c / M, m0 = c % M, g1 = (c + 1) / M, m1 = (c + 1) % M;
  const uint16_t* w0 = a.Wr + (static_cast<int64_t>(g0) * dm + 2 * p) * M + m0;
  const uint16_t* w1 = a.Wr + (static_cast<int64_t>(g1) * dm + 2 * p) * M + m1;
  reinterpret_cast<float4*>(a.wt)[d] =
      make_float4(bf16_bits_to_float(w0[0]), bf16_bits_to_float(w0[M]), bf16_bits_to_float(w1[0]),
                  bf16_bits_to_float(w1[M]));
}

template <int GM>
__global__ void __launch_bounds__(kWresThreads, 1) route_wres_kernel(const RouteArgs a) {
  grid_dep_wait();  // launched with launch_pdl
  using Sh = WresShape<GM>;
  constexpr int CPW = Sh::CPW, CGW = Sh::CGW, KS = Sh::KS;
  extern __shared__ __align__(128) uint8_t wres_smem_raw[];
  const int dm = a.dm;
  const WresLayout<GM> lay(dm);
  WresFixed<GM>& sm = *reinterpret_cast<WresFixed<GM>*>(wres_smem_raw + lay.fixed);
  const float2* Ws = reinterpret_cast<const float2*>(wres_smem_raw);
  float* part = reinterpret_cast<float*>(wres_smem_raw + lay.part);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cg = warp % CGW, ks = warp / CGW;
  const int slice = dm / KS;                 // values of d_model per K slice
  const int nq = slice / 8;                  // 8-value groups per slice
  const float cerr = static_cast<float>(slice / 2 + KS + 1) * 5.9604645e-8f * 1.01f;
  const int ntiles = (a.T + kWresTok - 1) / kWresTok;
  const int my_tiles = blockIdx.x < ntiles ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  // W_r pairs by one bulk copy
  const uint32_t wbytes = static_cast<uint32_t>(dm) * GM * 4;
  if (tid == 0) {
    mbar_init(&sm.wbar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0) {  // in 4 KB pieces, each CTA starting at a different one
    mbar_arrive_expect_tx(&sm.wbar, wbytes);
    const uint32_t npc = (wbytes + 4095) / 4096;
    for (uint32_t i = 0; i < npc; ++i) {
      const uint32_t pc = (i + blockIdx.x) % npc, off = pc * 4096;
      const uint32_t len = wbytes - off < 4096 ? wbytes - off : 4096;
      bulk_load(wres_smem_raw + off, reinterpret_cast<const uint8_t*>(a.wt) + off, len, &sm.wbar);
    }
  }

  // this warp's x groups, in the order it reduces them: groups 0..nq-1 of
  // tile blockIdx.x, then of tile blockIdx.x + gridDim.x, ...; lane l copies
  // tokens l and l + 32 of a group into ring slot (group number) % kWresRing
  uint16_t (*ring)[kWresTok * 8] = sm.ring[warp];
  int f_tile = blockIdx.x, f_q = 0, f_slot = 0;
  auto fetch = [&]() {
    if (f_tile < ntiles) {
      const int e = ks * slice + 8 * f_q;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int t = f_tile * kWresTok + lane + 32 * h;
        const bool in = t < a.T;
        cp_async_16(&ring[f_slot][(lane + 32 * h) * 8],
                    a.x + static_cast<int64_t>(in ? t : 0) * dm + e, in ? 16u : 0u);
      }
      if (++f_q == nq) {
        f_q = 0;
        f_tile += gridDim.x;
      }
    }
    cp_async_commit();
    f_slot = f_slot + 1 == kWresRing ? 0 : f_slot + 1;
  };
#pragma unroll
  for (int i = 0; i < kWresRing - 1; ++i) fetch();

  for (int c = tid; c < GM; c += kWresThreads) sm.bias[c] = a.bias ? a.bias[c] : 0.f;
  const bool wok = mbar_wait(&sm.wbar, 0, nullptr, a.status, kWaitLimitNs);
  if (__syncthreads_or(!wok)) {  // let this thread's copies land, then stop
    cp_async_wait_all();
    return;
  }
  // column norms: the lanes of a warp with the same column pair add their
  // row pairs (rows 2p, 2p+1 with p = warp-and-lane order), then the warps in order
  {
    const float4* Wv = reinterpret_cast<const float4*>(Ws);
    const int c = 2 * (tid % (GM / 2));
    float s0 = 0.f, s1 = 0.f;
    for (int d = tid; d < dm * GM / 4; d += kWresThreads) {
      const float4 f = Wv[d];
      s0 = fmaf(f.x, f.x, s0);
      s0 = fmaf(f.y, f.y, s0);
      s1 = fmaf(f.z, f.z, s1);
      s1 = fmaf(f.w, f.w, s1);
    }
#pragma unroll
    for (int off = GM / 2; off < 32; off <<= 1) {
      s0 += __shfl_xor_sync(0xFFFFFFFFu, s0, off);
      s1 += __shfl_xor_sync(0xFFFFFFFFu, s1, off);
    }
    if (lane < GM / 2) {
      sm.wsqp[warp][c] = s0;
      sm.wsqp[warp][c + 1] = s1;
    }
  }
  __syncthreads();
  for (int c = tid; c < GM; c += kWresThreads) {
    float s2 = 0.f;
    for (int r = 0; r < kWresWarps; ++r) s2 += sm.wsqp[r][c];
    sm.wnorm[c] = sqrtf(s2);
  }

  // this warp's W_r pairs start at row pair ks*slice/2, column cg*CPW
  const float4* wbase =
      reinterpret_cast<const float4*>(Ws + static_cast<int64_t>(ks) * (slice / 2) * GM + cg * CPW);
  int slot = 0;  // ring slot of this warp's next group
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const int t0 = tile * kWresTok;
    const int ntok = min(kWresTok, a.T - t0);
    if (tid == 0) sm.nflag = 0;
    uint64_t acc[2][CPW];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int c = 0; c < CPW; ++c) acc[h][c] = 0;  // the bits of (+0, +0)
    uint64_t xq[2] = {0, 0};
    const float4* wr = wbase;
#pragma unroll 1
    for (int q = 0; q < nq; ++q) {
      fetch();
      cp_async_wait_group<kWresRing - 1>();  // this lane's copies of the group have landed
      __syncwarp();
      const uint32_t* g32 = reinterpret_cast<const uint32_t*>(ring[slot]);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        // (x[2p], x[2p+1]) of the two tokens: the halves of one 32-bit word
        const uint32_t wa = g32[lane * 4 + r], wb = g32[(lane + 32) * 4 + r];
        const uint64_t x0 = f2_pack(__uint_as_float(wa << 16), __uint_as_float(wa & 0xFFFF0000u));
        const uint64_t x1 = f2_pack(__uint_as_float(wb << 16), __uint_as_float(wb & 0xFFFF0000u));
#pragma unroll
        for (int c2 = 0; c2 < CPW / 2; ++c2) {
          const float4 w4 = wr[c2];
          const uint64_t wlo = f2_pack(w4.x, w4.y), whi = f2_pack(w4.z, w4.w);
          acc[0][2 * c2] = f2_fma(x0, wlo, acc[0][2 * c2]);
          acc[0][2 * c2 + 1] = f2_fma(x0, whi, acc[0][2 * c2 + 1]);
          acc[1][2 * c2] = f2_fma(x1, wlo, acc[1][2 * c2]);
          acc[1][2 * c2 + 1] = f2_fma(x1, whi, acc[1][2 * c2 + 1]);
          if (c2 % 4 == 3) asm volatile("" ::: "memory");  // at most 4 loads ahead
        }
        if (cg == 0) {
          xq[0] = f2_fma(x0, x0, xq[0]);
          xq[1] = f2_fma(x1, x1, xq[1]);
        }
        wr += GM / 2;
        // keep the next row pair's loads below this one's FMAs (registers)
        asm volatile("" ::: "memory");
      }
      __syncwarp();  // the ring slot is read before a later fetch overwrites it
      slot = slot + 1 == kWresRing ? 0 : slot + 1;
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int c = 0; c < CPW; ++c) {
        float lo, hi;
        f2_unpack(acc[h][c], lo, hi);
        part[(ks * kWresTok + lane + 32 * h) * (GM + 1) + cg * CPW + c] = lo + hi;
      }
      if (cg == 0) {
        float lo, hi;
        f2_unpack(xq[h], lo, hi);
        sm.xsqp[ks][lane + 32 * h] = lo + hi;
      }
    }
    __syncthreads();

    // logits (slice sums in slice order, then the bias) and their bounds
    bool nonfinite = false;
    for (int qq = tid; qq < ntok * GM; qq += kWresThreads) {
      const int ql = qq / GM, col = qq % GM;
      const float bv = sm.bias[col];
      float l = part[ql * (GM + 1) + col], x2 = sm.xsqp[0][ql];
#pragma unroll
      for (int w = 1; w < KS; ++w) {
        l += part[(w * kWresTok + ql) * (GM + 1) + col];
        x2 += sm.xsqp[w][ql];
      }
      l += bv;
      sm.lgt[ql][col] = l;
      sm.err[ql][col] = cerr * fmaf(sqrtf(x2), sm.wnorm[col], fabsf(bv)) + 1e-36f;
      nonfinite |= !isfinite(l);
    }
    if (nonfinite) latch_status(a.status, GQE_ERR_NONFINITE);
    __syncthreads();
    route_tile_epilogue<GM>(a, &sm.lgt[0][0], &sm.err[0][0], t0, ntok, &sm.nflag, sm.flags,
                            sm.sel);
    __syncthreads();
  }
  cp_async_wait_all();  // the empty trailing groups
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

struct Exact {            // normalised: v[0..16] in [0, 2^32), top signed
  uint32_t v[kLimbs - 1];
  int32_t top;
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

// Terms of one exact logit: products x_j * w_jm (16-bit integer times
// 2^(pos-266)) and the bias (24-bit integer).  Returns 0 for a zero term.
struct Term {
  long long mant;
  int pos;
};

__device__ __forceinline__ Term product_term(uint32_t xb, uint32_t wb) {
  int sx, mx, ex, sw, mw, ew;
  bf16_decompose(xb, sx, mx, ex);
  bf16_decompose(wb, sw, mw, ew);
  long long prod = static_cast<long long>(mx) * mw;
  if (sx ^ sw) prod = -prod;
  return Term{prod, ex + ew + kExpBias};
}

__device__ __forceinline__ Term bias_term(float bias) {
  const uint32_t bb = __float_as_uint(bias);
  const int E = (bb >> 23) & 0xFF;
  long long mant = (E == 0) ? (bb & 0x7FFFFF) : ((bb & 0x7FFFFF) | 0x800000);
  if (bb >> 31) mant = -mant;
  return Term{mant, ((E == 0) ? -149 : E - 150) + kExpBias};
}

constexpr int kWin = 7;  // register window of 32-bit limbs

__device__ void exact_logit(const RouteArgs& a, int t, int g, int m, Exact& out, bool& bad) {
  const int lane = threadIdx.x & 31;
  const uint16_t* xr = a.x + static_cast<int64_t>(t) * a.dm;
  const uint16_t* wr = a.Wr + static_cast<int64_t>(g) * a.dm * a.M + m;
  const bool has_bias = (lane == 0) && a.bias;
  // pass 1: range of bit positions occupied by the terms
  int pmin = 1 << 30, tmax = -(1 << 30);
#pragma unroll 4
  for (int j = lane; j < a.dm; j += 32) {
    const uint32_t xb = xr[j], wb = wr[static_cast<int64_t>(j) * a.M];
    if (((xb >> 7) & 0xFF) == 0xFF || ((wb >> 7) & 0xFF) == 0xFF) {
      bad = true;
      continue;
    }
    const Term tm = product_term(xb, wb);
    if (tm.mant != 0) {
      pmin = min(pmin, tm.pos);
      tmax = max(tmax, tm.pos + 16);
    }
  }
  Term bt{0, 0};
  if (has_bias) {
    const float bv = a.bias[g * a.M + m];
    if (!isfinite(bv)) bad = true;
    else bt = bias_term(bv);
    if (bt.mant != 0) {
      pmin = min(pmin, bt.pos);
      tmax = max(tmax, bt.pos + 24);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    pmin = min(pmin, __shfl_xor_sync(0xFFFFFFFFu, pmin, off));
    tmax = max(tmax, __shfl_xor_sync(0xFFFFFFFFu, tmax, off));
  }
  long long full[kLimbs];
#pragma unroll
  for (int i = 0; i < kLimbs; ++i) full[i] = 0;
  if (tmax >= pmin) {  // at least one non-zero term
    const int base = pmin >> 5;
    // at most d_model + 1 terms: the sum stays below 2^(tmax + 13)
    if (tmax + 14 - 32 * base <= 32 * (kWin - 1) - 1) {
      // fast path: every term lands in limbs [base, base + kWin) held in registers
      long long w[kWin];
#pragma unroll
      for (int i = 0; i < kWin; ++i) w[i] = 0;
      auto add = [&](const Term& tm) {
        const int L = (tm.pos >> 5) - base, o = tm.pos & 31;
        const long long v = tm.mant * (1ll << o);
        const long long lo = v & 0xFFFFFFFFll, hi = v >> 32;
#pragma unroll
        for (int i = 0; i < kWin; ++i) w[i] += (i == L ? lo : 0) + (i == L + 1 ? hi : 0);
      };
      for (int j = lane; j < a.dm; j += 32) {
        const uint32_t xb = xr[j], wb = wr[static_cast<int64_t>(j) * a.M];
        if (((xb >> 7) & 0xFF) == 0xFF || ((wb >> 7) & 0xFF) == 0xFF) continue;
        const Term tm = product_term(xb, wb);
        if (tm.mant != 0) add(tm);
      }
      if (bt.mant != 0) add(bt);
#pragma unroll
      for (int i = 0; i < kWin; ++i) {
        long long v = w[i];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
        w[i] = v;
      }
      for (int i = 0; i < kWin && base + i < kLimbs; ++i) full[base + i] = w[i];
    } else {
      // wide exponent range: the full 18-limb accumulator
      for (int j = lane; j < a.dm; j += 32) {
        const uint32_t xb = xr[j], wb = wr[static_cast<int64_t>(j) * a.M];
        if (((xb >> 7) & 0xFF) == 0xFF || ((wb >> 7) & 0xFF) == 0xFF) continue;
        const Term tm = product_term(xb, wb);
        if (tm.mant != 0) limbs_add(full, tm.mant, tm.pos);
      }
      if (bt.mant != 0) limbs_add(full, bt.mant, bt.pos);
#pragma unroll
      for (int i = 0; i < kLimbs; ++i) {
        long long v = full[i];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
        full[i] = v;
      }
    }
  }
  // carry pass: limbs 0..16 into [0, 2^32), the top limb keeps the sign
#pragma unroll
  for (int i = 0; i < kLimbs - 1; ++i) {
    const long long c = full[i] >> 32;  // floor division by 2^32
    full[i] -= c * 4294967296ll;
    full[i + 1] += c;
  }
#pragma unroll
  for (int i = 0; i < kLimbs - 1; ++i) out.v[i] = static_cast<uint32_t>(full[i]);
  out.top = static_cast<int32_t>(full[kLimbs - 1]);  // |sum| < 2^540: top limb is tiny
}

// The value of an exact logit as a double (the limbs from the top down, then
// the 2^-266 scale): within a few ulps, enough for the softmax; the ordering
// itself uses exact_cmp.
__device__ __forceinline__ double exact_to_double(const Exact& e) {
  double v = static_cast<double>(e.top);
  for (int i = kLimbs - 2; i >= 0; --i) v = v * 4294967296.0 + static_cast<double>(e.v[i]);
  return ldexp(v, -kExpBias);
}

// -1, 0, +1 for a < b, a == b, a > b
__device__ __forceinline__ int exact_cmp(const Exact& a, const Exact& b) {
  if (a.top != b.top) return a.top < b.top ? -1 : 1;
  for (int i = kLimbs - 2; i >= 0; --i)
    if (a.v[i] != b.v[i]) return a.v[i] < b.v[i] ? -1 : 1;
  return 0;
}

// Float64 logits of one (token, group) pair, with a rigorous bound: every
// bf16*bf16 product is exact in float64; each lane sums its ceil(dm/32)
// products in order, the warp adds the 32 partial sums in a 5-level tree,
// and the bias is added last, so |l64 - l| <= (ceil(dm/32) + 7) 2^-53 A with
// A = sum |x_j w_j| + |bias| (bound doubled for the rounding of A itself).
__device__ void logit64(const RouteArgs& a, int t, int g, int m, double& l, double& err) {
  const int lane = threadIdx.x & 31;
  const uint16_t* xr = a.x + static_cast<int64_t>(t) * a.dm;
  const uint16_t* wr = a.Wr + static_cast<int64_t>(g) * a.dm * a.M + m;
  double s = 0.0, A = 0.0;
#pragma unroll 8
  for (int j = lane; j < a.dm; j += 32) {
    const double p = static_cast<double>(bf16_bits_to_float(xr[j])) *
                     static_cast<double>(bf16_bits_to_float(wr[static_cast<int64_t>(j) * a.M]));
    s += p;
    A += fabs(p);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    s += __shfl_xor_sync(0xFFFFFFFFu, s, off);
    A += __shfl_xor_sync(0xFFFFFFFFu, A, off);
  }
  if (a.bias) {
    const double b = a.bias[g * a.M + m];
    s += b;
    A += fabs(b);
  }
  l = s;
  err = 2.0 * ((a.dm + 31) / 32 + 7) * 1.1102230246251565e-16 * A;
}

// Exact top-k of one (token, group) pair by one warp: exact logits of the
// group's M experts, ranks by (logit desc, index asc), then w from p.  The
// float64 pass decides every pair whose gaps exceed its bound; only pairs
// still undecided (in practice exact ties) take the fixed-point path.
__device__ void exact_rank_pair(const RouteArgs& a, int t, int g, int* sel) {
  __shared__ Exact ex[kRouteMaxWarps][kMaxM];
  __shared__ double l64[kRouteMaxWarps][kMaxM], e64[kRouteMaxWarps][kMaxM];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int M = a.M, k = a.k;
  bool bad = false;
  for (int m = 0; m < M; ++m) {
    double l, e;
    logit64(a, t, g, m, l, e);
    if (lane == 0) {
      l64[warp][m] = l;
      e64[warp][m] = e;
    }
  }
  __syncwarp();
  // ranks from the float64 logits (ties -> lower index), certified when every
  // compared pair is separated by more than the two bounds
  bool certain = true;
  int rank = 0;
  if (lane < M) {
    const double la = l64[warp][lane], ea = e64[warp][lane];
    for (int b = 0; b < M; ++b) {
      if (b == lane) continue;
      const double lb = l64[warp][b], eb = e64[warp][b];
      if (lb > la || (lb == la && b < lane)) ++rank;
      if (!(fabs(la - lb) > (ea + eb) * 1.0000001)) certain = false;
    }
  }
  certain = __all_sync(0xFFFFFFFFu, certain);
  if (!certain) {
    for (int m = 0; m < M; ++m) {
      Exact e;
      exact_logit(a, t, g, m, e, bad);
      if (lane == 0) ex[warp][m] = e;
    }
    bad = __any_sync(0xFFFFFFFFu, bad);
    __syncwarp();
    if (lane < M) {
      rank = 0;
      for (int b = 0; b < M; ++b) {
        if (b == lane) continue;
        const int c = exact_cmp(ex[warp][b], ex[warp][lane]);
        if (c > 0 || (c == 0 && b < lane)) ++rank;
      }
    }
  }
  if (lane < M && rank < k) sel[rank] = lane;
  // p of this pair again, from the float64 logits or (when those could not
  // order the experts) the exact ones: the float32 logits of the main pass
  // may have cancelled catastrophically for a pair that needed this path
  if (lane < M && !certain) l64[warp][lane] = exact_to_double(ex[warp][lane]);
  __syncwarp();
  if (lane == 0) {
    if (bad) latch_status(a.status, GQE_ERR_NONFINITE);
    const int64_t row = static_cast<int64_t>(t) * a.G + g;
    float* prow = a.p + row * M;
    double mx = l64[warp][0];
    for (int m = 1; m < M; ++m) mx = fmax(mx, l64[warp][m]);
    double s = 0.0;
    for (int m = 0; m < M; ++m) s += exp(l64[warp][m] - mx);
    for (int m = 0; m < M; ++m) prow[m] = static_cast<float>(exp(l64[warp][m] - mx) / s);
    float den = 0.f;
    for (int j = 0; j < k; ++j) den += prow[sel[j]];
    for (int j = 0; j < k; ++j) {
      a.topk_idx[row * k + j] = sel[j];
      a.w[row * k + j] = (k == 1) ? 1.0f : prow[sel[j]] / den;
    }
  }
  __syncwarp();
}

template <int GM>
cudaError_t launch_route_gm(const RouteArgs& a, cudaStream_t st) {
  static int configured = -1;
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int smem = static_cast<int>(sizeof(RouteSmem<GM>));
  if (configured != dev) {
    e = cudaFuncSetAttribute(route_kernel<GM>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured = dev;
  }
  e = launch_pdl(route_prep_kernel<GM>, dim3((a.dm + 31) / 32), dim3(32 * GM), 0, st, a);
  if (e != cudaSuccess) return e;
  // tokens per tile: about two tiles per SM when the tokens allow it, at most
  // kTok (two per lane)
  RouteArgs b = a;
  const int64_t want = (static_cast<int64_t>(a.T) + 2 * sms - 1) / (2 * sms);
  b.tok = static_cast<int>(want < 1 ? 1 : (want > RouteShape<GM>::kTok ? RouteShape<GM>::kTok : want));
  const int ntiles = (a.T + b.tok - 1) / b.tok;
  const int grid = ntiles < 4 * sms ? ntiles : 4 * sms;
  return launch_pdl(route_kernel<GM>, dim3(grid), dim3(kRouteThreads), smem, st, b);
}

template <int GM>
cudaError_t launch_route_wres(const RouteArgs& a, cudaStream_t st) {
  static int configured = -1;
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int smem = static_cast<int>(WresLayout<GM>(a.dm).total);
  if (configured != dev) {  // the largest size this kernel is ever launched with
    e = cudaFuncSetAttribute(route_wres_kernel<GM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kWresMaxSmem);
    if (e != cudaSuccess) return e;
    configured = dev;
  }
  const int npairs = a.dm * GM / 4;
  e = launch_pdl(route_pairs_kernel<GM>, dim3((npairs + 255) / 256), dim3(256), 0, st, a);
  if (e != cudaSuccess) return e;
  const int ntiles = (a.T + kWresTok - 1) / kWresTok;
  const int grid = ntiles < sms ? ntiles : sms;
  return launch_pdl(route_wres_kernel<GM>, dim3(grid), dim3(kWresThreads), smem, st, a);
}

// The shared-memory-resident kernel when W_r fits, each K slice is a whole
// number of 8-value groups and there are at least kWresMinTiles tiles per SM
// (its per-CTA start, loading all of W_r, costs about as much as a tile; with
// fewer tokens the streamed kernel measured as fast or faster); the streamed
// kernel otherwise.
constexpr int kWresMinTiles = 3;

template <int GM>
cudaError_t launch_route_any(const RouteArgs& a, cudaStream_t st) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const bool fits = a.dm % (8 * WresShape<GM>::KS) == 0 &&
                    static_cast<int64_t>(a.dm) * GM * 4 <= kWresMaxW &&
                    WresLayout<GM>(a.dm).total <= static_cast<size_t>(kWresMaxSmem);
  const bool many = static_cast<int64_t>(a.T) >= static_cast<int64_t>(kWresMinTiles) * sms * kWresTok;
  return fits && (many || g_route_force_resident.load() != 0) ? launch_route_wres<GM>(a, st)
                                                  : launch_route_gm<GM>(a, st);
}

}  // namespace

int set_route_force_resident(int on) {
  return on < 0 ? g_route_force_resident.load() : g_route_force_resident.exchange(on != 0 ? 1 : 0);
}

cudaError_t launch_route(const RouteArgs& a, cudaStream_t st) {
  switch (a.G * a.M) {
    case 4: return launch_route_any<4>(a, st);
    case 8: return launch_route_any<8>(a, st);
    case 16: return launch_route_any<16>(a, st);
    case 32: return launch_route_any<32>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace gqe
