// Backward pass of the GQE prefill path on the sm_100a tensor cores.
//
// "AI 大模型之 GQA", 训练与部署 共享键值的梯度归约: every query head's attention
// backward is computed on its own, the gradients of a shared KV head are the
// SUM of the contributions of every head that reads it, and query gradients
// stay with their head.  Here the heads that read KV head g are the routed
// experts of group g (only for the tokens that selected them) and, for g = 0,
// the always-on shared head.  "论文综述：分组查询专家" §二 三个关键部件:
// o_bar = sum_j w_j o_j, so slot j's output receives dO_sel_j + w_j d(o_bar)
// and dw_j = <d(o_bar), o_j>.
//
// Per head and row, with P = softmax of the scaled scores (causal), O = P V:
//   dV = P^T dO, dP = dO V^T, dS = P * (dP - rowsum(dO * O)),
//   dQ = dS K / sqrt(d), dK = dS^T Q / sqrt(d).
//
// bwd_prep_kernel: per routed slot, dO_eff = dO_sel + w * d(o_bar) (bf16 for
//   the tensor cores), D = <dO_eff, O_sel>, dw = <d(o_bar), O_sel>; per token
//   of the shared head, dO = ds (bf16) and D = <ds, s>.
// bwd_kernel<D>: one CTA per (batch, group, KV tile of 128 keys).  It holds
//   K_t, V_t in shared memory and dK_t, dV_t in TMEM, and walks every query
//   tile that can see the tile: the bucket rows of each expert of the group
//   from the first position >= the tile's first key on, and for group 0 the
//   shared head's query tiles.  Per query tile:
//     S^T = K_t Q^T and dP^T = V_t dO^T        (UMMA, M = 128 keys)
//     P^T, dS^T from S^T, dP^T, the forward's log-sum-exp and D (thread =
//       key row), rounded to bf16 into shared memory
//     dV_t += P^T dO, dK_t += dS^T Q             (UMMA, A = P^T / dS^T)
//     dQ = dS K_t                                (UMMA, A = dS^T read M-major)
//   dQ is added into a float32 buffer with vector atomics (several KV tiles
//   contribute to a query row); dK_t, dV_t are written once at the end, so a
//   KV head's gradient is summed over all of its heads without atomics.
// Warp roles (192 threads): warps 0-3 math + epilogues, warp 4 loads (K/V by
// TMA once, Q and dO rows gathered by cp.async per query tile), warp 5 TMEM
// owner and tcgen05.mma issuer.
#include <cuda_bf16.h>

#include "gqe_device.cuh"

namespace gqe {
namespace {

constexpr int kBwdThreads = 192;
constexpr int kAtomB = kTileM * 128;  // 128 rows x 128 B (64 bf16)

template <int D>
struct BwdCfg {
  static constexpr int kKVBytes = kTileN * D * 2;  // one K or V tile
  static constexpr int kQBytes = kTileM * D * 2;   // one Q or dO tile
  static constexpr int kPBytes = kTileN * kTileM * 2;  // P^T or dS^T: 128 x 128 bf16
  // Q/dO tiles are double-buffered at d = 64; at d = 128 one buffer keeps the
  // CTA within the shared-memory limit
  static constexpr int kQBufs = D == 64 ? 2 : 1;
  static constexpr int kSmemK = 0;
  static constexpr int kSmemV = kSmemK + kKVBytes;
  static constexpr int kSmemQ = kSmemV + kKVBytes;
  static constexpr int kSmemDO = kSmemQ + kQBufs * kQBytes;
  static constexpr int kSmemP = kSmemDO + kQBufs * kQBytes;
  static constexpr int kSmemDS = kSmemP + kPBytes;
  static constexpr int kSmemVec = kSmemDS + kPBytes;       // kQBufs x (lse, D, pos) x 128
  static constexpr int kSmemBar = kSmemVec + kQBufs * 3 * 128 * 4;
  static constexpr int kSmemBytes = kSmemBar + 512 + 1024;  // barriers, lo/cnt, alignment
  // TMEM: S^T (128), dP^T (128), dV (D), dK (D); dQ reuses the S^T columns
  static constexpr uint32_t kTS = 0, kTdP = 128, kTdV = 256, kTdK = 256 + D;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kIdescKQ = make_idesc_f16(kTileM, kTileN, /*bf16*/ 1, 0, 0);
  static constexpr uint32_t kIdescPd = make_idesc_f16(kTileM, D, /*bf16*/ 1, 0, /*MN*/ 1);
  static constexpr uint32_t kIdescdQ = make_idesc_f16(kTileM, D, /*bf16*/ 1, /*MN*/ 1, /*MN*/ 1);
};

enum : int {
  kBbKV = 0,
  kBbQFull = 1,   // +buffer
  kBbQFree = 3,   // +buffer
  kBbSFull = 5,
  kBbPFull = 6,
  kBbDQFull = 7,
  kBbDQFree = 8,
  kBbAcc = 9,
  kBbSpare = 10,
  kBbNum = 11
};

struct BWaiter {
  volatile int* abort;
  int* status;
  uint64_t limit;
  __device__ bool operator()(uint64_t* bar, uint32_t parity) const {
    return mbar_wait(bar, parity, abort, status, limit);
  }
};

// The query tiles of one CTA, in the same order for every role: for each
// expert m of the group, rows [lo_m, cnt_m) of its bucket in chunks of 128,
// then (group 0) the shared head's query tiles from the KV tile's on.
struct TileWalk {
  int m, row, shared_q;  // current expert and row (routed), or shared query tile
};

struct BwdTile {
  int kind, m, row0, nrows;
};

__device__ __forceinline__ bool next_tile(TileWalk& w, const int* lo, const int* cnt, int M, int g,
                                          int t, int nq, int S, BwdTile& out) {
  while (w.m < M) {
    if (w.row < cnt[w.m]) {
      out = BwdTile{kRouted, w.m, w.row, min(kTileM, cnt[w.m] - w.row)};
      w.row += kTileM;
      return true;
    }
    ++w.m;
    if (w.m < M) w.row = lo[w.m];
  }
  if (g == 0 && w.shared_q < nq) {
    const int q = w.shared_q++;
    out = BwdTile{kShared, -1, q * kTileM, min(kTileM, S - q * kTileM)};
    return true;
  }
  return false;
}

// bf16 row of d values into the 128-byte-swizzled K-major layout (one row of
// a 128-row tile): 16-byte chunk c of row r at c ^ (r & 7) inside its
// 64-element atom.
template <int D>
__device__ __forceinline__ void gather_row(uint8_t* dst, int r, const uint16_t* src, bool valid) {
#pragma unroll
  for (int c = 0; c < D / 8; ++c)
    cp_async_16(dst + (c >> 3) * kAtomB + r * 128 + (((c & 7) ^ (r & 7)) << 4), src + c * 8,
                valid ? 16u : 0u);
}

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_kernel(const __grid_constant__ BwdArgs a) {
  grid_dep_wait();  // launched with launch_pdl
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.S, G = a.G, M = a.M, N = a.N, k = a.k;
  const int nq = (S + kTileM - 1) / kTileM;
  // heaviest first: the first KV tiles are seen by the most queries
  const int bg_count = a.B * G;
  const int t = static_cast<int>(blockIdx.x) / bg_count;
  const int bg = static_cast<int>(blockIdx.x) % bg_count;
  const int b = bg / G, g = bg % G;
  const int kv0 = t * kTileN;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kSmemBar);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + kBbNum);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + kBbNum + 1);
  int* lo = reinterpret_cast<int*>(bars + kBbNum + 2);  // [kMaxM]
  int* cnt = lo + kMaxM;                                 // [kMaxM]
  const BWaiter wait{abort_flag, a.status, a.wait_limit_ns};
  float* vec = reinterpret_cast<float*>(smem + C::kSmemVec);  // [buf][lse | D | pos][128]

  if (threadIdx.x == 0) {
    mbar_init(&bars[kBbKV], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[kBbQFull + s], 1);
      mbar_init(&bars[kBbQFree + s], 1);
    }
    mbar_init(&bars[kBbSFull], 1);
    mbar_init(&bars[kBbPFull], 4);
    mbar_init(&bars[kBbDQFull], 1);
    mbar_init(&bars[kBbDQFree], 4);
    mbar_init(&bars[kBbAcc], 1);
    mbar_init(&bars[kBbSpare], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  // first row of each expert's bucket at a position >= kv0 (binary search)
  if (warp == 0 && lane < M) {
    const int id = (b * G + g) * M + lane;
    const int s0 = a.bucket_off[id], s1 = a.bucket_off[id + 1];
    int lo_i = 0, hi = s1 - s0;
    while (lo_i < hi) {
      const int mid = (lo_i + hi) >> 1;
      if (a.bucket_tok[s0 + mid] < kv0) lo_i = mid + 1;
      else hi = mid;
    }
    lo[lane] = lo_i;
    cnt[lane] = s1 - s0;
  }
  if (warp == 5) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&a.tmK);
    tma_prefetch_desc(&a.tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;
  const float sl2 = a.scale_log2;

  if (warp == 4) {
    // ------------------------------------------------------ loads
    if (lane == 0) {
      mbar_arrive_expect_tx(&bars[kBbKV], 2 * C::kKVBytes);
#pragma unroll
      for (int at = 0; at < D / 64; ++at) {
        tma_load_4d(smem + C::kSmemK + at * kAtomB, &a.tmK, &bars[kBbKV], at * 64, g, kv0, b);
        tma_load_4d(smem + C::kSmemV + at * kAtomB, &a.tmV, &bars[kBbKV], at * 64, g, kv0, b);
      }
    }
    TileWalk wk{0, lo[0], t};
    BwdTile tl;
    for (int i = 0; next_tile(wk, lo, cnt, M, g, t, nq, S, tl); ++i) {
      const int buf = i % C::kQBufs, round = i / C::kQBufs;
      if (round > 0 && !__all_sync(0xFFFFFFFFu, wait(&bars[kBbQFree + buf], (round - 1) & 1)))
        break;
      uint8_t* sQ = smem + C::kSmemQ + buf * C::kQBytes;
      uint8_t* sDO = smem + C::kSmemDO + buf * C::kQBytes;
      float* vlse = vec + buf * 3 * 128;
      const int bstart =
          tl.kind == kRouted ? a.bucket_off[(b * G + g) * M + tl.m] : 0;
      const int h = g * M + tl.m;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int r = lane + 32 * q;
        const bool valid = r < tl.nrows;
        const int rv = valid ? r : tl.nrows - 1;
        const int pos = tl.kind == kRouted ? a.bucket_tok[bstart + tl.row0 + rv] : tl.row0 + rv;
        const int64_t tok = static_cast<int64_t>(b) * S + pos;
        const uint16_t *qsrc, *dosrc;
        float lse, dd;
        if (tl.kind == kRouted) {
          const int32_t* sel = a.topk_idx + (tok * G + g) * k;
          int slot = 0;
          for (int j = 0; j < k; ++j)
            if (sel[j] == tl.m) slot = j;
          const int64_t si = (tok * G + g) * k + slot;
          qsrc = a.Q + (tok * N + h) * D;
          dosrc = a.dO_r + si * D;
          lse = a.lse_sel[si];
          dd = a.D_r[si];
        } else {
          qsrc = a.Qs + tok * D;
          dosrc = a.dO_s + tok * D;
          lse = a.lse_s[tok];
          dd = a.D_s[tok];
        }
        gather_row<D>(sQ, r, qsrc, valid);
        gather_row<D>(sDO, r, dosrc, valid);
        vlse[r] = valid ? lse : INFINITY;  // P = 0 on rows past the tile
        vlse[128 + r] = valid ? dd : 0.f;
        vlse[256 + r] = __int_as_float(valid ? pos : -1);
      }
      cp_async_wait_all();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBbQFull + buf]);
    }
    if (lane == 0 && *abort_flag)
      mbar_wait(&bars[kBbKV], 0, nullptr, a.status, a.wait_limit_ns);
  } else if (warp == 5) {
    // ------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t tS = tbase + C::kTS, tdP = tbase + C::kTdP, tdV = tbase + C::kTdV,
                     tdK = tbase + C::kTdK;
      const uint32_t kaddr = smem_u32(smem + C::kSmemK), vaddr = smem_u32(smem + C::kSmemV);
      const uint32_t paddr = smem_u32(smem + C::kSmemP), dsaddr = smem_u32(smem + C::kSmemDS);
      bool ok = wait(&bars[kBbKV], 0);
      TileWalk wk{0, lo[0], t};
      BwdTile tl;
      int i = 0;
      for (; ok && next_tile(wk, lo, cnt, M, g, t, nq, S, tl); ++i) {
        const int buf = i % C::kQBufs;
        if (!wait(&bars[kBbQFull + buf], (i / C::kQBufs) & 1)) { ok = false; break; }
        if (i > 0 && !wait(&bars[kBbDQFree], (i - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t qaddr = smem_u32(smem + C::kSmemQ + buf * C::kQBytes);
        const uint32_t doaddr = smem_u32(smem + C::kSmemDO + buf * C::kQBytes);
        // S^T = K Q^T and dP^T = V dO^T: M = 128 keys, N = 128 queries, K = d
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kAtomB + (kk & 3) * 32;
          umma_ss(tS, make_sdesc_sw128(kaddr + off, 16, 1024),
                  make_sdesc_sw128(qaddr + off, 16, 1024), C::kIdescKQ, kk > 0 ? 1u : 0u);
          umma_ss(tdP, make_sdesc_sw128(vaddr + off, 16, 1024),
                  make_sdesc_sw128(doaddr + off, 16, 1024), C::kIdescKQ, kk > 0 ? 1u : 0u);
        }
        tc_commit(&bars[kBbSFull]);
        if (!wait(&bars[kBbPFull], i & 1)) { ok = false; break; }
        tc_fence_after();
        // dV += P^T dO, dK += dS^T Q: M = 128 keys, N = d, K = 128 queries
#pragma unroll
        for (int kk = 0; kk < kTileM / 16; ++kk) {
          const uint32_t aoff = (kk >> 2) * kAtomB + (kk & 3) * 32;
          umma_ss(tdV, make_sdesc_sw128(paddr + aoff, 16, 1024),
                  make_sdesc_sw128(doaddr + kk * 2048, kAtomB, 1024), C::kIdescPd,
                  (i > 0 || kk > 0) ? 1u : 0u);
          umma_ss(tdK, make_sdesc_sw128(dsaddr + aoff, 16, 1024),
                  make_sdesc_sw128(qaddr + kk * 2048, kAtomB, 1024), C::kIdescPd,
                  (i > 0 || kk > 0) ? 1u : 0u);
        }
        // dQ = dS K: M = 128 queries (dS^T read query-major), N = d, K = 128 keys
#pragma unroll
        for (int kk = 0; kk < kTileN / 16; ++kk)
          umma_ss(tS, make_sdesc_sw128(dsaddr + kk * 2048, kAtomB, 1024),
                  make_sdesc_sw128(kaddr + kk * 2048, kAtomB, 1024), C::kIdescdQ,
                  kk > 0 ? 1u : 0u);
        tc_commit(&bars[kBbDQFull]);
        tc_commit(&bars[kBbQFree + buf]);
      }
      if (ok) {
        tc_commit(&bars[kBbAcc]);
      } else {
        tc_commit(&bars[kBbSpare]);
        mbar_wait(&bars[kBbSpare], 0, nullptr, a.status, a.wait_limit_ns);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------ math warps
    const int r = warp * 32 + lane;  // key row of S^T / dP^T; query row of dQ
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const int key = kv0 + r;
    uint8_t* sP = smem + C::kSmemP;
    uint8_t* sDS = smem + C::kSmemDS;
    bool ok = true;
    TileWalk wk{0, lo[0], t};
    BwdTile tl;
    int i = 0;
    int ntiles = 0;
    for (; next_tile(wk, lo, cnt, M, g, t, nq, S, tl); ++i) {
      ++ntiles;
      const int buf = i % C::kQBufs;
      if (!__all_sync(0xFFFFFFFFu, wait(&bars[kBbSFull], i & 1))) { ok = false; break; }
      tc_fence_after();
      const float* vlse = vec + buf * 3 * 128;
      // this thread's query row of the tile (for its dQ row below): read now,
      // as the buffer may be refilled once this tile's products are issued
      const int my_pos = __float_as_int(vlse[256 + r]);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t sv[32], dv[32];
        tmem_ld32(tbase + lane_off + C::kTS + 32 * c, sv);
        tmem_ld32(tbase + lane_off + C::kTdP + 32 * c, dv);
        tmem_ld_wait(sv);
        tmem_ld_wait(dv);
        uint32_t pp[16], ss[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float p2[2], d2[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int q = 32 * c + e + u;
            const bool vis = key <= __float_as_int(vlse[256 + q]);
            const float p =
                vis ? ex2_approx(fmaf(__uint_as_float(sv[e + u]), sl2, -vlse[q])) : 0.f;
            p2[u] = p;
            d2[u] = p * (__uint_as_float(dv[e + u]) - vlse[128 + q]) * a.inv_sqrt_d;
          }
          __nv_bfloat162 hp = __floats2bfloat162_rn(p2[0], p2[1]);
          __nv_bfloat162 hd = __floats2bfloat162_rn(d2[0], d2[1]);
          pp[e / 2] = *reinterpret_cast<uint32_t*>(&hp);
          ss[e / 2] = *reinterpret_cast<uint32_t*>(&hd);
        }
        // row r (key) of P^T and dS^T: queries 32c .. 32c+31 are 4 chunks of 16 B
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int cq = 4 * c + u;  // 16-byte chunk of the 256-byte row
          const int off = (cq >> 3) * kAtomB + r * 128 + (((cq & 7) ^ (r & 7)) << 4);
          *reinterpret_cast<uint4*>(sP + off) =
              make_uint4(pp[4 * u], pp[4 * u + 1], pp[4 * u + 2], pp[4 * u + 3]);
          *reinterpret_cast<uint4*>(sDS + off) =
              make_uint4(ss[4 * u], ss[4 * u + 1], ss[4 * u + 2], ss[4 * u + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBbPFull]);
      // dQ rows of this query tile (thread = query row r): add into the
      // float32 accumulator
      if (!__all_sync(0xFFFFFFFFu, wait(&bars[kBbDQFull], i & 1))) { ok = false; break; }
      tc_fence_after();
      const bool valid = r < tl.nrows;
      float* dst = nullptr;
      if (valid) {
        const int64_t tok = static_cast<int64_t>(b) * S + my_pos;
        dst = tl.kind == kRouted ? a.dQ + (tok * N + g * M + tl.m) * D : a.dQs + tok * D;
      }
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tbase + lane_off + C::kTS + 32 * c, v);
        tmem_ld_wait(v);
        if (dst)
#pragma unroll
          for (int q = 0; q < 8; ++q)
            atomicAdd(reinterpret_cast<float4*>(dst + 32 * c) + q,
                      make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                  __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3])));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBbDQFree]);
    }
    // dK_t, dV_t (thread = key row): written once, summed over all heads
    ok = __all_sync(0xFFFFFFFFu, ok);
    if (ok && key < S) {
      float* dk = a.dK + ((static_cast<int64_t>(b) * S + key) * G + g) * D;
      float* dv = a.dV + ((static_cast<int64_t>(b) * S + key) * G + g) * D;
      if (ntiles == 0) {
        for (int c = 0; c < D; c += 4) {
          *reinterpret_cast<float4*>(dk + c) = make_float4(0.f, 0.f, 0.f, 0.f);
          *reinterpret_cast<float4*>(dv + c) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    }
    if (ok && ntiles > 0 && __all_sync(0xFFFFFFFFu, wait(&bars[kBbAcc], 0))) {
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t vk[32], vv[32];
        tmem_ld32(tbase + lane_off + C::kTdK + 32 * c, vk);
        tmem_ld32(tbase + lane_off + C::kTdV + 32 * c, vv);
        tmem_ld_wait(vk);
        tmem_ld_wait(vv);
        if (key < S) {
          float* dk = a.dK + ((static_cast<int64_t>(b) * S + key) * G + g) * D + 32 * c;
          float* dvp = a.dV + ((static_cast<int64_t>(b) * S + key) * G + g) * D + 32 * c;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            reinterpret_cast<float4*>(dk)[q] =
                make_float4(__uint_as_float(vk[4 * q]), __uint_as_float(vk[4 * q + 1]),
                            __uint_as_float(vk[4 * q + 2]), __uint_as_float(vk[4 * q + 3]));
            reinterpret_cast<float4*>(dvp)[q] =
                make_float4(__uint_as_float(vv[4 * q]), __uint_as_float(vv[4 * q + 1]),
                            __uint_as_float(vv[4 * q + 2]), __uint_as_float(vv[4 * q + 3]));
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tbase, C::kTmemCols);
  }
}

// One warp per row: routed slot (token, group, slot) or shared-head token.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const BwdArgs a) {
  grid_dep_wait();  // launched with launch_pdl
  const int lane = threadIdx.x & 31;
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t T = static_cast<int64_t>(a.B) * a.S;
  const int64_t n_routed = T * a.G * a.k;
  constexpr int E = D / 32;  // elements per lane
  if (wid < n_routed) {
    const int64_t tok = wid / (a.G * a.k);
    const int g = static_cast<int>((wid / a.k) % a.G), j = static_cast<int>(wid % a.k);
    const float* o = a.O_sel + tok * a.out_row_stride + (static_cast<int64_t>(g) * a.k + j) * D;
    const float* dsel =
        a.dO_sel + tok * a.dout_row_stride + (static_cast<int64_t>(g) * a.k + j) * D;
    const float* dbar = a.do_bar + tok * a.dout_row_stride + static_cast<int64_t>(g) * D;
    const float wj = a.w[wid];
    float dd = 0.f, dw = 0.f;
    uint16_t* dst = a.dO_r_out + wid * D;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int c = lane + 32 * e;
      const float ov = o[c], db = dbar[c];
      const float de = fmaf(wj, db, dsel[c]);
      dd = fmaf(de, ov, dd);
      dw = fmaf(db, ov, dw);
      __nv_bfloat16 hb = __float2bfloat16_rn(de);
      dst[c] = *reinterpret_cast<uint16_t*>(&hb);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      dd += __shfl_xor_sync(0xFFFFFFFFu, dd, off);
      dw += __shfl_xor_sync(0xFFFFFFFFu, dw, off);
    }
    if (lane == 0) {
      a.D_r_out[wid] = dd;
      a.dw[wid] = dw;
    }
  } else if (wid < n_routed + T) {
    const int64_t tok = wid - n_routed;
    const float* s = a.s_out + tok * a.out_row_stride;
    const float* dsv = a.ds + tok * a.dout_row_stride;
    uint16_t* dst = a.dO_s_out + tok * D;
    float dd = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int c = lane + 32 * e;
      const float v = dsv[c];
      dd = fmaf(v, s[c], dd);
      __nv_bfloat16 hb = __float2bfloat16_rn(v);
      dst[c] = *reinterpret_cast<uint16_t*>(&hb);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dd += __shfl_xor_sync(0xFFFFFFFFu, dd, off);
    if (lane == 0) a.D_s_out[tok] = dd;
  }
}

}  // namespace

cudaError_t launch_bwd(const BwdArgs& a, cudaStream_t st) {
  const int64_t T = static_cast<int64_t>(a.B) * a.S;
  const int64_t rows = T * a.G * a.k + T;
  const int64_t blocks = (rows * 32 + 255) / 256;
  const int nq = (a.S + kTileM - 1) / kTileM;
  const unsigned grid = static_cast<unsigned>(static_cast<int64_t>(a.B) * a.G * nq);
  cudaError_t e;
  if (a.d == 64) {
    if ((e = launch_pdl(bwd_prep_kernel<64>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st,
                        a)) != cudaSuccess)
      return e;
    if ((e = cudaFuncSetAttribute(bwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  BwdCfg<64>::kSmemBytes)) != cudaSuccess)
      return e;
    e = launch_pdl(bwd_kernel<64>, dim3(grid), dim3(kBwdThreads), BwdCfg<64>::kSmemBytes, st, a);
    if (e != cudaSuccess) return e;
  } else if (a.d == 128) {
    if ((e = launch_pdl(bwd_prep_kernel<128>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st,
                        a)) != cudaSuccess)
      return e;
    if ((e = cudaFuncSetAttribute(bwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  BwdCfg<128>::kSmemBytes)) != cudaSuccess)
      return e;
    e = launch_pdl(bwd_kernel<128>, dim3(grid), dim3(kBwdThreads), BwdCfg<128>::kSmemBytes, st, a);
    if (e != cudaSuccess) return e;
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace gqe
