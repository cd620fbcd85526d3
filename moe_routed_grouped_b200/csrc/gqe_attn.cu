// Causal flash attention on the sm_100a tensor cores for GQE prefill.
//
// One CTA computes one work item: 128 query rows against every KV tile they
// can see.  Three kinds of rows share the kernel:
//   routed  - the rows of one (batch, group, expert) bucket: the tokens whose
//             router picked query head h = g*M + m ("论文综述：分组查询专家"
//             §二 路由器), gathered by token index; they attend KV head g;
//   shared  - 128 consecutive tokens of the always-on shared head (§二 三个
//             关键部件), KV head 0;
//   dense   - 128 consecutive tokens of one query head h, KV head
//             floor(h / M) ("AI 大模型之 GQA", 技术深化: the explicit head map).
// K and V are read straight from the group's KV head; nothing is repeated.
// The causal rule is applied on absolute token positions (key <= query,
// "AI 大模型之 GQA" 工程实操), so gathered rows mask correctly and KV tiles past
// the last row's position are never visited.
//
// Warp roles (192 threads):
//   warps 0-3  softmax + epilogue; thread r owns query row r (TMEM lane r)
//   warp 4     producer: Q gather (cp.async) or TMA tile load; K/V via TMA
//   warp 5     TMEM owner and single-thread tcgen05.mma issuer
// TMEM: S = Q.K^T (128 fp32 columns), P (fp16, 64 columns), O (d columns).
// Per KV tile j: S_j = Q K_j^T (UMMA, smem x smem) -> softmax warps read S_j,
// release it, exponentiate, write P_j to TMEM -> O += P_j V_j (UMMA, A from
// TMEM).  Q.K^T of tile j+1 runs while the softmax of tile j is computed.
// The running max is only moved when it grows by more than 2^8, so O is
// rescaled rarely; the final division by the row sum makes this exact.
#include <atomic>

#include "gqe_device.cuh"

namespace gqe {
namespace {

template <int D>
struct Cfg {
  static constexpr int kStages = 2;
  static constexpr int kAtom = kTileM * 128;          // 128 rows x 128 B (64 elements)
  static constexpr int kQBytes = kTileM * D * 2;
  static constexpr int kKVBytes = kTileN * D * 2;
  static constexpr int kSmemQ = 0;
  static constexpr int kSmemK = kQBytes;
  static constexpr int kSmemV = kSmemK + kStages * kKVBytes;
  static constexpr int kSmemBar = kSmemV + kStages * kKVBytes;
  static constexpr int kSmemBytes = kSmemBar + 256 + 1024;  // barriers + alignment slack
  static constexpr uint32_t kTmemS = 0, kTmemP = 128, kTmemO = (D == 64 ? 192 : 256);
  static constexpr uint32_t kTmemCols = (D == 64 ? 256 : 512);
  static constexpr int kMinBlocks = (D == 64 ? 2 : 1);
  static constexpr uint32_t kIdescQK = make_idesc_f16(kTileM, kTileN, /*bf16*/ 1, 0, 0);
  static constexpr uint32_t kIdescPV = make_idesc_f16(kTileM, D, /*f16*/ 0, 0, /*MN*/ 1);
};

constexpr int kThreads = 192;
// Of every 8 column pairs, this many are exponentiated by a polynomial on the
// FMA pipe; the rest use the MUFU ex2 unit (16 lanes/clock/SM), which would
// otherwise bound d = 64 attention at about half the tensor-core rate.
constexpr int kPolyPairs = 2;
// The pair kernel runs the longest calls (K/V beyond L2, S around 1M), where
// the GPU sits at its power limit and clocks down: there the polynomial's
// extra instructions cost more than the MUFU time they save, and one pair in
// 8 is the measured optimum (A/B at S = 1M: 0 / 1 / 2 / 3 pairs took
// 1.92 / 1.87 / 2.01 / 2.16 s for the routed call).
constexpr int kPairPolyPairs = 1;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;

// barrier slots
enum {
  kBarQFull = 0,
  kBarKFull = 1,   // +stage
  kBarKEmpty = 3,  // +stage
  kBarVFull = 5,   // +stage
  kBarVEmpty = 7,  // +stage
  kBarSFull = 9,
  kBarSFree = 10,
  kBarPFull = 11,
  kBarODone = 12,
  kBarSpare = 13,
  kNumBars = 14
};

struct Waiter {
  volatile int* abort;
  int* status;
  uint64_t limit;
  __device__ bool operator()(uint64_t* bar, uint32_t parity) const {
    return mbar_wait(bar, parity, abort, status, limit);
  }
};

// ---------------------------------------------------------------------------
// The online softmax of one KV tile for the thread's query row (TMEM lane).
//
// S_j (128 fp32 columns) is read from TMEM into registers and released at
// once, so the MMA warp can start S_{j+1} = Q K_{j+1}^T while this tile is
// exponentiated.  P_j = 2^(S_j * scale * log2(e) - m) replaces S_j in the
// registers and is packed to fp16; it goes back to TMEM for the P.V product
// only after all of its exponentials, so the wait for the previous tile's
// P.V (which reads P from the same TMEM columns) comes that late.  m is the
// running maximum in log2 units, moved only when a tile's maximum exceeds it
// by more than 8 (so P <= 2^8 always fits fp16), which makes O rescales rare;
// the final division by the row sum l makes the result exact whatever m was
// used.
constexpr float kRescaleThreshold = 8.f;

__device__ __forceinline__ void tile_load_s(uint32_t taddr, uint32_t (&sv)[4][32]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) tmem_ld32(taddr + 32 * c, sv[c]);
#pragma unroll
  for (int c = 0; c < 4; ++c) tmem_ld_wait(sv[c]);
}

// Key t is visible to a row at absolute position pos iff kvs <= t <= pos.
// The causal part: columns past lim = pos - kbase are masked (one compare
// with a constant column index per element).
__device__ __forceinline__ void tile_mask_causal(uint32_t (&sv)[4][32], int lim) {
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int e = 0; e < 32; ++e)
      if (32 * c + e > lim) sv[c][e] = __float_as_uint(-INFINITY);
}
// The first-valid-slot part (left padding): columns before first are masked;
// only the tile that holds kv_start needs it.
__device__ __forceinline__ void tile_mask_below(uint32_t (&sv)[4][32], int first) {
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int e = 0; e < 32; ++e)
      if (32 * c + e < first) sv[c][e] = __float_as_uint(-INFINITY);
}

// Row maximum of the raw scores: 8 independent chains of 3-input max.
__device__ __forceinline__ float tile_max(const uint32_t (&sv)[4][32]) {
  float mxp[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) mxp[q] = -INFINITY;
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int e = 0; e < 32; e += 2)
      mxp[(e >> 1) & 7] = fmax3f(mxp[(e >> 1) & 7], __uint_as_float(sv[c][e]),
                                 __uint_as_float(sv[c][e + 1]));
  return fmax3f(fmax3f(mxp[0], mxp[1], mxp[2]), fmax3f(mxp[3], mxp[4], mxp[5]),
                fmaxf(mxp[6], mxp[7]));
}

// p = 2^(s * sl2 - m), packed to fp16 pairs into pk; returns the sum of the p.
// kPoly of every 8 column pairs go to the FMA-pipe polynomial.
template <int kPoly>
__device__ __forceinline__ float tile_exp(const uint32_t (&sv)[4][32], float sl2, float m,
                                          uint32_t (&pk)[4][16]) {
  const uint64_t sl2x2 = f2_pack(sl2, sl2), negm2 = f2_pack(-m, -m);
  uint64_t rs2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
  for (int c = 0; c < 4; ++c) {
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const uint64_t y2 =
          f2_fma(f2_pack(__uint_as_float(sv[c][e]), __uint_as_float(sv[c][e + 1])), sl2x2, negm2);
      float p0, p1;
      if (((e >> 1) & 7) < kPoly) {  // this pair on the FMA pipe
        exp2_poly_pair(y2, p0, p1);
      } else {                             // this pair on the MUFU unit
        float y0, y1;
        f2_unpack(y2, y0, y1);
        p0 = ex2_approx(y0);
        p1 = ex2_approx(y1);
      }
      rs2[(e >> 1) & 3] = f2_add(rs2[(e >> 1) & 3], f2_pack(p0, p1));
      pk[c][e / 2] = pack_half2(p0, p1);
    }
  }
  float r0, r1, r2, r3, r4, r5, r6, r7;
  f2_unpack(rs2[0], r0, r1);
  f2_unpack(rs2[1], r2, r3);
  f2_unpack(rs2[2], r4, r5);
  f2_unpack(rs2[3], r6, r7);
  return ((r0 + r1) + (r2 + r3)) + ((r4 + r5) + (r6 + r7));
}

// TMEM addresses and barriers of one 128-row tile's softmax.
struct SoftmaxCtx {
  uint32_t tS, tP, tO;  // this warp's lane quarter of S, P and O
  uint64_t *s_full, *s_free, *o_done, *p_full;
};

// One KV tile j of a softmax warp; returns false when a wait gave up (the
// lanes agree, as the tcgen05 instructions that follow are warp-collective).
// A row that has seen no visible key yet (all padding) keeps m = -inf and
// l = 0: its exponentials are taken against 0, which gives P = 0.
template <int D, int kPoly>
__device__ __forceinline__ bool softmax_tile(const SoftmaxCtx& x, const Waiter& wait, int j,
                                             bool diag, int kbase, int pos, int kvs, float sl2,
                                             float& m_used, float& l) {
  const int lane = threadIdx.x & 31;
  if (!__all_sync(0xFFFFFFFFu, wait(x.s_full, j & 1))) return false;
  tc_fence_after();
  uint32_t sv[4][32];
  tile_load_s(x.tS, sv);
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(x.s_free);  // S_j is in registers: S_{j+1} may start
  if (diag) tile_mask_causal(sv, pos - kbase);
  if (kbase < kvs) tile_mask_below(sv, kvs - kbase);
  float factor = 1.f;
  const float mnew = fmaxf(m_used, tile_max(sv) * sl2);  // j = 0: m_used = -inf, factor 0
  if (mnew - m_used > kRescaleThreshold) {
    factor = ex2_approx(m_used - mnew);
    m_used = mnew;
  }
  // P in fp16: 64 registers, 64 TMEM columns for the 128 keys
  uint32_t pk[4][16];
  l = l * factor + tile_exp<kPoly>(sv, sl2, m_used == -INFINITY ? 0.f : m_used, pk);
  // P.V of the previous tile must be done before P and O are touched
  if (j > 0) {
    if (!__all_sync(0xFFFFFFFFu, wait(x.o_done, (j - 1) & 1))) return false;
    tc_fence_after();
    if (__any_sync(0xFFFFFFFFu, factor != 1.f)) {  // rare: rescale O
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        tmem_ld32(x.tO + 32 * c, ov);
        tmem_ld_wait(ov);
#pragma unroll
        for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * factor);
        tmem_st32(x.tO + 32 * c, ov);
      }
    }
  }
#pragma unroll
  for (int c = 0; c < 4; ++c) tmem_st16(x.tP + 16 * c, pk[c]);
  tmem_st_wait();
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(x.p_full);
  return true;
}

// One query row of a routed tile: row r of the token's Q head, copied with
// cp.async into the 128-byte swizzle the UMMA descriptor expects (16-byte
// chunk c of row r at c ^ (r & 7)); zero-filled when the row is past the
// bucket's end.  Each softmax thread copies its own row, so the 128 rows are
// in flight at once; the copies are complete and visible to the tensor core
// when this returns.
template <int D, int kAtom>
__device__ __forceinline__ void gather_q_row(uint8_t* sQ, int r, const uint16_t* src, bool valid) {
#pragma unroll
  for (int c = 0; c < D / 8; ++c) {
    const int atom = c >> 3, ch = c & 7;
    cp_async_16(sQ + atom * kAtom + r * 128 + ((ch ^ (r & 7)) << 4), src + c * 8,
                valid ? 16u : 0u);
  }
  cp_async_wait_all();
  fence_proxy_async_smem();
}

// Output rows of one softmax warp: lane l holds query row l of the warp's
// TMEM lane quarter (O at taddr_o), its 1/l scale and its destination(s)
// (null: not stored).  The rows are normalised into shared memory (32 rows
// of D + 4 floats: conflict-free for both access patterns below) and then
// written row by row with consecutive lanes on consecutive 16-byte pieces, so
// each store instruction covers whole 128-byte segments of one or a few rows
// instead of 32 scattered pieces.
template <int D>
__device__ __noinline__ void store_rows_coalesced(float* stage, uint32_t taddr_o, float inv,
                                               uint8_t* dst, uint8_t* dst2, bool fp32) {
  constexpr int kStr = D + 4;
  const int lane = threadIdx.x & 31;
  float* mine = stage + lane * kStr;
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    uint32_t ov[32];
    tmem_ld32(taddr_o + 32 * c, ov);
    tmem_ld_wait(ov);
#pragma unroll
    for (int q = 0; q < 8; ++q)
      reinterpret_cast<float4*>(mine + 32 * c)[q] =
          make_float4(__uint_as_float(ov[4 * q]) * inv, __uint_as_float(ov[4 * q + 1]) * inv,
                      __uint_as_float(ov[4 * q + 2]) * inv, __uint_as_float(ov[4 * q + 3]) * inv);
  }
  __syncwarp();
  const unsigned long long d1 = reinterpret_cast<unsigned long long>(dst);
  const unsigned long long d2 = reinterpret_cast<unsigned long long>(dst2);
  if (fp32) {
    constexpr int kLanesPerRow = D / 4;  // 16-byte pieces of 4 floats
    constexpr int kRows = 32 / kLanesPerRow;
    const int sub = lane / kLanesPerRow, piece = lane % kLanesPerRow;
#pragma unroll 4
    for (int r0 = 0; r0 < 32; r0 += kRows) {
      const int row = r0 + sub;
      float4* o1 = reinterpret_cast<float4*>(__shfl_sync(0xFFFFFFFFu, d1, row));
      float4* o2 = reinterpret_cast<float4*>(__shfl_sync(0xFFFFFFFFu, d2, row));
      const float4 v = reinterpret_cast<const float4*>(stage + row * kStr)[piece];
      if (o1) o1[piece] = v;
      if (o2) o2[piece] = v;
    }
  } else {
    constexpr int kLanesPerRow = D / 8;  // 16-byte pieces of 8 bf16
    constexpr int kRows = 32 / kLanesPerRow;
    const int sub = lane / kLanesPerRow, piece = lane % kLanesPerRow;
#pragma unroll 4
    for (int r0 = 0; r0 < 32; r0 += kRows) {
      const int row = r0 + sub;
      uint4* o1 = reinterpret_cast<uint4*>(__shfl_sync(0xFFFFFFFFu, d1, row));
      uint4* o2 = reinterpret_cast<uint4*>(__shfl_sync(0xFFFFFFFFu, d2, row));
      const float4* src = reinterpret_cast<const float4*>(stage + row * kStr + 8 * piece);
      const float4 x0 = src[0], x1 = src[1];
      const float f[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
        w[e] = *reinterpret_cast<uint32_t*>(&h);
      }
      const uint4 v = make_uint4(w[0], w[1], w[2], w[3]);
      if (o1) o1[piece] = v;
      if (o2) o2[piece] = v;
    }
  }
  __syncwarp();
}

template <int D>
__global__ void __launch_bounds__(kThreads, Cfg<D>::kMinBlocks)
    attn_kernel(const __grid_constant__ AttnArgs a) {
  grid_dep_wait();  // launched with launch_pdl
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.S, N = a.N, G = a.G, M = a.M;

  // ---------------------------------------------------------- work item
  int kind, b, h = 0, g = 0, m = 0, row0, nrows, nkv, bstart = 0;
  if (a.dense) {
    const int nq = (S + kTileM - 1) / kTileM;
    const int64_t bn = static_cast<int64_t>(a.B) * N;
    const int64_t t = blockIdx.x;
    const int qt = nq - 1 - static_cast<int>(t / bn);
    const int bh = static_cast<int>(t % bn);
    kind = kDense;
    b = bh / N;
    h = bh % N;
    g = h / M;
    row0 = qt * kTileM;
    nrows = min(kTileM, S - row0);
    nkv = qt + 1;
  } else {
    // the list holds at least gridDim.x entries: read the entry and the count
    // together rather than one after the other
    const int count = *a.tile_count;
    const TileDesc td = a.tiles[blockIdx.x];
    if (static_cast<int>(blockIdx.x) >= count) return;
    if (td.nkv == 0) return;  // empty second half of a pair
    kind = td.code >> 24;
    const int id = td.code & 0xFFFFFF;
    if (kind == kRouted) {
      b = id / (G * M);
      g = (id / M) % G;
      m = id % M;
      h = g * M + m;
      bstart = a.bucket_off[id];
    } else {
      b = id;
      g = 0;  // the shared head reads KV head 0
    }
    row0 = td.row0;
    nrows = td.nrows;
    nkv = td.nkv;
  }
  // chunked prefill: absolute position of query row 0 and the first valid
  // KV slot of this sequence (0, 0 without offsets); KV tiles are visited
  // from the one that holds kv_start on
  int qoff = 0, kvs = 0;
  if (!a.dense) seq_offsets(a.q_off, a.kv_start, b, S, a.T, a.status, &qoff, &kvs);
  const int j0 = kvs / kTileN;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kSmemBar);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + kNumBars + 1);
  const Waiter wait{abort_flag, a.status, a.wait_limit_ns};

  if (threadIdx.x == 0) {
    // routed Q rows are gathered by the 4 softmax warps, other Q tiles by TMA
    mbar_init(&bars[kBarQFull], kind == kRouted ? 4 : 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&bars[kBarKFull + s], 1);
      mbar_init(&bars[kBarKEmpty + s], 1);
      mbar_init(&bars[kBarVFull + s], 1);
      mbar_init(&bars[kBarVEmpty + s], 1);
    }
    mbar_init(&bars[kBarSFull], 1);
    mbar_init(&bars[kBarSFree], 4);
    mbar_init(&bars[kBarPFull], 4);
    mbar_init(&bars[kBarODone], 1);
    mbar_init(&bars[kBarSpare], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&a.tmK);
    tma_prefetch_desc(&a.tmV);
    tma_prefetch_desc(kind == kDense ? &a.tmQ : &a.tmQs);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------ producer
    uint8_t* sQ = smem + C::kSmemQ;
    if (kind != kRouted && lane == 0) {
      mbar_arrive_expect_tx(&bars[kBarQFull], C::kQBytes);
#pragma unroll
      for (int atom = 0; atom < D / 64; ++atom) {
        if (kind == kDense)
          tma_load_4d(sQ + atom * C::kAtom, &a.tmQ, &bars[kBarQFull], atom * 64, h, row0, b);
        else
          tma_load_3d(sQ + atom * C::kAtom, &a.tmQs, &bars[kBarQFull], atom * 64, row0, b);
      }
    }
    if (lane == 0) {
      int issued = 0;
      for (int j = 0; j < nkv; ++j) {
        const int s = j & 1;
        const uint32_t round = static_cast<uint32_t>(j >> 1);
        if (round > 0 && !wait(&bars[kBarKEmpty + s], (round - 1) & 1)) break;
        mbar_arrive_expect_tx(&bars[kBarKFull + s], C::kKVBytes);
#pragma unroll
        for (int atom = 0; atom < D / 64; ++atom)
          tma_load_4d(smem + C::kSmemK + s * C::kKVBytes + atom * C::kAtom, &a.tmK,
                      &bars[kBarKFull + s], atom * 64, g, (j0 + j) * kTileN, b);
        if (round > 0 && !wait(&bars[kBarVEmpty + s], (round - 1) & 1)) {
          issued = 2 * j + 1;
          break;
        }
        mbar_arrive_expect_tx(&bars[kBarVFull + s], C::kKVBytes);
#pragma unroll
        for (int atom = 0; atom < D / 64; ++atom)
          tma_load_4d(smem + C::kSmemV + s * C::kKVBytes + atom * C::kAtom, &a.tmV,
                      &bars[kBarVFull + s], atom * 64, g, (j0 + j) * kTileN, b);
        issued = 2 * j + 2;
      }
      if (*abort_flag) {
        // let the copies already in flight land before the CTA exits
        const int nk = (issued + 1) / 2, nv = issued / 2;
        for (int q = max(0, nk - 2); q < nk; ++q)
          mbar_wait(&bars[kBarKFull + (q & 1)], (q >> 1) & 1, nullptr, a.status, a.wait_limit_ns);
        for (int q = max(0, nv - 2); q < nv; ++q)
          mbar_wait(&bars[kBarVFull + (q & 1)], (q >> 1) & 1, nullptr, a.status, a.wait_limit_ns);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t tS = tbase + C::kTmemS, tP = tbase + C::kTmemP, tO = tbase + C::kTmemO;
      const uint32_t qaddr = smem_u32(smem + C::kSmemQ);
      auto issue_pv = [&](int jj) -> bool {
        const int s = jj & 1;
        if (!wait(&bars[kBarPFull], jj & 1)) return false;
        if (!wait(&bars[kBarVFull + s], (jj >> 1) & 1)) return false;
        tc_fence_after();
        const uint32_t vaddr = smem_u32(smem + C::kSmemV + s * C::kKVBytes);
#pragma unroll
        for (int kk = 0; kk < kTileN / 16; ++kk)
          umma_ts(tO, tP + kk * 8, make_sdesc_sw128(vaddr + kk * 2048, C::kAtom, 1024),
                  C::kIdescPV, (jj > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&bars[kBarODone]);
        tc_commit(&bars[kBarVEmpty + s]);
        return true;
      };
      bool ok = wait(&bars[kBarQFull], 0);
      tc_fence_after();
      for (int j = 0; ok && j < nkv; ++j) {
        const int s = j & 1;
        if (!wait(&bars[kBarKFull + s], (j >> 1) & 1)) { ok = false; break; }
        if (j > 0 && !wait(&bars[kBarSFree], (j - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t kaddr = smem_u32(smem + C::kSmemK + s * C::kKVBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kAtom + (kk & 3) * 32;
          umma_ss(tS, make_sdesc_sw128(qaddr + off, 16, 1024),
                  make_sdesc_sw128(kaddr + off, 16, 1024), C::kIdescQK, kk > 0 ? 1u : 0u);
        }
        tc_commit(&bars[kBarSFull]);
        tc_commit(&bars[kBarKEmpty + s]);
        if (j > 0 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok) ok = issue_pv(nkv - 1);
      if (!ok) {
        // drain whatever was issued before giving up
        tc_commit(&bars[kBarSpare]);
        mbar_wait(&bars[kBarSpare], 0, nullptr, a.status, a.wait_limit_ns);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------ softmax warps
    const int r = warp * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const int rv = min(r, nrows - 1);
    int pos, pos_first, slot = 0;
    if (kind == kRouted) {
      pos = a.bucket_tok[bstart + row0 + rv];
      pos_first = a.bucket_tok[bstart + row0];
      gather_q_row<D, C::kAtom>(smem + C::kSmemQ, r,
                                a.Q + ((static_cast<int64_t>(b) * S + pos) * N + h) * D,
                                r < nrows);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBarQFull]);
      // the row's output slot (rank of expert m among its selections), read
      // now so the epilogue does not wait for it
      const int32_t* sel = a.topk_idx + ((static_cast<int64_t>(b) * S + pos) * G + g) * a.k;
      for (int q = 0; q < a.k; ++q)
        if (sel[q] == m) slot = q;
    } else {
      pos = row0 + rv;
      pos_first = row0;
    }
    const int apos = qoff + pos, apos_first = qoff + pos_first;  // absolute positions
    const float sl2 = a.scale_log2;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    const SoftmaxCtx sx{tbase + lane_off + C::kTmemS, tbase + lane_off + C::kTmemP,
                        tbase + lane_off + C::kTmemO, &bars[kBarSFull], &bars[kBarSFree],
                        &bars[kBarODone], &bars[kBarPFull]};
    for (int j = 0; j < nkv; ++j) {
      const int kbase = (j0 + j) * kTileN;
      const bool diag = kbase + kTileN - 1 > apos_first;
      if (!softmax_tile<D, kPolyPairs>(sx, wait, j, diag, kbase, apos, kvs, sl2, m_used, l)) {
        ok = false;
        break;
      }
    }
    if (ok) ok = wait(&bars[kBarODone], (nkv - 1) & 1);
    ok = __all_sync(0xFFFFFFFFu, ok);
    const bool fp32 = a.out_fp32 != 0;
    const size_t esz = fp32 ? 4 : 2;
    uint8_t* dst = nullptr;
    uint8_t* dst2 = nullptr;
    if (ok && r < nrows) {
      const int64_t tokrow = static_cast<int64_t>(b) * S + pos;
      if (kind == kDense) {
        dst = static_cast<uint8_t*>(a.O_dense) + ((tokrow * N + h) * D) * esz;
      } else if (kind == kShared) {
        dst = static_cast<uint8_t*>(a.s_out) + (tokrow * a.out_row_stride) * esz;
      } else {
        dst = static_cast<uint8_t*>(a.O_sel) +
              (tokrow * a.out_row_stride + static_cast<int64_t>(g * a.k + slot) * D) * esz;
        if (a.k == 1)
          dst2 = static_cast<uint8_t*>(a.o_bar) +
                 (tokrow * a.out_row_stride + static_cast<int64_t>(g) * D) * esz;
        if (a.lse_sel) a.lse_sel[(tokrow * G + g) * a.k + slot] = m_used + log2f(l);
      }
      if (kind == kShared && a.lse_s) a.lse_s[tokrow] = m_used + log2f(l);
    }
    if (ok) {
      tc_fence_after();
      // every product is done, so the K/V stages are free for the staging rows
      float* stage = reinterpret_cast<float*>(smem + C::kSmemK) + warp * 32 * (D + 4);
      // a padding row (no visible key) has l = 0 and is written as zeros
      store_rows_coalesced<D>(stage, tbase + lane_off + C::kTmemO, l > 0.f ? 1.f / l : 0.f, dst,
                              dst2, fp32);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tbase, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// d = 64, long sequences: the pair kernel.  One CTA (one per SM: it takes
// all 512 TMEM columns) computes TWO 128-row tiles that read the same KV
// head: two expert buckets of one (batch, group) or two query tiles of the
// shared head.  Each K/V tile is loaded once for both, which halves the K/V
// traffic.  That matters once K and V
// no longer fit in L2: CTAs that start at different times sweep the KV
// sequence at different offsets, so each tile read by attn_kernel comes from
// DRAM (at S = 1M the launch is bound by HBM bandwidth).  While K and V fit
// in L2 attn_kernel is faster (two independent CTAs per SM).  Dense calls
// keep attn_kernel: their query-tile-major order already lets the CTAs that
// run together share K/V tiles in L2.
// Warp roles (352 threads):
//   warps 0-3 / 4-7  softmax + epilogue of tile 0 / tile 1 (thread = row)
//   warp 8           producer: Q of both tiles, then K/V via TMA (3 stages)
//   warps 9 / 10     tcgen05.mma issuer of tile 0 / tile 1 (warp 9 owns TMEM)
// A K/V stage is refilled once both issuers are done with it, so the two
// tiles run independently within the depth of the stage ring.
// TMEM: tile s at column 256*s: S (128 fp32), P (128 fp16 = 64), O (64).
struct PairCfg {
  static constexpr int D = 64;
  static constexpr int kStages = 3;
  static constexpr int kAtom = kTileM * 128;
  static constexpr int kQBytes = kTileM * D * 2;
  static constexpr int kKVBytes = kTileN * D * 2;
  static constexpr int kSmemQ = 0;  // two Q tiles
  static constexpr int kSmemK = 2 * kQBytes;
  static constexpr int kSmemV = kSmemK + kStages * kKVBytes;
  // output staging: 8 softmax warps x 32 rows x (D + 4) floats
  static constexpr int kSmemStage = kSmemV + kStages * kKVBytes;
  static constexpr int kSmemBar = kSmemStage + 8 * 32 * (D + 4) * 4;
  static constexpr int kSmemBytes = kSmemBar + 256 + 1024;  // barriers + alignment slack
  static constexpr uint32_t kTmemSlot = 256, kTmemS = 0, kTmemP = 128, kTmemO = 192;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kIdescQK = make_idesc_f16(kTileM, kTileN, /*bf16*/ 1, 0, 0);
  static constexpr uint32_t kIdescPV = make_idesc_f16(kTileM, D, /*f16*/ 0, 0, /*MN*/ 1);
};
constexpr int kPairThreads = 352;
constexpr int kPairProducerWarp = 8;
constexpr int kPairMmaWarp = 9;

enum {
  kPbQFull = 0,    // +tile
  kPbKFull = 2,    // +stage
  kPbKEmpty = 5,   // +stage
  kPbVFull = 8,    // +stage
  kPbVEmpty = 11,  // +stage
  kPbSFull = 14,   // +tile
  kPbSFree = 16,   // +tile
  kPbPFull = 18,   // +tile
  kPbODone = 20,   // +tile
  kPbSpare = 22,   // +tile
  kPbNum = 24
};

struct Slot {
  int kind, b, h, g, m, row0, nrows, nkv, bstart;
};

__device__ __forceinline__ Slot decode_tile(const TileDesc& td, const AttnArgs& a) {
  Slot t{};
  t.nkv = td.nkv;
  if (td.nkv == 0) return t;
  t.kind = td.code >> 24;
  const int id = td.code & 0xFFFFFF;
  if (t.kind == kRouted) {
    t.b = id / (a.G * a.M);
    t.g = (id / a.M) % a.G;
    t.m = id % a.M;
    t.h = t.g * a.M + t.m;
    t.bstart = a.bucket_off[id];
  } else {
    t.b = id;
    t.g = 0;  // the shared head reads KV head 0
  }
  t.row0 = td.row0;
  t.nrows = td.nrows;
  return t;
}

__global__ void __launch_bounds__(kPairThreads, 1)
    attn_pair_kernel(const __grid_constant__ AttnArgs a) {
  grid_dep_wait();  // launched with launch_pdl
  using C = PairCfg;
  constexpr int D = C::D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.S, N = a.N, G = a.G;

  // ---------------------------------------------------------- work item
  Slot sl[2];
  {
    if (2 * static_cast<int>(blockIdx.x) >= *a.tile_count) return;
    sl[0] = decode_tile(a.tiles[2 * blockIdx.x], a);
    sl[1] = decode_tile(a.tiles[2 * blockIdx.x + 1], a);
    if (sl[0].nkv == 0) return;
    if (sl[1].nkv > 0 && (sl[1].b != sl[0].b || sl[1].g != sl[0].g || sl[1].nkv > sl[0].nkv)) {
      // not a valid pair (the scheduler writes none): refuse the second tile
      if (threadIdx.x == 0) latch_status(a.status, GQE_ERR_CUDA);
      sl[1].nkv = 0;
    }
  }
  const int b = sl[0].b, g = sl[0].g, nkv0 = sl[0].nkv;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kSmemBar);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + kPbNum);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + kPbNum + 1);
  const Waiter wait{abort_flag, a.status, a.wait_limit_ns};

  if (threadIdx.x == 0) {
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[kPbQFull + s], sl[s].kind == kRouted ? 4 : 1);
      mbar_init(&bars[kPbSFull + s], 1);
      mbar_init(&bars[kPbSFree + s], 4);
      mbar_init(&bars[kPbPFull + s], 4);
      mbar_init(&bars[kPbODone + s], 1);
    }
#pragma unroll
    for (int st = 0; st < C::kStages; ++st) {
      mbar_init(&bars[kPbKFull + st], 1);
      mbar_init(&bars[kPbKEmpty + st], 2);
      mbar_init(&bars[kPbVFull + st], 1);
      mbar_init(&bars[kPbVEmpty + st], 2);
    }
    mbar_init(&bars[kPbSpare], 1);
    mbar_init(&bars[kPbSpare + 1], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kPairMmaWarp) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == kPairProducerWarp && lane == 0) {
    tma_prefetch_desc(&a.tmK);
    tma_prefetch_desc(&a.tmV);
    tma_prefetch_desc(&a.tmQs);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;

  if (warp == kPairProducerWarp) {
    // ------------------------------------------------------ producer
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const Slot t = sl[s];
      if (t.nkv == 0) continue;
      uint8_t* sQ = smem + C::kSmemQ + s * C::kQBytes;
      if (t.kind != kRouted && lane == 0) {  // routed rows: gathered by the softmax warps
        mbar_arrive_expect_tx(&bars[kPbQFull + s], C::kQBytes);
        tma_load_3d(sQ, &a.tmQs, &bars[kPbQFull + s], 0, t.row0, t.b);
      }
    }
    if (lane == 0) {
      int nk = 0, nv = 0;  // K and V loads issued
      for (int j = 0; j < nkv0; ++j) {
        const int st = j % C::kStages;
        const uint32_t round = static_cast<uint32_t>(j / C::kStages);
        if (round > 0 && !wait(&bars[kPbKEmpty + st], (round - 1) & 1)) break;
        mbar_arrive_expect_tx(&bars[kPbKFull + st], C::kKVBytes);
        tma_load_4d(smem + C::kSmemK + st * C::kKVBytes, &a.tmK, &bars[kPbKFull + st], 0, g,
                    j * kTileN, b);
        ++nk;
        if (round > 0 && !wait(&bars[kPbVEmpty + st], (round - 1) & 1)) break;
        mbar_arrive_expect_tx(&bars[kPbVFull + st], C::kKVBytes);
        tma_load_4d(smem + C::kSmemV + st * C::kKVBytes, &a.tmV, &bars[kPbVFull + st], 0, g,
                    j * kTileN, b);
        ++nv;
      }
      if (*abort_flag) {
        // let the copies still in flight land before the CTA exits
        for (int s = 0; s < 2; ++s)
          if (sl[s].nkv > 0 && sl[s].kind != kRouted)
            mbar_wait(&bars[kPbQFull + s], 0, nullptr, a.status, a.wait_limit_ns);
        for (int q = max(0, nk - C::kStages); q < nk; ++q)
          mbar_wait(&bars[kPbKFull + q % C::kStages], (q / C::kStages) & 1, nullptr, a.status,
                    a.wait_limit_ns);
        for (int q = max(0, nv - C::kStages); q < nv; ++q)
          mbar_wait(&bars[kPbVFull + q % C::kStages], (q / C::kStages) & 1, nullptr, a.status,
                    a.wait_limit_ns);
      }
    }
  } else if (warp == kPairMmaWarp || warp == kPairMmaWarp + 1) {
    // ------------------------------------------------------ MMA issuers
    // one thread per tile: S_s = Q_s K_j^T, then O_s += P_s V_{j-1}.  Each K/V
    // stage is released when both tiles are done with it; the shorter tile
    // releases the longer one's remaining stages as they arrive.
    const int s = warp - kPairMmaWarp;
    const int nk = s ? sl[1].nkv : sl[0].nkv;
    if (lane == 0) {
      const uint32_t tS = tbase + s * C::kTmemSlot + C::kTmemS;
      const uint32_t tP = tbase + s * C::kTmemSlot + C::kTmemP;
      const uint32_t tO = tbase + s * C::kTmemSlot + C::kTmemO;
      const uint32_t qaddr = smem_u32(smem + C::kSmemQ) + s * C::kQBytes;
      auto issue_pv = [&](int jj) -> bool {
        const int st = jj % C::kStages;
        if (!wait(&bars[kPbVFull + st], (jj / C::kStages) & 1)) return false;
        if (!wait(&bars[kPbPFull + s], jj & 1)) return false;
        tc_fence_after();
        const uint32_t vaddr = smem_u32(smem + C::kSmemV + st * C::kKVBytes);
#pragma unroll
        for (int kk = 0; kk < kTileN / 16; ++kk)
          umma_ts(tO, tP + kk * 8, make_sdesc_sw128(vaddr + kk * 2048, C::kAtom, 1024),
                  C::kIdescPV, (jj > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&bars[kPbODone + s]);
        tc_commit(&bars[kPbVEmpty + st]);
        return true;
      };
      bool ok = nk == 0 || wait(&bars[kPbQFull + s], 0);
      tc_fence_after();
      for (int j = 0; ok && j < nk; ++j) {
        const int st = j % C::kStages;
        if (!wait(&bars[kPbKFull + st], (j / C::kStages) & 1)) { ok = false; break; }
        if (j > 0 && !wait(&bars[kPbSFree + s], (j - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t kaddr = smem_u32(smem + C::kSmemK + st * C::kKVBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_ss(tS, make_sdesc_sw128(qaddr + kk * 32, 16, 1024),
                  make_sdesc_sw128(kaddr + kk * 32, 16, 1024), C::kIdescQK, kk > 0 ? 1u : 0u);
        tc_commit(&bars[kPbSFull + s]);
        tc_commit(&bars[kPbKEmpty + st]);
        if (j > 0 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok && nk > 0) ok = issue_pv(nk - 1);
      for (int j = nk; ok && j < nkv0; ++j) {  // stages only the other tile uses
        const int st = j % C::kStages;
        if (!wait(&bars[kPbKFull + st], (j / C::kStages) & 1)) { ok = false; break; }
        mbar_arrive(&bars[kPbKEmpty + st]);
        if (!wait(&bars[kPbVFull + st], (j / C::kStages) & 1)) { ok = false; break; }
        mbar_arrive(&bars[kPbVEmpty + st]);
      }
      if (!ok) {
        // drain whatever was issued before giving up
        tc_commit(&bars[kPbSpare + s]);
        mbar_wait(&bars[kPbSpare + s], 0, nullptr, a.status, a.wait_limit_ns);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------ softmax warps
    const int s = warp >> 2, quarter = warp & 3;
    const Slot t = s ? sl[1] : sl[0];
    if (t.nkv > 0) {
      const int r = quarter * 32 + lane;
      const uint32_t tsl = tbase + (static_cast<uint32_t>(quarter * 32) << 16) + s * C::kTmemSlot;
      const int rv = min(r, t.nrows - 1);
      int pos, pos_first;
      if (t.kind == kRouted) {
        pos = a.bucket_tok[t.bstart + t.row0 + rv];
        pos_first = a.bucket_tok[t.bstart + t.row0];
        gather_q_row<D, C::kAtom>(smem + C::kSmemQ + s * C::kQBytes, r,
                                  a.Q + ((static_cast<int64_t>(t.b) * S + pos) * N + t.h) * D,
                                  r < t.nrows);
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kPbQFull + s]);
      } else {
        pos = t.row0 + rv;
        pos_first = t.row0;
      }
      const float sl2 = a.scale_log2;
      float m_used = -INFINITY, l = 0.f;
      bool ok = true;
      const SoftmaxCtx sx{tsl + C::kTmemS, tsl + C::kTmemP, tsl + C::kTmemO, &bars[kPbSFull + s],
                          &bars[kPbSFree + s], &bars[kPbODone + s], &bars[kPbPFull + s]};
      for (int j = 0; j < t.nkv; ++j) {
        const int kbase = j * kTileN;
        if (!softmax_tile<D, kPairPolyPairs>(sx, wait, j, kbase + kTileN - 1 > pos_first, kbase,
                                             pos, 0, sl2, m_used, l)) {
          ok = false;
          break;
        }
      }
      ok = __all_sync(0xFFFFFFFFu, ok && wait(&bars[kPbODone + s], (t.nkv - 1) & 1));
      const bool fp32 = a.out_fp32 != 0;
      const size_t esz = fp32 ? 4 : 2;
      uint8_t* dst = nullptr;
      uint8_t* dst2 = nullptr;
      if (ok && r < t.nrows) {
        const int64_t tokrow = static_cast<int64_t>(t.b) * S + pos;
        if (t.kind == kShared) {
          dst = static_cast<uint8_t*>(a.s_out) + (tokrow * a.out_row_stride) * esz;
        } else {
          const int32_t* sel = a.topk_idx + (tokrow * G + t.g) * a.k;
          int slot = 0;
          for (int q = 0; q < a.k; ++q)
            if (sel[q] == t.m) slot = q;
          dst = static_cast<uint8_t*>(a.O_sel) +
                (tokrow * a.out_row_stride + static_cast<int64_t>(t.g * a.k + slot) * D) * esz;
          if (a.k == 1)
            dst2 = static_cast<uint8_t*>(a.o_bar) +
                   (tokrow * a.out_row_stride + static_cast<int64_t>(t.g) * D) * esz;
          if (a.lse_sel) a.lse_sel[(tokrow * G + t.g) * a.k + slot] = m_used + log2f(l);
        }
        if (t.kind == kShared && a.lse_s) a.lse_s[tokrow] = m_used + log2f(l);
      }
      if (ok) {
        tc_fence_after();
        // K/V stages may still feed the other tile: stage in this warp's own region
        float* stage = reinterpret_cast<float*>(smem + C::kSmemStage) + warp * 32 * (D + 4);
        store_rows_coalesced<D>(stage, tsl + C::kTmemO, l > 0.f ? 1.f / l : 0.f, dst, dst2,
                                fp32);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kPairMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tbase, C::kTmemCols);
  }
}

__global__ void selftest_wait_kernel(int* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // nothing ever arrives on `bar`: the wait must give up by itself
  mbar_wait(&bar, 0, &abort_flag, status, limit_ns);
}

template <int D>
cudaError_t launch_d(const AttnArgs& a, int64_t grid, cudaStream_t st) {
  static int configured_device = -1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (configured_device != dev) {
    e = cudaFuncSetAttribute(attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg<D>::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  return launch_pdl(attn_kernel<D>, dim3(static_cast<unsigned>(grid)), dim3(kThreads),
                    Cfg<D>::kSmemBytes, st, a);
}

// K/V working set (bytes) from which the d = 64 calls use the pair kernel:
// below about 3/4 of the 126 MB L2 the K/V tiles are served from L2 and
// attn_kernel is faster.
std::atomic<int64_t> g_pair_min_kv_bytes{int64_t(96) << 20};

cudaError_t launch_pair(const AttnArgs& a, int64_t grid, cudaStream_t st) {
  static int configured_device = -1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (configured_device != dev) {
    e = cudaFuncSetAttribute(attn_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             PairCfg::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  return launch_pdl(attn_pair_kernel, dim3(static_cast<unsigned>(grid)), dim3(kPairThreads),
                    PairCfg::kSmemBytes, st, a);
}

}  // namespace

int64_t set_pair_threshold(int64_t kv_bytes) { return g_pair_min_kv_bytes.exchange(kv_bytes); }

bool pair_kernel_for(const gqe_dims& d) {
  if (d.d != 64) return false;
  // K (bf16) and V (fp16) of every KV head the call reads
  const int64_t kv_bytes = static_cast<int64_t>(d.B) * d.S * d.G * d.d * 4;
  const int64_t thr = g_pair_min_kv_bytes.load();
  return thr >= 0 && kv_bytes >= thr;
}

cudaError_t launch_attention(const AttnArgs& a, int64_t n_list, cudaStream_t st) {
  const int64_t nq = (a.S + kTileM - 1) / kTileM;
  if (a.d == 64) {
    if (a.pair && !a.dense) {
      const int64_t grid = n_list / 2;
      return grid > 0 ? launch_pair(a, grid, st) : cudaSuccess;
    }
    const int64_t grid = a.dense ? static_cast<int64_t>(a.B) * a.N * nq : n_list;
    return grid > 0 ? launch_d<64>(a, grid, st) : cudaSuccess;
  }
  if (a.d == 128) {
    const int64_t grid = a.dense ? static_cast<int64_t>(a.B) * a.N * nq : n_list;
    return grid > 0 ? launch_d<128>(a, grid, st) : cudaSuccess;
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_selftest_wait(int* status, uint64_t limit_ns, cudaStream_t st) {
  selftest_wait_kernel<<<1, 32, 0, st>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace gqe
