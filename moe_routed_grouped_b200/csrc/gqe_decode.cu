// Incremental decode step of GQE: one new token per sequence attends its
// cached history ("AI 大模型之 GQA", 工程实操 非方形因果遮罩: query length 1,
// key length the whole history, mask on the absolute position; with padding
// the mask is intersected with key validity, here a first valid slot per
// sequence for left-padded caches).
//
// A decode step reads every cached K/V row of each KV head once and does
// little arithmetic with it, so it is bound by HBM bandwidth, not by the
// tensor cores: the kernels below use plain vector loads and CUDA-core FMAs.
// The cache is split into chunks of keys (split-KV, so that B*G KV heads can
// fill 148 SMs); one CTA serves every selected head of its KV head over its
// chunk, so a cached row crosses HBM once however many heads use it.  Each
// CTA leaves the chunk's softmax state (running max, sum of exponentials,
// unnormalised output) in the workspace; decode_merge_kernel rescales and
// adds the chunks, then writes the routed slots, o_bar and the shared head.
#include <cuda_bf16.h>

#include "gqe_decode.h"
#include "gqe_device.cuh"

namespace gqe {
namespace {

// Running maximum before any visible key.  Finite, so that the first update's
// rescale factor exp2(m_old - m_new) is exp2(0) = 1 or 0, never NaN.
constexpr float kNoKeyMax = -1.0e30f;

__device__ __forceinline__ void unpack_bf16x8(const uint4 r, float (&f)[8]) {
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ void store_out(void* base, int64_t off, float v, int out_fp32) {
  if (out_fp32) {
    static_cast<float*>(base)[off] = v;
  } else {
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    static_cast<__nv_bfloat16*>(base)[off] = h;
  }
}

// Partial attention of one (b, g, chunk) for head slots pass*HB .. pass*HB+HB-1.
// MULTI (n_new > 1): slot r*(k+1) + j belongs to new token r, whose query sits
// at slot pos + r and sees keys up to there; each head slot then carries its
// own causal bound.  Without MULTI every slot is token 0's and the chunk's end
// is its bound.
//
// Lanes: a key row of D bf16 is read by L = D/8 lanes, 16 bytes each, so a
// warp reads 32/L consecutive rows per load; the key slots of the CTA are
// NS = 4 * 32/L rows apart and each takes kDecUnroll keys per step.  A score
// is the L lanes' partial dot products added with xor shuffles (every lane of
// the group ends with the same sum), then each slot keeps its own online
// softmax state per head; the slots are merged through shared memory at the
// end of the chunk.
template <int D, int HB, bool MULTI>
__global__ void __launch_bounds__(kDecThreads, 3) decode_partial_kernel(const DecodeArgs a) {
  grid_dep_wait();  // launched with launch_pdl
  constexpr int L = D / 8;
  constexpr int SPW = 32 / L;
  constexpr int NS = (kDecThreads / 32) * SPW;
  constexpr int U = kDecUnroll;
  __shared__ float sm_m[NS][HB];
  __shared__ float sm_l[NS][HB];
  __shared__ __align__(16) float sm_o[NS][HB][D];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slot = warp * SPW + lane / L;
  const int part = lane % L;

  int64_t unit = blockIdx.x;
  const int c = static_cast<int>(unit % a.nchunks);
  unit /= a.nchunks;
  const int pass = static_cast<int>(unit % a.passes);
  unit /= a.passes;
  const int g = static_cast<int>(unit % a.G);
  const int b = static_cast<int>(unit / a.G);

  // visible keys of sequence b: slots lo..pos + r for new token r (lo > 0
  // with left padding); `last` is the last new token's slot
  const int pos = a.pos[b];
  const int lo = a.kv_start ? a.kv_start[b] : 0;
  const int64_t last = static_cast<int64_t>(pos) + a.n_new - 1;
  if (pos < 0 || last >= a.T || lo < 0 || lo > pos) {
    if (threadIdx.x == 0 && c == 0 && pass == 0 && g == 0)
      latch_status(a.status, GQE_ERR_BAD_POSITION);
    return;
  }
  const int64_t c0 = static_cast<int64_t>(c) * a.chunk;
  if (c0 > last || c0 + a.chunk <= lo) return;  // no visible key here; the merge skips it
  const int64_t t0 = max(c0, static_cast<int64_t>(lo));
  const int64_t t1 = min(c0 + a.chunk, last + 1);

  // this pass's head slots: j < k routed (head g*M + topk_idx), j == k the
  // shared head (KV head 0 only); a slot that is not live is skipped
  const int64_t bg = static_cast<int64_t>(b) * a.G + g;
  float q[HB][8];
  bool live[HB];
  int qpos[HB];  // causal bound of each slot (MULTI)
#pragma unroll
  for (int h = 0; h < HB; ++h) {
    int r = 0, j = pass * HB + h;
    if (MULTI) {
      r = j / (a.k + 1);
      j -= r * (a.k + 1);
    }
    qpos[h] = pos + r;
    const int64_t tr = static_cast<int64_t>(b) * a.n_new + r;  // the token's row
    const uint16_t* qrow = nullptr;
    if (r < a.n_new && j < a.k) {
      const int m = a.topk_idx[(tr * a.G + g) * a.k + j];
      if (m >= 0 && m < a.M)
        qrow = a.Q + (tr * a.N + static_cast<int64_t>(g) * a.M + m) * D;
      else if (threadIdx.x == 0)
        latch_status(a.status, GQE_ERR_BAD_INDEX);
    } else if (r < a.n_new && j == a.k && g == 0) {
      qrow = a.Qs + tr * D;
    }
    live[h] = qrow != nullptr;
    if (live[h]) {
      unpack_bf16x8(__ldg(reinterpret_cast<const uint4*>(qrow + part * 8)), q[h]);
#pragma unroll
      for (int e = 0; e < 8; ++e) q[h][e] *= a.scale_log2;
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) q[h][e] = 0.f;
    }
  }

  float m_run[HB], l_run[HB], o[HB][8];
#pragma unroll
  for (int h = 0; h < HB; ++h) {
    m_run[h] = kNoKeyMax;
    l_run[h] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) o[h][e] = 0.f;
  }

  const int64_t row = static_cast<int64_t>(a.G) * D;  // elements between cached rows
  const uint16_t* kb = a.Kc + (static_cast<int64_t>(b) * a.T * a.G + g) * D + part * 8;
  const uint16_t* vb = a.Vc + (static_cast<int64_t>(b) * a.T * a.G + g) * D + part * 8;

  for (int64_t tb = t0; tb < t1; tb += NS * U) {
    uint4 kr[U], vr[U];
    bool ok[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t t = tb + u * NS + slot;
      ok[u] = t < t1;
      const int64_t tl = ok[u] ? t : t1 - 1;  // masked keys re-read a visible row
      kr[u] = __ldg(reinterpret_cast<const uint4*>(kb + tl * row));
      vr[u] = __ldg(reinterpret_cast<const uint4*>(vb + tl * row));
    }
#pragma unroll
    for (int h = 0; h < HB; ++h) {
      if (!live[h]) continue;  // uniform over the CTA
      float s[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float kf[8];
        unpack_bf16x8(kr[u], kf);
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc = fmaf(q[h][e], kf[e], acc);
#pragma unroll
        for (int off = L / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        bool vis = ok[u];
        if (MULTI) vis = vis && tb + u * NS + slot <= qpos[h];
        s[u] = vis ? acc : -INFINITY;
      }
      float mx = m_run[h];
#pragma unroll
      for (int u = 0; u < U; ++u) mx = fmaxf(mx, s[u]);
      const float alpha = exp2f(m_run[h] - mx);
      m_run[h] = mx;
      float p[U];
      float psum = 0.f;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        p[u] = exp2f(s[u] - mx);
        psum += p[u];
      }
      l_run[h] = fmaf(l_run[h], alpha, psum);
#pragma unroll
      for (int e = 0; e < 8; ++e) o[h][e] *= alpha;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float vf[8];
        unpack_bf16x8(vr[u], vf);
#pragma unroll
        for (int e = 0; e < 8; ++e) o[h][e] = fmaf(p[u], vf[e], o[h][e]);
      }
    }
  }

  // merge the key slots: rescale each to the CTA's maximum and add
#pragma unroll
  for (int h = 0; h < HB; ++h) {
    if (part == 0) {
      sm_m[slot][h] = m_run[h];
      sm_l[slot][h] = l_run[h];
    }
    float4* dst = reinterpret_cast<float4*>(&sm_o[slot][h][part * 8]);
    dst[0] = make_float4(o[h][0], o[h][1], o[h][2], o[h][3]);
    dst[1] = make_float4(o[h][4], o[h][5], o[h][6], o[h][7]);
  }
  __syncthreads();
  for (int qi = threadIdx.x; qi < HB * D; qi += kDecThreads) {
    const int h = qi / D, e = qi % D;
    const int j = pass * HB + h;
    bool use = false;  // live[h], read with constant indices so live[] stays in registers
#pragma unroll
    for (int hh = 0; hh < HB; ++hh)
      if (hh == h) use = live[hh];
    if (!use) continue;
    float mx = kNoKeyMax;
    for (int s = 0; s < NS; ++s) mx = fmaxf(mx, sm_m[s][h]);
    float acc = 0.f, lsum = 0.f;
    for (int s = 0; s < NS; ++s) {
      const float sc = exp2f(sm_m[s][h] - mx);
      acc = fmaf(sm_o[s][h][e], sc, acc);
      lsum = fmaf(sm_l[s][h], sc, lsum);
    }
    const int64_t pi = (bg * a.heads + j) * a.nchunks + c;
    a.part_o[pi * D + e] = acc;
    if (e == 0) {
      a.part_m[pi] = mx;
      a.part_l[pi] = lsum;
    }
  }
}

// Merge of the chunks of one (new token, g): for each live head slot of that
// token, rescale every chunk that holds keys it sees (the partial kernel
// wrote those) to the common maximum, add, normalise; then
// o_bar = sum_j w_j * O_j in slot order (review §二 三个关键部件) and the
// shared head for g = 0.
//
// kMergeSplit groups of D threads (thread e of a group: output element e)
// take the chunks c = c_lo + q, c_lo + q + kMergeSplit, ... of a head, so the
// partial outputs are loaded by several groups at once; the groups' sums are
// then added in group order.  A head's chunk maxima and sums are first staged
// in shared memory by all threads.
constexpr int kMergeSplit = 4;

template <int D>
__global__ void __launch_bounds__(D * kMergeSplit) decode_merge_kernel(const DecodeArgs a) {
  grid_dep_wait();  // launched with launch_pdl
  __shared__ float sm_m[kDecMaxChunks];
  __shared__ float sm_l[kDecMaxChunks];
  __shared__ float sm_acc[kMergeSplit][D];
  __shared__ float sm_lsum[kMergeSplit];
  // one CTA per (new token row, g); row tr = b * n_new + r
  const int g = static_cast<int>(blockIdx.x % a.G);
  const int64_t tr = blockIdx.x / a.G;
  const int b = static_cast<int>(tr / a.n_new);
  const int r = static_cast<int>(tr % a.n_new);
  const int64_t bg = static_cast<int64_t>(b) * a.G + g;  // partials are per (b, g)
  const int64_t rg = tr * a.G + g;                       // router outputs per (row, g)
  const int e = static_cast<int>(threadIdx.x) % D;
  const int q = static_cast<int>(threadIdx.x) / D;
  const int pos = a.pos[b];
  const int lo = a.kv_start ? a.kv_start[b] : 0;
  const bool pos_ok = pos >= 0 && static_cast<int64_t>(pos) + a.n_new - 1 < a.T && lo >= 0 &&
                      lo <= pos;
  const int c_lo = pos_ok ? lo / a.chunk : 0;  // chunks c_lo .. nc-1 hold visible keys
  const int nc = pos_ok ? (pos + r) / a.chunk + 1 : 0;
  const int nh = a.k + (g == 0 ? 1 : 0);
  const float nan = __int_as_float(0x7fc00000);
  const int64_t row = tr * a.out_row_stride;
  float obar = 0.f;
  for (int j = 0; j < nh; ++j) {
    bool ok = pos_ok;
    if (j < a.k) {
      const int m = a.topk_idx[rg * a.k + j];
      ok = ok && m >= 0 && m < a.M;
    }
    const int64_t p0 = (bg * a.heads + static_cast<int64_t>(r) * (a.k + 1) + j) * a.nchunks;
    if (j > 0) __syncthreads();  // the previous head's staged values are read
    if (ok)
      for (int c = c_lo + static_cast<int>(threadIdx.x); c < nc; c += D * kMergeSplit) {
        sm_m[c] = a.part_m[p0 + c];
        sm_l[c] = a.part_l[p0 + c];
      }
    __syncthreads();
    float acc = 0.f, lsum = 0.f;
    if (ok) {
      float mx = kNoKeyMax;
      for (int c = c_lo; c < nc; ++c) mx = fmaxf(mx, sm_m[c]);
      const float* po = a.part_o + p0 * D + e;
#pragma unroll 4
      for (int c = c_lo + q; c < nc; c += kMergeSplit) {
        const float sc = exp2f(sm_m[c] - mx);
        acc = fmaf(po[static_cast<int64_t>(c) * D], sc, acc);
        lsum = fmaf(sm_l[c], sc, lsum);
      }
    }
    sm_acc[q][e] = acc;
    if (e == 0) sm_lsum[q] = lsum;
    __syncthreads();
    if (q == 0) {
      float out = nan;  // a rejected position or expert index yields NaN
      if (ok) {
        float at = 0.f, lt = 0.f;
#pragma unroll
        for (int i = 0; i < kMergeSplit; ++i) {
          at += sm_acc[i][e];
          lt += sm_lsum[i];
        }
        out = at / lt;
      }
      if (j < a.k) {
        store_out(a.O_sel, row + (static_cast<int64_t>(g) * a.k + j) * D + e, out, a.out_fp32);
        obar = fmaf(a.w[rg * a.k + j], out, obar);
      } else {
        store_out(a.s_out, row + e, out, a.out_fp32);
      }
    }
  }
  if (q == 0) store_out(a.o_bar, row + static_cast<int64_t>(g) * D + e, obar, a.out_fp32);
}

template <int D, int HB, bool MULTI>
cudaError_t launch_decode_dh(const DecodeArgs& a, cudaStream_t st) {
  const int64_t ctas = static_cast<int64_t>(a.B) * a.G * a.passes * a.nchunks;
  cudaError_t e = launch_pdl(decode_partial_kernel<D, HB, MULTI>, dim3(static_cast<unsigned>(ctas)),
                             dim3(kDecThreads), 0, st, a);
  if (e != cudaSuccess) return e;
  const int64_t rows = static_cast<int64_t>(a.B) * a.n_new * a.G;
  return launch_pdl(decode_merge_kernel<D>, dim3(static_cast<unsigned>(rows)),
                    dim3(D * kMergeSplit), 0, st, a);
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st) {
  if (a.nchunks < 1 || a.nchunks > kDecMaxChunks) return cudaErrorInvalidValue;
  if (a.n_new > 1) {  // several new tokens: per-slot causal bounds
    if (a.d == 64) return launch_decode_dh<64, kDecHeads, true>(a, st);
    if (a.d == 128) return launch_decode_dh<128, kDecHeads, true>(a, st);
    return cudaErrorInvalidValue;
  }
  // two head slots cover k = 1 (a routed head, plus the shared one for g = 0)
  const bool narrow = a.heads <= 2;
  if (a.d == 64)
    return narrow ? launch_decode_dh<64, 2, false>(a, st)
                  : launch_decode_dh<64, kDecHeads, false>(a, st);
  if (a.d == 128)
    return narrow ? launch_decode_dh<128, 2, false>(a, st)
                  : launch_decode_dh<128, kDecHeads, false>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace gqe
