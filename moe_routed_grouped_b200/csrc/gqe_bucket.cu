// Bucketing, work-list scheduling, V conversion and the k>1 combine.
//
// bucket_body: one CTA per (batch, group).  Each token appears once in each
// of the k buckets its router picked ("论文综述：分组查询专家" §二 路由器:
// only the selected heads compute), so the (b, g) block of the token list has
// the fixed size S*k and starts at (b*G + g)*S*k; the per-expert offsets are
// a scan local to the CTA.  The scatter is a stable counting sort built from
// warp ballots, so each bucket lists its tokens in ascending position, which
// the attention kernel needs for causal tile skipping ("AI 大模型之 GQA",
// 工程实操: the mask is decided on absolute positions).
#include "gqe_device.cuh"

namespace gqe {
namespace {

constexpr int kBucketThreads = 1024;
constexpr int kBucketWarps = kBucketThreads / 32;

__device__ void bucket_body(const BucketArgs& a, int bg) {
  __shared__ int cnt[kMaxM];
  __shared__ int start[kMaxM];
  __shared__ int running[kMaxM];
  __shared__ int wcnt[kMaxM][kBucketWarps];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = bg / a.G, g = bg % a.G;
  const int S = a.S, G = a.G, M = a.M, k = a.k;
  const int64_t base = static_cast<int64_t>(bg) * S * k;
  if (tid < kMaxM) {
    cnt[tid] = 0;
    running[tid] = 0;
  }
  __syncthreads();

  // phase 1: bucket sizes (warp-aggregated counts)
  bool bad = false;
  for (int i0 = 0; i0 < S; i0 += kBucketThreads) {
    const int i = i0 + tid;
    uint32_t mine = 0;
    if (i < S) {
      const int32_t* row = a.topk_idx + ((static_cast<int64_t>(b) * S + i) * G + g) * k;
      for (int j = 0; j < k; ++j) {
        const int m = row[j];
        if (m < 0 || m >= M) bad = true;
        else mine |= 1u << m;
      }
    }
    for (int m = 0; m < M; ++m) {
      const uint32_t bal = __ballot_sync(0xFFFFFFFFu, (mine >> m) & 1u);
      if (lane == 0 && bal) atomicAdd(&cnt[m], __popc(bal));
    }
  }
  if (bad) latch_status(a.status, GQE_ERR_BAD_INDEX);
  __syncthreads();
  if (tid == 0) {
    int s = 0;
    for (int m = 0; m < M; ++m) {
      start[m] = s;
      s += cnt[m];
    }
  }
  __syncthreads();
  if (tid < M) a.bucket_off[bg * M + tid] = static_cast<int32_t>(base + start[tid]);
  if (bg == a.B * a.G - 1 && tid == 0)
    a.bucket_off[a.B * a.G * M] = static_cast<int32_t>(static_cast<int64_t>(a.B) * G * S * k);

  // phase 2: stable scatter, one chunk of 1024 tokens at a time
  for (int i0 = 0; i0 < S; i0 += kBucketThreads) {
    const int i = i0 + tid;
    uint32_t mine = 0;  // bit m set if this token picked expert m
    if (i < S) {
      const int32_t* row = a.topk_idx + ((static_cast<int64_t>(b) * S + i) * G + g) * k;
      for (int j = 0; j < k; ++j) {
        const int m = row[j];
        if (m >= 0 && m < M) mine |= 1u << m;
      }
    }
    for (int m = 0; m < M; ++m) {
      const uint32_t bal = __ballot_sync(0xFFFFFFFFu, (mine >> m) & 1u);
      if (lane == 0) wcnt[m][warp] = __popc(bal);
    }
    __syncthreads();
    if (tid < M) {
      int s = running[tid];
      for (int w = 0; w < kBucketWarps; ++w) {
        const int c = wcnt[tid][w];
        wcnt[tid][w] = s;
        s += c;
      }
      running[tid] = s;
    }
    __syncthreads();
    const uint32_t lt = (1u << lane) - 1u;
    for (int m = 0; m < M; ++m) {
      const uint32_t bal = __ballot_sync(0xFFFFFFFFu, (mine >> m) & 1u);
      if ((mine >> m) & 1u) {
        const int r = wcnt[m][warp] + __popc(bal & lt);
        a.bucket_tok[base + start[m] + r] = i;
      }
    }
    __syncthreads();
  }

  // routed work items: ceil(cnt/128) tiles per expert; unused slots get nkv 0
  TileDesc* slots = a.tiles_raw + static_cast<int64_t>(bg) * a.cap_bg;
  int qo, kvs;
  seq_offsets(a.q_off, a.kv_start, b, S, a.T, a.status, &qo, &kvs);
  const int j0 = kvs / kTileN;
  if (!a.pairs) {
    int first = 0;
    for (int m = 0; m < M; ++m) {
      const int nt = (cnt[m] + kTileM - 1) / kTileM;
      for (int t = tid; t < nt; t += kBucketThreads) {
        const int row0 = t * kTileM;
        const int nrows = min(kTileM, cnt[m] - row0);
        const int last = a.bucket_tok[base + start[m] + row0 + nrows - 1];
        TileDesc d;
        d.code = (kRouted << 24) | (bg * M + m);
        d.row0 = row0;
        d.nrows = nrows;
        // KV tiles from the one of kv_start to the last row's; at least one,
        // so rows that are all padding are still written (as zeros)
        d.nkv = max(1, (qo + last) / kTileN + 1 - j0);
        slots[first + t] = d;
      }
      first += nt;
    }
    for (int t = first + tid; t < a.cap_bg; t += kBucketThreads) slots[t] = TileDesc{0, 0, 0, 0};
    return;
  }
  // For the pair kernel the (b, g) block's tiles are placed in descending nkv
  // order, a stable merge of the M per-expert lists (each ascending, as the
  // bucket lists ascending positions), so that neighbours 2p, 2p+1 form a
  // pair of nearly equal length.
  __shared__ int tfirst[kMaxM + 1];
  if (tid == 0) {
    int s = 0;
    for (int m = 0; m < M; ++m) {
      tfirst[m] = s;
      s += (cnt[m] + kTileM - 1) / kTileM;
    }
    tfirst[M] = s;
  }
  __syncthreads();
  const int ntiles = tfirst[M];
  const int32_t* tok = a.bucket_tok + base;
  auto tile_nkv = [&](int m, int t) {
    return max(1, (qo + tok[start[m] + min(t * kTileM + kTileM - 1, cnt[m] - 1)]) / kTileN + 1 - j0);
  };
  for (int i = tid; i < ntiles; i += kBucketThreads) {
    int m = 0;
    while (i >= tfirst[m + 1]) ++m;
    const int t = i - tfirst[m];
    const int v = tile_nkv(m, t);
    // ascending position under the key (nkv, m, t): t tiles of expert m come
    // first, then, from every other expert, those with smaller nkv (or equal
    // nkv and smaller m), found by binary search
    int asc = t;
    for (int m2 = 0; m2 < M; ++m2) {
      if (m2 == m) continue;
      int lo = 0, hi = tfirst[m2 + 1] - tfirst[m2];
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        const int w = tile_nkv(m2, mid);
        if (m2 < m ? w <= v : w < v) lo = mid + 1;
        else hi = mid;
      }
      asc += lo;
    }
    const int row0 = t * kTileM;
    TileDesc d;
    d.code = (kRouted << 24) | (bg * M + m);
    d.row0 = row0;
    d.nrows = min(kTileM, cnt[m] - row0);
    d.nkv = v;
    slots[ntiles - 1 - asc] = d;
  }
  for (int t = ntiles + tid; t < a.cap_bg; t += kBucketThreads) slots[t] = TileDesc{0, 0, 0, 0};
}

// One CTA: the shared head's tiles are appended (for the pair kernel in
// pairs: query tiles q and q-1 of one batch), then the work items (tiles, or
// pairs by the KV-tile count of their first tile) are sorted longest first,
// so the heaviest work starts first and the grid's tail is short.  Counting
// sort on nkv in [1, ceil(T/128)].
constexpr int kSchedThreads = 1024;

__device__ void schedule_body(const BucketArgs& a, int* hist /* ceil(T/128) + 2 bins */) {
  const int tid = threadIdx.x;
  const int nq = (a.S + kTileM - 1) / kTileM;
  const int nq2 = nq + (nq & 1);
  const int nkv_max = (a.T + kTileN - 1) / kTileN;
  const int64_t n_routed = static_cast<int64_t>(a.B) * a.G * a.cap_bg;
  TileDesc* shared_tiles = a.tiles_raw + n_routed;
  for (int v = tid; v < nkv_max + 2; v += kSchedThreads) hist[v] = 0;
  // the shared head's tiles: every token, KV head 0; slot i of a batch holds
  // query tile nq-1-i (so pair i/2 is tiles nq-1-2(i/2) and nq-2-2(i/2))
  for (int64_t t = tid; t < static_cast<int64_t>(a.B) * nq2; t += kSchedThreads) {
    const int b = static_cast<int>(t / nq2), q = nq - 1 - static_cast<int>(t % nq2);
    TileDesc d{0, 0, 0, 0};
    if (q >= 0) {
      int qo, kvs;
      seq_offsets(a.q_off, a.kv_start, b, a.S, a.T, a.status, &qo, &kvs);
      d.code = (kShared << 24) | b;
      d.row0 = q * kTileM;
      d.nrows = min(kTileM, a.S - q * kTileM);
      d.nkv = max(1, (qo + d.row0 + d.nrows - 1) / kTileN + 1 - kvs / kTileN);
    }
    shared_tiles[t] = d;
  }
  __syncthreads();
  const int per = a.pairs ? 2 : 1;  // list entries per work item
  const int64_t nitems = a.n_raw_tiles / per;
  for (int64_t p = tid; p < nitems; p += kSchedThreads) {
    const int v = a.tiles_raw[per * p].nkv;
    if (v > 0) atomicAdd(&hist[v], 1);
  }
  __syncthreads();
  if (tid == 0) {  // exclusive scan from the largest nkv down
    int s = 0;
    for (int v = nkv_max; v >= 1; --v) {
      const int c = hist[v];
      hist[v] = s;
      s += c;
    }
    *a.tile_count = per * s;
  }
  __syncthreads();
  for (int64_t p = tid; p < nitems; p += kSchedThreads) {
    const TileDesc d0 = a.tiles_raw[per * p];
    if (d0.nkv > 0) {
      const int64_t dst = atomicAdd(&hist[d0.nkv], 1);
      a.tiles[per * dst] = d0;
      if (per == 2) a.tiles[2 * dst + 1] = a.tiles_raw[2 * p + 1];
    }
  }
}

// V (bf16) -> fp16 for the P.V product; P is rounded to fp16 (11-bit
// significand), which is what keeps the output within 1e-3 relative L2.
__device__ void convert_v_body(const ConvertArgs& a, int block, int nblocks) {
  const int64_t n8 = a.n / 8;
  bool bad = false;
  for (int64_t i = block * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<int64_t>(nblocks) * blockDim.x) {
    const uint4 v = reinterpret_cast<const uint4*>(a.V)[i];
    const uint32_t in[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float lo = __uint_as_float(in[q] << 16);
      const float hi = __uint_as_float(in[q] & 0xFFFF0000u);
      bad |= !(fabsf(lo) <= 65504.f) || !(fabsf(hi) <= 65504.f);
      out[q] = pack_half2(lo, hi);
    }
    reinterpret_cast<uint4*>(a.V16)[i] = make_uint4(out[0], out[1], out[2], out[3]);
  }
  if (bad) latch_status(a.status, GQE_ERR_NONFINITE);
}

// One launch for the work that precedes attention: CTAs [0, B*G) bucket one
// (batch, group) each, the remaining CTAs convert V to fp16, and the CTA that
// finishes last (fenced counter) sorts the work list.
__global__ void __launch_bounds__(kBucketThreads)
    prep_kernel(const BucketArgs a, const ConvertArgs cv, int with_schedule) {
  grid_dep_wait();  // launched with launch_pdl
  extern __shared__ int hist[];
  __shared__ int is_last;
  const int nbucket = a.B * a.G;
  if (static_cast<int>(blockIdx.x) < nbucket)
    bucket_body(a, blockIdx.x);
  else
    convert_v_body(cv, blockIdx.x - nbucket, gridDim.x - nbucket);
  if (!with_schedule) return;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(a.done, 1) == static_cast<int>(gridDim.x) - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  schedule_body(a, hist);
  if (threadIdx.x == 0) *a.done = 0;  // ready for the next call
}

__global__ void convert_v_kernel(const ConvertArgs a) {
  grid_dep_wait();  // launched with launch_pdl
  convert_v_body(a, blockIdx.x, gridDim.x);
}

// o_bar[t, g] = sum_j w[t, g, j] * O_sel[t, g, j] in slot order
// (review §二 三个关键部件, the renormalised weighted-sum slot); k > 1 only.
__global__ void combine_kernel(const CombineArgs a) {
  grid_dep_wait();  // launched with launch_pdl
  const int lanes_per_row = a.d / 4;  // 4 elements per thread
  const int64_t rows = static_cast<int64_t>(a.T) * a.G;
  const int64_t tid = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t q = tid; q < rows * lanes_per_row; q += nthreads) {
    const int64_t row = q / lanes_per_row;
    const int c = static_cast<int>(q % lanes_per_row) * 4;
    const int64_t t = row / a.G;
    const int g = static_cast<int>(row % a.G);
    const float* wr = a.w + row * a.k;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < a.k; ++j) {
      const int64_t off = t * a.out_row_stride + static_cast<int64_t>(g * a.k + j) * a.d + c;
      float v[4];
      if (a.out_fp32) {
        const float4 f = *reinterpret_cast<const float4*>(static_cast<const float*>(a.O_sel) + off);
        v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
      } else {
        const uint2 h = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(a.O_sel) + off);
        v[0] = __uint_as_float(h.x << 16); v[1] = __uint_as_float(h.x & 0xFFFF0000u);
        v[2] = __uint_as_float(h.y << 16); v[3] = __uint_as_float(h.y & 0xFFFF0000u);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[e] = fmaf(wr[j], v[e], acc[e]);
    }
    const int64_t off = t * a.out_row_stride + static_cast<int64_t>(g) * a.d + c;
    if (a.out_fp32) {
      *reinterpret_cast<float4*>(static_cast<float*>(a.o_bar) + off) =
          make_float4(acc[0], acc[1], acc[2], acc[3]);
    } else {
      __nv_bfloat162 lo = __floats2bfloat162_rn(acc[0], acc[1]);
      __nv_bfloat162 hi = __floats2bfloat162_rn(acc[2], acc[3]);
      uint2 h;
      h.x = *reinterpret_cast<uint32_t*>(&lo);
      h.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(static_cast<uint16_t*>(a.o_bar) + off) = h;
    }
  }
}

}  // namespace

cudaError_t launch_prep(const BucketArgs& a, const ConvertArgs* cv, bool with_schedule,
                        cudaStream_t st) {
  const int nkv_max = (a.T + kTileN - 1) / kTileN;
  const size_t smem = with_schedule ? sizeof(int) * (nkv_max + 2) : 0;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  int nconv = 0;
  ConvertArgs c{};
  if (cv) {
    c = *cv;
    // the conversion CTAs take the slots the bucket CTAs leave free (two
    // 1024-thread CTAs per SM), so the launch runs in one wave
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t n8 = c.n / 8;
    const int slots = 2 * sms, nb = a.B * a.G;
    const int cap = nb < slots - slots / 4 ? slots - nb : slots / 4;
    nconv = static_cast<int>((n8 + kBucketThreads - 1) / kBucketThreads);
    if (nconv > cap) nconv = cap;
    if (nconv < 1) nconv = 1;
  }
  return launch_pdl(prep_kernel, dim3(a.B * a.G + nconv), dim3(kBucketThreads), smem, st, a, c,
                    with_schedule ? 1 : 0);
}

cudaError_t launch_convert_v(const ConvertArgs& a, cudaStream_t st) {
  const int64_t n8 = a.n / 8;
  int64_t blocks = (n8 + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  return launch_pdl(convert_v_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, a);
}

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t st) {
  const int64_t work = static_cast<int64_t>(a.T) * a.G * (a.d / 4);
  int64_t blocks = (work + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  return launch_pdl(combine_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, a);
}

}  // namespace gqe
