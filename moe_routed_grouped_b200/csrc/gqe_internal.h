// Internal declarations shared by the GQE kernels and the C-ABI layer.
#pragma once

#include <utility>

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/gqe.h"

namespace gqe {

constexpr int kTileM = 128;      // query rows per attention tile (UMMA M)
constexpr int kTileN = 128;      // keys per KV tile (UMMA N of Q.K^T)
constexpr int kMaxM = 32;        // experts per group supported
constexpr uint64_t kWaitLimitNs = 4000000000ull;  // 4 s per bounded wait

// Tile kinds of the attention work list.
enum TileKind : int { kRouted = 0, kShared = 1, kDense = 2 };

// One attention work item: 128 query rows against the keys they can see.
//   code  = (kind << 24) | id   (routed: bucket (b*G+g)*M+m; shared: b)
//   row0  = first row inside the bucket (routed) or first token (shared)
//   nrows = valid rows (1..128); nkv = KV tiles to visit (0 = empty slot)
// For the pair kernel (d = 64, K and V larger than L2) the work list holds
// tiles in pairs (entries 2p, 2p+1) of the same batch and KV head, the first
// with the larger nkv; the second may be empty.  A pair is one CTA, which
// loads each K/V tile once for both.  Otherwise it is a list of single tiles.
struct TileDesc {
  int32_t code, row0, nrows, nkv;
};

// Work-list capacity: routed tile slots per (b, g) and the list length
// (routed slots, then the shared head's tiles), both even so pairs align.
inline void tile_list_dims(int64_t B, int64_t S, int64_t G, int64_t M, int64_t k,
                           int64_t* cap_bg, int64_t* n_raw_tiles) {
  const int64_t nq = (S + kTileM - 1) / kTileM;
  const int64_t c = (S * k + kTileM - 1) / kTileM + M;
  *cap_bg = c + (c & 1);
  *n_raw_tiles = B * G * *cap_bg + B * (nq + (nq & 1));
}

// Byte offsets of the regions inside the caller's workspace.
struct WsLayout {
  size_t status;      // int32 status word (latched errors)
  size_t counters;    // int32[16]: [0] exact router decisions (cumulative),
                      // [1] tile count, [2] prep-kernel completion counter
  size_t fix_list;    // int32[B*S*G]: (token*G + g) pairs needing exact routing
  size_t wt;          // float32 [d_model][G*M]: W_r transposed for the router
  size_t wsq;         // float32 [ceil(d_model/32)][G*M]: partial column sums of squares of W_r
  size_t v16;         // fp16 [B,S,G,d]: V converted for the P.V product
  size_t bucket_off;  // int32[B*G*M + 1]
  size_t bucket_tok;  // int32[B*G*S*k]
  size_t tiles_raw;   // TileDesc[n_raw_tiles], in pairs
  size_t tiles;       // TileDesc[n_raw_tiles]: pairs sorted by nkv, descending
  size_t total;
  int64_t cap_bg;       // routed tile slots per (b, g), even
  int64_t n_raw_tiles;  // B*G*cap_bg + B*nq rounded up to even (routed + shared)
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// T: KV slots per sequence (the V conversion's size); S when not chunked.
inline WsLayout make_ws_layout(const gqe_dims& d, int64_t T = -1) {
  WsLayout L{};
  const int64_t B = d.B, S = d.S, G = d.G, M = d.N / d.G, k = d.k, hd = d.d;
  if (T < S) T = S;
  tile_list_dims(B, S, G, M, k, &L.cap_bg, &L.n_raw_tiles);
  size_t off = 0;
  L.status = off;     off += 256;
  L.counters = off;   off += 256;
  L.fix_list = off;   off = align_up(off + sizeof(int32_t) * B * S * G, 256);
  L.wt = off;         off = align_up(off + sizeof(float) * d.d_model * G * M, 256);
  L.wsq = off;        off = align_up(off + sizeof(float) * ((d.d_model + 31) / 32) * G * M, 256);
  L.v16 = off;        off = align_up(off + sizeof(uint16_t) * B * T * G * hd, 256);
  L.bucket_off = off; off = align_up(off + sizeof(int32_t) * (B * G * M + 1), 256);
  L.bucket_tok = off; off = align_up(off + sizeof(int32_t) * B * G * S * k, 256);
  L.tiles_raw = off;  off = align_up(off + sizeof(TileDesc) * L.n_raw_tiles, 256);
  L.tiles = off;      off = align_up(off + sizeof(TileDesc) * L.n_raw_tiles, 256);
  L.total = off;
  return L;
}

// ------------------------------------------------------------ launchers
struct RouteArgs {
  const uint16_t* x;    // bf16 [T, dm]
  const uint16_t* Wr;   // bf16 [G, dm, M]
  float* wt;            // float32 [dm][G*M] (written by the prep kernel)
  float* wsq;           // float32 [ceil(dm/32)][G*M] (partial sums by route_prep_kernel)
  const float* bias;    // [G*M] or null
  int32_t* topk_idx;    // [T, G, k]
  float* p;             // [T, G, M]
  float* w;             // [T, G, k]
  int32_t* fix_list;
  int32_t* fix_count;
  int* status;
  int T, dm, G, M, k;
  int tok;              // tokens per route_kernel tile (set by the launcher)
};
// Launch with programmatic stream serialization: the kernel's CTAs may start
// as the previous kernel's CTAs retire; the kernel must call grid_dep_wait()
// before it touches global memory.
template <typename... Params, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

cudaError_t launch_route(const RouteArgs& a, cudaStream_t st);
// 1: the shared-memory-resident router whenever it fits; 0: by token count;
// negative: no change.  Returns the previous setting.
int set_route_force_resident(int on);

// Chunked prefill over a cache: query row i of sequence b sits at absolute
// position q_off[b] + i of a KV sequence of T slots, and sees slots
// kv_start[b]..q_off[b] + i ("AI 大模型之 GQA", 工程实操: the causal mask on
// absolute positions, intersected with key validity).  Null arrays mean 0.
// A value outside its range (q_off not in [0, T - S], kv_start not in
// [0, T)) latches GQE_ERR_BAD_POSITION and is taken as 0.
__device__ __forceinline__ void seq_offsets(const int32_t* q_off, const int32_t* kv_start, int b,
                                            int S, int T, int* status, int* qo, int* kvs) {
  int o = q_off ? q_off[b] : 0, v = kv_start ? kv_start[b] : 0;
  if (o < 0 || o > T - S) {
    atomicCAS(status, 0, GQE_ERR_BAD_POSITION);
    o = 0;
  }
  if (v < 0 || v >= T) {
    atomicCAS(status, 0, GQE_ERR_BAD_POSITION);
    v = 0;
  }
  *qo = o;
  *kvs = v;
}

struct BucketArgs {
  const int32_t* topk_idx;  // [B,S,G,k]
  int32_t* bucket_off;      // [B*G*M+1]
  int32_t* bucket_tok;      // [B*G*S*k]
  TileDesc* tiles_raw;      // routed slots then shared-head tiles
  TileDesc* tiles;          // sorted output
  int32_t* tile_count;
  int32_t* done;            // CTA completion counter (self-resetting)
  int* status;
  int B, S, G, M, k;
  int pairs;                // 1: build the paired list of the pair kernel
  int64_t cap_bg;
  int64_t n_raw_tiles;
  // chunked prefill (see seq_offsets); T = S and null arrays otherwise.  A
  // tile's nkv is then the number of KV tiles it visits, from the tile of
  // kv_start[b] on.
  const int32_t* q_off;
  const int32_t* kv_start;
  int T;
};

struct ConvertArgs {
  const uint16_t* V;  // bf16
  uint16_t* V16;      // fp16
  int64_t n;          // elements (multiple of 8)
  int* status;
};
// Bucketing (+ optional V conversion and work-list sort) in one launch.
cudaError_t launch_prep(const BucketArgs& a, const ConvertArgs* cv, bool with_schedule,
                        cudaStream_t st);
cudaError_t launch_convert_v(const ConvertArgs& a, cudaStream_t st);

struct AttnArgs {
  CUtensorMap tmK;    // bf16 K  [B,S,G,d]   box {64,1,128,1}
  CUtensorMap tmV;    // fp16 V  [B,S,G,d]   box {64,1,128,1}
  CUtensorMap tmQ;    // bf16 Q  [B,S,N,d]   box {64,1,128,1}   (dense tiles)
  CUtensorMap tmQs;   // bf16 Qs [B,S,d]     box {64,128,1}     (shared tiles)
  const uint16_t* Q;  // for the routed row gather
  const int32_t* bucket_off;
  const int32_t* bucket_tok;
  const int32_t* topk_idx;
  const TileDesc* tiles;      // pairs, sorted
  const int32_t* tile_count;  // list entries in use (2 x pairs)
  void* O_sel;
  void* o_bar;
  void* s_out;
  void* O_dense;
  int64_t out_row_stride;
  int* status;
  int B, S, N, G, M, k, d;
  int out_fp32;
  const int32_t* q_off;     // chunked prefill (see seq_offsets); null: 0
  const int32_t* kv_start;  // null: 0
  int T;                    // KV slots per sequence (K/V maps are [B, T, G, d])
  float* lse_sel;           // optional [B,S,G,k]: base-2 log-sum-exp of the scaled
  float* lse_s;             //   scores per routed slot / shared row (for the backward)
  int dense;          // 1: dense GQA tiles from blockIdx; 0: routed/shared list
  int pair;           // 1: the pair kernel on a paired list (d = 64 only)
  float scale_log2;   // log2(e) / sqrt(d)
  uint64_t wait_limit_ns;
};
// n_list: length of the work list (routed/shared); unused for dense tiles.
cudaError_t launch_attention(const AttnArgs& a, int64_t n_list, cudaStream_t st);

// Backward of the routed prefill (gqe_bwd.cu).
struct BwdArgs {
  CUtensorMap tmK;          // bf16 K [B,S,G,d], box {64,1,128,1}
  CUtensorMap tmV;          // bf16 V [B,S,G,d]
  const uint16_t* Q;        // bf16 [B,S,N,d]
  const uint16_t* Qs;       // bf16 [B,S,d]
  const int32_t* topk_idx;  // [B,S,G,k]
  const float* w;           // [B,S,G,k]
  const int32_t* bucket_off;
  const int32_t* bucket_tok;
  // forward outputs (float32 concat rows at out_row_stride) and statistics
  const float* O_sel;       // slot j of group g at (g*k + j)*d
  const float* s_out;
  int64_t out_row_stride;
  const float* lse_sel;     // [B,S,G,k] base-2 log-sum-exp of the scaled scores
  const float* lse_s;       // [B,S]
  // upstream gradients (float32 rows at dout_row_stride, the concat layout)
  const float* dO_sel;
  const float* do_bar;
  const float* ds;
  int64_t dout_row_stride;
  // workspace: effective dO of the slots and of the shared head, and D
  uint16_t* dO_r_out;       // [B,S,G,k,d] bf16 (written by the prep kernel)
  const uint16_t* dO_r;
  float* D_r_out;           // [B,S,G,k]
  const float* D_r;
  uint16_t* dO_s_out;       // [B,S,d] bf16
  const uint16_t* dO_s;
  float* D_s_out;           // [B,S]
  const float* D_s;
  // gradients (float32): dQ and dQs accumulated atomically (zeroed first)
  float* dQ;                // [B,S,N,d]
  float* dQs;               // [B,S,d]
  float* dK;                // [B,S,G,d]
  float* dV;                // [B,S,G,d]
  float* dw;                // [B,S,G,k]
  int* status;
  int B, S, N, G, M, k, d;
  float scale_log2;         // log2(e) / sqrt(d)
  float inv_sqrt_d;
  uint64_t wait_limit_ns;
};
cudaError_t launch_bwd(const BwdArgs& a, cudaStream_t st);
// K/V working-set size from which routed d = 64 calls use the pair kernel;
// returns the previous value (negative: never).  pair_kernel_for() is the
// decision for one call: taken once, then passed to the bucketing (list
// format) and to the attention launch.
int64_t set_pair_threshold(int64_t kv_bytes);
bool pair_kernel_for(const gqe_dims& d);

struct CombineArgs {
  const void* O_sel;
  void* o_bar;
  const float* w;
  int64_t out_row_stride;
  int T, G, k, d, out_fp32;
};
cudaError_t launch_combine(const CombineArgs& a, cudaStream_t st);

cudaError_t launch_selftest_wait(int* status, uint64_t limit_ns, cudaStream_t st);

// Projections (gqe_gemm.cu): bf16 operands, fp32 accumulation in TMEM.
struct GemmArgs {
  CUtensorMap tmA;      // dense form: bf16 A [rows, K] (row stride lda), box {64, 128}
  CUtensorMap tmB;      // bf16 B stack [nb, K, nc], box {64, 64, 1}
  const uint16_t* A;    // routed form: bf16 x [B, S, lda] (rows gathered)
  int64_t lda;
  void* C;              // dense form: [rows, ldc] (fp32 or bf16); routed form: bf16 Q [B,S,N,d]
  int64_t ldc;
  int c_fp32;
  int K;                // reduction length, a multiple of 64
  int nc;               // columns of one B matrix (a multiple of 64)
  int n_total;          // columns of C in the dense form (nb * nc or a part of it)
  int rows;             // rows of A and C in the dense form
  // routed form: the attention work list and the bucket lists
  const int32_t* bucket_off;
  const int32_t* bucket_tok;
  const TileDesc* tiles;
  const int32_t* tile_count;
  int B, S, N, G, M, d;
  int* status;
  uint64_t wait_limit_ns;
};
// C = A . B over 128-row tiles and bn-column tiles (bn in {64, 128, 256},
// n_total % bn == 0).
cudaError_t launch_gemm_dense(const GemmArgs& a, int bn, cudaStream_t st);
// Q of the selected heads, one CTA per routed tile of the work list.
cudaError_t launch_gemm_routed(const GemmArgs& a, int64_t n_list, cudaStream_t st);

// ------------------------------------------------------------ host helpers
// (gqe_host.cu; shared by every entry point)
bool aligned16(const void* p);
// Shape checks: unsupported combinations are refused, never remapped.
gqe_status check_dims(const gqe_dims* d, bool router);
// Tiled TMA map over a row-major tensor (dims innermost first, byte strides
// for dims 1..rank-1), 128-byte swizzle.
bool encode_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base,
                const uint64_t* dims, const uint64_t* strides, const uint32_t* box);
// [B, S, H, d] -> 4-D map with a {64, 1, 128, 1} box; [B, S, d] -> {64, 128, 1}.
bool map_bshd(CUtensorMap* m, CUtensorMapDataType dt, const void* base, int B, int S, int H,
              int d);
bool map_bsd(CUtensorMap* m, CUtensorMapDataType dt, const void* base, int B, int S, int d);
// The attention launch, bracketed by the profiling events when they are set.
void set_profile_events(cudaEvent_t begin, cudaEvent_t end);
cudaError_t timed_attention(const AttnArgs& a, int64_t n_list, cudaStream_t s);
// A non-blocking stream per device, created on first use and kept for the
// process: work that does not depend on the caller's stream runs there,
// ordered against it by events.
constexpr int kMaxSideDevices = 64;
cudaError_t side_stream(cudaStream_t* out);

}  // namespace gqe
