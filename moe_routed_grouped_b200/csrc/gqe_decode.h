// Split-KV decode and append (gqe_attention_decode / gqe_attention_append):
// plan, kernel arguments and launcher.  Kept apart from gqe_internal.h, which
// the prefill kernels share.
#pragma once

#include "gqe_internal.h"

namespace gqe {

// Split-KV plan of gqe_attention_decode / gqe_attention_append.  A CTA takes
// one chunk of keys of one (b, g) and up to kDecHeads of that group's head
// slots; slot r*(k+1) + j is new token r's routed head j (j < k) or its shared
// head (j = k, live only for g = 0).  A second kernel merges the chunks.  The
// plan depends on dims and n_new only, so the workspace size does too.
constexpr int kDecThreads = 128;     // 4 warps per partial-attention CTA
constexpr int kDecHeads = 4;         // head slots per CTA (registers bound it)
constexpr int kDecUnroll = 4;        // keys in flight per key slot
constexpr int64_t kDecTargetCtas = 4 * 148;
constexpr int64_t kDecMinChunk = 256;
// Chunks per (b, g) never exceed the CTA target: chunk >= ceil(T / want) with
// want <= kDecTargetCtas, so nchunks = ceil(T / chunk) <= want.
constexpr int kDecMaxChunks = static_cast<int>(kDecTargetCtas);
constexpr int kMaxAppend = 64;       // new tokens per sequence in one append call

struct DecodePlan {
  int64_t heads;    // head slots per (b, g): (k + 1) * n_new
  int64_t passes;   // ceil(heads / kDecHeads)
  int64_t chunk;    // keys per CTA (multiple of 64)
  int64_t nchunks;  // ceil(T / chunk)
  size_t status, part_m, part_l, part_o, total;  // workspace byte offsets
};

inline DecodePlan make_decode_plan(const gqe_dims& d, int64_t n_new = 1) {
  DecodePlan P{};
  const int64_t B = d.B, T = d.S, G = d.G, hd = d.d;
  P.heads = (d.k + 1) * n_new;
  P.passes = (P.heads + kDecHeads - 1) / kDecHeads;
  const int64_t groups = B * G * P.passes;
  const int64_t want = groups >= kDecTargetCtas ? 1 : (kDecTargetCtas + groups - 1) / groups;
  int64_t chunk = (T + want - 1) / want;
  chunk = (chunk + 63) / 64 * 64;
  P.chunk = chunk < kDecMinChunk ? kDecMinChunk : chunk;
  P.nchunks = (T + P.chunk - 1) / P.chunk;  // <= kDecMaxChunks (the merge stages that many)
  const int64_t parts = B * G * P.heads * P.nchunks;
  size_t off = 0;
  P.status = off;  off += 512;  // status word; bytes 256..511 stay the router's counters
  P.part_m = off;  off = align_up(off + sizeof(float) * parts, 256);
  P.part_l = off;  off = align_up(off + sizeof(float) * parts, 256);
  P.part_o = off;  off = align_up(off + sizeof(float) * parts * hd, 256);
  P.total = off;
  return P;
}

struct DecodeArgs {
  const uint16_t* Q;    // bf16 [B, n_new, N, d]
  const uint16_t* Qs;   // bf16 [B, n_new, d]
  const uint16_t* Kc;   // bf16 [B, T, G, d]
  const uint16_t* Vc;   // bf16 [B, T, G, d]
  const int32_t* pos;   // [B]: slot of new token 0 (token r at pos + r)
  const int32_t* kv_start;  // [B] first valid slot, or null (0)
  const int32_t* topk_idx;  // [B, n_new, G, k]
  const float* w;           // [B, n_new, G, k]
  float* part_m;        // [B, G, heads, nchunks]: running max (log2 units)
  float* part_l;        // [B, G, heads, nchunks]: sum of exponentials
  float* part_o;        // [B, G, heads, nchunks, d]: unnormalised output
  void* O_sel;
  void* o_bar;
  void* s_out;
  int64_t out_row_stride;
  int* status;
  int B, T, N, G, M, k, d;
  int n_new;            // new tokens per sequence (1: decode)
  int heads, passes, nchunks, chunk;
  int out_fp32;
  float scale_log2;     // log2(e) / sqrt(d)
};
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st);

}  // namespace gqe
