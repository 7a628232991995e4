// kvk_internal.cuh -- types shared by the host layer and the kernels of libkvk.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "kvk.h"

namespace kvk {

constexpr int kMaxRowElems = 2048;      // d + d_rope handled by the write kernel
constexpr size_t kArenaHeader = 256;    // status flags live in the first bytes of the arena
constexpr int kTcTileTokens = 64;       // tokens per tile of the tensor-core decode
// staged query rows of the tensor-core decode: heads rounded up to 8
inline int tc_query_rows(int H) { return (H + 7) / 8 * 8; }
// Work-split cost of one piece on the tensor-core decode, in tokens: query staging and the
// pipeline refill at a sequence boundary take about as long as 2.5 tiles.
constexpr int kTcPieceCost = 160;
// Default time limit of one wait inside the tensor-core decode (kvk_set_wait_limit).
constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;

struct AnchorDesc {
  int layer = 0;
  int d = 0;
  int b = 0;
  int n = 0;             // d + d_rope
  int row_bytes = 0;
  int sg = 1;            // fp16 scales per token: n / G in a group-scaled layout, else 1
  int64_t codes_off = 0;
  int64_t scales_off = 0;
  bool tmap_ok = false;
  CUtensorMap tmap_tile;     // 2D [rows = max_batch*max_tokens][row_bytes] uint8, 64-row box
};

}  // namespace kvk

struct kvk_layout {
  int n_layers = 0;
  int r = 0;
  int d_rope = 0;
  int max_batch = 0;
  int max_tokens = 0;
  int group = 0;                          // elements per scale (0: one scale per token)
  std::vector<int> anchor, d, b;
  std::vector<int> slot;                  // layer -> index into anchors (its anchor's)
  std::vector<kvk::AnchorDesc> anchors;
  uint8_t* arena = nullptr;
  size_t arena_bytes = 0;
  int64_t bits_per_token = 0;
  int path = KVK_PATH_AUTO;
  int ctas = 0;
  int device = -1;
  int num_sms = 0;
  uint64_t wait_limit_ns = 0;             // tensor-core decode wait limit (0: the default)
};

namespace kvk {

// ---------------------------------------------------------------------------
// decode parameters shared by both decode kernels and the merge
// ---------------------------------------------------------------------------
struct DecodeArgs {
  const uint8_t* codes;     // anchor's codes plane
  const __half* scales;     // anchor's scale plane
  int row_bytes, d, d_rope, n, b;
  int max_tokens;
  const void* q_lat;
  const void* q_rope;
  int64_t ql_ss, ql_sh, qr_ss, qr_sh;  // element strides
  int batch, H;
  const int32_t* seq_lens;
  const int32_t* keep_idx;   // nullable
  const int32_t* keep_len;
  int keep_stride;
  float sigma;
  float* out;
  float* lse;
  // workspace
  int32_t* seq_off;          // [batch + 1] token offsets of the flattened token space
  float* ws_ml;              // [slots][H][2]  (running max in log2 units, sum of weights)
  float* ws_o;               // [slots][H][d]  (un-normalised weighted sums)
  int G;                     // CTAs the flattened tokens are split over
  int split_x;               // cost of a piece in tokens (split_cost / split_token)
  uint32_t* flags;
  uint64_t limit_ns;         // time limit of one wait in the tensor-core kernel
  int group, sg;             // group-scaled cache: elements per scale and scales per token
                             // (group = 0, sg = 1: one scale per token)
  // fused append (kvk_mla_decode_append): before the decode reads it, the new token of
  // sequence i -- app_c[i * app_c_ss + k] (k < d) and app_kr[i * app_kr_ss + k] (k < d_rope),
  // dtype app_dtype -- is written at position seq_len_i - 1 of the cache.  app_c == nullptr:
  // no append.
  const void* app_c;
  const void* app_kr;
  int64_t app_c_ss, app_kr_ss;
  int app_dtype;
};

// Workspace carve-up: returns total bytes; fills pointers when base != nullptr.
size_t decode_workspace(int batch, int H, int d, int G, void* base, DecodeArgs* a);

// CTA count for a decode call (depends only on the layout and batch).
int decode_ctas(const kvk_layout* L, int batch, int path);

// launchers (return cudaGetLastError())
// The scale group of an anchor's writes (0 = one scale per token): the layout's, except that
// an uncompressed anchor always keeps one (unit) scale per token.
inline int anchor_group(const kvk_layout* L, const AnchorDesc& A) {
  return (A.b == KVK_BITS_BF16) ? 0 : L->group;
}
cudaError_t launch_quant_write(const kvk_layout* L, const AnchorDesc& A, const void* c_kv,
                               int dtype, int64_t c_ss, int64_t c_st, const void* k_rope,
                               int64_t kr_ss, int64_t kr_st, int batch, const int32_t* start_pos,
                               int n_new, cudaStream_t stream);
// One layer of a multi-layer quantise-on-write launch.
struct QuantLayer {
  uint8_t* codes;
  __half* scales;
  int row_bytes, d, b;
  int group;   // elements per scale (0: one per token)
  const void* c_kv;
  int64_t c_ss, c_st;
  const void* k_rope;
  int64_t kr_ss, kr_st;
};
struct QuantLayers {
  QuantLayer l[KVK_MAX_WRITE_LAYERS];
};
cudaError_t launch_quant_write_layers(const kvk_layout* L, const QuantLayers& Q, int n, int dtype,
                                      int batch, const int32_t* start_pos, int n_new,
                                      cudaStream_t stream);
// One new token per sequence written at position clamp(seq_lens[i], 0, max_tokens) - 1 (none
// for an empty sequence): the append of a fused append + decode when its decode kernel cannot
// take the append itself.
cudaError_t launch_quant_append(const kvk_layout* L, const AnchorDesc& A, const void* c_new,
                                int dtype, int64_t c_ss, const void* kr_new, int64_t kr_ss,
                                int batch, const int32_t* seq_lens, cudaStream_t stream);
cudaError_t launch_decode_fma(const DecodeArgs& a, int dtype, cudaStream_t stream);
// tmap: the codes plane the kernel streams (the anchor's, or a compacted keep-list copy)
// qmap_l / qmap_r: the query's latent and rope parts as 3D tensors [batch][H][d or d_rope] of
// 16-bit elements, boxes of 64 features x tc_query_rows(H) heads (128-byte swizzle)
cudaError_t launch_decode_tc(const DecodeArgs& a, const CUtensorMap& tmap, const CUtensorMap& qmap_l,
                             const CUtensorMap& qmap_r, int dtype, cudaStream_t st);
bool tc_supported(const kvk_layout* L, const AnchorDesc& A, int dtype, int H);
// The token-scale tensor-core kernel (kvk_decode_tc_token.cu): decode (and fused append) of
// b in {2, 4, 8, 16} codes with one scale per token and of bf16 rows; the query read with
// 16-byte loads (rows
// 16-byte aligned, as the general kernel's query tensor maps require).
cudaError_t launch_decode_tc_packed(const DecodeArgs& a, const CUtensorMap& tmap, int dtype,
                                    cudaStream_t st);
bool tc_packed_supported(const kvk_layout* L, const AnchorDesc& A, int dtype, int H);

inline size_t align_up_sz(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Keep-list compaction ahead of the tensor-core decode (kvk_compact.cu): the kept rows and
// scales of sequence i go, in keep order and without invalid entries, to rows
// [i * keep_stride, i * keep_stride + cnt[i]) of a dense scratch cache.
struct CompactArgs {
  const uint8_t* codes;      // anchor's codes plane [max_batch * max_tokens][row_bytes]
  const __half* scales;      // anchor's scale plane
  int row_bytes, max_tokens;
  const int32_t* seq_lens;
  const int32_t* keep_idx;   // [batch][keep_stride]
  const int32_t* keep_len;
  int keep_stride;
  int sg;                    // fp16 scales per token
  int32_t* cnt;              // [batch] valid kept entries per sequence (written)
  uint8_t* dst_codes;        // [batch * keep_stride][row_bytes]
  __half* dst_scales;        // [batch * keep_stride] (+ slack for the decode's scale windows)
  uint32_t* flags;
};
size_t compact_workspace_bytes(int batch, int keep_stride, int row_bytes, int sg);
void compact_carve(void* base, int batch, int keep_stride, int row_bytes, int sg, CompactArgs* c);
cudaError_t launch_compact(const CompactArgs& c, int batch, cudaStream_t stream);
cudaError_t launch_merge(const DecodeArgs& a, cudaStream_t stream);

// Absorbed projections (kvk_absorb.cu): y[b, h, j] = sum_k x[b, h, k] w[h, k, j].
size_t absorb_smem_bytes(int K, int x_f32);
cudaError_t launch_absorb(const void* x, int x_f32, int64_t x_ss, int64_t x_sh, const void* w,
                          int64_t w_sk, int64_t w_sh, void* y, int y_f32, int64_t y_ss,
                          int64_t y_sh, int batch, int heads, int K, int n, uint32_t* flags,
                          cudaStream_t st);

// Work split of the flattened tokens over G CTAs.  Sequence i occupies the cost range
// [off[i] + X i, off[i+1] + X (i+1)): X units standing for the fixed cost of a piece (query
// staging, partial write-back), then one unit per token; C = N + X batch in all.  CTA c owns
// the cost range [split_cost(c), split_cost(c+1)), i.e. the tokens t of sequence i whose cost
// position t + X (i + 1) lies in it: a CTA that takes the start of a sequence takes fewer
// tokens.  X = 0 is the plain even split of the tokens.
__host__ __device__ inline int64_t split_cost(int c, int64_t C, int G) {
  return ((int64_t)c * C) / G;
}
// The CTA whose cost range holds position u (the largest c with split_cost(c) <= u).
__host__ __device__ inline int split_cta(int64_t u, int64_t C, int G) {
  int64_t c = ((u + 1) * (int64_t)G + C - 1) / C - 1;
  return (int)(c < 0 ? 0 : (c >= G ? G - 1 : c));
}
// First token whose cost position is >= u (N when there is none); off has batch + 1 entries.
__host__ __device__ inline int64_t split_token(const int32_t* off, int batch, int X, int64_t u) {
  int L = 0, H = batch;   // the last i with off[i] + X i <= u
  while (L < H) {
    const int mid = (L + H + 1) >> 1;
    if (off[mid] + (int64_t)X * mid <= u) L = mid; else H = mid - 1;
  }
  if (L >= batch) return off[batch];
  const int64_t len = off[L + 1] - off[L];
  const int64_t into = u - (off[L] + (int64_t)X * L) - X;   // tokens of sequence L before u
  return off[L] + (into < 0 ? 0 : (into > len ? len : into));
}

}  // namespace kvk
