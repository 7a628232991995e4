// kvk_api.cu -- host side of libkvk: layout validation, arena planning, argument checks,
// kernel dispatch.  Every exported symbol is declared in include/kvk.h.
#include <string.h>

#include <algorithm>
#include <new>

#include "kvk_internal.cuh"

using kvk::AnchorDesc;

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A layout's arena lives on one device; a call made with another device current would
// hand that arena (and, for the no-allocation decode, that device's scratch array) to
// kernels running elsewhere.  Such calls are refused before anything is launched.
kvk_status check_device(const kvk_layout* L) {
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) {
    cudaGetLastError();
    return KVK_ERR_CUDA;
  }
  return cur == L->device ? KVK_OK : KVK_ERR_INVALID_ARG;
}

int row_bytes_of(int n, int b) {
  int raw = (n * b + 7) / 8;
  return (raw + 15) / 16 * 16;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Codes plane as a 2D uint8 tensor [rows][row_bytes]; inner box = one 128-feature group of
// packed codes (128*b/8 bytes, at most the row), outer box = `box_rows` token rows.
bool make_codes_tmap(CUtensorMap* m, void* base, int64_t rows, int row_bytes, int b,
                     int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  int inner = 128 * b / 8;   // 32, 64, 128 or 256 bytes
  // 16-bit elements (codes or bf16 values): one 64-feature atom per box (two boxes per group)
  if (b == 16 || b == KVK_BITS_BF16) inner = 128;
  CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_NONE;
  if (inner == 128) sw = CU_TENSOR_MAP_SWIZZLE_128B;
  else if (inner == 64) sw = CU_TENSOR_MAP_SWIZZLE_64B;
  else if (inner == 32) sw = CU_TENSOR_MAP_SWIZZLE_32B;
  cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {(cuuint32_t)inner, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// One part of the query (latent or rope) as a 3D tensor [batch][H][elems] of 16-bit elements
// with the caller's strides (in elements); box = 64 features x rows heads, 128-byte swizzle,
// so that a box lands as one UMMA K-major atom.  Heads >= H and features >= elems read zero.
bool make_query_tmap(CUtensorMap* m, const void* base, int64_t elems, int H, int batch,
                     int64_t stride_head, int64_t stride_seq, int rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || elems < 1) return false;
  cuuint64_t dims[3] = {(cuuint64_t)elems, (cuuint64_t)H, (cuuint64_t)batch};
  cuuint64_t strides[2] = {(cuuint64_t)stride_head * 2, (cuuint64_t)stride_seq * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

namespace kvk {

size_t decode_workspace(int batch, int H, int d, int G, void* base, DecodeArgs* a) {
  size_t off = 0;
  size_t o_seq = off;
  off = align_up(off + sizeof(int32_t) * (size_t)(batch + 1), kAlign);
  size_t slots = (size_t)G + (size_t)batch;
  size_t o_ml = off;
  off = align_up(off + sizeof(float) * slots * (size_t)H * 2, kAlign);
  size_t o_o = off;
  off = align_up(off + sizeof(float) * slots * (size_t)H * (size_t)d, kAlign);
  if (base && a) {
    uint8_t* p = static_cast<uint8_t*>(base);
    a->seq_off = reinterpret_cast<int32_t*>(p + o_seq);
    a->ws_ml = reinterpret_cast<float*>(p + o_ml);
    a->ws_o = reinterpret_cast<float*>(p + o_o);
    a->G = G;
  }
  return off;
}

int decode_ctas(const kvk_layout* L, int batch, int path) {
  if (L->ctas > 0) return L->ctas;
  int sms = L->num_sms > 0 ? L->num_sms : 148;
  int64_t tokens = (int64_t)batch * L->max_tokens;
  // at least ~256 tokens per CTA on the CUDA-core path, one tile per CTA on the tensor path
  int64_t per = (path == KVK_PATH_TENSOR) ? kTcTileTokens : 256;
  int64_t want = (tokens + per - 1) / per;
  int cap = (path == KVK_PATH_TENSOR) ? sms : 4 * sms;
  return (int)std::max<int64_t>(1, std::min<int64_t>(want, cap));
}

}  // namespace kvk

extern "C" {

const char* kvk_status_string(kvk_status s) {
  switch (s) {
    case KVK_OK: return "ok";
    case KVK_ERR_INVALID_ARG: return "invalid argument";
    case KVK_ERR_BAD_TABLE: return "per-layer table violates the action space";
    case KVK_ERR_BUDGET: return "plan exceeds the bits-per-token budget";
    case KVK_ERR_INHERITING_LAYER: return "layer inherits its cache and cannot be written";
    case KVK_ERR_WORKSPACE: return "arena or workspace too small";
    case KVK_ERR_ALIGNMENT: return "device pointer or stride misaligned";
    case KVK_ERR_CUDA: return "CUDA call failed";
    case KVK_ERR_UNSUPPORTED: return "shape not supported by the compiled kernels";
  }
  return "unknown status";
}

}  // extern "C"

// Layout with one fp16 scale per `group` consecutive elements of every quantised anchor's
// row (group = 0: one scale per token).
static kvk_status create_layout_impl(int n_layers, const int32_t* anchor, const int32_t* d,
                                     const int32_t* b, int r, int d_rope, int group,
                                     int max_batch, int max_tokens, int64_t budget_bits_per_token,
                                     void* dev_arena, size_t arena_bytes, kvk_layout** out,
                                     size_t* arena_bytes_needed, int64_t* bits_per_token) {
  if (out) *out = nullptr;
  if (n_layers < 1 || n_layers > 65536 || !anchor || !d || !b) return KVK_ERR_INVALID_ARG;
  if (group != 0 && group != 16 && group != 32 && group != 64) return KVK_ERR_INVALID_ARG;
  if (r < 16 || r % 16 != 0 || d_rope < 0 || d_rope % 8 != 0) return KVK_ERR_INVALID_ARG;
  if (max_batch < 1 || max_batch > 4096 || max_tokens < 1) return KVK_ERR_INVALID_ARG;
  if ((int64_t)max_batch * (int64_t)max_tokens >= (int64_t(1) << 31)) return KVK_ERR_INVALID_ARG;

  // depth axis: anchor[0] == 0; every other layer is an anchor or points at the nearest
  // preceding anchor.  rank / precision axes: 16 <= d <= r, d % 16 == 0, b in {2,4,8,16};
  // b = 0 keeps the anchor uncompressed (bf16 rows, 16 bits per element, no scale).
  int64_t bits = 0;
  int last = -1;
  for (int l = 0; l < n_layers; ++l) {
    if (anchor[l] == l) {
      if (d[l] < 16 || d[l] > r || d[l] % 16 != 0) return KVK_ERR_BAD_TABLE;
      if (b[l] != 2 && b[l] != 4 && b[l] != 8 && b[l] != 16 && b[l] != KVK_BITS_BF16)
        return KVK_ERR_BAD_TABLE;
      if (d[l] + d_rope > kvk::kMaxRowElems) return KVK_ERR_UNSUPPORTED;
      const int n = d[l] + d_rope;
      if (group && b[l] != KVK_BITS_BF16 && n % group != 0) return KVK_ERR_BAD_TABLE;
      if (b[l] == KVK_BITS_BF16)
        bits += (int64_t)n * 16;
      else
        bits += (int64_t)n * b[l] + (group ? (int64_t)16 * (n / group) : 16);
      last = l;
    } else {
      if (l == 0 || anchor[l] != last) return KVK_ERR_BAD_TABLE;
    }
  }
  if (bits_per_token) *bits_per_token = bits;

  // arena plan
  kvk_layout tmp;
  tmp.n_layers = n_layers;
  tmp.r = r;
  tmp.d_rope = d_rope;
  tmp.max_batch = max_batch;
  tmp.max_tokens = max_tokens;
  tmp.group = group;
  tmp.anchor.assign(anchor, anchor + n_layers);
  tmp.d.assign(d, d + n_layers);
  tmp.b.assign(b, b + n_layers);
  tmp.slot.assign(n_layers, -1);
  size_t off = kvk::kArenaHeader;
  int max_sg = 1;
  const size_t tokens = (size_t)max_batch * (size_t)max_tokens;
  for (int l = 0; l < n_layers; ++l) {
    if (anchor[l] == l) {
      AnchorDesc A;
      A.layer = l;
      A.d = d[l];
      A.b = b[l];
      A.n = d[l] + d_rope;
      A.row_bytes = row_bytes_of(A.n, A.b == KVK_BITS_BF16 ? 16 : A.b);
      A.sg = (group && A.b != KVK_BITS_BF16) ? A.n / group : 1;
      max_sg = std::max(max_sg, A.sg);
      off = align_up(off, kAlign);
      A.codes_off = (int64_t)off;
      off += tokens * (size_t)A.row_bytes;
      off = align_up(off, kAlign);
      A.scales_off = (int64_t)off;
      off += tokens * (size_t)A.sg * sizeof(__half);
      tmp.anchors.push_back(A);
    }
    tmp.slot[l] = (int)tmp.anchors.size() - 1;
  }
  // tail slack: the tensor-core decode reads each tile's scales (64 tokens) as one window from
  // the 16-byte boundary at or below the first, which can reach past the last scale plane by
  // up to 64 tokens' scales and 32 bytes
  off = align_up(off, kAlign) + align_up((size_t)64 * max_sg * sizeof(__half) + 32, kAlign);
  if (arena_bytes_needed) *arena_bytes_needed = off;
  if (budget_bits_per_token > 0 && bits > budget_bits_per_token) return KVK_ERR_BUDGET;
  if (!out) return KVK_OK;  // query mode

  if (dev_arena) {
    if ((reinterpret_cast<uintptr_t>(dev_arena) & (kAlign - 1)) != 0) return KVK_ERR_ALIGNMENT;
    if (arena_bytes < off) return KVK_ERR_WORKSPACE;
  }
  kvk_layout* L = new (std::nothrow) kvk_layout(std::move(tmp));
  if (!L) return KVK_ERR_INVALID_ARG;
  L->arena = static_cast<uint8_t*>(dev_arena);
  L->arena_bytes = arena_bytes;
  L->bits_per_token = bits;
  if (dev_arena) {
    if (cudaGetDevice(&L->device) != cudaSuccess ||
        cudaDeviceGetAttribute(&L->num_sms, cudaDevAttrMultiProcessorCount, L->device) !=
            cudaSuccess ||
        cudaMemset(dev_arena, 0, kvk::kArenaHeader) != cudaSuccess) {
      cudaGetLastError();
      delete L;
      return KVK_ERR_CUDA;
    }
    for (AnchorDesc& A : L->anchors) {
      void* base = L->arena + A.codes_off;
      A.tmap_ok = make_codes_tmap(&A.tmap_tile, base, (int64_t)tokens, A.row_bytes, A.b,
                                  kvk::kTcTileTokens);
    }
  }
  *out = L;
  return KVK_OK;
}

extern "C" {

kvk_status kvk_create_layout(int n_layers, const int32_t* anchor, const int32_t* d,
                             const int32_t* b, int r, int d_rope, int max_batch, int max_tokens,
                             int64_t budget_bits_per_token, void* dev_arena, size_t arena_bytes,
                             kvk_layout** out, size_t* arena_bytes_needed,
                             int64_t* bits_per_token) {
  return create_layout_impl(n_layers, anchor, d, b, r, d_rope, 0, max_batch, max_tokens,
                            budget_bits_per_token, dev_arena, arena_bytes, out,
                            arena_bytes_needed, bits_per_token);
}

kvk_status kvk_create_layout_grouped(int n_layers, const int32_t* anchor, const int32_t* d,
                                     const int32_t* b, int r, int d_rope, int scale_group,
                                     int max_batch, int max_tokens,
                                     int64_t budget_bits_per_token, void* dev_arena,
                                     size_t arena_bytes, kvk_layout** out,
                                     size_t* arena_bytes_needed, int64_t* bits_per_token) {
  if (scale_group == 0) return KVK_ERR_INVALID_ARG;
  return create_layout_impl(n_layers, anchor, d, b, r, d_rope, scale_group, max_batch,
                            max_tokens, budget_bits_per_token, dev_arena, arena_bytes, out,
                            arena_bytes_needed, bits_per_token);
}

void kvk_destroy(kvk_layout* L) { delete L; }

kvk_status kvk_get_layer_info(const kvk_layout* L, int layer, kvk_layer_info* info) {
  if (!L || !info || layer < 0 || layer >= L->n_layers) return KVK_ERR_INVALID_ARG;
  const AnchorDesc& A = L->anchors[L->slot[layer]];
  info->anchor = A.layer;
  info->d = A.d;
  info->b = A.b;
  info->row_bytes = A.row_bytes;
  info->codes = L->arena + A.codes_off;
  info->scales = L->arena + A.scales_off;
  info->codes_offset = A.codes_off;
  info->scales_offset = A.scales_off;
  info->max_batch = L->max_batch;
  info->max_tokens = L->max_tokens;
  info->r = L->r;
  info->d_rope = L->d_rope;
  info->scales_per_token = A.sg;
  info->scale_group = A.sg > 1 ? L->group : 0;
  return KVK_OK;
}

kvk_status kvk_quant_write(kvk_layout* L, int layer, const void* c_kv, int dtype,
                           int64_t c_stride_seq, int64_t c_stride_tok, const void* k_rope,
                           int64_t kr_stride_seq, int64_t kr_stride_tok, int batch,
                           const int32_t* dev_start_pos, int n_new, kvk_stream_t stream) {
  if (!L || layer < 0 || layer >= L->n_layers) return KVK_ERR_INVALID_ARG;
  if (L->anchor[layer] != layer) return KVK_ERR_INHERITING_LAYER;
  if (!L->arena) return KVK_ERR_INVALID_ARG;
  if (dtype != KVK_F32 && dtype != KVK_BF16) return KVK_ERR_INVALID_ARG;
  if (batch < 1 || batch > L->max_batch || n_new < 0) return KVK_ERR_INVALID_ARG;
  if (n_new == 0) return KVK_OK;
  if (kvk_status ds = check_device(L)) return ds;
  if (!c_kv || !dev_start_pos || (L->d_rope > 0 && !k_rope)) return KVK_ERR_INVALID_ARG;
  if (c_stride_seq < 0 || c_stride_tok < 0 || kr_stride_seq < 0 || kr_stride_tok < 0)
    return KVK_ERR_INVALID_ARG;
  if (!aligned16(c_kv) || (k_rope && !aligned16(k_rope)) ||
      (reinterpret_cast<uintptr_t>(dev_start_pos) & 3u))
    return KVK_ERR_ALIGNMENT;
  // strides in elements must keep every token's first element 16-byte aligned
  if (c_stride_seq % 8 || c_stride_tok % 8 || kr_stride_seq % 8 || kr_stride_tok % 8)
    return KVK_ERR_ALIGNMENT;
  const AnchorDesc& A = L->anchors[L->slot[layer]];
  cudaError_t e = kvk::launch_quant_write(L, A, c_kv, dtype, c_stride_seq, c_stride_tok, k_rope,
                                          kr_stride_seq, kr_stride_tok, batch, dev_start_pos,
                                          n_new, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVK_OK : KVK_ERR_CUDA;
}

kvk_status kvk_quant_write_layers(kvk_layout* L, int n, const int32_t* layers,
                                  const void* const* c_kv, int dtype,
                                  const int64_t* c_stride_seq, const int64_t* c_stride_tok,
                                  const void* const* k_rope, const int64_t* kr_stride_seq,
                                  const int64_t* kr_stride_tok, int batch,
                                  const int32_t* dev_start_pos, int n_new, kvk_stream_t stream) {
  if (!L || n < 1 || n > KVK_MAX_WRITE_LAYERS || !layers || !c_kv || !c_stride_seq ||
      !c_stride_tok || !k_rope || !kr_stride_seq || !kr_stride_tok)
    return KVK_ERR_INVALID_ARG;
  if (!L->arena) return KVK_ERR_INVALID_ARG;
  if (dtype != KVK_F32 && dtype != KVK_BF16) return KVK_ERR_INVALID_ARG;
  if (batch < 1 || batch > L->max_batch || n_new < 0) return KVK_ERR_INVALID_ARG;
  if (!dev_start_pos) return KVK_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(dev_start_pos) & 3u) return KVK_ERR_ALIGNMENT;
  kvk::QuantLayers Q;
  for (int k = 0; k < n; ++k) {
    const int layer = layers[k];
    if (layer < 0 || layer >= L->n_layers) return KVK_ERR_INVALID_ARG;
    if (L->anchor[layer] != layer) return KVK_ERR_INHERITING_LAYER;
    for (int j = 0; j < k; ++j)
      if (layers[j] == layer) return KVK_ERR_INVALID_ARG;
    if (!c_kv[k] || (L->d_rope > 0 && !k_rope[k])) return KVK_ERR_INVALID_ARG;
    if (c_stride_seq[k] < 0 || c_stride_tok[k] < 0 || kr_stride_seq[k] < 0 ||
        kr_stride_tok[k] < 0)
      return KVK_ERR_INVALID_ARG;
    if (!aligned16(c_kv[k]) || (k_rope[k] && !aligned16(k_rope[k]))) return KVK_ERR_ALIGNMENT;
    if (c_stride_seq[k] % 8 || c_stride_tok[k] % 8 || kr_stride_seq[k] % 8 ||
        kr_stride_tok[k] % 8)
      return KVK_ERR_ALIGNMENT;
    const AnchorDesc& A = L->anchors[L->slot[layer]];
    kvk::QuantLayer& q = Q.l[k];
    q.codes = L->arena + A.codes_off;
    q.scales = reinterpret_cast<__half*>(L->arena + A.scales_off);
    q.row_bytes = A.row_bytes;
    q.d = A.d;
    q.b = A.b;
    q.group = kvk::anchor_group(L, A);
    q.c_kv = c_kv[k];
    q.c_ss = c_stride_seq[k];
    q.c_st = c_stride_tok[k];
    q.k_rope = k_rope[k];
    q.kr_ss = kr_stride_seq[k];
    q.kr_st = kr_stride_tok[k];
  }
  if (n_new == 0) return KVK_OK;
  if (kvk_status ds = check_device(L)) return ds;
  cudaError_t e = kvk::launch_quant_write_layers(L, Q, n, dtype, batch, dev_start_pos, n_new,
                                                 reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVK_OK : KVK_ERR_CUDA;
}

// The kernel a call takes (a keep list does not change it: the tensor-core kernel then
// reads a compacted copy of the kept rows, given workspace for it).
static int choose_path(const kvk_layout* L, const AnchorDesc& A, int dtype, int H) {
  if (L->path == KVK_PATH_CUDA_CORE) return KVK_PATH_CUDA_CORE;
  bool tc = kvk::tc_supported(L, A, dtype, H);
  if (L->path == KVK_PATH_TENSOR || L->path == KVK_PATH_TENSOR_GENERAL)
    return tc ? KVK_PATH_TENSOR : -1;
  return tc ? KVK_PATH_TENSOR : KVK_PATH_CUDA_CORE;
}

kvk_status kvk_decode_workspace_bytes(const kvk_layout* L, int layer, int batch, int n_heads,
                                      size_t* bytes) {
  if (!L || !bytes || layer < 0 || layer >= L->n_layers || batch < 1 ||
      batch > L->max_batch || n_heads < 1)
    return KVK_ERR_INVALID_ARG;
  const AnchorDesc& A = L->anchors[L->slot[layer]];
  int G = std::max(kvk::decode_ctas(L, batch, KVK_PATH_TENSOR),
                   kvk::decode_ctas(L, batch, KVK_PATH_CUDA_CORE));
  *bytes = kvk::decode_workspace(batch, n_heads, A.d, G, nullptr, nullptr);
  return KVK_OK;
}

kvk_status kvk_decode_workspace_bytes_keep(const kvk_layout* L, int layer, int batch,
                                           int n_heads, int keep_stride, size_t* bytes) {
  if (keep_stride < 0) return KVK_ERR_INVALID_ARG;
  size_t base = 0;
  kvk_status st = kvk_decode_workspace_bytes(L, layer, batch, n_heads, &base);
  if (st != KVK_OK) return st;
  const AnchorDesc& A = L->anchors[L->slot[layer]];
  *bytes = align_up(base, kAlign) + kvk::compact_workspace_bytes(batch, keep_stride, A.row_bytes, A.sg);
  return KVK_OK;
}

kvk_status kvk_decode_path_for(const kvk_layout* L, int layer, int dtype, int n_heads,
                               int has_keep, int* path) {
  if (!L || !path || layer < 0 || layer >= L->n_layers || n_heads < 1) return KVK_ERR_INVALID_ARG;
  if (dtype != KVK_F32 && dtype != KVK_BF16 && dtype != KVK_F16) return KVK_ERR_INVALID_ARG;
  (void)has_keep;
  int p = choose_path(L, L->anchors[L->slot[layer]], dtype, n_heads);
  if (p < 0) return KVK_ERR_UNSUPPORTED;
  *path = p;
  return KVK_OK;
}

}  // extern "C"

namespace {

// The new tokens of a fused append + decode (kvk_mla_decode_append).
struct Append {
  const void* c;
  const void* kr;
  int64_t c_ss, kr_ss;
  int dtype;
};

kvk_status decode_impl(kvk_layout* L, int layer, const void* q_lat, const void* q_rope,
                       int dtype, int64_t q_lat_stride_seq, int64_t q_lat_stride_head,
                       int64_t q_rope_stride_seq, int64_t q_rope_stride_head, int batch,
                       int n_heads, const int32_t* dev_seq_lens, const int32_t* dev_keep_idx,
                       const int32_t* dev_keep_len, int keep_stride, float softmax_scale,
                       float* out, float* lse, void* workspace, size_t workspace_bytes,
                       kvk_stream_t stream, const Append* app) {
  if (!L || layer < 0 || layer >= L->n_layers || !L->arena) return KVK_ERR_INVALID_ARG;
  if (dtype != KVK_F32 && dtype != KVK_BF16 && dtype != KVK_F16) return KVK_ERR_INVALID_ARG;
  if (batch < 1 || batch > L->max_batch || n_heads < 1 || n_heads > 4096)
    return KVK_ERR_INVALID_ARG;
  if (!q_lat || (L->d_rope > 0 && !q_rope) || !dev_seq_lens || !out || !workspace)
    return KVK_ERR_INVALID_ARG;
  if ((dev_keep_idx == nullptr) != (dev_keep_len == nullptr)) return KVK_ERR_INVALID_ARG;
  if (dev_keep_idx && keep_stride < 0) return KVK_ERR_INVALID_ARG;
  if (q_lat_stride_seq < 0 || q_lat_stride_head < 0 || q_rope_stride_seq < 0 ||
      q_rope_stride_head < 0)
    return KVK_ERR_INVALID_ARG;
  if (!aligned16(q_lat) || (q_rope && !aligned16(q_rope)) || !aligned16(out) ||
      (lse && !aligned16(lse)) || !aligned16(workspace) ||
      (reinterpret_cast<uintptr_t>(dev_seq_lens) & 3u) ||
      (dev_keep_idx && (reinterpret_cast<uintptr_t>(dev_keep_idx) & 3u)) ||
      (dev_keep_len && (reinterpret_cast<uintptr_t>(dev_keep_len) & 3u)))
    return KVK_ERR_ALIGNMENT;
  if (q_lat_stride_seq % 8 || q_lat_stride_head % 8 || q_rope_stride_seq % 8 ||
      q_rope_stride_head % 8)
    return KVK_ERR_ALIGNMENT;
  if (kvk_status ds = check_device(L)) return ds;
  if (app) {
    if (L->anchor[layer] != layer) return KVK_ERR_INHERITING_LAYER;
    if (dev_keep_idx) return KVK_ERR_INVALID_ARG;
    if (app->dtype != KVK_F32 && app->dtype != KVK_BF16) return KVK_ERR_INVALID_ARG;
    if (!app->c || (L->d_rope > 0 && !app->kr) || app->c_ss < 0 || app->kr_ss < 0)
      return KVK_ERR_INVALID_ARG;
    if (!aligned16(app->c) || (app->kr && !aligned16(app->kr)) || app->c_ss % 8 ||
        app->kr_ss % 8)
      return KVK_ERR_ALIGNMENT;
  }
  const AnchorDesc& A = L->anchors[L->slot[layer]];
  int path = choose_path(L, A, dtype, n_heads);
  if (path < 0) return KVK_ERR_UNSUPPORTED;
  // With a keep list the tensor-core kernel reads a dense copy of the kept rows, placed after
  // the decode's own workspace; without room for it (or a tensor map over it) the call takes
  // the CUDA-core kernel, unless the tensor-core kernel was asked for.
  const bool keep = dev_keep_idx != nullptr;
  CUtensorMap keep_tmap;
  size_t keep_off = 0;
  if (keep && path == KVK_PATH_TENSOR) {
    const int Gt = kvk::decode_ctas(L, batch, KVK_PATH_TENSOR);
    keep_off = align_up(kvk::decode_workspace(batch, n_heads, A.d, Gt, nullptr, nullptr), kAlign);
    const bool room =
        workspace_bytes >= keep_off + kvk::compact_workspace_bytes(batch, keep_stride, A.row_bytes, A.sg);
    kvk::CompactArgs probe;
    if (room) kvk::compact_carve(static_cast<uint8_t*>(workspace) + keep_off, batch, keep_stride,
                                 A.row_bytes, A.sg, &probe);
    const bool ok = room && keep_stride > 0 &&
                    make_codes_tmap(&keep_tmap, probe.dst_codes, (int64_t)batch * keep_stride,
                                    A.row_bytes, A.b, kvk::kTcTileTokens);
    if (!ok) {
      if (L->path != KVK_PATH_AUTO) return room ? KVK_ERR_UNSUPPORTED : KVK_ERR_WORKSPACE;
      path = KVK_PATH_CUDA_CORE;
    }
  }

  // The tensor-core kernel copies each piece's query rows with TMA: tensor maps over the
  // caller's query tensors, built per call (their addresses and strides are the call's).
  CUtensorMap qmap_l, qmap_r;
  memset(&qmap_r, 0, sizeof(qmap_r));
  if (path == KVK_PATH_TENSOR) {
    const int rows = kvk::tc_query_rows(n_heads);
    bool ok = make_query_tmap(&qmap_l, q_lat, A.d, n_heads, batch, q_lat_stride_head,
                              q_lat_stride_seq, rows);
    if (ok && L->d_rope > 0)
      ok = make_query_tmap(&qmap_r, q_rope, L->d_rope, n_heads, batch, q_rope_stride_head,
                           q_rope_stride_seq, rows);
    if (!ok) {
      if (L->path != KVK_PATH_AUTO) return KVK_ERR_UNSUPPORTED;
      path = KVK_PATH_CUDA_CORE;
    }
  }

  kvk::DecodeArgs a;
  memset(&a, 0, sizeof(a));
  a.codes = L->arena + A.codes_off;
  a.scales = reinterpret_cast<const __half*>(L->arena + A.scales_off);
  a.row_bytes = A.row_bytes;
  a.d = A.d;
  a.d_rope = L->d_rope;
  a.n = A.n;
  a.b = A.b;
  a.max_tokens = L->max_tokens;
  a.q_lat = q_lat;
  a.q_rope = q_rope;
  a.ql_ss = q_lat_stride_seq;
  a.ql_sh = q_lat_stride_head;
  a.qr_ss = q_rope_stride_seq;
  a.qr_sh = q_rope_stride_head;
  a.batch = batch;
  a.H = n_heads;
  a.seq_lens = dev_seq_lens;
  a.keep_idx = dev_keep_idx;
  a.keep_len = dev_keep_len;
  a.keep_stride = keep_stride;
  a.sigma = softmax_scale;
  a.out = out;
  a.lse = lse;
  a.flags = reinterpret_cast<uint32_t*>(L->arena);
  a.limit_ns = L->wait_limit_ns ? L->wait_limit_ns : kvk::kDefaultWaitLimitNs;
  a.group = kvk::anchor_group(L, A);
  a.sg = A.sg;
  int G = kvk::decode_ctas(L, batch, path);
  size_t need = kvk::decode_workspace(batch, n_heads, A.d, G, workspace, &a);
  if (workspace_bytes < need) return KVK_ERR_WORKSPACE;
  a.split_x = (path == KVK_PATH_TENSOR) ? kvk::kTcPieceCost : 0;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  // Tensor-core launch over a codes plane: codes with one scale per token and bf16 rows take
  // the kernel specialised for them (unless the general one is asked for), group-scaled codes
  // the general one.
  const bool packed =
      L->path != KVK_PATH_TENSOR_GENERAL && kvk::tc_packed_supported(L, A, dtype, n_heads);
  auto launch_tc = [&](const CUtensorMap& codes_map) {
    return packed ? kvk::launch_decode_tc_packed(a, codes_map, dtype, st)
                  : kvk::launch_decode_tc(a, codes_map, qmap_l, qmap_r, dtype, st);
  };
  if (path == KVK_PATH_TENSOR && keep) {
    kvk::CompactArgs c;
    memset(&c, 0, sizeof(c));
    c.codes = a.codes;
    c.scales = a.scales;
    c.row_bytes = A.row_bytes;
    c.max_tokens = L->max_tokens;
    c.seq_lens = dev_seq_lens;
    c.keep_idx = dev_keep_idx;
    c.keep_len = dev_keep_len;
    c.keep_stride = keep_stride;
    c.flags = a.flags;
    kvk::compact_carve(static_cast<uint8_t*>(workspace) + keep_off, batch, keep_stride,
                       A.row_bytes, A.sg, &c);
    e = kvk::launch_compact(c, batch, st);
    // the decode proper: the dense copy as a cache of keep_stride rows per sequence
    a.codes = c.dst_codes;
    a.scales = c.dst_scales;
    a.max_tokens = keep_stride;
    a.seq_lens = c.cnt;
    a.keep_idx = nullptr;
    a.keep_len = nullptr;
    a.keep_stride = 0;
    if (e == cudaSuccess) e = launch_tc(keep_tmap);
  } else if (path == KVK_PATH_TENSOR) {
    if (app) {   // the decode kernel writes the new tokens itself
      a.app_c = app->c;
      a.app_kr = app->kr;
      a.app_c_ss = app->c_ss;
      a.app_kr_ss = app->kr_ss;
      a.app_dtype = app->dtype;
    }
    e = launch_tc(A.tmap_tile);
  } else {
    if (app)
      e = kvk::launch_quant_append(L, A, app->c, app->dtype, app->c_ss, app->kr, app->kr_ss,
                                   batch, dev_seq_lens, st);
    if (e == cudaSuccess) e = kvk::launch_decode_fma(a, dtype, st);
  }
  if (e == cudaSuccess) e = kvk::launch_merge(a, st);
  return e == cudaSuccess ? KVK_OK : KVK_ERR_CUDA;
}

}  // namespace

extern "C" {

kvk_status kvk_mla_decode(kvk_layout* L, int layer, const void* q_lat, const void* q_rope,
                          int dtype, int64_t q_lat_stride_seq, int64_t q_lat_stride_head,
                          int64_t q_rope_stride_seq, int64_t q_rope_stride_head, int batch,
                          int n_heads, const int32_t* dev_seq_lens, const int32_t* dev_keep_idx,
                          const int32_t* dev_keep_len, int keep_stride, float softmax_scale,
                          float* out, float* lse, void* workspace, size_t workspace_bytes,
                          kvk_stream_t stream) {
  return decode_impl(L, layer, q_lat, q_rope, dtype, q_lat_stride_seq, q_lat_stride_head,
                     q_rope_stride_seq, q_rope_stride_head, batch, n_heads, dev_seq_lens,
                     dev_keep_idx, dev_keep_len, keep_stride, softmax_scale, out, lse, workspace,
                     workspace_bytes, stream, nullptr);
}

kvk_status kvk_mla_decode_append(kvk_layout* L, int layer, const void* c_new,
                                 const void* k_rope_new, int new_dtype, int64_t c_new_stride_seq,
                                 int64_t k_rope_new_stride_seq, const void* q_lat,
                                 const void* q_rope, int dtype, int64_t q_lat_stride_seq,
                                 int64_t q_lat_stride_head, int64_t q_rope_stride_seq,
                                 int64_t q_rope_stride_head, int batch, int n_heads,
                                 const int32_t* dev_seq_lens, float softmax_scale, float* out,
                                 float* lse, void* workspace, size_t workspace_bytes,
                                 kvk_stream_t stream) {
  const Append app{c_new, k_rope_new, c_new_stride_seq, k_rope_new_stride_seq, new_dtype};
  return decode_impl(L, layer, q_lat, q_rope, dtype, q_lat_stride_seq, q_lat_stride_head,
                     q_rope_stride_seq, q_rope_stride_head, batch, n_heads, dev_seq_lens, nullptr,
                     nullptr, 0, softmax_scale, out, lse, workspace, workspace_bytes, stream,
                     &app);
}

kvk_status kvk_read_status(kvk_layout* L, uint32_t* flags, int clear, kvk_stream_t stream) {
  if (!L || !flags || !L->arena) return KVK_ERR_INVALID_ARG;
  if (kvk_status ds = check_device(L)) return ds;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, L->arena, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return KVK_ERR_CUDA;
  *flags = v;
  if (clear) {
    if (cudaMemsetAsync(L->arena, 0, sizeof(uint32_t), st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
      return KVK_ERR_CUDA;
  }
  return KVK_OK;
}

kvk_status kvk_set_decode_path(kvk_layout* L, int path) {
  if (!L || path < KVK_PATH_AUTO || path > KVK_PATH_TENSOR_GENERAL) return KVK_ERR_INVALID_ARG;
  L->path = path;
  return KVK_OK;
}

kvk_status kvk_set_decode_ctas(kvk_layout* L, int ctas) {
  if (!L || ctas < 0 || ctas > 65536) return KVK_ERR_INVALID_ARG;
  L->ctas = ctas;
  return KVK_OK;
}

kvk_status kvk_absorb(const void* x, int x_dtype, int64_t x_stride_seq, int64_t x_stride_head,
                      const void* w, int64_t w_stride_row, int64_t w_stride_head, void* y,
                      int y_dtype, int64_t y_stride_seq, int64_t y_stride_head, int batch,
                      int n_heads, int K, int n, kvk_stream_t stream) {
  if (!x || !w || !y) return KVK_ERR_INVALID_ARG;
  if ((x_dtype != KVK_BF16 && x_dtype != KVK_F32) || (y_dtype != KVK_BF16 && y_dtype != KVK_F32))
    return KVK_ERR_INVALID_ARG;
  if (batch < 1 || n_heads < 1 || n_heads > 65535 || K < 64 || K > 512 || K % 64 != 0 ||
      n < 16 || n % 16 != 0 || n > 65535 * 128)
    return KVK_ERR_INVALID_ARG;
  if (x_stride_seq < 0 || x_stride_head < 0 || y_stride_seq < 0 || y_stride_head < 0 ||
      w_stride_row < n || w_stride_head < (int64_t)K * w_stride_row)
    return KVK_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w) || !aligned16(y) || x_stride_seq % 8 || x_stride_head % 8 ||
      w_stride_row % 8 || w_stride_head % 8 || y_stride_seq % 8 || y_stride_head % 8)
    return KVK_ERR_ALIGNMENT;
  cudaError_t e = kvk::launch_absorb(x, x_dtype == KVK_F32, x_stride_seq, x_stride_head, w,
                                     w_stride_row, w_stride_head, y, y_dtype == KVK_F32,
                                     y_stride_seq, y_stride_head, batch, n_heads, K, n, nullptr,
                                     reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVK_OK : KVK_ERR_CUDA;
}

kvk_status kvk_set_wait_limit(kvk_layout* L, uint64_t ns) {
  if (!L) return KVK_ERR_INVALID_ARG;
  L->wait_limit_ns = ns;
  return KVK_OK;
}

}  // extern "C"
