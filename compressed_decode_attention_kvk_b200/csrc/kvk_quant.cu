// kvk_quant.cu -- quantise-on-write of one anchor layer's MLA cache (prefill and append).
//
// Method: KV-Kaizen, "Three Non-Eviction Compression Axes": the cached vector of a token is
// the latent c^KV truncated to its first d coordinates plus the decoupled RoPE key k^R
// (rank axis), stored at b bits by symmetric uniform quantisation with one scale per token
// (precision axis).  Scale dtype, rounding and bit layout follow the library's contract in
// include/kvk.h (fp16 scale rounded up, round-half-even codes, offset-binary fields
// little-endian in 16-byte padded rows, separate fp16 scale plane).
//
// Schedule: one warp per token.  Each lane owns groups of 8 consecutive elements
// (one 16-byte bf16 load or two 16-byte fp32 loads), keeps them in registers, the warp
// reduces |v| with shuffles, lane 0 stores the fp16 scale, and every lane stores its
// group's packed bytes (b bytes per group) -- consecutive lanes write consecutive bytes.
// The kernel is HBM bound: it reads (d + d_R) * sizeof(input) and writes row + 2 bytes
// per token.
#include "kvk_quant_common.cuh"

namespace kvk {
namespace {

constexpr int kWarpsPerBlock = 8;
constexpr int kMaxRounds = kMaxRowElems / (8 * 32);  // groups of 8 per lane

// One warp quantises token `tok` (of batch x n_new) of one anchor layer.
template <typename T>
__device__ __forceinline__ void quant_token(
    int64_t tok, uint8_t* __restrict__ codes, __half* __restrict__ scales, int row_bytes, int d,
    int d_rope, int b, int group, int max_tokens, const T* __restrict__ c_kv, int64_t c_ss,
    int64_t c_st,
    const T* __restrict__ k_rope, int64_t kr_ss, int64_t kr_st, int batch,
    const int32_t* __restrict__ start_pos, int n_new, uint32_t* __restrict__ flags) {
  const int lane = threadIdx.x & 31;
  if (tok >= (int64_t)batch * n_new) return;
  const int seq = (int)(tok / n_new);
  const int j = (int)(tok - (int64_t)seq * n_new);
  // the write position is loaded alongside the token's values (neither depends on the other)
  const int64_t pos = (int64_t)__ldg(start_pos + seq) + j;
  const int n = d + d_rope;
  const int groups = n >> 3;            // d % 16 == 0 and d_rope % 8 == 0
  const int d_groups = d >> 3;
  const T* crow = c_kv + (int64_t)seq * c_ss + (int64_t)j * c_st;
  const T* krow = k_rope + (int64_t)seq * kr_ss + (int64_t)j * kr_st;

  float v[kMaxRounds][8];
  float amax = 0.0f;
  bool finite = true;
#pragma unroll
  for (int r = 0; r < kMaxRounds; ++r) {
    const int g = r * 32 + lane;
    if (g < groups) {
      if (g < d_groups) load8<T>(crow + 8 * g, v[r]);
      else load8<T>(krow + 8 * (g - d_groups), v[r]);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        finite = finite && isfinite(v[r][k]);
        amax = fmaxf(amax, fabsf(v[r][k]));
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  finite = __all_sync(0xffffffffu, finite);
  if (pos < 0 || pos >= max_tokens) {
    if (lane == 0) atomicOr(flags, KVK_FLAG_WRITE_RANGE);
    return;
  }

  uint8_t* row = codes + ((int64_t)seq * max_tokens + pos) * row_bytes;
  if (group) {
    // one scale per `group` elements: each group of G elements is quantised like a token
    const int sg = n / group, lpg = group >> 3;   // scales per token, lanes per group
    __half* srow = scales + ((int64_t)seq * max_tokens + pos) * sg;
    bool bad = !finite;
#pragma unroll
    for (int r = 0; r < kMaxRounds; ++r) {
      const int g = r * 32 + lane;
      if (r * 32 >= groups) break;                        // warp-uniform
      float ga = 0.0f;
      if (g < groups) {
#pragma unroll
        for (int k = 0; k < 8; ++k) ga = fmaxf(ga, fabsf(v[r][k]));
      }
      for (int o = 1; o < lpg; o <<= 1) ga = fmaxf(ga, __shfl_xor_sync(0xffffffffu, ga, o));
      if (g >= groups) continue;
      const __half s16 = quant_scale(ga, b);
      const float s = __half2float(s16);
      bad = bad || isinf(s);
      if ((lane & (lpg - 1)) == 0) srow[(8 * g) / group] = s16;
      uint32_t u[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) u[k] = quant_field(v[r][k], s, b);
      store_fields8(row + (int64_t)g * b, u, b);
    }
    bad = __any_sync(0xffffffffu, bad);
    if (bad && lane == 0) atomicOr(flags, KVK_FLAG_NONFINITE);
    const int used = groups * b;
    if (lane < row_bytes - used) row[used + lane] = 0;
    return;
  }
  // uncompressed anchor: the bf16 of every element (round to nearest even) and scale 1
  const __half s16 = (b == KVK_BITS_BF16) ? __float2half(1.0f) : quant_scale(amax, b);
  const float s = __half2float(s16);
  if (lane == 0) {
    if (!finite || (b != KVK_BITS_BF16 && isinf(s))) atomicOr(flags, KVK_FLAG_NONFINITE);
    scales[(int64_t)seq * max_tokens + pos] = s16;
  }
  const int gb = group_bytes(b);
#pragma unroll
  for (int r = 0; r < kMaxRounds; ++r) {
    const int g = r * 32 + lane;
    if (g >= groups) continue;
    uint8_t* dst = row + (int64_t)g * gb;                // 8 elements: b bytes (16 for bf16)
    if (b == KVK_BITS_BF16) {
      store_bf16x8(dst, v[r]);
    } else {
      uint32_t u[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) u[k] = quant_field(v[r][k], s, b);
      store_fields8(dst, u, b);
    }
  }
  // zero the row padding (fewer than 16 bytes)
  const int used = groups * gb;
  if (lane < row_bytes - used) row[used + lane] = 0;
}

template <typename T>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
quant_write_kernel(uint8_t* __restrict__ codes, __half* __restrict__ scales, int row_bytes,
                   int d, int d_rope, int b, int group, int max_tokens, const T* __restrict__ c_kv,
                   int64_t c_ss, int64_t c_st, const T* __restrict__ k_rope, int64_t kr_ss,
                   int64_t kr_st, int batch, const int32_t* __restrict__ start_pos, int n_new,
                   uint32_t* __restrict__ flags) {
  quant_token<T>((int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5), codes, scales,
                 row_bytes, d, d_rope, b, group, max_tokens, c_kv, c_ss, c_st, k_rope, kr_ss,
                 kr_st, batch, start_pos, n_new, flags);
}

// Several anchor layers in one launch: blockIdx.y picks the layer.
template <typename T>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
quant_write_layers_kernel(const __grid_constant__ QuantLayers Q, int d_rope, int max_tokens,
                          int batch, const int32_t* __restrict__ start_pos, int n_new,
                          uint32_t* __restrict__ flags) {
  const QuantLayer& l = Q.l[blockIdx.y];
  quant_token<T>((int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5), l.codes, l.scales,
                 l.row_bytes, l.d, d_rope, l.b, l.group, max_tokens, static_cast<const T*>(l.c_kv),
                 l.c_ss, l.c_st, static_cast<const T*>(l.k_rope), l.kr_ss, l.kr_st, batch,
                 start_pos, n_new, flags);
}

// One warp per sequence: the new token goes to position clamp(len, 0, max_tokens) - 1.
template <typename T>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
quant_append_kernel(uint8_t* __restrict__ codes, __half* __restrict__ scales, int row_bytes,
                    int d, int d_rope, int b, int group, int max_tokens, const T* __restrict__ c_new,
                    int64_t c_ss, const T* __restrict__ kr_new, int64_t kr_ss, int batch,
                    const int32_t* __restrict__ seq_lens, uint32_t* __restrict__ flags) {
  const int i = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  if (i >= batch) return;
  const int len = min(max(__ldg(seq_lens + i), 0), max_tokens);
  if (len == 0) return;
  const int64_t r = (int64_t)i * max_tokens + (len - 1);
  const int sg = group ? (d + d_rope) / group : 1;
  if (!write_token_two_pass<T>(c_new + (int64_t)i * c_ss, kr_new + (int64_t)i * kr_ss, d,
                               d_rope, b, group, codes + r * row_bytes, row_bytes,
                               scales + r * sg) &&
      (threadIdx.x & 31) == 0)
    atomicOr(flags, KVK_FLAG_NONFINITE);
}

}  // namespace

cudaError_t launch_quant_append(const kvk_layout* L, const AnchorDesc& A, const void* c_new,
                                int dtype, int64_t c_ss, const void* kr_new, int64_t kr_ss,
                                int batch, const int32_t* seq_lens, cudaStream_t stream) {
  uint8_t* codes = L->arena + A.codes_off;
  __half* scales = reinterpret_cast<__half*>(L->arena + A.scales_off);
  uint32_t* flags = reinterpret_cast<uint32_t*>(L->arena);
  dim3 grid((unsigned)((batch + kWarpsPerBlock - 1) / kWarpsPerBlock)), block(kWarpsPerBlock * 32);
  if (dtype == KVK_BF16)
    quant_append_kernel<__nv_bfloat16><<<grid, block, 0, stream>>>(
        codes, scales, A.row_bytes, A.d, L->d_rope, A.b, anchor_group(L, A), L->max_tokens,
        static_cast<const __nv_bfloat16*>(c_new), c_ss, static_cast<const __nv_bfloat16*>(kr_new),
        kr_ss, batch, seq_lens, flags);
  else
    quant_append_kernel<float><<<grid, block, 0, stream>>>(
        codes, scales, A.row_bytes, A.d, L->d_rope, A.b, anchor_group(L, A), L->max_tokens,
        static_cast<const float*>(c_new), c_ss, static_cast<const float*>(kr_new), kr_ss, batch,
        seq_lens, flags);
  return cudaGetLastError();
}

cudaError_t launch_quant_write(const kvk_layout* L, const AnchorDesc& A, const void* c_kv,
                               int dtype, int64_t c_ss, int64_t c_st, const void* k_rope,
                               int64_t kr_ss, int64_t kr_st, int batch, const int32_t* start_pos,
                               int n_new, cudaStream_t stream) {
  const int64_t tokens = (int64_t)batch * n_new;
  const int64_t blocks = (tokens + kWarpsPerBlock - 1) / kWarpsPerBlock;
  if (blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
  uint8_t* codes = L->arena + A.codes_off;
  __half* scales = reinterpret_cast<__half*>(L->arena + A.scales_off);
  uint32_t* flags = reinterpret_cast<uint32_t*>(L->arena);
  dim3 grid((unsigned)blocks), block(kWarpsPerBlock * 32);
  if (dtype == KVK_BF16) {
    quant_write_kernel<__nv_bfloat16><<<grid, block, 0, stream>>>(
        codes, scales, A.row_bytes, A.d, L->d_rope, A.b, anchor_group(L, A), L->max_tokens,
        static_cast<const __nv_bfloat16*>(c_kv), c_ss, c_st,
        static_cast<const __nv_bfloat16*>(k_rope), kr_ss, kr_st, batch, start_pos, n_new, flags);
  } else {
    quant_write_kernel<float><<<grid, block, 0, stream>>>(
        codes, scales, A.row_bytes, A.d, L->d_rope, A.b, anchor_group(L, A), L->max_tokens,
        static_cast<const float*>(c_kv), c_ss, c_st, static_cast<const float*>(k_rope), kr_ss,
        kr_st, batch, start_pos, n_new, flags);
  }
  return cudaGetLastError();
}

cudaError_t launch_quant_write_layers(const kvk_layout* L, const QuantLayers& Q, int n, int dtype,
                                      int batch, const int32_t* start_pos, int n_new,
                                      cudaStream_t stream) {
  const int64_t tokens = (int64_t)batch * n_new;
  const int64_t blocks = (tokens + kWarpsPerBlock - 1) / kWarpsPerBlock;
  if (blocks > 0x7FFFFFFF || n < 1 || n > KVK_MAX_WRITE_LAYERS) return cudaErrorInvalidValue;
  uint32_t* flags = reinterpret_cast<uint32_t*>(L->arena);
  dim3 grid((unsigned)blocks, (unsigned)n), block(kWarpsPerBlock * 32);
  if (dtype == KVK_BF16)
    quant_write_layers_kernel<__nv_bfloat16><<<grid, block, 0, stream>>>(
        Q, L->d_rope, L->max_tokens, batch, start_pos, n_new, flags);
  else
    quant_write_layers_kernel<float><<<grid, block, 0, stream>>>(Q, L->d_rope, L->max_tokens,
                                                                 batch, start_pos, n_new, flags);
  return cudaGetLastError();
}

}  // namespace kvk
