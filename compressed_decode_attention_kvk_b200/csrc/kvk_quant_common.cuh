// kvk_quant_common.cuh -- the per-element steps of quantise-on-write, shared by the write
// kernel (kvk_quant.cu) and the decode kernel's fused append (kvk_decode_tc.cu), so that a
// token appended inside a decode is stored bit for bit as the write kernel stores it.
//
// KV-Kaizen, "Three Non-Eviction Compression Axes", item 3 (precision): b-bit symmetric
// uniform codes with one scale per token.  Scale: s = fp16(absmax / (2^(b-1) - 1)) rounded
// toward +inf (IEEE binary32 division first); code = clamp(round_half_even(v / s), +-q); the
// stored field is code + 2^(b-1), packed little-endian at b bits per element.  An
// uncompressed anchor (KVK_BITS_BF16) stores bf16(v) (round to nearest even) and scale 1.
#pragma once

#include "kvk_internal.cuh"

namespace kvk {

template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&v)[8]);

template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    // a bf16 is the high half of a binary32: widening is exact
    v[2 * k] = __uint_as_float(w[k] << 16);
    v[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
  }
}

// fp16 scale of a token with max |v| = amax at b bits
__device__ __forceinline__ __half quant_scale(float amax, int b) {
  const int q = (1 << (b - 1)) - 1;
  const float s32 = __fdiv_rn(amax, (float)q);   // IEEE binary32 division
  return __float2half_ru(s32);                    // rounded toward +inf
}

// offset-binary field of one element under the stored scale s
__device__ __forceinline__ uint32_t quant_field(float v, float s, int b) {
  const int q = (1 << (b - 1)) - 1;
  int c = 0;
  if (s != 0.0f) {
    c = __float2int_rn(__fdiv_rn(v, s));          // round half to even
    c = min(max(c, -q), q);
  }
  return (uint32_t)(c + (1 << (b - 1)));
}

// the b bytes holding eight consecutive fields (8 elements x b bits)
__device__ __forceinline__ void store_fields8(uint8_t* dst, const uint32_t (&u)[8], int b) {
  if (b == 16) {
    *reinterpret_cast<uint4*>(dst) = make_uint4(u[0] | (u[1] << 16), u[2] | (u[3] << 16),
                                                u[4] | (u[5] << 16), u[6] | (u[7] << 16));
  } else if (b == 8) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(u[0] | (u[1] << 8) | (u[2] << 16) | (u[3] << 24),
                                                u[4] | (u[5] << 8) | (u[6] << 16) | (u[7] << 24));
  } else if (b == 4) {
    uint32_t w = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) w |= u[k] << (4 * k);
    *reinterpret_cast<uint32_t*>(dst) = w;
  } else {   // b == 2
    uint32_t w = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) w |= u[k] << (2 * k);
    *reinterpret_cast<uint16_t*>(dst) = (uint16_t)w;
  }
}

// the 16 bytes holding eight consecutive bf16 elements of an uncompressed row
__device__ __forceinline__ void store_bf16x8(uint8_t* dst, const float (&v)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const __nv_bfloat162 h2 = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
    w[k] = *reinterpret_cast<const uint32_t*>(&h2);
  }
  *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
}

// Bytes of one packed group of eight elements.
__device__ __forceinline__ int group_bytes(int b) { return b == KVK_BITS_BF16 ? 16 : b; }

// One warp writes one token: v = [c[0..d) || k^R[0..d_rope)] read from crow / krow, stored in
// `row` (row_bytes, padding zeroed) with its scale(s) at `scale` (one per token, or one per
// `group` elements when group > 0).  Two passes over the inputs (the max, then the fields), so
// a lane holds only eight values at a time; the arithmetic is that of the single-pass write
// kernel.  Returns false (in every lane) if an input is not finite or a scale overflows fp16
// (the stored token is then unspecified).
template <typename T>
__device__ __forceinline__ bool write_token_two_pass(const T* crow, const T* krow, int d,
                                                     int d_rope, int b, int group, uint8_t* row,
                                                     int row_bytes, __half* scale) {
  const int lane = threadIdx.x & 31;
  const int groups = (d + d_rope) >> 3, d_groups = d >> 3;
  const int gb = group_bytes(b);
  auto load = [&](int g, float (&v)[8]) {
    if (g < d_groups) load8<T>(crow + 8 * g, v);
    else load8<T>(krow + 8 * (g - d_groups), v);
  };
  bool ok = true;
  if (group) {   // one scale per `group` elements: one pass, a round of 32 lanes at a time
    const int lpg = group >> 3;
    for (int g0 = 0; g0 < groups; g0 += 32) {
      const int g = g0 + lane;
      float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      float ga = 0.0f;
      if (g < groups) {
        load(g, v);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          ok = ok && isfinite(v[k]);
          ga = fmaxf(ga, fabsf(v[k]));
        }
      }
      for (int o = 1; o < lpg; o <<= 1) ga = fmaxf(ga, __shfl_xor_sync(0xffffffffu, ga, o));
      if (g < groups) {
        const __half s16 = quant_scale(ga, b);
        const float s = __half2float(s16);
        ok = ok && !isinf(s);
        if ((lane & (lpg - 1)) == 0) scale[(8 * g) / group] = s16;
        uint32_t u[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) u[k] = quant_field(v[k], s, b);
        store_fields8(row + (int64_t)g * gb, u, b);
      }
    }
  } else {
    float amax = 0.0f;
    for (int g = lane; g < groups; g += 32) {
      float v[8];
      load(g, v);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        ok = ok && isfinite(v[k]);
        amax = fmaxf(amax, fabsf(v[k]));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    __half s16 = __float2half(1.0f);
    if (b != KVK_BITS_BF16) s16 = quant_scale(amax, b);
    const float s = __half2float(s16);
    ok = ok && (b == KVK_BITS_BF16 || !isinf(s));
    if (lane == 0) *scale = s16;
    for (int g = lane; g < groups; g += 32) {
      float v[8];
      load(g, v);
      if (b == KVK_BITS_BF16) {
        store_bf16x8(row + (int64_t)g * gb, v);
      } else {
        uint32_t u[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) u[k] = quant_field(v[k], s, b);
        store_fields8(row + (int64_t)g * gb, u, b);
      }
    }
  }
  const int used = groups * gb;
  if (lane < row_bytes - used) row[used + lane] = 0;
  return __all_sync(0xffffffffu, ok);
}

}  // namespace kvk
