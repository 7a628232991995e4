// kvk_merge.cu -- log-sum-exp merge of the split-decode partials into the layer output.
//
// For sequence i and head h, the pieces j (one per CTA whose token slice meets the
// sequence) hold a running max m_j (log2 units), a weight sum l_j = sum 2^(z2 - m_j) and
// an un-normalised output o_j = sum 2^(z2 - m_j) * c_hat[:d].  With M = max_j m_j and
// w_j = 2^(m_j - M):
//     out = sum_j w_j o_j / sum_j w_j l_j,   lse = ln 2 * (M + log2 sum_j w_j l_j).
// An empty token set (no piece, or every weight zero) gives out = 0 and lse = -inf.
#include <float.h>

#include "kvk_decode_common.cuh"

namespace kvk {
namespace {

constexpr int kMergeThreads = 128;
constexpr int kChunk = 256;   // pieces whose weights are staged in shared memory at once
constexpr int kFew = 8;       // at most this many pieces: single-round register path
constexpr float kLn2 = 0.6931471805599453f;

template <bool kMax>
__device__ __forceinline__ float block_reduce(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float u = __shfl_xor_sync(0xffffffffu, v, o);
    v = kMax ? fmaxf(v, u) : v + u;
  }
  const int w = threadIdx.x >> 5;
  __syncthreads();   // red[] free from any earlier use
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  v = red[0];
  for (int k = 1; k < kMergeThreads / 32; ++k) v = kMax ? fmaxf(v, red[k]) : v + red[k];
  return v;
}

// One CTA per (sequence, head).  The pieces' (m, l) are reduced by the whole block; the
// outputs are then accumulated four features per thread, the pieces' loads independent of
// one another (weights staged in shared memory), so the kernel streams the partials instead
// of waiting on one load per piece.
__global__ void __launch_bounds__(kMergeThreads, 4) merge_kernel(DecodeArgs a) {
  __shared__ float w_s[kChunk];
  __shared__ float red[kMergeThreads / 32];
  // Let the next kernel in the stream (the next layer's decode) launch once every block of
  // this grid has started: its blocks then set up on the SMs this grid leaves and wait for
  // this grid to complete before they read or write anything it uses.
  griddep_trigger();
  griddep_wait();   // the decode's partials are complete and visible
  const int i = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  const int64_t C = a.seq_off[a.batch] + (int64_t)a.split_x * a.batch;
  const int64_t s0 = a.seq_off[i], s1 = a.seq_off[i + 1];
  float* out = a.out + ((int64_t)i * a.H + h) * a.d;
  int c0 = 0, np = 0;
  if (s1 > s0) {   // token t of sequence i sits at cost position t + X (i + 1)
    const int64_t u = (int64_t)a.split_x * (i + 1);
    c0 = split_cta(s0 + u, C, a.G);
    np = split_cta(s1 - 1 + u, C, a.G) - c0 + 1;
  }
  // CTAs c0 .. c0 + np - 1 hold the pieces; with fewer cost units than CTAs some of them own
  // nothing and wrote no partials (their slots are skipped)
  const bool dense = C >= a.G;
  auto live = [&](int k) {
    return dense || split_cost(c0 + k + 1, C, a.G) > split_cost(c0 + k, C, a.G);
  };
  auto ml = [&](int k) -> float2 {   // (m, l) of piece k of this sequence and head
    if (!live(k)) return make_float2(0.f, 0.f);
    const int64_t sh = (int64_t)(c0 + k + i) * a.H + h;
    return *reinterpret_cast<const float2*>(a.ws_ml + 2 * sh);
  };
  const int d4 = a.d >> 2;   // d is a multiple of 16
  if (np <= kFew && d4 <= kMergeThreads) {
    // Few pieces (the usual case): every thread loads all pieces' (m, l) and its four output
    // features of every piece in one round of independent loads, then reduces in registers.
    float2 mlv[kFew];
    float4 ov[kFew];
    const float4* src =
        reinterpret_cast<const float4*>(a.ws_o + ((int64_t)(c0 + i) * a.H + h) * a.d) + tid;
    const int64_t stride = (int64_t)a.H * d4;   // float4s between consecutive pieces
#pragma unroll
    for (int k = 0; k < kFew; ++k) {
      mlv[k] = make_float2(0.f, 0.f);
      ov[k] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (k < np && live(k)) {
        mlv[k] = ml(k);
        if (tid < d4) ov[k] = src[k * stride];
      }
    }
    float M = -INFINITY;
#pragma unroll
    for (int k = 0; k < kFew; ++k)
      if (k < np && mlv[k].y > 0.0f) M = fmaxf(M, mlv[k].x);
    if (M == -INFINITY) {
      if (tid < d4) reinterpret_cast<float4*>(out)[tid] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (a.lse && tid == 0) a.lse[(int64_t)i * a.H + h] = -INFINITY;
      return;
    }
    float lsum = 0.0f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < kFew; ++k) {
      if (k < np && mlv[k].y > 0.0f) {
        const float w = exp2f(mlv[k].x - M);
        lsum += w * mlv[k].y;
        acc.x = fmaf(w, ov[k].x, acc.x);
        acc.y = fmaf(w, ov[k].y, acc.y);
        acc.z = fmaf(w, ov[k].z, acc.z);
        acc.w = fmaf(w, ov[k].w, acc.w);
      }
    }
    const float inv = 1.0f / lsum;
    if (tid < d4)
      reinterpret_cast<float4*>(out)[tid] =
          make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    if (a.lse && tid == 0) a.lse[(int64_t)i * a.H + h] = kLn2 * (M + log2f(lsum));
    return;
  }
  float M = -INFINITY;
  for (int k = tid; k < np; k += kMergeThreads) {
    const float2 v = ml(k);
    if (v.y > 0.0f) M = fmaxf(M, v.x);
  }
  M = block_reduce<true>(M, red);
  if (M == -INFINITY) {
    for (int j = tid; j < a.d; j += kMergeThreads) out[j] = 0.0f;
    if (a.lse && tid == 0) a.lse[(int64_t)i * a.H + h] = -INFINITY;
    return;
  }
  float ls = 0.0f;
  for (int k = tid; k < np; k += kMergeThreads) {
    const float2 v = ml(k);
    if (v.y > 0.0f) ls += exp2f(v.x - M) * v.y;
  }
  const float lsum = block_reduce<false>(ls, red);
  const float inv = 1.0f / lsum;
  for (int j0 = 0; j0 < d4; j0 += kMergeThreads) {
    const int j = j0 + tid;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k0 = 0; k0 < np; k0 += kChunk) {
      const int nk = min(kChunk, np - k0);
      __syncthreads();   // previous chunk's weights consumed
      for (int k = tid; k < nk; k += kMergeThreads) {
        const float2 v = ml(k0 + k);
        w_s[k] = (v.y > 0.0f) ? exp2f(v.x - M) : 0.0f;
      }
      __syncthreads();
      if (j < d4) {
        const float4* src = reinterpret_cast<const float4*>(
            a.ws_o + ((int64_t)(c0 + k0 + i) * a.H + h) * a.d) + j;
        const int64_t stride = (int64_t)a.H * d4;   // float4s between consecutive pieces
#pragma unroll 4
        for (int k = 0; k < nk; ++k) {
          const float w = w_s[k];
          if (w != 0.0f) {
            const float4 v = src[k * stride];
            acc.x = fmaf(w, v.x, acc.x);
            acc.y = fmaf(w, v.y, acc.y);
            acc.z = fmaf(w, v.z, acc.z);
            acc.w = fmaf(w, v.w, acc.w);
          }
        }
      }
    }
    if (j < d4)
      reinterpret_cast<float4*>(out)[j] =
          make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  }
  if (a.lse && tid == 0) a.lse[(int64_t)i * a.H + h] = kLn2 * (M + log2f(lsum));
}

}  // namespace

cudaError_t launch_merge(const DecodeArgs& a, cudaStream_t st) {
  if (a.H > 65535) return cudaErrorInvalidValue;
  dim3 grid(a.batch, a.H), block(kMergeThreads);
  // a programmatic dependent of the decode: its blocks start as the decode's finish
  cudaError_t e = launch_pdl(merge_kernel, grid, block, 0, st, a);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace kvk
