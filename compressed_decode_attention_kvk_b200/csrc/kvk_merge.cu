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
constexpr float kLn2 = 0.6931471805599453f;

__global__ void __launch_bounds__(kMergeThreads) merge_kernel(DecodeArgs a) {
  const int i = blockIdx.x, h = blockIdx.y;
  const int64_t N = a.seq_off[a.batch];
  const int64_t s0 = a.seq_off[i], s1 = a.seq_off[i + 1];
  float* out = a.out + ((int64_t)i * a.H + h) * a.d;
  float M = -INFINITY;
  int c0 = 0, c1 = -1;
  if (s1 > s0) {
    c0 = cta_of(s0, N, a.G);
    c1 = cta_of(s1 - 1, N, a.G);
    for (int c = c0; c <= c1; ++c) {
      const int64_t sh = (int64_t)(c + i) * a.H + h;
      if (a.ws_ml[2 * sh + 1] > 0.0f) M = fmaxf(M, a.ws_ml[2 * sh]);
    }
  }
  if (M == -INFINITY) {
    for (int j = threadIdx.x; j < a.d; j += blockDim.x) out[j] = 0.0f;
    if (a.lse && threadIdx.x == 0) a.lse[(int64_t)i * a.H + h] = -INFINITY;
    return;
  }
  float lsum = 0.0f;
  for (int c = c0; c <= c1; ++c) {
    const int64_t sh = (int64_t)(c + i) * a.H + h;
    const float l = a.ws_ml[2 * sh + 1];
    if (l > 0.0f) lsum += exp2f(a.ws_ml[2 * sh] - M) * l;
  }
  const float inv = 1.0f / lsum;
  for (int j = threadIdx.x; j < a.d; j += blockDim.x) {
    float acc = 0.0f;
    for (int c = c0; c <= c1; ++c) {
      const int64_t sh = (int64_t)(c + i) * a.H + h;
      const float l = a.ws_ml[2 * sh + 1];
      if (l > 0.0f) acc = fmaf(exp2f(a.ws_ml[2 * sh] - M), a.ws_o[sh * a.d + j], acc);
    }
    out[j] = acc * inv;
  }
  if (a.lse && threadIdx.x == 0) a.lse[(int64_t)i * a.H + h] = kLn2 * (M + log2f(lsum));
}

}  // namespace

cudaError_t launch_merge(const DecodeArgs& a, cudaStream_t st) {
  if (a.H > 65535) return cudaErrorInvalidValue;
  dim3 grid(a.batch, a.H), block(kMergeThreads);
  merge_kernel<<<grid, block, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace kvk
