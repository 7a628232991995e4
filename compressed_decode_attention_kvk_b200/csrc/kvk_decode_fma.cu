// kvk_decode_fma.cu -- CUDA-core (FFMA) split decode over the packed cache.
//
// Decode attention of one layer over its anchor's compressed cache (KV-Kaizen, Background:
// "every decoded token reads the entire KV cache"; absorbed MLA form: all heads share one
// latent stream, score = sigma * s_t * (q_lat . code_t[:d] + q_rope . code_t[d:]),
// output = sum_t p_t * s_t * code_t[:d]).  This kernel runs any shape and any query dtype
// (fp32 queries always take it); the tensor-core kernel takes the large bf16/f16 shapes.
//
// Schedule: CTA c walks its slice of the flattened token space (kvk_decode_common.cuh).
// For each sequence piece and each group of 8 heads (one warp per head), tiles of TT
// tokens are dequantised into shared memory as exact integer codes (as float), every lane
// scores one token, the warp runs the online softmax (base 2), and the weighted codes
// accumulate in registers (lane j holds output features j, j+32, ...).  Partials
// (running max, weight sum, un-normalised output) go to the workspace slot of the piece.
#include <float.h>

#include "kvk_decode_common.cuh"

namespace kvk {
namespace {

constexpr int kHG = 8;   // heads per pass = warps per block
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float load_q(const float* p) { return __ldg(p); }
__device__ __forceinline__ float load_q(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ float load_q(const __half* p) { return __half2float(*p); }

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <int TT, int R, typename Tq>
__global__ void __launch_bounds__(kHG * 32) decode_fma_kernel(DecodeArgs a) {
  extern __shared__ float4 smem4[];
  float* smem = reinterpret_cast<float*>(smem4);
  const int n = a.n, d = a.d;
  const int ldc = n + 1;
  float* qs = smem;                                        // [kHG][n]
  float* cs = qs + kHG * n;                                // [TT][n + 1]
  float* ss = cs + TT * ldc;                               // [TT]
  int32_t* tokidx = reinterpret_cast<int32_t*>(ss + TT);   // [TT]
  int32_t* tmp = tokidx + TT;                              // [32]
  int32_t* off = tmp + 32;                                 // [batch + 1]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nt = blockDim.x;

  block_seq_offsets(a, off, tmp);
  if (blockIdx.x == 0)
    for (int i = tid; i <= a.batch; i += nt) a.seq_off[i] = off[i];
  const int64_t C = off[a.batch] + (int64_t)a.split_x * a.batch;
  const int c = blockIdx.x;
  const int64_t lo = split_token(off, a.batch, a.split_x, split_cost(c, C, a.G));
  const int64_t hi = split_token(off, a.batch, a.split_x, split_cost(c + 1, C, a.G));
  if (lo >= hi) return;
  // first sequence whose token range contains lo
  int seq = 0;
  {
    int L = 0, H = a.batch;  // largest i with off[i] <= lo
    while (L < H) {
      int mid = (L + H + 1) >> 1;
      if (off[mid] <= lo) L = mid; else H = mid - 1;
    }
    seq = L;
  }
  const Tq* qlat = static_cast<const Tq*>(a.q_lat);
  const Tq* qrope = static_cast<const Tq*>(a.q_rope);
  // b = KVK_BITS_BF16: 16-bit fields holding bf16 values instead of offset-binary codes
  const bool bf16_rows = (a.b == KVK_BITS_BF16);
  const int b = bf16_rows ? 16 : a.b;
  const uint32_t mask = (1u << b) - 1u;
  const int zero_off = 1 << (b - 1);
  const float zscale = a.sigma * kLog2e;

  for (; seq < a.batch && off[seq] < hi; ++seq) {
    const int64_t s0 = max(lo, (int64_t)off[seq]), s1 = min(hi, (int64_t)off[seq + 1]);
    if (s0 >= s1) continue;
    const int p0 = (int)(s0 - off[seq]), p1 = (int)(s1 - off[seq]);
    const int slot = c + seq;
    const int seq_len = clamped_len(a, seq);
    const int64_t seq_row0 = (int64_t)seq * a.max_tokens;
    for (int hg = 0; hg < a.H; hg += kHG) {
      const int h = hg + warp;
      const bool hv = h < a.H;
      __syncthreads();
      for (int k = lane; k < n; k += 32) {
        float v = 0.0f;
        if (hv) {
          v = (k < d) ? load_q(qlat + seq * a.ql_ss + h * a.ql_sh + k)
                      : load_q(qrope + seq * a.qr_ss + h * a.qr_sh + (k - d));
        }
        qs[warp * n + k] = v;
      }
      float m = -INFINITY;
      float l = 0.0f;
      float o[R];
#pragma unroll
      for (int r = 0; r < R; ++r) o[r] = 0.0f;

      for (int p = p0; p < p1; p += TT) {
        const int cnt = min(TT, p1 - p);
        __syncthreads();
        if (tid < TT) {
          int t = (tid < cnt) ? token_at(a, seq, p + tid, seq_len) : -1;
          tokidx[tid] = t;
          // a group-scaled cache carries its scales per element (below): unit token scale
          ss[tid] = (t >= 0) ? (a.group ? 1.0f : __half2float(a.scales[seq_row0 + t])) : 0.0f;
        }
        __syncthreads();
        for (int e = tid; e < TT * n; e += nt) {
          const int i = e / n, k = e - i * n;
          const int t = tokidx[i];
          float v = 0.0f;
          if (t >= 0) {
            const uint32_t* row =
                reinterpret_cast<const uint32_t*>(a.codes + (seq_row0 + t) * a.row_bytes);
            const int bit = k * b;
            const uint32_t w = __ldg(row + (bit >> 5));
            const uint32_t u = (w >> (bit & 31)) & mask;
            v = bf16_rows ? __uint_as_float(u << 16) : (float)((int)u - zero_off);
            if (a.group) v *= __half2float(a.scales[(seq_row0 + t) * a.sg + k / a.group]);
          }
          cs[i * ldc + k] = v;
        }
        __syncthreads();
        float z2 = -INFINITY;
        if (hv && lane < cnt && tokidx[lane] >= 0) {
          float acc = 0.0f;
          const float* qr = qs + warp * n;
          const float* cr = cs + lane * ldc;
          for (int k = 0; k < n; ++k) acc = fmaf(qr[k], cr[k], acc);
          z2 = acc * ss[lane] * zscale;
        }
        const float mn = fmaxf(m, warp_max(z2));
        const float alpha = (m == -INFINITY || mn == -INFINITY) ? 0.0f : exp2f(m - mn);
        const float pz = (z2 == -INFINITY) ? 0.0f : exp2f(z2 - mn);
        l = l * alpha + warp_sum(pz);
        const float wgt = pz * ss[lane];
#pragma unroll
        for (int r = 0; r < R; ++r) o[r] *= alpha;
        for (int i = 0; i < cnt; ++i) {
          const float wi = __shfl_sync(0xffffffffu, wgt, i);
          const float* cr = cs + i * ldc;
#pragma unroll
          for (int r = 0; r < R; ++r) {
            const int j = lane + 32 * r;
            if (j < d) o[r] = fmaf(wi, cr[j], o[r]);
          }
        }
        m = mn;
      }
      if (hv) {
        const int64_t sh = (int64_t)slot * a.H + h;
        if (lane == 0) {
          a.ws_ml[2 * sh] = m;
          a.ws_ml[2 * sh + 1] = l;
        }
        float* dst = a.ws_o + sh * d;
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const int j = lane + 32 * r;
          if (j < d) dst[j] = o[r];
        }
      }
    }
  }
}

template <int TT, int R>
cudaError_t launch_tt_r(const DecodeArgs& a, int dtype, size_t smem, cudaStream_t st) {
  dim3 grid(a.G), block(kHG * 32);
  cudaError_t e = cudaSuccess;
#define KVK_LAUNCH(T)                                                                   \
  do {                                                                                  \
    auto k = decode_fma_kernel<TT, R, T>;                                               \
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
    if (e != cudaSuccess) return e;                                                     \
    k<<<grid, block, smem, st>>>(a);                                                    \
  } while (0)
  if (dtype == KVK_F32) KVK_LAUNCH(float);
  else if (dtype == KVK_BF16) KVK_LAUNCH(__nv_bfloat16);
  else KVK_LAUNCH(__half);
#undef KVK_LAUNCH
  return cudaGetLastError();
}

template <int TT>
cudaError_t launch_tt(const DecodeArgs& a, int dtype, size_t smem, cudaStream_t st) {
  if (a.d <= 64) return launch_tt_r<TT, 2>(a, dtype, smem, st);
  if (a.d <= 128) return launch_tt_r<TT, 4>(a, dtype, smem, st);
  if (a.d <= 512) return launch_tt_r<TT, 16>(a, dtype, smem, st);
  return launch_tt_r<TT, 64>(a, dtype, smem, st);
}

size_t smem_bytes(int TT, int n, int batch) {
  return sizeof(float) * ((size_t)kHG * n + (size_t)TT * (n + 1) + TT) +
         sizeof(int32_t) * ((size_t)TT + 32 + batch + 1);
}

}  // namespace

cudaError_t launch_decode_fma(const DecodeArgs& a, int dtype, cudaStream_t st) {
  size_t s32 = smem_bytes(32, a.n, a.batch);
  if (s32 <= 227 * 1024) return launch_tt<32>(a, dtype, s32, st);
  size_t s16 = smem_bytes(16, a.n, a.batch);
  if (s16 <= 227 * 1024) return launch_tt<16>(a, dtype, s16, st);
  return cudaErrorInvalidValue;
}

}  // namespace kvk
