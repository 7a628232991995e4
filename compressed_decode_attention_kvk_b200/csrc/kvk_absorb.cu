// kvk_absorb.cu -- the absorbed MLA projections on either side of the decode, on the
// 5th-generation tensor core:
//     y[b, h, j] = sum_k x[b, h, k] * w[h, k, j]        (b < batch, h < heads, j < n, k < K)
// q_lat = q_nope . W_UK (the query taken into the latent space, only the first d columns a
// layer keeps: the rank axis) and the heads' values = out_lat . W_UV (the decode output taken
// back out of it, only the first d rows), "Three Non-Eviction Compression Axes", item 2, with
// the absorbed MLA form of the decode.
//
// One CTA per (head, 128 columns of y, 32 rows of the batch): the weight tile w[h, 0..K,
// j0..j0+128) arrives by TMA as MN-major 128-byte-swizzled boxes of 64 rows x 64 columns, the
// batch rows of x are written by the CTA's threads as K-major 128-byte-swizzled rows (an fp32
// x as two bf16 parts, hi = bf16(x) and lo = bf16(x - hi), each its own set of MMAs), one
// thread issues the K / 16 MMAs D[128 x 32] (+)= W^T . X^T (M = 128 columns of y on the TMEM
// lanes, N = 32 batch rows), and the epilogue reads D back (32 lanes per warp) and writes y.
// Weights are read once per batch chunk; the kernel is bound by the weight bytes.
#include <string.h>

#include "kvk_internal.cuh"
#include "kvk_sm100.cuh"

namespace kvk {
namespace {

using namespace sm100;

constexpr int kAbThreads = 128;
constexpr int kAbM = 128;          // columns of y per CTA (TMEM lanes)
constexpr int kAbN = 32;           // batch rows per CTA (MMA N, TMEM columns)
constexpr int kBox = 8192;         // one TMA box: 64 weight rows x 64 columns of bf16
constexpr uint64_t kAbLimitNs = 2000000000ull;

struct AbsorbParams {
  const void* x;
  int64_t x_ss, x_sh;
  int x_f32;
  void* y;
  int64_t y_ss, y_sh;
  int y_f32;
  int batch, heads, K, n;
  uint32_t idesc;
  uint32_t* flags;   // nullable: KVK_FLAG_TIMEOUT on a wait that ran out
};

// bf16 instruction descriptor, f32 accumulation: A MN-major (the weight), B K-major (x rows)
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ uint32_t bf16x2_bits(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__global__ void __launch_bounds__(kAbThreads, 1)
absorb_kernel(const __grid_constant__ AbsorbParams P, const __grid_constant__ CUtensorMap wmap) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int K = P.K, nkb = K / 64;
  // layout: weight boxes [nkb][2] (8 KB each), x rows (hi, then lo for fp32 x) as K-major
  // 128-byte-swizzled atoms [nkb][32 rows][128 B], then two mbarriers and the TMEM address
  uint8_t* wbuf = smem;
  uint8_t* xhi = wbuf + (size_t)nkb * 2 * kBox;
  uint8_t* xlo = xhi + (size_t)nkb * kAbN * 128;
  uint8_t* tail = xlo + (P.x_f32 ? (size_t)nkb * kAbN * 128 : 0);
  uint64_t* bar_w = reinterpret_cast<uint64_t*>(tail);
  uint64_t* bar_d = bar_w + 1;
  uint32_t* tbase = reinterpret_cast<uint32_t*>(bar_d + 1);
  uint32_t* abort_word = tbase + 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x, j0 = blockIdx.y * kAbM, b0 = blockIdx.z * kAbN;
  if (tid == 0) {
    mbar_init(bar_w, 1);
    mbar_init(bar_d, 1);
    *abort_word = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tbase, 32);
    tmem_relinquish();
  }
  __syncthreads();
  // the weight tile: rows 0..K of head h, columns j0..j0+128 (columns past n read as zero)
  if (tid == 0) {
    tma_prefetch_desc(&wmap);
    mbar_arrive_expect_tx(bar_w, (uint32_t)(nkb * 2 * kBox));
    for (int kb = 0; kb < nkb; ++kb)
      for (int a = 0; a < 2; ++a)
        tma_load_3d(wbuf + (size_t)(kb * 2 + a) * kBox, &wmap, j0 + 64 * a, 64 * kb, h, bar_w);
  }
  // the batch rows of x, as 16-byte chunks of 8 elements: row r, chunk c (k = 8c .. 8c+7)
  // goes to atom c / 8, row r, 16-byte slot (c % 8) ^ (r % 8); rows past the batch are zero
  const int chunks = K / 8;
  for (int e = tid; e < kAbN * chunks; e += kAbThreads) {
    const int r = e / chunks, c = e - r * chunks;
    const int b = b0 + r;
    uint4 hi = make_uint4(0u, 0u, 0u, 0u), lo = hi;
    if (b < P.batch) {
      if (P.x_f32) {
        const float* px = static_cast<const float*>(P.x) + (int64_t)b * P.x_ss +
                          (int64_t)h * P.x_sh + 8 * c;
        const float4 u = *reinterpret_cast<const float4*>(px);
        const float4 v = *reinterpret_cast<const float4*>(px + 4);
        const float f[8] = {u.x, u.y, u.z, u.w, v.x, v.y, v.z, v.w};
        uint32_t wh[4], wl[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          wh[i] = bf16x2_bits(f[2 * i], f[2 * i + 1]);
          const float h0 = __uint_as_float(wh[i] << 16), h1 = __uint_as_float(wh[i] & 0xFFFF0000u);
          wl[i] = bf16x2_bits(f[2 * i] - h0, f[2 * i + 1] - h1);   // exact differences
        }
        hi = make_uint4(wh[0], wh[1], wh[2], wh[3]);
        lo = make_uint4(wl[0], wl[1], wl[2], wl[3]);
      } else {
        hi = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(P.x) +
                                             (int64_t)b * P.x_ss + (int64_t)h * P.x_sh + 8 * c);
      }
    }
    const size_t at = (size_t)(c >> 3) * kAbN * 128 + r * 128 + (((c & 7) ^ (r & 7)) << 4);
    *reinterpret_cast<uint4*>(xhi + at) = hi;
    if (P.x_f32) *reinterpret_cast<uint4*>(xlo + at) = lo;
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tbase;
  const uint32_t abort = smem_u32(abort_word);
  bool ok = true;
  if (warp == 0) {
    ok = __all_sync(0xffffffffu, mbar_wait(bar_w, 0u, abort, kAbLimitNs));
    if (ok) {
      tc_fence_after();
      // A = W^T (M = 128 columns, MN-major): the two 64-column boxes of a row block are 8 KB
      // apart (leading byte offset), 8-row groups 1024 B apart (stride byte offset); K step 16
      // = 2048 B inside a box.  B = x rows (N = 32, K-major): 8-row groups 1024 B apart.
      const uint64_t a0 = sdesc(smem_u32(wbuf), (uint32_t)kBox, 1024u, kLayoutSw128);
      const uint64_t bh0 = sdesc(smem_u32(xhi), 16u, 1024u, kLayoutSw128);
      const uint64_t bl0 = sdesc(smem_u32(xlo), 16u, 1024u, kLayoutSw128);
      const int parts = P.x_f32 ? 2 : 1;
      for (int kb = 0; kb < nkb; ++kb) {
        const uint64_t ad = a0 + ((uint32_t)(kb * 2 * kBox) >> 4);
        for (int part = 0; part < parts; ++part) {
          const uint64_t bd = (part ? bl0 : bh0) + ((uint32_t)(kb * kAbN * 128) >> 4);
          mma4_elect(tmem, ad, 2048u >> 4, bd, 32u >> 4, P.idesc, (kb > 0 || part > 0) ? 1u : 0u);
        }
      }
      commit_elect(bar_d);
    }
  }
  __syncwarp();
  // every warp waits for the MMAs (or, after a failed weight wait, stops at once)
  ok = __all_sync(0xffffffffu, ok && mbar_wait(bar_d, 0u, abort, kAbLimitNs));
  tc_fence_after();
  if (ok) {
    // epilogue: warp w holds columns j0 + 32 w + lane of y, every batch row of the chunk
    float v[32];
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(tmem + ((uint32_t)(32 * warp) << 16)));
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
    const int j = j0 + 32 * warp + lane;
    if (j < P.n) {
#pragma unroll
      for (int i = 0; i < kAbN; ++i) {
        const int b = b0 + i;
        if (b >= P.batch) break;
        const int64_t o = (int64_t)b * P.y_ss + (int64_t)h * P.y_sh + j;
        if (P.y_f32) static_cast<float*>(P.y)[o] = v[i];
        else static_cast<__nv_bfloat16*>(P.y)[o] = __float2bfloat16_rn(v[i]);
      }
    }
  } else if (tid == 0 && P.flags) {
    atomicOr(P.flags, KVK_FLAG_TIMEOUT);
  }
  // the weight loads have landed before the block exits (a normal run waited for them)
  if (tid == 0) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try(bar_w, 0u) && globaltimer() - t0 < kAbLimitNs) {
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 32);
  }
}

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

}  // namespace

size_t absorb_smem_bytes(int K, int x_f32) {
  const size_t nkb = (size_t)K / 64;
  return nkb * 2 * kBox + nkb * kAbN * 128 * (x_f32 ? 2 : 1) + 64 + 1024;
}

// w: [heads][K rows][n columns] at w[h * w_sh + k * w_sk + j] (bf16; strides in elements)
cudaError_t launch_absorb(const void* x, int x_f32, int64_t x_ss, int64_t x_sh, const void* w,
                          int64_t w_sk, int64_t w_sh, void* y, int y_f32, int64_t y_ss,
                          int64_t y_sh, int batch, int heads, int K, int n, uint32_t* flags,
                          cudaStream_t st) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  CUtensorMap m;
  const cuuint64_t dims[3] = {(cuuint64_t)n, (cuuint64_t)K, (cuuint64_t)heads};
  const cuuint64_t strides[2] = {(cuuint64_t)w_sk * 2, (cuuint64_t)w_sh * 2};
  const cuuint32_t box[3] = {64, 64, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  if (fn(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(w), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  AbsorbParams P;
  memset(&P, 0, sizeof(P));
  P.x = x;
  P.x_ss = x_ss;
  P.x_sh = x_sh;
  P.x_f32 = x_f32;
  P.y = y;
  P.y_ss = y_ss;
  P.y_sh = y_sh;
  P.y_f32 = y_f32;
  P.batch = batch;
  P.heads = heads;
  P.K = K;
  P.n = n;
  P.idesc = idesc_bf16(kAbM, kAbN, true, false);
  P.flags = flags;
  const size_t smem = absorb_smem_bytes(K, x_f32);
  cudaError_t e =
      cudaFuncSetAttribute(absorb_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(heads, (n + kAbM - 1) / kAbM, (batch + kAbN - 1) / kAbN);
  absorb_kernel<<<grid, kAbThreads, smem, st>>>(P, m);
  return cudaGetLastError();
}

}  // namespace kvk
