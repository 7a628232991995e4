// kvk_decode_common.cuh -- pieces shared by the two decode kernels: the balanced split of
// the flattened token space over CTAs, and the per-sequence token lists.
//
// Token space: sequence i contributes n_i tokens (its seq_len, or its keep_len when a keep
// list is given); the n_i are laid end to end, N = sum n_i, and CTA c owns positions
// [c*N/G, (c+1)*N/G).  A CTA whose range crosses sequence boundaries produces one partial
// result ("piece") per sequence it touches, written to workspace slot c + i.  The merge
// combines, for sequence i, the slots c + i of every CTA c whose range meets it.
#pragma once

#include <utility>

#include "kvk_internal.cuh"

namespace kvk {

// Programmatic dependent launch.  The decode kernels and the merge are launched with
// programmatic stream serialisation: a kernel may start while the one before it in the
// stream finishes, and griddep_wait() returns once that kernel has completed and its memory
// is visible (at once when it was launched the ordinary way).  griddep_trigger() lets the
// next kernel launch before this one completes.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// cudaLaunchKernelEx with programmatic stream serialisation
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Clamped token count of sequence i without raising flags.
__device__ __forceinline__ int seq_tokens_quiet(const DecodeArgs& a, int i, bool* bad) {
  int len = __ldg(a.seq_lens + i);
  int cl = min(max(len, 0), a.max_tokens);
  *bad = (cl != len);
  if (a.keep_idx) {
    int k = __ldg(a.keep_len + i);
    int ck = min(max(k, 0), a.keep_stride);
    *bad = *bad || (ck != k);
    cl = ck;
  }
  return cl;
}

// Exclusive prefix sum of the token counts into smem_off[0..batch], computed by the whole
// block (blockDim a multiple of 32, at most 1024).  smem_tmp needs 32 entries.  Only block 0
// raises KVK_FLAG_SEQ_LEN, so each condition is reported once per call.
__device__ inline void block_seq_offsets(const DecodeArgs& a, int32_t* smem_off,
                                         int32_t* smem_tmp) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int per = (a.batch + nt - 1) / nt;
  const int begin = min(a.batch, tid * per), end = min(a.batch, begin + per);
  int local = 0;
  bool bad_any = false;
  for (int i = begin; i < end; ++i) {
    bool bad;
    local += seq_tokens_quiet(a, i, &bad);
    bad_any = bad_any || bad;
  }
  if (bad_any && blockIdx.x == 0) atomicOr(a.flags, KVK_FLAG_SEQ_LEN);
  const int lane = tid & 31, w = tid >> 5;
  int x = local;  // inclusive warp scan
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) smem_tmp[w] = x;
  __syncthreads();
  if (w == 0) {
    const int nw = nt >> 5;
    int t = lane < nw ? smem_tmp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    __syncwarp();
    if (lane < nw) smem_tmp[lane] = t;  // inclusive prefix of warp totals
  }
  __syncthreads();
  int run = x - local + (w > 0 ? smem_tmp[w - 1] : 0);
  for (int i = begin; i < end; ++i) {
    bool bad;
    smem_off[i] = run;
    run += seq_tokens_quiet(a, i, &bad);
  }
  if (begin < end && end == a.batch) smem_off[a.batch] = run;
  __syncthreads();
}

// Physical token index of position p of sequence i (the keep list maps positions to
// tokens).  Returns -1 for an invalid keep entry.
__device__ __forceinline__ int token_at(const DecodeArgs& a, int i, int p, int seq_len) {
  if (!a.keep_idx) return p;
  int t = __ldg(a.keep_idx + (int64_t)i * a.keep_stride + p);
  if (t < 0 || t >= seq_len) {
    atomicOr(a.flags, KVK_FLAG_KEEP_INDEX);
    return -1;
  }
  return t;
}

__device__ __forceinline__ int clamped_len(const DecodeArgs& a, int i) {
  int len = __ldg(a.seq_lens + i);
  return min(max(len, 0), a.max_tokens);
}

}  // namespace kvk
