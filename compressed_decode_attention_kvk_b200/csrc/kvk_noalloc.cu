// kvk_noalloc.cu -- kvk_mla_decode_noalloc: the decode entry point for callers that cannot
// allocate device memory.  The workspace of kvk_mla_decode is replaced by one file-scope
// device array; nothing here allocates (no cudaMalloc / cudaFree, no allocating library
// call).  See include/kvk.h for the contract (size limit, first-call set-up, sharing).
#include <atomic>

#include "kvk_internal.cuh"

namespace {

// Scratch for the split-decode partials and sequence offsets.  Lives as long as the
// library's module is loaded on a device; contents persist from call to call.
static __device__ __align__(256) unsigned char g_noalloc_scratch[KVK_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_ptr[kMaxDevices];

// Device address of the scratch array on device `dev` (which is current), looked up once per
// device.  The array's name in host code is only a host-side handle; the kernels must be
// given the address cudaGetSymbolAddress returns.
kvk_status scratch_for_device(int dev, void** out) {
  if (dev < 0 || dev >= kMaxDevices) return KVK_ERR_INVALID_ARG;
  void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (!p) {
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return KVK_ERR_CUDA;
    }
    g_scratch_ptr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return KVK_OK;
}

}  // namespace

extern "C" kvk_status kvk_mla_decode_noalloc(
    kvk_layout* layout, int layer, const void* q_lat, const void* q_rope, int dtype,
    int64_t q_lat_stride_seq, int64_t q_lat_stride_head, int64_t q_rope_stride_seq,
    int64_t q_rope_stride_head, int batch, int n_heads, const int32_t* dev_seq_lens,
    const int32_t* dev_keep_idx, const int32_t* dev_keep_len, int keep_stride,
    float softmax_scale, float* out, float* lse, kvk_stream_t stream) {
  if (!layout || !layout->arena) return KVK_ERR_INVALID_ARG;
  // the scratch address is per device: look it up only with the layout's device current
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) {
    cudaGetLastError();
    return KVK_ERR_CUDA;
  }
  if (cur != layout->device) return KVK_ERR_INVALID_ARG;
  void* scratch = nullptr;
  kvk_status st = scratch_for_device(cur, &scratch);
  if (st != KVK_OK) return st;
  // kvk_mla_decode checks the workspace against the need of the kernel it takes and
  // returns KVK_ERR_WORKSPACE (launching nothing) when the scratch is too small for it
  return kvk_mla_decode(layout, layer, q_lat, q_rope, dtype, q_lat_stride_seq,
                        q_lat_stride_head, q_rope_stride_seq, q_rope_stride_head, batch,
                        n_heads, dev_seq_lens, dev_keep_idx, dev_keep_len, keep_stride,
                        softmax_scale, out, lse, scratch, KVK_NOALLOC_SCRATCH_BYTES, stream);
}
