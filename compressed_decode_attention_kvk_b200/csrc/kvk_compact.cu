// kvk_compact.cu -- keep-list compaction in front of the tensor-core decode.
//
// A decode with a keep list (token eviction composed with the compressed cache: "Main
// Results", Table 2 of the KV-Kaizen page, representation compression times a SnapKV-style
// keep set) reads only the kept rows.  The tensor-core kernel streams whole 64-row tiles
// with the tensor memory accelerator, so the kept rows of each sequence (and their fp16
// scales) are first copied, in keep order, into a dense scratch cache [batch][keep_stride]
// in the workspace.  Entries outside [0, seq_len) are skipped and flagged
// (KVK_FLAG_KEEP_INDEX), exactly as the CUDA-core kernel skips them; the dense length of a
// sequence is its count of valid entries.  The decode then reads the scratch cache as a
// cache without a keep list, with those lengths.
#include "kvk_internal.cuh"

namespace kvk {
namespace {

constexpr int kCompactThreads = 256;   // keep entries per CTA (one chunk)
constexpr int kCompactWarps = kCompactThreads / 32;
constexpr int kCopyUnroll = 8;        // 16-byte loads in flight per thread

// One CTA per (sequence, chunk of 256 keep entries).  The CTA counts the valid entries of
// the earlier chunks itself (a few KB of keep indices from L2), so one launch suffices.
__global__ void __launch_bounds__(kCompactThreads) compact_kernel(CompactArgs c) {
  __shared__ int s_tok[kCompactThreads];
  __shared__ int s_warp[kCompactWarps], s_before[kCompactWarps];
  const int i = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int p0 = blockIdx.y * kCompactThreads;
  const int len_raw = __ldg(c.seq_lens + i), k_raw = __ldg(c.keep_len + i);
  const int len = min(max(len_raw, 0), c.max_tokens);
  const int k = min(max(k_raw, 0), c.keep_stride);
  if (blockIdx.y == 0 && tid == 0 && (len != len_raw || k != k_raw))
    atomicOr(c.flags, KVK_FLAG_SEQ_LEN);
  if (p0 >= max(k, 1)) return;   // chunk 0 always runs (it writes the count of k = 0)
  const int32_t* keep = c.keep_idx + (int64_t)i * c.keep_stride;

  // valid entries before this chunk
  int before = 0;
  for (int p = tid; p < p0; p += kCompactThreads) {
    const int t = __ldg(keep + p);
    before += (t >= 0 && t < len) ? 1 : 0;
  }
  // this chunk's entry, and its rank among the chunk's valid entries
  const int p = p0 + tid;
  bool v = false;
  int t = -1;
  if (p < k) {
    t = __ldg(keep + p);
    v = (t >= 0 && t < len);
    if (!v) atomicOr(c.flags, KVK_FLAG_KEEP_INDEX);
  }
  const unsigned ball = __ballot_sync(0xffffffffu, v);
  const int rank_in_warp = __popc(ball & ((1u << lane) - 1u));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) before += __shfl_xor_sync(0xffffffffu, before, o);
  if (lane == 0) s_warp[warp] = __popc(ball);
  if (lane == 0) s_before[warp] = before;
  __syncthreads();
  int base = 0, total = 0, prior = 0;
#pragma unroll
  for (int w = 0; w < kCompactWarps; ++w) {
    prior += s_before[w];
    if (w < warp) base += s_warp[w];
    total += s_warp[w];
  }
  if (v) s_tok[base + rank_in_warp] = t;
  if (tid == 0 && p0 + kCompactThreads >= k) c.cnt[i] = prior + total;   // holds the last entry
  __syncthreads();

  // copy the chunk's valid rows as 16-byte words (row_bytes is a multiple of 16): thread tid
  // takes words tid, tid + 256, ... of the chunk's rows laid end to end, kCopyUnroll loads in
  // flight before their stores
  const int w16 = c.row_bytes >> 4, nw = total * w16;
  const uint4* __restrict__ src = reinterpret_cast<const uint4*>(c.codes);
  uint4* __restrict__ dst = reinterpret_cast<uint4*>(c.dst_codes);
  const int64_t src_seq = (int64_t)i * c.max_tokens, dst_seq = (int64_t)i * c.keep_stride + prior;
  for (int e0 = tid; e0 < nw; e0 += kCompactThreads * kCopyUnroll) {
    uint4 v[kCopyUnroll];
    int64_t to[kCopyUnroll];
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
      const int e = e0 + u * kCompactThreads;
      if (e < nw) {
        const int r = e / w16, col = e - r * w16;
        v[u] = __ldg(src + (src_seq + s_tok[r]) * w16 + col);
        to[u] = (dst_seq + r) * w16 + col;
      }
    }
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u)
      if (e0 + u * kCompactThreads < nw) dst[to[u]] = v[u];
  }
  // the rows' scales: one per token, or sg per token in a group-scaled cache
  for (int e = tid; e < total * c.sg; e += kCompactThreads) {
    const int r = e / c.sg, j = e - r * c.sg;
    c.dst_scales[(dst_seq + r) * c.sg + j] = c.scales[(src_seq + s_tok[r]) * c.sg + j];
  }
}

}  // namespace

size_t compact_workspace_bytes(int batch, int keep_stride, int row_bytes, int sg) {
  size_t off = align_up_sz(sizeof(int32_t) * (size_t)batch, 256);
  off = align_up_sz(off + (size_t)batch * (size_t)keep_stride * (size_t)row_bytes, 256);
  // fp16 scales (sg per token), plus slack: the decode reads each tile's scales as one window
  // from the 16-byte boundary at or below the tile's first scale, up to 64 tokens' scales and
  // 32 bytes past the last kept row
  off = align_up_sz(off + (size_t)batch * (size_t)keep_stride * 2 * sg + 64 * 2 * sg + 32, 256);
  return off;
}

void compact_carve(void* base, int batch, int keep_stride, int row_bytes, int sg, CompactArgs* c) {
  c->sg = sg;
  uint8_t* p = static_cast<uint8_t*>(base);
  c->cnt = reinterpret_cast<int32_t*>(p);
  size_t off = align_up_sz(sizeof(int32_t) * (size_t)batch, 256);
  c->dst_codes = p + off;
  off = align_up_sz(off + (size_t)batch * (size_t)keep_stride * (size_t)row_bytes, 256);
  c->dst_scales = reinterpret_cast<__half*>(p + off);
}

cudaError_t launch_compact(const CompactArgs& c, int batch, cudaStream_t st) {
  const int chunks = (c.keep_stride + kCompactThreads - 1) / kCompactThreads;
  if (batch < 1 || chunks > 65535) return cudaErrorInvalidValue;
  dim3 grid(batch, chunks > 0 ? chunks : 1);
  compact_kernel<<<grid, kCompactThreads, 0, st>>>(c);
  return cudaGetLastError();
}

}  // namespace kvk
