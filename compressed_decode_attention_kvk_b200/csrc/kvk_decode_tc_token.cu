// kvk_decode_tc_token.cu -- tensor-core (tcgen05) split decode over b-bit codes with one
// fp16 scale per token (b in {2, 4, 8, 16}) and over uncompressed bf16 rows: the decode, and
// the fused append, of such layers.
//
// Computes the same partials as the CUDA-core kernel (kvk_decode_fma.cu) and the general
// tensor-core kernel (kvk_decode_tc.cu): for every piece of a sequence that the CTA owns, the
// running max m (log2 units), the weight sum l = sum 2^(z2 - m) and the un-normalised output
// o = sum 2^(z2 - m) c_hat[:d], where
// z2 = log2(e) * sigma * s_t * (q_lat . code_t[:d] + q_rope . code_t[d:])  (absorbed MLA
// attention over the dequantised cache; KV-Kaizen "Background": each decode step reads the
// whole cache).
//
// Scores are exact: codes of at most 8 bits are exact in f16 (score MMA M = 64); a 16-bit code
// c is split into hi = f16(c) and lo = c - hi, both exact, stacked per 16-token block into one
// M = 128 score MMA whose low-part rows land 16 TMEM lanes below the high-part rows (the
// softmax adds the two).  The conversion of every 128-feature group is spread over all eight
// convert warps (16 features each), and the softmax reads S with the 16x256b shape, two tokens
// per thread; measured on B200 at 32 x 8192 tokens, 40 heads, d = 512, this kernel is faster
// than the general one (kvk_decode_tc.cu) for every width it covers.  The general kernel keeps
// what this one lacks: group scales.  bf16 rows are exact in f16 (in its normal range) and are
// converted in place; rows past a piece's end are zeroed (bf16 garbage can be NaN).
//
// One persistent CTA per SM walks its slice of the flattened token space (the split charges
// each piece a fixed cost, so a CTA that starts a sequence takes fewer tokens) in tiles of
// 64 tokens.  Warp roles (512 threads, four warpgroups with their own register budgets):
//   warps 0-3  softmax: read S from TMEM, per-token scale, lazy online softmax, write P
//              (f16) to shared memory, rescale O in TMEM when a max grows, write partials
//   warps 4-11 convert: b-bit codes -> f16 operand tiles (UMMA 128-byte-swizzled, K-major;
//              16-bit codes as stacked high and low parts) and their transpose into TMEM;
//              staged query (power-of-two scaled).
//              Two warps per SM sub-partition, 16 features of every 128-feature group each.
//   warp 12    TMA producer: 128-feature groups of 64 rows into a ring (16-bit codes and bf16
//              rows straight into the group slots, narrower codes into a raw ring), and each
//              tile's token scales (none for bf16 rows); the stream is read once, so it
//              carries an evict-first L2 policy
//   warp 13    score-MMA issuer (one thread) and TMEM owner
//   warp 14    output-MMA issuer (one thread)
//   warp 15    the fused append's new tokens; then warms L2 with the queries of the CTA's
//              later pieces
// Launched with 128 registers per thread; the softmax warpgroup raises its budget to
// kRegsSoftmax, the conversion warpgroups lower theirs to kRegsConvert and the last
// warpgroup to kRegsIssue (4 x 32 x (192 + 2 x 120 + 80) = 65536).
// Per tile:  S^T[64 tok x N1 heads]  = C[64 x n] . Q^T   (M=64, or M=128 stacked x N2; A in
//                                                          smem, TMEM f32)
//            O^T[128 feat x N2 heads] += C^T[128 x 64] . P    (M=128 per 128 latent features,
//                                                               A = C^T in TMEM)
// Heads sit on N, so 40 heads cost N = 40 / 48, never M = 128.  The convert warps unpack each
// 128-feature group from a raw ring into an f16 slot (UMMA 128-byte swizzled, K-major: the
// score MMA's A), or convert 16-bit rows in place (codes split, bf16 rounded to f16), and put
// their 16 features of it, transposed with ldmatrix.trans, into TMEM (tcgen05.st); the output
// MMA reads C^T from TMEM (for 16-bit codes the high parts: f16(code), relative 2^-12 on the
// output, inside its tolerance).
// The transpose fragment orders the 16 tokens of each K step as 0,1,8,9,2,3,10,11,4,5,12,13,
// 6,7,14,15; the softmax warps write P's K rows in that same order.
// The per-token scale s_t (1 for bf16 rows) multiplies the S row and is folded into P as
// p * s_t / S_run, with S_run a running power of two >= every scale seen so far (when it grows,
// O is rescaled by the exact ratio).
// Every wait is bounded (the call's wait limit); on expiry the kernel records
// KVK_FLAG_TIMEOUT, drains its own TMA loads and MMAs, frees TMEM and exits.
#include <string.h>

#include "kvk_decode_common.cuh"
#include "kvk_quant_common.cuh"
#include "kvk_sm100.cuh"

namespace kvk {
namespace {

using namespace sm100;

constexpr int kThreads = 512;   // 16 warps = 4 warpgroups (warp 15 has no role)
constexpr int kConvWarp0 = 4;
constexpr int kConvWarps = 8;
constexpr int kConvThreads = 32 * kConvWarps;
constexpr int kTmaWarp = 12;
constexpr int kMmaWarp = 13;   // score MMAs; owns TMEM
constexpr int kMma2Warp = 14;  // output MMAs
// Register budgets.  The block is launched with kLaunchRegs per thread (the host checks that
// ptxas allocated exactly that before choosing this kernel); a warpgroup whose budget is
// above it raises it (setmaxnreg.inc), one below lowers it (.dec) -- never the other way,
// which would be an illegal instruction -- and the budgets sum to no more than the launch.
constexpr uint32_t kLaunchRegs = 65536 / kThreads;   // 128
constexpr uint32_t kRegsSoftmax = 192, kRegsConvert = 120, kRegsIssue = 80;
static_assert(128 * (kRegsSoftmax + 2 * kRegsConvert + kRegsIssue) <= 65536, "register split");
template <uint32_t N>
__device__ __forceinline__ void regs_set() {
  if constexpr (N > kLaunchRegs) regs_inc<N>();
  else if constexpr (N < kLaunchRegs) regs_dec<N>();
}
constexpr int kTile = kTcTileTokens;   // 64
constexpr int kAtom = 8192;            // 64 rows x 128 bytes (64 f16 features)
constexpr int kPair = 2 * kAtom;       // 128 features
// Group slot geometry.  Plain slots (b <= 8) hold each 64-feature atom's 64 f16 rows
// contiguously.  16-bit codes use stacked slots: per 16-token block, the 16 rows of exact high
// parts and then the 16 rows of low parts of the same tokens (4 KB blocks, low rows at +
// kLoOff), so that one M = 128 score MMA yields both partial scores of 64 tokens.
template <int BITS>
constexpr bool kStacked = (BITS == 16);
// 16-bit codes and bf16 rows are converted in place, in the group slot TMA filled
template <int BITS>
constexpr bool kInPlace = (BITS == 16 || BITS == KVK_BITS_BF16);
template <int BITS>
constexpr uint32_t kAtomB = kStacked<BITS> ? 2u * kAtom : (uint32_t)kAtom;
template <int BITS>
constexpr uint32_t kSlotB = 2u * kAtomB<BITS>;
constexpr uint32_t kLoOff = 2048;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSCol = 0;          // scores S^T, one buffer (N1 <= 64 columns)
constexpr uint32_t kCtCol0 = 64;       // C^T double buffer: 64 + 128 b, latent group p at + 32 p
constexpr uint32_t kOCol0 = 320;       // O^T group p at 320 + N2 p
// limit of the waits that drain a stopping kernel's own loads and MMAs (they always end)
constexpr uint64_t kDrainLimitNs = 2000000000ull;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kSmemLimit = 232448;
constexpr int kQC = 3;   // 16-byte chunks per lane per query row (rows of up to 768 features)
constexpr int kQD = 1;   // query rows in flight per convert warp while staging
// Token-scale ring: per tile a 144-byte window (the tile's 64 fp16 scales from the 16-byte
// boundary at or below the first), loaded by the TMA warp with a plain bulk copy.
constexpr int kScSlots = 4;
constexpr uint32_t kScBytes = 144;
// barriers besides the rings: s full/empty, P full/empty (2), C^T full/empty (2), q full/empty,
// o empty, two MMA drains, q seen, appended, scale full/empty (kScSlots each)
constexpr int kFixedBars = 2 + 4 + 4 + 7 + 2 * kScSlots;

struct TcParams {
  DecodeArgs a;
  int N1, N2;           // N of the score MMA (heads rounded to 8) and of the output MMA (16)
  int NP, NPd;          // 128-feature groups per row, and those holding latent features
  int NQA, NK16;        // 64-feature query atoms, 16-feature K steps
  int PR, RR, raw_slot; // ring slots (f16 groups, packed groups) and packed-group bytes
  uint32_t lbo_p;       // bytes between the 8-token core-matrix rows of P (16 N2 + 32)
  uint32_t p_bytes;     // one P buffer: 8 lbo_p
  uint32_t off_p, off_pairs, off_raw, off_bar, off_misc;
  uint32_t idesc1, idesc2;
  int qdtype;           // KVK_BF16 or KVK_F16
};

struct Misc {
  alignas(16) uint8_t sc[kScSlots][kScBytes];   // token-scale windows
  uint32_t tmem_base;
  int abort;
  float qs_inv[2][64];   // per piece parity and head: 2^-e of the staged query row
  int vote[2][4];
  float m_ref[64];
  float alpha[64];
  float red[4][64];
  float sred[4];
  int32_t scan_tmp[32];
};

// Position in a ring of n slots: slot index and the phase parity of its mbarriers.
struct Ring {
  uint32_t slot = 0, phase = 0;
  __device__ __forceinline__ void next(int n) {
    if (++slot == (uint32_t)n) {
      slot = 0;
      phase ^= 1u;
    }
  }
};

struct Cursor {
  int seq, pos, p0, p1, cnt, tile, piece;
  bool valid, first, last;
};

__device__ __forceinline__ bool find_piece(Cursor& c, const int32_t* off, int batch, int64_t lo,
                                           int64_t hi) {
  while (c.seq < batch && off[c.seq] < hi) {
    const int64_t s0 = max(lo, (int64_t)off[c.seq]), s1 = min(hi, (int64_t)off[c.seq + 1]);
    if (s0 < s1) {
      c.p0 = (int)(s0 - off[c.seq]);
      c.p1 = (int)(s1 - off[c.seq]);
      c.pos = c.p0;
      return true;
    }
    ++c.seq;
  }
  return false;
}
__device__ __forceinline__ void set_tile(Cursor& c) {
  c.cnt = min(kTile, c.p1 - c.pos);
  c.first = (c.pos == c.p0);
  c.last = (c.pos + kTile >= c.p1);
}
__device__ __forceinline__ void cursor_start(Cursor& c, int seq0, const int32_t* off, int batch,
                                             int64_t lo, int64_t hi) {
  c.seq = seq0;
  c.tile = 0;
  c.piece = 0;
  c.valid = find_piece(c, off, batch, lo, hi);
  if (c.valid) set_tile(c);
}
__device__ __forceinline__ void cursor_next(Cursor& c, const int32_t* off, int batch, int64_t lo,
                                            int64_t hi) {
  ++c.tile;
  c.pos += kTile;
  if (c.pos >= c.p1) {
    ++c.seq;
    ++c.piece;
    c.valid = find_piece(c, off, batch, lo, hi);
  }
  if (c.valid) set_tile(c);
}

__device__ __forceinline__ bool wait_noabort(uint64_t* b, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try(b, parity)) {
    if (globaltimer() - t0 > kDrainLimitNs) return false;
  }
  return true;
}

// mbar_wait by every lane of a warp, with one warp-uniform answer (the lanes of a warp then
// never diverge around the .sync.aligned instructions that follow a wait).
__device__ __forceinline__ bool wait_warp(uint64_t* b, uint32_t parity, uint32_t abort_saddr,
                                          uint64_t limit_ns) {
  return __all_sync(0xffffffffu, mbar_wait(b, parity, abort_saddr, limit_ns));
}

__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 bits_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// Two 16-bit offset-binary codes, each split exactly into two f16 parts, hi = f16(code)
// (rounded to nearest) and lo = code - hi: with hb, lb the code's bytes (exact in f16),
// t = (hb - 128) * 256 - hi is an integer of magnitude <= 263 (so the fused multiply-add is
// exact), and lo = t + lb an integer of magnitude <= 8 (f16 spacing is at most 16 below 2^15):
// q . code = q . hi + q . lo exactly.
__device__ __forceinline__ void cvt_code16_split(uint32_t w, uint32_t& hi, uint32_t& lo) {
  const __half2 hs = __hsub2(bits_h2(__byte_perm(w, 0x64u, 0x4341u)), __float2half2_rn(1152.f));
  const __half2 ls = __hsub2(bits_h2(__byte_perm(w, 0x64u, 0x4240u)), __float2half2_rn(1024.f));
  const __half2 h = __hfma2(hs, __float2half2_rn(256.f), ls);
  const __half2 t = __hfma2(hs, __float2half2_rn(256.f), __hneg2(h));
  hi = h2_bits(h);
  lo = h2_bits(__hadd2(t, ls));
}
// two bf16 values -> f16x2, round to nearest: exact for values in the f16 normal range
// (bf16 keeps 8 significant bits, f16 11); beyond +-65504 a value becomes +-inf
__device__ __forceinline__ uint32_t cvt_bf16x2(uint32_t w) {
  return h2_bits(__floats2half2_rn(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u)));
}
// bytes of w selected by `sel` (each a field u < 1024) -> f16x2 of (u - bias), exact
__device__ __forceinline__ uint32_t cvt_small(uint32_t w, uint32_t sel, __half2 bias) {
  return h2_bits(__hsub2(bits_h2(__byte_perm(w, 0x64u, sel)), bias));
}
__device__ __forceinline__ uint32_t spread2(uint32_t x) {  // 4 x 2-bit fields -> 4 bytes
  x = (x | (x << 12)) & 0x000F000Fu;
  x = (x | (x << 6)) & 0x03030303u;
  return x;
}

// Row handled by `lane` in pass k of a convert warp (two lanes per row, one 16-byte chunk
// each): rows 16k + 8(u/8) + (0,2,4,6,1,3,5,7)[u%8], u = lane/2.  Every 8-lane phase then
// touches rows that differ in bits 1 and 2 (distinct chunks of the 128-byte swizzle) and
// every 16-lane phase eight rows with distinct (row % 8), so the convert loops are free of
// shared-memory bank conflicts for 16- and 8-byte accesses.
__device__ __forceinline__ int conv_row(int lane, int k) {
  const int u = lane >> 1, x = u & 7;
  return 16 * k + 8 * (u >> 3) + (((x & 3) << 1) | (x >> 2));
}

// Packed b-bit group (64 rows x 128 features, TMA-swizzled) -> f16 pair slot, for the 16
// features fb .. fb+15 (eight-feature groups g = fb/8 + {0, 1} of every row).  All four
// packed words of a lane are loaded before the first store.
template <int BITS>
__device__ __forceinline__ void convert_group(const uint8_t* rawslot, uint8_t* pair, int lane,
                                              int fb) {
  const int g = (fb >> 3) + (lane & 1);
  uint32_t w[4][BITS == 8 ? 2 : 1];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = conv_row(lane, k);
    if constexpr (BITS == 8) {
      const uint2 u = *reinterpret_cast<const uint2*>(rawslot + r * 128 +
                                                      (((g >> 1) ^ (r & 7)) << 4) + ((g & 1) << 3));
      w[k][0] = u.x;
      w[k][BITS == 8 ? 1 : 0] = u.y;
    } else if constexpr (BITS == 4) {
      w[k][0] = *reinterpret_cast<const uint32_t*>(
          rawslot + r * 64 + (((g >> 2) ^ ((r >> 1) & 3)) << 4) + ((g & 3) << 2));
    } else {   // BITS == 2
      w[k][0] = *reinterpret_cast<const uint16_t*>(
          rawslot + r * 32 + (((g >> 3) ^ ((r >> 2) & 1)) << 4) + ((g & 7) << 1));
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = conv_row(lane, k);
    uint4 o;
    if constexpr (BITS == 8) {
      const __half2 bias = __float2half2_rn(1152.f);
      o.x = cvt_small(w[k][0], 0x4140u, bias);
      o.y = cvt_small(w[k][0], 0x4342u, bias);
      o.z = cvt_small(w[k][BITS == 8 ? 1 : 0], 0x4140u, bias);
      o.w = cvt_small(w[k][BITS == 8 ? 1 : 0], 0x4342u, bias);
    } else if constexpr (BITS == 4) {
      const __half2 bias = __float2half2_rn(1032.f);
      const uint32_t x = w[k][0] & 0x0F0F0F0Fu, y = (w[k][0] >> 4) & 0x0F0F0F0Fu;
      const uint32_t u01 = __byte_perm(x, y, 0x5140u), u45 = __byte_perm(x, y, 0x7362u);
      o.x = cvt_small(u01, 0x4140u, bias);
      o.y = cvt_small(u01, 0x4342u, bias);
      o.z = cvt_small(u45, 0x4140u, bias);
      o.w = cvt_small(u45, 0x4342u, bias);
    } else {   // BITS == 2
      const __half2 bias = __float2half2_rn(1026.f);
      const uint32_t u0 = spread2(w[k][0] & 0xFFu), u1 = spread2(w[k][0] >> 8);
      o.x = cvt_small(u0, 0x4140u, bias);
      o.y = cvt_small(u0, 0x4342u, bias);
      o.z = cvt_small(u1, 0x4140u, bias);
      o.w = cvt_small(u1, 0x4342u, bias);
    }
    *reinterpret_cast<uint4*>(pair + (g >> 3) * kAtom + r * 128 + (((g & 7) ^ (r & 7)) << 4)) = o;
  }
}

__device__ __forceinline__ void load8_bits(const uint4 u, int dtype, float (&v)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if (dtype == KVK_BF16) {
      v[2 * k] = __uint_as_float(w[k] << 16);
      v[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    } else {
      const float2 f = __half22float2(bits_h2(w[k]));
      v[2 * k] = f.x;
      v[2 * k + 1] = f.y;
    }
  }
}

template <int BITS, int NH>
__global__ void __launch_bounds__(kThreads, 1)
decode_tc_kernel(const __grid_constant__ TcParams P, const __grid_constant__ CUtensorMap tmap) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, derived from the shared array by an offset so that every
  // pointer below stays in the shared state space (plain LDS / STS, not generic accesses)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const DecodeArgs& a = P.a;
  uint8_t* q_s = smem;
  uint8_t* p_s = smem + P.off_p;
  uint8_t* pairs = smem + P.off_pairs;
  uint8_t* raw = smem + P.off_raw;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + P.off_bar);
  uint64_t* b_pfull = bars;               // [PR] group converted, visible to the tensor core
  uint64_t* b_pempty = b_pfull + P.PR;    // [PR] group released by the MMAs
  uint64_t* b_tfull = b_pempty + P.PR;    // [PR] 16-bit: TMA landed in the group slot
  uint64_t* b_rfull = b_tfull + P.PR;     // [RR] packed group landed
  uint64_t* b_rempty = b_rfull + P.RR;    // [RR] packed group consumed
  uint64_t* b_sfull = b_rempty + P.RR;    // scores ready in TMEM
  uint64_t* b_sempty = b_sfull + 1;       // scores read
  uint64_t* b_Pfull = b_sempty + 1;       // [2] P written
  uint64_t* b_Pempty = b_Pfull + 2;       // [2] output MMA of that P done
  uint64_t* b_ctfull = b_Pempty + 2;      // [2] C^T of a tile in TMEM
  uint64_t* b_ctempty = b_ctfull + 2;     // [2] output MMA of that C^T done
  uint64_t* b_qfull = b_ctempty + 2;      // query staged
  uint64_t* b_qempty = b_qfull + 1;       // query no longer read
  uint64_t* b_oempty = b_qempty + 1;      // O read out by the epilogue
  uint64_t* b_final = b_oempty + 1;       // score-MMA drain
  uint64_t* b_final2 = b_final + 1;       // output-MMA drain
  uint64_t* b_qseen = b_final2 + 1;       // softmax has taken the piece's query scale
  uint64_t* b_app = b_qseen + 1;          // fused append: new tokens written
  uint64_t* b_scfull = b_app + 1;         // [kScSlots] scale window landed
  uint64_t* b_scempty = b_scfull + kScSlots;   // [kScSlots] scale window read (last)
  Misc* m = reinterpret_cast<Misc*>(smem + P.off_misc);
  int32_t* off = reinterpret_cast<int32_t*>(m + 1);
  const uint32_t abort = smem_u32(&m->abort);   // shared abort word (abort_read / abort_set)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // Launched as a programmatic dependent: let the merge launch now (its blocks take SMs as
  // this kernel's blocks exit, and it waits for this grid to complete).  (The grid is at most
  // one block per SM, so every block of this grid is resident.)  The set-up below touches only
  // this block's shared memory, TMEM and the kernel parameters, so it may overlap the kernel
  // before this one; the wait before the first global access (block_seq_offsets) holds every
  // read of an input or of the workspace until that kernel has completed.
  griddep_trigger();

  if (tid == 0) {
    for (int i = 0; i < P.PR; ++i) {
      mbar_init(&b_pfull[i], kConvWarps);
      // score MMAs (commit), plus the convert warps where they read the slot back (b <= 8)
      mbar_init(&b_pempty[i], kInPlace<BITS> ? 1 : 1 + kConvWarps);
      mbar_init(&b_tfull[i], 1);
    }
    for (int i = 0; i < P.RR; ++i) {
      mbar_init(&b_rfull[i], 1);
      mbar_init(&b_rempty[i], kConvWarps);
    }
    mbar_init(b_sfull, 1);
    mbar_init(b_sempty, 4);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&b_Pfull[i], 4);
      mbar_init(&b_Pempty[i], 1);
      mbar_init(&b_ctfull[i], kConvWarps);
      mbar_init(&b_ctempty[i], 1);
    }
    mbar_init(b_qfull, kConvWarps);
    mbar_init(b_qempty, 1);
    mbar_init(b_oempty, 4);
    mbar_init(b_final, 1);
    mbar_init(b_final2, 1);
    mbar_init(b_qseen, 4);
    mbar_init(b_app, 1);
    for (int i = 0; i < kScSlots; ++i) {
      mbar_init(&b_scfull[i], 1);
      mbar_init(&b_scempty[i], 4);
    }
    m->abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&m->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kTmaWarp && lane == 0) tma_prefetch_desc(&tmap);
  griddep_wait();
  block_seq_offsets(a, off, m->scan_tmp);   // contains __syncthreads
  if (blockIdx.x == 0)
    for (int i = tid; i <= a.batch; i += kThreads) a.seq_off[i] = off[i];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = m->tmem_base;

  const int64_t C = off[a.batch] + (int64_t)a.split_x * a.batch;
  const int64_t lo = split_token(off, a.batch, a.split_x, split_cost(blockIdx.x, C, a.G));
  const int64_t hi = split_token(off, a.batch, a.split_x, split_cost(blockIdx.x + 1, C, a.G));
  int seq0 = 0;
  {
    int L = 0, H = a.batch;
    while (L < H) {
      const int mid = (L + H + 1) >> 1;
      if (off[mid] <= lo) L = mid; else H = mid - 1;
    }
    seq0 = L;
  }
  const bool has_work = lo < hi;

  // Roles by warpgroup; each warpgroup first sets its register budget (one call site per
  // warpgroup, executed by all four of its warps).
  if (has_work && warp >= kTmaWarp) {
    regs_set<kRegsIssue>();
    if (warp == kTmaWarp) {
      // ------------------------------------------------------------------ TMA producer
      if (lane == 0) {
        Cursor c;
        cursor_start(c, seq0, off, a.batch, lo, hi);
        uint32_t cnt = 0;
        Ring rg;
        const int slots = kInPlace<BITS> ? P.PR : P.RR;
        // The first cache loads go out at once, while the convert warps stage the first query
        // (measured faster than holding them until the query is staged).  A fused append
        // writes this CTA's new tokens first (the spare warp).
        if (a.app_c) mbar_wait(b_app, 0u, abort, a.limit_ns);
        Ring sr;   // scale ring
        uint32_t nsc = 0;
        const uint64_t pol = policy_evict_first();   // the cache and its scales are read once
        while (c.valid && !abort_read(abort)) {
          const int row0 = c.seq * a.max_tokens + c.pos;
          bool ok = true;
          if constexpr (BITS != KVK_BITS_BF16) {   // this tile's scale window (the arena has
                                                   // tail slack for the last one)
            const uintptr_t sp = reinterpret_cast<uintptr_t>(a.scales + row0);
            if (!(ok = mbar_wait(&b_scempty[sr.slot], sr.phase ^ 1u, abort, a.limit_ns))) break;
            mbar_arrive_expect_tx(&b_scfull[sr.slot], kScBytes);
            bulk_load_hint(m->sc[sr.slot], reinterpret_cast<const void*>(sp & ~uintptr_t(15)),
                           kScBytes, &b_scfull[sr.slot], pol);
            sr.next(kScSlots);
            ++nsc;
          }
          for (int p = 0; p < P.NP && ok; ++p) {
            const uint32_t s = rg.slot, ph = rg.phase;
            if constexpr (kInPlace<BITS>) {
              // 16-bit rows land in the group slot itself: each atom's 64 rows contiguously at
              // the start of the atom's place (the convert warps move them into the stacked
              // layout); the slot is re-armed once the score MMAs have read it
              if (!(ok = mbar_wait(&b_pempty[s], ph ^ 1u, abort, a.limit_ns))) break;
              const int nat = ((2 * p + 1) * 64 < a.n) ? 2 : 1;
              mbar_arrive_expect_tx(&b_tfull[s], nat * kAtom);
              for (int t = 0; t < nat; ++t)
                tma_load_2d_hint(pairs + s * kSlotB<BITS> + t * kAtomB<BITS>, &tmap,
                                 (2 * p + t) * 128, row0, &b_tfull[s], pol);
            } else {
              if (!(ok = mbar_wait(&b_rempty[s], ph ^ 1u, abort, a.limit_ns))) break;
              mbar_arrive_expect_tx(&b_rfull[s], P.raw_slot);
              tma_load_2d_hint(raw + s * P.raw_slot, &tmap, p * 16 * BITS, row0, &b_rfull[s],
                               pol);
            }
            ++cnt;
            rg.next(slots);
          }
          if (!ok) break;
          cursor_next(c, off, a.batch, lo, hi);
        }
        // Let every load this thread issued land before the block exits.  A slot is re-armed
        // only after its consumers saw the previous load complete, so only the last load of
        // each slot can still be in flight (after an abort); in a normal run all have landed.
        for (uint32_t k = nsc > (uint32_t)kScSlots ? nsc - kScSlots : 0u; k < nsc; ++k)
          wait_noabort(&b_scfull[k % kScSlots], (k / kScSlots) & 1u);
        const uint32_t first = cnt > (uint32_t)slots ? cnt - slots : 0u;
        for (uint32_t k = first; k < cnt; ++k) {
          const uint32_t s = k % slots, ph = (k / slots) & 1u;
          wait_noabort(kInPlace<BITS> ? &b_tfull[s] : &b_rfull[s], ph);
        }
      }
    } else if (warp == kMmaWarp) {
      // ------------------------------------------------------------------ score MMAs
      // The whole warp runs the schedule (warp-uniform waits); one elected lane issues the
      // MMAs in groups of four, and commits them.
      Cursor g;
      cursor_start(g, seq0, off, a.batch, lo, hi);
      Ring rg;
      // descriptors of slot 0 / atom 0; every other operand differs only in its start address
      // (bits 0-13, address >> 4), so each operand adds its byte offset >> 4
      const uint64_t a0 = sdesc(smem_u32(pairs), 16u, 1024u, kLayoutSw128);
      const uint64_t b0 = sdesc(smem_u32(q_s), 16u, 1024u, kLayoutSw128);
      const uint32_t q_atom = (uint32_t)P.N1 * 128u;
      bool ok = true;
      while (g.valid && ok) {
        ok = mbar_wait(b_sempty, ((uint32_t)g.tile & 1u) ^ 1u, abort, a.limit_ns);
        if (ok && g.first) ok = mbar_wait(b_qfull, (uint32_t)g.piece & 1u, abort, a.limit_ns);
        ok = __all_sync(0xffffffffu, ok);
        for (int p = 0; p < P.NP && ok; ++p) {
          const uint32_t s = rg.slot;
          ok = __all_sync(0xffffffffu, mbar_wait(&b_pfull[s], rg.phase, abort, a.limit_ns));
          if (!ok) break;
          tc_fence_after();
          for (int t = 0; t < 2; ++t) {
            const int atom = 2 * p + t;
            if (atom * 64 >= a.n) break;
            const uint64_t ad = a0 + ((s * kSlotB<BITS> + t * kAtomB<BITS>) >> 4);
            const uint64_t bd = b0 + ((atom * q_atom) >> 4);
            const int k0 = atom * 4;
            if (k0 + 4 <= P.NK16) {
              mma4_elect(tmem + kSCol, ad, 2u, bd, 2u, P.idesc1, k0 > 0 ? 1u : 0u);
            } else {
              for (int ks = 0; k0 + ks < P.NK16; ++ks)
                mma1_elect(tmem + kSCol, ad + 2u * ks, bd + 2u * ks, P.idesc1, (k0 + ks) > 0);
            }
          }
          commit_elect(&b_pempty[s]);   // this group's share of the slot release
          rg.next(P.PR);
        }
        if (!ok) break;
        commit_elect(b_sfull);
        if (g.last) commit_elect(b_qempty);
        cursor_next(g, off, a.batch, lo, hi);
      }
      commit_elect(b_final);          // every MMA issued above has completed after this
      if (lane == 0) wait_noabort(b_final, 0);
      __syncwarp();
    } else if (warp == kMma2Warp) {
      // ------------------------------------------------------------------ output MMAs
      Cursor g;
      cursor_start(g, seq0, off, a.batch, lo, hi);
      const uint32_t lbo_p = P.lbo_p;
      const uint64_t b0 = sdesc(smem_u32(p_s), lbo_p, 128u, kLayoutNone);
      bool ok = true;
      while (g.valid && ok) {
        const int sb = g.tile & 1;
        ok = mbar_wait(&b_Pfull[sb], (uint32_t)(g.tile >> 1) & 1u, abort, a.limit_ns);
        if (ok) ok = mbar_wait(&b_ctfull[sb], (uint32_t)(g.tile >> 1) & 1u, abort, a.limit_ns);
        if (ok && g.first && g.piece > 0)
          ok = mbar_wait(b_oempty, (uint32_t)(g.piece - 1) & 1u, abort, a.limit_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const uint64_t bd = b0 + ((sb * P.p_bytes) >> 4);
        for (int p = 0; p < P.NPd; ++p) {
          // K = 64 tokens in four steps of 16: A advances 8 TMEM columns, B two core-matrix
          // rows of P
          mma4_ts_elect(tmem + kOCol0 + (uint32_t)P.N2 * p, tmem + kCtCol0 + 128u * sb + 32u * p,
                        8u, bd, (2u * lbo_p) >> 4, P.idesc2, g.first ? 0u : 1u);
        }
        commit_elect(&b_ctempty[sb]);
        commit_elect(&b_Pempty[sb]);
        cursor_next(g, off, a.batch, lo, hi);
      }
      commit_elect(b_final2);
      if (lane == 0) wait_noabort(b_final2, 0);
      __syncwarp();
    } else {
      // ------------------------------------------------------------------ spare warp
      // Fused append: the new token of every sequence whose last position this CTA owns is
      // quantised (the write kernel's arithmetic) and stored before the TMA warp issues any
      // cache load; the proxy fence makes those generic stores visible to its async-proxy reads.
      if (a.app_c) {
        uint8_t* codes_w = const_cast<uint8_t*>(a.codes);
        __half* scales_w = const_cast<__half*>(a.scales);
        bool ok = true;
        for (int i = seq0; i < a.batch && off[i] < hi; ++i) {
          const int len = off[i + 1] - off[i];
          const int64_t last = (int64_t)off[i + 1] - 1;
          if (len == 0 || last < lo || last >= hi) continue;
          const int64_t r = (int64_t)i * a.max_tokens + (len - 1);
          if (a.app_dtype == KVK_BF16)
            ok = write_token_two_pass<__nv_bfloat16>(
                     static_cast<const __nv_bfloat16*>(a.app_c) + (int64_t)i * a.app_c_ss,
                     static_cast<const __nv_bfloat16*>(a.app_kr) + (int64_t)i * a.app_kr_ss,
                     a.d, a.d_rope, a.b, a.group, codes_w + r * a.row_bytes, a.row_bytes,
                     scales_w + r * a.sg) &&
                 ok;
          else
            ok = write_token_two_pass<float>(
                     static_cast<const float*>(a.app_c) + (int64_t)i * a.app_c_ss,
                     static_cast<const float*>(a.app_kr) + (int64_t)i * a.app_kr_ss, a.d,
                     a.d_rope, a.b, a.group, codes_w + r * a.row_bytes, a.row_bytes,
                     scales_w + r * a.sg) &&
                 ok;
        }
        if (!ok && lane == 0) atomicOr(a.flags, KVK_FLAG_NONFINITE);
        fence_proxy_async_global();
        __syncwarp();
        if (lane == 0) mbar_arrive(b_app);
      }
      // Warm L2 with the queries of the sequences after the first that this CTA touches
      // (the convert warps stage the first one at once).
      Cursor c;
      cursor_start(c, seq0, off, a.batch, lo, hi);
      const int lat_lines = (2 * a.d + 127) / 128, rope_lines = (2 * a.d_rope + 127) / 128;
      const int lines = lat_lines + rope_lines;
      while (c.valid) {
        ++c.seq;
        if (!(c.valid = find_piece(c, off, a.batch, lo, hi))) break;
        const uint8_t* ql = static_cast<const uint8_t*>(a.q_lat) + 2 * ((int64_t)c.seq * a.ql_ss);
        const uint8_t* qr = static_cast<const uint8_t*>(a.q_rope) + 2 * ((int64_t)c.seq * a.qr_ss);
        for (int i = lane; i < a.H * lines; i += 32) {
          const int h = i / lines, k = i - h * lines;
          if (k < lat_lines) prefetch_l2(ql + 2 * ((int64_t)h * a.ql_sh) + 128 * k);
          else prefetch_l2(qr + 2 * ((int64_t)h * a.qr_sh) + 128 * (k - lat_lines));
        }
      }
    }
  } else if (has_work && warp >= kConvWarp0) {
    regs_set<kRegsConvert>();
    // ------------------------------------------------------------------ convert
    // The convert warps leave their loop only together (named_or agreement at the top of
    // every tile), so their named barriers never wait for a warp that has gone.  Warp cw
    // sits in TMEM lane quarter cq = cw % 4 and owns features fb .. fb+15 of every group,
    // fb = 32 cq + 16 ch (ch = cw / 4): TMEM lanes fb .. fb+15 of C^T.
    const int cw = warp - kConvWarp0;
    const int cq = cw & 3, ch = cw >> 2, fb = 32 * cq + 16 * ch;
    // 16-bit codes: this lane's ldmatrix row address inside a stacked group slot, per 16-token
    // block tg (token 16tg + 8((lane/8)%2) + lane%8, 16-byte chunk 4(cq%2) + 2ch + (lane/8)/2
    // of atom cq/2), where TMA put the row (roff: the atom's 64 rows contiguous from the
    // atom's start) and in the stacked layout (aoff; low part at + kLoOff).  Both keep the
    // 128-byte swizzle phase (token % 8), so a warp's cells stay in its own 16-byte columns:
    // it reads all of them (ldmatrix) before it writes any, and no other warp touches them.
    uint32_t roff[4] = {}, aoff[4] = {};
    if constexpr (kInPlace<BITS>) {
      const int mi = lane >> 3, r8 = lane & 7;
      const uint32_t col = (uint32_t)(((4 * (cq & 1) + 2 * ch + (mi >> 1)) ^ r8) << 4);
#pragma unroll
      for (int tg = 0; tg < 4; ++tg) {
        const uint32_t tok = (uint32_t)(16 * tg + 8 * (mi & 1) + r8);
        roff[tg] = (uint32_t)(cq >> 1) * kAtomB<BITS> + tok * 128u + col;
        // bf16 rows stay where TMA put them (a plain slot's layout)
        aoff[tg] = kStacked<BITS> ? (uint32_t)(cq >> 1) * kAtomB<BITS> + (tok >> 4) * 4096u +
                                        (tok & 15u) * 128u + col
                                  : roff[tg];
      }
    }
    Ring pr, rr;   // f16 group ring, packed group ring
    int last_piece = -1;
    bool fail = false;
    const int cpr = P.NQA * 8;   // 16-byte chunks per staged query row
    Cursor c;
    cursor_start(c, seq0, off, a.batch, lo, hi);
    while (c.valid) {
      if (named_or(2, kConvThreads, fail || abort_read(abort))) break;
      if (c.piece != last_piece) {
        // Stage this sequence's query as f16 rows [N1][n], scaled by 2^e so that max |q|
        // lands in [2^14, 2^15) (exact for bf16 inputs in range); rows >= H and features
        // >= n are zero.  Wait until the previous piece's scores no longer read it and the
        // softmax warps have taken the previous piece's scale (bounds q_full to one phase
        // ahead of its slowest waiter).
        fail = fail || !wait_warp(b_qempty, ((uint32_t)c.piece & 1u) ^ 1u, abort, a.limit_ns);
        if (c.piece > 0)
          fail = fail || !wait_warp(b_qseen, ((uint32_t)c.piece - 1u) & 1u, abort, a.limit_ns);
        const uint8_t* qlat = static_cast<const uint8_t*>(a.q_lat) + 2 * ((int64_t)c.seq * a.ql_ss);
        const uint8_t* qrope =
            static_cast<const uint8_t*>(a.q_rope) + 2 * ((int64_t)c.seq * a.qr_ss);
        // One pass: warp cw stages heads cw, cw + 8, ...; lane l holds chunks l, l + 32, ... of
        // a row, the warp reduces the row's max |q|, and the row is written scaled by 2^e_h
        // (max |q_h| in [2^14, 2^15), exact for bf16 inputs in range).  Rows >= H and chunks
        // >= n are zero.  The loop body is one row (a small code footprint: this code runs
        // once per piece and would otherwise be fetched cold); the loads of the next kQD rows
        // are in flight while a row is processed.
        auto load_row = [&](int h, uint4 (&v)[kQC]) {
#pragma unroll
          for (int j = 0; j < kQC; ++j) {
            const int f0 = 8 * (lane + 32 * j);
            v[j] = make_uint4(0u, 0u, 0u, 0u);
            if (h < a.H && f0 < a.n)
              v[j] = *reinterpret_cast<const uint4*>(
                  (f0 < a.d) ? qlat + 2 * ((int64_t)h * a.ql_sh + f0)
                             : qrope + 2 * ((int64_t)h * a.qr_sh + (f0 - a.d)));
          }
        };
        uint4 v[kQD + 1][kQC];
#pragma unroll
        for (int i = 0; i < kQD; ++i)
          if (cw + kConvWarps * i < P.N1) load_row(cw + kConvWarps * i, v[i]);
#pragma unroll 1
        for (int h = cw; h < P.N1; h += kConvWarps) {
          if (h + kConvWarps * kQD < P.N1) load_row(h + kConvWarps * kQD, v[kQD]);
          float f[kQC][8];
          float mx = 0.f;
#pragma unroll
          for (int j = 0; j < kQC; ++j) {
            load8_bits(v[0][j], P.qdtype, f[j]);
#pragma unroll
            for (int e = 0; e < 8; ++e) mx = fmaxf(mx, fabsf(f[j][e]));
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          // e = 14 - floor(log2 max |q|) from the exponent field (a subnormal max counts as
          // 2^-126), at most 126 so that 2^e and 2^-e are normal floats
          int e = 0;
          if (mx > 0.f && isfinite(mx))
            e = min(14 - (max((__float_as_int(mx) >> 23) & 0xff, 1) - 127), 126);
          const float qscale = __int_as_float((127 + e) << 23);
          if (lane == 0) m->qs_inv[c.piece & 1][h] = __int_as_float((127 - e) << 23);
#pragma unroll
          for (int j = 0; j < kQC; ++j) {
            const int fc = lane + 32 * j;
            if (fc >= cpr) break;
            uint4 o;
            o.x = h2_bits(__floats2half2_rn(f[j][0] * qscale, f[j][1] * qscale));
            o.y = h2_bits(__floats2half2_rn(f[j][2] * qscale, f[j][3] * qscale));
            o.z = h2_bits(__floats2half2_rn(f[j][4] * qscale, f[j][5] * qscale));
            o.w = h2_bits(__floats2half2_rn(f[j][6] * qscale, f[j][7] * qscale));
            const int at = fc >> 3, jj = fc & 7;
            *reinterpret_cast<uint4*>(q_s + at * (P.N1 * 128) + h * 128 + ((jj ^ (h & 7)) << 4)) = o;
          }
#pragma unroll
          for (int i = 0; i < kQD; ++i)
#pragma unroll
            for (int j = 0; j < kQC; ++j) v[i][j] = v[i + 1][j];
        }
        fence_proxy_async_smem();
        named_sync(2, kConvThreads);   // every warp's rows written before q_full
        if (lane == 0) mbar_arrive(b_qfull);
        last_piece = c.piece;
      }
      const int ctb = c.tile & 1;   // C^T buffer of this tile
      for (int p = 0; p < P.NP; ++p) {
        const uint32_t s = pr.slot, ph = pr.phase;
        uint8_t* pair = pairs + s * kSlotB<BITS>;
        const int nat = ((2 * p + 1) * 64 < a.n) ? 2 : 1;
        // this warp owns features fb .. fb+15 of the group: atom cq/2, chunks
        // 4(cq%2) + 2ch + {0, 1} of every token row; it converts them and later transposes them
        const bool owns = (cq >> 1) < nat;
        if constexpr (kInPlace<BITS>) {
          // In place, 16-bit codes -> exact f16 high and low parts (bf16 rows -> f16), in one pass through
          // registers: each 8x8 block (8 tokens x 8 features) is loaded transposed from where
          // TMA put it, split element by element, stored back transposed into the stacked
          // layout (high parts, and low parts kLoOff further), and the high parts, now
          // feature-major, go to C^T in TMEM (lanes fb .. fb+15 of latent group p).  The slot is
          // not read after p_full, so only the score MMAs release it.
          fail = fail || !wait_warp(&b_tfull[s], ph, abort, a.limit_ns);
          const bool go = !fail && owns;
          const uint32_t sbase = smem_u32(pair);
          uint32_t x[16], xl[16];
          if (go) {
#pragma unroll
            for (int tg = 0; tg < 4; ++tg) {
              uint32_t d4[4];
              ldsm_x4_trans(sbase + roff[tg], d4);
#pragma unroll
              for (int i = 0; i < 4; ++i) x[4 * tg + i] = d4[i];
            }
            if constexpr (kStacked<BITS>) {
#pragma unroll
              for (int i = 0; i < 16; ++i) cvt_code16_split(x[i], x[i], xl[i]);
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i) x[i] = cvt_bf16x2(x[i]);
              if (c.cnt < kTile) {
                // rows past the piece's end hold whatever the cache or scratch holds there
                // (as bf16 possibly a NaN, and P = 0 times NaN is NaN): zero them.  Register
                // 4tg + i holds tokens 16tg + 8(i%2) + 2(lane%4) + {0, 1}.
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                  const int t0 = 16 * (i >> 2) + 8 * (i & 1) + 2 * (lane & 3);
                  x[i] &= (t0 < c.cnt ? 0x0000FFFFu : 0u) | (t0 + 1 < c.cnt ? 0xFFFF0000u : 0u);
                }
              }
            }
#pragma unroll
            for (int tg = 0; tg < 4; ++tg) {
              const uint32_t h4[4] = {x[4 * tg], x[4 * tg + 1], x[4 * tg + 2], x[4 * tg + 3]};
              stsm_x4_trans(sbase + aoff[tg], h4);
              if constexpr (kStacked<BITS>) {
                const uint32_t l4[4] = {xl[4 * tg], xl[4 * tg + 1], xl[4 * tg + 2], xl[4 * tg + 3]};
                stsm_x4_trans(sbase + kLoOff + aoff[tg], l4);
              }
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&b_pfull[s]);
          if (p < P.NPd) {
            if (p == 0) {   // the output MMAs of tile - 2 have finished reading this buffer
              fail = fail || !wait_warp(&b_ctempty[ctb], ((uint32_t)(c.tile >> 1) & 1u) ^ 1u,
                                        abort, a.limit_ns);
              tc_fence_after();
            }
            if (go && !fail)
              tmem_st16x256b_x4(tmem + ((uint32_t)fb << 16) + kCtCol0 + 128u * ctb + 32u * p, x);
          }
        } else {
          const uint32_t rs = rr.slot, rph = rr.phase;
          fail = fail || !wait_warp(&b_rfull[rs], rph, abort, a.limit_ns);
          fail = fail || !wait_warp(&b_pempty[s], ph ^ 1u, abort, a.limit_ns);
          if (!fail) convert_group<BITS>(raw + rs * P.raw_slot, pair, lane, fb);
          __syncwarp();
          if (lane == 0) mbar_arrive(&b_rempty[rs]);
          rr.next(P.RR);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&b_pfull[s]);
          if (p < P.NPd) {
            // transpose this warp's 16 features x 64 tokens into C^T (TMEM lanes fb .. fb+15
            // of latent group p): four 16-token blocks
            if (p == 0) {   // the output MMAs of tile - 2 have finished reading this buffer
              fail = fail || !wait_warp(&b_ctempty[ctb], ((uint32_t)(c.tile >> 1) & 1u) ^ 1u, abort,
                                        a.limit_ns);
              tc_fence_after();
            }
            if (!fail && owns) {
              const uint32_t abase = smem_u32(pair + (cq >> 1) * kAtom);
              const int mi = lane >> 3, r8 = lane & 7;
              const int cc = 4 * (cq & 1) + 2 * ch + (mi >> 1);
              uint32_t rr[16];
#pragma unroll
              for (int tg = 0; tg < 4; ++tg) {
                const int tok = 16 * tg + 8 * (mi & 1) + r8;
                uint32_t d4[4];
                ldsm_x4_trans(abase + tok * 128 + ((cc ^ (tok & 7)) << 4), d4);
#pragma unroll
                for (int i = 0; i < 4; ++i) rr[4 * tg + i] = d4[i];
              }
              tmem_st16x256b_x4(tmem + ((uint32_t)fb << 16) + kCtCol0 + 128u * ctb + 32u * p, rr);
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&b_pempty[s]);   // this warp is done reading the slot
        }
        pr.next(P.PR);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&b_ctfull[ctb]);
      cursor_next(c, off, a.batch, lo, hi);
    }
  } else if (has_work) {
    regs_set<kRegsSoftmax>();
    // ------------------------------------------------------------------ softmax
    // TMEM holds S^T with tokens on lanes: the M = 64 layout puts rows 16q .. 16q+15 in
    // lanes 32q .. 32q+15.  Loaded with the 16x256b shape, thread t of warp q holds rows
    // ra = 16q + t/4 and rb = ra + 8, heads 8j + 2(t%4) + {0, 1} of every 8-head block j.
    // The four warps leave the loop only together (named_or agreement every tile).
    constexpr int NB = NH / 8;
    const int q = warp;
    const uint32_t lb = tmem + ((uint32_t)(32 * q) << 16);
    const int ra = 16 * q + (lane >> 2), rb = ra + 8;
    const int hc = 2 * (lane & 3);
    bool fail = false;

    // S_run: running power of two >= every token scale seen so far (P = p * s / S_run keeps
    // P <= 2^8 in f16).  It only grows; when a tile brings a larger scale the slow path
    // rescales O by S_old / S_new, exactly (powers of two), together with any max update.
    float srun = 0.f, inv_srun = 0.f;

    float l[2 * NB];    // partial weight sums of this thread's heads
    float mr[2 * NB];   // reference max of this thread's heads (log2 units)
    float qh[2 * NB];   // 2^-e_h of this thread's heads 8j + hc + {0, 1} in the current piece
    int pt = 0;
    Cursor c;
    cursor_start(c, seq0, off, a.batch, lo, hi);
    const float coef0 = a.sigma * kLog2e;
    // K slot of this thread's rows in P: the transposed C^T holds, in the 16 K slots of each
    // step, tokens 0,1,8,9,2,3,10,11,4,5,12,13,6,7,14,15 of the step's 16 tokens
    const int ka = 16 * q + 4 * (lane >> 3) + ((lane >> 2) & 1), kb = ka + 2;
    // Token scales of rows ra / rb come from the tile's scale window in shared memory
    // (bulk-copied by the TMA warp at least a tile ahead): no global loads in this role, so
    // the proxy fence after each P write has nothing outstanding to wait for.
    Ring sr;
    while (c.valid) {
      const int t = c.tile, sb = t & 1;
      float s_a = 0.f, s_b = 0.f;
      if constexpr (BITS == KVK_BITS_BF16) {   // uncompressed rows: unit token scale
        s_a = (ra < c.cnt) ? 1.f : 0.f;
        s_b = (rb < c.cnt) ? 1.f : 0.f;
      } else {
        fail = fail || !wait_warp(&b_scfull[sr.slot], sr.phase, abort, a.limit_ns);
        const __half* w = reinterpret_cast<const __half*>(m->sc[sr.slot]) +
                          ((reinterpret_cast<uintptr_t>(a.scales + (int64_t)c.seq * a.max_tokens +
                                                        c.pos) & 15u) >> 1);
        if (ra < c.cnt) s_a = __half2float(w[ra]);
        if (rb < c.cnt) s_b = __half2float(w[rb]);
        __syncwarp();
        if (lane == 0) mbar_arrive(&b_scempty[sr.slot]);
        sr.next(kScSlots);
      }
      if (c.first) {
        fail = fail || !wait_warp(b_qfull, (uint32_t)c.piece & 1u, abort, a.limit_ns);
#pragma unroll
        for (int j = 0; j < NB; ++j)
#pragma unroll
          for (int e = 0; e < 2; ++e) qh[2 * j + e] = m->qs_inv[c.piece & 1][8 * j + hc + e];
        __syncwarp();
        if (lane == 0) mbar_arrive(b_qseen);
#pragma unroll
        for (int i = 0; i < 2 * NB; ++i) {
          l[i] = 0.f;
          mr[i] = -INFINITY;
        }
        pt = 0;
      }
      const bool va = ra < c.cnt, vb = rb < c.cnt;
      const float ca = coef0 * s_a, cbf = coef0 * s_b;
      fail = fail || !wait_warp(b_sfull, (uint32_t)t & 1u, abort, a.limit_ns);
      tc_fence_after();
      // S^T rows of this thread (16x256b shape over 16 lanes from `at`); with stacked 16-bit
      // codes the low-part scores of the same tokens sit 16 lanes further and are added
      auto load_s = [&](uint32_t at, float (&x)[4 * NB]) {
        if constexpr (NB == 8) {
          tmem_ld16x256b_x8(at, *reinterpret_cast<float(*)[32]>(x));
        } else if constexpr (NB == 6) {   // columns 0-31 and 32-47
          tmem_ld16x256b_x4(at, *reinterpret_cast<float(*)[16]>(x));
          tmem_ld16x256b_x2(at + 32u, *reinterpret_cast<float(*)[8]>(x + 16));
        } else if constexpr (NB == 4) {
          tmem_ld16x256b_x4(at, *reinterpret_cast<float(*)[16]>(x));
        } else {
          tmem_ld16x256b_x2(at, *reinterpret_cast<float(*)[8]>(x));
        }
      };
      float x[4 * NB];
      load_s(lb + kSCol, x);
      if constexpr (kStacked<BITS>) {
        float xlo[4 * NB];
        load_s(lb + (16u << 16) + kSCol, xlo);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 4 * NB; ++i) x[i] += xlo[i];
      }
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_sempty);
      bool mine = (pt == 0) || s_a > srun || s_b > srun;
#pragma unroll
      for (int j = 0; j < NB; ++j) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const bool hv = (8 * j + hc + e) < a.H;
          x[4 * j + e] = (va && hv) ? x[4 * j + e] * qh[2 * j + e] * ca : -INFINITY;
          x[4 * j + 2 + e] = (vb && hv) ? x[4 * j + 2 + e] * qh[2 * j + e] * cbf : -INFINITY;
          mine = mine || (x[4 * j + e] > mr[2 * j + e] + 8.f) ||
                 (x[4 * j + 2 + e] > mr[2 * j + e] + 8.f);
        }
      }
      // lazy running max: recompute (and rescale) only when a score exceeds the reference
      // by more than 2^8, so P stays within f16 range without touching O every tile
      if (named_or(1, 128, mine || fail || abort_read(abort))) {
        if (named_or(1, 128, fail || abort_read(abort))) break;
#pragma unroll
        for (int j = 0; j < NB; ++j) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            float v = fmaxf(x[4 * j + e], x[4 * j + 2 + e]);
            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
            if (lane < 4) m->red[q][8 * j + 2 * lane + e] = v;
          }
        }
        {
          float sm = fmaxf(s_a, s_b);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) sm = fmaxf(sm, __shfl_xor_sync(0xffffffffu, sm, o));
          if (lane == 0) m->sred[q] = sm;
        }
        named_sync(1, 128);
        float ratio = 1.f;   // S_old / S_new, applied to O only (l sums p, not p * s)
        {
          const float sm = fmaxf(fmaxf(m->sred[0], m->sred[1]), fmaxf(m->sred[2], m->sred[3]));
          if (sm > srun && isfinite(sm)) {
            int ex;
            const float fr = frexpf(sm, &ex);   // sm = fr * 2^ex, fr in [0.5, 1)
            const float sn = (fr == 0.5f) ? sm : ldexpf(1.f, ex);
            ratio = srun / sn;
            srun = sn;
            inv_srun = 1.f / sn;
          }
        }
        if (tid < NH) {   // one thread per head: new reference and the factor for old sums
          const float tm = fmaxf(fmaxf(m->red[0][tid], m->red[1][tid]),
                                 fmaxf(m->red[2][tid], m->red[3][tid]));
          const float mo = (pt == 0) ? -INFINITY : m->m_ref[tid];
          const float mn = fmaxf(mo, tm);
          m->alpha[tid] = (mo == -INFINITY) ? 0.f : exp2f(mo - mn);
          m->m_ref[tid] = mn;
        }
        named_sync(1, 128);
#pragma unroll
        for (int j = 0; j < NB; ++j) {
#pragma unroll
          for (int e = 0; e < 2; ++e) mr[2 * j + e] = m->m_ref[8 * j + hc + e];
        }
        if (pt > 0) {
#pragma unroll
          for (int j = 0; j < NB; ++j) {
#pragma unroll
            for (int e = 0; e < 2; ++e) l[2 * j + e] *= m->alpha[8 * j + hc + e];
          }
          // rescale O once the previous tile's output MMAs are done
          const int tp = t - 1;
          fail = fail ||
                 !wait_warp(&b_Pempty[tp & 1], (uint32_t)(tp >> 1) & 1u, abort, a.limit_ns);
          tc_fence_after();
          for (int p = 0; p < P.NPd; ++p) {
#pragma unroll
            for (int cb = 0; cb < NH; cb += 8) {
              float v[8];
              const uint32_t ta = lb + kOCol0 + (uint32_t)P.N2 * p + cb;
              tmem_ld8(ta, v);
              tmem_wait_ld();
#pragma unroll
              for (int k = 0; k < 8; ++k) v[k] *= m->alpha[cb + k] * ratio;
              tmem_st8(ta, v);
            }
          }
          tmem_wait_st();
          tc_fence_before();
        }
      }

      // P tile (MN-major core matrices, no swizzle): K slot k, heads 8j..8j+7 at
      // (k/8) lbo_p + 128 j + (k%8) 16; this thread's word for heads 8j + hc + {0, 1} is at
      // + 4 (lane % 4).  lbo_p = 16 N2 + 32 puts the two core rows a warp writes in
      // disjoint banks.
      fail = fail || !wait_warp(&b_Pempty[sb], ((uint32_t)(t >> 1) & 1u) ^ 1u, abort, a.limit_ns);
      {
        const float wa = s_a * inv_srun, wb = s_b * inv_srun;
        uint8_t* pbuf = p_s + sb * P.p_bytes + 4 * (lane & 3);
        uint8_t* pa = pbuf + (ka >> 3) * P.lbo_p + (ka & 7) * 16;
        uint8_t* pbp = pbuf + (kb >> 3) * P.lbo_p + (kb & 7) * 16;
#pragma unroll
        for (int j = 0; j < NB; ++j) {
          float ea[2], eb[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            // a head whose reference is still -inf has only -inf scores so far (any finite
            // score takes the slow path), so a finite stand-in gives 2^-inf = 0 without NaN
            const float m0 = (mr[2 * j + e] == -INFINITY) ? 0.f : mr[2 * j + e];
            ea[e] = ex2_approx(x[4 * j + e] - m0);
            eb[e] = ex2_approx(x[4 * j + 2 + e] - m0);
            l[2 * j + e] += ea[e] + eb[e];
          }
          *reinterpret_cast<uint32_t*>(pa + 128 * j) = h2_bits(__floats2half2_rn(ea[0] * wa, ea[1] * wa));
          *reinterpret_cast<uint32_t*>(pbp + 128 * j) = h2_bits(__floats2half2_rn(eb[0] * wb, eb[1] * wb));
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&b_Pfull[sb]);
      ++pt;

      if (c.last) {
        // -------- epilogue of the piece: partials to the workspace slot blockIdx.x + seq
        fail = fail || !wait_warp(&b_Pempty[sb], (uint32_t)(t >> 1) & 1u, abort, a.limit_ns);
        tc_fence_after();
#pragma unroll
        for (int j = 0; j < NB; ++j) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            float v = l[2 * j + e];
            v += __shfl_xor_sync(0xffffffffu, v, 4);
            v += __shfl_xor_sync(0xffffffffu, v, 8);
            v += __shfl_xor_sync(0xffffffffu, v, 16);
            if (lane < 4) m->red[q][8 * j + 2 * lane + e] = v;
          }
        }
        named_sync(1, 128);
        const int64_t slot = (int64_t)blockIdx.x + c.seq;
        for (int h = tid; h < a.H; h += 128) {
          const float L = (m->red[0][h] + m->red[1][h]) + (m->red[2][h] + m->red[3][h]);
          a.ws_ml[2 * (slot * a.H + h)] = m->m_ref[h];
          a.ws_ml[2 * (slot * a.H + h) + 1] = L;
        }
        if (!fail) {
          float* wo = a.ws_o + slot * a.H * a.d + 32 * q + lane;   // feature 32q + lane, head 0
#pragma unroll 1
          for (int p = 0; p < P.NPd; ++p) {
            const bool fv = 128 * p + 32 * q + lane < a.d;
#pragma unroll 1
            for (int cb = 0; cb < NH; cb += 8) {
              float v[8];
              tmem_ld8(lb + kOCol0 + (uint32_t)P.N2 * p + cb, v);
              tmem_wait_ld();
              if (fv) {
#pragma unroll
                for (int k = 0; k < 8; ++k)
                  if (cb + k < a.H) wo[(int64_t)(cb + k) * a.d + 128 * p] = v[k] * srun;
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(b_oempty);
        named_sync(1, 128);   // red / m_ref reads done before the next piece writes them
      }
      cursor_next(c, off, a.batch, lo, hi);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (tid == 0 && abort_read(abort)) atomicOr(a.flags, KVK_FLAG_TIMEOUT);
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------

struct Plan {
  TcParams p;
  size_t smem;
  bool ok;
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

Plan make_plan(int d, int d_rope, int b, int H, int batch) {
  Plan pl;
  memset(&pl, 0, sizeof(pl));
  TcParams& P = pl.p;
  if (b != 2 && b != 4 && b != 8 && b != 16 && b != KVK_BITS_BF16) return pl;
  const bool stacked = (b == 16);
  const bool in_place = stacked || b == KVK_BITS_BF16;
  const int n = d + d_rope;
  P.N1 = (H + 7) / 8 * 8;
  P.N2 = (H + 15) / 16 * 16;
  P.NP = (n + 127) / 128;
  P.NPd = (d + 127) / 128;
  P.NQA = (n + 63) / 64;
  P.NK16 = (n + 15) / 16;
  // TMEM: S^T (N1 <= 64 columns), two C^T buffers of 4 x 32 columns, O^T NPd x N2 columns
  if (H < 1 || P.N2 > 64 || P.NPd > 4 || kOCol0 + (uint32_t)(P.NPd * P.N2) > kTmemCols) return pl;
  if (P.NQA * 8 > 32 * kQC) return pl;   // staged query rows of up to 768 features
  const size_t q_bytes = (size_t)P.NQA * P.N1 * 128;
  P.lbo_p = (uint32_t)P.N2 * 16u + 32u;
  P.p_bytes = 8u * P.lbo_p;
  const size_t p_bytes = 2 * (size_t)P.p_bytes;
  const size_t misc_bytes = sizeof(Misc) + sizeof(int32_t) * (size_t)(batch + 1);
  const int raw_slot = in_place ? 0 : 64 * 16 * b;   // 16-bit rows land in the slots
  const size_t slot_bytes = stacked ? 4u * kAtom : (size_t)kPair;
  P.raw_slot = raw_slot;
  // try the largest rings that fit
  const size_t fixed = align_up(q_bytes, 1024) + align_up(p_bytes, 1024);
  auto total_for = [&](int PR, int RR) {
    size_t off = fixed;
    off += (size_t)PR * slot_bytes;
    off = align_up(off + (size_t)RR * raw_slot, 1024);
    off = align_up(off + (size_t)(3 * PR + 2 * RR + kFixedBars) * 8, 16);
    off += misc_bytes;
    return off + 1024;   // runtime alignment slack of the dynamic shared memory base
  };
  int PR = 0, RR = 0;
  if (in_place) {
    // TMA lands in the slots: at least a tile's groups
    for (PR = 3 * P.NP; PR >= P.NP; --PR)
      if (total_for(PR, 0) <= (size_t)kSmemLimit) break;
    if (PR < P.NP) return pl;
  } else {
    // f16 slots for one and a half tiles of groups, and the largest raw ring that then fits
    const int want = P.NP + (P.NP + 1) / 2;
    for (PR = want; PR >= P.NP; --PR) {
      for (RR = 4 * P.NP; RR >= 2; --RR)
        if (total_for(PR, RR) <= (size_t)kSmemLimit) break;
      if (RR >= 2 && total_for(PR, RR) <= (size_t)kSmemLimit) break;
    }
    if (PR < P.NP || RR < 2) return pl;
  }
  P.PR = PR;
  P.RR = RR;
  size_t off = fixed;
  P.off_p = (uint32_t)align_up(q_bytes, 1024);
  P.off_pairs = (uint32_t)fixed;
  off += (size_t)PR * slot_bytes;
  P.off_raw = (uint32_t)off;
  off = align_up(off + (size_t)RR * raw_slot, 1024);
  P.off_bar = (uint32_t)off;
  off = align_up(off + (size_t)(3 * PR + 2 * RR + kFixedBars) * 8, 16);
  P.off_misc = (uint32_t)off;
  pl.smem = off + misc_bytes + 1024;
  // score MMA: M = 64 tokens x N1 heads, or stacked M = 128 (high and low rows) x N2 heads
  // (B rows past N1 are read from the next query atom, or from the P buffers after the last
  // one, and give score columns of heads >= H, which the softmax ignores)
  P.idesc1 = stacked ? sm100::idesc_f16(128, P.N2, false, false)
                     : sm100::idesc_f16(64, P.N1, false, false);
  P.idesc2 = sm100::idesc_f16(128, P.N2, false, true);   // A = C^T from TMEM, B = P MN-major
  pl.ok = pl.smem <= (size_t)kSmemLimit;
  return pl;
}

// Registers per thread ptxas allocated to an instance (0 if it cannot be queried, e.g. no GPU).
template <int BITS, int NH>
int instance_regs() {
  static int regs = -1;
  if (regs < 0) {
    cudaFuncAttributes fa;
    regs = (cudaFuncGetAttributes(&fa, decode_tc_kernel<BITS, NH>) == cudaSuccess) ? fa.numRegs : 0;
  }
  return regs;
}
template <int BITS>
int instance_regs_nh(int N2) {
  switch (N2) {
    case 16: return instance_regs<BITS, 16>();
    case 32: return instance_regs<BITS, 32>();
    case 48: return instance_regs<BITS, 48>();
    case 64: return instance_regs<BITS, 64>();
  }
  return 0;
}
// The register budgets assume the launch allocation kLaunchRegs; anything else would make
// the budget changes invalid or leave an increase waiting for registers that never come.
bool launch_regs_ok(int b, int N2) {
  int r = 0;
  switch (b) {
    case 16: r = instance_regs_nh<16>(N2); break;
    case KVK_BITS_BF16: r = instance_regs_nh<KVK_BITS_BF16>(N2); break;
    case 8: r = instance_regs_nh<8>(N2); break;
    case 4: r = instance_regs_nh<4>(N2); break;
    case 2: r = instance_regs_nh<2>(N2); break;
  }
  return r == (int)kLaunchRegs;
}

template <int BITS, int NH>
cudaError_t launch_bits_nh(const TcParams& P, const CUtensorMap& tmap, size_t smem, int grid,
                           cudaStream_t st) {
  auto k = decode_tc_kernel<BITS, NH>;
  if (instance_regs<BITS, NH>() != (int)kLaunchRegs) return cudaErrorNotSupported;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // a programmatic dependent of the kernel before it (see the kernel's prologue)
  e = launch_pdl(k, dim3(grid), dim3(kThreads), smem, st, P, tmap);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int BITS>
cudaError_t launch_bits(const TcParams& P, const CUtensorMap& tmap, size_t smem, int grid,
                        cudaStream_t st) {
  switch (P.N2) {
    case 16: return launch_bits_nh<BITS, 16>(P, tmap, smem, grid, st);
    case 32: return launch_bits_nh<BITS, 32>(P, tmap, smem, grid, st);
    case 48: return launch_bits_nh<BITS, 48>(P, tmap, smem, grid, st);
    case 64: return launch_bits_nh<BITS, 64>(P, tmap, smem, grid, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool tc_packed_supported(const kvk_layout* L, const AnchorDesc& A, int dtype, int H) {
  if (dtype != KVK_BF16 && dtype != KVK_F16) return false;
  if (!A.tmap_ok || anchor_group(L, A) != 0) return false;
  const Plan pl = make_plan(A.d, L->d_rope, A.b, H, L->max_batch);
  return pl.ok && launch_regs_ok(A.b, pl.p.N2);
}

cudaError_t launch_decode_tc_packed(const DecodeArgs& a, const CUtensorMap& tmap, int dtype,
                                    cudaStream_t st) {
  if (a.group != 0) return cudaErrorInvalidValue;
  Plan pl = make_plan(a.d, a.d_rope, a.b, a.H, a.batch);
  if (!pl.ok) return cudaErrorInvalidValue;
  pl.p.a = a;
  pl.p.qdtype = dtype;
  switch (a.b) {
    case 16: return launch_bits<16>(pl.p, tmap, pl.smem, a.G, st);
    case KVK_BITS_BF16: return launch_bits<KVK_BITS_BF16>(pl.p, tmap, pl.smem, a.G, st);
    case 8: return launch_bits<8>(pl.p, tmap, pl.smem, a.G, st);
    case 4: return launch_bits<4>(pl.p, tmap, pl.smem, a.G, st);
    case 2: return launch_bits<2>(pl.p, tmap, pl.smem, a.G, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace kvk
