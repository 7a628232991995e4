// kvk_decode_tc.cu -- tensor-core (tcgen05) split decode over the packed KV-Kaizen cache.
//
// Computes the same partials as the CUDA-core kernel (kvk_decode_fma.cu): for every piece of
// a sequence that the CTA owns, the running max m (log2 units), the weight sum
// l = sum 2^(z2 - m) and the un-normalised output o = sum 2^(z2 - m) c_hat[:d], where
// z2 = log2(e) * sigma * s_t * (q_lat . code_t[:d] + q_rope . code_t[d:])  (absorbed MLA
// attention over the dequantised cache; KV-Kaizen "Background": each decode step reads the
// whole cache).
//
// One persistent CTA per SM walks its slice of the flattened token space (the split charges
// each piece a fixed cost, so a CTA that starts a sequence takes fewer tokens) in tiles of
// 64 tokens.  Warp roles (512 threads, four warpgroups with their own register budgets):
//   warps 0-3  softmax: read S from TMEM, per-token scale, lazy online softmax, write P
//              (f16) to shared memory, rescale O in TMEM when a max grows, write partials
//   warps 4-11 convert: 16-bit rows or packed b-bit codes -> f16 operand tiles (UMMA
//              128-byte-swizzled, K-major) and their transpose into TMEM.  16-bit rows: all
//              eight warps on every 128-feature group, 16 features each; packed
//              (group-scaled) codes: two teams of four warps on alternate groups, 32 features
//              each.  A warp's features are in its TMEM lane quarter of C^T.
//   warp 12    TMA producer: 128-feature groups of 64 packed rows into a ring, and each
//              tile's scales; the stream is read once, so it carries an evict-first L2 policy
//   warp 13    score-MMA issuer (one thread) and TMEM owner
//   warp 14    output-MMA issuer (one thread)
//   warp 15    query warp: each piece's query rows by TMA, scaled to f16 in place; the fused
//              append's new tokens; warms L2 with the queries of later pieces
// Launched with 128 registers per thread; the softmax warpgroup raises its budget to
// kRegsSoftmax, the conversion warpgroups lower theirs to kRegsConvert and the last
// warpgroup to kRegsIssue (4 x 32 x (192 + 2 x 120 + 80) = 65536).
// Per tile:  S^T[64 tok x N heads]   = C[64 x n] . Q^T         (A in smem, TMEM f32)
//            O^T[128 feat x N2 heads] += C^T[128 x 64] . P    (M=128 per 128 latent features,
//                                                               A = C^T in TMEM)
// Heads sit on N, so 40 heads cost N = 40 / 48, never M = 128.  Scores are exact for every
// format: codes of b <= 8 bits and bf16 values are exact in f16; a 16-bit code c is split into
// hi = f16(c) and lo = c - hi (both exact), and a group-scaled value c * s likewise.  Those
// two parts form a stacked A operand: per 16-token block, the 16 rows of high parts and the 16
// rows of low parts, so one M = 128 MMA per K step yields both partial scores, the high ones
// of tokens 16q .. 16q + 15 in TMEM lanes 32q .. 32q + 15 and the low ones in lanes
// 32q + 16 .. 32q + 31, which the softmax adds.  Otherwise the score MMA is M = 64.
// The convert warps turn each group into f16 (in place for 16-bit rows, from a raw ring for
// packed codes) and put their 32 features of it, transposed, into TMEM (tcgen05.st), so a ring
// slot is free as soon as the score MMA has read it; the output MMA reads C^T from TMEM.  The
// transpose fragment orders the 16 tokens of each K step as 0,1,8,9,2,3,10,11,4,5,12,13,6,7,
// 14,15; the softmax warps write P's K rows in that same order.  C^T holds f16(code) (for 16-bit
// codes rounded, relative 2^-12 on the output, inside its tolerance).
// The per-token scale s_t multiplies the S row and is folded into P as p * s_t / S_run, with
// S_run a running power of two >= every scale seen so far (when it grows, O is rescaled by the
// exact ratio).
// Every wait is bounded in time; on expiry the kernel records KVK_FLAG_TIMEOUT, drains its
// own TMA loads and MMAs, frees TMEM and exits.
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
constexpr int kTeamWarps = kConvWarps / 2;   // two conversion teams take alternate groups
constexpr int kTmaWarp = 12;
constexpr int kMmaWarp = 13;   // score MMAs; owns TMEM
constexpr int kMma2Warp = 14;  // output MMAs
constexpr int kQueryWarp = 15; // query staging, fused append
// Register budgets.  The block is launched with kLaunchRegs per thread (the host checks that
// ptxas allocated exactly that before choosing this kernel); a warpgroup whose budget is
// above it raises it (setmaxnreg.inc), one below lowers it (.dec) -- never the other way,
// which would be an illegal instruction -- and the budgets sum to no more than the launch.
constexpr uint32_t kLaunchRegs = 65536 / kThreads;   // 128
constexpr uint32_t kRegsSoftmax = 192, kRegsConvert = 120, kRegsIssue = 80;
static_assert(128 * (kRegsSoftmax + 2 * kRegsConvert + kRegsIssue) <= 65536, "register split");
// 16-bit rows (int16 codes, or the bf16 values of an uncompressed anchor) are converted in
// place in the slot the tensor memory accelerator filled; narrower codes go through a raw ring
template <int BITS>
constexpr bool kInPlace = (BITS == 16 || BITS == KVK_BITS_BF16);
template <uint32_t N>
__device__ __forceinline__ void regs_set() {
  if constexpr (N > kLaunchRegs) regs_inc<N>();
  else if constexpr (N < kLaunchRegs) regs_dec<N>();
}
constexpr int kTile = kTcTileTokens;   // 64
constexpr int kAtom = 8192;            // 64 rows x 128 bytes (64 f16 features)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSCol = 0;          // scores S^T, one buffer (N1 <= 64 columns)
constexpr uint32_t kCtCol0 = 64;       // C^T double buffer: 64 + 128 b, latent group p at + 32 p
constexpr uint32_t kOCol0 = 320;       // O^T group p at 320 + N2 p
// limit of the waits that drain a stopping kernel's own loads and MMAs (they always end)
constexpr uint64_t kDrainLimitNs = 2000000000ull;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kSmemLimit = 232448;
// 16-byte chunks per lane of a half warp per staged query row (rows of up to 768 features)
constexpr int kQL = 6;   // (a bound on the row: 16 kQL chunks of 8 features)
// Scale ring: per tile one window of the tile's fp16 scales (64 tokens x sg scales, from the
// 16-byte boundary at or below the first, rounded up to 16 bytes: 144 bytes for one scale per
// token), loaded by the TMA warp with a plain bulk copy.
constexpr int kScSlots = 4;
// barriers besides the rings: s full/empty, P full/empty (2), C^T full/empty (2), q full/empty,
// o empty, two MMA drains, q seen, appended, q landed, scale full/empty (kScSlots each)
constexpr int kFixedBars = 2 + 4 + 4 + 8 + 2 * kScSlots;

struct TcParams {
  DecodeArgs a;
  int N1, N2;           // staged query rows (heads rounded to 8); N of the output MMA (to 16)
  int NP, NPd;          // 128-feature groups per row, and those holding latent features
  int NQA, NK16;        // 64-feature query atoms, 16-feature K steps
  int PR, RR, raw_slot; // ring slots (f16 groups, packed groups) and packed-group bytes
  int stacked;          // score A = exact high + low parts (16-bit codes, group scales): M = 128
  uint32_t atom_bytes;  // one 64-feature atom of a group slot (8 KB, 16 KB stacked)
  uint32_t slot_bytes;  // one group slot: 2 atoms
  uint32_t rbs;         // bytes per 16-token block of an atom (2048, 4096 stacked)
  uint32_t lbo_p;       // bytes between the 8-token core-matrix rows of P (16 N2 + 32)
  uint32_t p_bytes;     // one P buffer: 8 lbo_p
  uint32_t off_p, off_pairs, off_raw, off_bar, off_misc;
  uint32_t idesc1, idesc2;
  int qdtype;           // KVK_BF16 or KVK_F16
  uint32_t off_sc, sc_bytes;   // scale windows: ring offset and bytes per window (0: none)
  int grouped;          // scales per element group, applied by the convert warps
};

struct Misc {
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
// (rounded to nearest) and
// lo = code - hi: with hb, lb the code's bytes (exact in f16), t = (hb - 128) * 256 - hi is an
// integer of magnitude <= 263 (so the fused multiply-add is exact), and lo = t + lb an integer
// of magnitude <= 8 (f16 spacing is at most 16 below 2^15): q . code = q . hi + q . lo exactly.
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

// Byte offset of token row r (0..63) of 64-feature atom a inside a group slot.  A plain slot
// holds each atom's 64 rows contiguously (rbs = 2048: 16 rows of 128 bytes per block); a
// stacked slot interleaves, per 16-token block, the 16 rows of high parts with the 16 rows of
// low parts of the same tokens (rbs = 4096, low block at + kLoOff), so that one M = 128 score
// MMA reads A rows [hi 0-15, lo 0-15, hi 16-31, lo 16-31, ...] and TMEM lane quarter q receives
// the high and the low scores of tokens 16q .. 16q + 15.
constexpr uint32_t kLoOff = 2048;
__device__ __forceinline__ uint32_t slot_addr(int a, int r, uint32_t atom_bytes, uint32_t rbs) {
  return (uint32_t)a * atom_bytes + (uint32_t)(r >> 4) * rbs + (uint32_t)(r & 15) * 128u;
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
// features fb .. fb+15 (eight-feature groups g = fb/8 + {0, 1} of every row), in two halves:
// load_group reads this lane's packed words (all four rows before any use), store_group
// unpacks them and writes the f16 rows.
template <int BITS>
constexpr int kPackedWords = (BITS == 8) ? 2 : 1;   // 32-bit words per row chunk of a lane

template <int BITS>
__device__ __forceinline__ void load_group(const uint8_t* rawslot, int lane, int fb,
                                           uint32_t (&w)[4][kPackedWords<BITS>]) {
  const int g = (fb >> 3) + (lane & 1);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = conv_row(lane, k);
    if constexpr (BITS == 8) {
      const uint2 u = *reinterpret_cast<const uint2*>(rawslot + r * 128 +
                                                      (((g >> 1) ^ (r & 7)) << 4) + ((g & 1) << 3));
      w[k][0] = u.x;
      w[k][kPackedWords<BITS> - 1] = u.y;
    } else if constexpr (BITS == 4) {
      w[k][0] = *reinterpret_cast<const uint32_t*>(
          rawslot + r * 64 + (((g >> 2) ^ ((r >> 1) & 3)) << 4) + ((g & 3) << 2));
    } else {   // BITS == 2
      w[k][0] = *reinterpret_cast<const uint16_t*>(
          rawslot + r * 32 + (((g >> 3) ^ ((r >> 2) & 1)) << 4) + ((g & 7) << 1));
    }
  }
}

// SCALED: each row's f16 values are multiplied by that row's group scale sc[k] (both halves):
// the dequantised value code * s of a group-scaled cache, split exactly into hi = f16(code * s)
// (stored at the row's place) and lo = code * s - hi (stored kLoOff bytes further, in the
// stacked slot's low-part block of the same 16 tokens; the fused multiply-add is exact, the
// product of a b <= 8 bit code and an 11-bit scale having at most 18 significant bits).
// Token row r of atom a sits at a * atom_bytes + (r / 16) * rbs + (r % 16) * 128 (slot_addr).
template <int BITS, bool SCALED>
__device__ __forceinline__ void store_group(const uint32_t (&w)[4][kPackedWords<BITS>],
                                            uint8_t* pair, int lane, int fb,
                                            const __half2 (&sc)[4], uint32_t atom_bytes,
                                            uint32_t rbs) {
  const int g = (fb >> 3) + (lane & 1);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = conv_row(lane, k);
    uint4 o;
    if constexpr (BITS == 8) {
      const __half2 bias = __float2half2_rn(1152.f);
      o.x = cvt_small(w[k][0], 0x4140u, bias);
      o.y = cvt_small(w[k][0], 0x4342u, bias);
      o.z = cvt_small(w[k][kPackedWords<BITS> - 1], 0x4140u, bias);
      o.w = cvt_small(w[k][kPackedWords<BITS> - 1], 0x4342u, bias);
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
    const uint32_t at = slot_addr(g >> 3, r, atom_bytes, rbs) + (((g & 7) ^ (r & 7)) << 4);
    if constexpr (SCALED) {
      uint4 h, l;
      h.x = h2_bits(__hmul2(bits_h2(o.x), sc[k]));
      h.y = h2_bits(__hmul2(bits_h2(o.y), sc[k]));
      h.z = h2_bits(__hmul2(bits_h2(o.z), sc[k]));
      h.w = h2_bits(__hmul2(bits_h2(o.w), sc[k]));
      l.x = h2_bits(__hfma2(bits_h2(o.x), sc[k], __hneg2(bits_h2(h.x))));
      l.y = h2_bits(__hfma2(bits_h2(o.y), sc[k], __hneg2(bits_h2(h.y))));
      l.z = h2_bits(__hfma2(bits_h2(o.z), sc[k], __hneg2(bits_h2(h.z))));
      l.w = h2_bits(__hfma2(bits_h2(o.w), sc[k], __hneg2(bits_h2(h.w))));
      *reinterpret_cast<uint4*>(pair + at) = h;
      *reinterpret_cast<uint4*>(pair + at + kLoOff) = l;
    } else {
      *reinterpret_cast<uint4*>(pair + at) = o;
    }
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
decode_tc_kernel(const __grid_constant__ TcParams P, const __grid_constant__ CUtensorMap tmap,
                 const __grid_constant__ CUtensorMap qmap_l, const __grid_constant__ CUtensorMap qmap_r) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, derived from the shared array by an offset so that every
  // pointer below stays in the shared state space (plain LDS / STS, not generic accesses)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const DecodeArgs& a = P.a;
  uint8_t* q_s = smem;
  uint8_t* p_s = smem + P.off_p;
  uint8_t* pairs = smem + P.off_pairs;
  uint8_t* raw = smem + P.off_raw;
  uint8_t* scw = smem + P.off_sc;         // [kScSlots] scale windows
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
  uint64_t* b_qload = b_app + 1;          // a piece's query rows landed (TMA)
  uint64_t* b_scfull = b_qload + 1;       // [kScSlots] scale window landed
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
      // every convert warp (16-bit rows), or the team converting the group (packed codes)
      mbar_init(&b_pfull[i], kInPlace<BITS> ? kConvWarps : kTeamWarps);
      // score MMAs (commit), plus the convert warps where they read the slot after q_full
      mbar_init(&b_pempty[i], kInPlace<BITS> ? 1 : 1 + kTeamWarps);
      mbar_init(&b_tfull[i], 1);
    }
    for (int i = 0; i < P.RR; ++i) {
      mbar_init(&b_rfull[i], 1);
      mbar_init(&b_rempty[i], kTeamWarps);
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
    mbar_init(b_qload, 1);
    for (int i = 0; i < kScSlots; ++i) {
      mbar_init(&b_scfull[i], 1);
      // released by the softmax warps (token scales) or the convert warps (group scales)
      mbar_init(&b_scempty[i], P.grouped ? kConvWarps : 4);
    }
    m->abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&m->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kTmaWarp && lane == 0) tma_prefetch_desc(&tmap);
  if (warp == kQueryWarp && lane == 0) {
    tma_prefetch_desc(&qmap_l);
    if (a.d_rope > 0) tma_prefetch_desc(&qmap_r);
  }
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
        // hold the first cache loads until the first query rows have landed: their loads then
        // do not queue behind every CTA's ring fill
        mbar_wait(b_qload, 0u, abort, a.limit_ns);
        // a fused append writes this CTA's new tokens first (the spare warp)
        if (a.app_c) mbar_wait(b_app, 0u, abort, a.limit_ns);
        Ring sr;   // scale ring
        uint32_t nsc = 0;
        const uint64_t pol = policy_evict_first();   // the cache and its scales are read once
        while (c.valid && !abort_read(abort)) {
          const int row0 = c.seq * a.max_tokens + c.pos;
          bool ok = true;
          if constexpr (BITS != 0) {   // this tile's scale window (the arena has tail slack)
            const uintptr_t sp = reinterpret_cast<uintptr_t>(a.scales + (int64_t)row0 * a.sg);
            if (!(ok = mbar_wait(&b_scempty[sr.slot], sr.phase ^ 1u, abort, a.limit_ns))) break;
            mbar_arrive_expect_tx(&b_scfull[sr.slot], P.sc_bytes);
            bulk_load_hint(scw + sr.slot * P.sc_bytes,
                           reinterpret_cast<const void*>(sp & ~uintptr_t(15)), P.sc_bytes,
                           &b_scfull[sr.slot], pol);
            sr.next(kScSlots);
            ++nsc;
          }
          for (int p = 0; p < P.NP && ok; ++p) {
            const uint32_t s = rg.slot, ph = rg.phase;
            if (kInPlace<BITS>) {
              if (!(ok = mbar_wait(&b_pempty[s], ph ^ 1u, abort, a.limit_ns))) break;
              // each atom's 64 rows land contiguously at the start of the atom's place (a
              // stacked slot's convert warps then move them into the interleaved layout)
              const int nat = ((2 * p + 1) * 64 < a.n) ? 2 : 1;
              mbar_arrive_expect_tx(&b_tfull[s], nat * kAtom);
              for (int t = 0; t < nat; ++t)
                tma_load_2d_hint(pairs + s * P.slot_bytes + t * P.atom_bytes, &tmap,
                                 (2 * p + t) * 128, row0, &b_tfull[s], pol);
            } else {
              if (!(ok = mbar_wait(&b_rempty[s], ph ^ 1u, abort, a.limit_ns))) break;
              mbar_arrive_expect_tx(&b_rfull[s], P.raw_slot);
              tma_load_2d_hint(raw + s * P.raw_slot, &tmap, p * 16 * BITS, row0, &b_rfull[s], pol);
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
      // A: M = 64 rows of one atom, or (stacked) M = 128 rows, the atom's interleaved high- and
      // low-part blocks; B: the staged query atom (N = heads rounded to 8, or to 16 when
      // stacked: rows past N1 are read from the next atom, or from the P buffers after the
      // last one, and give score columns of heads >= H, which the softmax ignores)
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
            const uint64_t ad = a0 + ((s * P.slot_bytes + t * P.atom_bytes) >> 4);
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
      // ------------------------------------------------------------------ query warp
      // Loads each piece's query rows [N1][n] with TMA into the 64-feature atoms of the score
      // MMAs' B (heads >= H and features past each part zero-filled); the convert warps then
      // scale and convert them in place.
      const int lat_atoms = a.d / 64;
      const uint32_t q_atom = (uint32_t)P.N1 * 128u;
      auto issue_q = [&](int seq) {
        if (lane == 0) {
          mbar_arrive_expect_tx(b_qload, (uint32_t)P.NQA * q_atom);
          for (int at = 0; at < P.NQA; ++at) {
            if (at < lat_atoms) tma_load_3d(q_s + at * q_atom, &qmap_l, 64 * at, 0, seq, b_qload);
            else tma_load_3d(q_s + at * q_atom, &qmap_r, 64 * (at - lat_atoms), 0, seq, b_qload);
          }
        }
        __syncwarp();
      };
      Cursor c;
      cursor_start(c, seq0, off, a.batch, lo, hi);
      uint32_t nq = 0;   // query loads issued
      if (c.valid) {
        issue_q(c.seq);
        ++nq;
      }
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
      // Warm L2 with the queries of the later pieces (their TMA loads then hit L2).
      {
        Cursor w = c;
        const int lat_lines = (2 * a.d + 127) / 128, rope_lines = (2 * a.d_rope + 127) / 128;
        const int lines = lat_lines + rope_lines;
        while (w.valid) {
          ++w.seq;
          if (!(w.valid = find_piece(w, off, a.batch, lo, hi))) break;
          const uint8_t* ql = static_cast<const uint8_t*>(a.q_lat) + 2 * ((int64_t)w.seq * a.ql_ss);
          const uint8_t* qr =
              static_cast<const uint8_t*>(a.q_rope) + 2 * ((int64_t)w.seq * a.qr_ss);
          for (int i = lane; i < a.H * lines; i += 32) {
            const int h = i / lines, k = i - h * lines;
            if (k < lat_lines) prefetch_l2(ql + 2 * ((int64_t)h * a.ql_sh) + 128 * k);
            else prefetch_l2(qr + 2 * ((int64_t)h * a.qr_sh) + 128 * (k - lat_lines));
          }
        }
      }
      // Later pieces: the rows of piece k are loaded once piece k-1's score MMAs are done
      // with the atoms and the softmax warps have taken its scales; the convert warps scale
      // them when they reach the piece.
      bool fail = false;
      for (int piece = 1; !fail; ++piece) {
        ++c.seq;
        if (!(c.valid = find_piece(c, off, a.batch, lo, hi))) break;
        fail = !wait_warp(b_qempty, ((uint32_t)piece & 1u) ^ 1u, abort, a.limit_ns) ||
               !wait_warp(b_qseen, ((uint32_t)piece - 1u) & 1u, abort, a.limit_ns);
        if (!fail) {
          issue_q(c.seq);
          ++nq;
        }
      }
      // the last query load this warp issued has landed before the block exits (after an
      // abort it may still be in flight)
      if (nq > 0 && lane == 0) wait_noabort(b_qload, (nq - 1) & 1u);
      __syncwarp();
    }
  } else if (has_work && warp >= kConvWarp0) {
    regs_set<kRegsConvert>();
    // ------------------------------------------------------------------ convert
    // 16-bit rows: every warp converts every group, warp cw the 16 features 32 cq + 16 (cw / 4)
    // .. + 15 (cq = cw % 4).  Packed codes: two teams of four warps take alternate groups (team
    // cw / 4 converts the CTA's groups with the team's parity), so two groups are in flight; in
    // its team's groups warp cw owns the 32 features 32 cq .. 32 cq + 31.  Either way a warp's
    // features are in its own TMEM lane quarter of C^T.
    // The warps share no barrier among themselves (every hand-off is an mbarrier), so a warp
    // that stops on a failed wait leaves its loop alone; it then arrives on nothing more, and
    // everything downstream of the group it stopped at waits until it sees the abort word.
    const int cw = warp - kConvWarp0;
    const int cq = cw & 3, team = cw >> 2;
    Ring pr, rr;   // f16 group ring, packed group ring
    Ring sr;       // scale windows (group-scaled cache only)
    bool fail = false;
    // this lane's ldmatrix row address inside a group slot, per 16-feature half h and 16-token
    // block tg: atom cq/2, 16-byte chunk 4(cq%2) + 2h + (lane/8)/2 of token
    // 16tg + 8((lane/8)%2) + lane%8, in the slot's layout (aoff; the low part of a stacked
    // slot at + kLoOff) and, for 16-bit rows, where TMA put it (roff: the atom's 64 rows
    // contiguous from the atom's start; the same as aoff in a plain slot).  Both keep the
    // 128-byte swizzle phase (token % 8), so a warp's cells stay in its own 16-byte columns:
    // it reads all of them (ldmatrix) before it writes any, and no other warp touches them.
    uint32_t aoff[2][4], roff[2][4];
    {
      const int mi = lane >> 3, r8 = lane & 7;
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int tg = 0; tg < 4; ++tg) {
          const int tok = 16 * tg + 8 * (mi & 1) + r8;
          const uint32_t col = (uint32_t)(((4 * (cq & 1) + 2 * h + (mi >> 1)) ^ r8) << 4);
          aoff[h][tg] = slot_addr(cq >> 1, tok, P.atom_bytes, P.rbs) + col;
          roff[h][tg] = (uint32_t)(cq >> 1) * P.atom_bytes + (uint32_t)tok * 128u + col;
        }
    }
    const uint32_t pairs_u = smem_u32(pairs);
    // does this warp own features of group p (the last group may hold only one atom)?
    auto owns_group = [&](int p) { return (cq >> 1) < (((2 * p + 1) * 64 < a.n) ? 2 : 1); };
    // ldmatrix (transposed) of this warp's 32 features x 64 tokens of a group slot, in the
    // slot layout (off = aoff) or as TMA left them (off = roff)
    auto ldsm32 = [&](uint32_t base, const uint32_t (&off)[2][4], uint32_t (&x)[32]) {
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int tg = 0; tg < 4; ++tg) {
          uint32_t d4[4];
          ldsm_x4_trans(base + off[h][tg], d4);
#pragma unroll
          for (int i = 0; i < 4; ++i) x[16 * h + 4 * tg + i] = d4[i];
        }
    };
    // the same for 16 features (one half's offsets; register 4 tg + i: 16-token block tg)
    auto ldsm16 = [&](uint32_t base, const uint32_t (&off)[4], uint32_t (&x)[16]) {
#pragma unroll
      for (int tg = 0; tg < 4; ++tg) {
        uint32_t d4[4];
        ldsm_x4_trans(base + off[tg], d4);
#pragma unroll
        for (int i = 0; i < 4; ++i) x[4 * tg + i] = d4[i];
      }
    };
    auto stsm16 = [&](uint32_t base, const uint32_t (&off)[4], const uint32_t (&x)[16]) {
#pragma unroll
      for (int tg = 0; tg < 4; ++tg) {
        const uint32_t d4[4] = {x[4 * tg], x[4 * tg + 1], x[4 * tg + 2], x[4 * tg + 3]};
        stsm_x4_trans(base + off[tg], d4);
      }
    };
    // this warp's C^T: TMEM lanes 32 cq .. 32 cq + 31, columns of latent group p
    auto tmem_st32 = [&](uint32_t col, const uint32_t (&x)[32]) {
      const uint32_t* x0 = x;
      tmem_st16x256b_x4(tmem + ((uint32_t)(32 * cq) << 16) + col,
                        *reinterpret_cast<const uint32_t(*)[16]>(x0));
      tmem_st16x256b_x4(tmem + ((uint32_t)(32 * cq + 16) << 16) + col,
                        *reinterpret_cast<const uint32_t(*)[16]>(x0 + 16));
    };
    Cursor c;
    cursor_start(c, seq0, off, a.batch, lo, hi);
    const uint32_t q_atom = (uint32_t)P.N1 * 128u;
    const int cpr = P.NQA * 8;   // 16-byte chunks per staged query row
    const int hs = lane >> 4, l16 = lane & 15;
    while (c.valid) {
      if (fail || abort_read(abort)) break;
      if (c.first) {
        // Stage the piece's query once its rows have landed: row h scaled by 2^e_h so that
        // max |q_h| lands in [2^14, 2^15) (exact for bf16 inputs in range) and rounded to f16
        // in place; the softmax warps apply 2^-e_h.  Each warp takes row pairs 2 cw + 16 i
        // (one row per half warp; lane l16 holds the row's 16-byte chunks l16, l16 + 16, ...).
        fail = fail || !wait_warp(b_qload, (uint32_t)c.piece & 1u, abort, a.limit_ns);
        if (fail) break;
#pragma unroll 1
        for (int hb = 2 * cw; hb < P.N1; hb += 2 * kConvWarps) {
          // compact loops: this code runs once per piece, so it is mostly fetched cold
          const int h = hb + hs;
          const uint32_t rbase = smem_u32(q_s) + (uint32_t)h * 128u;
          float mx = 0.f;
#pragma unroll 1
          for (int fc = l16; fc < cpr; fc += 16) {
            float f[8];
            load8_bits(lds128(rbase + (fc >> 3) * q_atom + (((fc & 7) ^ (h & 7)) << 4)), P.qdtype,
                       f);
#pragma unroll
            for (int e = 0; e < 8; ++e) mx = fmaxf(mx, fabsf(f[e]));
          }
#pragma unroll
          for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          // e = 14 - floor(log2 max |q|) from the exponent field (a subnormal max counts as
          // 2^-126), at most 126 so that 2^e and 2^-e are normal floats
          int e = 0;
          if (mx > 0.f && isfinite(mx))
            e = min(14 - (max((__float_as_int(mx) >> 23) & 0xff, 1) - 127), 126);
          const float qscale = __int_as_float((127 + e) << 23);
          if (l16 == 0) m->qs_inv[c.piece & 1][h] = __int_as_float((127 - e) << 23);
#pragma unroll 1
          for (int fc = l16; fc < cpr; fc += 16) {
            const uint32_t addr = rbase + (fc >> 3) * q_atom + (((fc & 7) ^ (h & 7)) << 4);
            float f[8];
            load8_bits(lds128(addr), P.qdtype, f);
            uint4 o;
            o.x = h2_bits(__floats2half2_rn(f[0] * qscale, f[1] * qscale));
            o.y = h2_bits(__floats2half2_rn(f[2] * qscale, f[3] * qscale));
            o.z = h2_bits(__floats2half2_rn(f[4] * qscale, f[5] * qscale));
            o.w = h2_bits(__floats2half2_rn(f[6] * qscale, f[7] * qscale));
            sts128(addr, o);
          }
        }
        fence_proxy_async_smem();   // the generic writes, visible to the score MMAs
        __syncwarp();
        if (lane == 0) mbar_arrive(b_qfull);
      }
      const int ctb = c.tile & 1;   // C^T buffer of this tile
      const uint32_t ct_col = kCtCol0 + 128u * ctb;
      // the output MMAs of tile - 2 have finished reading this C^T buffer (waited before the
      // team's first store of the tile, and by every warp before it arrives on the buffer's
      // full barrier: a team that stores no C^T -- the one converting only the rope group when
      // d <= 128 -- would otherwise run two tiles ahead and arrive twice in one phase)
      bool ct_waited = false;
      // the teams take alternate groups of the CTA's whole group sequence (with an odd number
      // of groups per tile, each team's share alternates between tiles)
      const int gbase = c.tile * P.NP;
      auto wait_ct = [&]() {
        fail = fail || !wait_warp(&b_ctempty[ctb], ((uint32_t)(c.tile >> 1) & 1u) ^ 1u, abort,
                                  a.limit_ns);
        tc_fence_after();
        ct_waited = true;
      };
      if constexpr (kInPlace<BITS>) {
        // In place, 16-bit codes (or bf16 values) -> f16, in one pass through registers, by all
        // eight convert warps on every group: warp cw takes the 16 features of half hf = cw / 4
        // of its lane quarter's 32 (a group's conversion then takes half as long as with one
        // team of four).  Each 8x8 block (8 tokens x 8 features) is loaded transposed, converted
        // element by element, stored back transposed (row-major again, for the score MMAs;
        // 16-bit codes as exact high and low parts in the stacked slot) and the same registers,
        // now feature-major, go to C^T in TMEM (lanes 32 cq + 16 hf ..).  The relocation from
        // where TMA put the rows stays inside the warp's own 16-byte columns, all of which it
        // reads before it writes any.  The slot is not read after p_full, so only the score MMAs
        // release it.
        const int hf = team;
        uint32_t ao[4], ro[4];   // this warp's half of aoff / roff
#pragma unroll
        for (int tg = 0; tg < 4; ++tg) {
          ao[tg] = hf ? aoff[1][tg] : aoff[0][tg];
          ro[tg] = hf ? roff[1][tg] : roff[0][tg];
        }
        for (int p = 0; p < P.NP; ++p) {
          const uint32_t s = pr.slot;
          fail = fail || !wait_warp(&b_tfull[s], pr.phase, abort, a.limit_ns);
          const bool go = !fail && owns_group(p);
          const uint32_t sbase = pairs_u + s * P.slot_bytes;
          uint32_t x[16], xl[16];
          if (go) {
            ldsm16(sbase, ro, x);
            if constexpr (BITS == 16) {
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
          }
          if (go && !fail) {
            stsm16(sbase, ao, x);
            if constexpr (BITS == 16) stsm16(sbase + kLoOff, ao, xl);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && !fail) mbar_arrive(&b_pfull[s]);
          if (p < P.NPd) {
            if (!ct_waited) wait_ct();
            if (go && !fail)
              tmem_st16x256b_x4(tmem + ((uint32_t)(32 * cq + 16 * hf) << 16) + ct_col + 32u * p, x);
          }
          pr.next(P.PR);
        }
      } else {
        // Packed codes: the team's group is read from the raw ring into registers (and the raw
        // slot released), unpacked into its f16 slot -- with a group-scaled cache multiplied by
        // the group scales and split into exact high and low parts -- and this warp's 32
        // features are read back transposed into C^T.
        constexpr int NW = kPackedWords<BITS>;
        // group-scaled cache: this tile's scale window (rows past the piece's end get scale 0)
        const __half* wsc = nullptr;
        if (P.grouped) {
          fail = fail || !wait_warp(&b_scfull[sr.slot], sr.phase, abort, a.limit_ns);
          wsc = reinterpret_cast<const __half*>(scw + sr.slot * P.sc_bytes) +
                ((reinterpret_cast<uintptr_t>(a.scales + ((int64_t)c.seq * a.max_tokens + c.pos) *
                                                             a.sg) & 15u) >> 1);
        }
        for (int p = 0; p < P.NP; ++p) {
          if (((p + gbase) & 1) == team) {
            const uint32_t s = pr.slot, ph = pr.phase, rs = rr.slot;
            uint8_t* pair = pairs + s * P.slot_bytes;
            uint32_t w[2][4][NW];
            fail = fail || !wait_warp(&b_rfull[rs], rr.phase, abort, a.limit_ns);
            if (!fail) {
              load_group<BITS>(raw + rs * P.raw_slot, lane, 32 * cq, w[0]);
              load_group<BITS>(raw + rs * P.raw_slot, lane, 32 * cq + 16, w[1]);
            }
            __syncwarp();
            if (lane == 0 && !fail) mbar_arrive(&b_rempty[rs]);
            fail = fail || !wait_warp(&b_pempty[s], ph ^ 1u, abort, a.limit_ns);
            if (!fail) {
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int fb = 32 * cq + 16 * h;
                if (P.grouped) {
                  // scale index of this lane's eight features: (128 p + fb + 8 (lane % 2)) / G
                  const int j = (128 * p + fb + 8 * (lane & 1)) / a.group;
                  __half2 sc[4];
#pragma unroll
                  for (int k = 0; k < 4; ++k) {
                    const int r = conv_row(lane, k);
                    const __half sv = (r < c.cnt) ? wsc[r * a.sg + j] : __float2half(0.f);
                    sc[k] = __halves2half2(sv, sv);
                  }
                  store_group<BITS, true>(w[h], pair, lane, fb, sc, P.atom_bytes, P.rbs);
                } else {
                  const __half2 one[4] = {};
                  store_group<BITS, false>(w[h], pair, lane, fb, one, P.atom_bytes, P.rbs);
                }
              }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && !fail) mbar_arrive(&b_pfull[s]);
            if (p < P.NPd) {
              if (!ct_waited) wait_ct();
              if (!fail && owns_group(p)) {
                uint32_t x[32];
                ldsm32(smem_u32(pair), aoff, x);
                tmem_st32(ct_col + 32u * p, x);
              }
            }
            __syncwarp();
            if (lane == 0 && !fail) mbar_arrive(&b_pempty[s]);   // this warp is done with the slot
          }
          pr.next(P.PR);
          rr.next(P.RR);
        }
        if (P.grouped) {   // the tile's scale window is no longer read by this warp
          __syncwarp();
          if (lane == 0 && !fail) mbar_arrive(&b_scempty[sr.slot]);
          sr.next(kScSlots);
        }
      }
      if (!ct_waited) wait_ct();
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && !fail) mbar_arrive(&b_ctfull[ctb]);
      cursor_next(c, off, a.batch, lo, hi);
    }
    tmem_wait_st();   // no TMEM store of this warp is outstanding when the role ends
  } else if (has_work) {
    regs_set<kRegsSoftmax>();
    // ------------------------------------------------------------------ softmax
    // Thread layout: lane t of warp q holds token r = 16q + t % 16 of the tile and the HH = NH/2
    // heads h0 .. h0 + HH - 1, h0 = HH (t / 16).  S^T is read with the 32x32b shape (thread t
    // <-> TMEM lane 32q + t, every column):
    //  - M = 64 score MMA: rows 16q .. 16q + 15 sit in lanes 32q .. 32q + 15 and lanes 16-31 of
    //    the quarter hold nothing, so thread t >= 16 takes its heads of token 16q + t - 16 from
    //    lane t - 16;
    //  - stacked M = 128 score MMA: lane 32q + t (t < 16) holds the high-part scores of token
    //    16q + t and lane 32q + 16 + t its low-part scores, and each thread adds the other
    //    lane's partial scores of its heads.
    // One shuffle per head either way.  The four warps leave the loop only together (named_or
    // agreement every tile).
    constexpr int HH = NH / 2;
    constexpr int NHB = HH / 8;   // 8-head blocks of a thread
    const int q = warp;
    const uint32_t lb = tmem + ((uint32_t)(32 * q) << 16);
    const int hf = lane >> 4;
    const int u = lane & 15;
    const int r = 16 * q + u;     // this thread's token in the tile
    const int h0 = HH * hf;       // this thread's first head
    const bool stacked = P.stacked != 0;
    bool fail = false;

    // S_run: running power of two >= every token scale seen so far (P = p * s / S_run keeps
    // P <= 2^8 in f16).  It only grows; when a tile brings a larger scale the slow path
    // rescales O by S_old / S_new, exactly (powers of two), together with any max update.
    float srun = 0.f, inv_srun = 0.f;

    float l[HH];    // partial weight sums of this thread's heads (its token)
    float mr[HH];   // reference max of this thread's heads (log2 units)
    float qh[HH];   // 2^-e_h of this thread's heads in the current piece
    int pt = 0;
    Cursor c;
    cursor_start(c, seq0, off, a.batch, lo, hi);
    const float coef0 = a.sigma * kLog2e;
    // K slot of token r in P: the transposed C^T holds, in the 16 K slots of each step, tokens
    // 0,1,8,9,2,3,10,11,4,5,12,13,6,7,14,15 of the step's 16 tokens
    const int kslot = 16 * q + 4 * ((u & 7) >> 1) + 2 * (u >> 3) + (u & 1);
    // Token scales come from the tile's scale window in shared memory (bulk-copied by the TMA
    // warp at least a tile ahead): no global loads in this role, so the proxy fence after each
    // P write has nothing outstanding to wait for.
    Ring sr;
    while (c.valid) {
      const int t = c.tile, sb = t & 1;
      float s_r = 0.f;
      if (BITS == 0 || (!kInPlace<BITS> && P.grouped)) {
        // uncompressed rows, or scales applied per group by the convert warps: unit token scale
        s_r = (r < c.cnt) ? 1.f : 0.f;
      } else {
        fail = fail || !mbar_wait(&b_scfull[sr.slot], sr.phase, abort, a.limit_ns);
        const __half* w = reinterpret_cast<const __half*>(scw + sr.slot * P.sc_bytes) +
                          ((reinterpret_cast<uintptr_t>(a.scales + (int64_t)c.seq * a.max_tokens +
                                                        c.pos) & 15u) >> 1);
        if (r < c.cnt) s_r = __half2float(w[r]);
        __syncwarp();
        if (lane == 0 && !fail) mbar_arrive(&b_scempty[sr.slot]);
        sr.next(kScSlots);
      }
      if (c.first) {
        fail = fail || !mbar_wait(b_qfull, (uint32_t)c.piece & 1u, abort, a.limit_ns);
#pragma unroll
        for (int j = 0; j < HH; ++j) qh[j] = m->qs_inv[c.piece & 1][h0 + j];
        __syncwarp();
        if (lane == 0 && !fail) mbar_arrive(b_qseen);
#pragma unroll
        for (int j = 0; j < HH; ++j) {
          l[j] = 0.f;
          mr[j] = -INFINITY;
        }
        pt = 0;
      }
      const bool vr = r < c.cnt;
      const float cr = coef0 * s_r;
      fail = fail || !mbar_wait(b_sfull, (uint32_t)t & 1u, abort, a.limit_ns);
      tc_fence_after();
      float x[HH];
      // columns j and HH + j of the thread's lane, in kSplit rounds (fewer live registers at
      // 64 heads)
      constexpr int kSplit = (NH == 64) ? 2 : 1;
      constexpr int CH = HH / kSplit;
#pragma unroll
      for (int sp = 0; sp < kSplit; ++sp) {
        float v[2 * CH];
#pragma unroll
        for (int k = 0; k < CH / 8; ++k) {
          tmem_ld8(lb + kSCol + (uint32_t)(sp * CH + 8 * k), *reinterpret_cast<float(*)[8]>(v + 8 * k));
          tmem_ld8(lb + kSCol + (uint32_t)(HH + sp * CH + 8 * k),
                   *reinterpret_cast<float(*)[8]>(v + CH + 8 * k));
        }
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < CH; ++j) {
          const float send = (stacked && hf) ? v[j] : v[CH + j];
          const float y = __shfl_xor_sync(0xffffffffu, send, 16);
          const float own = hf ? v[CH + j] : v[j];
          x[sp * CH + j] = stacked ? own + y : (hf ? y : own);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0 && !fail) mbar_arrive(b_sempty);
      bool mine = (pt == 0) || s_r > srun;
#pragma unroll
      for (int j = 0; j < HH; ++j) {
        const bool hv = (h0 + j) < a.H;
        x[j] = (vr && hv) ? x[j] * qh[j] * cr : -INFINITY;
        mine = mine || (x[j] > mr[j] + 8.f);
      }
      // lazy running max: recompute (and rescale) only when a score exceeds the reference
      // by more than 2^8, so P stays within f16 range without touching O every tile
      if (named_or(1, 128, mine || fail || abort_read(abort))) {
        if (named_or(1, 128, fail || abort_read(abort))) break;
#pragma unroll
        for (int j = 0; j < HH; ++j) {   // tile max per head over the warp's 16 tokens
          float v = x[j];
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
          if (u == 0) m->red[q][h0 + j] = v;
        }
        {
          float sm = s_r;
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
        for (int j = 0; j < HH; ++j) mr[j] = m->m_ref[h0 + j];
        if (pt > 0) {
#pragma unroll
          for (int j = 0; j < HH; ++j) l[j] *= m->alpha[h0 + j];
          // rescale O once the previous tile's output MMAs are done
          const int tp = t - 1;
          fail = fail ||
                 !mbar_wait(&b_Pempty[tp & 1], (uint32_t)(tp >> 1) & 1u, abort, a.limit_ns);
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
      // (k/8) lbo_p + 128 j + (k%8) 16; a thread writes its token's HH heads as NHB 16-byte
      // rows.  lbo_p = 16 N2 + 32 puts the eight rows of each 8-lane phase in distinct banks.
      fail = fail || !mbar_wait(&b_Pempty[sb], ((uint32_t)(t >> 1) & 1u) ^ 1u, abort, a.limit_ns);
      {
        const float wr = s_r * inv_srun;
        uint8_t* prow = p_s + sb * P.p_bytes + (kslot >> 3) * P.lbo_p + (kslot & 7) * 16 +
                        128 * (h0 >> 3);
#pragma unroll
        for (int b8 = 0; b8 < NHB; ++b8) {
          float e[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int j = 8 * b8 + k;
            // a head whose reference is still -inf has only -inf scores so far (any finite
            // score takes the slow path), so a finite stand-in gives 2^-inf = 0 without NaN
            const float m0 = (mr[j] == -INFINITY) ? 0.f : mr[j];
            e[k] = ex2_approx(x[j] - m0);
            l[j] += e[k];
          }
          uint4 o;
          o.x = h2_bits(__floats2half2_rn(e[0] * wr, e[1] * wr));
          o.y = h2_bits(__floats2half2_rn(e[2] * wr, e[3] * wr));
          o.z = h2_bits(__floats2half2_rn(e[4] * wr, e[5] * wr));
          o.w = h2_bits(__floats2half2_rn(e[6] * wr, e[7] * wr));
          *reinterpret_cast<uint4*>(prow + 128 * b8) = o;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && !fail) mbar_arrive(&b_Pfull[sb]);
      ++pt;

      if (c.last) {
        // -------- epilogue of the piece: partials to the workspace slot blockIdx.x + seq
        fail = fail || !mbar_wait(&b_Pempty[sb], (uint32_t)(t >> 1) & 1u, abort, a.limit_ns);
        tc_fence_after();
#pragma unroll
        for (int j = 0; j < HH; ++j) {
          float v = l[j];
          v += __shfl_xor_sync(0xffffffffu, v, 1);
          v += __shfl_xor_sync(0xffffffffu, v, 2);
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          v += __shfl_xor_sync(0xffffffffu, v, 8);
          if (u == 0) m->red[q][h0 + j] = v;
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
        if (lane == 0 && !fail) mbar_arrive(b_oempty);
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

// sg: fp16 scales per token (group > 0: a group-scaled cache, scales applied in conversion)
Plan make_plan(int d, int d_rope, int b, int H, int batch, int group, int sg) {
  Plan pl;
  memset(&pl, 0, sizeof(pl));
  TcParams& P = pl.p;
  const int n = d + d_rope;
  const bool in_place = (b == 16 || b == KVK_BITS_BF16);
  // group scales are applied while the packed codes are unpacked (b < 16): 16-bit codes
  // converted in place, and uncompressed rows, take the CUDA-core kernel in such a layout
  if (group && in_place) return pl;
  // exact scores from high and low parts: 16-bit codes and group-scaled caches
  const bool stacked = (b == 16) || group;
  P.stacked = stacked ? 1 : 0;
  P.N1 = tc_query_rows(H);
  P.N2 = (H + 15) / 16 * 16;
  P.NP = (n + 127) / 128;
  P.NPd = (d + 127) / 128;
  P.NQA = (n + 63) / 64;
  P.NK16 = (n + 15) / 16;
  // TMEM: S^T (N2 <= 64 columns), two C^T buffers of 4 x 32 columns, O^T NPd x N2 columns
  if (H < 1 || P.N2 > 64 || P.NPd > 4 || kOCol0 + (uint32_t)(P.NPd * P.N2) > kTmemCols) return pl;
  if (P.NQA * 8 > 16 * kQL) return pl;   // staged query rows of up to 768 features
  if (d % 64) return pl;                  // latent query atoms copied whole by TMA
  const size_t q_bytes = (size_t)P.NQA * P.N1 * 128;
  P.lbo_p = (uint32_t)P.N2 * 16u + 32u;
  P.p_bytes = 8u * P.lbo_p;
  const size_t p_bytes = 2 * (size_t)P.p_bytes;
  const size_t misc_bytes = sizeof(Misc) + sizeof(int32_t) * (size_t)(batch + 1);
  P.atom_bytes = stacked ? 2u * kAtom : (uint32_t)kAtom;
  P.slot_bytes = 2u * P.atom_bytes;
  P.rbs = stacked ? 2u * kLoOff : kLoOff;
  const int raw_slot = in_place ? 0 : 64 * 16 * b;
  P.raw_slot = raw_slot;
  P.grouped = group ? 1 : 0;
  // a tile's scale window: 64 tokens x sg scales from a 16-byte boundary, rounded up to 16
  P.sc_bytes = (b == KVK_BITS_BF16) ? 0u : (uint32_t)align_up((size_t)64 * sg * 2 + 16, 16);
  const size_t sc_ring = align_up((size_t)kScSlots * P.sc_bytes, 1024);
  // try the largest rings that fit
  const size_t fixed = align_up(q_bytes, 1024) + align_up(p_bytes, 1024) + sc_ring;
  auto total_for = [&](int PR, int RR) {
    size_t off = fixed;
    off += (size_t)PR * P.slot_bytes;
    off = align_up(off + (size_t)RR * raw_slot, 1024);
    off = align_up(off + (size_t)(3 * PR + 2 * RR + kFixedBars) * 8, 16);
    off += misc_bytes;
    return off + 1024;   // runtime alignment slack of the dynamic shared memory base
  };
  int PR = 0, RR = 0;
  if (in_place) {
    // the TMA lands in the f16 slots: at least a tile's groups
    for (PR = 3 * P.NP; PR >= P.NP; --PR)
      if (total_for(PR, 0) <= (size_t)kSmemLimit) break;
    if (PR < P.NP) return pl;
  } else {
    // packed codes land in the raw ring; the f16 slots only span conversion to score MMA, so
    // fewer than a tile's groups still flow (a group's slot is that of the group PR earlier,
    // released by its score MMAs, which never wait for a later group)
    const int want = P.NP + (P.NP + 1) / 2;
    bool fit = false;
    for (PR = want; PR >= 2 && !fit; --PR) {
      for (RR = 4 * P.NP; RR >= 2; --RR)
        if (total_for(PR, RR) <= (size_t)kSmemLimit) {
          fit = true;
          break;
        }
      if (fit) break;
    }
    if (!fit) return pl;
  }
  P.PR = PR;
  P.RR = RR;
  size_t off = fixed;
  P.off_p = (uint32_t)align_up(q_bytes, 1024);
  P.off_sc = P.off_p + (uint32_t)align_up(p_bytes, 1024);
  P.off_pairs = (uint32_t)fixed;
  off += (size_t)PR * P.slot_bytes;
  P.off_raw = (uint32_t)off;
  off = align_up(off + (size_t)RR * raw_slot, 1024);
  P.off_bar = (uint32_t)off;
  off = align_up(off + (size_t)(3 * PR + 2 * RR + kFixedBars) * 8, 16);
  P.off_misc = (uint32_t)off;
  pl.smem = off + misc_bytes + 1024;
  // score MMA: M = 64 tokens x N1 heads, or stacked M = 128 (high and low rows) x N2 heads
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

struct Maps {
  const CUtensorMap& codes;
  const CUtensorMap& ql;
  const CUtensorMap& qr;
};

template <int BITS, int NH>
cudaError_t launch_bits_nh(const TcParams& P, const Maps& mp, size_t smem, int grid,
                           cudaStream_t st) {
  auto k = decode_tc_kernel<BITS, NH>;
  if (instance_regs<BITS, NH>() != (int)kLaunchRegs) return cudaErrorNotSupported;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(k, dim3(grid), dim3(kThreads), smem, st, P, mp.codes, mp.ql, mp.qr);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int BITS>
cudaError_t launch_bits(const TcParams& P, const Maps& mp, size_t smem, int grid,
                        cudaStream_t st) {
  switch (P.N2) {
    case 16: return launch_bits_nh<BITS, 16>(P, mp, smem, grid, st);
    case 32: return launch_bits_nh<BITS, 32>(P, mp, smem, grid, st);
    case 48: return launch_bits_nh<BITS, 48>(P, mp, smem, grid, st);
    case 64: return launch_bits_nh<BITS, 64>(P, mp, smem, grid, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool tc_supported(const kvk_layout* L, const AnchorDesc& A, int dtype, int H) {
  if (dtype != KVK_BF16 && dtype != KVK_F16) return false;
  if (!A.tmap_ok) return false;
  const Plan pl = make_plan(A.d, L->d_rope, A.b, H, L->max_batch, anchor_group(L, A), A.sg);
  return pl.ok && launch_regs_ok(A.b, pl.p.N2);
}

cudaError_t launch_decode_tc(const DecodeArgs& a, const CUtensorMap& tmap, const CUtensorMap& qmap_l,
                             const CUtensorMap& qmap_r, int dtype, cudaStream_t st) {
  Plan pl = make_plan(a.d, a.d_rope, a.b, a.H, a.batch, a.group, a.sg);
  if (!pl.ok) return cudaErrorInvalidValue;
  pl.p.a = a;
  pl.p.qdtype = dtype;
  const Maps mp{tmap, qmap_l, qmap_r};
  switch (a.b) {
    case 16: return launch_bits<16>(pl.p, mp, pl.smem, a.G, st);
    case KVK_BITS_BF16: return launch_bits<KVK_BITS_BF16>(pl.p, mp, pl.smem, a.G, st);
    case 8: return launch_bits<8>(pl.p, mp, pl.smem, a.G, st);
    case 4: return launch_bits<4>(pl.p, mp, pl.smem, a.G, st);
    case 2: return launch_bits<2>(pl.p, mp, pl.smem, a.G, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace kvk
