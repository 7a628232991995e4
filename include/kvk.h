/*
 * kvk.h -- C ABI of libkvk, the B200 (sm_100a) library for the KV-Kaizen compressed
 * MLA KV cache: quantise-on-write of each anchor layer's cache and the decode-step
 * attention that reads the packed cache back.
 *
 * Source of the method: "KV-Kaizen: Learning Context-Adaptive Cache Compression Choices"
 * (whiteboard summary on picx.dev), sections "Three Non-Eviction Compression Axes"
 * (depth / rank / precision) and "Action Space and Cost Model".
 *
 * Conventions shared by every entry point
 *   - Plain pointers and sizes only.  "dev_" pointers are CUDA device pointers; every
 *     other pointer is host memory.  The caller owns all device memory (arena, inputs,
 *     outputs, workspace); a layout owns only its host-side metadata.
 *   - Argument and table checks are synchronous and happen before any launch; a failed
 *     check returns its status and launches nothing.  Launches are asynchronous on the
 *     given stream (a cudaStream_t; NULL is the legacy default stream).  A launch error
 *     returns KVK_ERR_CUDA.
 *   - Device-side conditions that the host cannot see (positions and lengths held in
 *     device memory, non-finite inputs) never fault: the kernel skips or clamps the
 *     offending item and sets a sticky flag, read with kvk_read_status().
 *   - Every device pointer must be 16-byte aligned (the arena: 256-byte aligned), or the
 *     call returns KVK_ERR_ALIGNMENT.
 *   - A layout belongs to the device that was current when it was created with an arena.
 *     Every call that launches work (writes, decodes, kvk_read_status) must be made with
 *     that device current; otherwise it returns KVK_ERR_INVALID_ARG and launches nothing.
 *   - Nothing here allocates device memory except kvk_create_layout's one synchronous
 *     cudaMemset of the arena header; nothing falls back to the CPU.
 */
#ifndef KVK_H_
#define KVK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* kvk_stream_t;

/* Opaque host-side handle: per-layer table, anchor map, arena offsets, TMA descriptors. */
typedef struct kvk_layout kvk_layout;

typedef enum {
    KVK_OK = 0,
    KVK_ERR_INVALID_ARG = 1,      /* null / out-of-range argument, or a layout without arena */
    KVK_ERR_BAD_TABLE = 2,        /* anchor / d / b table violates the action space          */
    KVK_ERR_BUDGET = 3,           /* plan's bits per token exceed the given budget            */
    KVK_ERR_INHERITING_LAYER = 4, /* quant-write addressed a layer that inherits its cache    */
    KVK_ERR_WORKSPACE = 5,        /* arena or workspace smaller than required                 */
    KVK_ERR_ALIGNMENT = 6,        /* device pointer or stride not aligned as required         */
    KVK_ERR_CUDA = 7,             /* a CUDA runtime / driver call or a launch failed          */
    KVK_ERR_UNSUPPORTED = 8       /* shape outside what the compiled kernels handle           */
} kvk_status;

typedef enum { KVK_F32 = 0, KVK_BF16 = 1, KVK_F16 = 2 } kvk_dtype;

/* Sticky device flags (kvk_read_status). */
#define KVK_FLAG_NONFINITE   0x1u /* quant-write: non-finite input, or scale above the fp16 range */
#define KVK_FLAG_WRITE_RANGE 0x2u /* quant-write: position outside [0, max_tokens); token skipped  */
#define KVK_FLAG_SEQ_LEN     0x4u /* decode: seq_len outside [0, max_tokens], clamped; or keep_len
                                     outside [0, keep_stride], clamped                             */
#define KVK_FLAG_KEEP_INDEX  0x8u /* decode: keep index outside [0, seq_len); entry skipped        */
#define KVK_FLAG_TIMEOUT     0x10u /* decode: a tensor-core kernel wait exceeded its time limit and
                                      the kernel stopped early; that call's outputs are unspecified */

/* Bit width of an anchor that keeps its cache uncompressed: rows of bfloat16 values (16 bits
 * per element, no quantisation and no scale) -- the bf16 MLA cache the compressed choices are
 * measured against.  Such an anchor costs (d + d_rope) * 16 bits per token. */
#define KVK_BITS_BF16 0

/* Decode kernel selection (kvk_set_decode_path). */
#define KVK_PATH_AUTO      0 /* tensor-core kernel where it applies, else the CUDA-core kernel  */
#define KVK_PATH_TENSOR    1 /* tcgen05 kernel only (KVK_ERR_UNSUPPORTED where it cannot run)   */
#define KVK_PATH_CUDA_CORE 2 /* FFMA kernel (any shape, any dtype)                                */
/* The general tcgen05 kernel (the one bf16 rows and group-scaled codes take) also where the
 * token-scale kernel would run (codes with one scale per token): a second tensor-core
 * implementation of those widths to check against; KVK_ERR_UNSUPPORTED where it cannot run. */
#define KVK_PATH_TENSOR_GENERAL 3

/*
 * kvk_create_layout -- validate a per-layer plan and lay out its cache in an arena.
 *
 * Defines: the depth axis (a layer either is an anchor with its own cache or inherits the
 * nearest anchor before it), the rank axis (an anchor keeps the first d of r latent
 * coordinates plus the d_rope-wide RoPE key) and the precision axis (b-bit symmetric
 * codes, one scale per token) -- "Three Non-Eviction Compression Axes"; and the budget
 * check of "Action Space and Cost Model" with the fp16 scale counted:
 *     bits_per_token = sum over anchors l of ((d_l + d_rope) * b_l + 16)
 * (an uncompressed bf16 anchor counts (d_l + d_rope) * 16).
 *
 *   n_layers            L >= 1
 *   anchor[L]           anchor[l] == l for an anchor; otherwise the largest l' < l with
 *                       anchor[l'] == l' (the nearest preceding anchor).  anchor[0] == 0.
 *   d[L], b[L]          for anchors: 16 <= d <= r, d % 16 == 0; b in {2, 4, 8, 16}, or
 *                       KVK_BITS_BF16 (0) for an uncompressed bf16 anchor.  Ignored for
 *                       inheriting layers.
 *   r, d_rope           latent width (multiple of 16) and RoPE width (multiple of 8, >= 0)
 *   max_batch, max_tokens  capacity of every anchor's cache (max_batch <= 4096,
 *                       max_batch * max_tokens < 2^31)
 *   budget_bits_per_token  <= 0: no check; else KVK_ERR_BUDGET when the plan costs more
 *   dev_arena, arena_bytes caller-owned device memory (256-byte aligned), size >= needed
 *   out                 receives the handle; NULL = query only (sizes and bits filled in)
 *   arena_bytes_needed, bits_per_token  optional outputs (may be NULL)
 *
 * With out != NULL and dev_arena == NULL a planning-only layout is returned: its offsets
 * can be inspected (kvk_get_layer_info) but it cannot write or decode.  With an arena, the
 * arena header (status flags) is zeroed by one synchronous cudaMemset.
 * Arena layout: 256-byte header, then per anchor (in layer order) a codes plane
 * [max_batch][max_tokens][row_bytes] and an fp16 scale plane [max_batch][max_tokens],
 * each 256-byte aligned, and 256 bytes of tail slack (read, never written, by the decode).
 * row_bytes = ceil((d + d_rope) * b / 8) rounded up to 16.
 * Packed row format: field u_i = code_i + 2^(b-1) (offset binary) at bit i*b of the row
 * read as a little-endian bit stream, i over [c[0..d) || k^R[0..d_rope)], zero padding.
 * An uncompressed anchor (b = KVK_BITS_BF16) stores element i as the bfloat16 of v_i
 * (round to nearest even) at bytes 2i, 2i+1 of the row, row_bytes = 2 (d + d_rope) rounded up
 * to 16, and its scale plane holds 1.0 for every written token.
 */
kvk_status kvk_create_layout(int n_layers, const int32_t* anchor, const int32_t* d,
                             const int32_t* b, int r, int d_rope, int max_batch, int max_tokens,
                             int64_t budget_bits_per_token, void* dev_arena, size_t arena_bytes,
                             kvk_layout** out, size_t* arena_bytes_needed,
                             int64_t* bits_per_token);

/*
 * kvk_create_layout_grouped -- kvk_create_layout with one fp16 scale per group of
 * `scale_group` consecutive elements of each quantised anchor's row instead of one per token:
 * the group-scale comparison point of the precision axis (a 4-bit cache with a scale per 32
 * elements costs 4.5 bits per element, the figure behind the 152x composition of "Hardware
 * Benchmarking (Apple M3 Ultra)"; KIVI-style grouping in "Main Results / Table 2").
 *
 *   scale_group  G in {16, 32, 64}; every quantised anchor needs (d + d_rope) % G == 0
 *                (else KVK_ERR_BAD_TABLE); uncompressed anchors keep one unit scale per token
 *   other arguments as kvk_create_layout, and
 *     bits_per_token = sum over quantised anchors of ((d + d_rope) * b + 16 * (d + d_rope) / G)
 *                      (+ (d + d_rope) * 16 for uncompressed anchors).
 * Scale plane of such an anchor: [max_batch][max_tokens][(d + d_rope) / G] fp16, scale j of a
 * token covering elements [j G, (j + 1) G).  Each group is quantised as kvk_quant_write
 * quantises a token (its own absmax, scale rounded up, round-half-even codes), and decode
 * dequantises each element with its group's scale.  Every other entry point takes such a
 * layout unchanged.
 */
kvk_status kvk_create_layout_grouped(int n_layers, const int32_t* anchor, const int32_t* d,
                                     const int32_t* b, int r, int d_rope, int scale_group,
                                     int max_batch, int max_tokens,
                                     int64_t budget_bits_per_token, void* dev_arena,
                                     size_t arena_bytes, kvk_layout** out,
                                     size_t* arena_bytes_needed, int64_t* bits_per_token);

/* Frees the host-side handle only (never the arena).  NULL is ignored. */
void kvk_destroy(kvk_layout* layout);

/* Where a layer's cache lives.  For an inheriting layer this describes its anchor's cache
 * (the depth axis: the cache is never duplicated).  codes / scales are device pointers
 * into the arena (offsets from 0 for a planning-only layout). */
typedef struct {
    int32_t anchor;         /* anchor layer whose cache this layer reads                  */
    int32_t d;              /* latent coordinates kept by that anchor                      */
    int32_t b;              /* bits per stored element                                     */
    int32_t row_bytes;      /* bytes of one packed token row                               */
    void* codes;            /* [max_batch][max_tokens][row_bytes] uint8                    */
    void* scales;           /* [max_batch][max_tokens] fp16                                */
    int64_t codes_offset;   /* byte offsets of the two planes inside the arena             */
    int64_t scales_offset;
    int32_t max_batch;
    int32_t max_tokens;
    int32_t r;
    int32_t d_rope;
    int32_t scales_per_token; /* fp16 scales per token in the scale plane (1, or (d+d_rope)/G) */
    int32_t scale_group;      /* elements per scale G of a group-scaled anchor, 0: per token    */
} kvk_layer_info;

kvk_status kvk_get_layer_info(const kvk_layout* layout, int layer, kvk_layer_info* info);

/*
 * kvk_quant_write -- quantise and store new tokens of one anchor layer (prefill or append).
 *
 * Defines the precision axis ("one scale per token", symmetric uniform, b bits) applied to
 * the rank-truncated MLA vector v = [c_kv[0..d) || k_rope[0..d_rope)] of each token:
 *     A = max_i |v_i| (fp32);  s32 = A / (2^(b-1) - 1) (IEEE fp32 division);
 *     s = fp16(s32) rounded toward +inf, stored in the scale plane;
 *     code_i = clamp(round_half_even(v_i / s), -(2^(b-1)-1), 2^(b-1)-1) with the stored
 *     scale (IEEE fp32 division); s == 0 gives all-zero codes.
 * An uncompressed anchor (KVK_BITS_BF16) stores bf16(v_i) instead, and the scale 1.0.
 * Token j (0 <= j < n_new) of sequence i (0 <= i < batch) goes to position
 * dev_start_pos[i] + j of sequence i's cache.
 *
 *   layer        an anchor layer (an inheriting layer -> KVK_ERR_INHERITING_LAYER)
 *   c_kv         device, element (i, j, k) at c_kv[i*c_stride_seq + j*c_stride_tok + k],
 *                k < d read (features contiguous); dtype KVK_F32 or KVK_BF16
 *   k_rope       device, element (i, j, k) at k_rope[i*kr_stride_seq + j*kr_stride_tok + k],
 *                k < d_rope; same dtype.  Strides in elements, multiples of 8 (16 B).
 *   batch        1 <= batch <= max_batch;  n_new >= 0 (0: nothing launched)
 *   dev_start_pos  device int32 [batch]; a position outside [0, max_tokens) skips the token
 *                and sets KVK_FLAG_WRITE_RANGE; non-finite input or a scale beyond the
 *                fp16 range sets KVK_FLAG_NONFINITE (the stored token is then unspecified).
 */
kvk_status kvk_quant_write(kvk_layout* layout, int layer, const void* c_kv, int dtype,
                           int64_t c_stride_seq, int64_t c_stride_tok, const void* k_rope,
                           int64_t kr_stride_seq, int64_t kr_stride_tok, int batch,
                           const int32_t* dev_start_pos, int n_new, kvk_stream_t stream);

/*
 * kvk_quant_write_layers -- the same write for n distinct anchor layers in one launch (for
 * example one decode step's append to every anchor), all with the same dtype, batch,
 * dev_start_pos and n_new.  Layer layers[k] takes c_kv[k] / k_rope[k] with strides
 * c_stride_seq[k], c_stride_tok[k], kr_stride_seq[k], kr_stride_tok[k] (host arrays of n
 * entries, device tensors as in kvk_quant_write).  The result is the one n separate
 * kvk_quant_write calls would produce.  1 <= n <= KVK_MAX_WRITE_LAYERS; every argument of
 * every layer is checked before anything is launched, with kvk_quant_write's statuses, and a
 * repeated layer is KVK_ERR_INVALID_ARG.
 */
#define KVK_MAX_WRITE_LAYERS 64
kvk_status kvk_quant_write_layers(kvk_layout* layout, int n, const int32_t* layers,
                                  const void* const* c_kv, int dtype,
                                  const int64_t* c_stride_seq, const int64_t* c_stride_tok,
                                  const void* const* k_rope, const int64_t* kr_stride_seq,
                                  const int64_t* kr_stride_tok, int batch,
                                  const int32_t* dev_start_pos, int n_new, kvk_stream_t stream);

/* Bytes of device workspace kvk_mla_decode needs for (layer, batch, n_heads), covering
 * both decode kernels. */
kvk_status kvk_decode_workspace_bytes(const kvk_layout* layout, int layer, int batch,
                                      int n_heads, size_t* bytes);

/* Bytes of device workspace for a call with a keep list of row stride keep_stride to take
 * the tensor-core kernel: the bytes above plus a dense copy of the kept rows
 * (batch * keep_stride * row_bytes of the layer's anchor) and their scales.  With less, such
 * a call takes the CUDA-core kernel (or returns KVK_ERR_WORKSPACE when the tensor-core
 * kernel is forced).  keep_stride < 0 is KVK_ERR_INVALID_ARG. */
kvk_status kvk_decode_workspace_bytes_keep(const kvk_layout* layout, int layer, int batch,
                                           int n_heads, int keep_stride, size_t* bytes);

/*
 * kvk_mla_decode -- one decode step of attention for one layer over its anchor's cache.
 *
 * Defines decode attention over the compressed cache ("every decoded token reads the
 * entire KV cache", Background; the absorbed MLA form): with a = anchor(layer), d = d_a,
 * c_hat_t = code_t * s_t the dequantised row of token t,
 *     z_{h,t} = softmax_scale * (q_lat[h, 0..d) . c_hat_t[0..d) + q_rope[h] . c_hat_t[d..d+d_rope))
 *     out[h]  = sum_t softmax_t(z_{h,.}) * c_hat_t[0..d),   lse[h] = log sum_t exp(z_{h,t})
 * over t in 0..seq_len-1, or over the keep list when one is given (composition with token
 * eviction).  An empty token set gives out = 0 and lse = -inf.
 *
 *   layer        any layer; an inheriting layer reads its anchor's cache (no copy)
 *   q_lat        device [batch][n_heads][>= d] at q_lat[i*q_lat_stride_seq + h*q_lat_stride_head + k]
 *   q_rope       device [batch][n_heads][d_rope], strides likewise (elements, multiples of 8)
 *   dtype        KVK_BF16 / KVK_F16 (tensor-core kernel eligible) or KVK_F32 (CUDA-core kernel)
 *   batch        1 <= batch <= max_batch;  n_heads >= 1
 *   dev_seq_lens device int32 [batch], clamped to [0, max_tokens] (KVK_FLAG_SEQ_LEN)
 *   dev_keep_idx nullable device int32 [batch][keep_stride]: ascending, unique token indices;
 *                entries >= seq_len or < 0 are skipped (KVK_FLAG_KEEP_INDEX)
 *   dev_keep_len device int32 [batch], required iff dev_keep_idx; clamped to [0, keep_stride]
 *   softmax_scale  sigma above
 *   out          device fp32 [batch][n_heads][d], written completely
 *   lse          nullable device fp32 [batch][n_heads] (natural log)
 *   workspace    device, >= kvk_decode_workspace_bytes(); contents are scratch.  With a
 *                keep list and at least kvk_decode_workspace_bytes_keep() bytes, the kept
 *                rows are first copied densely into the workspace (one extra launch) and the
 *                tensor-core kernel reads that copy; otherwise the CUDA-core kernel gathers
 *                them itself.
 */
kvk_status kvk_mla_decode(kvk_layout* layout, int layer, const void* q_lat, const void* q_rope,
                          int dtype, int64_t q_lat_stride_seq, int64_t q_lat_stride_head,
                          int64_t q_rope_stride_seq, int64_t q_rope_stride_head, int batch,
                          int n_heads, const int32_t* dev_seq_lens, const int32_t* dev_keep_idx,
                          const int32_t* dev_keep_len, int keep_stride, float softmax_scale,
                          float* out, float* lse, void* workspace, size_t workspace_bytes,
                          kvk_stream_t stream);

/*
 * kvk_mla_decode_append -- one decode step of an anchor layer with its new token: quantise
 * and store the token, then decode over the cache that includes it, in one launch where the
 * tensor-core kernel runs ("Three Non-Eviction Compression Axes", item 3, applied to the
 * token a decode step appends, followed by the decode of kvk_mla_decode).
 *
 * The result is the one of kvk_quant_write (n_new = 1, dev_start_pos[i] = seq_len_i - 1)
 * followed by kvk_mla_decode over seq_len_i tokens: dev_seq_lens counts the new token.  In
 * the tensor-core kernel the CTA that owns position seq_len_i - 1 writes the token before
 * it loads that position; the CUDA-core kernel (fp32 queries, shapes the tensor-core kernel
 * does not take) gets the write as a separate launch first.
 *
 *   layer        an anchor layer (an inheriting layer -> KVK_ERR_INHERITING_LAYER: its
 *                anchor's step writes the token)
 *   c_new        device [batch][>= d] at c_new[i * c_new_stride_seq + k]; dtype new_dtype
 *                (KVK_BF16 or KVK_F32); k_rope_new [batch][d_rope] likewise.  Strides in
 *                elements, multiples of 8.
 *   dev_seq_lens clamped to [0, max_tokens] as in kvk_mla_decode; a sequence of length 0
 *                appends nothing
 *   the query, output and workspace arguments are those of kvk_mla_decode (no keep list:
 *   with token eviction write with kvk_quant_write and decode with kvk_mla_decode).
 */
kvk_status kvk_mla_decode_append(kvk_layout* layout, int layer, const void* c_new,
                                 const void* k_rope_new, int new_dtype, int64_t c_new_stride_seq,
                                 int64_t k_rope_new_stride_seq, const void* q_lat,
                                 const void* q_rope, int dtype, int64_t q_lat_stride_seq,
                                 int64_t q_lat_stride_head, int64_t q_rope_stride_seq,
                                 int64_t q_rope_stride_head, int batch, int n_heads,
                                 const int32_t* dev_seq_lens, float softmax_scale, float* out,
                                 float* lse, void* workspace, size_t workspace_bytes,
                                 kvk_stream_t stream);

/*
 * kvk_mla_decode_noalloc -- kvk_mla_decode without a caller-provided workspace.
 *
 * The paper has no counterpart to this entry point; it exists for callers that cannot
 * allocate device memory for the workspace: for example a host application that reserves
 * the whole device memory budget up front and hands plugins only fixed buffers, or a
 * latency-critical loop where an allocation (and the synchronisation it may bring) is not
 * acceptable.  Such a caller still passes its inputs and outputs; the scratch space comes
 * from a file-scope __device__ array of KVK_NOALLOC_SCRATCH_BYTES bytes inside libkvk,
 * which every GPU that loads the library holds until the process exits.
 *
 * Arguments and results are those of kvk_mla_decode minus (workspace, workspace_bytes).
 * The call takes the kernel kvk_mla_decode would take (kvk_decode_path_for) and needs, for
 * that kernel, the workspace kvk_mla_decode needs; when that exceeds
 * KVK_NOALLOC_SCRATCH_BYTES it returns KVK_ERR_WORKSPACE and launches nothing.  (The
 * tensor-core kernel needs (G + batch) * n_heads * (d + 2) * 4 bytes plus a little, G the
 * SM count; kvk_decode_workspace_bytes, which covers both kernels, can be larger.)  A call
 * with a keep list takes the tensor-core kernel only if the scratch also holds the dense
 * copy of the kept rows, else the CUDA-core kernel.  This entry point allocates nothing: no
 * cudaMalloc, no cudaFree, no allocating library routine.
 *
 * Set-up: the first call on a device (the layout's device, which must be current) looks
 * up the array's device address with cudaGetSymbolAddress and caches it per device; make
 * that first call before any stream capture.  The cached address is that of the library's
 * module in the device's primary context: after cudaDeviceReset it is stale, and calls
 * made after a reset are unsupported.  All calls share the one array and it keeps the
 * previous call's contents (no part of it needs to start at zero), so calls whose
 * executions overlap on the GPU -- on different streams, or from different host threads --
 * race on it and give undefined results; order them on one stream or serialise them.
 */
#define KVK_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

kvk_status kvk_mla_decode_noalloc(kvk_layout* layout, int layer, const void* q_lat,
                                  const void* q_rope, int dtype, int64_t q_lat_stride_seq,
                                  int64_t q_lat_stride_head, int64_t q_rope_stride_seq,
                                  int64_t q_rope_stride_head, int batch, int n_heads,
                                  const int32_t* dev_seq_lens, const int32_t* dev_keep_idx,
                                  const int32_t* dev_keep_len, int keep_stride,
                                  float softmax_scale, float* out, float* lse,
                                  kvk_stream_t stream);

/*
 * kvk_absorb -- the absorbed MLA projections on either side of the decode, on the tensor
 * cores ("Three Non-Eviction Compression Axes", item 2: only the first d latent coordinates
 * a layer keeps are produced or consumed):
 *     y[b][h][j] = sum_{k < K} x[b][h][k] * w[h][k][j]      for b < batch, h < n_heads, j < n
 * Query side: x = q_nope (bf16, K = the head dim), w = W_UK restricted to its first d columns,
 * y = q_lat (bf16, n = d) for kvk_mla_decode.  Output side: x = the decode output (fp32, K = d),
 * w = W_UV restricted to its first d rows, y = the heads' values (fp32, n = the value dim).
 *
 *   x       device, x_dtype KVK_BF16 or KVK_F32, element (b, h, k) at
 *           x[b * x_stride_seq + h * x_stride_head + k]; an fp32 x enters the tensor cores
 *           as two bf16 parts (hi = bf16(x), lo = bf16(x - hi)), about 16 significant bits
 *   w       device bf16, element (h, k, j) at w[h * w_stride_head + k * w_stride_row + j]
 *           (w_stride_row >= n, w_stride_head >= K * w_stride_row)
 *   y       device, y_dtype KVK_BF16 (rounded to nearest even) or KVK_F32, element (b, h, j) at
 *           y[b * y_stride_seq + h * y_stride_head + j]; written completely
 *   K       64 <= K <= 512, K % 64 == 0;  n >= 16, n % 16 == 0;  1 <= n_heads <= 65535
 *   All strides are in elements and multiples of 8; pointers 16-byte aligned
 *   (KVK_ERR_ALIGNMENT otherwise).  Accumulation is fp32.  No layout is involved; a wait that
 *   runs out (2 s) leaves y unspecified.
 */
kvk_status kvk_absorb(const void* x, int x_dtype, int64_t x_stride_seq, int64_t x_stride_head,
                      const void* w, int64_t w_stride_row, int64_t w_stride_head, void* y,
                      int y_dtype, int64_t y_stride_seq, int64_t y_stride_head, int batch,
                      int n_heads, int K, int n, kvk_stream_t stream);

/* Copy the sticky device flags to *flags (synchronises the stream); clear != 0 resets them
 * to zero afterwards. */
kvk_status kvk_read_status(kvk_layout* layout, uint32_t* flags, int clear, kvk_stream_t stream);

/* Decode kernel choice (KVK_PATH_*) and the number of CTAs the decode splits the tokens
 * over (0 = automatic).  Both only steer the schedule: results stay within tolerance of
 * the same definition. */
kvk_status kvk_set_decode_path(kvk_layout* layout, int path);
kvk_status kvk_set_decode_ctas(kvk_layout* layout, int ctas);

/* Failure detection of the tensor-core decode: every wait inside the kernel (for a tile to
 * land, for a stage of the pipeline to finish) gives up after `ns` nanoseconds; the kernel
 * then sets KVK_FLAG_TIMEOUT, lets its own loads and tensor-core operations finish, and
 * exits, so the stream and the context stay usable and the call's outputs are unspecified.
 * ns = 0 restores the default limit of 2 s.  A short limit (microseconds) makes a wait run
 * out on purpose, to exercise that path. */
kvk_status kvk_set_wait_limit(kvk_layout* layout, uint64_t ns);

/* Which kernel kvk_mla_decode would run for these arguments (KVK_PATH_TENSOR or
 * KVK_PATH_CUDA_CORE), without launching anything.  has_keep != 0: a keep list is given;
 * it does not change the answer, but a keep-list call takes the tensor-core kernel only with
 * a workspace of kvk_decode_workspace_bytes_keep() bytes (else the CUDA-core kernel). */
kvk_status kvk_decode_path_for(const kvk_layout* layout, int layer, int dtype, int n_heads,
                               int has_keep, int* path);

/* Static description of a status code. */
const char* kvk_status_string(kvk_status status);

#ifdef __cplusplus
}
#endif
#endif /* KVK_H_ */
