/*
 * mla.h -- C ABI of libmla: absorbed Multi-head Latent Attention decode over a
 * paged latent KV cache, for NVIDIA B200 (sm_100a).
 *
 * Sources of the operations:
 *   [T27] Day 27 tutorial "Multi-Head Latent Attention: How DeepSeek Compressed
 *         the Cache Further" (kgptalkie), sections named per call below.
 *   [RK]  "RedKnot-MLA: Multi-Head Offline-Online Reuse for DeepSeek-V4
 *         Long-Context Serving", abstract.
 *
 * Conventions shared by every call
 *   - Every pointer is a DEVICE pointer owned by the caller unless a comment
 *     says "host".  The library never allocates device memory and keeps no
 *     state between calls except cached per-device properties and TMA
 *     descriptors (mla_decode_static_ws adds one fixed static scratch
 *     array).  Buffers must not alias unless a call says so.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream) and returns an mla_status_t synchronously.
 *     Argument errors are reported before anything is launched and leave the
 *     outputs untouched.  MLA_ERR_CUDA reports a failed launch.
 *   - Errors found by a kernel while it runs (a page id out of range, a row
 *     outside every segment) are written to a device status word; the
 *     offending work item is skipped (its outputs are set to NaN), the kernel
 *     never traps.  mla_get_status() reads and clears that word.
 *   - Storage types: dims.dtype == MLA_BF16 means q_nope, q_rope, q_abs, the
 *     cache, W_UK, W_UV and W_O hold bfloat16; MLA_F32 means they hold float.
 *     Accumulation is always fp32; o_lat, lse, v and out are always float.
 *   - Layouts are dense row-major in the index order written in brackets.
 *   - No C++ exception crosses this interface.
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MLA_ABI_VERSION 1

/* A cudaStream_t, declared without including the CUDA headers. */
typedef struct CUstream_st* mla_stream_t;

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned buffer       */
  MLA_ERR_UNSUPPORTED = 2,  /* valid arguments with no kernel for them          */
  MLA_ERR_WORKSPACE = 3,    /* workspace smaller than mla_decode_workspace_size */
  MLA_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed             */
  MLA_ERR_TIMEOUT = 5,      /* a bounded device-side wait gave up               */
  MLA_ERR_BAD_INDEX = 6     /* a kernel met a page id / row / segment out of range */
} mla_status_t;

typedef enum { MLA_F32 = 0, MLA_BF16 = 1 } mla_dtype_t;

/* Model dimensions of one attention layer.
 *   H          query heads
 *   d_c        width of the shared content latent c_KV ([T27] "Learn a Smaller
 *              Shared Representation")
 *   d_r        width of the decoupled rotary key ([T27] "Position Rotations
 *              Complicate the Absorption"); even
 *   d_n, d_v   per-head no-position key width and value width
 *   d_model    output width of the shared output projection W_O
 *   page_size  cache rows per page; must be 64
 *   dtype      MLA_F32 or MLA_BF16 (storage type, see above)
 *   scale      softmax scale applied to every score (1/sqrt(d_n + d_r) is the
 *              scale of the expanded query/key width)
 *   rope_base  RoPE base: feature pair i of a vector at position p is rotated
 *              by p * rope_base^(-2i/d_r); pairs are adjacent (2i, 2i+1). */
typedef struct {
  int32_t H, d_c, d_r, d_n, d_v, d_model, page_size;
  int32_t dtype;
  float scale;
  double rope_base;
} mla_dims_t;

/* One segment of a sequence's logical row space.  Rows [row_begin, row_end)
 * hold cache rows whose request positions are key_pos_base + (r - row_begin);
 * their rotary keys were cached at (request position - delta[q_version]),
 * where delta[] are the relocation offsets given to mla_absorb_q.  A document
 * cached offline at canonical position 0 and placed at request offset P is
 * the segment {P, P + len, v, P} with delta[v] = P ([RK]: query-side RoPE
 * relocation restores the document's request position).  row_begin must be
 * a multiple of page_size; row_begin == row_end marks an unused slot. */
typedef struct {
  int32_t row_begin, row_end, q_version, key_pos_base;
} mla_seg_t;

/* ABI version of the loaded library (MLA_ABI_VERSION). */
int32_t mla_abi_version(void);

/* Static string naming a status code. */
const char* mla_status_str(mla_status_t status);

/* Waits for `stream`, then returns and clears the device status word that
 * kernels set when they skip bad work items (MLA_OK if none). */
mla_status_t mla_get_status(mla_stream_t stream);

/* ---------------------------------------------------------------------------
 * mla_absorb_q -- projection absorption plus query-side RoPE relocation.
 * [T27] "Move the Key Projection Into the Query": q . (U_K c) = (U_K^T q) . c,
 * so the newest query is transformed once per step instead of expanding every
 * cached latent.  [T27] "Position Rotations Complicate the Absorption": the
 * rotary part stays a separate term.  [RK]: the rotary query is rotated at
 * (q_pos - delta[v]) so that keys cached at shifted positions need no rewrite.
 *
 *   q_nope [n_q, H, d_n]   no-position query per head            (dtype)
 *   q_rope [n_q, H, d_r]   rotary query per head, unrotated       (dtype)
 *   q_pos  [n_q]           request position of each query token   (int32)
 *   delta  [n_ver]  HOST   relocation offsets; version v rotates the rotary
 *                          query at q_pos - delta[v]; 1 <= n_ver <= 8
 *   w_uk   [H, d_n, d_c]   W_UK[h]: c -> content key              (dtype)
 *   q_abs  [n_ver, n_q, H, d_c + d_r]  out: [W_UK[h]^T q_nope | R(q_pos -
 *                          delta[v]) q_rope], rounded to dtype
 * Angles are computed in double precision.  Errors: INVALID_ARG for null
 * pointers, n_q < 0, n_ver outside [1, 8], odd d_r. */
mla_status_t mla_absorb_q(const mla_dims_t* dims, int32_t n_q, const void* q_nope,
                          const void* q_rope, const int32_t* q_pos, const int32_t* delta,
                          int32_t n_ver, const void* w_uk, void* q_abs,
                          mla_stream_t stream);

/* ---------------------------------------------------------------------------
 * mla_decode -- absorbed attention of every query token over its sequence's
 * packed latent cache, for a list of heads.
 * [T27] "Move the Key Projection Into the Query" and "Position Rotations
 * Complicate the Absorption": score(t) = scale * (q_abs_content . c_t +
 * q_abs_rope . k_rope_t), masked where key_pos(t) > q_pos, softmaxed.
 * [T27] "Move the Value Expansion After the Weighted Sum": the output is the
 * weighted latent o_lat = sum_t a_t c_t; the value expansion happens later
 * (mla_out_proj).  Long sequences are split across SMs and the splits are
 * merged by log-sum-exp inside this call.
 *
 *   B, s_q        sequences and query tokens per sequence; query row i =
 *                 b * s_q + j
 *   q_abs         [n_ver, B*s_q, H, d_c + d_r] from mla_absorb_q (dtype)
 *   head_ids      [n_h] distinct head ids in [0, H) (int32, device), or NULL
 *                 for heads 0 .. n_h-1.  [RK]: the Local and Global heads
 *                 are sets of head ids, decoded by separate calls over the
 *                 same q_abs and cache.  An id outside [0, H) records
 *                 BAD_INDEX and that head's results are not written.
 *   n_h           heads decoded, 1 <= n_h <= H
 *   cache         [n_pages, page_size, d_c + d_r]: row = [c_KV | k_rope],
 *                 k_rope already rotated at its cache position (dtype);
 *                 256-byte aligned
 *   block_table   [B, max_pages]: page id of each page_size-row block of a
 *                 sequence's logical row space (int32)
 *   segs          [B, max_segs] (mla_seg_t): a sequence's segments, sorted,
 *                 disjoint; its rows are the union of its segments
 *   gather_rows   NULL, or [B, max_gather] logical rows to attend instead of
 *                 all segment rows ([RK]: protected token rows recomputed
 *                 online); n_gather [B] gives how many entries are used.
 *                 Every gathered row must lie in a segment, and the rows of
 *                 each group of entries [128 k, 128 k + 128) in segments of
 *                 one q_version (they share one query panel); a sequence
 *                 that breaks either rule records BAD_INDEX and gets NaN
 *                 o_lat and lse.
 *   q_pos         [B*s_q] request positions (int32)
 *   o_lat         [B*s_q, H, d_c] out (float), indexed by head id: heads
 *                 not listed are not written
 *   lse           [B*s_q, H] out (float): natural-log sum of exp of the
 *                 scaled visible scores; a query that sees no row gets
 *                 o_lat = 0 and lse = -inf
 *   workspace     scratch of ws_bytes >= mla_decode_workspace_size(dims, B,
 *                 s_q, n_ver, n_h),
 *                 256-byte aligned; contents need not be initialised
 * Rows past the end of a segment in its last page, and pages no table
 * references, may hold anything (NaN included) without affecting results.
 * Errors: INVALID_ARG (null/size/alignment), UNSUPPORTED (page_size != 64,
 * n_ver > 8, or n_pages * page_size, max_pages * page_size or
 * n_ver * B * s_q * H beyond 2^31 - 1: device indices are 32-bit),
 * WORKSPACE (ws_bytes too small). */
mla_status_t mla_decode(const mla_dims_t* dims, int32_t B, int32_t s_q, const void* q_abs,
                        int32_t n_ver, const int32_t* head_ids, int32_t n_h,
                        const void* cache,
                        int64_t n_pages, const int32_t* block_table, int32_t max_pages,
                        const mla_seg_t* segs, int32_t max_segs, const int32_t* gather_rows,
                        const int32_t* n_gather, int32_t max_gather, const int32_t* q_pos,
                        float* o_lat, float* lse, void* workspace, size_t ws_bytes,
                        mla_stream_t stream);

/* Bytes of workspace mla_decode needs for these sizes on the current device,
 * with or without a head list (0 if the arguments are invalid or the device
 * cannot be queried). */
size_t mla_decode_workspace_size(const mla_dims_t* dims, int32_t B, int32_t s_q,
                                 int32_t n_ver, int32_t n_h);

/* ---------------------------------------------------------------------------
 * mla_decode_static_ws -- mla_decode without a caller workspace.  The papers
 * have no counterpart: this is a library convenience for callers that cannot
 * allocate device memory at decode time (a server whose KV page pool holds
 * all free device memory; a C host without a device allocator).
 *
 * Arguments, layouts, results and errors are those of mla_decode minus
 * workspace/ws_bytes.  The scratch is a static device array of
 * MLA_DECODE_STATIC_WS_BYTES (48 MiB) inside the library, reserved when its
 * module loads; nothing is allocated per call.
 *   - Sizes whose mla_decode_workspace_size exceeds the array are rejected
 *     with MLA_ERR_WORKSPACE before anything is launched (on a 148-SM device
 *     the split partials take 38.9 MB; the rest holds the plan of up to
 *     B * s_q * ceil(n_h / 128) streams and the packed queries of a head
 *     list, n_ver * B * s_q * n_h * 1152 bytes).  Invalid dims or sizes give
 *     MLA_ERR_INVALID_ARG; a device that cannot be queried gives
 *     MLA_ERR_CUDA.
 *   - The array is reserved when the library's module for it loads, which
 *     the runtime does lazily, at the first call of mla_decode_static_ws_init
 *     or mla_decode_static_ws on a device.  A host that reserves the rest of
 *     device memory (a KV page pool) must make one of those calls first, and
 *     before any stream capture.  Every call looks the address up again, so
 *     a device reset or a new context needs only that first call again.
 *   - Every call on a device shares the one array, which keeps the previous
 *     call's contents (nothing in it needs clearing).  Calls that overlap on
 *     the GPU -- other streams, other host threads -- race on it: serialise
 *     them on one stream. */
#define MLA_DECODE_STATIC_WS_BYTES ((size_t)48 << 20)

/* Loads the static scratch array on the current device (reserving its 48 MiB)
 * and checks that its address resolves; launches nothing.  MLA_OK, or
 * MLA_ERR_CUDA when the module cannot be loaded (e.g. no room left). */
mla_status_t mla_decode_static_ws_init(void);

mla_status_t mla_decode_static_ws(const mla_dims_t* dims, int32_t B, int32_t s_q,
                                  const void* q_abs, int32_t n_ver, const int32_t* head_ids,
                                  int32_t n_h,
                                  const void* cache, int64_t n_pages,
                                  const int32_t* block_table, int32_t max_pages,
                                  const mla_seg_t* segs, int32_t max_segs,
                                  const int32_t* gather_rows, const int32_t* n_gather,
                                  int32_t max_gather, const int32_t* q_pos, float* o_lat,
                                  float* lse, mla_stream_t stream);

/* ---------------------------------------------------------------------------
 * mla_merge_lse -- merge two partial attentions over disjoint key sets.
 * [RK]: certified Local-head contributions kept offline (MLA-Off) and the
 * rows recomputed online (MLA-Online) are merged before the single shared
 * output projection.  For each query row q and listed head h = head_ids[k]
 * (k < n_h; NULL lists heads 0 .. n_h-1; an id outside [0, H) records
 * BAD_INDEX and is skipped):
 *   lse = log(exp(lse_a) + exp(lse_b))
 *   o   = exp(lse_a - lse) * o_a + exp(lse_b - lse) * o_b
 * with lse = -inf and o = 0 when both sides are empty.
 *   o_a, o_b, o     [n_q, H, d]   (float)
 *   lse_a, lse_b, lse [n_q, H]    (float)
 * o may equal o_a or o_b and lse may equal lse_a or lse_b (in place); no
 * other aliasing.  Errors: INVALID_ARG. */
mla_status_t mla_merge_lse(int32_t n_q, int32_t H, const int32_t* head_ids, int32_t n_h,
                           int32_t d, const float* o_a, const float* lse_a, const float* o_b,
                           const float* lse_b, float* o, float* lse, mla_stream_t stream);

/* ---------------------------------------------------------------------------
 * mla_out_proj -- value up-projection per head, then the shared output
 * projection.  [T27] "Move the Value Expansion After the Weighted Sum": the
 * one mixed latent is expanded once, v_h = W_UV[h] o_lat_h, and each head's
 * value joins the final output projection, out = W_O [v_0; ...; v_{H-1}].
 *   o_lat [n_q, H, d_c]     (float)
 *   w_uv  [H, d_v, d_c]     (dtype)
 *   w_o   [d_model, H*d_v]  (dtype) or NULL to stop after v
 *   v     [n_q, H, d_v]     out (float)
 *   out   [n_q, d_model]    out (float); ignored when w_o is NULL
 * For dtype MLA_BF16 the float operands o_lat and v are rounded to bfloat16
 * on their way into the tensor-core products (accumulation stays fp32).
 * Errors: INVALID_ARG. */
mla_status_t mla_out_proj(const mla_dims_t* dims, int32_t n_q, const float* o_lat,
                          const void* w_uv, const void* w_o, float* v, float* out,
                          mla_stream_t stream);

/* ---------------------------------------------------------------------------
 * mla_append_rows -- write new tokens into the paged latent cache (the cache
 * writer upstream of mla_decode).
 * [T27] "Position Rotations Complicate the Absorption": the decoupled rotary
 * key is cached beside the latent, already rotated.  [RK]: a document is
 * cached at canonical positions 0, 1, ... and relocated on the query side.
 * Entry i becomes the cache row of logical row row[i] of sequence seq[i]
 * (page block_table[seq[i]][row[i] / page_size], slot row[i] % page_size):
 *     [ c_new[i] | R(cache_pos[i]) k_rope_raw[i] ]
 * with the rotation of mla_absorb_q (adjacent pairs, angle cache_pos *
 * rope_base^(-2j/d_r) in double, result rounded to dtype).  cache_pos is the
 * row's request position minus the relocation offset it will be served with
 * (a prefix row: its request position; a document cached on its own: 0, 1, ...).
 *
 *   n_new         entries (0 is a no-op)
 *   c_new         [n_new, d_c] latents (dtype)
 *   k_rope_raw    [n_new, d_r] rotary keys before rotation (dtype)
 *   cache_pos     [n_new] int32 rotation positions
 *   seq, row      [n_new] int32 sequence index (< B) and logical row
 *   cache         [n_pages, page_size, d_c + d_r] (dtype), written in place
 *   block_table   [B, max_pages] int32 page ids
 *   key_gram      NULL for plain rows; for a QK-normed cache ("QK-Normed
 *                 MLA" abstract) the Gram matrix [d_c, d_c] (float) from
 *                 mla_qknorm_key_gram.  Then each written row also gets
 *                 key_inv_rms[page * page_size + slot] = 1 / sqrt(c^T G c +
 *                 qk_eps), the inverse RMS of its H * d_n content keys, and
 *                 its rotary key is stored multiplied by sqrt(c^T G c +
 *                 qk_eps), the form mla_decode_qknorm reads.
 *   qk_eps        RMSNorm epsilon (>= 0; read with key_gram only)
 *   key_inv_rms   [n_pages * page_size] float, written in place; NULL
 *                 exactly when key_gram is NULL
 * Only the addressed rows change.  Two entries naming one row race.
 * Errors: INVALID_ARG (null pointers, sizes, misaligned element pointers),
 * UNSUPPORTED (page_size != 64).  An entry whose sequence, row or page id is
 * out of range is skipped and records BAD_INDEX in the status word. */
mla_status_t mla_append_rows(const mla_dims_t* dims, int32_t n_new, const void* c_new,
                             const void* k_rope_raw, const int32_t* cache_pos,
                             const int32_t* seq, const int32_t* row, int32_t B, void* cache,
                             int64_t n_pages, const int32_t* block_table, int32_t max_pages,
                             const float* key_gram, float qk_eps, float* key_inv_rms,
                             mla_stream_t stream);

/* mla_debug_wait_probe -- checks the bounded-wait path without a fault: one
 * thread waits, through the decode kernels' own bounded wait, on a barrier
 * phase that never completes, gives up after limit_ns (1 us .. 100 ms), and
 * records MLA_ERR_TIMEOUT in the status word as a decode role does; nothing
 * is in flight, so the kernel returns and the context stays usable.
 * waited_us (device, int32) receives the time it waited, in microseconds.
 * Errors: INVALID_ARG for a limit out of range or a null / misaligned
 * waited_us. */
mla_status_t mla_debug_wait_probe(int64_t limit_ns, int32_t* waited_us, mla_stream_t stream);

/* ---------------------------------------------------------------------------
 * Low-bit latent cache (QuantMLA abstract: the content and rotary caches
 * kept as INT4 / INT4 or INT2 / INT4 codes, unpacked and dequantised inside
 * the attention).  A packed row is d_c content codes of bits_c bits, then
 * d_r rotary codes of bits_r bits, little-end first: code k of a segment
 * occupies bits [bits*k mod 8, ...) of byte bits*k/8 of the segment, as a
 * two's complement field.  Row bytes: (d_c*bits_c + d_r*bits_r) / 8 (288 at
 * INT4/INT4, 160 at INT2/INT4 for 512 + 64 channels).  One static scale per
 * channel: a code stands for code * scale_c[k] (content channel k) or
 * code * scale_r[k] (rotary channel k).  (bits_c, bits_r) is (4, 4) or
 * (2, 4), and d_c * bits_c and d_r * bits_r must be multiples of 32.
 *
 * mla_pack_rows -- packed[i] = codes of rows[i] [n_rows, d_c + d_r] (dtype):
 *   code = round-half-even(x / scale) in fp32, clamped to the signed range.
 *   packed [n_rows, row bytes], 4-byte aligned.
 * mla_decode_lowbit -- mla_decode over a pool of packed rows
 *   cache [n_pages, page_size, row bytes] (4-byte aligned): the result is
 *   attention over the dequantised rows.  The scales are folded into the
 *   query and the output (scores of the scaled query against the codes; the
 *   weighted sum of codes times scale_c), so no row is ever dequantised in
 *   memory.  Head lists, segments, gathered rows, masking and outputs are
 *   those of mla_decode; no workspace.  UNSUPPORTED for other bit pairs.
 *   This kernel is a SIMT kernel: one CTA per (head, query row). */
mla_status_t mla_pack_rows(const mla_dims_t* dims, int32_t bits_c, int32_t bits_r,
                           int64_t n_rows, const void* rows, const float* scale_c,
                           const float* scale_r, void* packed, mla_stream_t stream);

mla_status_t mla_decode_lowbit(const mla_dims_t* dims, int32_t bits_c, int32_t bits_r,
                               int32_t B, int32_t s_q, const void* q_abs, int32_t n_ver,
                               const int32_t* head_ids, int32_t n_h, const void* cache,
                               const float* scale_c, const float* scale_r, int64_t n_pages,
                               const int32_t* block_table, int32_t max_pages,
                               const mla_seg_t* segs, int32_t max_segs,
                               const int32_t* gather_rows, const int32_t* n_gather,
                               int32_t max_gather, const int32_t* q_pos, float* o_lat,
                               float* lse, mla_stream_t stream);

/* ---------------------------------------------------------------------------
 * Tensor-core route of the low-bit cache (same packed rows, same scales).
 *
 * mla_lowbit_dequant_bytes -- bytes of a pool of n_pages pages of dtype rows
 *   (n_pages * page_size * (d_c + d_r) * sizeof(dtype)); 0 for bad dims.
 * mla_dequant_rows -- out[i][k] = code_k(packed[i]) * scale_k, the product in
 *   fp32, rounded to dims->dtype (round to nearest even for bf16).  packed
 *   [n_rows, row bytes] 4-byte aligned; out [n_rows, d_c + d_r] 16-byte
 *   aligned.  Bit pairs and dims as mla_pack_rows; UNSUPPORTED when
 *   d_c + d_r > 8192.
 * mla_decode_lowbit_tc -- the result of mla_decode_lowbit computed as
 *   mla_dequant_rows over the whole packed pool (n_pages * page_size rows)
 *   into the caller's scratch pool `dequant` (>= mla_lowbit_dequant_bytes,
 *   256-byte aligned, else MLA_ERR_WORKSPACE / MLA_ERR_INVALID_ARG), then
 *   mla_decode over that pool with the workspace (its rules and its errors;
 *   the bf16 decode runs on the tensor cores).  The difference from
 *   mla_decode_lowbit is where the scales act: here on each dequantised
 *   element, rounded to dtype; there on the query and the output.  The
 *   scratch pool's contents afterwards are the dequantised rows (or
 *   unspecified when the decode refused the call).  Cost: one read of the
 *   packed pool, one write of the dequantised pool, then the decode, which
 *   reads the pool back from L2 when it fits there. */
size_t mla_lowbit_dequant_bytes(const mla_dims_t* dims, int64_t n_pages);

mla_status_t mla_dequant_rows(const mla_dims_t* dims, int32_t bits_c, int32_t bits_r,
                              int64_t n_rows, const void* packed, const float* scale_c,
                              const float* scale_r, void* out, mla_stream_t stream);

mla_status_t mla_decode_lowbit_tc(const mla_dims_t* dims, int32_t bits_c, int32_t bits_r,
                                  int32_t B, int32_t s_q, const void* q_abs, int32_t n_ver,
                                  const int32_t* head_ids, int32_t n_h, const void* cache,
                                  const float* scale_c, const float* scale_r, int64_t n_pages,
                                  const int32_t* block_table, int32_t max_pages,
                                  const mla_seg_t* segs, int32_t max_segs,
                                  const int32_t* gather_rows, const int32_t* n_gather,
                                  int32_t max_gather, const int32_t* q_pos, float* o_lat,
                                  float* lse, void* dequant, size_t dequant_bytes,
                                  void* workspace, size_t ws_bytes, mla_stream_t stream);

/* ---------------------------------------------------------------------------
 * QK-normed MLA ("QK-Normed MLA" abstract): RMSNorm of the content query and
 * of each token's content keys after the key up-projection, with all heads
 * one group (statistics over H * d_n values).  In the absorbed form the
 * query carries both norm weights and is absorbed as usual; the key side is
 * one inverse RMS per cached token, applied per score column:
 *   score(t) = scale * (q_abs_content . c_t * inv_t + q_abs_rope . k_rope_t)
 * with the cached rotary key of a QK-normed cache stored times 1 / inv_t
 * (mla_append_rows with key_gram), so the score is scale * inv_t times the
 * plain 576-wide product.
 *
 * mla_qknorm_query -- q_out[r] = q_nope[r] / sqrt(mean(q_nope[r]^2) + eps)
 *   * g_q * g_k over the H * d_n values of query row r (rounded to dtype);
 *   pass q_out to mla_absorb_q as q_nope.
 *   q_nope, q_out [n_rows, H, d_n] (dtype); g_q, g_k [H * d_n] (float).
 * mla_qknorm_key_gram -- gram = W_UK^T W_UK / (H * d_n), [d_c, d_c] float,
 *   with W_UK [H, d_n, d_c] (dtype) seen as [H * d_n, d_c]: then
 *   mean_j (W_UK c)_j^2 = c^T gram c.  Depends on the weights only.
 * mla_decode_qknorm -- mla_decode with the per-column factor inv_t read from
 *   key_inv_rms [n_pages * page_size] (float, 16-byte aligned; a row's
 *   entry at page * page_size + slot, as the writer stores it).  Page mode
 *   only: no gathered rows.  Other arguments, layouts and errors are those
 *   of mla_decode; INVALID_ARG when key_inv_rms is NULL. */
mla_status_t mla_qknorm_query(const mla_dims_t* dims, int32_t n_rows, const void* q_nope,
                              const float* g_q, const float* g_k, float eps, void* q_out,
                              mla_stream_t stream);

mla_status_t mla_qknorm_key_gram(const mla_dims_t* dims, const void* w_uk, float* gram,
                                 mla_stream_t stream);

mla_status_t mla_decode_qknorm(const mla_dims_t* dims, int32_t B, int32_t s_q,
                               const void* q_abs, int32_t n_ver, const int32_t* head_ids,
                               int32_t n_h, const void* cache, const float* key_inv_rms,
                               int64_t n_pages, const int32_t* block_table, int32_t max_pages,
                               const mla_seg_t* segs, int32_t max_segs, const int32_t* q_pos,
                               float* o_lat, float* lse, void* workspace, size_t ws_bytes,
                               mla_stream_t stream);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* MLA_H_ */
