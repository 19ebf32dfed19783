/*
 * axr.h -- C ABI of the B200 (sm_100a) implementation of AXELRAM decode-time attention from quantized key indices.
 *
 * Method source: "AXELRAM: Quantize Once, Never Dequantize" (arXiv 2604.02638), as carried by the ai-navigate-news
 * digest (Key Points, Abstract) and the mlsanity index card (Abstract).  Keys are written once through a fixed
 * orthogonal transform and a design-time scalar codebook ("transform on write"); attention scores are read by table
 * lookup on the stored indices with no inverse transform and no reconstruction of the key ("table lookup on read").
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Plain C types only.  fp16 tensors are passed as uint16_t* holding IEEE binary16 bit patterns.  `stream` is a
 *    cudaStream_t (NULL = the legacy default stream).  Device pointers are marked [dev], host pointers [host].
 *  - The caller owns every buffer.  No entry point allocates device memory per call; entry points that need scratch
 *    take a caller-provided workspace whose size comes from the matching *_workspace_bytes() function.  The one
 *    exception is axr_attend_decode_static, which uses a fixed 4 MiB module-scope device array instead.
 *  - Device work is asynchronous on `stream`.  Argument errors are detected on the host and returned before any
 *    launch (no device work is queued).  Launch errors come from cudaGetLastError and return AXR_ECUDA.
 *  - The decode entry points launch their split merge as a programmatic dependent of the decode kernel on the same
 *    stream (its blocks wait on the device for the decode kernel's completion); work the caller enqueues before or
 *    after keeps plain stream order.
 *  - On any status other than AXR_OK, axr_last_error() returns a thread-local human-readable message.
 *  - Fixed notation: d head dim (power of two), b bits per index, L = 2^b levels, s the +-1 sign vector, H the
 *    Sylvester Walsh-Hadamard matrix scaled by 1/sqrt(d) (symmetric, H*H = I), G = Hq/Hkv (query head h reads KV
 *    head h / G).
 *  - Cache layouts (row-major, innermost last):
 *      codes  [B, Hkv, Tcap, R] uint8, R = d*b/8 bytes per token: an LSB-first bitstream in which coordinate j
 *             holds bits [j*b, j*b+b); index k means centroid c_k, k = 0 the most negative;
 *      norms  [B, Hkv, Tcap] fp16, the token's L2 norm rounded to nearest even;
 *      values [B, Hkv, Tcap, d] fp16 (AXR_V_F16), or codes + norms of the same shape as the keys (AXR_V_QUANT);
 *      q      [B, Hq, d] fp32;  out [B, Hq, d] fp32;  scores [B, Hq, T] fp32.
 *    Tcap >= T is the allocated capacity (row stride); only tokens t < seq_lens[b] (or t < T when seq_lens is
 *    NULL) are read.
 *  - Alignment: codes base 16 bytes, norms 4 bytes, q/out/scores 16 bytes, fp16 values 16 bytes.
 *  - Supported: d in {64, 128} (the writer and the selector also take d = 8), b in {1, 2, 3, 4},
 *    G in {1, 2, 4, 8}.  Anything else returns AXR_EUNSUPPORTED.
 */
#ifndef AXR_H_
#define AXR_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define AXR_API __attribute__((visibility("default")))
#else
#define AXR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum axr_status {
  AXR_OK = 0,
  AXR_EINVAL = 1,        /* null pointer, negative or inconsistent size, misaligned pointer */
  AXR_EUNSUPPORTED = 2,  /* d, b or G outside the compiled set */
  AXR_ECUDA = 3,         /* a CUDA runtime call or a kernel launch failed */
  AXR_EWORKSPACE = 4     /* workspace missing or smaller than the matching *_workspace_bytes() */
} axr_status;

typedef enum axr_dtype { AXR_F32 = 0, AXR_F16 = 1 } axr_dtype;
/* Value storage for axr_attend_decode: fp16 rows, quantized rows (the keys' layout), or quantized and tiled
 * (axr_write_values_tiled's layout, d = 128). */
typedef enum axr_vkind { AXR_V_F16 = 0, AXR_V_QUANT = 1, AXR_V_QUANT_TILED = 2 } axr_vkind;

/* Thread-local message for the last non-OK status returned on this thread (empty string if none). */
AXR_API const char* axr_last_error(void);

/*
 * Device status word.  Every spin-wait inside the library's kernels (on an mbarrier that a bulk copy completes, or on
 * a pipeline stage being armed) gives up after a bounded number of polls, about a second, instead of hanging the
 * GPU.  A block that gave up writes NaN into the outputs it owns and sets AXR_STATUS_WAIT_TIMEOUT in the status word
 * of its device; the call that launched it has already returned AXR_OK.  The word is sticky (calls never clear it).
 *
 * axr_device_status -- synchronizes the current device (cudaDeviceSynchronize), then copies its status word to
 * *flags [host].  clear != 0 resets the word to 0 after reading.  Returns AXR_ECUDA with a message when
 * AXR_STATUS_WAIT_TIMEOUT is set, AXR_OK otherwise; AXR_EINVAL for a null flags pointer.  A caller that wants to
 * tell a timed-out call from NaN inputs checks the word after the call.
 *
 * axr_selftest_wait_timeout -- the library's test of that give-up path: one block waits on an mbarrier that nothing
 * arrives on (no copy pending), gives up after `polls` polls (1 .. 2^20), sets AXR_STATUS_WAIT_TIMEOUT and returns.
 * The GPU context stays usable.  Asynchronous on `stream`.  Not part of the method.
 */
#define AXR_STATUS_WAIT_TIMEOUT 1u
AXR_API axr_status axr_device_status(unsigned int* flags, int clear);
AXR_API axr_status axr_selftest_wait_timeout(int polls, void* stream);

/* ABI version: major*10000 + minor*100 + patch. */
AXR_API int axr_version(void);

/*
 * axr_codebook -- design-time codebook (AXELRAM Abstract: the transform makes each coordinate ~N(0, 1/d), so the
 * optimal scalar quantizer depends only on d and b).  Lloyd-Max quantizer of N(0,1), symmetrised, scaled by
 * 1/sqrt(d).  Host only; no CUDA call.
 *   centroids  [host] out, L doubles, increasing (unit scale: gamma_k / sqrt(d));
 *   thresholds [host] out, L-1 doubles, increasing, t_k = (c_{k-1} + c_k) / 2.
 * Errors: AXR_EINVAL for null outputs; AXR_EUNSUPPORTED for d not a power of two in [1, 4096] or b outside 1..4.
 */
AXR_API axr_status axr_codebook(int d, int bits, double* centroids, double* thresholds);

/*
 * axr_write_keys -- write path (AXELRAM Key Points, 2nd item, and Abstract: transform on write).  For each input
 * vector x (also used for V when values are quantized):
 *   n = ||x||_2 (fp32);  y = H (s .* x);  u = y / n (u = 0 when n = 0);
 *   idx_j = #{k >= 1 : u_j >= t_k}  (a value on a threshold goes up);  pack idx LSB-first;  norm = fp16_rne(n).
 *   x         [dev] [n_vec, d] of x_dtype (AXR_F32 or AXR_F16), contiguous rows;
 *   signs     [dev] [d] int8, negative = -1, otherwise +1;
 *   dst_rows  [dev] [n_vec] int64 destination row of each vector in codes/norms, or NULL for row i -> row i
 *             (appending one token per (batch, KV head) into a [B, Hkv, Tcap] cache uses (b*Hkv + h)*Tcap + t);
 *   codes     [dev] out, rows of R = d*b/8 bytes;  norms [dev] out, fp16 per row.
 * Errors: AXR_EINVAL (null pointer, n_vec < 0, bad dtype, misalignment), AXR_EUNSUPPORTED (d or b), AXR_ECUDA.
 * n_vec == 0 is a no-op.
 */
AXR_API axr_status axr_write_keys(const void* x, axr_dtype x_dtype, int64_t n_vec, int d, int bits, const int8_t* signs,
                          const int64_t* dst_rows, uint8_t* codes, uint16_t* norms, void* stream);

/*
 * axr_write_values_tiled -- the write path of axr_write_keys (same transform, norm, codebook and tie rule) with the
 * codes stored for the tensor-core value product: the cache is cut into tiles of 128 tokens and within a tile each
 * coordinate's 128 codes form one LSB-first bitstream, token o at bits [o*b, o*b + b).  The pages fix no layout
 * (AXELRAM Key Points, 2nd item, quantizes the cache once; the values are quantized the same way); this one lets
 * the read path gather two tokens' values of a coordinate with one lookup.
 *   x         [dev] [n_vec, d] of x_dtype, contiguous rows;  signs [dev] [d] int8;
 *   dst_rows  [dev] [n_vec] int64 destination rows r = (b*Hkv + h)*Tcap + t, distinct, or NULL for rows 0..n_vec-1;
 *   Tcap      tokens per (batch, KV head) in the cache, a positive multiple of 128;
 *   codes     [dev] out, [B*Hkv][Tcap/128][d][16*b] bytes (4-byte aligned);  norms [dev] out, fp16 per row r.
 * With dst_rows NULL and n_vec a multiple of 128 whole tiles are written with plain stores; otherwise each code is
 * replaced in place with word atomics (other tokens of the tile keep theirs).
 * Errors: AXR_EINVAL (null pointer, n_vec < 0, bad dtype, Tcap, misalignment), AXR_EUNSUPPORTED (d != 128, b),
 * AXR_ECUDA.  n_vec == 0 is a no-op.
 */
AXR_API axr_status axr_write_values_tiled(const void* x, axr_dtype x_dtype, int64_t n_vec, int d, int bits,
                                          const int8_t* signs, const int64_t* dst_rows, int Tcap, uint8_t* codes,
                                          uint16_t* norms, void* stream);

/*
 * axr_score -- read-path scores (AXELRAM Key Points, 1st and 2nd items; Abstract: scores straight from the indices
 * by table lookup, no inverse transform).  Per (batch b, query head h): q~ = H (s .* q); a d x L table
 * LUT[j][k] = scale * q~_j * c_k is built in shared memory; for each token t < len_b
 *   scores[b, h, t] = norm_t * sum_j LUT[j][idx_{t,j}],   and scores[b, h, t] = -inf for len_b <= t < T.
 *   q [dev] [B,Hq,d] f32;  kcodes/knorms [dev] cache layout;  seq_lens [dev] [B] int32 or NULL (all T);
 *   scores [dev] out [B, Hq, T] f32.
 * Errors: AXR_EINVAL (pointers, sizes, T > Tcap, Hq not a multiple of Hkv, alignment), AXR_EUNSUPPORTED, AXR_ECUDA.
 * T == 0 or B == 0 is a no-op.  seq_lens entries are clamped to [0, T].
 */
AXR_API axr_status axr_score(const float* q, const uint8_t* kcodes, const uint16_t* knorms, const int32_t* seq_lens, int B,
                     int Hq, int Hkv, int T, int Tcap, int d, int bits, const int8_t* signs, float scale,
                     float* scores, void* stream);

/*
 * Table read mode of axr_score (process-wide; default AXR_GATHER_MMA, the fastest on B200).  Every mode computes the same table
 * entries LUT[j][k] = scale * q~_j * c_k (AXELRAM Key Points, 2nd item) summed at each token's indices, and they agree
 * to within the score tolerance:
 *   AXR_GATHER_TABLE     the table itself sits in shared memory, G heads wide (one 16-byte entry serves four
 *                        heads), and each token is one thread summing one lookup per field of its code row: a
 *                        field of W bits covers W/b coordinates, its entry the sum of their q~_j c_k -- W = 8 at
 *                        b <= 2 (byte-indexed tables of 4 or 8 coordinates), 6 at b = 3, 8 or 4 at b = 4 (by
 *                        G, as the tables fit); axr_attend_decode over fp16 values in this mode also reads the
 *                        keys through it (values on the CUDA cores);
 *   AXR_GATHER_FACTORED  the table is held factored -- row factor q~_j in registers, column factor c_k gathered two
 *                        coordinates at a time from a byte-indexed pair table -- and each entry is formed by the
 *                        packed fp32 FMA that accumulates it; half the shared-memory wavefronts of TABLE;
 *   AXR_GATHER_TENSOR    the same factored table on the tensor cores: each token's gathered column factors (split
 *                        into hi and lo fp16 planes, about 22 bits) form a row of an MMA operand in tensor memory,
 *                        the row factors (split the same way) the other operand, and tcgen05.mma accumulates the
 *                        G sums per token in fp32;
 *   AXR_GATHER_MMA       the same hi/lo operands as warp-level MMAs (mma.sync, operands in registers): one table
 *                        lookup gives a token's hi and lo registers for two coordinates;
 *   AXR_GATHER_DIRECT    the AXR_GATHER_MMA arithmetic with every lane's code slice loaded from global memory
 *                        straight into registers (coalesced, several groups in flight per warp; no staging tile,
 *                        no block barrier): shared memory serves the table lookups alone.  The decode entry
 *                        points treat it as AXR_GATHER_MMA.
 * axr_attend_decode reads the key table in factored form; with tiled values the value product runs as warp-level
 * MMAs, or, in AXR_GATHER_TENSOR mode, both products run as tcgen05 MMAs.  Errors: AXR_EINVAL for an unknown mode.
 */
typedef enum axr_gather {
  AXR_GATHER_FACTORED = 0,
  AXR_GATHER_TABLE = 1,
  AXR_GATHER_TENSOR = 2,
  AXR_GATHER_MMA = 3,
  AXR_GATHER_DIRECT = 4
} axr_gather;
AXR_API axr_status axr_set_gather(axr_gather mode);
AXR_API axr_gather axr_get_gather(void);

/* Bytes of workspace that axr_attend_decode / axr_dense_decode need for these sizes (0 when B, Hq or T is 0).
 * Depends only on the arguments. */
AXR_API size_t axr_attend_workspace_bytes(int B, int Hq, int Hkv, int T, int d);

/*
 * axr_attend_decode -- one decode step of attention over a quantized key cache: the scores of axr_score (scaled by
 * `scale`, typically 1/sqrt(d)), an online softmax per split of the token axis, the value product, and a merge of
 * the splits.  Values are fp16 (AXR_V_F16: out = sum_t p_t v_t) or quantized like the keys with the same signs
 * (AXR_V_QUANT: the weighted sum is formed in the rotated domain and mapped back once, out = s .* H (sum_t p_t
 * n^V_t c[idx^V_t])).  AXR_V_QUANT_TILED takes the value codes in axr_write_values_tiled's layout (d = 128, Tcap
 * a multiple of 128) and forms the value product on the tensor cores: per 128-token tile an M = 128 (coordinates) x
 * N = 16 (heads) x K = 128 (tokens) MMA of the fp16 value centroids with the fp16 weights p_t n^V_t, accumulated in
 * fp32.  The softmax, the value product and the split merge are not on the pages (an SRAM macro only scores); they
 * are the standard definitions.  A batch row with len_b = 0 gets out = 0.
 *   v [dev] fp16 values or value codes;  vnorms [dev] value norms (quantized kinds) or NULL (AXR_V_F16);
 *   out [dev] [B, Hq, d] f32;  workspace [dev] >= axr_attend_workspace_bytes(B, Hq, Hkv, T, d) bytes, 16-aligned.
 * Errors: as axr_score, plus AXR_EWORKSPACE.
 */
AXR_API axr_status axr_attend_decode(const float* q, const uint8_t* kcodes, const uint16_t* knorms, axr_vkind vkind,
                             const void* v, const uint16_t* vnorms, const int32_t* seq_lens, int B, int Hq, int Hkv,
                             int T, int Tcap, int d, int bits, const int8_t* signs, float scale, float* out,
                             void* workspace, size_t ws_bytes, void* stream);

/*
 * axr_decode_step -- one decode step in one call.  The new token's key and value (k_new, v_new: [B, Hkv, d] fp16)
 * are written into the cache at position len_b - 1 of each batch row (len_b = seq_lens[b], or T): keys through the
 * write path of axr_write_keys (codes and fp16 norm), values the same way (AXR_V_QUANT) or as they are (AXR_V_F16).
 * Then axr_attend_decode runs over positions [0, len_b), the new token included.  The write happens inside the
 * decode launch, by the block that attends over that position, before that block copies the position's tile in, so
 * the step needs no separate append launch.  Digest, Key Points 2 ("transform on write") for the write, and
 * axr_attend_decode for the read.  Row value layouts only (AXR_V_F16, AXR_V_QUANT).  Batch rows with len_b = 0 get
 * out = 0 and nothing is written.
 *   kcodes, knorms, v, vnorms [dev]: the cache as for axr_attend_decode; one position per (b, KV head) is written;
 *   k_new, v_new [dev] [B, Hkv, d] fp16, 16-byte aligned.
 * Errors: as axr_attend_decode; AXR_EINVAL for the tiled value layout or a null or misaligned k_new / v_new.
 */
AXR_API axr_status axr_decode_step(const float* q, const uint16_t* k_new, const uint16_t* v_new, uint8_t* kcodes,
                                   uint16_t* knorms, axr_vkind vkind, void* v, uint16_t* vnorms,
                                   const int32_t* seq_lens, int B, int Hq, int Hkv, int T, int Tcap, int d, int bits,
                                   const int8_t* signs, float scale, float* out, void* workspace, size_t ws_bytes,
                                   void* stream);

/*
 * Paged caches.  A serving KV cache is allocated in blocks: the pages quantize every token once on write and read it
 * many times (AXELRAM Key Points, 2nd item), and a server hands out cache space a block at a time.  The paged entry
 * points read (and axr_decode_step_paged writes) the same per-token rows through a block table:
 *   block_table [dev] [B, max_blocks] int32: logical block j of batch row b (tokens [j bt, (j + 1) bt)) lives in
 *               pool block block_table[b * max_blocks + j]; only the entries of blocks below ceil(len_b / bt) are
 *               read, and each must be a valid block of the pools;
 *   block_tokens bt, a power of two in [16, 2^20];
 *   pools       codes [num_blocks, Hkv, bt, R] uint8, norms [num_blocks, Hkv, bt] fp16, values [num_blocks, Hkv, bt,
 *               d] fp16 (AXR_V_F16) or codes + norms shaped like the keys (AXR_V_QUANT): the bt rows of one (block,
 *               KV head) are contiguous.  Row r = (p Hkv + hk) bt + o of a pool is token o of block p for KV head
 *               hk, so axr_write_keys with dst_rows fills a pool (prefill) the same way;
 *   T           an upper bound of the sequence lengths, <= max_blocks * bt (it sizes the workspace and the splits);
 *               seq_lens [B] (or NULL: every row has T tokens).
 * Everything else (arguments, results, alignment, workspace, errors) is as in axr_attend_decode / axr_decode_step;
 * AXR_EINVAL also for a bad block size, T above the table's reach, a null or misaligned table, or tiled values.
 */
AXR_API axr_status axr_attend_decode_paged(const float* q, const uint8_t* kcodes, const uint16_t* knorms,
                                           axr_vkind vkind, const void* v, const uint16_t* vnorms,
                                           const int32_t* block_table, int max_blocks, int block_tokens,
                                           const int32_t* seq_lens, int B, int Hq, int Hkv, int T, int d, int bits,
                                           const int8_t* signs, float scale, float* out, void* workspace,
                                           size_t ws_bytes, void* stream);
AXR_API axr_status axr_decode_step_paged(const float* q, const uint16_t* k_new, const uint16_t* v_new,
                                         uint8_t* kcodes, uint16_t* knorms, axr_vkind vkind, void* v,
                                         uint16_t* vnorms, const int32_t* block_table, int max_blocks,
                                         int block_tokens, const int32_t* seq_lens, int B, int Hq, int Hkv, int T,
                                         int d, int bits, const int8_t* signs, float scale, float* out,
                                         void* workspace, size_t ws_bytes, void* stream);

/*
 * axr_attend_decode_static -- axr_attend_decode without a workspace argument, for callers that cannot allocate
 * device memory (code running inside a memory pool it does not own, plugins handed only input and output pointers,
 * decode steps that must not touch an allocator).  The paper has no counterpart: this is a deployment convenience.
 * The split partials live in a fixed library-owned device array of axr_attend_static_scratch_bytes() bytes (4 MiB),
 * which every GPU that loads the library holds until the process exits.  Nothing is allocated per call: no
 * cudaMalloc, cudaFree or allocating library routine.
 *   Arguments, layouts and results are those of axr_attend_decode.
 *   Sizes whose axr_attend_workspace_bytes() exceeds the fixed array return AXR_EWORKSPACE (use axr_attend_decode).
 *   The first call on a device looks up the array's device address (cudaGetSymbolAddress, with that device
 *   current) and keeps it; make that first call before any stream capture.  The kept address dies with the
 *   device's context: do not call this entry point on a device after cudaDeviceReset in the same process.
 *   All calls share the one array: calls that may overlap on the GPU (different streams, or different host threads
 *   on one device) race and must be serialised by the caller.  The array keeps the last call's contents; every slot
 *   a call reads is written by that call first, so no clearing is needed.
 */
AXR_API axr_status axr_attend_decode_static(const float* q, const uint8_t* kcodes, const uint16_t* knorms,
                                            axr_vkind vkind, const void* v, const uint16_t* vnorms,
                                            const int32_t* seq_lens, int B, int Hq, int Hkv, int T, int Tcap, int d,
                                            int bits, const int8_t* signs, float scale, float* out, void* stream);
/* Size in bytes of the fixed device array axr_attend_decode_static uses. */
AXR_API size_t axr_attend_static_scratch_bytes(void);

/*
 * axr_dense_decode -- the same decode step over an unquantized fp16 K/V cache (k, v [dev] [B, Hkv, Tcap, d] fp16):
 * out = softmax(scale * q . k_t) . v.  Not part of the method: the bandwidth reference the quantized path is
 * measured against.  Same workspace rule and errors as axr_attend_decode.
 */
AXR_API axr_status axr_dense_decode(const float* q, const uint16_t* k, const uint16_t* v, const int32_t* seq_lens, int B,
                            int Hq, int Hkv, int T, int Tcap, int d, float scale, float* out, void* workspace,
                            size_t ws_bytes, void* stream);

/*
 * LOOKAT product quantization (the newx.sg summary and abstract of "LOOKAT: Lookup-Optimized Key-Attention for
 * Memory-Efficient Transformers"): keys are cut into m subspaces of d/m coordinates (subspace i = coordinates
 * [i d/m, (i+1) d/m)), each with a codebook of K <= 256 centroids learned by k-means; a key is stored as m one-byte
 * indices; a query scores it through a per-query table T[i][k] = q^(i) . C_i[k] (asymmetric distance computation:
 * the query is exact, no key is reconstructed).  The pages print no formulas; these are the textbook definitions.
 * Supported: d in {64, 128}, m in {2, 4, 8, 16}, 1 <= K <= 256, G in {1, 2, 4, 8}.
 *
 * axr_pq_train -- Lloyd's k-means of one head's keys, per subspace, from the initial centroids in codebooks:
 *   each of `iters` iterations assigns every subvector to its nearest centroid (the rule of axr_pq_encode) and
 *   moves every centroid with members to their mean (fp64 sums, rounded to fp32); a centroid without members
 *   stays.  x [dev] [n_vec, d] (AXR_F16 or AXR_F32); codebooks [dev] in/out [m, K, d/m] f32;
 *   workspace [dev] >= axr_pq_train_workspace_bytes(d, m, K), 16-aligned.
 * axr_pq_encode -- the nearest centroid of every subvector: squared Euclidean distance formed in fp32 as
 *   sum_j (x_j - c_j)^2 in increasing j, each operation rounded (no fused multiply-add), lowest index on a tie.
 *   x [dev] [n_vec, d]; codebooks [dev] [heads, m, K, d/m] f32, vector r using set (r / head_period) % heads
 *   (a [B, Hkv, Tcap, d] cache: heads = Hkv, head_period = Tcap; new tokens [B, Hkv, d]: head_period = 1);
 *   dst_rows [dev] [n_vec] int64 destination rows, or NULL for row r; codes [dev] out [rows, m] uint8.
 * axr_pq_score -- scores[b, h, t] = scale * sum_i T[i][codes[b, hk, t, i]] for t < len_b, -inf for len_b <= t < T;
 *   q [dev] [B, Hq, d] f32; codes [dev] [B, Hkv, Tcap, m]; codebooks [dev] [Hkv, m, K, d/m] f32 (one set per KV
 *   head); the table is built in shared memory per (batch row, KV head), G heads wide.
 * axr_pq_attend_decode -- decode attention with those scores (times `scale`) over fp16 values [dev]
 *   [B, Hkv, Tcap, d]: online softmax per split of the token axis, the value product, the split merge;
 *   workspace as axr_attend_decode (axr_attend_workspace_bytes).
 * Errors: AXR_EINVAL (pointers, sizes, alignment: q/v/out 16 bytes, codes 4 (m >= 4) or 2, codebooks 4),
 * AXR_EUNSUPPORTED (d, m, K, G, subspace width), AXR_EWORKSPACE, AXR_ECUDA.  n_vec == 0 / B == 0 are no-ops.
 */
AXR_API size_t axr_pq_train_workspace_bytes(int d, int m, int K);
AXR_API axr_status axr_pq_train(const void* x, axr_dtype x_dtype, int64_t n_vec, int d, int m, int K, int iters,
                                float* codebooks, void* workspace, size_t ws_bytes, void* stream);
AXR_API axr_status axr_pq_encode(const void* x, axr_dtype x_dtype, int64_t n_vec, int d, int m, int K,
                                 const float* codebooks, int heads, int head_period, const int64_t* dst_rows,
                                 uint8_t* codes, void* stream);
AXR_API axr_status axr_pq_score(const float* q, const uint8_t* codes, const float* codebooks, const int32_t* seq_lens,
                                int B, int Hq, int Hkv, int T, int Tcap, int d, int m, int K, float scale,
                                float* scores, void* stream);
AXR_API axr_status axr_pq_attend_decode(const float* q, const uint8_t* codes, const float* codebooks,
                                        const uint16_t* v, const int32_t* seq_lens, int B, int Hq, int Hkv, int T,
                                        int Tcap, int d, int m, int K, float scale, float* out, void* workspace,
                                        size_t ws_bytes, void* stream);

/*
 * Power-of-two shift-accumulate keys (the arxivdaily page of the shift-accumulate attention paper): a second codec
 * through the same split-T reducer.  The page gives no formulas; the reading implemented here:
 *   write: alpha = max_j |k_j| (fp16, exact); u = k / alpha (fp32); |u_j| to the nearest magnitude level
 *     2^-e (1 + mu / 2^M) in linear value (a value on a midpoint goes up; e in [0, 2^E - 1], mu in [0, 2^M - 1]);
 *     code = sign << (E + M) | l with l = (e_max - e) 2^M + mu the level's rank from the smallest; 1 + E + M bits per
 *     coordinate packed LSB-first (rows of d (1 + E + M) / 8 bytes), alpha per row.
 *   scores: the query in fixed point, Q_j = rint(q_j / s_q), s_q = max |q| / 32767 (fp32); S = sum_j sigma_j
 *     ((Q_j << (F - e_j)) + mu_j (Q_j << (F - e_j - M))) with head-room F = e_max + M, an exact integer; the score is
 *     scale * s_q * alpha * 2^-F * S.
 *   attend: r_t = rint(float(S) * (s_q * (scale * log2 e) * alpha_t) * 2^-F) (fp32, in that order) is an integer
 *     log2 weight; out = sum_t 2^(r_t - R) v_t / sum_t 2^(r_t - R), R = max_t r_t -- every weight and every rescale
 *     (the running maximum, the split merge) an exact power of two.  fp16 values.
 * Formats (E, M): (1, 0), (2, 0), (3, 0), (1, 1), (2, 1); d in {64, 128}; G in {1, 2, 4, 8}.
 *   axr_pot_write: x [dev] [n_vec, d] fp16 (8-byte aligned rows); dst_rows [dev] int64 or NULL; codes [dev] out;
 *     alpha [dev] out fp16 per row.
 *   axr_pot_score: q [dev] [B, Hq, d] f32; codes [dev] [B, Hkv, Tcap, row] (16-byte aligned); alpha [dev]
 *     [B, Hkv, Tcap] fp16; S_out [dev] out [B, Hq, T] int32 and/or scores [dev] out [B, Hq, T] f32 (either NULL;
 *     past len_b: S = 0 and score -inf).
 *   axr_pot_attend_decode: v [dev] [B, Hkv, Tcap, d] fp16; out [dev] [B, Hq, d] f32; workspace as
 *     axr_attend_decode (axr_attend_workspace_bytes).
 * Errors: AXR_EINVAL (pointers, sizes, alignment), AXR_EUNSUPPORTED (d, format, G), AXR_EWORKSPACE, AXR_ECUDA.
 */
AXR_API axr_status axr_pot_write(const uint16_t* x, int64_t n_vec, int d, int E, int M, const int64_t* dst_rows,
                                 uint8_t* codes, uint16_t* alpha, void* stream);
AXR_API axr_status axr_pot_score(const float* q, const uint8_t* codes, const uint16_t* alpha, const int32_t* seq_lens,
                                 int B, int Hq, int Hkv, int T, int Tcap, int d, int E, int M, float scale,
                                 int32_t* S_out, float* scores, void* stream);
AXR_API axr_status axr_pot_attend_decode(const float* q, const uint8_t* codes, const uint16_t* alpha,
                                         const uint16_t* v, const int32_t* seq_lens, int B, int Hq, int Hkv, int T,
                                         int Tcap, int d, int E, int M, float scale, float* out, void* workspace,
                                         size_t ws_bytes, void* stream);

/* Bytes of workspace for axr_select_signs with these sizes. */
AXR_API size_t axr_select_workspace_bytes(int n_layers, int n_seq, int n_tok, int Hq, int Hkv, int d, int n_cand);

/*
 * axr_select_signs -- one-time, gradient-free sign-pattern selection (AXELRAM Key Points, 4th item; Abstract:
 * candidates scored on a few calibration samples, no hardware cost).  Objective per candidate s^(c): the mean over
 * every (layer, sequence, query head, position, coordinate) of (o_quant - o_ref)^2, where o_ref is unquantized
 * softmax attention (computed once in fp64) and o_quant the same attention with every key written through
 * axr_write_keys' path with signs s^(c) (values unquantized).  Softmax scale 1/sqrt(d); causal != 0 lets
 * position i see keys 0..i only.
 *   q [dev] [n_layers, n_seq, Hq, n_tok, d] f32;  k, v [dev] [n_layers, n_seq, Hkv, n_tok, d] fp16 (q and v
 *   16-byte aligned for d >= 64, where the candidate attention runs on the tensor cores: q and the reconstructed keys
 *   as hi and lo fp16 planes, three products a step, the weights split the same way against the fp16 values, fp32
 *   accumulation; d = 8 runs in fp32 on the CUDA cores);
 *   candidates [dev] [n_cand, d] int8 (+-1);  mse_out [dev] out [n_cand] f64;
 *   best_out [dev] out, one int32: the first index of the minimum of mse_out;
 *   workspace [dev] >= axr_select_workspace_bytes(...) bytes, 16-aligned.
 * Errors: AXR_EINVAL, AXR_EUNSUPPORTED (d not in {8, 64, 128}, b, G), AXR_EWORKSPACE, AXR_ECUDA.
 */
AXR_API axr_status axr_select_signs(const float* q, const uint16_t* k, const uint16_t* v, int n_layers, int n_seq, int n_tok,
                            int Hq, int Hkv, int d, int bits, const int8_t* candidates, int n_cand, int causal,
                            double* mse_out, int32_t* best_out, void* workspace, size_t ws_bytes, void* stream);

/*
 * axr_select_signs_per_layer -- the same one-time selection with one sign vector per layer.  The pages trace the
 * sign sensitivity to layer-wise norm heterogeneity (AXELRAM Abstract; Key Points, 3rd and 4th items): a pattern
 * that suits the high-norm layers need not suit the others, and the write path takes its sign vector per call,
 * so a model may hold one per layer.  Objective of candidate c for layer l: the mean over every (sequence, query
 * head, position, coordinate) of layer l of (o_quant - o_ref)^2, with o_quant, o_ref and the causal rule as in
 * axr_select_signs.  The mean over layers of mse_layers_out[:, c] equals axr_select_signs' mse_out[c].
 *   inputs and workspace as axr_select_signs (the same axr_select_workspace_bytes);
 *   mse_layers_out [dev] out [n_layers, n_cand] f64;
 *   best_layers_out [dev] out [n_layers] int32: per layer the first index of the minimum of its row;
 *   mse_parts_out [dev] out [n_layers, n_seq, n_cand] f64, the MSE of each (layer, calibration sequence), or NULL.
 * Errors: as axr_select_signs.
 */
AXR_API axr_status axr_select_signs_per_layer(const float* q, const uint16_t* k, const uint16_t* v, int n_layers,
                                              int n_seq, int n_tok, int Hq, int Hkv, int d, int bits,
                                              const int8_t* candidates, int n_cand, int causal,
                                              double* mse_layers_out, int32_t* best_layers_out,
                                              double* mse_parts_out, void* workspace, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* AXR_H_ */
