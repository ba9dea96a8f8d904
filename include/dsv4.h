/*
 * dsv4.h -- C ABI of the DeepSeek-V4 hybrid CSA/HCA attention hot path on NVIDIA B200
 * (sm_100a).
 *
 * The operations are defined on the page "CSA And HCA: Definition, State, And Cost
 * Model" (cited below as [CSA-DEF] with its section) and, for the per-query valid-count
 * idea, on pypto-lib PR #834 ("accelerate DeepSeek V4 Flash prefill sparse attention").
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor arguments are DEVICE pointers owned by the caller, densely packed,
 *    row-major, in the layout stated per argument. The library never frees, keeps or
 *    aliases them beyond the call's stream-ordered execution.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream). Every
 *    call only enqueues work; nothing synchronises the host except dsv4_check_errors.
 *  - The library allocates no device memory. Scratch space comes from a caller
 *    workspace sized by the matching *_workspace_size function.
 *  - Return value: a dsv4_status. Argument errors are detected on the host before any
 *    launch (nothing is enqueued then). Launch failures return DSV4_ERR_CUDA. Errors
 *    that only the device can see (an index outside the visible range, a bounded wait
 *    that gave up) are recorded in a per-device status word that dsv4_check_errors
 *    reads and clears; the offending element is skipped, never read out of bounds.
 *    No call aborts, traps or throws across the ABI. dsv4_last_error_message gives a
 *    human-readable reason for the last failing call on the calling thread.
 *  - Positions: query i of sequence b sits at position t = q_pos0[b] + i. Prefill uses
 *    q_pos0 = 0 and nq = n; decode uses nq = 1 and t = L_b - 1.
 *  - Pools of several sequences are stacked row-wise; sequence b's compressed entry s is
 *    row kv_row_off[b] + s.
 */
#ifndef DSV4_H
#define DSV4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum dsv4_status {
  DSV4_OK = 0,
  DSV4_ERR_INVALID_ARG = 1,    /* bad pointer, size, alignment or combination          */
  DSV4_ERR_UNSUPPORTED = 2,    /* valid request this build has no kernel for           */
  DSV4_ERR_CUDA = 3,           /* a CUDA runtime call or launch failed                 */
  DSV4_ERR_DEVICE_TIMEOUT = 4, /* a bounded device-side wait gave up (device word)     */
  DSV4_ERR_DEVICE_BOUNDS = 5,  /* an index/offset outside its range was skipped        */
  DSV4_ERR_WORKSPACE = 6       /* workspace pointer/size too small for the request     */
} dsv4_status;

typedef enum dsv4_dtype {
  DSV4_F32 = 0,   /* IEEE binary32                                                    */
  DSV4_BF16 = 1,  /* bfloat16                                                         */
  DSV4_FP4 = 2    /* e2m1 codes, 2 per byte (element 2j in the low nibble), plus one
                     E4M3 (fn) scale byte per 16 consecutive elements                 */
} dsv4_dtype;

/* Version of this ABI (incremented on any incompatible change). */
int dsv4_abi_version(void);

/* Static description of a status code. Never NULL. */
const char* dsv4_status_string(int status);

/* Reason for the last non-OK status returned on the calling thread ("" if none). */
const char* dsv4_last_error_message(void);

/* Synchronises `stream`, then reads and clears the current device's status word.
 * Returns DSV4_OK, DSV4_ERR_DEVICE_TIMEOUT, DSV4_ERR_DEVICE_BOUNDS or DSV4_ERR_CUDA. */
int dsv4_check_errors(void* stream);

/*
 * dsv4_compress -- learned compressor, [CSA-DEF] s2.1 (CSA, overlap = 1) and s2.2
 * (HCA, overlap = 0); the CSA indexer keys are a second instance ([CSA-DEF] s3.1).
 *
 * For every sequence b, entry i < floor(n/m) and channel ch, one softmax over positions
 * (per channel) of the logits Z + bias, then the weighted sum of the entry stream C:
 *   positions = block i from stream a (bias[0]) and, when overlap and i > 0, block i-1
 *   from stream b (bias[1]). For i = 0 the preceding block has zero weight. The
 *   trailing incomplete block (n mod m tokens) is never pooled.
 *
 *   dtype  DSV4_F32 or DSV4_BF16: element type of C, Z and out (math is fp32).
 *   C, Z   [B, n, S*c] with S = 1 + overlap; columns [0,c) = stream a, [c,2c) = b.
 *   bias   fp32 [S, m, c]: bias[0] = B^a, bias[1] = B^b.
 *   out    [B, floor(n/m), c] (dtype).
 *   Requires B >= 0, n >= 0, c >= 1, m >= 1, overlap in {0,1}. B*n == 0 is a no-op.
 */
int dsv4_compress(int dtype, const void* C, const void* Z, const float* bias, void* out,
                  int B, int n, int c, int m, int overlap, void* stream);

/*
 * dsv4_compress_decode -- one token of the compressor state machine of [CSA-DEF] s7
 * (steps 2-4: update the compressor state; when t + 1 is a multiple of m, emit and append
 * the completed entry) for each of B sequences. The emitted entry is the s2.1 (overlap = 1)
 * or s2.2 (overlap = 0) entry dsv4_compress computes from the whole stream; an incomplete
 * block exposes nothing.
 *
 *   dtype         DSV4_F32 or DSV4_BF16: element type of C_new, Z_new, tail and pool.
 *   C_new, Z_new  [B, S*c], S = 1 + overlap: the new token's entry and gate rows (columns
 *                 [0,c) stream a, [c,2c) stream b, as for dsv4_compress).
 *   bias          fp32 [S, m, c].
 *   tail          [B, T, 2, S*c], T = S*m, caller-owned state, updated in place: slot
 *                 p mod T holds position p's C row ([., ., 0, .]) and Z row ([., ., 1, .]).
 *                 Before the first call for a sequence whose prefix has n0 tokens, slots
 *                 p mod T for p in [max(0, n0 - T), n0) hold the prefix's rows (nothing
 *                 else is read; for n0 = 0 the tail needs no initialisation).
 *   pool          [pool_rows, c]: sequence b's entry i is row pool_row_off[b] + i.
 *   pos           int32 [B]: position t of each sequence's new token.
 * Writes pool row pool_row_off[b] + (t+1)/m - 1 when (t + 1) % m == 0, so that attention
 * of token t launched after this call sees the completed entry. Device-side errors
 * (t < 0, a pool row outside [0, pool_rows)) skip the sequence and set
 * DSV4_ERR_DEVICE_BOUNDS. Requires B >= 0, c >= 1, m >= 1, overlap in {0,1}; B == 0 is a
 * no-op.
 */
int dsv4_compress_decode(int dtype, const void* C_new, const void* Z_new, const float* bias,
                         void* tail, void* pool, const int64_t* pool_row_off, int64_t pool_rows,
                         const int32_t* pos, int B, int c, int m, int overlap, void* stream);

/*
 * dsv4_ring_write -- [CSA-DEF] s7 step 1: each sequence's new shared-KV entry overwrites
 * slot t mod R of its local ring (the layout dsv4_hybrid_sparse_attn reads: position j in
 * slot j mod R).
 *
 *   dtype   DSV4_F32 or DSV4_BF16.
 *   kv_new  [B, c]; local [B, R, c]; pos int32 [B] (t; t < 0 skips the sequence and sets
 *           DSV4_ERR_DEVICE_BOUNDS).
 * Requires B >= 0, R >= 1, c >= 1; B == 0 is a no-op.
 */
int dsv4_ring_write(int dtype, const void* kv_new, void* local, int R, const int32_t* pos,
                    int B, int c, void* stream);

/*
 * dsv4_decode_state -- a token's whole state update ([CSA-DEF] s7 steps 1-4 for every layer)
 * in one launch: each job is a dsv4_ring_write or a compressor token of one layer for the same
 * B sequences at positions pos, with the arguments, results, device-side errors and
 * requirements of those calls: DSV4_JOB_COMPRESS as dsv4_compress_decode (entry into a pool of
 * dtype), DSV4_JOB_COMPRESS_FP8 as dsv4_compress_decode_fp8 (the main-KV FP8 entry),
 * DSV4_JOB_COMPRESS_FP4 emits the entry rounded to dtype and quantised exactly as
 * dsv4_quantize_fp4 quantises that row (the FP4 index-key pool; c % 16 == 0, codes 8-byte
 * aligned). Jobs run concurrently, so two jobs must not write the same memory. At most
 * DSV4_DECODE_MAX_JOBS jobs; the job array is read on the host before the call returns.
 */
#define DSV4_DECODE_MAX_JOBS 32
typedef enum dsv4_job_kind {
  DSV4_JOB_RING = 0,          /* x_new = kv_new [B, c], out = local ring [B, R, c] */
  DSV4_JOB_COMPRESS = 1,      /* x_new = C_new, z_new = Z_new [B, S*c], bias [S, m, c],
                                 tail [B, S*m, 2, S*c], out = pool [pool_rows, c] */
  DSV4_JOB_COMPRESS_FP8 = 2,  /* as 1; out = FP8 codes [pool_rows, c - rope_dims], out_scales =
                                 fp32 [pool_rows, (c - rope_dims)/64], out_rope = bf16
                                 [pool_rows, rope_dims] */
  DSV4_JOB_COMPRESS_FP4 = 3   /* as 1; out = e2m1 codes [pool_rows, c/2], out_scales = E4M3
                                 bytes [pool_rows, c/16] */
} dsv4_job_kind;
typedef struct dsv4_decode_job {
  int kind;              /* dsv4_job_kind */
  int c;                 /* channels of the entry */
  int m;                 /* compressor: ratio */
  int overlap;           /* compressor: 1 = CSA (two streams), 0 = HCA */
  int R;                 /* ring: slots per sequence */
  int rope_dims;         /* FP8: bf16 RoPE channels at the end of the entry */
  const void* x_new;
  const void* z_new;
  const float* bias;
  void* tail;
  void* out;
  void* out_scales;
  void* out_rope;
  const int64_t* pool_row_off;
  int64_t pool_rows;
} dsv4_decode_job;
int dsv4_decode_state(int dtype, const dsv4_decode_job* jobs, int n_jobs, const int32_t* pos,
                      int B, void* stream);

/*
 * dsv4_quantize_fp4 -- FP4 indexer operands ([CSA-DEF] s3.1 and s8: the indexer Q/K are
 * multiplied in 4-bit floating point). Per group of 16 consecutive elements of a row:
 *   scale = RNE_E4M3(amax / 6) (fp32 quotient, saturating at 448);
 *   code  = RNE_e2m1(x / scale) (fp32 quotient, saturating at +-6; IEEE sign, so a
 *           negative value that rounds to zero is code 0x8); a zero scale gives codes 0.
 *
 *   x       bf16 [rows, cols]; cols % 16 == 0; x 16-byte aligned.
 *   codes   uint8 [rows, cols/2] (element 2j in the low nibble of byte j).
 *   scales  uint8 [rows, cols/16] (E4M3 fn bytes).
 */
int dsv4_quantize_fp4(const void* x, uint8_t* codes, uint8_t* scales, int64_t rows, int cols,
                      void* stream);

/* Bytes of workspace dsv4_index_topk needs for a bf16 / fp32 request: per chunk of queries
 * (at most 256 MiB of rows) the fp32 score rows (4 * round4(max_entries) bytes each) and,
 * for rows longer than 16384 entries, a top-k region per row: with at most 1024 rows in the
 * request and k <= 4096 the threshold top-k's (a 2048-bin histogram and counters, the
 * entries above the threshold and up to 8192 boundary candidates: 8448 bytes +
 * round256(4k) + 64 KiB), otherwise the
 * per-segment candidates (8k bytes per 16384-entry segment). Each of the two regions is
 * rounded up to 256 bytes. A smaller workspace makes smaller chunks; a larger one is not
 * used.
 * max_entries = the largest number of completed entries any query of the request can see. */
size_t dsv4_index_topk_workspace_size(int B, int nq, int max_entries, int k);

/* The same for any operand type. FP4 operands at H_I = 64, c_I = 128 are scored on the
 * tensor cores after an exact expansion of the chunk's q^I rows in the workspace and, for
 * requests with several queries per sequence, of K^I to bf16 (ki_rows x c_I) too; one query
 * per sequence (decode) with 16-byte aligned KI and KI_scales and at least 130 key rows reads
 * the FP4 key pool itself and expands it inside the score kernel. This size includes the room
 * for the K^I expansion either way. With less room (or with scores_out and a workspace too
 * small for the expansion of every query) FP4 is scored on CUDA cores. */
size_t dsv4_index_topk_workspace_size_ex(int qdtype, int B, int nq, int H_I, int c_I,
                                         int max_entries, int k, int64_t ki_rows);

/*
 * dsv4_index_topk -- lightning-indexer score and per-query TopK, [CSA-DEF] s3.1:
 *   I_{t,s} = sum_h w_{t,h} * ReLU(qI_{t,h} . KI_s)    for s < floor((t+1)/m)
 *   S_t     = TopK_s(I_{t,s}, k)
 * Scores are accumulated in fp32. k_eff = min(k, floor((t+1)/m)) entries are returned,
 * as a set listed in ascending entry order (ties at the k-th score go to the lower entry
 * index); slots k_eff..k-1 hold -1.
 *
 *   qdtype     DSV4_F32, DSV4_BF16 or DSV4_FP4: element type of qI and KI.
 *   qI         [B, nq, H_I, c_I] (FP4: codes [B*nq*H_I, c_I/2] + qI_scales [.., c_I/16]).
 *   w          fp32 [B, nq, H_I] head weights.
 *   KI         [ki_rows, c_I] keys of all sequences (FP4: codes + KI_scales).
 *   kv_row_off int64 [B] first KI row of each sequence.
 *   q_pos0     int32 [B] position of query 0 of each sequence.
 *   idx        int32 [B, nq, k] output; counts int32 [B, nq] output (= k_eff).
 *   scores_out optional fp32 [B, nq, scores_ld]: if non-NULL receives I_{t,s} for
 *              s < floor((t+1)/m) (other columns untouched); scores_ld >= max_entries.
 *   workspace  device scratch of >= dsv4_index_topk_workspace_size(...) bytes (256-byte
 *              aligned), or NULL/0 when scores_out is given.
 *   Requires c_I % 16 == 0 (FP4: c_I % 64 == 0), H_I >= 1, m >= 1, 0 <= k <= 4096.
 *   Device-checked: kv_row_off[b] + floor((q_pos0[b]+nq)/m) <= ki_rows.
 */
int dsv4_index_topk(int qdtype, const void* qI, const uint8_t* qI_scales, const float* w,
                    const void* KI, const uint8_t* KI_scales, int64_t ki_rows,
                    const int64_t* kv_row_off, const int32_t* q_pos0,
                    int B, int nq, int H_I, int c_I, int m, int k, int max_entries,
                    int32_t* idx, int32_t* counts, float* scores_out, int64_t scores_ld,
                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * dsv4_index_topk_noalloc -- the same indexer score + TopK as dsv4_index_topk, for
 * callers that cannot allocate device memory (a runtime that only hands out buffers it
 * planned in advance, plain C code without a device allocator, or a serving loop that
 * must not call cudaMalloc because it can synchronise the device and fail under
 * fragmentation). The pages have no counterpart of this entry point; it is a property
 * of this library's interface only.
 *
 * Instead of a caller workspace it uses a fixed 8 MiB scratch array compiled into the
 * library (a __device__ array that every GPU which loads the library keeps until the
 * process exits). It allocates nothing: no cudaMalloc, no cudaFree, no allocating
 * library routine. Arguments and outputs are those of dsv4_index_topk without
 * scores_out, scores_ld, workspace and workspace_bytes.
 *   - max_entries above 2,097,152 (one score row larger than the scratch) is rejected
 *     with DSV4_ERR_INVALID_ARG before anything is enqueued.
 *   - Queries are processed in chunks whose score rows fit in the scratch; long rows
 *     (more than 16384 entries) also need their top-k region there and get smaller chunks.
 *   - DSV4_FP4 operands of requests with several queries per sequence are scored on the
 *     tensor cores only while the exact bf16 expansion of the whole key pool (256 bytes per
 *     key row at c_I = 128) fits in the scratch beside at least one score row: above roughly
 *     32,000 key rows such requests are scored on CUDA cores instead (same results up to
 *     fp32 rounding order, lower throughput). One query per sequence (decode) needs no such
 *     room: the score kernel expands the FP4 keys it streams.
 *   - The first call on a device looks up the array's device address (once per device,
 *     with that device current); make that first call before any stream capture.
 *   - Every call on a device shares the one array. The scratch holds score rows that
 *     each call writes before it reads them, so nothing needs to start at zero, but two
 *     calls whose work overlaps on the GPU (different streams, no ordering between them)
 *     race on the array and may return wrong indices. Order such calls on one stream.
 */
int dsv4_index_topk_noalloc(int qdtype, const void* qI, const uint8_t* qI_scales,
                            const float* w, const void* KI, const uint8_t* KI_scales,
                            int64_t ki_rows, const int64_t* kv_row_off, const int32_t* q_pos0,
                            int B, int nq, int H_I, int c_I, int m, int k, int max_entries,
                            int32_t* idx, int32_t* counts, void* stream);

/*
 * dsv4_hybrid_sparse_attn -- shared-KV MQA over one candidate list per query,
 * [CSA-DEF] s3.2, s4, s5.1-s5.3:
 *   A_t = {pool[s] : s in S_t}            (CSA: idx/counts from dsv4_index_topk)
 *       or {pool[s] : s < floor((t+1)/m)} (HCA dense read: idx == NULL)
 *     ++ {local[j mod R] : max(0,t-w+1) <= j <= t}
 *   z_{h,j} = scale * q_{t,h} . A_j ;  a_{h,j} = exp(z_{h,j}) / (sum_u exp(z_{h,u}) + exp(sink_h))
 *   O_{t,h} = sum_j a_{h,j} A_j ;       LSE_{t,h} = log(sum_u exp(z_{h,u}) + exp(sink_h))
 * Each candidate row is both key and value for every head. The sink term is omitted
 * when sink == NULL. Softmax and accumulation are fp32.
 *
 *   dtype      DSV4_F32 or DSV4_BF16: element type of Q, pool, local and O.
 *   Q          [B, nq, H, c].
 *   pool       [pool_rows, c] compressed entries of all sequences; kv_row_off int64 [B].
 *   idx        int32 [B, nq, k] selected entries (first counts[b,i] valid) or NULL.
 *              With k == 0 and a non-NULL idx (never read) the list is the window only.
 *   counts     int32 [B, nq] or NULL (required when idx != NULL).
 *   local      [B, R, c] uncompressed local entries; position j lives in slot j mod R
 *              (prefill: R = n; decode ring: R >= w).
 *   q_pos0     int32 [B].
 *   m          compression ratio used for the dense read (idx == NULL); ignored otherwise.
 *   w          local window, >= 1 (so every candidate list is non-empty).
 *   sink       fp32 [H] or NULL.  scale: logit scale (1/sqrt(c) in the model).
 *   O          [B, nq, H, c] (dtype) output.  lse: fp32 [B, nq, H] output or NULL.
 *   workspace  device scratch (256-byte aligned) of workspace_bytes, or NULL / 0. When the
 *              request has fewer (query, 64-head group) items than the device has SMs
 *              (decode), the tensor-core path splits each candidate list into up to 8
 *              parts that run on separate SMs and are merged afterwards (exact up to fp32
 *              rounding order); the parts live here. Without workspace nothing is split.
 *              dsv4_hybrid_sparse_attn_workspace_size gives the size that allows all splits.
 *   Requires c % 8 == 0 for bf16 (c % 4 for fp32), R >= min(w, q_pos0+nq).
 *   Device-checked: every used idx value in [0, floor((t+1)/m_csa)) when `m` > 0, and
 *   every pool row < pool_rows; out-of-range candidates are skipped and flagged.
 */
int dsv4_hybrid_sparse_attn(int dtype, const void* Q, const void* pool, int64_t pool_rows,
                            const int64_t* kv_row_off, const int32_t* idx,
                            const int32_t* counts, int k, const void* local, int R,
                            const int32_t* q_pos0, int B, int nq, int H, int c, int m, int w,
                            const float* sink, float scale, void* O, float* lse,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * dsv4_hybrid_sparse_attn_rope -- dsv4_hybrid_sparse_attn with the output side of the
 * [CSA-DEF] s5.2 contract fused in: the last rope_dims channels of every output row O_{t,h}
 * are rotated back by the query's position t (inverse RoPE; the channel pairing and angles
 * of dsv4_norm_rope) before O is stored. Q, pool and local hold rows that dsv4_norm_rope
 * (or an upstream kernel) already normalised and rotated: the query at t, compressed entry
 * s at m*s (m' for HCA), local entry j at j. LSE is unchanged by the rotation.
 *   rope_dims  even, 0 <= rope_dims <= c (0: same as dsv4_hybrid_sparse_attn). The tensor-core
 *              path takes rope_dims = 64 at c = 512; other values run on CUDA cores.
 * All other arguments, layouts and errors are those of dsv4_hybrid_sparse_attn.
 */
int dsv4_hybrid_sparse_attn_rope(int dtype, const void* Q, const void* pool, int64_t pool_rows,
                                 const int64_t* kv_row_off, const int32_t* idx,
                                 const int32_t* counts, int k, const void* local, int R,
                                 const int32_t* q_pos0, int B, int nq, int H, int c, int m, int w,
                                 const float* sink, float scale, void* O, float* lse,
                                 void* workspace, size_t workspace_bytes, int rope_dims,
                                 void* stream);

/*
 * dsv4_norm_rope -- [CSA-DEF] s5.2: RMS normalisation of attention rows and rotary position
 * embedding of their last `rope` channels, in place. For each row r of x [rows, c]:
 *   norm = 1:  x_r <- x_r / sqrt(mean(x_r^2) + eps)      (fp32, no learned gain)
 *   then channel pair i (channels c - rope + 2i, c - rope + 2i + 1) is rotated by the angle
 *   p * 10000^(-2i / rope), p = pos[r / rows_per_pos] (inverse = 1: by minus that angle).
 * The angle is formed and reduced in double precision; the result is rounded once to dtype.
 * Uses: query heads (rows_per_pos = H, pos = query positions), compressed entries (pos = m*s),
 * local entries (pos = j), and the inverse rotation of an output (norm = 0, inverse = 1).
 *   dtype  DSV4_F32 or DSV4_BF16.   pos  int32 [ceil(rows / rows_per_pos)], >= 0 (a negative
 *   position skips its rows and sets DSV4_ERR_DEVICE_BOUNDS).
 *   Requires rows >= 0, rows_per_pos >= 1, c >= 1, 0 <= rope <= c, rope even, eps >= 0.
 */
int dsv4_norm_rope(int dtype, void* x, const int32_t* pos, int64_t rows, int rows_per_pos, int c,
                   int rope, int norm, int inverse, float eps, void* stream);

/*
 * Production main-KV entries, [CSA-DEF] s8 precision table ("main KV: 448 FP8 + 64 BF16 RoPE
 * channels"). The pages leave the FP8 scale metadata open; this library keeps one fp32 scale
 * per 64 consecutive FP8 channels. A pool of `rows` entries of c channels whose last `rope`
 * channels carry RoPE ((c - rope) % 64 == 0) is three caller-owned arrays:
 *   codes   uint8 [rows, c - rope]  E4M3 (fn) bytes, sign << 7 | magnitude code
 *   scales  fp32  [rows, (c - rope) / 64]
 *   rope    bf16  [rows, rope]
 * V4 shapes: c = 512, rope = 64 -> 448 + 28 + 128 = 604 bytes per entry (bf16: 1024).
 */

/* dsv4_quantize_main_kv -- rows x [rows, c] (dtype F32 or BF16) into the FP8 entry format:
 * per 64-channel group scale = fp32(amax / 448), code = RNE_E4M3(fp32(x / scale)) saturating
 * at 448 with the IEEE sign (a negative value that rounds to zero is 0x80); a zero scale gives
 * zero codes; the RoPE channels are rounded to bf16. codes 2-byte aligned, x 4-byte aligned. */
int dsv4_quantize_main_kv(int dtype, const void* x, uint8_t* codes, float* scales, void* rope,
                          int64_t rows, int c, int rope_dims, void* stream);

/* dsv4_dequantize_main_kv -- FP8 entries back to bf16 rows out [rows, c]: each FP8 channel is
 * RNE_bf16(E4M3 value * scale) (the product carries up to 28 significant bits, so it is
 * rounded once), the RoPE channels are copied. */
int dsv4_dequantize_main_kv(const uint8_t* codes, const float* scales, const void* rope,
                            void* out, int64_t rows, int c, int rope_dims, void* stream);

/* dsv4_compress_decode_fp8 -- dsv4_compress_decode with the completed entry emitted in the
 * FP8 entry format (quantise on emission, [CSA-DEF] s7 step 4 + s8): the entry is rounded to
 * dtype and then quantised exactly as dsv4_quantize_main_kv would quantise that row, into
 * row pool_row_off[b] + (t+1)/m - 1 of (codes, scales, rope). Tail, positions, errors and
 * requirements are those of dsv4_compress_decode, plus (c - rope_dims) % 64 == 0 and
 * c <= 12288. */
int dsv4_compress_decode_fp8(int dtype, const void* C_new, const void* Z_new, const float* bias,
                             void* tail, uint8_t* codes, float* scales, void* rope,
                             int rope_dims, const int64_t* pool_row_off, int64_t pool_rows,
                             const int32_t* pos, int B, int c, int m, int overlap, void* stream);

/* Workspace bytes of dsv4_hybrid_sparse_attn_fp8: the gathered bf16 rows (B*k*c*2), their
 * candidate lists and row offsets, and the split-list partials. */
size_t dsv4_hybrid_sparse_attn_fp8_workspace_size(int B, int H, int c, int k);

/*
 * dsv4_hybrid_sparse_attn_fp8 -- decode attention (one query per sequence, t = q_pos0[b])
 * over a compressed pool stored as FP8 entries: the selected entries idx[b, 0..counts[b])
 * are read in the FP8 format (604 bytes per V4 entry instead of 1024), expanded to bf16 rows
 * as in dsv4_dequantize_main_kv next to the query, and attended with the bf16 local ring
 * exactly as dsv4_hybrid_sparse_attn attends bf16 rows (selected entries, then the window,
 * one softmax, sink, LSE). Q, local, O: bf16 [B, H, c], [B, R, c], [B, H, c]; lse fp32 [B, H]
 * or NULL. A selection outside [0, floor((t+1)/m)) or beyond pool_rows is skipped and
 * reported (DSV4_ERR_DEVICE_BOUNDS). workspace: >= dsv4_hybrid_sparse_attn_fp8_workspace_size
 * bytes, 256-byte aligned (DSV4_ERR_WORKSPACE otherwise). Requires k >= 1, w >= 1, R >= w,
 * (c - rope_dims) % 64 == 0.
 */
int dsv4_hybrid_sparse_attn_fp8(const void* Q, const uint8_t* pool_codes, const float* pool_scales,
                                const void* pool_rope, int64_t pool_rows,
                                const int64_t* kv_row_off, const int32_t* idx,
                                const int32_t* counts, int k, const void* local, int R,
                                const int32_t* q_pos0, int B, int H, int c, int rope_dims, int m,
                                int w, const float* sink, float scale, void* O, float* lse,
                                void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes for dsv4_hybrid_sparse_attn to split every candidate list of a request of
 * B x nq queries with H heads of dimension c (0 when no split would be used). */
size_t dsv4_hybrid_sparse_attn_workspace_size(int B, int nq, int H, int c);

#ifdef __cplusplus
}
#endif

#endif /* DSV4_H */
