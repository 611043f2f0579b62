/*
 * csa.h -- C ABI of libcsa.so: the CSA / HCA hybrid-attention hot path on
 * NVIDIA B200 (sm_100a).
 *
 * Sources (page title, then section):
 *   [HA] "DeepSeek-V4 混合注意力：从压缩记忆到百万上下文"
 *   [P1] "揭秘DeepSeek-V4-Pro-MXFP4稀疏注意力：哈希索引与DSA如何撑起1M超长上下文？"
 *   [P2] "解密DeepSeek-V4-Flash-NVFP4的混合注意力机制：压缩稀疏注意力如何提升长文本处理能力"
 *
 * Conventions for every entry point:
 *   - Tensors are dense, row-major ("C order"), in device memory, with the
 *     shapes stated below.  Pointers to bf16 / fp32 / e4m3 data must be
 *     16-byte aligned; the innermost dimension must be a multiple of 8.
 *   - The caller owns every buffer, including workspaces.  The library never
 *     allocates, frees or synchronises; every call only enqueues kernels on
 *     `stream` (a cudaStream_t; NULL = legacy default stream) and returns.
 *   - Arguments are validated on the host before anything is launched.  On
 *     CSA_ERR_INVALID or CSA_ERR_UNSUPPORTED nothing is launched and no output
 *     is touched.  CSA_ERR_CUDA reports a launch failure (cudaGetLastError).
 *   - Kernels never wait without bound: a wait that runs out records
 *     CSA_ERR_TIMEOUT in a device status word that csa_poll_status() returns.
 *   - dtype codes: CSA_F32 (fp32), CSA_BF16 (bfloat16), CSA_E4M3 (OCP FP8 e4m3,
 *     one byte per element), CSA_BF16_KV8 (attention only: bf16 q / swa_kv / out,
 *     memory rows kv stored as mixed-precision entries, see csa_quantize_kv8).
 */
#ifndef CSA_H_
#define CSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  CSA_OK = 0,
  CSA_ERR_INVALID = 1,     /* bad pointer, size, alignment or dtype code */
  CSA_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. D not 128/256/512) */
  CSA_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
  CSA_ERR_TIMEOUT = 4      /* a kernel gave up a bounded wait (see csa_poll_status) */
};

enum { CSA_F32 = 0, CSA_BF16 = 1, CSA_E4M3 = 2, CSA_BF16_KV8 = 3, CSA_MXFP4 = 4 };

#define CSA_INDEX_HEADS 64   /* index heads per query ([HA] §2 table, §4.2) */
#define CSA_INDEX_DIM 128    /* dims per index head */
#define CSA_SWA_WINDOW 128   /* SWA tokens per query ([HA] §6; [P1] window_size 128) */
#define CSA_MAX_TOPK 2048
#define CSA_MAX_SHARDS 16    /* GPUs one sequence's entries may be sharded over */

/* Human-readable name of a status code (static string). */
const char *csa_status_string(int status);

/* Library ABI version (major * 100 + minor). */
int csa_version(void);

/*
 * csa_n_valid -- how many compressed entries each query may see ([HA] §6: a query at
 * absolute position t attends to entry i only once its block of `ratio` raw tokens
 * is complete, (i + 1) * ratio <= t + 1):
 *   n_valid[i] = clamp(floor((q_pos[i] + 1) / ratio) - lo, 0, hi - lo)   (0 for q_pos[i] < 0)
 * for a device that holds the sequence's entries [lo, hi); a device that holds all N
 * entries passes lo = 0, hi = N.  The result is the n_valid argument of
 * csa_index_scores, csa_topk and csa_topk_select.
 *   q_pos   : [count] int64 absolute positions (device)
 *   n_valid : [count] int32 (device)
 *   ratio >= 1, 0 <= lo <= hi, hi - lo <= INT32_MAX; CSA_ERR_INVALID otherwise.
 */
int csa_n_valid(const int64_t *q_pos, int64_t count, int ratio, int64_t lo, int64_t hi, int32_t *n_valid,
                void *stream);

/*
 * csa_compress -- token-level Compressor ([HA] §4.1 for ratio 4, §5 for 128).
 *
 * ratio 4 (CSA, overlapped two-branch pooling):
 *   out[b,i,j] = sum_{r<2m} alpha_r * V_r,  alpha = softmax_r(Zcat_r) per channel j,
 *   with positions r = 0..3 the b-branch rows (i-1)*4+r of C_b / Z_b and
 *   r = 4..7 the a-branch rows i*4+(r-4) of C_a / Z_a.  For entry 0 the
 *   b-branch rows are prev_Cb / prev_Zb (the b branch of the 4 raw rows just
 *   before this chunk), or absent when those are NULL.
 * ratio 128 (HCA, non-overlapped): out[b,i,j] = sum_{r<128} beta_r * C[b,128i+r,j],
 *   beta = softmax_r(Z[b,128i+r,j]); C_b, Z_b, prev_* must be NULL.
 *
 *   C_a, Z_a (C, Z for ratio 128), C_b, Z_b : [B, L, c], dtype in_dtype (F32|BF16)
 *   prev_Cb, prev_Zb : [B, 4, c] in_dtype, or both NULL
 *   out   : [B, L/ratio, c], dtype out_dtype (F32|BF16); a partial trailing block
 *           (L % ratio rows) produces no entry
 *   c     : multiple of 8 (ratio 4) or of 128 (ratio 128)
 * Softmax and sums in fp32.  Streaming, HBM-bound.
 */
int csa_compress(const void *C_a, const void *C_b, const void *Z_a, const void *Z_b, const void *prev_Cb,
                 const void *prev_Zb, int B, int64_t L, int c, int ratio, int in_dtype, int out_dtype, void *out,
                 void *stream);

/*
 * csa_compress_index_keys -- a step's new index-key entries, written straight into the
 * indexer's caches in one launch ([HA] §4.1 compressor over the index keys; §7: the
 * Indexer compresses its own keys; §4.2: its QK runs in low precision):
 *   entry i of sequence b = csa_compress(ratio 4) of the c = 128 index-key channels, bit
 *   for bit, rounded to bf16 and stored at row pos0 + i of kI [B, n_cap, 128] bf16;
 *   with k8 != NULL that stored bf16 row is also quantised exactly as
 *   csa_quantize_e4m3_hadamard (hadamard != 0) or csa_quantize_e4m3 (hadamard == 0)
 *   quantises it, into row pos0 + i of k8 [B, n_cap, 128] e4m3 and k_scale [B, n_cap] fp32.
 *   C_a, C_b, Z_a, Z_b : [B, L, 128] in_dtype (F32|BF16); prev_Cb, prev_Zb : [B, 4, 128] or
 *   both NULL (see csa_compress); L / 4 entries per sequence (a partial block makes none);
 *   0 <= pos0, pos0 + L/4 <= n_cap.  k8 and k_scale are both NULL or both set.
 *   Pointers 16-byte aligned.  CSA_ERR_INVALID otherwise.
 */
int csa_compress_index_keys(const void *C_a, const void *C_b, const void *Z_a, const void *Z_b, const void *prev_Cb,
                            const void *prev_Zb, int B, int64_t L, int in_dtype, int hadamard, int64_t n_cap,
                            int64_t pos0, void *kI, uint8_t *k8, float *k_scale, void *stream);

/*
 * csa_quantize_e4m3 -- per-row symmetric e4m3 quantisation for the
 * low-precision index QK path ([HA] §4.2 and §9: the index QK runs in low
 * precision; this library's variant is e4m3 with a per-row scale).
 *   x      : [rows, cols] F32 or BF16 (x_dtype)
 *   codes  : [rows, cols] uint8 e4m3, code = RN-even(x / scale), saturating to +-448
 *   scale  : [rows] fp32, scale = amax(|x_row|) / 448 (IEEE fp32 division); 1 for an all-zero row
 * Use it for index keys ([B*N, 128] -> k_scale [B, N]) and index queries
 * ([B*T*64, 128] -> q_scale [B, T, 64]).
 */
int csa_quantize_e4m3(const void *x, int x_dtype, int64_t rows, int cols, uint8_t *codes, float *scale,
                      void *stream);

/*
 * csa_quantize_e4m3_hadamard -- csa_quantize_e4m3 of the Hadamard-rotated rows
 * ([P1], the Indexer paragraph: the index query is Hadamard-rotated before it is
 * scored against the compressed keys).  Give the index keys the same rotation: the
 * rotation is orthonormal, so <Rq, Rk> = <q, k> and the scores keep their value,
 * while channels that dominate q and k are spread over all dims before the e4m3
 * rounding.  The exact bf16 rerank (csa_topk_select, csa_index_rerank) takes the
 * UNROTATED bf16 operands.
 *   y = H_n x / sqrt(n) per row, H_n the Walsh-Hadamard matrix in Sylvester (natural)
 *       order, H[i][j] = (-1)^popcount(i & j); the sums are taken in fp64 (exact while
 *       a row spans at most 53 - 8 - log2(n) binary orders for BF16 input, 53 - 24 -
 *       log2(n) for F32), times 1/sqrt(n) in fp64, rounded to fp32; a zero is +0
 *   then codes / scale exactly as csa_quantize_e4m3 computes them from y.
 *   x     : [rows, cols] F32 or BF16 (x_dtype), 16-byte aligned;  cols = 32, 64, 128 or 256
 *   codes : [rows, cols] uint8 e4m3, 16-byte aligned;  scale : [rows] fp32
 * NaN inputs are not supported.  Returns CSA_ERR_INVALID for any other cols or dtype,
 * or for an x or codes pointer that is not 16-byte aligned.
 */
int csa_quantize_e4m3_hadamard(const void *x, int x_dtype, int64_t rows, int cols, uint8_t *codes, float *scale,
                               void *stream);

/*
 * csa_quantize_mxfp4 -- MXFP4 operands for the FP4 index QK ([HA] §2 table and §4.2:
 * the index QK path runs in FP4; the format is this library's reading, OCP MXFP4).
 *   per block of 32 consecutive values of a row: X = 2^(floor(log2 amax) - 2), clamped
 *   to 2^-127 .. 2^127, X = 1 for an all-zero block; element = nearest FP4 E2M1 value
 *   of v / X (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), ties to the even mantissa,
 *   saturating at 6; the sign is kept (also for zero).
 *   hadamard != 0: the rows are first rotated as in csa_quantize_e4m3_hadamard (the
 *   rounded fp32 rotated values are the v above).
 *   x      : [rows, cols] F32 or BF16 (x_dtype), 16-byte aligned;  cols = 32, 64, 128 or 256
 *   codes  : [rows, cols/2] bytes, 16-byte aligned; value 2j in the low nibble, 2j+1 in
 *            the high nibble (sign bit 3, exponent bits 2..1, mantissa bit 0)
 *   scales : [rows, cols/32] E8M0 bytes (X = 2^(byte - 127))
 * NaN inputs are not supported.  Returns CSA_ERR_INVALID for any other cols or dtype,
 * or for an x or codes pointer that is not 16-byte aligned.
 */
int csa_quantize_mxfp4(const void *x, int x_dtype, int64_t rows, int cols, int hadamard, uint8_t *codes,
                       uint8_t *scales, void *stream);

/*
 * csa_quantize_mxfp4_sf128 -- csa_quantize_mxfp4 of rows of 128 values (cols = 128) with the
 * E8M0 scales written in the layout the block-scaled tensor-core MMA reads, the operands of
 * csa_index_scores with dtype CSA_MXFP4: the rows of each of `batches` batches (rows_per_batch
 * each) in tiles of 128; tile j of batch b is one 512-byte atom at byte (b * ceil(rpb/128) + j) *
 * 512, holding row i = 128 j + m0 + 32 m1 (m0 < 32, m1 < 4) at byte 16 m0 + 4 m1 + s for its
 * scale s < 4 (dims 32 s .. 32 s + 31).  Bytes of rows past rows_per_batch are not written.
 *   codes : [batches * rows_per_batch, 64] bytes as csa_quantize_mxfp4; sf : 16-byte aligned,
 *   csa_mxfp4_sf128_bytes(batches, rows_per_batch) bytes.
 */
size_t csa_mxfp4_sf128_bytes(int64_t batches, int64_t rows_per_batch);
int csa_quantize_mxfp4_sf128(const void *x, int x_dtype, int64_t batches, int64_t rows_per_batch, int hadamard,
                             uint8_t *codes, uint8_t *sf, void *stream);

/*
 * csa_index_scores -- Lightning Indexer ([HA] §4.2):
 *   scores[b,t,i] = sum_{h<64} w[b,t,h] * ReLU(<qI[b,t,h,:], kI[b,i,:]>)   for i < n_valid[b,t]
 *   scores[b,t,i] = -inf                                                   for n_valid[b,t] <= i < N
 * with dequantised values (code * scale) when dtype = CSA_E4M3, and (code * 2^(e - 127)) per
 * block of 32 dims when dtype = CSA_MXFP4 (the FP4 index QK of [HA] §2 / §4.2).
 *   qI      : [B, T, 64, 128] dtype
 *   q_scale : [B, T, 64] fp32 (E4M3 only, else NULL)
 *   w       : [B, T, 64] fp32
 *   kI      : [B, N, 128] dtype   (keys shared by the 64 heads)
 *   k_scale : [B, N] fp32 (E4M3 only, else NULL)
 *   n_valid : [B, T] int32, 0 <= n_valid <= N (visible complete entries: csa_n_valid)
 *   CSA_MXFP4: qI [B, T, 64, 64] and kI [B, N, 64] packed E2M1 codes (csa_quantize_mxfp4_sf128);
 *              q_scale / k_scale are the byte arrays of their scales in the tensor-core layout
 *              (rows_per_batch T * 64 and N), 16-byte aligned.
 *   scores  : [B, T, N] fp32
 *   select_ws : NULL, or (T == 1 only) a csa_topk_select workspace: the call then
 *               also accumulates each row's 4096-bin histogram of its valid scores
 *               there, to be consumed by the next csa_topk_select on that workspace.
 * BF16 / E4M3 run on tcgen05 tensor cores (fp32 accumulation); F32 runs on
 * the fp32 FMA pipes.
 */
int csa_index_scores(const void *qI, const float *q_scale, const float *w, const void *kI, const float *k_scale,
                     int dtype, const int32_t *n_valid, int B, int T, int64_t N, float *scores, void *select_ws,
                     void *stream);

/*
 * csa_index_scores_ex -- csa_index_scores with flags (0: the same call).
 *   CSA_INDEX_KEYS_READY: the caller states that kI and k_scale were not written by the
 *     launch just before this call on `stream` (they were written earlier, or on another
 *     stream whose work this stream already waited for).  The library's kernels start
 *     their successor on the stream before they finish (programmatic dependent launch);
 *     with this flag the indexer streams its first key tiles into shared memory while
 *     its predecessor (say, the query quantiser) still runs, and waits for that launch only
 *     before it reads the queries.  Without the flag nothing is read before the wait.
 *     Giving the flag when the predecessor does write the keys is a race (stale keys).
 *   Other bits: CSA_ERR_INVALID.  T = 1 decode launches (B x 1 queries) are the intended use.
 */
#define CSA_INDEX_KEYS_READY 1u
int csa_index_scores_ex(const void *qI, const float *q_scale, const float *w, const void *kI, const float *k_scale,
                        int dtype, const int32_t *n_valid, int B, int T, int64_t N, float *scores, void *select_ws,
                        unsigned flags, void *stream);

/*
 * csa_index_topk -- the indexer and the top-k in one call, without writing the score
 * matrix ([HA] §4.2: a cheap scan of every compressed key, the expensive work only for
 * the top-k; the chunked-prefill shapes).  The result equals, index for index,
 * csa_index_scores followed by csa_topk on the same arguments (the same kernel computes
 * every score, so the values are bit-identical).  Steps, in stream order:
 *   1. every 16th key of each sequence (and its scale) is gathered and scored;
 *   2. per row, the r-th largest sampled score (r = max(48, ceil(4k / 16))) is the
 *      row's threshold: about 16r keys are expected at or above it, and at least r are
 *      (a row with r samples or fewer takes every valid key);
 *   3. the indexer scores every key; each valid score at or above its row's threshold
 *      goes into the row's candidate list (score key, index); nothing else is written;
 *   4. per row with at least k and at most cap = min(8192, max(4096, 16k)) candidates, the exact
 *      top-k of the list (ties toward the lower index), ascending; other rows are
 *      counted as failed;
 *   5. a fallback, launched every time and doing nothing unless a row failed: the
 *      scores of every row into the workspace, then the row top-k of csa_topk.
 *   Arguments as csa_index_scores / csa_topk; dtype CSA_BF16 or CSA_E4M3 (others:
 *   CSA_ERR_UNSUPPORTED); k <= 1024, N <= 32768 (the fallback's row top-k holds a row in
 *   shared memory).
 *   idx         : [B, T, k] int32, ascending, -1 padded when n_valid < k.
 *   failed_rows : NULL, or one device int32 (caller-owned): the number of rows that
 *                 took the fallback (0 unless the sample misled a row's threshold or
 *                 the row is dominated by ties).
 *   workspace   : csa_index_topk_workspace_size(B, T, N, k, dtype) bytes, 256-byte
 *                 aligned, no initial contents.  It includes room for the fallback's
 *                 [B, T, N] fp32 scores, which only a failed row makes the call write.
 */
size_t csa_index_topk_workspace_size(int B, int T, int64_t N, int k, int dtype);
int csa_index_topk(const void *qI, const float *q_scale, const float *w, const void *kI, const float *k_scale,
                   int dtype, const int32_t *n_valid, int B, int T, int64_t N, int k, int32_t *idx,
                   int32_t *failed_rows, void *workspace, size_t ws_bytes, void *stream);

/*
 * csa_topk -- top-k of each score row ([HA] §4.2 / §7 topk(scores, k);
 * k = 512 Flash, 1024 Pro):
 *   idx[b,t,:] = the k indices i < n_valid[b,t] with the largest scores[b,t,i],
 *   ties toward the lower index, in ascending index order; when
 *   n_valid[b,t] < k the row holds 0..n_valid-1 followed by -1.
 *   -0.0 equals +0.0; NaN scores are not supported.
 *   scores  : [B, T, N] fp32;  n_valid : [B, T] int32;  idx : [B, T, k] int32
 *   1 <= k <= CSA_MAX_TOPK;  N <= 2^20
 *   workspace : csa_topk_workspace_size(B, T, N, k) bytes of device memory,
 *               16-byte aligned, ZERO-FILLED by the caller before its first use;
 *               every call leaves it zero-filled again.  Calls that share a
 *               workspace must be ordered on one stream.
 */
size_t csa_topk_workspace_size(int B, int T, int64_t N, int k);
int csa_topk(const float *scores, const int32_t *n_valid, int B, int T, int64_t N, int k, int32_t *idx,
             void *workspace, size_t ws_bytes, void *stream);

/*
 * csa_topk_noalloc -- csa_topk without a caller-provided workspace.  The pages have
 * no counterpart: this entry point is for callers that cannot allocate device
 * memory themselves -- a host that reserves its whole device-memory budget at
 * start-up and forbids allocation afterwards (embedded or latency-critical
 * serving), a plug-in that runs inside another application which owns the device
 * allocator, or plain C code with no device allocator of its own.
 *   Same arguments, checks and results as csa_topk, minus the workspace.  Rows that
 *   need scratch (see csa_topk_workspace_size) use a library-owned device array of
 *   CSA_NOALLOC_SCRATCH_BYTES (16 MiB), which every GPU that loads the library
 *   holds until the process exits; a call whose csa_topk_workspace_size exceeds
 *   it returns CSA_ERR_UNSUPPORTED.  Every argument is checked before the array is
 *   touched: a rejected call enqueues nothing.  No cudaMalloc / cudaFree (or any
 *   allocating routine) is ever made; each call clears the part of the array it
 *   uses with cudaMemsetAsync on `stream`: a completed call leaves that part zeroed,
 *   but one cut short (an error) or one that overlapped another would not, and the
 *   clear makes every call independent of the previous one.
 *   Each call looks up the array's device address (cudaGetSymbolAddress) with the
 *   call's device current, so the entry point stays valid after a cudaDeviceReset
 *   (the array may then sit at another address).  All calls share
 *   the one array: calls that may overlap on the GPU (different streams, or work
 *   replayed concurrently) race on it and give wrong results -- order them on one
 *   stream.
 */
#define CSA_NOALLOC_SCRATCH_BYTES (16u << 20)
int csa_topk_noalloc(const float *scores, const int32_t *n_valid, int B, int T, int64_t N, int k, int32_t *idx,
                     void *stream);

/*
 * csa_index_rerank -- exact rescoring of a candidate list, then top-k among it
 * ([HA] §9: the indexer forms its candidates at twice top-k; this is the
 * second stage that makes a low-precision first pass exact on its candidates).
 *   cand[b,t,:] (kc ascending indices, -1 padded; typically csa_topk of the e4m3
 *   scores with 2k) is rescored with the plain definition of csa_index_scores on
 *   the full-precision qI / kI (dtype F32 or BF16, fp32 accumulation), then
 *   idx[b,t,:] = the k best candidates (ties toward the lower index), ascending,
 *   -1 padded -- equal to csa_topk of the full-precision scores whenever the true
 *   top-k lies inside the candidate list.
 *   qI [B,T,64,128], w [B,T,64] fp32, kI [B,N,128], cand [B,T,kc] int32,
 *   cand_scores [B,T,kc] fp32 (caller scratch), idx [B,T,k] int32;
 *   k <= kc <= 32768.
 */
int csa_index_rerank(const void *qI, const float *w, const void *kI, int dtype, const int32_t *cand, int kc, int B,
                     int T, int64_t N, int k, float *cand_scores, int32_t *idx, void *stream);

/*
 * csa_topk_select -- decode top-k in one launch, fed by the histogram that
 * csa_index_scores(..., select_ws) accumulated ([HA] §4.2 / §7 topk; §9: the
 * indexer forms its candidates at twice top-k).  One query per sequence (T == 1):
 * scores [B, N] fp32, n_valid [B] int32, idx [B, k] int32.
 *   qI == NULL : idx = the exact top-k of each row (as csa_topk).
 *   qI != NULL : candidates = every index whose score lies in the histogram bin of
 *                the kc-th largest score or above (a superset of the kc largest);
 *                each is rescored with the plain indexer definition on the
 *                full-precision qI [B, 64, 128] / kI [B, N, 128] (dtype F32 or BF16)
 *                and w [B, 64], and idx = the k best rescored candidates.
 *   Ties go to the lower index; rows are ascending and -1 padded (n_valid < k).
 *   idx_scores : NULL, or [B, k] fp32 (caller-owned): beside each idx entry the score
 *               that ranked it -- the rescored exact score when qI != NULL, else the
 *               input score -- and -inf beside a -1 pad.  With qI != NULL a row of
 *               0 < n_valid <= k entries is then rescored too (every entry is taken).
 *               The sharded decode packs these scores for its all-gather.
 *   k <= CSA_MAX_TOPK, k <= kc, N <= 2^19.
 *   workspace : csa_select_workspace_size(B, N) bytes, 16-byte aligned, ZERO-FILLED
 *               before first use; csa_index_scores(..., workspace) fills the
 *               histograms and this call consumes them and leaves the workspace
 *               ready (zeroed histograms) for the next pair of calls.
 */
size_t csa_select_workspace_size(int B, int64_t N);
/* csa_score_histogram -- accumulate the per-row histogram of scores [B, N] (entries
 * i < n_valid[b]) into a csa_topk_select workspace, for scores that did not come
 * from csa_index_scores(..., select_ws). */
int csa_score_histogram(const float *scores, const int32_t *n_valid, int B, int64_t N, void *workspace,
                        size_t ws_bytes, void *stream);
int csa_topk_select(const float *scores, const int32_t *n_valid, int B, int64_t N, int k, int kc, const void *qI,
                    const float *w, const void *kI, int dtype, int32_t *idx, float *idx_scores, void *workspace,
                    size_t ws_bytes, void *stream);

/*
 * csa_quantize_kv8 -- mixed-precision storage of compressed KV entries ([HA] §4.2,
 * storage precision: the RoPE dims stay BF16, the rest of each compressed entry
 * is FP8).  D = 512 only; the last 64 dims are the RoPE dims.
 *   kv      : [rows, 512] bf16 (device), 16-byte aligned
 *   entries : [rows, csa_kv8_entry_bytes(512) = 608] bytes (device), 16-byte aligned:
 *             bytes [0, 448)   e4m3 codes of dims 0..447,
 *                   [448, 576) bf16 dims 448..511 (bit copy),
 *                   [576, 604) seven fp32 block scales s = 2^e (block = 64 dims), e the
 *                              smallest integer with max|x| <= 448 * 2^e (0 for a zero block),
 *                   [604, 608) zero.
 *             code = e4m3 of x / s, nearest, ties to even (x / s is exact), so code * s is
 *             exactly a bf16 value.
 *   CSA_ERR_UNSUPPORTED for D != 512; CSA_ERR_INVALID for null or misaligned pointers.
 * Such entries are the kv argument of sparse_attn / hca_attn with dtype CSA_BF16_KV8,
 * which attend over the dequantised rows (code * s, and the bf16 dims as stored).
 */
long long csa_kv8_entry_bytes(int D);
int csa_quantize_kv8(const void *kv, int64_t rows, int D, void *entries, void *stream);

/*
 * sparse_attn -- CSA core attention ([P2] sparse_attn(q, kv, attn_sink,
 * topk_idxs, softmax_scale); [HA] §4.2 Shared-KV MQA, §6 SWA + sink, §7 call chain):
 *   for query (b,t) at absolute position pos = q_pos[b,t] and head h:
 *     memory = [swa_kv rows of positions max(0,pos-127)..pos held in the buffer
 *               (buffer row = position - swa_pos0[b])] ++ [kv[b, idx[b,t,e]] for e < k]
 *     z_j = scale * <q[b,t,h,:], memory_j>,
 *     out[b,t,h,:] = sum_j exp(z_j) memory_j / (exp(sink[h]) + sum_l exp(z_l))
 *   The latent row is both key and value.  idx entries outside [0, N) (e.g.
 *   the -1 padding of csa_topk) contribute nothing.
 *   q      : [B, T, H, D] dtype;  kv : [B, N, D] dtype;  swa_kv : [B, W, D] dtype
 *   swa_pos0 : [B] int64;  q_pos : [B, T] int64;  sink : [H] fp32 (unscaled logit)
 *   idx    : [B, T, k] int32;  out : [B, T, H, D] dtype
 *   dtype CSA_BF16 (tcgen05, fp32 softmax and accumulation; H <= 128,
 *   D in {128, 256, 512}), CSA_BF16_KV8 (as CSA_BF16 with kv [B, N, 608] bytes of
 *   csa_quantize_kv8 entries; D = 512) or CSA_F32 (fp32 FMA; D multiple of 32, <= 512).
 *   workspace : csa_attn_workspace_size(B, T, H, D, rows_per_query, dtype) bytes
 *               (16-byte aligned, device memory, owned by the caller, contents
 *               need not be kept between calls), rows_per_query = min(W, 128) + k
 *               for sparse_attn and min(W, 128) + N for hca_attn (a larger value
 *               gives a size that is also enough); may be NULL when that size is 0.
 *               With few queries (B * T * ceil(H / 64) below the SM count) the
 *               CSA_BF16 row list of a query is split over up to 16 CTAs of one
 *               thread-block cluster that write their unnormalised partial
 *               outputs and (m, l) there and merge them after a cluster barrier;
 *               CSA_BF16_KV8 and CSA_F32 need none (size 0).  Too small or
 *               misaligned -> CSA_ERR_INVALID, nothing launched.
 */
size_t csa_attn_workspace_size(int B, int T, int H, int D, int64_t rows_per_query, int dtype);
int sparse_attn(const void *q, const void *kv, const void *swa_kv, const int64_t *swa_pos0, int W,
                const int64_t *q_pos, const float *sink, const int32_t *idx, int k, float scale, int B, int T,
                int H, int D, int64_t N, int dtype, void *out, void *workspace, size_t ws_bytes, void *stream);

/*
 * hca_attn -- HCA core attention ([HA] §5: dense MQA over every compressed
 * summary plus the SWA rows, no indexer): as sparse_attn with the memory rows
 * kv[b, 0 .. min(N, (pos+1)/ratio) - 1] (complete blocks only).
 */
int hca_attn(const void *q, const void *kv, const void *swa_kv, const int64_t *swa_pos0, int W,
             const int64_t *q_pos, const float *sink, int ratio, float scale, int B, int T, int H, int D, int64_t N,
             int dtype, void *out, void *workspace, size_t ws_bytes, void *stream);

/*
 * Partial RoPE ([HA] §6: only the last 64 dims of each head carry the rotary position
 * embedding; after the core attention the output's same dims get the inverse rotation,
 * before the grouped output projection).  The pages give no pairing, base or position
 * rule; this library's reading: the RoFormer rotation of the pairs (D-64+2i, D-64+2i+1),
 * i < 32, by the angle pos * theta^(-2i/64) (theta > 1; the MXFP4 page's
 * compress_rope_theta is 160000), a compressed entry i standing at position i * ratio,
 * SWA rows and queries at their token positions.  Angles and their cos / sin are formed
 * in fp64, the rotation runs in fp32.
 *
 * csa_rope -- rows x [B, R, D] (F32|BF16) -> out (the same pointer for in place): dims
 *   D-64.. turned at position pos(b, r) = (pos_base ? pos_base[b] : 0) + r * stride, the
 *   others copied; inverse != 0 turns the other way.  Use it when rows enter a cache:
 *   compressed entries (pos_base NULL, stride = ratio) and raw SWA rows (pos_base =
 *   swa_pos0, stride 1).  D even and >= 64.
 */
int csa_rope(const void *x, int dtype, int B, int64_t R, int D, const int64_t *pos_base, int64_t stride,
             double theta, int inverse, void *out, void *stream);

/*
 * sparse_attn_rope / hca_attn_rope -- sparse_attn / hca_attn with the partial RoPE around
 * the attention: q (as given, not rotated) is turned at q_pos inside the kernel, the memory
 * and SWA rows are taken as stored (rotated when they entered the cache, csa_rope), and the
 * output's last 64 dims are turned back at q_pos.  So out = inverse_rope(attn(rope(q),
 * rows)) ([HA] §7 call chain).  rope_theta > 1; dtype CSA_BF16 or CSA_F32 (CSA_BF16_KV8:
 * CSA_ERR_UNSUPPORTED); D >= 64.  Other arguments as sparse_attn / hca_attn.
 */
int sparse_attn_rope(const void *q, const void *kv, const void *swa_kv, const int64_t *swa_pos0, int W,
                     const int64_t *q_pos, const float *sink, const int32_t *idx, int k, float scale,
                     double rope_theta, int B, int T, int H, int D, int64_t N, int dtype, void *out, void *workspace,
                     size_t ws_bytes, void *stream);
int hca_attn_rope(const void *q, const void *kv, const void *swa_kv, const int64_t *swa_pos0, int W,
                  const int64_t *q_pos, const float *sink, int ratio, float scale, double rope_theta, int B, int T,
                  int H, int D, int64_t N, int dtype, void *out, void *workspace, size_t ws_bytes, void *stream);

/*
 * Sharded decode of one long sequence over G GPUs (the compressed entries split into
 * G contiguous ranges, one per GPU).  Per step, on every GPU g owning entries [lo, hi):
 *   1. csa_index_scores + csa_topk_select over the local entries (local indices, with
 *      the exact rescored scores of the local winners in idx_scores), and csa_shard_pack
 *      -> (score, global index) pairs;
 *   2. one all-gather of the pairs, shard-major [G][B][k]; csa_shard_select -> the
 *      global top-k, the same on every GPU;
 *   3. csa_shard_remap -> the winners inside [lo, hi) as local indices;
 *      sparse_attn_partial over them (the SWA rows on one GPU only: W = 0 elsewhere),
 *      its output and (m, l) written into one buffer;
 *   4. one all-gather of those buffers; csa_attn_combine adds the sink once.
 * The attention identity behind 3-4: [HA] §6 p_i = e^{z_i} / (e^{z_s} + sum_j e^{z_j})
 * over a union of disjoint row sets, put together from per-set pieces.
 */

/*
 * sparse_attn_partial -- sparse_attn over this GPU's rows without the sink:
 *   out[b,t,h,:] = sum_j e^{z_j - m} row_j / l,  l = sum_j e^{z_j - m},
 *   ml[b,t,h] = (m, l) as two fp32 (natural-log units; m is a reference value near the
 *   largest z, so m + ln(l) is the log-sum-exp of the z_j); no rows -> (-inf, 0), out 0.
 *   Arguments as sparse_attn (no sink); W = 0 leaves the SWA rows out.
 *   dtype CSA_BF16 or CSA_BF16_KV8 (CSA_F32: CSA_ERR_UNSUPPORTED).
 *   out [B,T,H,D] bf16; ml [B,T,H,2] fp32, 8-byte aligned.
 */
int sparse_attn_partial(const void *q, const void *kv, const void *swa_kv, const int64_t *swa_pos0, int W,
                        const int64_t *q_pos, const int32_t *idx, int k, float scale, int B, int T, int H, int D,
                        int64_t N, int dtype, void *out, float *ml, void *workspace, size_t ws_bytes, void *stream);

/*
 * csa_attn_combine -- G partial results -> the attention output with the sink added once:
 *   M = max(sink[h], m_g), den = e^{sink[h] - M} + sum_g l_g e^{m_g - M},
 *   out = sum_g l_g e^{m_g - M} o_g / den   (pieces with l_g = 0 are skipped).
 *   Shard g's outputs o_g [B,T,H,D] bf16 start at parts + g * part_stride bytes and its
 *   (m, l) [B,T,H,2] fp32 at ml + g * ml_stride bytes (e.g. one gathered buffer per shard:
 *   the same stride for both); sink [H] fp32; out [B,T,H,D] bf16.
 *   1 <= G <= CSA_MAX_SHARDS; D a multiple of 8; parts, out 16-byte aligned, part_stride a
 *   multiple of 16, ml and ml_stride multiples of 8.
 */
int csa_attn_combine(const void *parts, int64_t part_stride, const float *ml, int64_t ml_stride, const float *sink,
                     int G, int B, int T, int H, int D, void *out, void *stream);

/*
 * csa_shard_pack -- this shard's winners as (score, global index) pairs: n entries,
 *   loc[i] in [0, ns) -> (scores[i], loc[i] + lo); anything else -> (-inf, -1).
 *   pairs: n x {fp32 score, int32 index}, 8-byte aligned.
 */
int csa_shard_pack(const float *scores, const int32_t *loc, int64_t n, int64_t ns, int64_t lo, void *pairs,
                   void *stream);

/*
 * csa_shard_select -- global top-k from the gathered pairs [G][B][k] (csa_shard_pack's
 * layout; each shard's list ascending, -1 padded; the shards in ascending entry order)
 * -> idx [B][k], the k best by score, ties toward the lower global index (position
 * order), padding never before a real entry.
 * workspace: csa_shard_select_workspace_size(G, B, k) bytes.  G * k <= 32768.
 */
size_t csa_shard_select_workspace_size(int G, int B, int k);
int csa_shard_select(const void *pairs, int G, int B, int k, int32_t *idx, void *workspace, size_t ws_bytes,
                     void *stream);

/*
 * csa_shard_remap -- out[i] = in[i] - lo + add if lo <= in[i] < hi, else -1 (n entries,
 * int32).  Global -> local indices: the shard's [lo, hi), add = 0; local -> global:
 * lo = 0, hi = the shard's entry count, add = its first entry.
 */
int csa_shard_remap(const int32_t *in, int64_t n, int64_t lo, int64_t hi, int64_t add, int32_t *out, void *stream);

/*
 * csa_launch_count -- number of kernels this library has enqueued in this
 * process so far (all devices, all streams; captured launches included).
 */
unsigned long long csa_launch_count(void);

/*
 * csa_poll_status -- synchronise `stream`, then return and clear the device
 * status word (CSA_OK, or CSA_ERR_TIMEOUT if a kernel abandoned a bounded
 * wait since the last poll).  CSA_ERR_CUDA if synchronisation fails.
 */
int csa_poll_status(void *stream);

/*
 * csa_test_bounded_wait -- a check of the failure-detection path (no counterpart in
 * the pages): one kernel thread waits on a shared-memory barrier that completes only
 * if `complete` is non-zero, with the bound limit_ns nanoseconds of the GPU's global
 * timer.  If the bound runs out the kernel records CSA_ERR_TIMEOUT in the device status
 * word and returns, exactly as every wait inside the library's kernels does; the
 * next csa_poll_status returns that code and clears it.  No GPU fault is involved.
 *   1000 <= limit_ns <= 10^9; CSA_ERR_INVALID otherwise.
 */
int csa_test_bounded_wait(int complete, long long limit_ns, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* CSA_H_ */
