/*
 * qsa.h -- C ABI of the B200 (sm_100a) Qwen Sparse Attention (QSA) hot path.
 *
 * The method (from "Qwen3.8-Flash-Next architecture", flozi.net, section "Der Weg eines Tokens
 * durch das Modell", item 2 "Die zwei Stufen von QSA"; and "Qwen3.8-Flash-Next", studioglobal.ai,
 * section "Hybride Aufmerksamkeit fuer sehr lange Kontexte"):
 *   1. an indexer maps tokens to light keys; groups of `blk` (= 4) consecutive keys are averaged
 *      into one micro-block key, and RoPE is applied after the averaging;
 *   2. every query is scored against its causally visible micro-blocks with Hi (= 4) indexer
 *      query heads sharing one key head;
 *   3. each query keeps its top-k blocks (k = 512 blocks = 2048 tokens) plus its own, possibly
 *      incomplete, block;
 *   4. exact softmax attention (GQA) runs over only the tokens of the kept blocks.
 * Readings where the pages leave a step open (all fixed here, and in the CPU oracle):
 *   - score s(t,b) = sum_h w_h * max(0, qi[t,h] . kp[b])  (QSA_SCORE_LINEAR drops the max);
 *   - the candidates of the query at position p are the complete blocks b < floor(p/blk); the own
 *     block (tokens blk*floor(p/blk) .. p) is always attended and never scored;
 *   - top-k is taken on the fp32 scores; equal scores go to the lower block index; the list is
 *     ascending and padded with -1 when fewer than k candidates exist;
 *   - one index list per query, shared by all attention heads (one shared key head);
 *   - pooled keys and rotated indexer queries are stored as bf16 (round to nearest even);
 *   - RoPE is the half-split rotation of pairs (i, i + Di/2) by pos * theta^(-2i/Di); a pooled key
 *     sits at the position of its block's first token.
 *
 * Conventions for every call:
 *   - All tensor pointers are caller-owned, contiguous, 16-byte-aligned DEVICE memory; bf16
 *     tensors are passed as `const void*` / `void*` (bf16 bit patterns).  Layouts are given per
 *     call, outermost dimension first.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work is enqueued on it
 *     asynchronously; no call synchronises except qsa_get_device_status.  No call allocates
 *     device memory; scratch memory comes from the caller's `workspace`.
 *   - Arguments are checked on the host before any launch.  On a non-QSA_OK return nothing was
 *     launched and no output was touched (QSA_ERR_CUDA: a launch was rejected by the runtime).
 *   - Faults found on the device (an index list entry outside its query's causal range, a
 *     sequence length outside the cache, a wait that ran out of time) are skipped by the kernel
 *     and recorded in a per-device status word that qsa_get_device_status reads and clears.
 *   - Supported shapes: blk = 4; Di = 64 for scoring (any even Di <= 256 for pooling/RoPE);
 *     Hi in {1, 2, 4, 8}; attention D in {128, 256}, Hkv in {1, 2}, Hq/Hkv <= 16 (the decode
 *     split merge inside thread-block clusters needs D = 128 and Hq/Hkv <= 8; other decode shapes
 *     merge through the workspace).  Other shapes return QSA_ERR_UNSUPPORTED.
 *   - Calls are thread-safe.  The library keeps only per-device caches (device attributes, the
 *     status word) and no other mutable global state.
 *   - Every call opens an NVTX range named after the function (visible in Nsight Systems and
 *     Nsight Compute; costs one pointer test when no tool is attached).
 *   - The debug build of the library (libqsa_b200_debug.so, compiled with -DQSA_DEBUG) has the
 *     same ABI.  Its kernels check the data-dependent addresses they form (gathered K/V rows,
 *     output and partial rows, tile-union entries and chunk records) against the sizes of the
 *     call; a failed check skips the access and records QSA_ERR_DEVICE_CHECK.  In a correct
 *     library no check fails; the release build compiles them out.
 */
#ifndef QSA_H
#define QSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define QSA_ABI_VERSION 1

#if defined(__GNUC__)
#define QSA_API __attribute__((visibility("default")))
#else
#define QSA_API
#endif

typedef enum {
  QSA_OK = 0,
  QSA_ERR_INVALID_ARGUMENT = 1,    /* null pointer, negative size, misaligned pointer, bad index */
  QSA_ERR_UNSUPPORTED = 2,         /* a shape outside the supported set above */
  QSA_ERR_WORKSPACE_TOO_SMALL = 3, /* ws_bytes below what the call needs */
  QSA_ERR_CUDA = 4,                /* the CUDA runtime rejected a launch or query */
  QSA_ERR_TIMEOUT = 5,             /* a device-side wait ran out of time (device status only) */
  QSA_ERR_DEVICE_CHECK = 6         /* debug build only: a device-side bounds check failed and the
                                      access was skipped (device status only) */
} qsa_status_t;

typedef enum {
  QSA_SCORE_RELU_SUM = 0, /* s = sum_h w_h * max(0, qi_h . kp)   (the QSA indexer) */
  QSA_SCORE_LINEAR = 1    /* s = sum_h w_h * (qi_h . kp)          (test mode: one GEMM) */
} qsa_score_mode_t;

typedef enum {
  QSA_OP_SELECT_TOPK = 1,       /* qsa_select_topk with scores == NULL */
  QSA_OP_SPARSE_ATTN_DECODE = 2, /* qsa_sparse_attn_decode with num_splits > 1 */
  QSA_OP_SPARSE_ATTN_PREFILL = 3 /* qsa_sparse_attn_prefill_ws (query tiles) */
} qsa_op_t;

/* Human-readable name of a status code (static string, never NULL). */
QSA_API const char* qsa_status_string(qsa_status_t status);

/* QSA_ABI_VERSION of the loaded library. */
QSA_API int qsa_abi_version(void);

/*
 * Micro-block key pooling (step 1: mean of each group of four keys, then RoPE).
 *   ki [B][L][Di] bf16  ->  kp [B][floor(L/blk)][Di] bf16
 *   kp[b][j] = bf16( rope( (1/blk) * sum_{i<blk} ki[b][blk*j + i], pos0 + blk*j ) )
 * The mean is formed exactly (double) and rounded once to bf16.  rope_theta <= 0 disables RoPE.
 * A trailing partial group (L mod blk tokens) is not pooled.  Batch strides are in elements
 * (0 = packed: L*Di for ki, floor(L/blk)*Di for kp), so a decode step can pool the newest block
 * j of every sequence of a [B][Lmax][Di] cache in one call: ki = &ki[0][blk*j][0], L = blk,
 * ki_batch_stride = Lmax*Di, kp = &kp[0][j][0], kp_batch_stride = NBk*Di, pos0 = blk*j.
 * Errors: INVALID_ARGUMENT (null, B/L < 0, Di odd or > 256), UNSUPPORTED (blk != 4).
 */
QSA_API qsa_status_t qsa_pool_block_keys(const void* ki, void* kp, int B, int L, int Di, int blk,
                                         float rope_theta, int64_t pos0, int64_t ki_batch_stride,
                                         int64_t kp_batch_stride, void* stream);

/*
 * Rotary parameters of the indexer, for the _rope variants below.  theta <= 0: no rotation.
 * yarn_factor > 1 scales the frequencies for contexts beyond yarn_orig_ctx positions with YaRN
 * ("YaRN: Efficient Context Window Extension of Large Language Models", Peng et al. 2023, sections
 * 3.2 and 3.4; the pages name YaRN for the 1M-token context but give no parameters).  For the pair
 * with base frequency f = theta^(-2i/Di) and r = yarn_orig_ctx * f / (2 pi) rotations over the
 * original context, g = clamp((r - yarn_alpha) / (yarn_beta - yarn_alpha), 0, 1) and the frequency
 * becomes (1 - g) f / yarn_factor + g f; the rotated pair is multiplied by yarn_mscale (<= 0: the
 * paper's 0.1 ln(yarn_factor) + 1).  Typical ramp: yarn_alpha = 1, yarn_beta = 32.
 */
typedef struct qsa_rope_params {
  double theta;
  double yarn_factor;    /* <= 1: plain RoPE */
  double yarn_orig_ctx;  /* > 0 when yarn_factor > 1 */
  double yarn_alpha;
  double yarn_beta;      /* > yarn_alpha */
  double yarn_mscale;
} qsa_rope_params_t;

/*
 * qsa_pool_block_keys with rotary parameters (NULL: no rotation).  Errors as above, and
 * INVALID_ARGUMENT for inconsistent YaRN parameters.
 */
QSA_API qsa_status_t qsa_pool_block_keys_rope(const void* ki, void* kp, int B, int L, int Di, int blk,
                                              const qsa_rope_params_t* rope, int64_t pos0,
                                              int64_t ki_batch_stride, int64_t kp_batch_stride,
                                              void* stream);

/*
 * RoPE of the indexer queries at their own positions (the query side of the rotation that the
 * keys receive after pooling).
 *   qi [B][Tq][Hi][Di] bf16 -> qi_out (same layout; may alias qi)
 *   row t of batch b sits at position q_pos0 + t, or at seqlens[b] - 1 when seqlens != NULL
 *   (decode: Tq must be 1).  Call it before qsa_index_score / qsa_select_topk when RoPE is on.
 * Errors: INVALID_ARGUMENT (null, sizes, Di odd or > 256, rope_theta <= 0).
 */
QSA_API qsa_status_t qsa_rope_index_queries(const void* qi, void* qi_out, int B, int Tq, int Hi, int Di,
                                    int64_t q_pos0, const int32_t* seqlens, float rope_theta,
                                    void* stream);

/*
 * qsa_rope_index_queries with rotary parameters (theta must be > 0); use the same parameters as
 * for the keys.  Errors as above.
 */
QSA_API qsa_status_t qsa_rope_index_queries_rope(const void* qi, void* qi_out, int B, int Tq, int Hi,
                                                 int Di, int64_t q_pos0, const int32_t* seqlens,
                                                 const qsa_rope_params_t* rope, void* stream);

/*
 * Indexer block scores (step 2: four indexer query heads against one shared key head).
 *   qi [B][Tq][Hi][Di] bf16 (already rotated if RoPE is used), kp [B][NBk][Di] bf16,
 *   head_w [Hi] fp32 or NULL (all ones)  ->  scores [B][Tq][ld_scores] fp32:
 *   scores[b][t][j] = s(t, j) for j < NB(p) = floor(p/blk), p = q_pos0 + t (or seqlens[b]-1 with
 *   seqlens != NULL, Tq == 1).  Entries j >= NB(p) are not written.
 * Prefill runs on tcgen05 tensor cores (TMEM accumulators, TMA-fed); decode (seqlens != NULL)
 * is a bandwidth-bound pass over the pooled-key cache on warp-level tensor-core MMAs (mma.sync,
 * fp32 accumulate): its fp32 sums may differ from the prefill kernel's in the last bit.
 * Requires floor((q_pos0 + Tq - 1)/blk) <= NBk (prefill) and ld_scores >= NBk.
 * Errors: INVALID_ARGUMENT, UNSUPPORTED (Di != 64, Hi not in {1,2,4,8}, blk != 4).
 */
QSA_API qsa_status_t qsa_index_score(const void* qi, const void* kp, const float* head_w,
                             const int32_t* seqlens, int B, int Tq, int NBk, int Hi, int Di,
                             int blk, int64_t q_pos0, qsa_score_mode_t mode, float* scores,
                             int64_t ld_scores, void* stream);

/*
 * Per-query top-k block selection (step 3: a budget of 512 whole blocks, i.e. 2048 tokens).
 *   -> idx [B][Tq][k] int32: the k candidates with the largest fp32 score (equal scores: lower
 *   index first), in ascending block order, -1 padded when NB(p) < k.  The own block is never
 *   listed (it is implicit).
 * scores != NULL: select from scores [B][Tq][ld_scores] (as written by qsa_index_score); qi, kp,
 *   head_w, mode and workspace are ignored.
 * scores == NULL: the scores are computed here.  Arguments as for qsa_index_score.  Two ways,
 *   both selecting the top k of the same tensor-core fp32 scores (rows redone exactly, see below,
 *   use CUDA-core fp32 scores, which may differ in the last bit, so such a row can differ from the
 *   other way only by blocks tied within that rounding); qsa_set_select_options can force one:
 *   - materialised (decode; Hi of 1 or 2; short prefills): the scores are computed chunk by chunk
 *     into `workspace` (at least one score row of NBk floats; decode: B rows).  In decode, with
 *     few sequences (2 or more SMs per sequence), k <= 1024 and more than 6144 blocks, each
 *     sequence's top-k runs on a thread-block cluster of up to 8 CTAs, one slice of the scores
 *     each, merged through distributed shared memory; the lists equal those of one CTA per
 *     sequence.  With more than one chunk the
 *     workspace is split in two halves and the top-k of one chunk runs on a per-device internal
 *     stream while the next chunk is scored on `stream`; the internal stream is joined back into
 *     `stream` before the call returns, so the call keeps the usual stream-ordered semantics.
 *   - filtered (prefill with Hi of 4 or 8 and k <= 1024, chosen automatically when the call's last
 *     row sits at position 16384 or later, q_pos0 + Tq >= 16384, and the workspace holds 4096 rows
 *     or all of them): the scores are never stored.  Every 16th
 *     pooled block is scored first; per row, a threshold with about 2 k (at least 1024) of the
 *     row's scores expected above it is read off these samples; the tensor-core score kernel then
 *     keeps only the scores at or above the threshold, in block order, and the top-k is selected
 *     from that list.  A row whose list is shorter than k or longer than its capacity is redone
 *     exactly over all its scores (CUDA-core fp32 scores), so a threshold decides only which rows
 *     are redone, never which blocks a row keeps beyond last-bit ties.  Workspace per
 *     row of a chunk: about 4 * NBk / 16 + 256 * max(64, ceil(2 k / 16)) bytes, plus
 *     128 * NBk * 4 bytes for the redo.
 *   qsa_workspace_size(QSA_OP_SELECT_TOPK, ...) gives a size that fits either way in few chunks
 *   (up to about 4 GiB).
 * Errors: INVALID_ARGUMENT (k < 1, ...), UNSUPPORTED, WORKSPACE_TOO_SMALL.
 */
QSA_API qsa_status_t qsa_select_topk(const float* scores, int64_t ld_scores, const void* qi,
                             const void* kp, const float* head_w, const int32_t* seqlens, int B,
                             int Tq, int NBk, int Hi, int Di, int blk, int64_t q_pos0,
                             qsa_score_mode_t mode, int k, int32_t* idx, void* workspace,
                             size_t ws_bytes, void* stream);

/*
 * Decode selection with the pooling of the newest block folded in (one decode step's steps 1-3).
 *   qi [B][Hi][Di] bf16 (rotated if RoPE is used), kp [B][NBk][Di] bf16 (read and written),
 *   ki [B][Lmax][Di] bf16 key cache, row b at ki + b * ki_batch_stride (elements; 0 = NBk * blk *
 *   Di), seqlens [B] -> idx [B][k] as qsa_select_topk with seqlens.
 * For every sequence whose new token completes a block (seqlens[b] a multiple of blk and
 * seqlens[b] / blk <= NBk), kp[b][seqlens[b]/blk - 1] is first set to the pooled (and, with rope,
 * rotated) key of cache rows seqlens[b] - blk .. seqlens[b] - 1, exactly as qsa_pool_block_keys
 * would write it.  That block is the query's own block, so the selection does not depend on it;
 * the pooling runs inside the score kernel and saves a launch per step.  rope may be NULL (no
 * rotation).  Workspace: at least B * NBk * 4 bytes (the score rows).
 * Errors: as for qsa_select_topk.
 */
QSA_API qsa_status_t qsa_decode_select(const void* qi, void* kp, const void* ki, int64_t ki_batch_stride,
                                       const float* head_w, const int32_t* seqlens, int B, int NBk, int Hi,
                                       int Di, int blk, qsa_score_mode_t mode,
                                       const qsa_rope_params_t* rope, int k, int32_t* idx, void* workspace,
                                       size_t ws_bytes, void* stream);

/*
 * Gather-sparse attention, prefill (step 4: exact attention over the selected tokens, GQA).
 *   q [B][Tq][Hq][D] bf16 for positions q_pos0 .. q_pos0+Tq-1 (q_pos0 + Tq <= Tk),
 *   k, v [B][Tk][Hkv][D] bf16, idx [B][Tq][k_blocks] int32 (from qsa_select_topk; entries -1
 *   and entries equal to the own block are skipped; other entries outside [0, own) are skipped
 *   and flagged in the device status)  ->  out [B][Tq][Hq][D] bf16,
 *   lse [B][Tq][Hq] fp32 (natural-log log-sum-exp of the scaled logits; may be NULL).
 *   o(t,h) = sum_{j in S(t)} softmax_j(scale * q(t,h) . k(j,g)) v(j,g),  g = h / (Hq/Hkv),
 *   S(t) = tokens of the listed blocks  U  { blk*floor(p/blk) .. p }.
 * The softmax is kept in fp32 (online, exp2 form); products run on bf16 tensor cores.
 * Shapes: D = 128 or 256, Hkv = 1 or 2, Hq/Hkv up to 16 -- the benchmark shape (16 query heads
 * over 2 KV heads, D = 128) and the model shape of "Qwen3.8-Flash-Next architecture" (flozi.net),
 * "Der Weg eines Tokens durch das Modell" (24 query heads over 2 KV heads, D = 256).
 * Errors: INVALID_ARGUMENT, UNSUPPORTED (D not in {128, 256}, Hkv not in {1,2}, Hq/Hkv > 16,
 * blk != 4).
 */
QSA_API qsa_status_t qsa_sparse_attn_prefill(const void* q, const void* k, const void* v,
                                     const int32_t* idx, int B, int Tq, int Tk, int Hq, int Hkv,
                                     int D, int k_blocks, int blk, int64_t q_pos0, float scale,
                                     void* out, float* lse, void* stream);

/*
 * qsa_sparse_attn_prefill with a workspace: the same arguments, result and errors, plus `workspace`
 * (caller-owned device memory, 16-byte aligned) of ws_bytes.
 * With the query-tile path chosen (qsa_set_attn_options(2); the automatic choice is row by row,
 * the faster of the two on workloads whose consecutive rows share little of their selections), and
 * when D = 128, Hq = 8 * Hkv (groups of 8 query heads), k_blocks <= 1024 and the workspace holds at
 * least one tile (512 + 8 * (16 * k_blocks + 16) + 128 * (k_blocks + 1) + 4 bytes; qsa_workspace_size(
 * QSA_OP_SPARSE_ATTN_PREFILL, B, Tq, 0, k_blocks, Hq, D, 0) gives room for up to 4096 tiles), the
 * rows are processed in tiles of 16 consecutive query rows on tcgen05 tensor cores: a tile attends
 * over the union of its rows' listed blocks and own blocks, gathered once per tile, and each row
 * masks out the union blocks it did not list ("Qwen3.8-Flash-Next architecture" (flozi.net), "Der
 * Weg eines Tokens durch das Modell", item 2: exact attention over the selected tokens;
 * consecutive queries select overlapping blocks).  The result is the same exact attention up to
 * fp32 summation order.  The order of the entries in a list does not matter.  A non-finite K/V value in
 * a block that one row of a tile lists reaches the other rows of the tile (0 * inf); positions
 * past the call's last query are never read.  Calls with more tiles than the workspace holds are
 * processed in ranges of tiles.
 * The automatic choice (qsa_set_attn_options(0)) runs row by row; when the shape is one that
 * qsa_sparse_attn_prefill_kv takes and the workspace holds K and V interleaved by block
 * (ws_bytes >= B * ceil(Tk / 4) * 2 * 4 * Hkv * D * 2; qsa_attn_prefill_workspace_size covers it),
 * it first writes the interleaved blocks of the positions the rows can see (qsa_interleave_kv)
 * into the workspace and then runs qsa_sparse_attn_prefill_kv: the same result bit for bit, with
 * each block's K and V fetched by one copy.  Otherwise, and with qsa_set_attn_options(1), it runs
 * the row-by-row kernel of qsa_sparse_attn_prefill.
 */
QSA_API qsa_status_t qsa_sparse_attn_prefill_ws(const void* q, const void* k, const void* v,
                                        const int32_t* idx, int B, int Tq, int Tk, int Hq, int Hkv,
                                        int D, int k_blocks, int blk, int64_t q_pos0, float scale,
                                        void* out, float* lse, void* workspace, size_t ws_bytes,
                                        void* stream);

/*
 * Bytes of workspace with which qsa_sparse_attn_prefill_ws can take every path it has for these
 * sizes: the query-tile unions (up to 4096 tiles) and, for the shapes of
 * qsa_sparse_attn_prefill_kv, K and V interleaved by block.  0 for invalid sizes.
 */
QSA_API size_t qsa_attn_prefill_workspace_size(int B, int Tq, int Tk, int Hq, int Hkv, int D, int k_blocks);

/*
 * K and V interleaved by micro-block, the layout qsa_sparse_attn_prefill_kv reads.  (The pages have
 * no counterpart: a layout for the attention's gather, "Qwen3.8-Flash-Next architecture"
 * (flozi.net), "Der Weg eines Tokens durch das Modell", item 2.)
 *   k, v [B][Tk][Hkv][D] bf16  ->  kv [B][ceil(Tk/blk)][2][blk][Hkv][D] bf16
 *   kv[b][j][0][i] = k[b][blk*j + i], kv[b][j][1][i] = v[b][blk*j + i]; positions >= Tk are zero.
 * Writes the blocks that hold positions [pos_lo, pos_hi) (0 <= pos_lo <= pos_hi <= Tk; a block is
 * rewritten whole, so a block that straddles pos_hi also receives the positions after pos_hi that
 * it holds, read from k and v as they are).  D = 128, Hkv in {1, 2}, blk = 4.
 * Errors: INVALID_ARGUMENT (null or misaligned pointer, sizes, blk), UNSUPPORTED (D, Hkv).
 */
QSA_API qsa_status_t qsa_interleave_kv(const void* k, const void* v, void* kv, int B, int Tk, int Hkv, int D,
                                       int blk, int64_t pos_lo, int64_t pos_hi, void* stream);

/*
 * qsa_sparse_attn_prefill over K and V interleaved by block (kv as qsa_interleave_kv writes it, for
 * at least the positions < q_pos0 + Tq): the same arguments otherwise, the same result bit for bit.
 * A block's K and V are one contiguous run, fetched with one copy.  D = 128, Hkv in {1, 2}, groups
 * of up to 8 query heads; other shapes return UNSUPPORTED.
 */
QSA_API qsa_status_t qsa_sparse_attn_prefill_kv(const void* q, const void* kv, const int32_t* idx, int B, int Tq,
                                                int Tk, int Hq, int Hkv, int D, int k_blocks, int blk,
                                                int64_t q_pos0, float scale, void* out, float* lse,
                                                void* stream);

/*
 * Chooses the prefill attention of qsa_sparse_attn_prefill_ws for all later calls from this
 * process: 0 = automatic (row by row, over interleaved K/V when the workspace holds them), 1 = row by
 * row over k and v as given, 2 = query tiles (UNSUPPORTED for other
 * shapes, WORKSPACE_TOO_SMALL without room for one tile).  Errors: INVALID_ARGUMENT (path outside
 * 0..2).
 */
QSA_API qsa_status_t qsa_set_attn_options(int path);

/*
 * The whole QSA layer for one prefill whose inputs and output live in HOST memory
 * ("Qwen3.8-Flash-Next architecture" (flozi.net), "Der Weg eines Tokens durch das Modell", item 2:
 * pooling, block selection and attention over the selected tokens), with the transfers overlapped
 * with the kernels.  (The pages have no host-side counterpart: this is the library's own schedule
 * of the three calls above around the copies.)
 *   host, read:    q [B][Tq][Hq][D], k, v [B][Tk][Hkv][D], qi [B][Tq][Hi][Di], ki [B][Tk][Di] (bf16)
 *   host, written: out [B][Tq][Hq][D] bf16
 *   Host buffers should be page-locked (cudaHostAlloc / cudaHostRegister) for the copies to
 *   overlap; pageable memory gives the same result without the overlap.
 *   Query row t sits at position q_pos0 + t; Tk >= q_pos0 + Tq.  mode, head_w (device, or NULL) and
 *   rope (NULL or theta <= 0: no rotation) as for qsa_select_topk / qsa_pool_block_keys_rope;
 *   scale > 0 as for qsa_sparse_attn_prefill.
 * Schedule (B = 1): ki and qi are sent first in `sel_chunks` causal row chunks and each chunk's
 * pooling and selection starts as soon as it has arrived (only when Tk = q_pos0 + Tq and
 * q_pos0 % 4 == 0; else one chunk); q, k, v follow in causal row chunks (K/V only up to each
 * chunk's last position, each row sent once), each chunk's attention starts when it has arrived
 * and its output rows go back while the next chunk is computed: `chunks` equal chunks, or with
 * chunks == 0 three chunks of a quarter of the rows and then chunks that halve the rest down to
 * about 2048 rows (fewer partial last waves, a small last output copy).  B > 1: one chunk of each.
 * The kernels run on `stream`; the copies on two streams of the library's own (one per direction
 * and device), ordered against `stream` with events.  The call returns once everything is
 * enqueued; `out` is complete when `stream` reaches the point of the call (synchronise it, or
 * record an event after the call).
 * Device memory: `dev` (256-byte aligned, dev_bytes >= qsa_prefill_host_device_bytes(...)) holds
 * the device copies of the inputs, the pooled keys, the rotated queries, the output rows and both
 * workspaces; it must not be used by other work until the call's work on `stream` is done.
 * idx_out [B][Tq][k_blocks] int32 and lse_out [B][Tq][Hq] fp32 (device, may be NULL: then kept in
 * `dev`) receive the index lists and log-sum-exps.
 * Calls on one device enqueue one at a time (a lock); their work may overlap on the GPU only if
 * they use different `dev` buffers.
 * Errors: INVALID_ARGUMENT (null pointer, dev misaligned, sizes, Tk < q_pos0 + Tq, blk != 4,
 * chunks < 0, sel_chunks < 1, scale <= 0), WORKSPACE_TOO_SMALL (dev_bytes), both before anything is
 * enqueued; a failing step (for example UNSUPPORTED for a shape the kernels do not take) returns
 * its own status with the work before it already enqueued; CUDA on a runtime error.
 */
QSA_API qsa_status_t qsa_prefill_host(const void* q, const void* k, const void* v, const void* qi, const void* ki,
                                      void* out, int B, int Tq, int Tk, int Hq, int Hkv, int D, int Hi, int Di,
                                      int k_blocks, int blk, int64_t q_pos0, float scale, qsa_score_mode_t mode,
                                      const float* head_w, const qsa_rope_params_t* rope, int chunks,
                                      int sel_chunks, void* dev, size_t dev_bytes, int32_t* idx_out,
                                      float* lse_out, void* stream);

/*
 * Bytes of the `dev` buffer qsa_prefill_host needs for these sizes (rope: 1 if the indexer RoPE
 * is on).  0 for invalid sizes.  Host arithmetic only.
 */
QSA_API size_t qsa_prefill_host_device_bytes(int B, int Tq, int Tk, int Hq, int Hkv, int D, int Hi, int Di,
                                             int k_blocks, int blk, int64_t q_pos0, int rope, int chunks,
                                             int sel_chunks);

/*
 * Gather-sparse attention, decode (split-KV).  One new token per sequence.
 *   q [B][Hq][D] bf16; caches k, v [B][Lmax][Hkv][D] bf16 holding seqlens[b] tokens (the new
 *   token included, so the query sits at position seqlens[b] - 1); idx [B][k_blocks] int32
 *   -> out [B][Hq][D] bf16, lse [B][Hq] fp32 (may be NULL).
 * The index list of each sequence is cut into num_splits ranges (0 = choose from the GPU size)
 * that run in parallel; their partial softmax states are merged by log-sum-exp: inside the
 * attention kernel when the splits of a sequence can run as one thread-block cluster (D = 128,
 * groups of up to 8 heads, 2 .. 8 splits, B * num_splits <= SMs, every cluster resident at once;
 * the partials meet in distributed shared memory), otherwise by a second kernel over partials in
 * `workspace` (qsa_decode_split_merge tells which).  num_splits > 1 needs workspace >=
 * qsa_workspace_size(QSA_OP_SPARSE_ATTN_DECODE, B, 1, 0, k_blocks, Hq, D, num_splits) bytes
 * either way.
 * Errors: as for prefill, plus WORKSPACE_TOO_SMALL.
 */
QSA_API qsa_status_t qsa_sparse_attn_decode(const void* q, const void* kcache, const void* vcache,
                                    const int32_t* seqlens, const int32_t* idx, int B, int Lmax,
                                    int Hq, int Hkv, int D, int k_blocks, int blk, float scale,
                                    int num_splits, void* out, float* lse, void* workspace,
                                    size_t ws_bytes, void* stream);

/*
 * Decode attention for callers that cannot allocate device memory.
 * (No counterpart on the pages: this is a deployment variant of qsa_sparse_attn_decode.)
 * Some callers have no way to hand the library a workspace: code that runs while a stream is
 * being captured into a CUDA graph (cudaMalloc is not allowed there), plugins of inference
 * engines whose memory planner owns the whole device heap, and embedded hosts with a fixed device
 * budget.  This entry point takes the same inputs and outputs as qsa_sparse_attn_decode but keeps
 * the per-split partial results in a scratch array that is part of the library image itself
 * (QSA_NOALLOC_DECODE_SCRATCH_BYTES per GPU, held by every GPU that loads the library until the
 * process exits).  It calls no allocator.
 *   - num_splits == 0 picks the largest split count up to qsa_decode_default_splits that fits the
 *     array.  An explicit num_splits is first capped at max(k_blocks, 1), as in
 *     qsa_sparse_attn_decode; if the capped count s > 1 needs partials, B * s * Hq * (D + 2) * 4
 *     bytes, beyond QSA_NOALLOC_DECODE_SCRATCH_BYTES, the call returns QSA_ERR_WORKSPACE_TOO_SMALL.
 *   - The array is read only when the splits merge through partials (qsa_decode_split_merge
 *     returns 2); when they merge inside thread-block clusters it is not touched.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress) with
 *     that device current; make that first call before any stream capture that should contain it.
 *   - Every call, on every stream, shares the one array per device: calls whose kernels overlap on
 *     the GPU race and corrupt each other's partials.  Serialise them (one stream, or events).
 *   - Each call overwrites every partial it later reads, so nothing has to be cleared between
 *     calls even though the array keeps the previous call's contents.
 */
#define QSA_NOALLOC_DECODE_SCRATCH_BYTES (4u << 20)
QSA_API qsa_status_t qsa_sparse_attn_decode_noalloc(const void* q, const void* kcache,
                                                    const void* vcache, const int32_t* seqlens,
                                                    const int32_t* idx, int B, int Lmax, int Hq,
                                                    int Hkv, int D, int k_blocks, int blk,
                                                    float scale, int num_splits, void* out,
                                                    float* lse, void* stream);

/*
 * Workspace bytes for `op`.  QSA_OP_SELECT_TOPK: B, Tq, NBk (a chunk of score rows, capped);
 * QSA_OP_SPARSE_ATTN_DECODE: B, Hq, D, num_splits (0 = the count the call would choose).
 * Returns 0 for an unknown op or invalid sizes.
 */
QSA_API size_t qsa_workspace_size(qsa_op_t op, int B, int Tq, int NBk, int k, int Hq, int D,
                          int num_splits);

/* Split count qsa_sparse_attn_decode picks for num_splits == 0 on the current device. */
QSA_API int qsa_decode_default_splits(int B, int k_blocks);

/*
 * How qsa_sparse_attn_decode merges num_splits (>= 1, as passed after the default is resolved)
 * splits on the current device: 0 = one split, nothing to merge; 1 = inside the attention
 * kernel (thread-block clusters, one launch); 2 = a second kernel over partials in the
 * workspace.  -1 on invalid sizes or without a usable device.
 */
QSA_API int qsa_decode_split_merge(int B, int Hq, int Hkv, int D, int num_splits);

/*
 * Synchronises `stream`, then reads and clears the current device's status word:
 * QSA_OK, QSA_ERR_INVALID_ARGUMENT (an index or sequence length was out of range and skipped),
 * QSA_ERR_TIMEOUT (a device-side wait ran out of time and the kernel returned early),
 * QSA_ERR_DEVICE_CHECK (debug build: a device-side bounds check failed), or
 * QSA_ERR_CUDA (the synchronisation itself failed).
 */
QSA_API qsa_status_t qsa_get_device_status(void* stream);

/*
 * Chooses how qsa_select_topk computes a prefill selection when it is not given scores, for all
 * later calls from this process: path 0 = automatic (default), 1 = materialised scores,
 * 2 = filtered (UNSUPPORTED unless Hi is 4 or 8 and k <= 1024).  sample_rank > 0 replaces the filtered path's
 * rank of the threshold among a row's samples (a testing and tuning knob: a small rank makes
 * short lists and a large one overflowing lists, both redone exactly); 0 restores the default.
 * Errors: INVALID_ARGUMENT (path outside 0..2, sample_rank < 0).
 */
QSA_API qsa_status_t qsa_set_select_options(int path, int sample_rank);

/*
 * Device-side wait limit in nanoseconds for all later launches from this process (default
 * 2e9 = 2 s; 0 restores the default).  Every spin on an mbarrier in the kernels gives up after
 * this long, records QSA_ERR_TIMEOUT and returns.
 */
QSA_API void qsa_set_wait_timeout_ns(uint64_t ns);

/*
 * Self-test of the bounded waits: launches one CTA that waits on an mbarrier no thread ever
 * completes, with a `timeout_ns` limit.  Afterwards qsa_get_device_status returns
 * QSA_ERR_TIMEOUT and the context stays usable.
 */
QSA_API qsa_status_t qsa_wait_timeout_selftest(uint64_t timeout_ns, void* stream);

/*
 * Gather-rate probe (measurement only; not a step of the method).  The sparse attention fetches
 * every selected 4-token block of K and of V as one scattered chunk (2 KB at 2 KV heads x D 128)
 * into a shared-memory ring; this call measures how fast the SMs can do that alone, which is the
 * ceiling the attention's gather is compared with.  `ctas` CTAs (0 = one per SM) of `issuer_warps`
 * warps each keep `stages` x `slots_per_warp` chunks in flight per warp and refill them
 * `iterations` times from pseudo-random chunk-aligned offsets of src [src_bytes] (device memory,
 * 16-byte aligned; a buffer that fits in L2 gives the L2 -> SM ceiling).  method 0: 1-D bulk copies
 * (TMA engine, one per chunk); 1: 16-byte cp.async by every lane; 2: the two alternating by warp;
 * 3 and 4: tiled tensor copies with the 128-byte swizzle from src viewed as [tokens][2][128] bf16,
 * one box of [4 tokens][1 head][64] (chunk_bytes must be 512) or [4 tokens][2 heads][64] (1024).
 * Bytes delivered = CTAs * issuer_warps * iterations * slots_per_warp * chunk_bytes; time the
 * launch with events on `stream`.  The landed data are not read.
 * Errors: INVALID_ARGUMENT (null or misaligned src, chunk_bytes not a multiple of 16 in 16 .. 16384
 * or above src_bytes, method outside 0..4, issuer_warps outside 1..16, slots_per_warp outside
 * 1..32), UNSUPPORTED (stages outside 2..4, ring above 227 KB of shared memory).
 */
QSA_API qsa_status_t qsa_probe_gather(const void* src, size_t src_bytes, int chunk_bytes, int method,
                                      int issuer_warps, int stages, int slots_per_warp, int iterations,
                                      int ctas, uint64_t seed, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* QSA_H */
