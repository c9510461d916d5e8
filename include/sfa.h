/*
 * sfa.h - C ABI of libsfa: top-k sparse attention backward (SparseFlashAttentionGrad),
 * the dense varlen FlashAttention backward (FlashAttentionUnpaddingScoreGrad) and
 * the dense lightning-indexer gradient with KL loss (DenseLightningIndexerGradKLLoss)
 * for NVIDIA B200 (sm_100a).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every tensor argument is a DEVICE pointer to densely packed (contiguous,
 *    row-major) memory in the layout stated for it, unless the comment says
 *    "host".  The caller owns every buffer: inputs, outputs and workspace.
 *    The library allocates nothing and never synchronizes the stream.
 *  - Inputs are never written.  `value` may be the same pointer as `key`.
 *  - Outputs are fully overwritten (no accumulation into caller memory).
 *  - Two phases, as in the aclnn convention of the FlashAttentionUnpaddingScoreGrad
 *    page (函数原型 / 返回值): *_workspace_size() validates the arguments on the host
 *    and returns the workspace size; the compute call re-validates, then enqueues
 *    kernels on `stream` (a cudaStream_t; NULL = legacy default stream) and returns.
 *  - Errors are reported before any launch and leave outputs untouched:
 *      SFA_ERR_NULLPTR   a required pointer is NULL
 *      SFA_ERR_INVALID   shape / attribute outside the supported set
 *      SFA_ERR_WORKSPACE workspace_bytes smaller than the size query returned
 *      SFA_ERR_CUDA      a CUDA launch or copy failed (see sfa_last_error_string)
 *  - Out-of-range sparse index values and inconsistent sequence lengths are
 *    masked on the device (the affected keys are skipped); they never fault.
 *  - Not thread-safe for concurrent calls that share one workspace.
 */
#ifndef SFA_H_
#define SFA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t sfa_status;
#define SFA_OK 0
#define SFA_ERR_NULLPTR 161001   /* same codes as ACLNN_ERR_PARAM_NULLPTR / _INVALID */
#define SFA_ERR_INVALID 161002
#define SFA_ERR_WORKSPACE 161003
#define SFA_ERR_CUDA 161004
#define SFA_ERR_TIMEOUT 161005

#define SFA_LAYOUT_BSND 0
#define SFA_LAYOUT_TND 1

#define SFA_DTYPE_BF16 0
#define SFA_DTYPE_FP16 1

typedef struct CUstream_st *sfa_stream_t; /* == cudaStream_t */

/*
 * Problem sizes of a sparse attention call (SparseFlashAttentionGrad README,
 * 参数说明 and 约束说明).
 *   layout  SFA_LAYOUT_BSND: query [B,S1,N1,D], key/value [B,S2,N2,D],
 *                            queryRope [B,S1,N1,Dr], keyRope [B,S2,N2,Dr],
 *                            sparseIndices [B,S1,N2,topk], softmax stats [B,S1,N1];
 *                            T1/T2 are ignored (taken as B*S1, B*S2).
 *           SFA_LAYOUT_TND:  query [T1,N1,D], key/value [T2,N2,D], queryRope
 *                            [T1,N1,Dr], keyRope [T2,N2,Dr], sparseIndices
 *                            [T1,N2,topk], softmax stats [T1,N1]; S1/S2 ignored.
 *   dtype   SFA_DTYPE_BF16 or SFA_DTYPE_FP16 for every 16-bit tensor.
 *   Supported: N2 = 1, D = 512, Dr = 64, N1 in {1,2,4,...,128}, B in [1,256],
 *   S1, S2 (or per-sequence lengths) in [1, 128K], topk >= 1.
 */
typedef struct sfa_shape {
    int32_t layout;
    int32_t dtype;
    int64_t B;
    int64_t S1, S2;
    int64_t T1, T2;
    int64_t N1, N2;
    int64_t D, Dr;
    int64_t topk;
} sfa_shape;

/* ------------------------------------------------------------------------- */
/* Sparse attention backward                                                  */
/* ------------------------------------------------------------------------- */

/*
 * Phase 1 of sfa_grad: validate `shape` and the attributes, return the device
 * workspace size in *workspace_bytes.  Host only, no device work.
 * sparse_mode: 0 (no mask) or 3 (lower triangle split at the right vertex,
 * i.e. key j kept for query position i iff j <= i + S2_b - S1_b), per the
 * 约束说明 of the SparseFlashAttentionGrad README.
 */
sfa_status sfa_grad_workspace_size(const sfa_shape *shape, int64_t sparse_block_size, int64_t sparse_mode,
                                   int32_t deterministic, size_t *workspace_bytes);

/*
 * Phase 2: the training backward of top-k sparse attention (SparseFlashAttentionGrad
 * README, 功能说明): per query token, gather the key/value rows named by
 * sparseIndices in blocks of sparse_block_size, recompute
 *     P  = exp(scale * [q||qRope].[k||kRope]^T - softmaxMax) / softmaxSum,
 * then dP = dOut.V^T, dS = P o (dP - rowsum(dOut o out)),
 *      dQuery||dQueryRope = scale * dS.[k||kRope],
 *      dKey||dKeyRope    += scale * dS^T.[q||qRope],   dValue += P^T.dOut,
 * the key-side sums scatter-added in fp32 and cast once at the end.
 *
 *   query, query_rope, d_out, out   [.., N1, D|Dr] 16-bit, see sfa_shape
 *   key, value, key_rope            [.., N2=1, D|Dr] 16-bit; value may == key
 *   sparse_indices                  int32 [.., N2, topk]; entry i selects rows
 *                                   [i*bs, i*bs+bs) of the token's own batch
 *                                   (BSND) or sequence (TND); negative entries
 *                                   and blocks starting at/after S2_b are skipped,
 *                                   duplicates count with multiplicity
 *   softmax_max, softmax_sum        fp32 [.., N1]: max of the scaled scores and
 *                                   sum of exp(scaled - max) from the forward,
 *                                   used as given; softmax_sum == 0 gives P = 0
 *   actual_seq_lengths_q / _kv      int32, device.  BSND: per-batch valid lengths
 *                                   (length B) or NULL for S1/S2.  TND: required,
 *                                   cumulative end offsets (length B, last = T1/T2)
 *   scale                           scaleValue (applied in S, dQuery, dKey)
 *   pre_tokens, next_tokens         accepted and ignored (no effect for modes 0/3)
 *   deterministic                   0: fp32 atomic scatter (run-to-run order may
 *                                   differ); 1: bit-identical results run to run:
 *                                   the key-side sums are 64-bit fixed point on a
 *                                   power-of-two grid chosen per call from
 *                                   max|d_out|, T1*N1 and scale (dValue: 2^-e with
 *                                   e = 54 - ceil(log2(T1*N1)) - E(max|d_out|);
 *                                   dKey/dKeyRope: e = 42 - ceil(log2(T1*N1)) -
 *                                   E(max|d_out|) - E(|scale|), E(x) the least k
 *                                   with x <= 2^k).  Scaling d_out by 2^k scales
 *                                   the results by exactly 2^k, so the precision
 *                                   does not depend on the gradient's magnitude.
 *                                   The grid leaves 2^8 of range for dValue over
 *                                   the bound T1*N1*max|d_out| (which holds when
 *                                   softmax_max/_sum are the forward's statistics,
 *                                   so that every row's P sums to 1) and about 2^11
 *                                   for dKey over unit-scale activations; inputs
 *                                   outside that range may saturate.
 *   workspace, workspace_bytes      >= sfa_grad_workspace_size(); 256-byte aligned
 *   d_query, d_query_rope           [.., N1, D|Dr] 16-bit outputs; rows of BSND
 *                                   padding tokens (position >= S1_b) are zero
 *   d_key, d_value, d_key_rope      [.., N2, D|Dr] 16-bit outputs; d_key excludes
 *                                   d_value's share even when value == key
 */
sfa_status sfa_grad(const void *query, const void *key, const void *value, const int32_t *sparse_indices,
                    const void *d_out, const void *out, const float *softmax_max, const float *softmax_sum,
                    const int32_t *actual_seq_lengths_q, const int32_t *actual_seq_lengths_kv,
                    const void *query_rope, const void *key_rope, float scale, int64_t sparse_block_size,
                    int64_t sparse_mode, int64_t pre_tokens, int64_t next_tokens, int32_t deterministic,
                    const sfa_shape *shape, void *workspace, size_t workspace_bytes, sfa_stream_t stream,
                    void *d_query, void *d_key, void *d_value, void *d_query_rope, void *d_key_rope);

/*
 * Query-row sharding of sfa_grad (for data parallelism over query rows with a
 * replicated key/value: each GPU runs its own rows, then the key-side sums are
 * added across GPUs).  The pages' operator runs all rows at once; splitting it
 * this way computes the same sums (SparseFlashAttentionGrad README, 功能说明:
 * dKey / dValue are sums over every query row that selected a key, so partial
 * sums over disjoint row sets add up to the whole).
 *
 * sfa_dkv_accum_size - bytes of the key-side accumulator: [T2][1088] (columns
 * dKey 0-511 | dKeyRope 512-575 | dValue 576-1087), fp32 when deterministic == 0,
 * int64 fixed point (the grid of sfa_grad's deterministic mode) when 1.  Host only.
 */
sfa_status sfa_dkv_accum_size(const sfa_shape *shape, int32_t deterministic, size_t *accum_bytes);

/*
 * sfa_grad_rows - sfa_grad restricted to query rows [row_begin, row_end) of the
 * flattened [T1] row index (BSND: b * S1 + s; TND: the token index).
 *   - Same inputs, workspace and validation as sfa_grad; 0 <= row_begin <=
 *     row_end <= T1, else SFA_ERR_INVALID before any device work.
 *   - Of sparse_indices, query, query_rope, d_out, out, softmax_max and
 *     softmax_sum only the range's rows are read (a pipeline may copy the other
 *     rows while this call runs); key / key_rope are read whole.
 *   - d_query / d_query_rope: the rows in the range are written (zero for rows
 *     with no selected key); rows outside the range are not touched.
 *   - dkv_accum (caller-owned, 256-byte aligned, sfa_dkv_accum_size bytes): the
 *     range's dKey | dKeyRope | dValue contributions are ADDED to it; the caller
 *     zeroes it before the first range and may add accumulators of other ranges
 *     (other GPUs) element-wise before sfa_dkv_finalize.  With deterministic == 1
 *     the accumulator is integer, so that element-wise addition is exact and
 *     order-independent; when every range boundary is an even row the final
 *     outputs are bit-identical to sfa_grad's (N1 = 128 processes rows 2m and
 *     2m + 1 with identical block lists as one pair, whose key-side sums are
 *     formed together: a boundary between them changes the rounding, not the
 *     tolerance).
 *   - dout_absmax (device fp32, deterministic mode only; may be NULL otherwise):
 *     max|d_out| over EVERY row whose contributions go into this accumulator (on
 *     every GPU), which fixes the fixed-point grid: zero it, add each range with
 *     sfa_dout_absmax and, across GPUs, combine the values with a max-reduction
 *     before the first sfa_grad_rows call.  All calls on one accumulator (and
 *     sfa_dkv_finalize) must see the same value and the same scale.
 *   - Enqueued on `stream`; nothing is allocated and nothing synchronizes.
 */
sfa_status sfa_grad_rows(const void *query, const void *key, const void *value, const int32_t *sparse_indices,
                         const void *d_out, const void *out, const float *softmax_max, const float *softmax_sum,
                         const int32_t *actual_seq_lengths_q, const int32_t *actual_seq_lengths_kv,
                         const void *query_rope, const void *key_rope, float scale, int64_t sparse_block_size,
                         int64_t sparse_mode, int32_t deterministic, int64_t row_begin, int64_t row_end,
                         const sfa_shape *shape, void *workspace, size_t workspace_bytes, sfa_stream_t stream,
                         void *dkv_accum, const float *dout_absmax, void *d_query, void *d_query_rope);

/*
 * sfa_dout_absmax - max-merges max|d_out| over query rows [row_begin, row_end)
 * into *dout_absmax (device fp32, caller-zeroed before the first range).  The
 * value sets the fixed-point grid of deterministic row ranges (sfa_grad_rows).
 */
sfa_status sfa_dout_absmax(const void *d_out, const sfa_shape *shape, int64_t row_begin, int64_t row_end,
                           sfa_stream_t stream, float *dout_absmax);

/*
 * sfa_dkv_finalize - casts a (summed) key-side accumulator into the 16-bit
 * d_key [.., N2, D], d_value [.., N2, D] and d_key_rope [.., N2, Dr] outputs
 * (round to nearest even; fixed point is scaled back by its grid first).
 * `shape` gives T1, N1, T2 and the dtype; `deterministic` selects the
 * accumulator format; dout_absmax and scale must be the ones the accumulator
 * was filled with (dout_absmax may be NULL when deterministic == 0).
 */
sfa_status sfa_dkv_finalize(const void *dkv_accum, const sfa_shape *shape, int32_t deterministic,
                            const float *dout_absmax, float scale, sfa_stream_t stream, void *d_key, void *d_value,
                            void *d_key_rope);

/*
 * sfa_grad_noalloc - sfa_grad for callers that cannot allocate device memory.
 * (The source pages have no counterpart: it exists for this library's callers.)
 *
 * Some callers cannot supply a workspace: code running under another
 * framework's memory pool (a raw allocation would escape its accounting),
 * plugins and embedded runtimes that are handed only input and output buffers,
 * and code where allocating would synchronize the device.  This call takes the
 * same arguments as sfa_grad minus the workspace, and allocates nothing: its
 * scratch is a 64 MiB array that is part of the library's device image, so
 * every GPU that loads the library holds those 64 MiB until the process exits.
 *  - Computes with the CUDA-core backward kernel; results match sfa_grad within
 *    the bf16 tolerance (and are bit-identical run to run when deterministic).
 *  - Problems whose scratch would exceed 64 MiB (the dKey/dValue accumulator,
 *    T2 x 1088 x 4 bytes, or x 8 when deterministic, plus T1 x topk x 4 bytes of
 *    index tables) are rejected with SFA_ERR_WORKSPACE before any device work.
 *  - The first call on each device looks up the array's device address with
 *    cudaGetSymbolAddress (with that device current) and keeps it for the life
 *    of the process; make that first call before any stream capture on the
 *    device.  Calls after a reset of the device (cudaDeviceReset, or the primary
 *    context being torn down and re-created) are not supported: the kept address
 *    belongs to the old context.
 *  - All calls on a device share the array, which keeps the previous call's
 *    contents (the accumulator is cleared on the call's stream).  Calls whose
 *    work overlaps on the GPU (other streams, other threads) race on it and
 *    must be serialized by the caller.
 */
sfa_status sfa_grad_noalloc(const void *query, const void *key, const void *value, const int32_t *sparse_indices,
                            const void *d_out, const void *out, const float *softmax_max, const float *softmax_sum,
                            const int32_t *actual_seq_lengths_q, const int32_t *actual_seq_lengths_kv,
                            const void *query_rope, const void *key_rope, float scale, int64_t sparse_block_size,
                            int64_t sparse_mode, int64_t pre_tokens, int64_t next_tokens, int32_t deterministic,
                            const sfa_shape *shape, sfa_stream_t stream, void *d_query, void *d_key, void *d_value,
                            void *d_query_rope, void *d_key_rope);

/* ------------------------------------------------------------------------- */
/* Sparse attention forward (produces the inputs `out`, softmax_max/_sum)     */
/* ------------------------------------------------------------------------- */

sfa_status sfa_fwd_workspace_size(const sfa_shape *shape, int64_t sparse_block_size, int64_t sparse_mode,
                                  size_t *workspace_bytes);

/*
 * Forward of the same attention (FlashAttentionUnpaddingScoreGrad page, 计算公式:
 * S = scale*Q.K^T, P = Softmax(S), Y = P.V) over the gathered rows:
 *   out [.., N1, D] 16-bit, softmax_max / softmax_sum fp32 [.., N1] (max of the
 *   scaled scores, sum of exp(scaled - max)).  A query row with no valid key
 *   gets out = 0, softmax_max = 0, softmax_sum = 0.  Arguments as in sfa_grad.
 */
sfa_status sfa_fwd(const void *query, const void *key, const void *value, const int32_t *sparse_indices,
                   const int32_t *actual_seq_lengths_q, const int32_t *actual_seq_lengths_kv,
                   const void *query_rope, const void *key_rope, float scale, int64_t sparse_block_size,
                   int64_t sparse_mode, const sfa_shape *shape, void *workspace, size_t workspace_bytes,
                   sfa_stream_t stream, void *out, float *softmax_max, float *softmax_sum);

/* ------------------------------------------------------------------------- */
/* Hot-path sub-steps, exported for bit-exact testing and reuse               */
/* ------------------------------------------------------------------------- */

/*
 * Index compaction (the Gather of the SparseFlashAttentionGrad README, 功能说明,
 * with the sparseMode mask of its 约束说明): for each query row t, copy the valid
 * block indices of sparse_indices[t, 0, :] in their original order to
 * blocks_out[t*topk + 0 .. n-1] (the rest is left unwritten), the count n to
 * nblocks_out[t] and the number of valid key rows (after the S2_b cut and the
 * mode-3 causal cut, row by row) to nrows_out[t].  A block is valid iff its
 * index i >= 0, i*bs < S2_b and, in mode 3, i*bs <= pos + S2_b - S1_b.  BSND
 * padding rows (position >= S1_b) get n = 0.  All outputs int32, device.
 */
sfa_status sfa_compact_indices(const int32_t *sparse_indices, const int32_t *actual_seq_lengths_q,
                               const int32_t *actual_seq_lengths_kv, int64_t sparse_block_size, int64_t sparse_mode,
                               const sfa_shape *shape, sfa_stream_t stream, int32_t *blocks_out,
                               int32_t *nblocks_out, int32_t *nrows_out);

/*
 * The gathered key rows of every query row, as the fused kernels read them
 * (the Gather of the SparseFlashAttentionGrad README, 功能说明: an index i selects
 * rows [i*bs, i*bs+bs) of the token's batch / sequence, cut by S2_b and by the
 * sparseMode 3 bound of 约束说明).  Runs the index compaction (outputs as in
 * sfa_compact_indices), optionally sorts each row's kept blocks ascending
 * (sorted != 0; topk <= 4096), then expands the blocks into global key-row ids
 * (flattened [T2] view):
 *   block_aligned == 0: rows_out[t*topk*bs + 0 .. n-1] = the kept rows in block
 *     order, count_out[t] = n (the row count of sfa_compact_indices);
 *   block_aligned != 0: block i of row t takes slots [i*bs, i*bs+bs) holding the
 *     block's consecutive rows, slots past the block's kept rows carrying the row
 *     id with bit 31 set; count_out[t] = blocks * bs.
 * blocks_out [T1*topk], nblocks_out / count_out [T1], rows_out [T1*topk*bs]:
 * int32, device.  Slots past count_out[t] are left unwritten.
 */
sfa_status sfa_key_rows(const int32_t *sparse_indices, const int32_t *actual_seq_lengths_q,
                        const int32_t *actual_seq_lengths_kv, int64_t sparse_block_size, int64_t sparse_mode,
                        const sfa_shape *shape, int32_t sorted, int32_t block_aligned, sfa_stream_t stream,
                        int32_t *blocks_out, int32_t *nblocks_out, int32_t *rows_out, int32_t *count_out);

/*
 * FlashSoftmaxGrad(dO, O) of stage 2 (SparseFlashAttentionGrad README): the fp32
 * row sum over the D value dims of dOut o out, one value per (query row, head):
 * rowsum_out fp32 [T1, N1] (BSND: [B*S1, N1]).
 */
sfa_status sfa_softmax_grad_rowsum(const void *d_out, const void *out, const sfa_shape *shape, sfa_stream_t stream,
                                   float *rowsum_out);

/* ------------------------------------------------------------------------- */
/* Dense varlen FlashAttention backward (TND), FlashAttentionUnpaddingScoreGrad */
/* ------------------------------------------------------------------------- */

typedef struct fa_shape {
    int32_t dtype; /* SFA_DTYPE_BF16 | SFA_DTYPE_FP16 */
    int32_t reserved;
    int64_t B;     /* number of sequences */
    int64_t T1, T2;
    int64_t Nq, Nkv; /* Nq % Nkv == 0 (GQA), 1..256 */
    int64_t D;       /* head dim, multiple of 8, 8..256 */
} fa_shape;

sfa_status fa_grad_workspace_size(const fa_shape *shape, int64_t sparse_mode, int32_t deterministic,
                                  size_t *workspace_bytes);

/*
 * aclnnFlashAttentionUnpaddingScoreGrad (计算公式): with S = scale*Q.K^T (kept pairs
 * only), P = exp(S - softmaxMax)/softmaxSum, dV = P^T.dY,
 * dS = P o (dY.V^T - rowsum(dY o attentionIn)), dQ = scale*dS.K, dK = scale*dS^T.Q;
 * query head h uses kv head h / (Nq/Nkv) and kv gradients sum over their heads.
 *   q, dy, attention_in [T1, Nq, D]; k, v [T2, Nkv, D]; dq [T1,Nq,D]; dk, dv
 *   [T2,Nkv,D] (16-bit).  softmax_max / softmax_sum fp32 [T1, Nq, 8] (8 equal
 *   copies, lane 0 read), as in 关于softmaxMax与softmaxSum参数的约束.
 *   actual_seq_qlen / actual_seq_kvlen: HOST int64 arrays of length B holding
 *   cumulative end offsets (last = T1 / T2); copied into the workspace before
 *   the call returns.  keep_prob must be 1 (no dropout); pre/next_tokens are
 *   ignored for sparse_mode 0 / 3; head_num must equal Nq.
 *   deterministic: 0 fp32 atomics; 1 bit-identical run to run, every atomically
 *   summed gradient in 64-bit fixed point on the per-call grid of sfa_grad's
 *   deterministic mode (max|dy|, T1 * Nq/Nkv and scale; dq: e = 42 - E(max|dy|)
 *   - E(|scale|)).
 */
sfa_status fa_grad(const void *q, const void *k, const void *v, const void *dy, const float *softmax_max,
                   const float *softmax_sum, const void *attention_in, const int64_t *actual_seq_qlen,
                   const int64_t *actual_seq_kvlen, double scale, double keep_prob, int64_t pre_tokens,
                   int64_t next_tokens, int64_t head_num, int64_t sparse_mode, int32_t deterministic,
                   const fa_shape *shape, void *workspace, size_t workspace_bytes, sfa_stream_t stream, void *dq,
                   void *dk, void *dv);

sfa_status fa_fwd_workspace_size(const fa_shape *shape, int64_t sparse_mode, size_t *workspace_bytes);

/* Forward of the dense attention above: out [T1,Nq,D] 16-bit, softmax_max /
 * softmax_sum fp32 [T1, Nq, 8] (8 equal copies).  Host cumulative seqlens as in fa_grad. */
sfa_status fa_fwd(const void *q, const void *k, const void *v, const int64_t *actual_seq_qlen,
                  const int64_t *actual_seq_kvlen, double scale, int64_t sparse_mode, const fa_shape *shape,
                  void *workspace, size_t workspace_bytes, sfa_stream_t stream, void *out, float *softmax_max,
                  float *softmax_sum);

/* ------------------------------------------------------------------------- */
/* Dense lightning-indexer gradient with KL loss (DenseLightningIndexerGradKLLoss) */
/* ------------------------------------------------------------------------- */

/*
 * Problem sizes of an indexer-gradient call.
 *   layout  SFA_LAYOUT_BSND: query [B,S1,N1,D], queryRope [B,S1,N1,Dr], key [B,S2,1,D],
 *                            keyRope [B,S2,1,Dr], queryIndex [B,S1,G,Di], keyIndex
 *                            [B,S2,1,Di], weights [B,S1,G], softmaxMax/Sum [B,S1,N1],
 *                            softmaxMaxIndex/SumIndex [B,S1]; T1/T2 ignored.
 *           SFA_LAYOUT_TND:  the same with [T1,...] / [T2,...] leading dims; S1/S2 ignored.
 *   Supported: D = 512, Dr = 64 (the main attention's MLA shape, one key head),
 *   N1 in {64, 128}, G = 64, Di = 128 (one indexer key head), B in [1, 256].
 */
typedef struct lig_shape {
    int32_t layout;
    int32_t dtype;  /* SFA_DTYPE_BF16 | SFA_DTYPE_FP16 for every 16-bit tensor */
    int64_t B;
    int64_t S1, S2;
    int64_t T1, T2;
    int64_t N1;     /* main-attention query heads */
    int64_t D, Dr;
    int64_t G;      /* indexer query heads */
    int64_t Di;     /* indexer head dim */
} lig_shape;

sfa_status lig_kl_grad_workspace_size(const lig_shape *shape, int64_t sparse_mode, size_t *workspace_bytes);

/*
 * DenseLightningIndexerGradKLLoss README (功能说明, formulas 1-4; 参数说明 for the
 * argument list).  Per query token t and every key row j it sees (sparse_mode 0:
 * its whole batch / sequence; 3: j <= pos + S2_b - S1_b):
 *   I_tj  = sum_g W[t,g] ReLU(queryIndex[t,g] . keyIndex[j])
 *   p_tj  = (1/N1) sum_h exp(scale * Q~[t,h].K~[j] - softmaxMax[t,h]) / softmaxSum[t,h]
 *           (Q~ = query || queryRope, K~ = key || keyRope; a softmaxSum of 0 gives 0)
 *   sI_tj = exp(I_tj - softmaxMaxIndex[t]) / softmaxSumIndex[t]
 *   loss  = sum_t sum_j p_tj (log p_tj - log sI_tj)          (0 where p = 0)
 *   dI    = sI - p;  dWeights[t,g] = sum_j dI_tj ReLU(S_tgj)   (S = queryIndex . keyIndex)
 *   dQueryIndex[t,g] = sum_j dI_tj W[t,g] [S_tgj > 0] keyIndex[j]
 *   dKeyIndex[j]     = sum_{t,g} dI_tj W[t,g] [S_tgj > 0] queryIndex[t,g]
 * Statistics are used as given (they are the forward's outputs).  A token with no
 * visible key (BSND padding rows included) gets zero dQueryIndex / dWeights rows.
 *   actual_seq_lengths_query / _key: DEVICE int64 [B] (the page's INT64 tensors):
 *     BSND per-batch valid lengths (NULL = S1 / S2), TND cumulative end offsets
 *     (required).  pre_tokens / next_tokens are ignored (modes 0 and 3 only).
 *   Outputs: d_query_index [.., G, Di], d_key_index [.., 1, Di], d_weights [.., G]
 *     (16-bit), loss: one fp32 (device).  dKeyIndex is summed with fp32 atomics
 *     (run-to-run differences in the last bits); loss is a fixed-order sum.
 *   The 16-bit inputs must be 16-byte aligned (they are read by TMA) and the
 *   workspace 256-byte aligned (SFA_ERR_INVALID otherwise).
 */
sfa_status lig_kl_grad(const void *query, const void *key, const void *query_index, const void *key_index,
                       const void *weights, const float *softmax_max, const float *softmax_sum,
                       const float *softmax_max_index, const float *softmax_sum_index, const void *query_rope,
                       const void *key_rope, const int64_t *actual_seq_lengths_query,
                       const int64_t *actual_seq_lengths_key, double scale, int64_t sparse_mode, int64_t pre_tokens,
                       int64_t next_tokens, const lig_shape *shape, void *workspace, size_t workspace_bytes,
                       sfa_stream_t stream, void *d_query_index, void *d_key_index, void *d_weights, float *loss);

/* ------------------------------------------------------------------------- */
/* Diagnostics                                                                */
/* ------------------------------------------------------------------------- */

/*
 * Timing hook for benchmarks: the next sfa_grad / sfa_grad_rows / sfa_fwd /
 * fa_grad / lig_kl_grad call on the calling thread records `event_before` immediately before
 * and `event_after` immediately after launching its main kernel (the fused
 * tensor-core kernel or the CUDA-core kernel), on that call's stream.  Both are cudaEvent_t
 * handles created by the caller; NULL clears the hook.  Consumed by one call.
 */
sfa_status sfa_set_kernel_events(void *event_before, void *event_after);

/*
 * Failure detection.  Every wait of the fused kernels on an mbarrier (a load, an
 * MMA or another warp role) is bounded: past the limit the kernel writes a
 * non-zero wait-site code into its workspace's error word (the first 4 bytes of
 * the workspace of sfa_grad / sfa_grad_rows / sfa_fwd / fa_grad / fa_fwd /
 * lig_kl_grad, zeroed
 * at the start of each such call), stops issuing work, drains what it issued,
 * frees its tensor memory and exits; the CUDA context stays usable.  (The pages
 * name only an AI Core "timeout or trap" error for oversized problems, 约束说明 of
 * aclnnFlashAttentionUnpaddingScoreGrad.)
 *
 * sfa_workspace_status - synchronizes `stream`, reads the error word of
 * `workspace` (device pointer) and returns SFA_OK, or SFA_ERR_TIMEOUT with the
 * wait-site code in *site_out (may be NULL) when the last call on it gave up.
 *
 * sfa_set_wait_limit - limit in nanoseconds of every such wait in fused kernels
 * launched afterwards from the calling thread; 0 restores the default (4 s).
 * A tiny limit (the tests use 1 ns) makes a launch give up at its first wait that is
 * not already satisfied, which exercises the path above without any fault.
 */
sfa_status sfa_workspace_status(const void *workspace, sfa_stream_t stream, int32_t *site_out);
sfa_status sfa_set_wait_limit(uint64_t limit_ns);

/* Static string naming a status code. */
const char *sfa_status_string(sfa_status status);
/* Message of the last error on the calling thread ("" if none). */
const char *sfa_last_error_string(void);
/* Library version, "major.minor.patch". */
const char *sfa_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SFA_H_ */
