/*
 * attn.h -- C ABI of libattn.so: scaled-dot-product attention forward on NVIDIA B200 (sm_100a).
 *
 * The operations, each an asynchronous launch on the caller's CUDA stream:
 *
 *   attn_fwd         O = softmax(scale * Q K^T + mask) V, with per-row softmax max and sum.
 *   attn_sparse_csr  the same softmax restricted to the entries of a CSR pattern (fp32).
 *   attn_merge       merge of two partial attention results from their max/sum statistics.
 *   attn_fwd_accumulate  attn_fwd over one chunk of keys folded into a running merge result.
 *   attn_fwd_masked  attn_fwd with band limits, an explicit mask and a value head size Dv.
 *   attn_sparse_csr_tc  attn_sparse_csr in bf16 / fp16 on the tensor cores.
 *   attn_csr_plan    the pattern bookkeeping of attn_sparse_csr_tc, once per pattern, into a
 *                    caller-owned buffer that attn_sparse_csr_tc_planned then reads.
 *
 * Conventions shared by every call
 *   - All tensor pointers are DEVICE pointers owned by the caller. The library allocates no
 *     device memory, keeps no reference to any argument after the call returns, and never
 *     synchronises the stream (except attn_get_last_error, which says so).
 *   - Tensors are dense and contiguous in the layout stated for each argument (row-major,
 *     last index fastest).
 *   - `stream` is a cudaStream_t passed as void*; NULL means the legacy default stream.
 *   - Shape and argument errors are found on the host before anything is launched and are
 *     returned as an attn_status; nothing is written in that case.
 *   - Errors that depend on device data (cumulative lengths that are not monotone or do not
 *     end at the total, CSR columns out of range, a row pointer that decreases, a pipeline
 *     wait that timed out) are recorded in a per-device status word that
 *     attn_get_last_error() reads. The kernel skips the offending unit of work (its outputs
 *     are left as zeros where that is stated below) and never traps or aborts.
 *   - Results are deterministic: the same inputs give bitwise-identical outputs (no atomics
 *     take part in any result).
 *   - Every function is thread-safe; calls on different streams may overlap.
 *   - No call allocates device memory. The library's own device memory, per device: the status
 *     word, the work counters of attn_fwd's persistent grid (one pair for each of the first 256
 *     streams that call it; launches on further streams, and launches being captured into a CUDA
 *     graph, divide their work statically instead, with the same results) and the fixed scratch
 *     of attn_sparse_csr_tc_noalloc.
 *
 * Softmax statistics (all calls): softmax_max is max_j s_ij, with s_ij = scale * q_i . k_j, in
 * natural-log units; softmax_sum is sum_j exp(s_ij - softmax_max). A row that sees no key has
 * output 0, softmax_max = -inf and softmax_sum = 0.
 */
#ifndef SDPA_B200_ATTN_H
#define SDPA_B200_ATTN_H

#include <stdint.h>

#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID = 1,     /* bad shape, null pointer, inconsistent sizes              */
  ATTN_ERR_UNSUPPORTED = 2, /* valid request this library does not run (e.g. bf16, D=96) */
  ATTN_ERR_CUDA = 3,        /* a CUDA runtime call failed (launch, device query)        */
  ATTN_ERR_DATA = 4,        /* device-side: bad cumulative lengths or CSR indices       */
  ATTN_ERR_TIMEOUT = 5      /* device-side: a pipeline wait exceeded its bound          */
} attn_status;

typedef enum { ATTN_BF16 = 0, ATTN_F32 = 1, ATTN_F16 = 2 } attn_dtype;

typedef enum { ATTN_BHSD = 0, ATTN_TND = 1 } attn_layout;

typedef enum {
  ATTN_MASK_NONE = 0,
  ATTN_MASK_CAUSAL_TOPLEFT = 1,    /* key j visible to query i iff j <= i                  */
  ATTN_MASK_CAUSAL_BOTTOMRIGHT = 2, /* key j visible iff j <= i + Skv_b - Sq_b (per sequence) */
  ATTN_MASK_BAND = 3               /* attn_fwd_masked only: i - pre_tokens <= j <= i + next_tokens */
} attn_mask;

/*
 * attn_fwd -- fused attention forward (FlashAttention-style tiling with an online softmax).
 *
 * Defined by: "paddle.nn.functional.sparse_attention" (Paddle 2.3 API doc), formula
 * result = softmax(Q K^T / sqrt(d)) V, here with a general `scale`; "aclnnFlashAttentionVarLenScore"
 * (CANN 8.5 API doc), 功能说明 (function) and 约束说明 (constraints): the packed TND layout,
 * cumulative sequence lengths, GQA/MQA head ratios, lower-triangular masks and the shape limits.
 *
 * Layouts (layout = ATTN_BHSD):
 *   q   [B, Nq,  Sq,  D]     k, v [B, Nkv, Skv, D]     out [B, Nq, Sq, D]
 *   softmax_max, softmax_sum  float32 [B, Nq, Sq]
 * Layouts (layout = ATTN_TND, packed variable-length batch):
 *   q   [Tq, Nq, D]          k, v [Tkv, Nkv, D]        out [Tq, Nq, D]
 *   softmax_max, softmax_sum  float32 [Tq, Nq]
 *   Sq and Skv are the totals Tq and Tkv. cu_seqlens_q / cu_seqlens_kv are device int32
 *   arrays of B entries holding cumulative lengths WITHOUT a leading zero: sequence b
 *   occupies tokens [cu[b-1], cu[b]) with cu[-1] = 0, and cu[B-1] must equal the total.
 *   Lengths [2,2,0,2,2] are passed as [2,4,4,6,8]; zero-length sequences are allowed.
 * GQA/MQA: query head h reads key/value head h / (Nq / Nkv); Nq must be a multiple of Nkv.
 * dtype: ATTN_BF16 or ATTN_F16 (q, k, v, out bfloat16 or float16; tensor cores with fp32
 *        accumulation; D = 64 or 128), or ATTN_F32 (float32 throughout, CUDA-core FMA;
 *        1 <= D <= 256).
 * softmax_max / softmax_sum may both be NULL to skip the statistics. mask_mode is 0, 1 or 2
 * (the band needs attn_fwd_masked).
 * Limits (from the constraints): 1 <= Nq <= 256, D <= 768 (larger D is ATTN_ERR_INVALID;
 * sizes this library does not run are ATTN_ERR_UNSUPPORTED), Tq, Tkv <= 1M tokens and
 * B <= 2048 for TND; scale must be finite and > 0. Empty problems (B = 0, Sq = 0 or a total
 * of 0 tokens) return ATTN_OK without a launch. For ATTN_BF16 and ATTN_F16, q, k, v and out
 * must be 16-byte aligned.
 * Data errors: cumulative lengths that decrease or do not end at the totals set ATTN_ERR_DATA
 * in the status word; the affected outputs are not written.
 */
ATTN_API int attn_fwd(const void* q, const void* k, const void* v,
             const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_kv,
             int B, int Sq, int Skv, int Nq, int Nkv, int D,
             float scale, int mask_mode, int dtype, int layout,
             void* out, float* softmax_max, float* softmax_sum, void* stream);

/*
 * attn_fwd_accumulate -- attention forward over one chunk of keys, folded into a running
 * accumulator (the fused form of attn_fwd followed by attn_merge).
 *
 * Defined by: the attn_fwd definition above for this chunk's keys, and the lane-wise update of
 * "npu_ring_attention_update" (MindSpeed op doc, 小算子等价计算逻辑) for the fold: for each of
 * the 8 statistic lanes m = max(pm, m_c), ps' = ps e^(pm - m), cs' = l_c e^(m_c - m),
 * l = ps' + cs'; out = acc_out * ps'_0 / l_0 + o_c * cs'_0 / l_0, where (o_c, m_c, l_c) are this
 * chunk's output row and statistics, computed in fp32 and never rounded before the fold.
 * Calling it for every chunk of a split key range (first = 1 for the first chunk) gives the
 * attention over the whole key range, as a ring of devices would compute it.
 *
 * Arguments are those of attn_fwd (k, v, cu_seqlens_kv and Skv describe this chunk of keys),
 * except the outputs, which are the accumulator in the layouts of attn_merge:
 *   layout = ATTN_BHSD: acc_out [Sq, B, Nq*D] ("SBH"), acc_max / acc_sum float32 [B, Nq, Sq, 8]
 *   layout = ATTN_TND:  acc_out [Tq, Nq*D],             acc_max / acc_sum float32 [Tq, Nq, 8]
 * acc_out has the element type `dtype`. first = 1 overwrites the accumulator (all 8 lanes get
 * this chunk's statistics); first = 0 folds into it (it must hold an earlier call's result).
 * Calls that fold into the same accumulator must not overlap on the device.
 * For ATTN_BF16 and ATTN_F16, acc_out, acc_max and acc_sum must be 16-byte aligned (otherwise
 * ATTN_ERR_INVALID): a row's 8 statistic lanes are moved as two 16-byte vectors.
 */
ATTN_API int attn_fwd_accumulate(const void* q, const void* k, const void* v,
                                 const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_kv,
                                 int B, int Sq, int Skv, int Nq, int Nkv, int D,
                                 float scale, int mask_mode, int dtype, int layout, int first,
                                 void* acc_out, float* acc_max, float* acc_sum, void* stream);

/*
 * attn_fwd_masked -- attn_fwd with a band (preTokens / nextTokens), an optional explicit mask
 * and a value head size of its own.
 *
 * Defined by: the attn_fwd definition above, restricted to the keys that pass both the mode
 * and the mask; "aclnnFlashAttentionVarLenScore" (CANN 8.5 API doc), 约束说明, which lists
 * preTokens / nextTokens, attenMaskOptional and the head-size rule qD == kD >= vD. The page
 * does not carry the table that defines the sparse modes, so this call takes these readings:
 *   mask_mode ATTN_MASK_BAND: key j is visible to query row i iff
 *     i - pre_tokens <= j <= i + next_tokens, with i and j positions within the sequence
 *     (top-left aligned); pre_tokens + next_tokens must be >= 0 (the band is not empty).
 *     pre_tokens and next_tokens are ignored by the other modes. Values beyond +-2^30 act as
 *     unbounded.
 *   atten_mask (may be NULL): uint8, 1 = the key is masked out, 0 = it may be attended; the
 *     entry for (sequence b, query position i, key position j) is
 *     atten_mask[b * mask_batch_stride + i * mask_row_stride + j] (positions within the
 *     sequence for TND; mask_batch_stride = 0 shares one mask across the batch). The caller
 *     guarantees that every addressed entry lies inside its buffer: for BHSD,
 *     mask_row_stride >= Skv; for TND, the mask must cover each sequence's lengths.
 *     A key must pass both the mode and the mask.
 *   Dv: v is [B, Nkv, Skv, Dv] (BHSD) or [Tkv, Nkv, Dv] (TND) and out is [B, Nq, Sq, Dv] or
 *     [Tq, Nq, Dv]; 1 <= Dv <= Dqk. q and k have head size Dqk.
 * Other arguments, statistics, limits and errors are those of attn_fwd (D there is Dqk).
 * Supported: ATTN_F32 with Dv <= Dqk <= 256; ATTN_BF16 and ATTN_F16 with (Dqk, Dv) =
 * (64, 64), (128, 128) or (128, 64) (other pairs are ATTN_ERR_UNSUPPORTED there). On the
 * tensor-core path a mask given with atten_mask, mask_row_stride and mask_batch_stride all
 * 16-byte aligned is read 16 bytes at a time, otherwise byte by byte.
 * Errors: mask_mode outside 0..3, pre_tokens + next_tokens < 0 with the band, negative
 * strides, Dv outside 1..Dqk, or a BHSD mask_row_stride < Skv give ATTN_ERR_INVALID.
 */
ATTN_API int attn_fwd_masked(const void* q, const void* k, const void* v,
                             const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_kv,
                             int B, int Sq, int Skv, int Nq, int Nkv, int Dqk, int Dv,
                             float scale, int mask_mode, int64_t pre_tokens, int64_t next_tokens,
                             const uint8_t* atten_mask, int64_t mask_batch_stride,
                             int64_t mask_row_stride, int dtype, int layout,
                             void* out, float* softmax_max, float* softmax_sum, void* stream);

/*
 * attn_sparse_csr -- CSR-sparse attention forward, float32.
 *
 * Defined by: "paddle.nn.functional.sparse_attention" (Paddle 2.3 API doc), formula and
 * 参数 (parameters): for every (b, h, i), the softmax of q_i . k_j / sqrt(D) runs over the
 * stored entries c of row i only, j = columns[b, h, c], and the output is the weighted sum of
 * the v_j. The offset array is read as a row pointer (the page's worked example is one).
 *
 *   q, k, v, out   float32 [B, H, S, D]
 *   csr_offset     int32 [B, H, S+1]: per (b, h) row pointer, offset[0] = 0, non-decreasing,
 *                  offset[S] <= nnz_cap
 *   csr_columns    int32 [B, H, nnz_cap]: column of each stored entry, 0 <= j < S; order
 *                  within a row is free and a repeated column counts once per entry
 * An empty row gives an output row of zeros. 1 <= D <= 256. D = 64 or 128 with 16-byte aligned
 * q, k, v, out and S <= 32768 run a kernel tiled over each block's union of columns; other
 * shapes run a warp per row. Both compute in float32 with the same definition.
 * Data errors: a column outside [0, S), or a row pointer that starts above 0, decreases or
 * passes nnz_cap, set ATTN_ERR_DATA; the affected rows are written as zeros.
 */
ATTN_API int attn_sparse_csr(const float* q, const float* k, const float* v,
                    const int32_t* csr_offset, const int32_t* csr_columns,
                    int B, int H, int S, int D, int64_t nnz_cap,
                    float* out, void* stream);

/*
 * attn_sparse_csr_tc -- CSR-sparse attention forward in bf16 or fp16 on the tensor cores.
 *
 * Defined by: the attn_sparse_csr definition above ("paddle.nn.functional.sparse_attention",
 * formula and 参数), with 16-bit inputs and output and fp32 accumulation. Each block of 128
 * query rows gathers the union of its rows' columns into tiles of 128 keys and multiplies
 * those on the tensor cores; each row's softmax keeps exactly its own stored entries.
 *
 *   q, k, v, out   dtype (ATTN_BF16 or ATTN_F16) [B, H, S, D], 16-byte aligned; D = 64 or 128
 *   csr_offset     int32 [B, H, S+1], as for attn_sparse_csr
 *   csr_columns    int32 [B, H, nnz_cap]: column of each stored entry, 0 <= j < S, order free;
 *                  the columns of one row must be distinct
 * Scale 1/sqrt(D). An empty row gives zeros. S <= 32768 (larger is ATTN_ERR_UNSUPPORTED).
 * Data errors: a column outside [0, S), a row pointer that starts above 0, decreases or passes
 * nnz_cap, or a column stored twice in one row, set ATTN_ERR_DATA; those rows are written as
 * zeros. Other dtypes are ATTN_ERR_INVALID.
 */
ATTN_API int attn_sparse_csr_tc(const void* q, const void* k, const void* v,
                                const int32_t* csr_offset, const int32_t* csr_columns,
                                int B, int H, int S, int D, int64_t nnz_cap, int dtype,
                                void* out, void* stream);

/*
 * CSR pattern plans -- the pattern bookkeeping of attn_sparse_csr_tc, done once per pattern.
 *
 * Defined by: "paddle.nn.functional.sparse_attention" (Paddle 2.3 API doc), 参数: the pattern is
 * offset [B, H, S+1] (a row pointer per (b, h)) and columns [B, H, nnz_cap]. The two-phase form
 * (size the caller-owned buffer, then run) follows "aclnnFlashAttentionVarLenScore" (CANN 8.5
 * API doc), 函数原型 (GetWorkspaceSize, then the call that takes the workspace).
 *
 * A plan holds, for every block of 128 query rows of every (b, h): the sorted union of the
 * columns the block's rows store, a bit per (row, union column) saying which of them the row
 * stores, and which rows are bad. It depends on the pattern only, so a model with a fixed
 * sparsity pattern builds it once and reuses it for every call.
 *
 * attn_csr_plan_size: *bytes = the plan's size for this shape, computed on the host from the
 *   arguments alone: B * H * ceil(S/128) * (64 + 20 * ucap) with ucap = min(S, nnz_cap) rounded
 *   up to 128. S <= 32768 (larger is ATTN_ERR_UNSUPPORTED); negative sizes or a null `bytes`
 *   are ATTN_ERR_INVALID. Launches nothing.
 * attn_csr_plan: fills `plan` (device memory owned by the caller, 16-byte aligned, at least
 *   attn_csr_plan_size bytes, else ATTN_ERR_INVALID) from csr_offset / csr_columns (as for
 *   attn_sparse_csr). Asynchronous on `stream`; the plan may be used by later launches on the
 *   same stream. Data errors are recorded in the status word and in the plan: a row pointer that
 *   starts above 0, decreases or passes nnz_cap, a column outside [0, S), or a column stored
 *   twice in one row make that row bad (its output zeros, ATTN_ERR_DATA).
 * attn_sparse_csr_tc_planned: attn_sparse_csr_tc (same definition, types, shapes and limits)
 *   computed from a plan of the pattern instead of the pattern itself. plan / plan_bytes must
 *   satisfy the rules above for the same B, H, S and nnz_cap; a plan record that was not built
 *   for this S and nnz_cap (or not built at all) is not used: its rows are written as zeros and
 *   ATTN_ERR_DATA is recorded. Each plan must not be rewritten while a call that reads it runs.
 */
ATTN_API int attn_csr_plan_size(int B, int H, int S, int64_t nnz_cap, int64_t* bytes);
ATTN_API int attn_csr_plan(const int32_t* csr_offset, const int32_t* csr_columns, int B, int H,
                           int S, int64_t nnz_cap, void* plan, int64_t plan_bytes, void* stream);
ATTN_API int attn_sparse_csr_tc_planned(const void* q, const void* k, const void* v,
                                        const void* plan, int64_t plan_bytes, int B, int H, int S,
                                        int D, int64_t nnz_cap, int dtype, void* out, void* stream);

/*
 * attn_sparse_csr_tc_noalloc -- attn_sparse_csr_tc for callers that cannot allocate device memory.
 *
 * The pages have no counterpart of this call; it exists for this library's users. The planned
 * form above is the fastest, but it needs a plan buffer the caller allocates. A caller that runs
 * inside a host application owning all GPU memory through its own pool (a plugin that is given
 * no workspace), or on a path where cudaMalloc's possible device synchronisation or failure is
 * not acceptable, cannot provide one. This call keeps a fixed scratch array of 48 MiB inside the
 * library (a static device variable, held on every GPU where the library's code is loaded until
 * the process exits), builds the plan there and runs the planned kernel. It allocates nothing
 * and frees nothing.
 *
 * Arguments, layouts, limits, results and data errors are those of attn_sparse_csr_tc (the result
 * is that of attn_sparse_csr_tc_planned on the same pattern). A pattern whose plan
 * (attn_csr_plan_size) exceeds 48 MiB is refused with ATTN_ERR_UNSUPPORTED before any launch;
 * workload 4's shape (B=2, H=8, S=4096, nnz_cap=1,278,208) needs 41,975,808 bytes.
 * The first call on each device looks up the scratch array's device address with that device
 * current; make that first call before any stream capture. Every call shares the one array:
 * calls whose kernels can overlap on the GPU (other streams, other host threads) race on it and
 * must be ordered by the caller. The array keeps the last call's plan; nothing in it needs to
 * start at zero, since each call's plan kernel writes every byte its planned kernel reads.
 */
ATTN_API int attn_sparse_csr_tc_noalloc(const void* q, const void* k, const void* v,
                                        const int32_t* csr_offset, const int32_t* csr_columns,
                                        int B, int H, int S, int D, int64_t nnz_cap, int dtype,
                                        void* out, void* stream);

/*
 * attn_merge -- merge two partial attention results (the ring-attention update).
 *
 * Defined by: "npu_ring_attention_update" (MindSpeed op doc), 小算子等价计算逻辑 (equivalent
 * small-op logic) and 前向接口 (forward interface). For every statistic lane (8 per row):
 *     m = max(pm, cm); ps' = ps * exp(pm - m); cs' = cs * exp(cm - m); l = ps' + cs'
 * and out = prev_out * (ps'/l) + cur_out * (cs'/l) with the lane-0 values of each row,
 * computed in float32 and rounded once (to nearest even) to the output type.
 *
 * layout = ATTN_BHSD means the page's "SBH" layout:
 *   prev_out, cur_out, out     [S, B, N*D] of `dtype` (ATTN_BF16, ATTN_F16 or ATTN_F32)
 *   prev_/cur_/out_ max, sum   float32 [B, N, S, 8]
 *   actual_seq_qlen must be NULL.
 * layout = ATTN_TND (packed tokens; S is the total token count T):
 *   prev_out, cur_out, out     [T, N*D] of `dtype`
 *   prev_/cur_/out_ max, sum   float32 [T, N, 8] (token-major, like the TND tensors)
 *   actual_seq_qlen            NULL, or a device int64 array of B cumulative query lengths
 *                              (no leading zero, as attn_fwd's cu_seqlens). The merge is per
 *                              token, so the lengths only fix T: if they decrease or do not
 *                              end at T the status word records ATTN_ERR_DATA (the merge still
 *                              runs over all T tokens).
 * A lane whose two maxima are both -inf (two empty partials) gives m = -inf, l = 0 and, on
 * lane 0, an output row of zeros; where the lane-0 l is 0 the output scales are 0.
 * Outputs may alias the prev_* inputs (in-place accumulation); no other overlap is allowed.
 */
ATTN_API int attn_merge(const void* prev_out, const float* prev_max, const float* prev_sum,
               const void* cur_out, const float* cur_max, const float* cur_sum,
               int S, int B, int N, int D, int dtype, int layout,
               const int64_t* actual_seq_qlen,
               void* out, float* out_max, float* out_sum, void* stream);

/*
 * attn_get_last_error -- read and clear the calling device's status word.
 * Enqueues on `stream` a one-thread kernel that exchanges the word for 0 in one atomic step,
 * copies the old value back and synchronises `stream`. *device_status is then the first
 * device-side error (ATTN_ERR_DATA or ATTN_ERR_TIMEOUT) recorded by any launch on the current
 * device since the previous read, or ATTN_OK. The word is per device, shared by all streams:
 * every launch that finished before the exchange is covered, and an error that a launch still
 * running on another stream records later is kept for the next read (none is lost). Calls on
 * one device are serialised by a host lock. The return value is ATTN_OK, or ATTN_ERR_CUDA if
 * the launch, the copy or the synchronisation failed.
 */
ATTN_API int attn_get_last_error(void* stream, int* device_status);

/* Static description of a status code. */
ATTN_API const char* attn_status_string(int status);

/* ABI version of this header: (major << 16) | minor. */
ATTN_API int attn_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SDPA_B200_ATTN_H */
