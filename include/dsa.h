/*
 * dsa.h -- C interface of the B200 (sm_100a) DeepSeek Sparse Attention hot path.
 *
 * The path has three stages, each a hand-written CUDA kernel, plus a split
 * merge:
 *   1. lightning-indexer scores   I[t,s] = sum_j w[t,j] * ReLU(q_I[t,j] . k_I[s])
 *   2. per-query causal top-k     the min(k, n_t) highest scores of row t
 *   3. sparse MLA attention       softmax over the selected latent rows only,
 *                                 every query head sharing each row (MQA mode)
 * Sources (page title, section):
 *   - "DeepSeek Sparse Attention Explained" (kgptalkie): "How Does the Lightning
 *     Indexer Score a Token?", "How Does the Selector Pick 1,024?", "What Does
 *     the Whole Block Look Like?", "What Does the GPU Actually Run?".
 *   - "DeepSeek Sparse Attention" (lizeman), section 2 (two stages) and
 *     section 3 (the dsa_layer sketch whose arguments this interface follows).
 *   - "DeepSeek V3.2-Exp Cuts Long-Context Costs" (kiadev), "How DSA works" and
 *     "Training and implementation details" (FP8 indexer, top-k = 2048, MLA in
 *     MQA mode).
 *
 * Conventions shared by every entry point:
 *   - All pointers marked (device) are CUDA device pointers owned by the caller;
 *     the library never allocates, frees or keeps them.  Every call is
 *     asynchronous on `stream` (a cudaStream_t passed as void*, NULL = legacy
 *     default stream) and returns once the kernels are queued.
 *   - Arguments are checked on the host before any launch: NULL pointers,
 *     16-byte alignment of every tensor base, supported sizes.  A failed check
 *     returns an error status and launches nothing.
 *   - Device-side errors (an index >= q_len, q_len > T_max, a bounded wait that
 *     ran out) are recorded in a status word at the start of the workspace and
 *     read back with dsa_get_device_status().  Kernels never trap.
 *   - Query row t belongs to sequence q_seq[t] and sees the causal candidate
 *     positions s in [0, q_len[t]).  Decode: q_len[t] is the cached length of
 *     the sequence.  Prefill: q_len[t] = t + 1 (the token sees itself).
 *
 * Tensor layouts (row-major, contiguous, element counts):
 *   q_I      [Nq, H_I, d_I]   FP8 e4m3 bytes (idx_dtype DSA_FP8_E4M3) or float
 *   q_scale  [Nq, H_I]        float, > 0 (FP8 only; may be NULL for float)
 *   w        [Nq, H_I]        bfloat16 (FP8 mode) or float (float mode)
 *   k_I      [B, T_max, d_I]  FP8 e4m3 bytes or float
 *   k_scale  [B, T_max]       float, > 0 (FP8 only; may be NULL for float)
 *   q        [Nq, H, 576]     bfloat16 or float (absorbed MLA query: 512 latent + 64 rope)
 *   kv       [B, T_max, 576]  bfloat16 or float (latent cache; value = first 512), or
 *            [B, T_max, 656]  bytes with kv_dtype DSA_FP8_E4M3: the FP8 latent entry of
 *                             kgptalkie "What Does the GPU Actually Run?" -- bytes 0..511 the
 *                             e4m3 codes of latent values 0..511, bytes 512..527 four fp32
 *                             scales (value i = e4m3(code i) * scale[i / 128]), bytes
 *                             528..655 the 64 rope values in bf16; q and out stay bf16
 *   out      [Nq, H, 512]     same element type as kv
 *   lse      [Nq, H]          float, natural-log sum of exp(scale * q.c) over the selection
 *   scores   [Nq, ld_scores]  float, entries s >= q_len[t] are not written
 *   idx      [Nq, k]          int32, ascending positions, -1 padded
 *   q_seq, q_len [Nq]         int32
 */
#ifndef DSA_B200_H
#define DSA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DSA_OK = 0,
    DSA_ERR_INVALID_ARG = 1,   /* NULL, misaligned or inconsistent argument */
    DSA_ERR_UNSUPPORTED = 2,   /* valid but not built: e.g. d_I not 64/128, H != 128 for bf16 */
    DSA_ERR_WORKSPACE = 3,     /* workspace NULL or smaller than dsa_workspace_size() */
    DSA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed (see dsa_last_cuda_error) */
    DSA_ERR_TIMEOUT = 5,       /* device: a bounded wait inside a kernel ran out */
    DSA_ERR_INDEX_OOB = 6,     /* device: an idx entry outside [-1, q_len[t]) (treated as -1) */
    DSA_ERR_LENGTH = 7         /* device: q_len[t] > T_max or > ld_scores, or q_seq[t] outside [0, B) (row skipped) */
} dsa_status_t;

typedef enum { DSA_F32 = 0, DSA_BF16 = 1, DSA_FP8_E4M3 = 2 } dsa_dtype_t;

typedef enum {
    DSA_OP_INDEXER = 0,
    DSA_OP_TOPK = 1,
    DSA_OP_SPARSE_MLA = 2,
    DSA_OP_DECODE = 3,
    DSA_OP_PREFILL = 4,
    DSA_OP_DENSE_MLA = 5
} dsa_op_t;

/* Problem sizes.  Supported builds:
 *   idx_dtype DSA_FP8_E4M3: d_I in {64, 128}, H_I = 64 (the MMA N dimension of the
 *                           tensor-core kernel), T_max a multiple of 4; w is bfloat16.
 *   idx_dtype DSA_F32:      d_I in {64, 128}, 1 <= H_I <= 64; w is float.
 *   kv_dtype  DSA_BF16 or DSA_FP8_E4M3 (656-byte entries): H = 128 (MMA M dimension).
 *   kv_dtype  DSA_F32:      1 <= H <= 128.
 *   1 <= k <= 2048; 1 <= T_max; ld_scores >= 1 and a multiple of 4. */
typedef struct {
    int32_t B;          /* sequences held in the cache */
    int32_t Nq;         /* query rows */
    int32_t H_I;        /* indexer heads */
    int32_t d_I;        /* indexer head width */
    int32_t H;          /* MLA query heads */
    int32_t k;          /* top-k budget */
    int32_t T_max;      /* cache capacity per sequence, tokens (row stride of k_I/kv per sequence) */
    int32_t idx_dtype;  /* dsa_dtype_t of q_I/k_I: DSA_FP8_E4M3 or DSA_F32 */
    int32_t kv_dtype;   /* dsa_dtype_t of the cache: DSA_BF16, DSA_F32 or DSA_FP8_E4M3 (656-byte entries) */
    int32_t reserved;   /* must be 0 */
    int64_t ld_scores;  /* row stride of the scores matrix, elements */
} dsa_dims;

/* Optional per-stage timing: cudaEvent_t handles (as void*) recorded on the
 * call's stream before the first stage and after each stage (indexer, top-k,
 * attention, merge).  Any entry may be NULL. */
typedef struct {
    void* ev[5];
} dsa_stage_events;

/* Bytes of workspace the given operation needs for these sizes (0 when none
 * beyond the 256-byte status block).  The plan depends on the current
 * device's SM count.  Returns DSA_OK and writes *bytes, or DSA_ERR_INVALID_ARG /
 * DSA_ERR_UNSUPPORTED. */
dsa_status_t dsa_workspace_size(const dsa_dims* dims, int32_t op, size_t* bytes);

/* Zero the workspace's status block (call once after allocating a workspace). */
dsa_status_t dsa_workspace_init(void* workspace, size_t ws_bytes, void* stream);

/* Stage 1 -- lightning-indexer scores (kgptalkie, "How Does the Lightning
 * Indexer Score a Token?"; kiadev, "How DSA works": FP8, few small heads, ReLU).
 * scores[t,s] = k_scale[b,s] * sum_j (w[t,j] q_scale[t,j]) * ReLU(sum_x q_I[t,j,x] k_I[b,s,x])
 * for s < q_len[t], b = q_seq[t]; in float mode the scales are 1.  The per-head
 * dot products are never written out.  Device errors go to workspace's status
 * word (workspace may be NULL, then length errors are only skipped rows). */
dsa_status_t dsa_indexer_scores(const dsa_dims* dims, const void* q_I, const float* q_scale,
                                const void* w, const void* k_I, const float* k_scale,
                                const int32_t* q_seq, const int32_t* q_len, float* scores,
                                void* workspace, size_t ws_bytes, void* stream);

/* Stage 1 for the rows of one prompt (prefill): the same scores as
 * dsa_indexer_scores, with four consecutive query rows served by one
 * tensor-core pass (MMA N = 4 x 64 heads), so that each cached key tile is read
 * once per four rows.  Precondition: rows 4u .. 4u+3 belong to one sequence
 * (q_seq equal); a group that does not is skipped and DSA_ERR_INVALID_ARG is
 * recorded in the workspace's status word.  FP8 only (idx_dtype
 * DSA_FP8_E4M3, H_I = 64, d_I 64 or 128); other dims return
 * DSA_ERR_UNSUPPORTED.  Arguments, layouts and ownership as for
 * dsa_indexer_scores. */
dsa_status_t dsa_prefill_indexer_scores(const dsa_dims* dims, const void* q_I, const float* q_scale,
                                        const void* w, const void* k_I, const float* k_scale,
                                        const int32_t* q_seq, const int32_t* q_len, float* scores,
                                        void* workspace, size_t ws_bytes, void* stream);

/* Stage 2 -- per-row causal top-k (kgptalkie, "How Does the Selector Pick
 * 1,024?": keep the highest index_topk scores, min(budget, tokens so far),
 * redone for every query).  idx[t] holds the min(k, q_len[t]) positions of the
 * largest scores[t, 0:q_len[t]] under the order (score descending, position
 * ascending; -0.0 == +0.0), written in ascending position order, then -1.
 * NaN scores are not supported.  Bit-exact and deterministic. */
dsa_status_t dsa_topk(const dsa_dims* dims, const float* scores, const int32_t* q_len,
                      int32_t* idx, void* workspace, size_t ws_bytes, void* stream);

/* Stage 3 -- sparse MLA attention in MQA mode (kgptalkie, "What Does the
 * Whole Block Look Like?": the softmax denominator runs over the selected
 * tokens only; kiadev, "Training and implementation details": MQA mode, each
 * latent row shared by all heads).  For each row t and head h:
 *   out[t,h,:] = sum_{s in idx[t], s>=0} softmax_s(softmax_scale * q[t,h,:] . kv[b,s,:]) kv[b,s,0:512]
 *   lse[t,h]   = ln sum_s exp(softmax_scale * q[t,h,:] . kv[b,s,:])
 * An empty selection gives out = 0, lse = -inf.  lse may be NULL.
 * Entries of idx outside [-1, q_len[t]) are treated as -1 and flagged
 * DSA_ERR_INDEX_OOB in the status word.  The k positions of a row are split
 * across CTAs; up to 8 splits of a row run as one thread-block cluster and
 * merge on chip, more (small Nq) write fp32 partial results into the
 * workspace (sized for DSA_OP_SPARSE_MLA) for a merge pass. */
dsa_status_t dsa_sparse_mla_attn(const dsa_dims* dims, const void* q, const void* kv,
                                 const int32_t* idx, const int32_t* q_seq, const int32_t* q_len,
                                 float softmax_scale, void* out, float* lse,
                                 void* workspace, size_t ws_bytes, void* stream);

/* Dense MLA in MQA mode, the comparison the pages measure DSA against
 * (kgptalkie "How Much Does DSA Save?": dense attention over every cached
 * token vs the indexer plus attention over 2,048; kiadev "Efficiency,
 * benchmarks and operational signals": decode cost at 128K).  Same formula and
 * outputs as dsa_sparse_mla_attn with the selection replaced by every position
 * s < q_len[t]: out[t,h,:] = sum_{s < q_len[t]} softmax_s(...) kv[b,s,0:512].
 * The same kernel runs with each split walking a contiguous block of
 * positions instead of an index list; dims->k is ignored (the plan uses T_max).
 * kv_dtype DSA_BF16 or DSA_FP8_E4M3.  Workspace sized for DSA_OP_DENSE_MLA. */
dsa_status_t dsa_dense_mla_attn(const dsa_dims* dims, const void* q, const void* kv,
                                const int32_t* q_seq, const int32_t* q_len, float softmax_scale,
                                void* out, float* lse, void* workspace, size_t ws_bytes, void* stream);

/* Stage 3 for callers that cannot allocate device memory.  No counterpart in
 * the paper: it exists for callers embedded in a host that owns all device
 * memory -- plugin interfaces that hand a kernel only its input and output
 * buffers, or serving loops whose device-memory budget is fixed at start-up --
 * and so can neither call cudaMalloc nor size a workspace for
 * dsa_sparse_mla_attn.  Same arguments and results as dsa_sparse_mla_attn with
 * kv_dtype DSA_BF16 or DSA_FP8_E4M3, minus the workspace: the split partials live in a buffer
 * the library holds statically on every GPU that loads it (about 16.1 MiB,
 * kept until the process exits).
 * Limit: when the split count is above 8 (the partials path of
 * dsa_sparse_mla_attn), (number of splits) x Nq <= 64 partial rows of 128
 * heads.  The split count is the one dsa_sparse_mla_attn uses:
 * S = clamp(SMs / (2 Nq), 1, 16), rows per split = ceil(k / S) rounded up to
 * a multiple of 64, splits = ceil(k / rows per split).  1 to 8 splits merge on
 * chip and need no scratch at all.  At k = 2048 on a 148-SM B200 that means:
 * Nq <= 5 uses the buffer (Nq 1..4: 16 splits, Nq 5: 11), Nq = 6 (11 splits,
 * 66 partial rows) is refused, Nq >= 7 merges on chip.
 * Larger requests return DSA_ERR_UNSUPPORTED before any launch.  kv_dtype
 * DSA_F32 returns DSA_ERR_UNSUPPORTED.
 * The first call on a device looks up the buffer's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  All calls share the buffer, so calls whose kernels overlap on the
 * GPU (other streams, other host threads) race on it: serialise them.  No
 * status word exists here, so device-side errors are not reported: entries
 * outside [-1, q_len[t]) are still treated as -1 without a flag, and a
 * bounded wait that runs out (a stalled GPU) ends the kernel early with
 * incomplete outputs and no error code.  Callers that need those reports use
 * dsa_sparse_mla_attn.  Allocates nothing; calls no cudaMalloc or cudaFree. */
dsa_status_t dsa_sparse_mla_attn_noalloc(const dsa_dims* dims, const void* q, const void* kv,
                                         const int32_t* idx, const int32_t* q_seq, const int32_t* q_len,
                                         float softmax_scale, void* out, float* lse, void* stream);

/* The whole decode step: stages 1-3 back to back on `stream` (lizeman,
 * section 3 sketch: indexer, top-K gather, attention over the K positions).
 * scores_out / idx_out may be NULL (then the workspace holds them; size the
 * workspace for DSA_OP_DECODE); when given they receive the intermediate
 * results.  Short-context dispatch: a row with q_len[t] <= k selects every
 * position (kgptalkie, "How Does the Selector Pick 1,024?": a short prompt is
 * read in full), so when scores_out is NULL the indexer skips such rows and
 * the top-k writes 0 .. q_len[t]-1 without reading scores; the outputs are
 * the same.  When the whole cache is that short (T_max <= k and
 * ld_scores >= T_max, a bf16 or FP8 latent cache), the step is attention over
 * every position s < q_len[t]: it runs the attention kernel's dense form (the
 * computation of dsa_dense_mla_attn, same output bits), and the indexer and
 * the top-k run only to fill scores_out / idx_out when those are given.  A
 * stage with nothing to run still records its events.  events may be NULL. */
dsa_status_t dsa_decode_step(const dsa_dims* dims,
                             const void* q_I, const float* q_scale, const void* w,
                             const void* k_I, const float* k_scale,
                             const void* q, const void* kv,
                             const int32_t* q_seq, const int32_t* q_len, float softmax_scale,
                             void* out, float* lse, float* scores_out, int32_t* idx_out,
                             void* workspace, size_t ws_bytes, void* stream,
                             const dsa_stage_events* events);

/* A paged cache (kgptalkie "How Does the Selector Pick 1,024?": the selection
 * is an address list into the paged KV cache).  Every sequence's cache lives in
 * fixed-size blocks of shared pools, found through its row of a block table:
 * token s of sequence b is row block_table[b * max_blocks + s / block_size] *
 * block_size + s % block_size of each pool.  Caller-owned device memory. */
typedef struct {
    const void* k_I;             /* [num_blocks, block_size, d_I] e4m3 indexer keys */
    const float* k_scale;        /* [num_blocks, block_size] fp32 key scales (16-byte aligned) */
    const void* kv;              /* [num_blocks, block_size, 576] bf16 or [.., 656] FP8 latent entries */
    const int32_t* block_table;  /* [B, max_blocks] physical block of logical block j of sequence b */
    int32_t block_size;          /* tokens per block: a power of two >= 64 */
    int32_t num_blocks;          /* blocks in each pool */
    int32_t max_blocks;          /* table row length; dims->T_max must equal max_blocks * block_size */
    int32_t reserved;            /* must be 0 */
} dsa_paged_cache;

/* dsa_decode_step over a paged cache: the same stages, dispatch and outputs,
 * with the indexer's key and scale copies (16-byte asynchronous copies, each
 * within one block) and the attention's row gather translated through the
 * block table.  Only blocks
 * holding positions s < q_len[t] are read; a table entry outside
 * [0, num_blocks) for such a block records DSA_ERR_INDEX_OOB in the status
 * word (its rows are skipped).  FP8 indexer; bf16 or FP8 (656-byte) latent pool
 * ([num_blocks, block_size, 576] bf16 or [num_blocks, block_size, 656] bytes). */
dsa_status_t dsa_decode_step_paged(const dsa_dims* dims,
                                   const void* q_I, const float* q_scale, const void* w,
                                   const dsa_paged_cache* cache, const void* q,
                                   const int32_t* q_seq, const int32_t* q_len, float softmax_scale,
                                   void* out, float* lse, float* scores_out, int32_t* idx_out,
                                   void* workspace, size_t ws_bytes, void* stream,
                                   const dsa_stage_events* events);

/* Write n new tokens into the caches (kgptalkie, "What Does the Whole Block
 * Look Like?": on the precise path the token is compressed and written to the
 * KV cache; "What Does the GPU Actually Run?": FP8 entries with fp32 scales).
 * Token i goes to sequence seq[i], position pos[i] (0 <= pos < T_max):
 *   k_new [n, d_I] fp32 -> with idx_dtype DSA_FP8_E4M3, e4m3 codes of
 *       k_new / s, s = max|k_new| / 448 (1 if all zero), round to nearest even,
 *       clamped to +-448, into k_I, and s into k_scale; with DSA_F32 copied;
 *   kv_new [n, 576] bf16 -> copied (kv_dtype DSA_BF16) or packed into the
 *       656-byte FP8 entry (kv_dtype DSA_FP8_E4M3: each 128-value latent group
 *       quantised like the key with its own scale; rope values copied).
 * paged == NULL: kv, k_I, k_scale are the contiguous caches ([B, T_max, ..]);
 * otherwise the pools and block table of *paged are used and kv, k_I,
 * k_scale are ignored.  A token whose sequence or position is out of range,
 * or whose block id is outside the pool, is skipped and recorded in the
 * workspace's status word (workspace may be NULL).  n <= 65535. */
dsa_status_t dsa_append_tokens(const dsa_dims* dims, int32_t n, const int32_t* seq, const int32_t* pos,
                               const void* kv_new, const float* k_new, void* kv, void* k_I, float* k_scale,
                               const dsa_paged_cache* paged, void* workspace, size_t ws_bytes, void* stream);

/* Prefill: the same three stages for many query rows of ONE sequence (every
 * position of a prompt), processed in row chunks so the transient score rows
 * fit the workspace (size it for DSA_OP_PREFILL).  Semantics per row are
 * exactly those of dsa_decode_step; q_len[t] = t + 1 for a causal prompt
 * (rows t < k skip the indexer, as in dsa_decode_step).
 * The indexer serves four consecutive rows per tensor-core pass, so every
 * q_seq[t] must name the same sequence: groups of four rows that do not are
 * skipped and DSA_ERR_INVALID_ARG is recorded in the device status word.
 * idx_out may be NULL. */
dsa_status_t dsa_prefill(const dsa_dims* dims,
                         const void* q_I, const float* q_scale, const void* w,
                         const void* k_I, const float* k_scale,
                         const void* q, const void* kv,
                         const int32_t* q_seq, const int32_t* q_len, float softmax_scale,
                         void* out, float* lse, int32_t* idx_out,
                         void* workspace, size_t ws_bytes, void* stream);

/* Read and clear the device status word: synchronises `stream`, writes the
 * first device-side error recorded since the last read into *status (DSA_OK if
 * none) and resets it. */
dsa_status_t dsa_get_device_status(void* workspace, void* stream, int32_t* status);

/* Short text for a status code (static storage). */
const char* dsa_status_string(int32_t status);

/* The last CUDA runtime error seen by this thread inside the library (a
 * cudaError_t value; 0 when none). */
int32_t dsa_last_cuda_error(void);

/* Self-test of the bounded wait used by every kernel: one CTA waits on a
 * barrier that nothing arrives at, for about `timeout_us` microseconds, then
 * records DSA_ERR_TIMEOUT in the status word and exits normally. */
dsa_status_t dsa_selftest_wait_timeout(void* workspace, size_t ws_bytes, int32_t timeout_us,
                                       void* stream);

/* Self-test of a production kernel's bounded waits: dsa_sparse_mla_attn's
 * kernel (kv_dtype DSA_BF16, same arguments and workspace) with one fault
 * planted on the host's request: its gather warps never signal that the
 * first tile has landed.  The MMA warp's wait for that tile runs out after
 * about `timeout_us` microseconds (1 .. 5,000,000); the kernel then records
 * DSA_ERR_TIMEOUT in the workspace status word, every role of every CTA
 * leaves its loop, copies still in flight land, tensor memory is freed and the
 * kernel exits.  out and lse hold zeros / -inf or partial results afterwards.
 * The CUDA context stays usable.  No counterpart on the pages: it checks the
 * failure handling that every kernel's waits rely on. */
dsa_status_t dsa_selftest_attention_stall(const dsa_dims* dims, const void* q, const void* kv, const int32_t* idx,
                                          const int32_t* q_seq, const int32_t* q_len, float softmax_scale,
                                          void* out, float* lse, void* workspace, size_t ws_bytes,
                                          int32_t timeout_us, void* stream);

/* Library version string. */
const char* dsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_B200_H */
