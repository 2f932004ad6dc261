/*
 * dsa.h -- C ABI of the DSA sparse-attention step for NVIDIA B200 (sm_100a).
 *
 * The step has two parts, as the pages describe it:
 *
 *  1. Index stage ("Day0 Adaptation and Performance Optimization for Novel
 *     Long-Sequence Reasoning Models", section 3; "Large Model Inference
 *     Acceleration: Day-0 Adaptation and Performance Optimization for New
 *     Architectures", section 1.1 "Indexer Fusion: Three Kernels into One"):
 *     relevance scoring of every cached position, head-weight weighting and
 *     Top-K selection in ONE kernel that reads the paged indexer-key cache in
 *     place and writes only the final index list.  The score is the Lightning
 *     Indexer form with a ReLU gate:
 *         score(t, s) = sum_h w[t,h] * max(0, q[t,h,:] . k[s,:])
 *     Ties are broken by position (the lower position wins).
 *
 *  2. Sparse read stage ("Day0 Adaptation and Sparse Attention Optimization
 *     for Long-Sequence LLM Inference", section 4): Sparse Flash Attention
 *     gathers only the selected rows of the MLA latent cache (512 latent +
 *     64 RoPE, shared by all query heads) and computes softmax attention over
 *     them: logits = sm_scale * q . row[0:576], output = softmax . row[0:512].
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers unless stated; the caller owns
 *    every buffer (inputs, outputs and the workspace).  The library never
 *    allocates or frees memory and never synchronizes the stream, except
 *    dsa_get_status(), which synchronizes by design.
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t, passed as
 *    void*; NULL = legacy default stream).  Pointers must stay valid until
 *    that work completes.
 *  - Host-side validation failures return before anything is launched.
 *    Launch failures return DSA_ERR_CUDA.  Errors found by the kernels
 *    (out-of-range block ids, a co-scheduling wait that timed out) are
 *    recorded in a status word inside the workspace and read with
 *    dsa_get_status().
 *  - Layouts are dense, row-major, with the innermost dimension last.
 *    Query tokens are sequence-major: tokens cu_q[b] .. cu_q[b+1]-1 belong to
 *    sequence b and sit at positions seq_lens[b]-nq_b .. seq_lens[b]-1; token
 *    j of a sequence sees positions 0..its own position (causal).
 *  - Paged caches: page size 64 tokens.  block_table[b, i] is the physical
 *    page holding positions 64*i .. 64*i+63 of sequence b.  The indexer-key
 *    cache and the latent cache share the table.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DSA_API __attribute__((visibility("default")))
#else
#define DSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DSA_OK = 0,
    DSA_ERR_INVALID_ARG = 1,    /* a pointer, size or shape failed validation       */
    DSA_ERR_UNSUPPORTED = 2,    /* valid request outside what the kernels implement */
    DSA_ERR_WORKSPACE = 3,      /* workspace NULL, too small or misaligned          */
    DSA_ERR_CUDA = 4,           /* a CUDA runtime / driver call failed              */
    DSA_ERR_TIMEOUT = 5,        /* device: a bounded wait expired (kernel returned) */
    DSA_ERR_DEVICE_BOUNDS = 6,  /* device: block id or index out of range (skipped) */
    DSA_ERR_CAPACITY = 7        /* device: a key chunk exceeded on-chip capacity    */
} dsa_status;

typedef enum {
    DSA_KEY_BF16 = 0,           /* indexer keys: bf16 [num_blocks, 64, D_I]                       */
    DSA_KEY_FP8_E4M3 = 1,       /* indexer keys: e4m3fn codes [num_blocks, 64, D_I] (uint8) plus  */
                                /* fp32 scales [num_blocks, 64, D_I/64], one per 64 elements      */
    DSA_KEY_MXFP8 = 2           /* indexer keys in MXFP8: e4m3fn codes [num_blocks, 64, D_I]      */
                                /* (uint8) plus one shared scale per 32 elements, [num_blocks,   */
                                /* 64, D_I/32] uint8 exponents e (scale 2^(e-127)); needs MXFP8   */
                                /* queries.  "Day0 Adaptation and Performance Optimization for   */
                                /* Novel Long-Sequence Reasoning Models", section 4: full MXFP8   */
                                /* quantization of index Q/K, every 32 elements share a scale.   */
} dsa_key_dtype;

typedef enum {
    DSA_Q_BF16 = 0,             /* indexer queries: bf16 [T, H_I, D_I]                             */
    DSA_Q_MXFP8 = 1             /* indexer queries in MXFP8: e4m3fn codes [T, H_I, D_I] (uint8) in */
                                /* q_idx plus q_scale [T, H_I, D_I/32] uint8 exponents            */
} dsa_query_dtype;

/* Batch and paging description shared by all entry points. */
typedef struct {
    int32_t batch;              /* B sequences                                            */
    int32_t num_tokens;         /* T query tokens in total                                */
    const int32_t* seq_lens;    /* device [B]: cached length INCLUDING this step's tokens */
    const int32_t* cu_q;        /* device [B+1]: query-token offsets, cu_q[0] = 0         */
    const int32_t* block_table; /* device [B, max_blocks_per_seq]                         */
    int32_t max_blocks_per_seq;
    int32_t num_blocks;         /* physical pages in each cache (bounds checks)           */
    int32_t max_seq_len;        /* host-side upper bound on every seq_lens[b]             */
    int32_t max_q_per_seq;      /* host-side upper bound on cu_q[b+1] - cu_q[b]           */
} dsa_batch;

/* Indexer inputs (Lightning Indexer + Top-K). */
typedef struct {
    const void* q_idx;          /* device [T, H_I, D_I] bf16 (or e4m3 codes, see q_dtype)      */
    const float* w;             /* device [T, H_I] fp32 head weights (any sign)                */
    const void* k_cache;        /* device indexer-key cache, layout per key_dtype              */
    const float* k_scale;       /* device key scales: [num_blocks, 64, D_I/64] fp32 (fp8 keys, */
                                /* 4-byte aligned) or [num_blocks, 64, D_I/32] uint8 exponents */
                                /* (MXFP8 keys, 16-byte aligned); NULL for bf16 keys           */
    int32_t key_dtype;          /* dsa_key_dtype                                               */
    int32_t H_I;                /* indexer heads: 8, 16, 32 or 64                              */
    int32_t D_I;                /* indexer dim: 64 or 128                                      */
    int32_t K;                  /* Top-K, 1..2048                                              */
    int32_t q_dtype;            /* dsa_query_dtype (MXFP8 exactly when key_dtype is MXFP8)     */
    const uint8_t* q_scale;     /* device [T, H_I, D_I/32] exponents of MXFP8 queries, or NULL */
} dsa_indexer_inputs;

typedef enum {
    DSA_KV_BF16 = 0,            /* latent cache rows in bf16 [num_blocks, 64, 576]                              */
    DSA_KV_FP8 = 1              /* FP8 latent cache: e4m3fn codes [num_blocks, 64, 576] (uint8, 16-byte aligned)  */
                                /* plus fp32 scales [num_blocks, 64, 5]: one per 128-element tile of a row, the  */
                                /* fifth covering the 64 RoPE elements ("Day0 Adaptation and Performance         */
                                /* Optimization ...", section 4: FP8 KV cache per token and head, tiles of 128). */
                                /* The selected rows are dequantized to bf16 (code x scale, rounded once) into   */
                                /* the workspace, 64 tokens at a time, before the attention                      */
} dsa_kv_dtype;

/* Sparse MLA attention inputs. */
typedef struct {
    const void* q;              /* device [T, H, 576] bf16 (512 latent + 64 RoPE)   */
    const void* kv_cache;       /* device latent cache, layout per kv_dtype         */
    int32_t H;                  /* query heads, 1..128                              */
    float sm_scale;             /* softmax scale applied to q . row[0:576]          */
    int32_t kv_dtype;           /* dsa_kv_dtype                                     */
    const float* kv_scale;      /* device [num_blocks, 64, 5] fp32 (FP8), else NULL */
} dsa_attn_inputs;

/*
 * Bytes of workspace needed for this batch shape by indexer_topk (ix given),
 * sparse_mla_attn (at given) or both / dsa_decode (both given).  The
 * layout is [256-byte status area][indexer group region and published-key
 * slots, a fixed size per device][attention partial slots of tokens shared
 * by several SM pairs, a fixed size per device]; one buffer sized with both
 * serves all three entry points, for any mix of shapes.  With an FP8 latent
 * cache (at->kv_dtype) a staging region follows: the selected rows of up to
 * 64 tokens as bf16 plus their per-token batch (sized for ix->K, or for
 * K = 2048 when ix is NULL); its contents are scratch.
 * The workspace must be 256-byte aligned and ZERO-FILLED before its first
 * use.  After that the library keeps it consistent by itself (a call that
 * completes without a device error leaves its histograms zero and its
 * barrier words at rest), so it can be reused by later calls on the same
 * stream; the caller must not modify it.  After a device error
 * (dsa_get_status != OK) zero-fill it again.  Calls sharing one workspace
 * must not overlap in time.
 * Status area: int32 word 0 is the device status read by dsa_get_status.
 * Words 1 and 2 are test hooks of the library's own failure tests and must
 * stay zero in normal use: word 1 shortens every bounded device wait to that
 * many microseconds (0 = the default of one second), word 2 injects a wait
 * that runs out (bit 0: an indexer group barrier waits for one CTA more than
 * its group has; bit 1: in the attention kernel the second CTA of each pair
 * never reports its first rows).
 * Returns 0 if the shape is invalid.
 */
DSA_API size_t dsa_workspace_size(const dsa_batch* batch, const dsa_indexer_inputs* ix,
                          const dsa_attn_inputs* at);

/*
 * Fused Lightning Indexer + Top-K.
 * out_idx   device [T, K] int32: the selected positions of each token in
 *           ascending order, -1 padded when fewer than K positions are
 *           visible (then every visible position is selected).
 * out_score device [T, K] fp32 score of each selected position (-inf on
 *           padding) or NULL.
 * Score rows are never written to global memory.
 */
DSA_API dsa_status indexer_topk(const dsa_batch* batch, const dsa_indexer_inputs* ix,
                        int32_t* out_idx, float* out_score,
                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * Sparse Flash Attention over the rows listed in idx (device [T, K] int32
 * logical positions; negative entries are skipped).
 * out device [T, H, 512] bf16; lse device [T, H] fp32 natural-log
 * log-sum-exp of the scaled logits (-inf if a token selects nothing) or NULL.
 * The launch is a programmatic dependent of the preceding kernel on the
 * stream: its prologue may overlap that kernel's end, and it reads nothing
 * (inputs, index list, workspace) before that kernel has completed.  When a
 * token's rows are spread over several SM pairs (few tokens), a second, small
 * kernel merges the pairs' partial results (normalised bf16 O and softmax
 * statistics, kept in the workspace) into out and lse.
 */
DSA_API dsa_status sparse_mla_attn(const dsa_batch* batch, const dsa_attn_inputs* at,
                           const int32_t* idx, int32_t K,
                           void* out, float* lse,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * sparse_mla_attn without a caller workspace (the pages have no counterpart:
 * this is a convenience of this library).  For callers that cannot provide
 * device memory for the workspace -- code that must not allocate on the
 * device, or that has no device allocator at hand.  The function itself
 * allocates nothing: it uses a fixed 20 MiB scratch array inside the library
 * module (status area and partial slots), which every GPU that loads the
 * library holds until the process exits.
 * Arguments, layouts and results are those of sparse_mla_attn.
 *  - The first call on a device (and the first after that device's context
 *    changes) looks up the scratch address with the device current; make it
 *    before any latency-critical use.
 *  - Each call first clears the scratch's status area on the stream (one
 *    memset), so a call that ended in a device error leaves nothing behind
 *    for later calls.
 *  - Shapes whose plan needs more scratch than 20 MiB are rejected with
 *    DSA_ERR_WORKSPACE (dsa_last_error() gives both sizes); on a 148-SM B200
 *    every shape fits.
 *  - All calls on a device share the one scratch: calls whose device work
 *    overlaps in time (other streams, other host threads) race and must not
 *    be issued.
 *  - Errors found by the kernels go to the scratch's status word, which this
 *    API does not expose; use sparse_mla_attn when device-side status is
 *    needed.
 */
DSA_API dsa_status sparse_mla_attn_static(const dsa_batch* batch, const dsa_attn_inputs* at,
                                          const int32_t* idx, int32_t K, void* out, float* lse,
                                          void* stream);

/*
 * The whole decode step: indexer_topk then sparse_mla_attn on one stream,
 * without a host synchronization in between.  out_idx [T, K] is required
 * (it carries the index list between the stages); out_score and lse may be
 * NULL.  The attention launch depends programmatically on the indexer
 * launch: its prologue and the first token's query load overlap the end of
 * the indexer, and it reads the index list only after the indexer completed.
 */
DSA_API dsa_status dsa_decode(const dsa_batch* batch, const dsa_indexer_inputs* ix,
                      const dsa_attn_inputs* at,
                      int32_t* out_idx, float* out_score, void* out, float* lse,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * Synchronizes `stream`, reads the device status word kept in `workspace`
 * (DSA_OK if no kernel reported an error since the last read) into
 * *device_status and clears it.  Returns DSA_ERR_CUDA if the stream itself
 * failed.
 */
DSA_API dsa_status dsa_get_status(void* workspace, void* stream, int32_t* device_status);

/*
 * Number of kernel launches dsa_decode enqueues for this shape (indexer
 * launches + the attention launch + the merge launch when tokens are shared
 * by several SM pairs), or -1 if the shape is invalid.  Useful for
 * sizing CUDA graphs and for launch accounting; performs no launch.
 */
DSA_API int32_t dsa_decode_launch_count(const dsa_batch* batch, const dsa_indexer_inputs* ix,
                                        const dsa_attn_inputs* at);

/*
 * Indexer prolog: the input preparation of the index stage ("Day0 Adaptation
 * and Performance Optimization for Novel Long-Sequence Reasoning Models",
 * section 3: query projection, key RMS normalization, query quantization and
 * head-weight projection, projections kept in bf16 (section 4); "Large Model
 * Inference Acceleration ...", section 1.2).  For each query token t with
 * hidden state x[t, :] and p = W . x[t, :] (fp32 accumulation of bf16 inputs):
 *     q[t, h, i] = p[h*D_I + i]
 *     k[t, i]    = p[HD + i] / sqrt(mean_j p[HD + j]^2 + eps) * k_gamma[i]
 *     w[t, h]    = p[HD + D_I + h]                         (HD = H_I * D_I)
 * q is written to q_out in q_dtype (bf16, round to nearest even; or MXFP8:
 * e4m3fn codes [T, H_I, D_I] plus one shared exponent per 32 elements in
 * q_scale_out [T, H_I, D_I/32], scale 2^(floor(log2 amax) - 8)); w to w_out
 * [T, H_I] fp32; k into the token's row of the paged indexer-key cache
 * (position seq_lens[b] - nq_b + j for token j of sequence b, page from the
 * block table) in key_dtype: bf16; e4m3fn codes with one fp32 scale
 * amax/448 per 64 elements in k_scale [num_blocks, 64, D_I/64]; or MXFP8
 * codes with k_scale [num_blocks, 64, D_I/32] exponents.  e4m3fn codes are
 * rounded to nearest even and saturated at +-448; a zero is stored as +0.
 * All four come out of one kernel (a tensor-core GEMM over the stacked weight
 * rows with the normalization and encoding applied to its accumulators).
 */
typedef enum {
    DSA_W_ROW_MAJOR = 0,        /* w_proj row-major [H_I*D_I + D_I + H_I, d_model]                          */
    DSA_W_TILE_PACKED = 1       /* w_proj as written by indexer_prolog_pack: each 128-row x 64-column block */
                                /* contiguous, so that the weights stream from HBM in 16 KB pieces         */
} dsa_weight_layout;

typedef struct {
    const void* x;              /* device [T, d_model] bf16 hidden states of the step's tokens, 16-byte aligned */
    const void* w_proj;         /* device [H_I*D_I + D_I + H_I, d_model] bf16, 16-byte aligned: the query    */
                                /* rows (head h, element i at row h*D_I + i), then the D_I key rows, then   */
                                /* the H_I head-weight rows                                                 */
    const float* k_gamma;       /* device [D_I] key RMS-normalization weight                                */
    float eps;                  /* RMS-normalization epsilon, >= 0                                           */
    int32_t d_model;            /* hidden size: a multiple of 8                                              */
    int32_t H_I;                /* 8, 16, 32 or 64                                                           */
    int32_t D_I;                /* 64 or 128                                                                 */
    int32_t key_dtype;          /* dsa_key_dtype of the key cache written                                    */
    int32_t q_dtype;            /* dsa_query_dtype of q_out (MXFP8 exactly when key_dtype is MXFP8)          */
    int32_t w_layout;           /* dsa_weight_layout of w_proj                                               */
} dsa_prolog_inputs;

/*
 * Bytes of the tile-packed copy of the prolog weights (0 for invalid sizes):
 * ceil(n_out/128) * ceil(d_model/64) blocks of 128 x 64 bf16, n_out =
 * H_I*D_I + D_I + H_I.  Block (i, j) holds rows 128i.. and columns 64j.. of
 * the row-major matrix (zeros past its edges), row-major, at element offset
 * (i * ceil(d_model/64) + j) * 8192.
 */
DSA_API size_t dsa_prolog_packed_bytes(int32_t H_I, int32_t D_I, int32_t d_model);

/*
 * Writes the tile-packed copy of the row-major prolog weights w_proj into
 * w_packed (dsa_prolog_packed_bytes bytes, 16-byte aligned; both device
 * pointers), enqueued on `stream`.  Done once when the weights are loaded
 * ("Day0 Adaptation and Performance Optimization ...", section 2: hardware-
 * friendly weight layouts).  Returns DSA_ERR_INVALID_ARG for bad sizes or
 * pointers, DSA_ERR_CUDA if the launch fails.
 */
DSA_API dsa_status indexer_prolog_pack(const void* w_proj, void* w_packed, int32_t H_I, int32_t D_I,
                                       int32_t d_model, void* stream);

/*
 * Bytes of workspace indexer_prolog needs for this shape (0 if the arguments
 * are invalid).  Layout: [256-byte status area][split counters][fp32 partial
 * tiles when the contraction is split along d_model].  The status area and
 * the counters must be zero-filled before the first call and stay so after
 * every successful call; the partial tiles are scratch, so a workspace that
 * indexer_prolog has used must be zero-filled again before indexer_topk,
 * sparse_mla_attn or dsa_decode use it.
 */
DSA_API size_t dsa_prolog_workspace_size(const dsa_batch* batch, const dsa_prolog_inputs* pr);

/*
 * Runs the prolog for the batch's T tokens (batch->max_seq_len and
 * max_q_per_seq are not used).  Outputs: q_out (bf16 [T, H_I, D_I], or e4m3
 * codes with q_scale_out for MXFP8), w_out [T, H_I] fp32, and the tokens'
 * rows of k_cache / k_scale (layouts of dsa_indexer_inputs); no other cache
 * row is touched.  A token whose page id is out of range is skipped and
 * recorded as DSA_ERR_DEVICE_BOUNDS in the status word.  Returns
 * DSA_ERR_INVALID_ARG / DSA_ERR_UNSUPPORTED / DSA_ERR_WORKSPACE before
 * launching anything, DSA_ERR_CUDA if the launch fails.
 */
DSA_API dsa_status indexer_prolog(const dsa_batch* batch, const dsa_prolog_inputs* pr, void* q_out,
                                  uint8_t* q_scale_out, float* w_out, void* k_cache, void* k_scale,
                                  void* workspace, size_t workspace_bytes, void* stream);

/* Static description of a status code. */
DSA_API const char* dsa_status_str(int32_t status);

/*
 * Text of the last failure an entry point recorded on the calling host thread
 * (the CUDA call and its error name for DSA_ERR_CUDA), or "" if none.  The
 * string is owned by the library and stays valid until the next call on that
 * thread.
 */
DSA_API const char* dsa_last_error(void);

/* Library version string. */
DSA_API const char* dsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
