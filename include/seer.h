/*
 * seer.h — C ABI of libseer, a B200 (sm_100a) implementation of the
 * SeerAttention long-context prefill hot path:
 *
 *   AttnGate soft scores  ->  threshold / per-row TopK block mask
 *   ->  block-sparse causal FlashAttention prefill (GQA)
 *   plus the companion pass that returns O and the 2D max-pooled map A.
 *
 * Sources (web pages about SeerAttention):
 *  - "SeerAttention: Learning Intrinsic Sparse Attention in Your LLMs",
 *    rebuttal: Weakness 2 (per-row TopK, [Seq/Block, TopK] indices, gate is
 *    self-attention without V), Weakness 3 (pooling shapes), Weakness 4
 *    (padding), Weakness 5 (inference kernel pseudocode), Q1 (block RoPE).
 *  - "SeerAttention-Llama-3.1-8B-AttnGates" model card (threshold/TopK on
 *    the soft scores drives a block-sparse FlashAttention kernel).
 *  - "SeerAttention: Self-distilled Attention Gating for Efficient
 *    Long-context Prefilling": Figure 8 (O plus max-pooled attention map),
 *    Sec. 4 (block size 64).
 *
 * Conventions for every call:
 *  - Tensors are caller-owned DEVICE memory, contiguous, row-major.  Q, K, V
 *    and O are bf16 in [B, H, S, d] order (Hq heads for Q/O, Hkv for K/V;
 *    query head h reads KV head h / (Hq/Hkv)).  Block size is fixed at 64.
 *  - The library never allocates device memory.  Calls that need scratch
 *    take a caller-provided workspace of at least seer_workspace_bytes().
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream).  Argument checks run on the host before any launch
 *    and return an error without touching the device.  A launch failure
 *    returns SEER_ERR_CUDA.  Errors found on the device (a bounded wait that
 *    ran out) are recorded in a device status word and reported by
 *    seer_check_status().
 *  - seer_last_error() returns a thread-local text for the last failure.
 *  - Supported: any S >= 1 with nb = ceil(S/64) <= 16384, d in {64, 128},
 *    Hq % Hkv == 0, B * Hq <= 65535.  Other shapes return
 *    SEER_ERR_UNSUPPORTED.
 *  - S not a multiple of 64 ("Learning Intrinsic Sparse Attention",
 *    rebuttal Weakness 4: padding, ceil-mode pooling): the last block holds
 *    the S - 64 (nb - 1) remaining tokens; it pools only those tokens, and no
 *    query or key exists past S (rows past S are never written).
 */
#ifndef SEER_H
#define SEER_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SEER_API __attribute__((visibility("default")))
#else
#define SEER_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum seer_status {
    SEER_OK = 0,
    SEER_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad shape value  */
    SEER_ERR_UNSUPPORTED = 2,  /* valid but not implemented (S%64, d, ...)  */
    SEER_ERR_WORKSPACE = 3,    /* workspace missing or too small            */
    SEER_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed         */
    SEER_ERR_TIMEOUT = 5,      /* a device-side bounded wait ran out        */
    SEER_ERR_DEVICE = 6        /* another device-side check failed          */
} seer_status;

/* Problem shape.  nb = ceil(S / 64) query/key blocks. */
typedef struct seer_shape {
    int B, Hq, Hkv, S, d;
} seer_shape;

/* AttnGate parameters ("Learning Intrinsic Sparse Attention", rebuttal Q1 on
 * AttnGate's RoPE and Weakness 3): per-head linear maps d -> d_gate (no bias),
 * block RoPE at position = block index with base rope_theta, rotate-half
 * pairs (t, t + d_gate/2).  Weights are bf16 [d, d_gate] row-major per head;
 * *_head_stride is the element distance between consecutive heads' matrices
 * (0 = one matrix shared by all heads).  d_gate must be even, 2..256. */
typedef struct seer_gate_params {
    int d_gate;
    float rope_theta;
    long long wq_head_stride;
    long long wk_head_stride;
    int k_pooling;            /* SEER_KPOOL_AVG (0) or SEER_KPOOL_MAXMIN (1)          */
} seer_gate_params;

/* K pooling of the gate ("Learning Intrinsic Sparse Attention", rebuttal
 * Weakness 3 and Question 1): average like Q, or per-block max and min
 * concatenated along the feature axis ([max | min], 2d features; W_k is then
 * bf16 [2d, d_gate] per KV head). */
enum { SEER_KPOOL_AVG = 0, SEER_KPOOL_MAXMIN = 1 };

/* Mask modes ("SeerAttention-Llama-3.1-8B-AttnGates": threshold/TopK on the
 * soft scores; "Learning Intrinsic Sparse Attention", Weakness 2: TopK is
 * per row). */
enum { SEER_MASK_THRESHOLD = 0, SEER_MASK_TOPK = 1 };

typedef struct seer_mask_params {
    int mode;                   /* SEER_MASK_THRESHOLD or SEER_MASK_TOPK            */
    float threshold;            /* THRESHOLD: keep j <= i with score > threshold   */
    double density;             /* TOPK: k_i = ceil(density * (i+1)), when neither  */
                                /*       k_per_row nor k_fixed is given             */
    int k_fixed;                /* TOPK: if > 0, k_i = k_fixed                      */
    const int32_t *k_per_row;   /* TOPK: DEVICE int32 [nb] or NULL; overrides both  */
                                /*       (seer_topk_from_density fills a host copy) */
    int force_first;            /* keep block 0 in every row (counts toward k_i)    */
    int force_diag;             /* keep block i in row i (counts toward k_i)        */
} seer_mask_params;

/* which_call values for seer_workspace_bytes(). */
enum {
    SEER_CALL_GATE_SCORES = 0,
    SEER_CALL_BLOCK_SPARSE_PREFILL = 1,
    SEER_CALL_ATTN_POOLED_MAP = 2,
    SEER_CALL_DECODE_GATE_SCORES = 3,
    SEER_CALL_BLOCK_SPARSE_DECODE = 4,
    SEER_CALL_GATE_KEY_CACHE = 5,
    SEER_CALL_DECODE_GATE_CACHED = 6
};

/*
 * seer_gate_scores — AttnGate soft scores.
 * ("Learning Intrinsic Sparse Attention", rebuttal Weakness 3: pool along
 * the sequence axis, [B, H, S/64, d], before the linear layer; Q1: block
 * RoPE on the non-RoPE'd pooled Q/K; Weakness 2: softmax like attention
 * without V; Question 2: rows sum to 1.)
 *   Qp = mean over each block's tokens of q   (K likewise: average pooling)
 *   Qt = RoPE_i(Qp @ Wq[h]),  Kt = RoPE_j(Kp @ Wk[h_kv])
 *   scores[b,h,i,j] = softmax_{j<=i}(Qt_i . Kt_j / sqrt(d_gate)); 0 for j > i.
 * With k_pooling = SEER_KPOOL_MAXMIN, Kp = [max | min] over each block (2d
 * features) and W_k is [2d, d_gate].
 * q: bf16 [B,Hq,S,d]; k: bf16 [B,Hkv,S,d]; wq/wk: bf16 per the params;
 * scores: fp32 [B,Hq,nb,nb] (fully written).  Workspace:
 * seer_workspace_bytes(SEER_CALL_GATE_SCORES, shape) bytes, 256-B aligned.
 */
SEER_API seer_status seer_gate_scores(const seer_shape *shape, const void *q, const void *k,
                             const void *wq, const void *wk, const seer_gate_params *gp,
                             float *scores, void *workspace, size_t ws_bytes, void *stream);

/*
 * seer_block_mask — binary block mask from soft scores (threshold or per-row
 * TopK).  TopK keeps exactly k_i = clamp(k_i, |forced|, i+1) blocks of row i:
 * the forced blocks, then the largest scores, ties to the lower block index.
 * scores: fp32 [B,Hq,nb,nb] (entries j > i are ignored; scores must not be
 * NaN); mask: u8 [B,Hq,nb,nb], fully written, 0 for j > i.  No workspace.
 * Given identical scores the mask is bit-exact across runs and with the
 * reference definition.
 */
SEER_API seer_status seer_block_mask(const seer_shape *shape, const float *scores,
                            const seer_mask_params *mp, uint8_t *mask, void *stream);

/*
 * seer_topk_from_density — per-row TopK counts for a target density
 * ("Learning Intrinsic Sparse Attention", rebuttal Weakness 2: TopK is taken
 * per query-block row).  Host function, no device work:
 *   k_out[i] = clamp(ceil(density * (i + 1)), n_forced(i), i + 1),  0 <= i < nb,
 * with ceil taken in double precision — the rule seer_block_mask applies on
 * the device when it is given `density` — and n_forced(i) the blocks the flags
 * force in row i (block 0 and the diagonal, one block in row 0).
 * k_out: caller-owned HOST int32 [nb].  density: finite, >= 0 (values above 1
 * give k_i = i + 1).  nb in [1, 16384].  Invalid arguments return
 * SEER_ERR_INVALID_ARG and leave k_out untouched.  A caller that wants these
 * counts on the device copies k_out there and passes it as k_per_row.
 */
SEER_API seer_status seer_topk_from_density(double density, int nb, int force_first, int force_diag,
                                            int32_t *k_out);

/*
 * seer_compact_mask — per (b, h, i) ascending list of active key blocks
 * ("Learning Intrinsic Sparse Attention", Weakness 5: the kernel loops over
 * the selected blocks by index; Weakness 2: [Seq/Block, TopK] indices).
 * mask: u8 [B,Hq,nb,nb] (entries j > i ignored).  lists: int32
 * [B,Hq,nb*(nb+1)/2], causal-packed: row i starts at i*(i+1)/2 and holds
 * counts[b,h,i] entries (the rest of its i+1 slots are left untouched).
 * counts: int32 [B,Hq,nb].  No workspace.
 */
SEER_API seer_status seer_compact_mask(const seer_shape *shape, const uint8_t *mask, int32_t *lists,
                              int32_t *counts, void *stream);

/*
 * seer_block_sparse_prefill — block-sparse causal attention, GQA
 * ("Learning Intrinsic Sparse Attention", Weakness 5 pseudocode: per query
 * block, online softmax over the selected key blocks only).  For query token
 * r in block i of head h:  O_r = sum_c softmax(scale * q_r.k_c) v_c over keys
 * c <= r whose block is active in mask[b,h,i,:]; LSE_r = log sum exp.
 * Rows with no admissible key get O_r = 0 and LSE_r = -inf.
 * q: bf16 [B,Hq,S,d], k/v: bf16 [B,Hkv,S,d], mask: u8 [B,Hq,nb,nb]
 * (entries j > i ignored), o: bf16 [B,Hq,S,d], lse: fp32 [B,Hq,S] or NULL.
 * softmax_scale <= 0 selects 1/sqrt(d).  q, k, v, o must be 16-B aligned.
 * Workspace: seer_workspace_bytes(SEER_CALL_BLOCK_SPARSE_PREFILL) (may be 0;
 * workspace may then be NULL).
 * Scheduling: the persistent grid takes tiles from a counter that the call
 * seeds on `stream` (an 8-byte memset before the launch); counters come from
 * a per-device ring of 256, so up to 256 prefill / pooled-map launches may be
 * in flight at once on any streams.  A launch whose counter slot is re-seeded
 * by a later launch while it still runs stops taking tiles and records a
 * device error that seer_check_status reports as SEER_ERR_DEVICE.  A CUDA
 * graph that captured the call reuses its counter on every replay, so one
 * graph must not be replayed on two streams at once.
 * Shared memory: the kernel's layout grows with nb (two key-block lists of nb
 * entries); at d = 128 and the largest nb it leaves under 1 KB of the 227 KB
 * window for aligning the window's base to 1 KB.  The kernel checks that its
 * aligned layout fits before it touches shared memory; if not it writes
 * nothing and records a device error (SEER_ERR_DEVICE from seer_check_status).
 */
SEER_API seer_status seer_block_sparse_prefill(const seer_shape *shape, const void *q, const void *k,
                                      const void *v, const uint8_t *mask, float softmax_scale,
                                      void *o, float *lse, void *workspace, size_t ws_bytes,
                                      void *stream);

/*
 * seer_attn_pooled_map — dense causal attention returning O and the 2D
 * max-pooled attention map ("SeerAttention: Self-distilled Attention Gating",
 * Figure 8: store the block row max r_ij, then a_ij = exp(r_ij - m_i)/l_i and
 * A_ij = colmax(a_ij)):
 *   A[b,h,i,j] = max_{r in block i, c in block j, c <= r} P_rc, 0 for j > i,
 * with P the causal softmax of scale * q.k.  A is not row-normalised.
 * q/k/v/o as above; A: fp32 [B,Hq,nb,nb] (fully written).  Workspace:
 * seer_workspace_bytes(SEER_CALL_ATTN_POOLED_MAP, shape) bytes (holds the
 * per-row block maxima of the queries in flight).  Tiles are scheduled as in
 * seer_block_sparse_prefill (same counter ring and limits).
 */
SEER_API seer_status seer_attn_pooled_map(const seer_shape *shape, const void *q, const void *k,
                                 const void *v, float softmax_scale, void *o, float *A,
                                 void *workspace, size_t ws_bytes, void *stream);

/*
 * seer_gate_scores_noalloc — seer_gate_scores for callers that cannot
 * allocate device memory (an embedding application whose pool owns all device
 * memory, or a latency-critical path that must not call cudaMalloc).  The
 * pages have no counterpart; it is a deployment convenience.  Same inputs,
 * outputs and results as seer_gate_scores, but the workspace comes from a
 * fixed 24 MiB device array inside the library (held by every GPU that loads
 * the library until exit).  The gate needs, with nb = ceil(S/64),
 * dk = d (average K pooling) or 2d (max+min) and each term rounded up to a
 * multiple of 256 bytes,
 *   4 B*Hq*nb*d + 4 B*Hkv*nb*dk + 4 B*Hq*nb*d_gate + 4 B*Hkv*nb*d_gate  bytes;
 * shapes for which that exceeds 24 MiB (25165824 bytes) return
 * SEER_ERR_UNSUPPORTED and launch nothing.  (seer_workspace_bytes reports a
 * d_gate = 256, max+min bound and is not this call's limit.)  The first call on a
 * device looks up the array's device address; make it before any stream
 * capture.  All calls share the array: calls whose kernels overlap on the GPU
 * race and must be ordered (one stream, or events).
 */
SEER_API seer_status seer_gate_scores_noalloc(const seer_shape *shape, const void *q, const void *k,
                                              const void *wq, const void *wk, const seer_gate_params *gp,
                                              float *scores, void *stream);

/*
 * seer_distill_loss — the gate's distillation target and MSE loss
 * ("Learning Intrinsic Sparse Attention", rebuttal Question 2: the max-pooled
 * map is row-normalised to match the gate's softmax output; Q2 on the loss:
 * MSE against that target).  For soft scores G = scores and pooled map A
 * (fp32 [B,Hq,nb,nb], e.g. from seer_gate_scores and seer_attn_pooled_map):
 *   A_norm[i,j]     = A[i,j] / sum_{j'<=i} A[i,j']  (0 for j > i; zero rows stay 0)
 *   loss_rows[b,h,i] = sum_{j<=i} (G[i,j] - A_norm[i,j])^2        fp32 [B,Hq,nb]
 *   loss[b,h]       = sum_i loss_rows[b,h,i] / (nb(nb+1)/2)        fp32 [B,Hq]
 * (mean over the causal block entries).  A_norm may be NULL (not written).
 * Reductions run in a fixed order: results are reproducible.  No workspace.
 */
SEER_API seer_status seer_distill_loss(const seer_shape *shape, const float *scores, const float *A,
                                       float *A_norm, float *loss_rows, float *loss, void *stream);

/*
 * Decode step ("SeerAttention-R: Sparse Attention Adaptation for Long
 * Reasoning", abstract: the gate keeps its self-distilled design but drops
 * query pooling, and a sparse decoding kernel reads only the selected KV
 * blocks; "Learning Intrinsic Sparse Attention", rebuttal Weakness 4 on
 * decode: a per-Q-token AttnGate without pooling on the same weights).
 * One new token per sequence at position L - 1 of a KV cache of L tokens
 * that already holds its k and v; shape->S = L, nb = ceil(L/64), and the
 * token's block is the last one, i = nb - 1.
 *
 * seer_decode_gate_scores — the gate row of the token:
 *   qt = RoPE_{nb-1}(q_tok @ Wq[h])          (the token's own q, no pooling)
 *   Kt_j = RoPE_j(Kp_j @ Wk[h_kv])           (Kp as in seer_gate_scores)
 *   scores[b,h,j] = softmax_j(qt . Kt_j / sqrt(d_gate)), j < nb.
 * q_tok: bf16 [B,Hq,d]; k: bf16 [B,Hkv,L,d]; wq/wk and params as in
 * seer_gate_scores; scores: fp32 [B,Hq,nb].  Workspace:
 * seer_workspace_bytes(SEER_CALL_DECODE_GATE_SCORES, shape), 256-B aligned.
 */
SEER_API seer_status seer_decode_gate_scores(const seer_shape *shape, const void *q_tok, const void *k,
                                             const void *wq, const void *wk, const seer_gate_params *gp,
                                             float *scores, void *workspace, size_t ws_bytes, void *stream);

/*
 * seer_gate_key_cache — the gate's key rows Kt_j = RoPE_j(Kp_j @ Wk[h_kv])
 * for blocks j = first_block .. nb-1 of a cache of shape->S = L tokens (the K
 * side of seer_gate_scores and seer_decode_gate_scores).  A key row only
 * changes while its block fills, so a decoder keeps kt across steps and
 * refreshes from the last (partial) block on.  k: bf16 [B,Hkv,L,d]; wk and
 * params as in seer_gate_scores; kt: fp32 [B,Hkv,nb,d_gate], rows below
 * first_block untouched.  Workspace: seer_workspace_bytes(SEER_CALL_GATE_KEY_CACHE),
 * 256-B aligned.
 */
SEER_API seer_status seer_gate_key_cache(const seer_shape *shape, const void *k, const void *wk,
                                         const seer_gate_params *gp, int first_block, float *kt, void *workspace,
                                         size_t ws_bytes, void *stream);

/*
 * seer_decode_gate_scores_cached — seer_decode_gate_scores on cached key
 * rows: the token's q projected and rotated at block nb-1, softmax against
 * kt (fp32 [B,Hkv,nb,d_gate], from seer_gate_key_cache).  scores: fp32
 * [B,Hq,nb].  Workspace: seer_workspace_bytes(SEER_CALL_DECODE_GATE_CACHED),
 * 256-B aligned.
 */
SEER_API seer_status seer_decode_gate_scores_cached(const seer_shape *shape, const void *q_tok, const float *kt,
                                                    const void *wq, const seer_gate_params *gp, float *scores,
                                                    void *workspace, size_t ws_bytes, void *stream);

/*
 * seer_decode_block_mask — the mask row of the token: seer_block_mask's row
 * i = nb - 1 (threshold or TopK with k from k_fixed, k_per_row[nb-1] or
 * ceil(density * nb); block 0 and the last block forced as flagged).
 * scores: fp32 [B,Hq,nb]; mask: u8 [B,Hq,nb], fully written.  No workspace.
 */
SEER_API seer_status seer_decode_block_mask(const seer_shape *shape, const float *scores,
                                            const seer_mask_params *mp, uint8_t *mask, void *stream);

/*
 * seer_block_sparse_decode — attention of the token over the active blocks:
 *   o[b,h] = sum_{c < L, mask[b,h,c/64]} softmax(q_tok . k_c * scale) v_c,
 *   lse[b,h] = log sum exp (fp32, natural log; -inf and o = 0 when no block
 *   is active).  scale <= 0 means 1/sqrt(d).
 * q_tok: bf16 [B,Hq,d]; k/v: bf16 [B,Hkv,L,d]; mask: u8 [B,Hq,nb];
 * o: bf16 [B,Hq,d]; lse: fp32 [B,Hq] or NULL.  Workspace:
 * seer_workspace_bytes(SEER_CALL_BLOCK_SPARSE_DECODE, shape), 16-B aligned
 * (split-K partials).
 */
SEER_API seer_status seer_block_sparse_decode(const seer_shape *shape, const void *q_tok, const void *k,
                                              const void *v, const uint8_t *mask, float softmax_scale, void *o,
                                              float *lse, void *workspace, size_t ws_bytes, void *stream);

/* Workspace bytes a call needs for `shape` (0 for SEER_CALL_BLOCK_SPARSE_PREFILL).
 * Returns 0 and sets the last error for an invalid shape or call id. */
SEER_API size_t seer_workspace_bytes(int which_call, const seer_shape *shape);

/* Synchronise `stream`, read and clear the device status word.  Returns
 * SEER_OK, SEER_ERR_TIMEOUT, SEER_ERR_DEVICE or SEER_ERR_CUDA. */
SEER_API seer_status seer_check_status(void *stream);

/* Upper bound, in nanoseconds, on any single device-side wait of the
 * attention kernels (default 2e9).  A wait that runs out sets the device
 * status to SEER_ERR_TIMEOUT and the kernel exits cleanly.  0 means give up
 * at the first unsatisfied poll (used to test the timeout path). */
SEER_API void seer_set_wait_timeout_ns(unsigned long long ns);

/* Thread-local description of the last failure ("" if none). */
SEER_API const char *seer_last_error(void);

/* Library version string. */
SEER_API const char *seer_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SEER_H */
