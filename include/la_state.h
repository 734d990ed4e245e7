/*
 * la_state.h -- C ABI of liblastate.so: the fixed-size recurrent-state step of linear
 * attention (Gated DeltaNet family) on NVIDIA B200 (sm_100a).
 *
 * What the library computes.  Per state head the state S is a d_k x d_v matrix.  For
 * each token, with gate g and write strength beta:
 *
 *   u = b * (v - c * S^T k)          write (delta) vector, length d_v
 *   S <- a * S + k u^T               decay plus rank-one correction
 *   o = scale * S^T q                readout by the query, from the UPDATED state
 *
 *   rule         a   b     c       source
 *   linear       1   1     0       plain additive update
 *   gated        g   1     0       update decayed by a gate
 *   delta        1   beta  1       delta correction without a gate
 *   gated_delta  g   beta  g       S <- g (I - beta k k^T) S + beta k v^T (the default)
 *   kda          channel-wise gate: S <- (I - beta k k^T) Diag(alpha) S + beta k v^T,
 *                i.e. u = beta (v - (Diag(alpha) S)^T k), S <- Diag(alpha) S + k u^T,
 *                with alpha in R^{d_k} (one decay per key channel)
 *
 * The rule names, their one-line meanings and the default are those of the ONNX
 * LinearAttention operator described in "Seven Architectures Replacing KV Cache With
 * Bounded Mutable State" (section "ONNX LinearAttention / FlashInfer"); the
 * gated_delta recurrence is the one of the "Gated DeltaNet" glossary page (Technical
 * definition: decay by a gate, rank-one delta-rule correction, projection by the
 * query) and of the KDA formula in the "Kimi Linear" section of the same article,
 * read with a scalar gate; kda is that formula with its channel-wise gate alpha_t
 * (Kimi Delta Attention), the prediction taken from the decayed state.  The kernels
 * compute the readout in the rearranged form of the "Gated DeltaNet" page
 * (Engineering details),
 *   o = scale * ( a * (S_old^T q) + (k . q) * u )   (kda: (Diag(alpha) S_old)^T q),
 * so that the update and the readout share one pass over S.  All arithmetic is FP32;
 * the state is stored in FP32 or BF16 (rounded to nearest even), as in the "Recurrent
 * state" glossary page (Why it matters: BF16 storage, FP32 compute).
 *
 * Layouts (row-major, last index contiguous; all device memory):
 *   state pool   [n_slots, H_v, d_k, d_v]       (the ONNX past_state / present_state
 *                                                shape (B, H_kv, d_k, d_v) with B -> slots)
 *   q, k         [B or T, H_qk, d_k]   io dtype  state head h reads q/k head h / (H_v/H_qk)
 *   v, o         [B or T, H_v,  d_v]   io dtype
 *   g, beta      [B or T, H_v]         float32
 *   g (kda)      [B or T, H_v, d_k]    float32, 16-byte aligned
 * Supported (d_k, d_v): (16,16), (64,64), (128,64), (128,128).
 *
 * Slots.  A request reads its state from read_slot[b] of the source pool and writes
 * the new state to write_slot[b] of the destination pool ("Recurrent state" and "Gated
 * DeltaNet" glossary pages: separate slots for reading a prefix-cache checkpoint and
 * writing live state, so the checkpoint survives).  A NULL slot array means slot b for
 * request b ("dense" mode: the source pool is past_state, the destination pool is
 * present_state, and they may be the same pool for an in-place update).
 *
 * Conventions for every entry point.
 *   - Ownership: all buffers belong to the caller.  The library allocates, frees and
 *     synchronizes nothing; work is enqueued asynchronously on `stream` (a
 *     cudaStream_t; NULL = the legacy default stream).
 *   - Host-side errors (LA_ERR_*) are returned before anything is launched.
 *   - Device-side errors never trap: a tile with an out-of-range slot, or a sequence
 *     with inconsistent cu_seqlens, is skipped (its outputs and destination are left
 *     untouched) and a bit is OR-ed into *err_word (device int32, required).  The
 *     caller reads it after synchronizing.  Bits are LA_DEVERR_*.
 *   - Preconditions (not checked on the device; la_state_check_slots checks them on the
 *     host): write slots are distinct, and no write slot equals another request's read
 *     slot.  Read slots may repeat; a request may read and write the same slot.
 *   - LA_Q8 pools: la_state_step takes them as source and destination together (equal
 *     n_hp; the masks may differ, but the step is fastest when both pools use one mask
 *     array, as an in-place pool does); the token-serial scans and the one-launch chunked
 *     prefill (la_state_scan_chunked, its checkpointed form, la_state_scan_chunked_qgroups)
 *     take them as source and / or destination; the two-launch chunked forms, the
 *     convolution entry points, the kda chunked prefill and la_state_step_qgroups /
 *     la_state_scan_qgroups return LA_ERR_UNSUPPORTED.
 *   - Pointers to the pool, q, k, v, o and dense buffers must be 16-byte aligned;
 *     g, beta and int32 arrays 4-byte aligned.
 */
#ifndef LA_STATE_H
#define LA_STATE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LA_ABI_VERSION 4

typedef enum {
    LA_RULE_LINEAR = 0,
    LA_RULE_GATED = 1,
    LA_RULE_DELTA = 2,
    LA_RULE_GATED_DELTA = 3,
    LA_RULE_KDA = 4 /* channel-wise gate (Kimi Delta Attention); g holds d_k decays per head */
} la_rule;

/* LA_Q8 (state pools only): the mixed INT8 / BF16 storage described at la_pool. */
typedef enum { LA_F32 = 0, LA_BF16 = 1, LA_Q8 = 2 } la_dtype;

typedef enum {
    LA_OK = 0,
    LA_ERR_NULL = 1,        /* a required pointer is NULL */
    LA_ERR_SHAPE = 2,       /* a size is negative / zero where it must not be, or inconsistent */
    LA_ERR_UNSUPPORTED = 3, /* (d_k, d_v), dtype or rule outside the supported set */
    LA_ERR_ALIGN = 4,       /* a pointer violates the alignment rule above */
    LA_ERR_ALIAS = 5,       /* la_state_check_slots: slot preconditions violated */
    LA_ERR_CUDA = 6         /* the CUDA runtime refused the launch (see la_last_cuda_error) */
} la_status;

/* Bits OR-ed into *err_word by the kernels. */
#define LA_DEVERR_READ_SLOT 1u  /* a read / source slot index outside [0, n_slots) */
#define LA_DEVERR_WRITE_SLOT 2u /* a write / destination slot index outside [0, n_slots) */
#define LA_DEVERR_CU_SEQLENS 4u /* cu_seqlens not non-decreasing within [0, total_tokens], or a bad seq_order entry */
#define LA_DEVERR_TIMEOUT 8u    /* an internal pipeline wait gave up (should never happen) */
#define LA_DEVERR_Q8_MASK 16u   /* a q8 head's channel mask does not hold exactly n_hp rows */

typedef struct {
    int32_t n_qk_heads; /* H_qk: heads of q and k */
    int32_t n_v_heads;  /* H_v: heads of v, o and of the state; a multiple of H_qk */
    int32_t d_k;
    int32_t d_v;
} la_shape;

/* A slot pool: n_slots states of `shape`, contiguous, [n_slots, H_v, d_k, d_v].
 *
 * LA_Q8 pools hold the state in the mixed precision of DAMP ("Seven Architectures ...",
 * sections "ONNX LinearAttention / FlashInfer" and Practical Implications: the high-risk
 * key channels in a higher precision, the rest in INT8, about 9.9 bits per value).  The
 * pages fix no layout; this library's: per (slot, head) tile, the key channels (rows)
 * whose bit is set in the head's mask are kept in BF16, every other row in INT8 codes
 * with one FP32 scale per group of 32 columns:
 *   s = absmax * fl(1/127),  inv = fl(1/absmax) * 127,  code = clamp(rint(x * inv), -127, 127),
 *   x' = code * s
 * (NaN codes to 0; s = inv = 0 and codes 0 for an all-zero group; every operation a
 * correctly rounded FP32 one).  Tile
 * bytes: codes [d_k - n_hp][d_v] int8, scales [d_k - n_hp][d_v / 32] float32, BF16 rows
 * [n_hp][d_v], each block in increasing row order; n_hp = d_k / 8 gives 9.875 bits per
 * value.  (d_k, d_v) in {(64,64), (128,64), (128,128)}; n_hp even, 0 <= n_hp <= d_k / 4.
 * The mask (which channels are high-risk) comes from an offline calibration that is not
 * part of this library. */
typedef struct {
    void *data;     /* device pointer, 16-byte aligned */
    int32_t dtype;  /* la_dtype of the stored state */
    int32_t n_slots;
    la_shape shape;
    int32_t n_hp;             /* LA_Q8: BF16 key channels per head; ignored otherwise */
    const uint32_t *hp_mask;  /* LA_Q8: device uint32 [H_v][d_k / 32], bit i of head h's words
                                 set for a BF16 channel (exactly n_hp per head); else NULL */
} la_pool;

/* Bytes of one slot of `pool` for any dtype (q8 included); 0 for an invalid pool.  Pure
 * host function. */
size_t la_pool_slot_bytes(const la_pool *pool);

/* Bytes of one slot (one request's state for one layer) of an LA_F32 or LA_BF16 pool:
 * H_v * d_k * d_v * sizeof(dtype) (0 for LA_Q8: see la_pool_slot_bytes).
 * Pure host function; returns 0 for an invalid shape or dtype.  For 64 heads of 128 x 128
 * at 2 bytes this is 2 MiB, the per-request figure of the ONNX section of "Seven
 * Architectures ..."; for 128 heads of 128 x 64 at BF16 it is 2 MiB, the Nemotron-H-8B
 * per-layer figure of "SSM / linear-RNN decode: the constant-size recurrent state update". */
size_t la_state_bytes(const la_shape *shape, la_dtype dtype);

/* 1 if (d_k, d_v) is one of the compiled tile shapes, else 0.  Pure host function. */
int la_shape_supported(int32_t d_k, int32_t d_v);

/* One batched decode step (one token per request) for B requests and all H_v heads.
 *   src, dst     pools with identical shape and dtype (they may be the same pool)
 *   read_slot    device int32 [B] or NULL (request b reads src slot b)
 *   write_slot   device int32 [B] or NULL (request b writes dst slot b)
 *   q, k         [B, H_qk, d_k] io dtype;  v, o: [B, H_v, d_v] io dtype
 *   g            float32 [B, H_v]; required for gated / gated_delta, ignored otherwise;
 *                kda: float32 [B, H_v, d_k] (16-byte aligned), required
 *   beta         float32 [B, H_v]; required for delta / gated_delta, ignored otherwise
 *   scale        multiplies the readout (1.0 for pre-normalised queries)
 *   err_word     device int32, required; bits LA_DEVERR_* are OR-ed in
 * B == 0 is a no-op returning LA_OK.  With a NULL slot array, B must not exceed that
 * pool's n_slots (LA_ERR_SHAPE). */
la_status la_state_step(la_rule rule, const la_pool *src, const int32_t *read_slot,
                        const la_pool *dst, const int32_t *write_slot, int32_t B,
                        const void *q, const void *k, const void *v, la_dtype io,
                        const float *g, const float *beta, float scale, void *o,
                        int32_t *err_word, void *stream);

/* Token-serial scan (prefill) over n_seqs packed variable-length sequences.  The state
 * of each (sequence, head) stays on chip in FP32 across all of the sequence's tokens;
 * it is read once at the start and stored once at the end.
 *   src, read_slot  initial state: src slot read_slot[s]; if read_slot is NULL the
 *                   initial state is zero and src may be NULL.  src may have another
 *                   dtype than dst, but the same shape.
 *   dst, write_slot final state goes to dst slot write_slot[s] (NULL: slot s)
 *   cu_seqlens      device int32 [n_seqs + 1]: sequence s is tokens
 *                   [cu_seqlens[s], cu_seqlens[s+1]) of the packed arrays
 *   total_tokens    T, the leading size of q, k, v, g, beta, o
 *   seq_order       device int32 [n_seqs] or NULL: the order in which sequences are
 *                   handed to the SMs (longest first balances the load best); each
 *                   sequence must appear exactly once.  NULL = 0, 1, 2, ...
 *   q, k            [T, H_qk, d_k];  v, o: [T, H_v, d_v];  g, beta: [T, H_v]
 *                   (kda: g is [T, H_v, d_k], 16-byte aligned)
 * Empty sequences are allowed (their initial state is copied to the destination).
 * n_seqs == 0 is a no-op returning LA_OK. */
la_status la_state_scan(la_rule rule, const la_pool *src, const int32_t *read_slot,
                        const la_pool *dst, const int32_t *write_slot, int32_t n_seqs,
                        const int32_t *cu_seqlens, int32_t total_tokens, const int32_t *seq_order,
                        const void *q, const void *k, const void *v, la_dtype io,
                        const float *g, const float *beta, float scale, void *o,
                        int32_t *err_word, void *stream);

/* The scan of la_state_scan evaluated in chunks of 64 tokens on the tensor cores: the
 * chunkwise-parallel form of the "Kimi Linear" section and the chunkwise WY algorithm of
 * the "Gated DeltaNet-2" section of "Seven Architectures ...".  Within a chunk the
 * delta-rule corrections are solved exactly with a triangular (UT) transform; the
 * products run with BF16 operands and FP32 accumulation, and the state stays in FP32
 * across the sequence.  Results agree with la_state_scan to BF16 precision, not bit for
 * bit: within 1e-2 of the largest output or state value (up to 7e-3 measured over
 * sequences of 2,000 tokens, every rule, gates in [-1, 1] and beta in [0, 2] included).
 * Arguments, outputs and errors as la_state_scan.  Supported: d_k = d_v = 128 with BF16
 * q/k/v/o, the rules linear, gated, delta and gated_delta, gates of either sign, FP32, BF16
 * or q8 pools (LA_ERR_UNSUPPORTED otherwise; kda has the two-launch form
 * la_state_scan_chunked_ws, which takes FP32 or BF16 pools). */
la_status la_state_scan_chunked(la_rule rule, const la_pool *src, const int32_t *read_slot,
                                const la_pool *dst, const int32_t *write_slot, int32_t n_seqs,
                                const int32_t *cu_seqlens, int32_t total_tokens, const int32_t *seq_order,
                                const void *q, const void *k, const void *v, la_dtype io,
                                const float *g, const float *beta, float scale, void *o,
                                int32_t *err_word, void *stream);

/* la_state_scan_chunked in two launches: the intra-chunk part of every chunk as one parallel
 * launch writing a caller-owned workspace, then the recurrence over the chunks reading it,
 * on the fifth-generation tensor cores (tcgen05 MMAs, the state in tensor memory).  The
 * chunks are independent in the first launch, so it fills the SMs (several CTAs each)
 * instead of sitting on each sequence's critical path.  Same precision as
 * la_state_scan_chunked (BF16 products, FP32 accumulation and state), not bit for bit.
 *   delta rules      the first launch forms K K^T, the triangular inverse T,
 *                    Tw = T diag(beta gamma) and Tu = T diag(beta) (17.9 KB per chunk and head)
 *   kda              the channel-wise gate ("Kimi Linear": S <- (I - beta k k^T) Diag(alpha) S
 *                    + beta k v^T): the chunk's decay products Gamma_t (d_k vectors) are
 *                    absorbed into the operands, Q (.) Gamma, K (.) Gamma and
 *                    K (.) Gamma_C / Gamma, and into the intra-chunk products [Q; K] K^T, whose
 *                    ratios Gamma_t / Gamma_s are factored around the middle of each 16-token
 *                    block; the first launch writes those operands, P, Tw = T diag(beta) and
 *                    Gamma_C (65 KB per chunk and head).  Each token's decay magnitude is
 *                    taken within [e^-8, e^8]: magnitudes below e^-8, zero included, act as
 *                    e^-8 (sign kept), a change of at most e^-8 (3.4e-4) of a decayed state
 *                    row; within 1e-2 of la_state_scan for decays in [-1, 1] and beta in [0, 2].
 *   workspace        device, 16-byte aligned, at least
 *                    la_scan_chunked_workspace_bytes_rule(rule, total_tokens, n_seqs, H_v)
 *                    bytes (la_scan_chunked_workspace_bytes: the same for the delta rules);
 *                    contents are scratch (overwritten, not read back by the caller)
 * Other arguments, supported set and errors as la_state_scan_chunked (kda added); for the
 * delta rules and kda LA_ERR_SHAPE when workspace_bytes is too small and LA_ERR_NULL for a
 * NULL workspace.  The linear and gated rules have no intra-chunk launch and run the
 * one-launch form: the workspace and its size are ignored (NULL allowed, never touched), and
 * la_scan_chunked_workspace_bytes_rule returns 0 for them (and for an unknown rule). */
size_t la_scan_chunked_workspace_bytes(int32_t total_tokens, int32_t n_seqs, int32_t n_v_heads);
size_t la_scan_chunked_workspace_bytes_rule(la_rule rule, int32_t total_tokens, int32_t n_seqs,
                                            int32_t n_v_heads);
la_status la_state_scan_chunked_ws(la_rule rule, const la_pool *src, const int32_t *read_slot,
                                   const la_pool *dst, const int32_t *write_slot, int32_t n_seqs,
                                   const int32_t *cu_seqlens, int32_t total_tokens,
                                   const int32_t *seq_order, const void *q, const void *k,
                                   const void *v, la_dtype io, const float *g, const float *beta,
                                   float scale, void *o, void *workspace, size_t workspace_bytes,
                                   int32_t *err_word, void *stream);

/* la_state_scan_chunked_ws with the library's own workspace: a fixed 256 MiB device array
 * of this library (one per device), so the caller passes no scratch buffer.  The array is
 * a file-scope __device__ variable of the library's device code: it is reserved on a
 * device when the module holding it is loaded there, which under the CUDA runtime's lazy
 * module loading (the default) is this entry point's first call on that device, and under
 * CUDA_MODULE_LOADING=EAGER is context creation -- then every process that loads the
 * library pays the 256 MiB per device, callers of the other entry points included.  It
 * stays reserved until the process exits (or the device is reset).  The array is
 * shared by every call on a device: calls must not run concurrently on one device (the
 * caller orders them, for example on one stream).  A call of a delta rule or kda whose
 * workspace would exceed the array (la_scan_chunked_workspace_bytes_rule(rule,
 * total_tokens, n_seqs, H_v) > 256 MiB) returns LA_ERR_SHAPE before launching anything;
 * the linear and gated rules do not use the array and have no such limit.  A failed device query or symbol lookup
 * returns LA_ERR_CUDA.  Other arguments and errors as la_state_scan_chunked. */
la_status la_state_scan_chunked_noalloc(la_rule rule, const la_pool *src, const int32_t *read_slot,
                                        const la_pool *dst, const int32_t *write_slot, int32_t n_seqs,
                                        const int32_t *cu_seqlens, int32_t total_tokens,
                                        const int32_t *seq_order, const void *q, const void *k,
                                        const void *v, la_dtype io, const float *g, const float *beta,
                                        float scale, void *o, int32_t *err_word, void *stream);

/* The scan of la_state_scan that also stores intermediate states: the prefix-cache
 * checkpoints at KV-cache block boundaries of the "Gated DeltaNet" glossary page (Why
 * it matters), and state snapshots for speculative-decoding rollback ("Seven
 * Architectures ...", Limitations and Open Questions).
 *   ckpt_every  > 0; checkpoint j of sequence s is the state after the sequence's first
 *               (j + 1) * ckpt_every tokens (the state the next token would start from)
 *   ckpt_cu     device int32 [n_seqs + 1]: sequence s has checkpoints
 *               ckpt_slots[ckpt_cu[s] .. ckpt_cu[s+1]), at most len(s) / ckpt_every of them
 *   ckpt_slots  device int32: destination slots in dst (dst dtype), distinct from every
 *               write slot and every read slot
 * Other arguments and errors as la_state_scan.  A sequence with more checkpoints than fit
 * reports LA_DEVERR_CU_SEQLENS (the ones that fit are written); an out-of-range
 * checkpoint slot reports LA_DEVERR_WRITE_SLOT and is skipped.  Host errors: ckpt_every
 * <= 0 (LA_ERR_SHAPE), NULL ckpt arrays (LA_ERR_NULL). */
la_status la_state_scan_checkpointed(la_rule rule, const la_pool *src, const int32_t *read_slot,
                                     const la_pool *dst, const int32_t *write_slot, int32_t n_seqs,
                                     const int32_t *cu_seqlens, int32_t total_tokens,
                                     const int32_t *seq_order, const void *q, const void *k,
                                     const void *v, la_dtype io, const float *g, const float *beta,
                                     float scale, void *o, int32_t ckpt_every, const int32_t *ckpt_cu,
                                     const int32_t *ckpt_slots, int32_t *err_word, void *stream);

/* la_state_scan_checkpointed evaluated by la_state_scan_chunked (one launch): the checkpoints
 * fall on chunk boundaries, so ckpt_every must be a multiple of 64 (the chunk length); each
 * checkpoint is the FP32 state the chunked recurrence holds at that boundary, stored in the dst
 * dtype.  Arguments, checkpoint semantics and errors as la_state_scan_checkpointed; supported
 * set as la_state_scan_chunked; LA_ERR_UNSUPPORTED when ckpt_every is not a multiple of 64. */
la_status la_state_scan_chunked_checkpointed(la_rule rule, const la_pool *src, const int32_t *read_slot,
                                             const la_pool *dst, const int32_t *write_slot, int32_t n_seqs,
                                             const int32_t *cu_seqlens, int32_t total_tokens,
                                             const int32_t *seq_order, const void *q, const void *k,
                                             const void *v, la_dtype io, const float *g, const float *beta,
                                             float scale, void *o, int32_t ckpt_every,
                                             const int32_t *ckpt_cu, const int32_t *ckpt_slots,
                                             int32_t *err_word, void *stream);

/* The short causal convolution fused ahead of the decode step ("Gated DeltaNet" glossary,
 * Engineering details: Conv1D fused with the recurrence into one kernel).  The pages give
 * no width, activation or normalisation; this library's reading: per channel c of the q,
 * k and v projections, a depthwise causal convolution along time,
 *   y_t[c] = sum_{j < W} w[c][j] x_{t-W+1+j}[c],
 * optionally followed by SiLU (y / (1 + e^-y)), then q and k optionally scaled to unit
 * length per head (y / sqrt(|y|^2 + 1e-6)); the results (FP32, not rounded) are the q, k, v
 * of the step.  The W - 1 earlier inputs of every channel are kept per (slot, state head):
 * head h holds its q/k head's 2 d_k channels and its own d_v channels (heads sharing a q/k
 * head hold equal copies, so no two tiles ever write the same history). */
typedef struct {
    int32_t width;          /* W, 2 <= W <= 4 */
    int32_t activation;     /* 0: none, 1: SiLU */
    int32_t qk_l2norm;      /* 1: q and k scaled to unit length per head after the convolution */
    const float *w_q;       /* device float32 [H_qk][d_k][W] (w[c][W - 1] multiplies the newest
                               input); 16-byte aligned, like w_k and w_v */
    const float *w_k;       /* device float32 [H_qk][d_k][W] */
    const float *w_v;       /* device float32 [H_v][d_v][W] */
    const void *hist_src;   /* device, io dtype [src n_slots][H_v][2 d_k + d_v][W - 1] (q, k, v
                               channels; oldest input first), read at read_slot; 16-byte aligned */
    void *hist_dst;         /* same layout with dst n_slots, written at write_slot (may equal hist_src) */
} la_conv;

/* la_state_step with the convolution ahead of it: xq, xk, xv are the convolution's inputs
 * (layouts of q, k, v); everything else as la_state_step.  FP32 or BF16 pools (not q8). */
la_status la_state_step_conv(la_rule rule, const la_pool *src, const int32_t *read_slot,
                             const la_pool *dst, const int32_t *write_slot, int32_t B,
                             const la_conv *conv, const void *xq, const void *xk, const void *xv,
                             la_dtype io, const float *g, const float *beta, float scale, void *o,
                             int32_t *err_word, void *stream);

/* la_state_scan with the convolution ahead of every token: xq, xk, xv are the
 * convolution's inputs (layouts of q, k, v).  Each (sequence, head) history is read from
 * conv->hist_src at read_slot[s] (zero when read_slot is NULL: a fresh prefill), carried
 * through the sequence, and the history after its last token is written to
 * conv->hist_dst at write_slot[s] (an empty sequence passes its history through), ready
 * for la_state_step_conv.  FP32 or BF16 pools, the default head direction, no
 * checkpoints (LA_ERR_UNSUPPORTED otherwise).  Other arguments and errors as
 * la_state_scan. */
la_status la_state_scan_conv(la_rule rule, const la_pool *src, const int32_t *read_slot,
                             const la_pool *dst, const int32_t *write_slot, int32_t n_seqs,
                             const int32_t *cu_seqlens, int32_t total_tokens,
                             const int32_t *seq_order, const la_conv *conv, const void *xq,
                             const void *xk, const void *xv, la_dtype io, const float *g,
                             const float *beta, float scale, void *o, int32_t *err_word,
                             void *stream);

/* la_state_scan_chunked with the convolution of la_state_scan_conv ahead of every token, in
 * the same launch ("Gated DeltaNet" glossary, Engineering details: the convolution fused
 * with the recurrence): each chunk's raw xq, xk, xv are convolved (then SiLU, then q and k
 * to unit length, as conv asks) in place in shared memory after they are staged, two chunks
 * ahead of the chunk's products; each (sequence, head) carries the window of its last
 * W - 1 raw inputs from chunk to chunk, starting from conv->hist_src at read_slot[s] (zero
 * when read_slot is NULL) and leaving it in conv->hist_dst at write_slot[s] (an empty
 * sequence passes its history through).  The convolved q, k, v are rounded to BF16 before
 * the products (q and k normalised from the rounded values).  Supported: the scalar-gate
 * rules, d_k = d_v = 128, BF16 io and histories (LA_ERR_UNSUPPORTED otherwise, kda
 * included).  Other arguments and errors as la_state_scan_conv. */
la_status la_state_scan_chunked_conv(la_rule rule, const la_pool *src, const int32_t *read_slot,
                                     const la_pool *dst, const int32_t *write_slot, int32_t n_seqs,
                                     const int32_t *cu_seqlens, int32_t total_tokens,
                                     const int32_t *seq_order, const la_conv *conv, const void *xq,
                                     const void *xk, const void *xv, la_dtype io, const float *g,
                                     const float *beta, float scale, void *o, int32_t *err_word,
                                     void *stream);

/* la_state_scan_chunked_conv in two launches: the convolution of every (chunk, state head)
 * as a launch of its own (each chunk reads the raw rows before it, or the history at the
 * read slot, so every chunk is independent), writing the convolved q, k, v of every state
 * head to a caller-owned workspace, then the chunked prefill reading them.  Same results as
 * la_state_scan_chunked_conv up to the order of the products (histories identical).
 *   workspace        device, 16-byte aligned, at least
 *                    la_scan_chunked_conv_workspace_bytes(total_tokens, H_v) bytes (a header
 *                    and 3 T H_v 128 BF16 values); contents are scratch
 * LA_ERR_NULL for a NULL workspace, LA_ERR_SHAPE when it is too small; other arguments,
 * supported set and errors as la_state_scan_chunked_conv. */
size_t la_scan_chunked_conv_workspace_bytes(int32_t total_tokens, int32_t n_v_heads);
la_status la_state_scan_chunked_conv_ws(la_rule rule, const la_pool *src, const int32_t *read_slot,
                                        const la_pool *dst, const int32_t *write_slot, int32_t n_seqs,
                                        const int32_t *cu_seqlens, int32_t total_tokens,
                                        const int32_t *seq_order, const la_conv *conv, const void *xq,
                                        const void *xk, const void *xv, la_dtype io, const float *g,
                                        const float *beta, float scale, void *o, void *workspace,
                                        size_t workspace_bytes, int32_t *err_word, void *stream);

/* The query-group direction of the ONNX LinearAttention operator ("Seven Architectures
 * ...", section "ONNX LinearAttention / FlashInfer": each KV head and its recurrent state
 * shared by a group of query heads, q_num_heads / kv_num_heads).  The state of head h is
 * updated once per token with its own key k_h, value v_h and gates; query head i then
 * reads the updated state of head i / (n_q_heads / H_v):
 *   o_i = scale * S_h^T q_i        (rearranged in the kernels as for la_state_step)
 *   pools     n_qk_heads == n_v_heads (the key has one head per state head)
 *   q         [B or T, n_q_heads, d_k] io dtype;  k: [B or T, H_v, d_k];  v: [B or T, H_v, d_v]
 *   o         [B or T, n_q_heads, d_v] io dtype;  g, beta as for la_state_step / la_state_scan
 *   n_q_heads a multiple of H_v with n_q_heads / H_v <= 8 (LA_ERR_SHAPE when not a
 *             multiple or when n_qk_heads != n_v_heads; LA_ERR_UNSUPPORTED above 8)
 * Other arguments, supported shapes and errors as la_state_step / la_state_scan. */
la_status la_state_step_qgroups(la_rule rule, const la_pool *src, const int32_t *read_slot,
                                const la_pool *dst, const int32_t *write_slot, int32_t B,
                                int32_t n_q_heads, const void *q, const void *k, const void *v,
                                la_dtype io, const float *g, const float *beta, float scale,
                                void *o, int32_t *err_word, void *stream);
la_status la_state_scan_qgroups(la_rule rule, const la_pool *src, const int32_t *read_slot,
                                const la_pool *dst, const int32_t *write_slot, int32_t n_seqs,
                                const int32_t *cu_seqlens, int32_t total_tokens,
                                const int32_t *seq_order, int32_t n_q_heads, const void *q,
                                const void *k, const void *v, la_dtype io, const float *g,
                                const float *beta, float scale, void *o, int32_t *err_word,
                                void *stream);
/* The same on the chunked (WY/UT) form of la_state_scan_chunked, its precision claim and
 * supported shapes (d_k = d_v = 128, BF16 io, rules other than kda, FP32/BF16/q8 pools).
 * The one-launch chunked pass runs once per query of the group, each writing its query
 * head's outputs; the state is the same in every pass and is written by the last, so a
 * request may read and write one slot. */
la_status la_state_scan_chunked_qgroups(la_rule rule, const la_pool *src,
                                        const int32_t *read_slot, const la_pool *dst,
                                        const int32_t *write_slot, int32_t n_seqs,
                                        const int32_t *cu_seqlens, int32_t total_tokens,
                                        const int32_t *seq_order, int32_t n_q_heads,
                                        const void *q, const void *k, const void *v, la_dtype io,
                                        const float *g, const float *beta, float scale, void *o,
                                        int32_t *err_word, void *stream);

/* Slot-pool maintenance, bit-exact whole-slot copies ("Recurrent state" glossary: slot
 * allocation and prefix-cache checkpoints; "Seven Architectures ...", ONNX section:
 * snapshots saved and restored for speculative-decoding rollback, migrated between
 * places).  n == 0 is a no-op.  Slot arrays are device int32 [n].
 *   copy     pool[dst_slots[i]] <- pool[src_slots[i]]; the destination set must not
 *            intersect the source set (except a slot copied onto itself)
 *   gather   dense[i] <- pool[slots[i]]          dense: [n, H_v, d_k, d_v], pool dtype
 *   scatter  pool[slots[i]] <- dense[i]
 *   zero     pool[slots[i]] <- 0 */
la_status la_state_pool_copy(const la_pool *pool, int32_t n, const int32_t *src_slots,
                             const int32_t *dst_slots, int32_t *err_word, void *stream);
la_status la_state_pool_gather(const la_pool *pool, int32_t n, const int32_t *slots, void *dense,
                               int32_t *err_word, void *stream);
la_status la_state_pool_scatter(const la_pool *pool, int32_t n, const int32_t *slots,
                                const void *dense, int32_t *err_word, void *stream);
la_status la_state_pool_zero(const la_pool *pool, int32_t n, const int32_t *slots,
                             int32_t *err_word, void *stream);

/* Conversion between FP32 states and the slots of an LA_Q8 pool (for example, a prefill
 * state handed to a quantised decode pool, or a quantised state read back):
 *   encode   pool[slots[i]] <- q8(dense[i])      dense: float32 [n, H_v, d_k, d_v]
 *   decode   dense[i] <- values of pool[slots[i]]
 * A slot index outside the pool reports LA_DEVERR_WRITE_SLOT (encode) or
 * LA_DEVERR_READ_SLOT (decode); a head whose mask does not hold n_hp rows reports
 * LA_DEVERR_Q8_MASK; those tiles are skipped.  LA_ERR_UNSUPPORTED for a pool that is not
 * LA_Q8. */
la_status la_state_pool_encode(const la_pool *pool, int32_t n, const int32_t *slots,
                               const float *dense, int32_t *err_word, void *stream);
la_status la_state_pool_decode(const la_pool *pool, int32_t n, const int32_t *slots, float *dense,
                               int32_t *err_word, void *stream);

/* Host-side check of the slot preconditions of la_state_step / la_state_scan on HOST
 * copies of the slot arrays (either may be NULL = identity): every index in [0, n_slots),
 * write slots distinct, no write slot equal to another request's read slot.  Returns
 * LA_OK, LA_ERR_SHAPE (index out of range) or LA_ERR_ALIAS. */
la_status la_state_check_slots(int32_t B, const int32_t *read_slot_host,
                               const int32_t *write_slot_host, int32_t n_slots);

/* Human-readable name of a status. */
const char *la_status_str(la_status status);

/* The cudaError_t of the most recent LA_ERR_CUDA returned on the calling thread (0 if none). */
int32_t la_last_cuda_error(void);

/* LA_ABI_VERSION of the loaded library. */
int32_t la_abi_version(void);

/* Failure-path test hooks.  Every pipeline wait inside the kernels has a time limit after
 * which the kernel stops, reports LA_DEVERR_TIMEOUT through the error word and returns, so
 * the CUDA context stays usable.  These two calls let a test exercise that path without any
 * fault: they change nothing else, and results are unaffected while they are unused.
 *   la_debug_set_wait_limit_us  the limit of the decode step's (la_state_step and its
 *                               variants) waits on the calling thread, in microseconds;
 *                               0 restores the default of one second
 *   la_debug_withhold_step_tile the next decode step on the calling thread withholds the
 *                               given tile (its index in the first CTA's order, 0 = first):
 *                               the producer issues no copy for it and signals nothing, so
 *                               the consumers' waits run out (nothing is left in flight); one
 *                               call only affects one step; a negative tile cancels it */
void la_debug_set_wait_limit_us(uint32_t us);
void la_debug_withhold_step_tile(int32_t tile);

#ifdef __cplusplus
}
#endif

#endif /* LA_STATE_H */
