/*
 * sattn.h -- C ABI of libsattn.so: causal self-attention over a structured,
 * data-dependent key set, for NVIDIA B200 (sm_100a).
 *
 * For query row i the key set is the union of
 *   - the starting span  j < n_start                  ("LM-Infinite", NAACL
 *     2024 summary, section 方法, equation A_i),
 *   - the recent window  0 <= i-j <= window            (same equation),
 *   - every earlier separator token, j < i            ("SepLLM", CSDN
 *     article, section 五.2, mask M_ij),
 *   - optionally, per query head, the topk middle tokens with the largest
 *     attention logit                                  ("LM-Infinite",
 *     section 方法, optional top-k paragraph),
 * restricted to j <= i.  Masked keys get -inf before the softmax ("SepLLM",
 * section 6.1 read together with 五.2).  The distance cap of LM-Infinite
 * (section 方法, equations d_ij and d'_ij = min(d_ij, L)) applies to every
 * logit: when L_pretrain > 0 and i-j > L_pretrain the logit is
 * <R(L_pretrain) q_i, k_j> with k_j unrotated (the RoPE realisation in the
 * same section); otherwise <R(i) q_i, R(j) k_j>.  Logits are scaled by
 * 1/sqrt(d).  R(p) is rotate-half RoPE with inverse frequencies
 * theta^(-2c/d); rope_theta = 0 disables rotation.  Query head h uses
 * key/value head floor(h * Hkv / Hq).
 *
 * sattn_segment_fwd implements segmented execution ("Training-Inference
 * Consistent Segmented Execution for Long-Context LLMs", sections 整体框架
 * and 关键设计).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every function returns an int status (SATTN_OK or a negative code) and
 *    never throws.  sattn_strerror() gives the text.
 *  - Tensor arguments are DEVICE pointers owned by the caller.  The library
 *    never allocates: all scratch lives in the caller's workspace `ws` of at
 *    least the size returned by the matching *_workspace_size call.  `ws`
 *    must be 256-byte aligned.
 *  - Q/K/V/O are [B, H, T, d] with the head dimension contiguous and the
 *    element strides given in sattn_params (batch, head, token).  For bf16
 *    the token stride must make rows 16-byte aligned (stride * 2 % 16 == 0)
 *    and base pointers 16-byte aligned (the tensor-memory-access engine
 *    loads tiles straight from these tensors).
 *  - Launches are asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = the legacy default stream).  Argument errors are detected on
 *    the host before any launch and leave every output untouched.
 *  - Device-side failures (a bounded wait that timed out) are written to a
 *    status word inside the workspace; sattn_stream_status() synchronises
 *    the stream and reads it.  Each entry point clears the word first.
 *  - Results are deterministic: no floating-point atomics; repeated calls on
 *    the same inputs are bit-identical.
 */
#ifndef SATTN_H_
#define SATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SATTN_OK 0
#define SATTN_ERR_INVALID_ARG (-1)
#define SATTN_ERR_UNSUPPORTED (-2)
#define SATTN_ERR_CUDA (-3)
#define SATTN_ERR_TIMEOUT (-4)

#define SATTN_DTYPE_BF16 0
#define SATTN_DTYPE_F32 1

/* Problem description.  Field meanings follow the pages' problem statement. */
typedef struct sattn_params {
  int32_t B;          /* batch */
  int32_t Hq;         /* query heads */
  int32_t Hkv;        /* key/value heads; Hq % Hkv == 0 */
  int32_t T;          /* sequence length, >= 1 */
  int32_t d;          /* head dimension: 64 or 128 */
  int32_t dtype;      /* SATTN_DTYPE_BF16 or SATTN_DTYPE_F32 (O has this type too) */
  int64_t q_stride[3];  /* element strides of Q: batch, head, token */
  int64_t k_stride[3];  /* of K */
  int64_t v_stride[3];  /* of V */
  int64_t o_stride[3];  /* of O */
  int32_t n_start;    /* starting ("sink") span, >= 0           (LM-Infinite A_i; SepLLM a) */
  int32_t window;     /* recent window w: keys with i-j <= w, >= 0 (LM-Infinite L; SepLLM n) */
  int32_t L_pretrain; /* distance cap; 0 = no cap                 (LM-Infinite d'_ij) */
  int32_t topk;       /* extra middle tokens per row and query head; 0 = none, <= 16 */
  int32_t with_separators; /* nonzero: is_sep may be passed; the workspace then holds the
                              separator compaction and gathered K/V (worst case: every token) */
  double rope_theta;  /* rotary base; 0 = no rotation */
  double rope_pos_scale; /* position interpolation: rotary positions are multiplied by this
                            before rotation (distances too); 0 or 1 = none; (0, 1] */
  int32_t alibi;      /* nonzero: ALiBi bias instead of rotation (rope_theta must be 0):
                         s_ij = q.k/sqrt(d) - m_h * min(i-j, L_pretrain) (no clip when
                         L_pretrain == 0), head slopes m_h = 2^(-8 (h+1) / Hq)
                         ("LM-Infinite", section 方法: the bias clipped at the same cap).
                         SATTN_ERR_UNSUPPORTED: with top-k unless L_pretrain > 0 and
                         window >= L_pretrain; with separators on the bf16 path unless
                         L_pretrain > 0; in sattn_segment_fwd */
  int32_t tile_m;     /* query tile (rows per tile of the block map and the kernels): 0 or 128 */
  int32_t tile_n;     /* key tile: 0 or 128.  The kernels are built for 128 x 128 tiles (the
                         tensor-core tile and the TMEM layout); other sizes return
                         SATTN_ERR_UNSUPPORTED */
} sattn_params;

/* Text of a status code (static storage). */
const char* sattn_strerror(int status);

/* Library version: major*10000 + minor*100 + patch. */
int sattn_version(void);

/* Bytes of workspace needed by sattn_fwd, sattn_topk_select and
 * sattn_build_blockmap for these parameters (the same buffer serves all
 * three).  Returns SATTN_ERR_INVALID_ARG / SATTN_ERR_UNSUPPORTED for
 * parameters the entry points would reject. */
int sattn_workspace_size(const sattn_params* p, size_t* bytes);

/* Bytes of workspace needed by sattn_segment_fwd; is_long is the same [Hq]
 * HOST array the call will get (NULL: size for every head long). */
int sattn_segment_workspace_size(const sattn_params* p, int32_t S, int32_t M, int32_t R,
                                 int32_t retr_block, const uint8_t* is_long, size_t* bytes);

/* Block map and separator compaction (the structural mask of the header
 * comment, top-k excluded since it is per head), with 128x128 tiles.
 *   is_sep          [B, T] uint8 flags (nonzero = separator), or NULL = none.
 *   cls             [B, ceil(T/128), ceil(T/128)] uint8, out: 0 empty,
 *                   1 partial, 2 full, over in-range (i, j) pairs; may be NULL.
 *   sep_pos         [B, T] int32, out: positions j >= n_start of separators in
 *                   ascending order, then -1.
 *   sep_count       [B] int32, out: number of such separators.
 *   qtile_sep_range [B, ceil(T/128), 2] int32, out: per query tile t, the
 *                   number of separators with j < 128t - window (kept by every
 *                   row of the tile) and with j < last_row(t) - window (kept by
 *                   at least one row).
 * All outputs are device pointers. */
int sattn_build_blockmap(const sattn_params* p, const uint8_t* is_sep, uint8_t* cls, int32_t* sep_pos,
                         int32_t* sep_count, int32_t* qtile_sep_range, void* ws, size_t ws_bytes,
                         void* stream);

/* Top-k middle-token selection ("LM-Infinite", section 方法, optional top-k).
 * For every (b, query head h, row i) the p->topk keys j with
 * n_start <= j < i - window that are not separators, ranked by the unscaled
 * logit z_ij (capped rule of the header comment), ties to the smaller j.
 *   Q, K       inputs as in sattn_fwd (V is not needed).
 *   is_sep     [B, T] uint8 or NULL.
 *   idx        [B, Hq, T, topk] int32, out: selected j sorted by (z desc, j asc);
 *              -1 when fewer than topk candidates exist.
 *   logit      [B, Hq, T, topk] float, out: z_ij in fp32; -inf for padding.
 * bf16 only.  With 0 < window < L_pretrain a candidate with i - j <= L_pretrain
 * is scored with the uncapped logit <R(i) q, R(j) k>, a farther one with the
 * capped <R(L) q, k>. */
int sattn_topk_select(const sattn_params* p, const void* Q, const void* K, const uint8_t* is_sep,
                      int32_t* idx, float* logit, void* ws, size_t ws_bytes, void* stream);

/* Forward attention over the structured key set.
 *   Q [B,Hq,T,d], K,V [B,Hkv,T,d]   dtype p->dtype, strides in p.
 *   is_sep      [B, T] uint8 or NULL (no separators).
 *   topk_idx    [B, Hq, T, topk] int32 or NULL; topk_logit likewise (float).
 *               When p->topk > 0 and topk_idx is NULL the selection of
 *               sattn_topk_select runs inside this call.  When given, they
 *               must be a selection in that format (middle, non-separator
 *               keys; -1 padding); the logits are used as the keys' z.
 *   O           [B, Hq, T, d], out, dtype p->dtype, strides p->o_stride.
 *   lse         [B, Hq, T] float, out: natural-log logsumexp of the scaled
 *               logits of each row.
 * bf16 runs on the tensor cores; fp32 runs on the CUDA cores in fp32.
 * With bf16 and L_pretrain > 0: window <= L_pretrain (SATTN_ERR_UNSUPPORTED
 * otherwise).  Separators and top-k keys may sit on either side of the cap
 * when window < L_pretrain: those with window < i - j <= L_pretrain take the
 * uncapped logit, the farther ones the capped one. */
int sattn_fwd(const sattn_params* p, const void* Q, const void* K, const void* V, const uint8_t* is_sep,
              const int32_t* topk_idx, const float* topk_logit, void* O, float* lse, void* ws, size_t ws_bytes,
              void* stream);

/* Segmented execution of one layer ("Training-Inference Consistent Segmented
 * Execution", sections 整体框架 and 关键设计).  The sequence is cut into T/S
 * segments.  For a query in segment s:
 *   local heads (is_long[h] == 0): the carried tail, keys [sS-M, sS), at
 *     positions 0..P-1, then the segment's keys sS..i at P + (j - sS);
 *   long heads (is_long[h] != 0): a prefix of R keys retrieved from the pool
 *     [0, sS): the top R/retr_block blocks of retr_block keys scored by
 *     max_{j in block} <q_{sS-1}, k_j> (unrotated; ties to the lower block),
 *     in ascending block order at positions 0..P-1, then the segment.
 *   Segment 0 has neither tail nor prefix.  No distance cap, no sinks.
 *   is_long        [Hq] uint8 HOST array.
 *   prefix_blocks  [B, Hq, T/S, R/retr_block] int32, out: the retrieved block
 *                  indices, ascending; -1 for local heads, segment 0, or
 *                  when the pool holds fewer blocks.
 *   O, lse         as in sattn_fwd.
 * bf16 only; S % 128 == 0, T % S == 0, 1 <= retr_block, R % retr_block == 0,
 * R / retr_block <= 1024, Hq <= 256, and at most 16384 blocks in the largest
 * pool ((T - S) / retr_block), else SATTN_ERR_UNSUPPORTED. */
int sattn_segment_fwd(const sattn_params* p, int32_t S, int32_t M, int32_t R, int32_t retr_block,
                      const uint8_t* is_long, const void* Q, const void* K, const void* V, void* O, float* lse,
                      int32_t* prefix_blocks, void* ws, size_t ws_bytes, void* stream);

/* Bytes of workspace needed by sattn_segment_bwd. */
int sattn_segment_bwd_workspace_size(const sattn_params* p, int32_t S, int32_t M, int32_t R, int32_t retr_block,
                                     size_t* bytes);

/* Backward pass of sattn_segment_fwd ("Training-Inference Consistent
 * Segmented Execution", sections 整体框架 and 损失函数 / 训练策略: training
 * runs segment by segment): the gradients of sum(dO * O) with respect to Q,
 * K and V for the same parameters and key lists as the forward.  The
 * retrieved blocks are constants (the forward's prefix_blocks are an
 * input): a retrieved key's gradient returns to its source position through
 * the rotary position it had in the prefix, and a key used by several rows,
 * heads or segments sums their contributions.
 *   is_long        [Hq] uint8 HOST array, as for the forward.
 *   Q, K, V, O, lse, prefix_blocks   the forward's inputs and outputs.
 *   dO             gradient of the loss w.r.t. O, strides o_stride.
 *   dQ, dK, dV     out, shaped and strided like Q, K, V (bf16).
 * Runs on the CUDA cores in fp32 (a warp per query row for dQ, a warp per
 * key for dK and dV, each key's rows in a fixed order); deterministic.
 * Validation as sattn_segment_fwd.  Asynchronous on `stream`. */
int sattn_segment_bwd(const sattn_params* p, int32_t S, int32_t M, int32_t R, int32_t retr_block,
                      const uint8_t* is_long, const void* Q, const void* K, const void* V, const void* O,
                      const float* lse, const int32_t* prefix_blocks, const void* dO, void* dQ, void* dK, void* dV,
                      void* ws, size_t ws_bytes, void* stream);

/* ---- segmented execution one segment at a time (explicit carried state) ----
 *
 * "Training-Inference Consistent Segmented Execution for Long-Context LLMs"
 * (section 整体框架) applies the layer per segment,
 * (C_i, o^(i)) = F(x^(i), C_{i-1}, R_{i-1}): the local heads carry the tail
 * of the earlier tokens, the long heads retrieve from the pool of earlier
 * keys with the previous segment's last query.  These calls run that
 * operator on one segment at a time with the carried part in a caller-owned
 * device buffer (the state): every earlier token's raw K and V, its key
 * rotated at its position, the previous segment's last query of every head
 * and a header counting the segments taken.  Steps 0, 1, ..., N-1 give the
 * O, LSE and retrieved blocks of sattn_segment_fwd on the concatenated
 * segments (the same kernels on the same operands).
 *
 * Common arguments: p gives B, Hq, Hkv, d, the rotary base and scale, bf16,
 * and p->T = the capacity (the longest total length, a multiple of S); S, M,
 * R, retr_block as in sattn_segment_fwd, with the same rules
 * (SATTN_ERR_UNSUPPORTED / SATTN_ERR_INVALID_ARG). */

/* Bytes of the state for a capacity of p->T positions. */
int sattn_segment_state_size(const sattn_params* p, int32_t S, int32_t M, int32_t R, int32_t retr_block,
                             size_t* bytes);

/* Starts a sequence: no segment taken; builds the rotary table of every
 * position.  state: device, 256-byte aligned, at least the size above.
 * Asynchronous on `stream`. */
int sattn_segment_state_reset(const sattn_params* p, int32_t S, int32_t M, int32_t R, int32_t retr_block,
                              void* state, size_t state_bytes, void* stream);

/* Bytes of workspace needed by sattn_segment_step. */
int sattn_segment_step_workspace_size(const sattn_params* p, int32_t S, int32_t M, int32_t R, int32_t retr_block,
                                      const uint8_t* is_long, size_t* bytes);

/* Segment `seg` (0, 1, ... in order; (seg + 1) S <= p->T):
 *   is_long        [Hq] host flags, as in sattn_segment_fwd.
 *   Q, K, V        the segment's [B, Hq, S, d] / [B, Hkv, S, d] bf16 device
 *                  inputs (positions seg S ..), strides q/k/v_stride.
 *   state          the carried state; the segment is appended and its last
 *                  query kept for the next step.
 *   O, lse         [B, Hq, S, d] bf16 (o_stride) and [B, Hq, S] fp32, out.
 *   prefix_blocks  [B, Hq, R / retr_block] int32, out: the long heads'
 *                  retrieved blocks for this segment (-1 for local heads,
 *                  segment 0 and unused slots); may be NULL when R = 0.
 * A step that is not the next segment of the state (or a state that was
 * never reset) writes nothing and leaves SATTN_ERR_INVALID_ARG in the
 * workspace's status word (sattn_stream_status).  Asynchronous on `stream`. */
int sattn_segment_step(const sattn_params* p, int32_t S, int32_t M, int32_t R, int32_t retr_block,
                       const uint8_t* is_long, int32_t seg, const void* Q, const void* K, const void* V, void* state,
                       size_t state_bytes, void* O, float* lse, int32_t* prefix_blocks, void* ws, size_t ws_bytes,
                       void* stream);

/* Bytes of workspace needed by sattn_decode_fwd for *p (p->T = cache length). */
int sattn_decode_workspace_size(const sattn_params* p, size_t* bytes);

/* One decoding step: the query of the newest token, at position i = T-1,
 * attends over the structured key set of that position among the cache's
 * T entries (its own key and value are the last entry).  The key set and the
 * logits are those of sattn_fwd's row i: starting span j < n_start and
 * window i-w <= j <= i ("LM-Infinite", section 方法), earlier separators
 * n_start <= j < i-w ("SepLLM", section 五.2), the capped logit
 * <R(L) q, k_j> for i-j > L_pretrain and <R(i) q, R(j) k_j> otherwise.
 *   p        shape and mask parameters; T is the cache length, Hq/Hkv one
 *            of 1, 2, 4, 8, bf16 only.  topk > 0 adds the query's top-k
 *            middle tokens as in sattn_fwd (see sattn_decode_topk_fwd).
 *   Q        [B, Hq, 1, d] bf16 device, strides q_stride[0..1].
 *   K, V     [B, Hkv, T, d] bf16 device cache (keys unrotated), strides as
 *            in sattn_fwd.
 *   is_sep   [B, T] uint8 device flags or NULL (needs p->with_separators).
 *   O        [B, Hq, 1, d] bf16 device, out, strides o_stride[0..1].
 *   lse      [B, Hq] fp32 device, out (natural log).
 * Reads each kept key and value row once (split over chunks of 128 kept keys,
 * the query heads of a kv-head group together, then a merge of the chunks).
 * Asynchronous on `stream`; validation as sattn_fwd. */
int sattn_decode_fwd(const sattn_params* p, const void* Q, const void* K, const void* V, const uint8_t* is_sep,
                     void* O, float* lse, void* ws, size_t ws_bytes, void* stream);

/* sattn_decode_fwd that also returns the top-k selection of the decoding
 * query ("LM-Infinite", section 方法, optional top-k, applied at generation):
 * per query head the p->topk candidates n_start <= j < i-w (i = T-1) that are
 * not separators with the largest unscaled logit z_ij (the capped one past
 * L_pretrain), ties to the smaller j, computed in fp32 from the raw inputs;
 * they join the step's key set with those logits.
 *   topk_idx    [B, Hq, topk] int32 device, out, or NULL: positions sorted by
 *               (z desc, j asc); -1 when fewer than topk candidates exist.
 *   topk_logit  [B, Hq, topk] float device, out, or NULL: z; -inf padding.
 * Every candidate key row is read once per kv-head group (a logit pass over
 * the middle of the cache), then a block per (batch, head) selects and adds
 * the selected keys' partial to the chunk merge.  SATTN_ERR_UNSUPPORTED with
 * ALiBi unless L_pretrain > 0 and window >= L_pretrain.  Other arguments as
 * sattn_decode_fwd. */
int sattn_decode_topk_fwd(const sattn_params* p, const void* Q, const void* K, const void* V, const uint8_t* is_sep,
                          void* O, float* lse, int32_t* topk_idx, float* topk_logit, void* ws, size_t ws_bytes,
                          void* stream);

/* Bytes of workspace needed by sattn_bwd for *p. */
int sattn_bwd_workspace_size(const sattn_params* p, size_t* bytes);

/* Backward pass of sattn_fwd ("SepLLM", section 6.2: training runs the
 * forward and the backward pass through the masked product): the gradients
 * of sum(dO * O) with respect to Q, K and V for the same parameters, key
 * sets and logits as the forward.  With P_ij = exp(s_ij - LSE_i) and
 * dz_ij = P_ij (dO_i.v_j - dO_i.O_i) / sqrt(d):
 *   dV_j = sum_i P_ij dO_i;
 *   an uncapped pair (z = <R(i)q_i, R(j)k_j>) adds R(i)^T dz R(j)k_j to dq_i
 *   and R(j)^T dz R(i)q_i to dk_j; a capped pair (L_pretrain > 0, i-j > L;
 *   z = <R(L)q_i, k_j>, "LM-Infinite", section 方法) adds R(L)^T dz k_j to
 *   dq_i and dz R(L)q_i to dk_j.
 *   p          as for sattn_fwd (same validation).
 *   Q, K, V    the forward's inputs, strides q/k/v_stride.
 *   is_sep     [B, T] uint8 device flags or NULL, as for the forward.
 *   topk_idx   [B, Hq, T, topk] int32 device: the forward's top-k selection
 *              (required when topk > 0; the selection is a constant here).
 *   O, lse     the forward's outputs (O strides o_stride; lse [B, Hq, T]).
 *   dO         gradient of the loss w.r.t. O, strides o_stride.
 *   dQ, dK, dV out, shaped and strided like Q, K, V (dtype of the inputs).
 * fp32: CUDA cores, one kernel writes dq per query row, another dk and dv
 * per key.  bf16: tensor cores (a dq kernel per 128-row query tile, a dk/dv
 * kernel per 128-key tile of positions or of compacted separators, both
 * recomputing P from lse), the sink and top-k keys on CUDA cores (the top-k
 * key side through each key's list of selecting rows, summed in ascending
 * (head, row) order), fp32 partial sums combined in a fixed order.  bf16
 * with topk > 0 needs B * Hq * T * topk < 2^31 (else SATTN_ERR_UNSUPPORTED).
 * Deterministic (no floating-point atomics).  Asynchronous on `stream`. */
int sattn_bwd(const sattn_params* p, const void* Q, const void* K, const void* V, const uint8_t* is_sep,
              const int32_t* topk_idx, const void* O, const float* lse, const void* dO, void* dQ, void* dK,
              void* dV, void* ws, size_t ws_bytes, void* stream);

/* Bytes of workspace needed by sattn_tree_cross_fwd. */
int sattn_tree_cross_workspace_size(const sattn_params* p, int32_t n_chunks, int32_t chunk_len, int32_t depth,
                                    int32_t alpha_leaf, size_t* bytes);

/* SharedLLM's position-aware tree cross-attention ("SharedLLM", sections
 * 关键设计 2 and 4) with the language-modelling policy (the right child of a
 * context-tree node is always the one expanded):
 *   - the context is n_chunks chunks of chunk_len tokens; in each chunk,
 *     levels w = 1..depth keep the left child of the node being expanded and
 *     level `depth` also its right child (depth 0 keeps the whole chunk);
 *     a node of length m splits at floor(m/2);
 *   - a kept node of length m at level w keeps max(1, floor(m / a_w)) rows
 *     at offsets floor(k m / m'), a_w = alpha_leaf * 2^(depth - w);
 *   - the kept rows of chunk c take rotary position c, every query
 *     position n_chunks; O = softmax(Q K'^T / sqrt(d)) V' over all kept
 *     rows of all chunks (no mask).
 *   p          B, Hq, Hkv, d, rope_theta, rope_pos_scale; T = query rows;
 *              bf16 only; topk, L_pretrain, alibi, with_separators must be 0.
 *   Q          [B, Hq, T, d] bf16 device, strides q_stride.
 *   K, V       [B, Hkv, n_chunks * chunk_len, d] bf16 device (the context's
 *              keys, unrotated, and values), strides k_stride / v_stride.
 *   O, lse     [B, Hq, T, d] bf16 (strides o_stride), [B, Hq, T] fp32, out.
 *   kept_index [n_kept] int32 device, out, or NULL: the kept offsets within
 *              a chunk, in order (n_kept from the workspace query's rules).
 * Limits: 1 <= alpha_leaf <= 1024, 0 <= depth <= 20, else
 * SATTN_ERR_INVALID_ARG.  Asynchronous on `stream`. */
int sattn_tree_cross_fwd(const sattn_params* p, int32_t n_chunks, int32_t chunk_len, int32_t depth,
                         int32_t alpha_leaf, const void* Q, const void* K, const void* V, void* O, float* lse,
                         int32_t* kept_index, void* ws, size_t ws_bytes, void* stream);

/* ---- SepLLM streaming KV cache ("SepLLM", section 6.2) ----
 * Per sequence: an Initial cache (a slots, the first a tokens), a Separator
 * cache (s slots), a Local window (w slots, the newest tokens) and a Past
 * window that takes what leaves the Local window.  After each append, if the
 * running size reaches c, Past's separators move (in order) behind the
 * cached separators, the oldest separators go if more than s would stay,
 * and the rest of Past is dropped.  Slots are ordered Initial | Separator |
 * Past | Local (newest last); a decoding step attends over every slot with
 * rolled positions: key x at rotary position x, the query at the last slot
 * (the talk page, section "Streaming ARMS").  The state lives in caller-owned
 * device memory; every decision is taken on the device (no host round trip,
 * so the calls can be captured in a CUDA graph). */
typedef struct sattn_stream_config {
  int32_t B, Hkv, d; /* sequences, kv heads, head dim (64 or 128) */
  int32_t a, s, w;   /* Initial, Separator, Local window slots (w >= 1) */
  int32_t c;         /* capacity; a + s + w < c (SATTN_ERR_INVALID_ARG otherwise) */
} sattn_stream_config;

/* Bytes of device state for cfg (256-byte aligned buffer). */
int sattn_stream_state_size(const sattn_stream_config* cfg, size_t* bytes);
/* Empties every sequence's cache. */
int sattn_stream_reset(const sattn_stream_config* cfg, void* state, size_t state_bytes, void* stream);
/* Appends one token per sequence: K_new, V_new [B, Hkv, d] bf16 contiguous
 * device (keys unrotated), is_sep [B] uint8 device or NULL (no separator),
 * position = the token's index in the stream (recorded per slot). */
int sattn_stream_append(const sattn_stream_config* cfg, void* state, size_t state_bytes, const void* K_new,
                        const void* V_new, const uint8_t* is_sep, int64_t position, void* stream);
/* Synchronises `stream`, then copies the region sizes [B, 4] (Initial,
 * Separator, Past, Local) and, if positions != NULL, the stream index of
 * every slot [B, c] to host memory. */
int sattn_stream_read(const sattn_stream_config* cfg, const void* state, size_t state_bytes, int32_t* sizes,
                      int32_t* positions, void* stream);
/* Workspace for sattn_stream_decode: p gives Hq (Hq / Hkv in 1, 2, 4, 8),
 * rope_theta, rope_pos_scale and the q / o strides; B, Hkv, d equal cfg's. */
int sattn_stream_decode_workspace_size(const sattn_stream_config* cfg, const sattn_params* p, size_t* bytes);
/* One decoding step per sequence over its cache (after the token's append):
 * Q [B, Hq, 1, d] bf16 device, O [B, Hq, 1, d] bf16 out, lse [B, Hq] fp32 out. */
int sattn_stream_decode(const sattn_stream_config* cfg, const sattn_params* p, const void* state, size_t state_bytes,
                        const void* Q, void* O, float* lse, void* ws, size_t ws_bytes, void* stream);

/* Synchronises `stream` and reads the device status word of `ws` into
 * *device_status (SATTN_OK or SATTN_ERR_TIMEOUT).  Returns SATTN_ERR_CUDA if
 * the synchronisation itself failed (the CUDA error is then sticky). */
int sattn_stream_status(void* stream, const void* ws, int32_t* device_status);

/* Block map without a workspace (no counterpart on the pages: it exists for
 * callers that may not allocate device memory or hand over a workspace, e.g.
 * an extension running inside a host framework that owns all device memory,
 * or a latency-critical loop where an allocation -- which can synchronise
 * the device -- is not allowed).  Same arguments and outputs as
 * sattn_build_blockmap minus ws/ws_bytes; the scratch (a prefix count of
 * the separator flags and tile-class tables) lives in a fixed 4 MiB device
 * array that every GPU loading the library keeps until exit.
 *  - The scratch takes 8 * B * (floor(T / 32) + 1) bytes rounded up to 16,
 *    plus B * S_f + B * S_m with S_f = nQT rounded up to 16 and
 *    S_m = 16 * nQT * min(ceil(nQT / 16), floor(bt / 16) + 2), where
 *    nQT = ceil(T / 128) and bt = min(nQT, ceil(window / 128)).  Above
 *    4194304 bytes the call returns SATTN_ERR_UNSUPPORTED (nothing
 *    launched).
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - Allocates nothing: no cudaMalloc/cudaFree, no allocating library call.
 *  - All calls share the array, which keeps the last call's contents (no part
 *    of it needs to start at zero).  Calls that overlap on the GPU -- other
 *    streams, other host threads -- race on it: serialise them.
 *  - The looked-up address is kept for the life of the process; a
 *    cudaDeviceReset destroys the array with its context, so do not call
 *    this entry point again after resetting the device. */
int sattn_build_blockmap_noalloc(const sattn_params* p, const uint8_t* is_sep, uint8_t* cls, int32_t* sep_pos,
                                 int32_t* sep_count, int32_t* qtile_sep_range, void* stream);

/* Failure-path self-test (no counterpart on the pages).  Launches, on
 * `stream`, one small kernel that waits -- through the same bounded mbarrier
 * wait every kernel of the library uses -- on a barrier nothing arrives at.
 * After limit_ns nanoseconds (1 <= limit_ns <= 2e9) the wait gives up: the
 * kernel writes SATTN_ERR_TIMEOUT to the status word of `ws` (status[0]) and
 * the waiting site (99) to status[1], and returns normally, so the CUDA
 * context stays usable.  Read the result with sattn_stream_status.  The
 * status word is cleared first.  ws: device workspace of at least 256 bytes,
 * 256-byte aligned.  Returns SATTN_ERR_INVALID_ARG (nothing launched) for a
 * bad workspace or limit, SATTN_ERR_CUDA if the launch failed. */
int sattn_selftest_wait_timeout(void* ws, size_t ws_bytes, uint64_t limit_ns, void* stream);

/* Instrumentation (no counterpart on the pages).  While enabled, every kernel
 * launch group of the library is bracketed by CUDA events recorded on the
 * launch stream; the events cost a few hundred nanoseconds of device time
 * each.  sattn_profile_collect synchronises those events and reports, per
 * kernel group, the number of kernel launches and the summed device time
 * (milliseconds) since the previous collect, then resets the record.
 *   names     [max_groups][32] chars, out (NUL-terminated group names)
 *   launches  [max_groups] int32, out: kernels launched by the group
 *   total_ms  [max_groups] double, out
 *   n_groups  out: number of groups written
 * Host pointers.  Not thread-safe against concurrent entry-point calls. */
int sattn_profile_enable(int on);
int sattn_profile_collect(char* names, int32_t* launches, double* total_ms, int32_t max_groups,
                          int32_t* n_groups);

#ifdef __cplusplus
}
#endif

#endif /* SATTN_H_ */
