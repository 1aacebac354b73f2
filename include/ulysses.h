/*
 * ulysses.h -- C ABI of the single-GPU Ulysses attention layer (sm_100a).
 *
 * The method (Ulysses sequence parallelism):
 *   "Paralelismul de Secvență Ulysses: Antrenarea modelelor AI cu contexte de
 *    un milion de token-uri", section "Mecanismul de funcționare Ulysses",
 *    steps 1-6, and "Ulysses 序列平行化：突破百萬標記長上下文的訓練瓶頸",
 *    section "Ulysses 序列平行化的原理": the sequence is split over P ranks
 *   (rank r holds positions [r*n/P, (r+1)*n/P)); a first all-to-all gives
 *   every rank all n positions of H/P heads; each rank runs ordinary attention
 *   on its heads; a second all-to-all restores the sequence split.  The loss
 *   is aggregated over ranks weighted by each rank's count of valid tokens
 *   (same page, section "Integrarea cu Accelerate").
 *
 * Here the P ranks are logical: all of them live in one GPU's memory and the
 * two all-to-alls are layout permutations inside HBM.
 *
 * Layouts (row = head_dim contiguous elements):
 *   seq layout   X[P][B][n/P][heads][head_dim]   (rank-major stack of the
 *                per-rank [B][n/P][heads][d] buffers; for B = 1 this is the
 *                natural [n][heads][d] order)
 *   head layout  X[P][B][heads/P][n][head_dim]   (rank r holds heads
 *                [r*heads/P, (r+1)*heads/P) for all n positions)
 *   LSE          float[P][B][H/P][n] (natural log of the softmax denominator)
 * GQA: query head q uses KV head floor(q / (H/G)); rank r holds query heads
 * [r*H/P, (r+1)*H/P) and KV heads [r*G/P, (r+1)*G/P), so every rank's query
 * heads find their KV heads locally (needs H % P == G % P == H % G == 0).
 *
 * Conventions for every entry point:
 *  - All data pointers are DEVICE pointers owned by the caller; the library
 *    never allocates or frees device memory.  `stream` is a cudaStream_t (or
 *    NULL for the legacy default stream) passed as void*.
 *  - Every call is asynchronous on `stream`; nothing synchronises the host.
 *  - Errors detectable from the arguments are returned before any launch and
 *    then nothing is launched.  Data-dependent errors (a bad label, a bounded
 *    wait that ran out) are OR-ed as (1 << status) into a device error word,
 *    read with ulysses_read_error(); kernels never trap.
 *  - Pointers must be 16-byte aligned and rows (head_dim * element bytes) a
 *    multiple of 16 bytes.  Inputs and outputs must not overlap.
 */
#ifndef ULYSSES_H
#define ULYSSES_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ULY_OK = 0,
  ULY_ERR_NULL = 1,        /* a required pointer is NULL                          */
  ULY_ERR_SHAPE = 2,       /* n % P, H % P, G % P, H % G, non-positive sizes     */
  ULY_ERR_DTYPE = 3,       /* unknown dtype / element size                        */
  ULY_ERR_ALIGN = 4,       /* pointer or row not 16-byte aligned                  */
  ULY_ERR_ALIAS = 5,       /* input and output ranges overlap                     */
  ULY_ERR_UNSUPPORTED = 6, /* valid but not implemented (e.g. bf16 head_dim!=128)*/
  ULY_ERR_CUDA = 7,        /* a CUDA runtime call failed                          */
  ULY_ERR_LABEL = 8,       /* async: a label outside [0, V) and != ignore_index   */
  ULY_ERR_TIMEOUT = 9,     /* async: a bounded wait inside a kernel ran out       */
  ULY_ERR_WORKSPACE = 10   /* workspace missing or smaller than required          */
} uly_status;

typedef enum { ULY_F32 = 0, ULY_BF16 = 1 } uly_dtype;

typedef enum {
  ULY_MASK_NONE = 0,       /* every key visible                                   */
  ULY_MASK_CAUSAL = 1,     /* key j visible to query i iff j <= i                 */
  ULY_MASK_DOC_CAUSAL = 2  /* causal and same document (packed sequences)         */
} uly_mask;

/* Shape of one Ulysses attention layer (all P logical ranks at once). */
typedef struct {
  int32_t batch;           /* B                                                   */
  int32_t seq_len;         /* n (global, all ranks); n % world == 0               */
  int32_t world;           /* P logical ranks                                     */
  int32_t n_q_heads;       /* H                                                   */
  int32_t n_kv_heads;      /* G (GQA); H % G == 0                                 */
  int32_t head_dim;        /* d: f32 supports 64 and 128, bf16 supports 128       */
  int32_t dtype;           /* uly_dtype of q, k, v, o, dout, dq, dk, dv           */
  int32_t mask;            /* uly_mask                                            */
  const int32_t *cu_seqlens; /* DEVICE int32[num_docs+1], doc-causal only: document
                              * e covers positions [cu[e], cu[e+1]); cu[0] = 0 and
                              * cu[num_docs] = n; shared by all batch rows        */
  int32_t num_docs;
  float softmax_scale;     /* 0 => 1/sqrt(head_dim)                               */
  int32_t out_seq_layout;  /* 0: everything in the head layout.  1: the second
                            * all-to-all (step 5) is done by the producing kernel:
                            * o (fwd) and dq, dk, dv (bwd) are written straight into
                            * the seq layout [P][B][n/P][heads][d], and the bwd
                            * reads o in that layout too (as the fwd wrote it).
                            * q, k, v, dout and lse stay in the head layout.      */
  int32_t deterministic;   /* bf16 backward only.  0: one fused pass over the
                            * (key tile, query tile) pairs; dQ is summed with fp32
                            * adds in L2 and is not bitwise repeatable (dK, dV are).
                            * 1: two passes, no atomics, bitwise repeatable (the dQ
                            * pass recomputes the scores).  Needs a smaller
                            * workspace.  Ignored by the f32 path (repeatable).   */
} uly_attn_desc;

/*
 * First all-to-all (step 3): seq layout -> head layout.
 * src: [P][B][n/P][heads][head_dim], dst: [P][B][heads/P][n][head_dim]; the
 * element type is opaque (elem_bytes in {1,2,4,8}); the copy is bit-exact.
 * Requires n % P == 0, heads % P == 0, head_dim * elem_bytes % 16 == 0.
 */
uly_status ulysses_seq_to_head(int32_t batch, int32_t seq_len, int32_t world, int32_t heads,
                               int32_t head_dim, int32_t elem_bytes, const void *src,
                               void *dst, void *stream);

/* One tensor of a batched all-to-all (the source and destination of one
 * permutation and its number of heads). */
typedef struct {
  const void *src;
  void *dst;
  int32_t heads;
} uly_permute_item;

/*
 * The first (seq -> head) or second (head -> seq) all-to-all of `count`
 * tensors at once (1 <= count <= 4, e.g. Q, K and V), all with the same
 * batch, seq_len, world, head_dim and elem_bytes and each with its own number
 * of heads; `items` is a HOST array the call reads before it returns.  Every
 * tensor follows the rules of ulysses_seq_to_head; no destination may overlap
 * any source or destination of the call.  Bit-exact copies, one launch when
 * the shapes allow (up to 256 heads per tensor, rows of at most 1 KB).
 */
uly_status ulysses_seq_to_head_batch(int32_t batch, int32_t seq_len, int32_t world, int32_t head_dim,
                                     int32_t elem_bytes, int32_t count, const uly_permute_item *items,
                                     void *stream);
uly_status ulysses_head_to_seq_batch(int32_t batch, int32_t seq_len, int32_t world, int32_t head_dim,
                                     int32_t elem_bytes, int32_t count, const uly_permute_item *items,
                                     void *stream);

/* Second all-to-all (step 5): head layout -> seq layout; exact inverse of
 * ulysses_seq_to_head, same arguments and rules. */
uly_status ulysses_head_to_seq(int32_t batch, int32_t seq_len, int32_t world, int32_t heads,
                               int32_t head_dim, int32_t elem_bytes, const void *src,
                               void *dst, void *stream);

/*
 * First all-to-all of K or V when there are fewer KV heads than ranks
 * (G < P; "Ulysses 序列平行化", section "與 Ring Attention 的比較": the method
 * needs at least as many heads as ranks, and grouped KV heads fall short of it).
 * Rank r uses KV head floor(r*G/P) for all of its query heads, so that head is
 * copied whole to each of its P/G ranks:
 *   src: seq layout [P][B][n/P][G][head_dim]
 *   dst: [P][B][1][n][head_dim], dst[r][b][0][t] = src[t/s][b][t%s][r*G/P]
 * After it, ulysses_attn_fwd / _bwd run with n_kv_heads = P (one KV head per
 * rank); their results equal plain GQA attention with G KV heads.  The element
 * type is opaque (elem_bytes in {1,2,4,8}); the copy is bit-exact.  Requires
 * n % P == 0, P % G == 0, head_dim * elem_bytes % 16 == 0 and a power-of-two
 * number (<= 64) of 16-byte vectors per row.  dst must not overlap src.
 */
uly_status ulysses_kv_seq_to_head_replicated(int32_t batch, int32_t seq_len, int32_t world,
                                             int32_t kv_heads, int32_t head_dim,
                                             int32_t elem_bytes, const void *src, void *dst,
                                             void *stream);

/*
 * Reverse of ulysses_kv_seq_to_head_replicated for gradients: the gradient of
 * a KV head is the sum of the gradients its P/G copies received,
 *   dst[r][b][tt][k] = sum_{j < P/G} src[k*P/G + j][b][0][r*s + tt],
 * accumulated in fp32 in rank order and rounded once (RNE) to `dtype`
 * (ULY_BF16 or ULY_F32).  src [P][B][1][n][d], dst seq layout [P][B][n/P][G][d].
 * Same shape and alignment rules; dst must not overlap src.
 */
uly_status ulysses_kv_head_to_seq_reduce(int32_t batch, int32_t seq_len, int32_t world,
                                         int32_t kv_heads, int32_t head_dim, int32_t dtype,
                                         const void *src, void *dst, void *stream);

/*
 * Next-token labels, shifted on the whole sequence BEFORE it is sharded (the
 * last position of shard r needs the first token of shard r+1; the SFT
 * trainer's automatic label shift, "Ulysses 序列平行化", section
 * "在 Hugging Face 生態系統中的整合"; padding and packed sequences,
 * "Paralelismul de Secvență Ulysses", section "Integrarea cu Transformers
 * Trainer și TRL SFTTrainer"):
 *   labels[r][b][tt] (t = r*n/P + tt) = input_ids[b][t+1]  if t+1 < valid_len and
 *                                       t+1 is not a document start,
 *                                     = ignore_index       otherwise.
 * input_ids: DEVICE int32 [B][n] in sequence order.  labels: DEVICE int32
 * [P][B][n/P] (the layout ulysses_loss_aggregate reads as [P][tokens/P]).
 * cu_seqlens: NULL (num_docs = 0) for one document per row, else DEVICE int32
 * [num_docs+1] as in uly_attn_desc (cu[0] = 0, nondecreasing, cu[num_docs] = n;
 * another array gives unspecified but in-bounds labels); document starts are
 * cu[1..num_docs-1].  valid_len in [0, n]: positions >= valid_len are padding
 * (padding to a multiple of P), and the token before them gets ignore_index.
 * labels must not overlap input_ids or cu_seqlens.
 */
uly_status ulysses_shift_labels(int32_t batch, int32_t seq_len, int32_t world,
                                const int32_t *input_ids, const int32_t *cu_seqlens,
                                int32_t num_docs, int32_t valid_len, int32_t ignore_index,
                                int32_t *labels, void *stream);

/*
 * Rotary position table for ulysses_qkv_proj_rope: for every position
 * p < max_pos and pair e < head_dim/2, table[p][e] = (cos, sin) of the angle
 * p * base^(-2e/head_dim), computed in double precision and rounded once to
 * float.  table: DEVICE float [max_pos][head_dim/2][2], 16-byte aligned.
 * base > 1 (Qwen3 uses 1e6).  Positions are those of the WHOLE sequence.
 */
uly_status ulysses_rope_table(int32_t max_pos, int32_t head_dim, double base, float *table,
                              void *stream);

/*
 * Steps 2-3 ("Paralelismul de Secvență Ulysses", section "Mecanismul de
 * funcționare Ulysses"): every rank projects its own tokens,
 *   [Q K V](t) = x(t) W_qkv^T,
 * rotates Q and K by the token's position in the whole sequence (rank r's
 * local token tt is at t = r*n/P + tt; the ms-swift page, section 6.2, names a
 * rotation that ignores the shard's offset as the cause of repeated tokens),
 * and writes the results directly in the head layout (the first all-to-all
 * happens in the same kernel).  bf16 in and out, fp32 accumulation, one
 * rounding.  Rotation: rotate-half pairing, element e with e + head_dim/2:
 *   y[e] = x[e] cos - x[e+d/2] sin,  y[e+d/2] = x[e+d/2] cos + x[e] sin,
 * cos/sin from `rope_table` (ulysses_rope_table) at the token's position.
 *   x:      DEVICE bf16 seq layout [P][B][n/P][hidden]
 *   w_qkv:  DEVICE bf16 [(H + 2G) * head_dim][hidden] (nn.Linear weight: H query
 *           heads, then G key heads, then G value heads, head_dim rows each)
 *   positions: NULL (position = t, needs max_pos >= n) or DEVICE int32 [B][n]
 *           in sequence order (e.g. restarting at every packed document); a
 *           position outside [0, max_pos) sets ULY_ERR_SHAPE in the error word
 *           and that row is rotated as position 0
 *   q:      DEVICE bf16 [P][B][H/P][n][head_dim];  k, v: [P][B][G/P][n][head_dim]
 * Needs n % P == H % P == G % P == H % G == 0, head_dim == 128, H + 2G even,
 * hidden % 64 == 0 (else ULY_ERR_SHAPE / ULY_ERR_UNSUPPORTED; with fewer KV
 * heads than ranks, project K/V in the seq layout and use
 * ulysses_kv_seq_to_head_replicated).  Outputs must not overlap any input or
 * each other.
 */
uly_status ulysses_qkv_proj_rope(int32_t batch, int32_t seq_len, int32_t world, int32_t hidden,
                                 int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                 const void *x, const void *w_qkv, const float *rope_table,
                                 int32_t max_pos, const int32_t *positions, void *q, void *k,
                                 void *v, void *stream);

/*
 * Steps 5-6: the second all-to-all and the output projection in one kernel:
 * the attention output is read in the head layout and every rank's tokens
 * are projected,  y(t) = [O_0(t) ... O_{H-1}(t)] W_o^T.
 *   o:   DEVICE bf16 [P][B][H/P][n][head_dim]
 *   w_o: DEVICE bf16 [hidden][H * head_dim]
 *   y:   DEVICE bf16 seq layout [P][B][n/P][hidden]
 * bf16 in and out, fp32 accumulation, one rounding.  Needs n % P == H % P == 0,
 * head_dim == 128, hidden % 256 == 0.  y must not overlap o or w_o.
 */
uly_status ulysses_o_proj(int32_t batch, int32_t seq_len, int32_t world, int32_t hidden,
                          int32_t n_q_heads, int32_t head_dim, const void *o, const void *w_o,
                          void *y, void *stream);

/* Bytes of device workspace ulysses_qkv_proj_rope_bwd needs: the projection's
 * output gradient dY, bf16 [B*n][(H + 2G) * head_dim]. */
uly_status ulysses_qkv_proj_rope_bwd_workspace_size(int32_t batch, int32_t seq_len, int32_t n_q_heads,
                                                   int32_t n_kv_heads, int32_t head_dim, size_t *bytes);

/*
 * Backward of steps 2-3 (the adjoint of ulysses_qkv_proj_rope):
 *   dY(t) = [R(-pos) dQ(t) | R(-pos) dK(t) | dV(t)]   (the gradients back
 *           through the folded all-to-all and through the rotation, whose
 *           transpose is the rotation by -pos), written to `workspace`;
 *   dX = dY W_qkv          (bf16, seq layout [P][B][n/P][hidden]);
 *   dW = sum over all tokens of dY^T X   (fp32 [(H+2G)*head_dim][hidden]).
 * dq [P][B][H/P][n][d], dk, dv [P][B][G/P][n][d] (bf16 head layout); x, w_qkv,
 * rope_table, max_pos, positions as for the forward.  Needs G % P == 0 (with
 * fewer KV heads than ranks, sum the copies' gradients first), head_dim ==
 * 128, H + 2G even, hidden % 256 == 0.  Tensor-core GEMMs with fp32
 * accumulation; the pre-pass is HBM-bound.  Outputs must not overlap inputs.
 */
uly_status ulysses_qkv_proj_rope_bwd(int32_t batch, int32_t seq_len, int32_t world, int32_t hidden,
                                     int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, const void *x,
                                     const void *w_qkv, const float *rope_table, int32_t max_pos,
                                     const int32_t *positions, const void *dq, const void *dk, const void *dv,
                                     void *dx, float *dw, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Backward of steps 5-6 (the adjoint of ulysses_o_proj):
 *   dO = dY W_o   written straight into the head layout [P][B][H/P][n][d]
 *                 (bf16; the first all-to-all in the GEMM's epilogue);
 *   dW_o = sum over all tokens of dY^T O   (fp32 [hidden][H * head_dim]).
 * o_seq: the attention output in the seq layout [P][B][n/P][H][d] (as
 * ulysses_attn_fwd writes it with out_seq_layout = 1); w_o [hidden][H*d];
 * dy: the layer output's gradient, seq layout [P][B][n/P][hidden] (bf16).
 * Needs head_dim == 128, H even, hidden % 256 == 0.
 */
uly_status ulysses_o_proj_bwd(int32_t batch, int32_t seq_len, int32_t world, int32_t hidden, int32_t n_q_heads,
                              int32_t head_dim, const void *o_seq, const void *w_o, const void *dy, void *do_head,
                              float *dw_o, void *stream);

/*
 * Local attention (step 4) of every logical rank, head layout in and out:
 * q, o [P][B][H/P][n][d]; k, v [P][B][G/P][n][d]; lse [P][B][H/P][n] (fp32).
 * O = softmax(scale * Q K^T + mask) V per query head, LSE its log-sum-exp.
 * bf16: tensor-core path (fp32 accumulation), needs head_dim == 128; any
 * group size H/G (an odd one, MHA included, runs one query head per CTA of the
 * forward instead of two, at about half its rate).  f32: exact-fp32 SIMT path.
 */
uly_status ulysses_attn_fwd(const uly_attn_desc *desc, const void *q, const void *k,
                            const void *v, void *o, float *lse, void *stream);

/* Bytes of device workspace ulysses_attn_bwd needs for this shape. */
uly_status ulysses_attn_bwd_workspace_size(const uly_attn_desc *desc, size_t *bytes);

/*
 * Backward of the local attention (gradients of sum(O * dO)), head layout:
 * dout, dq like q; dk, dv like k (summed over the query heads of each KV
 * head); o and lse are the forward's outputs.  With desc->out_seq_layout = 1,
 * dq, dk, dv are written in the seq layout instead.  `workspace` must hold
 * ulysses_attn_bwd_workspace_size() bytes (caller owned, 256-byte aligned,
 * contents need not be initialised): per query row D_i = <dO_i, O_i> and
 * LSE_i log2(e), and, for the fused bf16 backward (deterministic = 0), an fp32
 * dQ accumulator of 512 bytes per query row (n rounded up to 128 per head).
 * A malformed cu_seqlens (not starting at 0, decreasing, or not ending at n)
 * sets ULY_ERR_SHAPE in the error word (fwd and bwd); its kernels stay inside
 * their operands.
 */
uly_status ulysses_attn_bwd(const uly_attn_desc *desc, const void *q, const void *k,
                            const void *v, const void *o, const float *lse, const void *dout,
                            void *dq, void *dk, void *dv, void *workspace,
                            size_t workspace_bytes, void *stream);

/* Bytes of device workspace ulysses_loss_aggregate needs. */
uly_status ulysses_loss_workspace_size(int32_t world, int64_t tokens, int32_t vocab,
                                       size_t *bytes);

/*
 * Token-weighted cross-entropy over the P shards ("Integrarea cu Accelerate":
 * weight every rank's loss by its count of valid tokens):
 *   l_t = logsumexp(z_t) - z_t[y_t] for every token with y_t != ignore_index,
 *   shard_sum[r] = sum of l_t over shard r, shard_count[r] = its valid count,
 *   *loss = sum_r shard_sum[r] / sum_r shard_count[r]  (NaN if no valid token).
 * logits: [P][tokens/P][vocab] (ULY_BF16 or ULY_F32), labels int32 [P][tokens/P].
 * Needs tokens % P == 0.  A label outside [0, vocab) that is not ignore_index
 * sets ULY_ERR_LABEL in the error word and is not counted.  The reduction order
 * is fixed, so repeated calls give bitwise-equal results.
 */
uly_status ulysses_loss_aggregate(int32_t world, int64_t tokens, int32_t vocab,
                                  int32_t logit_dtype, const void *logits,
                                  const int32_t *labels, int32_t ignore_index,
                                  float *shard_sum, int64_t *shard_count, float *loss,
                                  void *workspace, size_t workspace_bytes, void *stream);

/* Bytes of device workspace ulysses_loss_aggregate_bwd needs. */
uly_status ulysses_loss_bwd_workspace_size(int32_t world, int64_t tokens, int32_t vocab,
                                           size_t *bytes);

/*
 * The aggregated loss and its gradient in one pass over the logits (the
 * training step after the aggregation; "Integrarea cu Accelerate": every
 * shard's loss is weighted by its valid-token count, so the gradient of
 * L = sum_r S_r / sum_r C_r has the global count C = sum_r C_r as its only
 * denominator):
 *   dlogits[t][v] = (softmax(z_t)_v - [v == y_t]) / C  for counted tokens,
 *   dlogits[t][v] = 0                                   for ignored or invalid ones.
 * shard_sum, shard_count and *loss as ulysses_loss_aggregate (bitwise the same
 * values).  dlogits: same shape and dtype as logits, written in full; it must
 * not overlap any other argument.  Logits are read once from HBM and dlogits
 * written once.  Errors as ulysses_loss_aggregate; with no counted token
 * every dlogits row is 0 and *loss is NaN.
 */
uly_status ulysses_loss_aggregate_bwd(int32_t world, int64_t tokens, int32_t vocab,
                                      int32_t logit_dtype, const void *logits,
                                      const int32_t *labels, int32_t ignore_index,
                                      void *dlogits, float *shard_sum, int64_t *shard_count,
                                      float *loss, void *workspace, size_t workspace_bytes,
                                      void *stream);

/* Size of the fixed scratch array behind ulysses_loss_aggregate_noalloc. */
#define ULYSSES_NOALLOC_LOSS_SCRATCH_BYTES 65536

/*
 * ulysses_loss_aggregate without a workspace argument, for callers that
 * cannot allocate device memory: hosts that pass the library only their input
 * and output buffers and own every allocation, or processes that allow no
 * device allocation after start-up.  The method's pages have no counterpart
 * of this call; it exists for those callers.
 * Same arguments, results and errors as ulysses_loss_aggregate, except:
 *  - the partial sums live in a fixed 64 KiB device array inside the library
 *    (held on every GPU that loads it until the process exits); shapes whose
 *    partials need more (more than 4096 of them: P * blocks per shard, about
 *    P > 3500 ranks) return ULY_ERR_WORKSPACE and launch nothing;
 *  - all calls share that array: calls that overlap on the GPU (unordered
 *    streams) race and give wrong results; nothing in it needs clearing
 *    between calls (every slot is written before it is read within a call);
 *  - the first call on a device looks up the array's address on that device,
 *    so make that first call before any stream capture.
 * It calls no cudaMalloc, cudaFree or other allocating routine.
 */
uly_status ulysses_loss_aggregate_noalloc(int32_t world, int64_t tokens, int32_t vocab,
                                          int32_t logit_dtype, const void *logits,
                                          const int32_t *labels, int32_t ignore_index,
                                          float *shard_sum, int64_t *shard_count, float *loss,
                                          void *stream);

/* Device address of the current device's asynchronous error word (int32;
 * bit s set <=> status s was raised by a kernel since it was last cleared),
 * for callers that poll it themselves (e.g. with their own stream-ordered
 * copy) instead of ulysses_read_error.  The word is owned by the library and
 * lives as long as the process's context on that device. */
uly_status ulysses_error_word(int32_t **dev_word);

/* Asynchronous error word of the current device: reads it (synchronising the
 * device) into *word (bit s set <=> status s was raised) and clears it. */
uly_status ulysses_read_error(int32_t *word);

/* Like ulysses_read_error, but copies up to n words of the error record:
 * info[0] = the error word; if a bounded wait ran out, info[1] = 1 and
 * info[2..8] = CTA x, CTA y, thread, shared-memory barrier address, phase
 * parity, cycles waited >> 20, and polls of the first wait that gave up.
 * The record is cleared. */
uly_status ulysses_read_error_info(int32_t *info, int32_t n);

/*
 * Failure detection (no counterpart on the pages: the tcgen05 kernels wait on
 * mbarriers, and every such wait is bounded).  Sets how many SM clock cycles a
 * pipeline wait of the attention and projection kernels launched from now on
 * may last before the kernel records ULY_ERR_TIMEOUT (and where, see
 * ulysses_read_error_info), drains its copies and MMAs, frees its tensor
 * memory and returns.  cycles = 0 restores the built-in limit (2e9 cycles,
 * about a second); a shorter limit also makes the waits poll without
 * suspending.  Meant for tests of that path: a limit of a few hundred cycles
 * makes the first wait for a tile copy run out.  Process-wide, host only.
 * Returns ULY_ERR_SHAPE for a negative value.
 */
uly_status ulysses_set_wait_limit(int64_t cycles);

/*
 * Block order of the attention kernels launched from now on (no counterpart
 * on the pages; a scheduling choice that leaves every result unchanged).
 * ULY_BLOCK_ORDER_AUTO (the default): the CTAs of one KV head start together
 * (heaviest tiles first) when a KV head has more than twice as many CTAs along
 * the sequence as the device has SMs and the mask is not a document mask, so
 * that the CTAs in flight share one GQA group's K/V (forward) or Q/dO and dQ
 * rows (backward) in L2; otherwise the heaviest tiles of every head start
 * first, which balances few waves best.  ULY_BLOCK_ORDER_KV_HEAD_MAJOR and
 * ULY_BLOCK_ORDER_HEAVIEST_FIRST fix one of the two, for tests that compare
 * them.  O, LSE, dK, dV and the deterministic backward's dQ are bitwise the
 * same under both; the fused backward's dQ varies at the fp32 rounding level
 * from run to run under either.  Process-wide, host only.  Returns
 * ULY_ERR_SHAPE for any other value.
 */
enum { ULY_BLOCK_ORDER_AUTO = 0, ULY_BLOCK_ORDER_KV_HEAD_MAJOR = 1, ULY_BLOCK_ORDER_HEAVIEST_FIRST = 2 };
uly_status ulysses_set_attn_block_order(int32_t order);

/* Human-readable name of a status. */
const char *ulysses_status_string(uly_status status);

/* Number of kernels launched by this process through the library so far. */
uint64_t ulysses_launch_count(void);

/* Per-kernel device timing.  ulysses_profile_enable(1) clears the totals and
 * makes every later launch record two CUDA events on its own stream (a few
 * microseconds of host time per launch); ulysses_profile_enable(0) stops.
 * ulysses_profile_read() waits for the recorded events and returns, for
 * kernel id `kernel` (0 <= kernel < ulysses_kernel_count()), the summed
 * device milliseconds and the number of timed launches. */
uly_status ulysses_profile_enable(int32_t on);
uly_status ulysses_profile_read(int32_t kernel, double *total_ms, int64_t *launches);
int32_t ulysses_kernel_count(void);
const char *ulysses_kernel_name(int32_t kernel);

#ifdef __cplusplus
}
#endif
#endif /* ULYSSES_H */
