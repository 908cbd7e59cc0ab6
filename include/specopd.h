/*
 * specopd.h -- C ABI of the SpecOPD branch-parallel target-scoring library
 * for NVIDIA B200 (sm_100a).
 *
 * The method: "SpecOPD: Branch-Parallel On-Policy Distillation for Speculative
 * Decoding".  Draft branches sampled at reference anchors are packed after a
 * shared reference trunk (Fig 2, step 3); one tree-masked attention pass scores
 * every packed row (Fig 3); the full-vocabulary overlap alpha and the E2E-TV
 * loss with its gradient complete the path (daiwk.github.io write-up of the
 * paper, section "Equations").
 *
 * Conventions for every entry point:
 *   - The caller owns every buffer.  Pointers named *_dev or documented as
 *     "device" are device memory of the current CUDA device; "host" pointers
 *     are ordinary host memory read during the call only.
 *   - The library allocates nothing and never synchronises: every kernel is
 *     enqueued on the given stream and the call returns at once.
 *   - A negative return value (specopd_status) means an argument error found
 *     on the host; nothing was enqueued.  SPECOPD_ERR_CUDA means a launch
 *     failed.
 *   - Errors that depend on device data (an anchor outside the reference,
 *     a non-finite teacher logit, a bounded wait that ran out) are OR-ed as
 *     SPECOPD_FLAG_* bits into the caller's device word `status`.  The word is
 *     never cleared by the library: zero it before the calls you want to check
 *     and read it after the stream has synchronised.
 *   - Tensors are row-major with the innermost dimension contiguous.
 *   - All entry points may be called from several host threads on different
 *     streams, but calls that share a workspace or a status word must be
 *     ordered on one stream.
 */
#ifndef SPECOPD_H_
#define SPECOPD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* cudaStream_t without pulling in the CUDA headers */
typedef struct CUstream_st* specopd_stream_t;

typedef enum {
  SPECOPD_OK = 0,
  SPECOPD_ERR_ARG = -1,        /* null pointer, bad count, bad tree description */
  SPECOPD_ERR_SHAPE = -2,      /* sizes out of the supported range */
  SPECOPD_ERR_DTYPE = -3,      /* dtype not supported for this entry point */
  SPECOPD_ERR_CUDA = -4,       /* a CUDA launch or driver call failed */
  SPECOPD_ERR_WORKSPACE = -5,  /* workspace missing, too small or misaligned */
  SPECOPD_ERR_ALIGN = -6       /* a pointer or leading dimension breaks 16-byte alignment */
} specopd_status;

/* bits OR-ed into the device status word */
#define SPECOPD_FLAG_ANCHOR 1u     /* an anchor lies outside [P, T-1]; it was clamped */
#define SPECOPD_FLAG_NONFINITE 2u  /* a teacher logit is NaN/inf, or a draft logit is +inf */
#define SPECOPD_FLAG_TIMEOUT 4u    /* a bounded in-kernel wait gave up; outputs are invalid */

typedef enum { SPECOPD_F32 = 0, SPECOPD_BF16 = 1 } specopd_dtype;

#define SPECOPD_MAX_TREES 512
#define SPECOPD_MAX_W 64
#define SPECOPD_TILE_ROWS 128

/*
 * A batch of proposal trees (Fig 2, step 3; Fig 3).
 *
 * Tree t has a trunk of trunk_len[t] tokens, the first prompt_len[t] of them
 * the prompt and the rest the reference response, and num_branches[t]
 * branches of W drafted samples y_{b,1..W}.  Branch b hangs off trunk token
 * anchors[b] (zero-based within its tree, in [prompt_len, trunk_len-1]; the
 * write-up's section "Inputs and code mapping" fixes zero-based anchors).
 *
 * Packing: tree t occupies packed rows [cu_rows[t], cu_rows[t+1]): the trunk
 * first, then each branch's samples contiguously, branches in the order given.
 * With pack_terminal = 1 every sample has a row (W rows per branch); with 0
 * the terminal sample y_{b,W} gets none (W-1 rows per branch), since its
 * prediction reads its predecessor's row and nothing reads its own (Fig 3).
 *
 * trunk_len, prompt_len, num_branches: host arrays [num_trees].
 * anchors: DEVICE array [sum num_branches], tree-major.
 */
typedef struct {
  int32_t num_trees;       /* 1 .. SPECOPD_MAX_TREES */
  int32_t W;               /* 1 .. SPECOPD_MAX_W */
  int32_t pack_terminal;   /* 0 or 1 */
  const int32_t* trunk_len;
  const int32_t* prompt_len;
  const int32_t* num_branches;
  const int32_t* anchors;  /* device */
} specopd_tree_desc;

/*
 * Per query tile of up to SPECOPD_TILE_ROWS packed rows of one tree: the
 * column ranges the rows of the tile can see.  All values are global packed
 * indices.  Written by specopd_build_tree_mask, read by
 * specopd_tree_attention.
 */
typedef struct {
  int32_t row_start;   /* first row of the tile */
  int32_t row_end;     /* one past its last row (same tree) */
  int32_t tree_base;   /* first packed row of the tree */
  int32_t trunk_hi;    /* one past the last trunk column any row of the tile sees */
  int32_t trunk_full;  /* every row of the tile sees every trunk column < trunk_full */
  int32_t br_lo;       /* first branch column any row sees (br_lo == br_hi: none) */
  int32_t br_hi;       /* one past the last branch column any row sees */
  int32_t reserved;
} specopd_tile_meta;

/* Number of packed rows N of the batch, or a negative specopd_status. */
int64_t specopd_tree_packed_rows(const specopd_tree_desc* desc);
/* Number of query tiles (tiles never straddle two trees), or a negative status. */
int64_t specopd_tree_num_tiles(const specopd_tree_desc* desc);
/* Number of predictions sum_b W, or a negative status. */
int64_t specopd_tree_num_predictions(const specopd_tree_desc* desc);

/*
 * specopd_build_tree_mask -- tree packing and the compact tree mask.
 *
 * Fig 3 (each row sees itself and its ancestors; siblings are hidden), the
 * write-up's section "Equations" (history (x_{<=a_b}, y_{b,<i}); semantic
 * position a_b + i; the anchor row predicts the first sample and the row of
 * y_{b,i-1} predicts y_{b,i}).
 *
 * Outputs (device, written in full):
 *   pos[N]          semantic position: trunk token j -> j, y_{b,i} -> a_b + i
 *   trunk_limit[N]  largest tree-local trunk index the row sees: j on the trunk, a_b on a branch
 *   branch_of[N]    global branch index of the row, -1 on the trunk
 *   anc_bits[N]     bit k-1 set iff the row sees y_{b,k} of its own branch (0 on the trunk)
 *   pred_rows[P]    P = sum_b W; entry b*W + i-1 is the packed row whose query
 *                   predicts y_{b,i} (b-major over the whole batch)
 *   cu_rows[num_trees+1]
 *   tile_meta[num_tiles]
 * So row r sees column c iff c lies in r's tree and either c is a trunk
 * column with tree-local index <= trunk_limit[r], or c = row of y_{b,k} of
 * r's own branch with bit k-1 of anc_bits[r] set.
 *
 * An anchor outside [prompt_len, trunk_len-1] sets SPECOPD_FLAG_ANCHOR in
 * *status and is clamped into range so later kernels stay in bounds.
 */
int specopd_build_tree_mask(const specopd_tree_desc* desc, int32_t* pos, int32_t* trunk_limit,
                            int32_t* branch_of, uint64_t* anc_bits, int32_t* pred_rows,
                            int32_t* cu_rows, specopd_tile_meta* tile_meta, int32_t* status,
                            specopd_stream_t stream);

/*
 * specopd_rope -- rotate-half rotary embedding at semantic positions.
 *
 * The write-up's section "Equations": branch token y_{b,i} takes position
 * a_b + i, not its packed offset.  Element k of each head pairs with element
 * k + d/2 and both rotate by pos[r] * theta^(-2k/d); the angle is formed in
 * fp64.  q [N, Hq, d] -> q_out, k [N, Hkv, d] -> k_out (same dtype, may not
 * alias the inputs).  Hq or Hkv may be 0 (that tensor is skipped and its two
 * pointers may be null), so a caller can rotate a range of query rows and all
 * key rows with two calls.  d a multiple of 4 with 4 <= d <= 256 (the kernel
 * moves each half-head in 2-element pairs); other d return SPECOPD_ERR_SHAPE.
 */
int specopd_rope(const void* q, const void* k, void* q_out, void* k_out, specopd_dtype dtype, int64_t N,
                 int Hq, int Hkv, int d, const int32_t* pos, float theta, specopd_stream_t stream);

/* Bytes of workspace specopd_tree_attention needs (rotated Q and K). */
size_t specopd_attention_workspace_bytes(specopd_dtype dtype, int64_t N, int Hq, int Hkv, int d);

/*
 * specopd_tree_attention -- one tree-masked GQA attention pass over all packed rows.
 *
 * Fig 3: packed queries share trunk keys/values; every row attends to itself
 * and its ancestors only.  O[r, h] = sum_{c visible to r} softmax_c(q_r.k_c *
 * scale) v_c with q, k rotated at pos (specopd_rope), query head h reading
 * KV head h / (Hq / Hkv).
 *
 * q [N, Hq, d], k and v [N, Hkv, d], out [N, Hq, d]: device, dtype `dtype`,
 * 16-byte aligned.  rope_theta > 0 rotates q and k at pos first (into the
 * workspace); rope_theta <= 0 takes q and k as already rotated.
 * softmax_scale <= 0 means 1/sqrt(d).  pos, trunk_limit, anc_bits: outputs
 * of specopd_build_tree_mask for the same trees.  tile_meta: num_tiles of its
 * tile records, all of them or any contiguous run (tile_meta offset by the
 * run's first tile); only the rows of the given tiles are written to out, so
 * ranks that split a batch by query rows each pass their own run (q rows
 * outside the run are not read; every key row the run's rows see must be
 * present).  num_tiles == 0 does nothing.
 * bf16 with d = 128 runs the tcgen05/TMEM kernel; fp32 (any d) and bf16 with
 * other d (multiple of 32, <= 256) run a SIMT kernel with fp32 arithmetic.
 * Accumulation is fp32 in both.
 * workspace: device, >= specopd_attention_workspace_bytes, 256-byte aligned
 * (may be null when rope_theta <= 0).
 * status: device word; SPECOPD_FLAG_TIMEOUT if an in-kernel wait gave up.
 */
int specopd_tree_attention(const void* q, const void* k, const void* v, void* out, specopd_dtype dtype,
                           int64_t N, int Hq, int Hkv, int d, float rope_theta, float softmax_scale,
                           const int32_t* pos, const int32_t* trunk_limit, const uint64_t* anc_bits,
                           const specopd_tile_meta* tile_meta, int64_t num_tiles, void* workspace,
                           size_t workspace_bytes, int32_t* status, specopd_stream_t stream);

/* Bytes of workspace specopd_tv_overlap_e2e needs. */
size_t specopd_overlap_workspace_bytes(int64_t rows, int64_t V, int64_t num_branches);

/*
 * specopd_tv_overlap -- per-row full-vocabulary overlap, unfused.
 *
 * The write-up's section "Equations": alpha = sum_v min(q(v), p(v)) with q the
 * draft softmax and p the teacher softmax over the FULL vocabulary (teacher
 * mass outside the draft support is kept, never renormalised).  Section
 * "Inputs and code mapping": draft entries that are NaN or -inf are outside
 * the draft support; the teacher must be finite; bf16 work is promoted to fp32.
 *
 * draft [rows, ld_draft], teacher [rows, ld_teacher]: device, dtype `dtype`;
 * the first V entries of each row are used.  Rows must start on 16-byte
 * boundaries (base pointer and ld * element size).
 * alpha[rows] (fp32, device) is written; q_less[rows] = sum_v q_v [q_v < p_v],
 * lse_draft[rows], lse_teacher[rows] (natural-log normalisers) are written
 * when non-null.  A row with an empty draft support gets alpha = 0.
 * A non-finite teacher logit or a +inf draft logit sets SPECOPD_FLAG_NONFINITE.
 */
int specopd_tv_overlap(const void* draft, const void* teacher, specopd_dtype dtype, int64_t rows, int64_t V,
                       int64_t ld_draft, int64_t ld_teacher, float* alpha, float* q_less, float* lse_draft,
                       float* lse_teacher, int32_t* status, specopd_stream_t stream);

/*
 * specopd_e2e_tv_loss -- E2E-TV loss from per-prediction overlaps, unfused.
 *
 * The write-up's section "Equations": L = 1 - (1/count) sum_b sum_{j<=W}
 * prod_{i<=j} alpha_{b,i}.  alpha: device [num_branches * W], b-major.
 * count <= 0 means num_branches * W.  loss: device scalar.  grad_alpha
 * (nullable, device [num_branches * W]) receives dL/dalpha.  An empty batch
 * writes loss = 0.
 */
int specopd_e2e_tv_loss(const float* alpha, int64_t num_branches, int W, double count, float* loss,
                        float* grad_alpha, specopd_stream_t stream);

/*
 * specopd_tv_overlap_e2e -- fused overlap, E2E-TV loss and gradient.
 *
 * One pass computes alpha for every prediction row; the last row of each
 * branch to finish forms that branch's prefix products and dL/dalpha, and the
 * last branch forms L.  With grad_draft non-null a second streaming pass
 * writes dL/dz = dL/dalpha * q (1[q < p] - sum_v q_v 1[q_v < p_v]) (zero on
 * entries outside the draft support); samples and teacher are held fixed
 * (write-up, section "Equations").  For bf16 with a gradient, both passes run
 * in one cooperative launch with one CTA per SM (the gradient of a branch
 * starts on the SMs as soon as its dL/dalpha is final); if the device
 * refuses the cooperative launch the call returns SPECOPD_ERR_CUDA.
 *
 * Rows are predictions b-major: row b*W + i-1 holds the logits read out for
 * y_{b,i}.  rows must equal num_branches * W.  count <= 0 means rows.
 * grad_draft [rows, ld_grad] fp32 device (16-byte aligned rows).
 * workspace: device, >= specopd_overlap_workspace_bytes, 256-byte aligned.
 * alpha[rows] and loss (scalar) are device fp32 outputs.
 */
int specopd_tv_overlap_e2e(const void* draft, const void* teacher, specopd_dtype dtype, int64_t rows,
                           int64_t V, int64_t ld_draft, int64_t ld_teacher, int64_t num_branches, int W,
                           double count, float* alpha, float* loss, float* grad_draft, int64_t ld_grad,
                           void* workspace, size_t workspace_bytes, int32_t* status, specopd_stream_t stream);

/*
 * specopd_diag_overlap_wait_timeout -- failure-detection diagnostic: makes a
 * bounded in-kernel wait of the fused overlap kernel run out on purpose.
 *
 * Launches the bf16 kernel of specopd_tv_overlap_e2e (cooperative, one CTA per
 * SM) with the gradient of every row requested but no row's statistics, so
 * no branch's dL/dalpha is ever published: every gradient unit waits for a
 * publication that never comes.  The wait gives up after its time limit
 * (about one second), ORs SPECOPD_FLAG_TIMEOUT into *status, raises the CTA's
 * abort flag so its other waits stop, and the kernel returns; no copy is in
 * flight at that point and the stream stays usable.  grad_draft is left
 * unwritten.  Arguments as specopd_tv_overlap_e2e (bf16 only, grad_draft and
 * workspace required, num_branches >= 1).
 */
int specopd_diag_overlap_wait_timeout(const void* draft, const void* teacher, int64_t rows, int64_t V,
                                      int64_t ld_draft, int64_t ld_teacher, int64_t num_branches, int W,
                                      float* grad_draft, int64_t ld_grad, void* workspace, size_t workspace_bytes,
                                      int32_t* status, specopd_stream_t stream);

/*
 * specopd_tree_causal_conv -- short causal convolution along each packed row's
 * own history.
 *
 * SpecOPD (thelatestinai.com listing), Fig 5: the causal convolution of the
 * GDN branch path follows branch ancestry, so a branch token's window holds
 * its own history (the trunk through its anchor, then its branch's earlier
 * samples), never its packed neighbours or a sibling's tokens.  Reading (the
 * figure prints no formula): a depthwise convolution of width Kw,
 *   out[r, c] = act(bias[c] + sum_{j<Kw} weight[c, j] * x[h_j(r), c]),
 * h_j(r) the row j steps back in r's history (j = 0: r itself), zero before
 * the start of the history; act is the identity (silu = 0) or SiLU
 * u / (1 + e^-u) (silu = 1).  fp32 arithmetic.
 *
 * x, out [N, C]: device, dtype `dtype` (out in the same dtype), row-major,
 * 16-byte aligned, C a multiple of 8 (bf16) or 4 (fp32); a feature tensor
 * [N, H, d] is passed with C = H d.  weight [C, Kw] and bias [C] (nullable):
 * device fp32.  1 <= Kw <= 8.  pos, trunk_limit, cu_rows (num_trees + 1
 * entries): outputs of specopd_build_tree_mask for the same trees.  out may
 * not alias x.  Returns SPECOPD_ERR_* before anything is enqueued.
 */
int specopd_tree_causal_conv(const void* x, void* out, specopd_dtype dtype, int64_t N, int C, const float* weight,
                             const float* bias, int Kw, int silu, const int32_t* pos, const int32_t* trunk_limit,
                             const int32_t* cu_rows, int num_trees, specopd_stream_t stream);

/* Bytes of workspace specopd_gdn_tree needs: the fp32 trunk checkpoints,
 * (sum over trees of T / 64) * H * 128 * 128 * 4, then the chunked form's
 * record of every trunk chunk and head, (sum over trees of ceil(T / 64)) * H
 * * 20,612 * 4, each rounded up to 256 (0 for an invalid description). */
size_t specopd_gdn_workspace_bytes(const specopd_tree_desc* desc, int H);

/*
 * specopd_gdn_tree -- Gated DeltaNet linear attention over a proposal tree,
 * every packed row reading the recurrent state of its own history, with
 * indexed state replay.
 *
 * SpecOPD (thelatestinai.com listing), Fig 5: a shared trunk pass caches an
 * fp32 GDN state at every C = 64 boundary; each branch copies the checkpoint
 * at or before its anchor, replays the trunk features up to the anchor, then
 * updates the state over its own tokens and reads it with each token's query;
 * checkpoints stay immutable.  Reading (the pages print no formula): the
 * gated delta rule per head, state S in R^{dv x dk} starting at zero,
 *   S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *   o_t = S_t q_t.
 * A branch's history is the trunk through its anchor, then its own earlier
 * tokens (the packing of specopd_build_tree_mask for the same description).
 * The library computes the same outputs in the chunked form of the rule (64
 * tokens per chunk: a per-chunk triangular solve and products, the state
 * carried from chunk to chunk in fp32), with the products on the tensor cores
 * and fp32 operands split into bf16 pairs; a branch's state at its anchor is
 * formed from the checkpoint and that chunk's cached update vectors, and its
 * samples run as one chunk from there.
 *
 * q, k, v [N, H, 128] bf16 (dk = dv = 128; k normalised upstream), alpha,
 * beta [N, H] fp32, out [N, H, 128] fp32: device, row-major, 16-byte aligned.
 * The features are consumed as given (projections, short convolution and
 * normalisation happen upstream).  workspace: device, >=
 * specopd_gdn_workspace_bytes, 256-byte aligned; it holds the checkpoints
 * after the call.  Anchors outside [P, T-1] set SPECOPD_FLAG_ANCHOR and are
 * clamped.  Returns SPECOPD_ERR_SHAPE for dk or dv other than 128 or N not
 * the packed row count, SPECOPD_ERR_ARG / _ALIGN / _WORKSPACE before anything
 * is enqueued, SPECOPD_ERR_CUDA if a launch fails.
 */
int specopd_gdn_tree(const specopd_tree_desc* desc, const void* q, const void* k, const void* v,
                     const float* alpha, const float* beta, float* out, int64_t N, int H, int dk, int dv,
                     void* workspace, size_t workspace_bytes, int32_t* status, specopd_stream_t stream);

/* Bytes of workspace specopd_sparse_tree_attention needs: rotated Q and K
 * (bf16), the trunk group keys and the keys of the groups holding branch
 * tokens (fp32), the chosen groups [N][Hkv][topk] (int32) and the per-row
 * selection words (uint32), each rounded up to 256 bytes (0 for an invalid
 * description). */
size_t specopd_sparse_workspace_bytes(const specopd_tree_desc* desc, int Hq, int Hkv, int di, int g, int topk);

/*
 * specopd_sparse_tree_attention -- sparse attention with branch-consistent
 * indexer groups over a proposal tree.
 *
 * SpecOPD (thelatestinai.com listing), Fig 4: rows reuse complete trunk group
 * keys; an incomplete boundary group stays in the causal tail; a group
 * completed by branch tokens gets a branch-specific indexer key; indexer
 * queries select complete groups with top-k; attention reads the selected
 * groups plus the causal tail, which bypasses top-k.  Readings (the figure
 * prints no formula): groups are g consecutive semantic positions of the
 * row's own history (trunk through the anchor, then its branch); a complete
 * group's key is the mean of its members' indexer keys; the score is the
 * indexer query dotted with it, taken in fp32 in a fixed order (members
 * summed in position order, products summed by a fixed reduction tree); the
 * k best per KV head, ties to the earlier
 * group; attention as specopd_tree_attention (rotate-half RoPE at `pos`,
 * scale softmax_scale or 1/sqrt(d) when <= 0) over the chosen members and the
 * tail, fp32 accumulation.  For g a multiple of 64 the attention runs on the
 * tensor cores (the tree-attention kernel with a per-row group filter); other
 * g run a SIMT kernel.
 *
 * q [N, Hq, 128], k, v [N, Hkv, 128], qi, ki [N, Hkv, di] (di <= 256), out
 * [N, Hq, 128]: device bf16, row-major, 16-byte aligned.  pos, trunk_limit,
 * anc_bits, tile_meta (num_tiles entries): outputs of specopd_build_tree_mask
 * for the same description.  1 <= topk <= 64; a tree's trunk plus one branch
 * must hold at most 1,024 complete groups.  selected (nullable, device int32
 * [N, Hkv, topk]) receives each (row, KV head)'s chosen complete groups in
 * ascending order (group m covers positions m g .. m g + g - 1), -1 past the
 * row's count (min(topk, complete groups)).  workspace >=
 * specopd_sparse_workspace_bytes, 256-byte aligned.  Returns
 * SPECOPD_ERR_SHAPE / _ARG / _ALIGN / _WORKSPACE before anything is enqueued,
 * SPECOPD_ERR_CUDA if a launch fails; a timed-out in-kernel wait sets
 * SPECOPD_FLAG_TIMEOUT in *status.
 */
int specopd_sparse_tree_attention(const specopd_tree_desc* desc, const void* q, const void* k, const void* v,
                                  const void* qi, const void* ki, void* out, int64_t N, int Hq, int Hkv, int d,
                                  int di, int g, int topk, float rope_theta, float softmax_scale, const int32_t* pos,
                                  const int32_t* trunk_limit, const uint64_t* anc_bits,
                                  const specopd_tile_meta* tile_meta, int64_t num_tiles, int32_t* selected,
                                  void* workspace, size_t workspace_bytes, int32_t* status,
                                  specopd_stream_t stream);

/* Bytes of workspace specopd_lm_head_overlap needs (0 for invalid sizes). */
size_t specopd_lm_head_workspace_bytes(int64_t rows, int64_t V);

/*
 * specopd_lm_head_overlap -- overlap, E2E-TV loss and dL/dalpha straight from
 * hidden states and LM heads, without materialising the [rows, V] logits.
 *
 * The write-up's section "Inputs and code mapping": prediction_logits reads
 * supplied hidden states and a supplied head, and e2e_tv_loss consumes the
 * same-history aligned logits of draft and teacher.  Reading (the pages name
 * nothing more): logits = h head^T, no bias, temperature 1, every vocabulary
 * entry active.  alpha, L, dL/dalpha and dL/dz are those of
 * specopd_tv_overlap_e2e (section "Equations").  The logits of a row are formed
 * tile by tile in TMEM (bf16 products, fp32 accumulation) twice, once for the
 * normalisers and once for alpha and q_less, and with grad_draft a third time
 * (draft only) to write dL/dz = dL/dalpha * q (1[q < p] - q_less).
 *
 * h_draft [rows, Hd], head_draft [V, Hd], h_teacher [rows, Ht],
 * head_teacher [V, Ht]: device bf16, row-major and contiguous, 16-byte
 * aligned; Hd and Ht are multiples of 64.  Rows are predictions b-major (row
 * b*W + i-1 holds y_{b,i}); rows must equal num_branches * W; count <= 0
 * means rows.  Outputs (device fp32): alpha [rows] (nullable: then kept in the
 * workspace), q_less [rows], lse_draft / lse_teacher [rows] (natural log),
 * loss (scalar), grad_alpha [rows] and grad_draft [rows, ld_grad] (16-byte
 * aligned rows, ld_grad >= V), all but loss nullable.  workspace:
 * device, >= specopd_lm_head_workspace_bytes(rows, V), 256-byte aligned;
 * the caller owns every buffer.  A non-finite logit sets
 * SPECOPD_FLAG_NONFINITE in *status; a timed-out in-kernel wait sets
 * SPECOPD_FLAG_TIMEOUT.  Returns SPECOPD_ERR_SHAPE / _ARG / _ALIGN /
 * _WORKSPACE before anything is enqueued, SPECOPD_ERR_CUDA if a launch fails.
 */
int specopd_lm_head_overlap(const void* h_draft, const void* head_draft, int Hd, const void* h_teacher,
                            const void* head_teacher, int Ht, int64_t rows, int64_t V, int64_t num_branches, int W,
                            double count, float* alpha, float* q_less, float* lse_draft, float* lse_teacher,
                            float* loss, float* grad_alpha, float* grad_draft, int64_t ld_grad, void* workspace,
                            size_t workspace_bytes, int32_t* status, specopd_stream_t stream);

/*
 * specopd_lm_head_shard_phase -- the LM head + overlap of specopd_lm_head_overlap
 * split over vocabulary shards (one shard per GPU), one phase at a time.
 *
 * The write-up's section "Inputs and code mapping" (prediction_logits from
 * supplied hidden states and head; e2e_tv_loss on the aligned logits), with
 * the vocabulary split: every rank holds all hidden states and the rows
 * [v0, v0 + V_shard) of both heads.  alpha needs both full-vocabulary
 * normalisers before any min, so the phases are separated by three per-row
 * exchanges of the ranks' partials (gather them in rank order, combine with
 * specopd_merge_parts):
 *   phase 0 -- out1 / out2 = the shard's base-2 log-sum-exps of draft /
 *              teacher logits per row [rows] (gather, merge with mode 1 ->
 *              the global lz2, lt2);
 *   phase 1 -- with the global lz2, lt2: out1 / out2 = the shard's alpha /
 *              q_less shares [rows] (gather, merge with mode 0 -> alpha,
 *              q_less; then specopd_e2e_tv_loss on alpha gives L and dL/dalpha);
 *              the [q < p] bits of the shard stay in the workspace;
 *   phase 2 -- with the global lz2, q_less and dL/dalpha (grad_alpha): out1 =
 *              dL/dz of the shard's columns, [rows, ld_grad] fp32 (16-byte
 *              aligned rows), from the bits phase 1 left in the same workspace.
 * Arguments as specopd_lm_head_overlap, heads of V_shard rows; lz2 / lt2 are
 * base-2 (log2 of the softmax normaliser).  workspace >=
 * specopd_lm_head_workspace_bytes(rows, V_shard), kept between phases 1 and 2.
 * A non-finite logit sets SPECOPD_FLAG_NONFINITE (phase 0).  One GPU runs the
 * same steps with one shard; the result equals specopd_lm_head_overlap up to
 * summation order.
 */
int specopd_lm_head_shard_phase(int phase, const void* h_draft, const void* head_draft, int Hd, const void* h_teacher,
                                const void* head_teacher, int Ht, int64_t rows, int64_t V_shard, const float* lz2,
                                const float* lt2, const float* q_less, const float* grad_alpha, float* out1,
                                float* out2, int64_t ld_grad, void* workspace, size_t workspace_bytes,
                                int32_t* status, specopd_stream_t stream);

/*
 * specopd_merge_parts -- out[i] from parts[k][i], k = 0 .. nparts-1, combined
 * in part order: mode 0 the sum, mode 1 the base-2 log-sum-exp (the maximum,
 * then log2 of the sum of 2^(x - maximum); a part of +inf or NaN is passed
 * on, all -inf gives -inf).  parts [nparts][n], out [n]: device fp32.  Used
 * between the phases of specopd_lm_head_shard_phase.
 */
int specopd_merge_parts(const float* parts, int nparts, int64_t n, int mode, float* out, specopd_stream_t stream);

/*
 * specopd_tv_overlap_e2e_static -- specopd_tv_overlap_e2e without a workspace.
 *
 * The paper has no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory for a workspace: programs whose device
 * memory belongs to another allocator they must not bypass, and hot loops
 * that must not call cudaMalloc/cudaFree because those calls can stall the
 * whole device.  The scratch is a fixed array of SPECOPD_STATIC_SCRATCH_BYTES
 * inside the library; every GPU that loads the library holds it until the
 * process exits.  Arguments, outputs and results are those of
 * specopd_tv_overlap_e2e minus the workspace; the call allocates nothing.
 *
 * Limits and caveats:
 *   - a batch whose specopd_overlap_workspace_bytes(rows, V, num_branches)
 *     exceeds SPECOPD_STATIC_SCRATCH_BYTES is rejected with
 *     SPECOPD_ERR_WORKSPACE before anything is enqueued (32 MiB holds, e.g.,
 *     1,600 rows of a 151,936-entry vocabulary);
 *   - arguments are checked as in specopd_tv_overlap_e2e first, then the
 *     batch against the fixed size;
 *   - the first call on a device looks up the array's device address and the
 *     library keeps it for the life of the process; make that first call
 *     before starting any stream capture, and do not use this entry point on
 *     a device after cudaDeviceReset (the kept address would be stale);
 *   - all calls on a device share the one array and it keeps the previous
 *     call's contents (the call clears what must start at zero itself), so
 *     calls that may run at the same time on the GPU -- e.g. on two streams --
 *     race and corrupt each other: order them on one stream.
 */
#define SPECOPD_STATIC_SCRATCH_BYTES ((size_t)32 << 20)
int specopd_tv_overlap_e2e_static(const void* draft, const void* teacher, specopd_dtype dtype, int64_t rows,
                                  int64_t V, int64_t ld_draft, int64_t ld_teacher, int64_t num_branches, int W,
                                  double count, float* alpha, float* loss, float* grad_draft, int64_t ld_grad,
                                  int32_t* status, specopd_stream_t stream);

/* Human-readable name of a specopd_status value. */
const char* specopd_status_string(int status);

#ifdef __cplusplus
}
#endif
#endif /* SPECOPD_H_ */
