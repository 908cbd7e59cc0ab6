// Internal launch interfaces shared by the kernel files and the C ABI layer.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/specopd.h"

namespace specopd {

// Per-tree layout of a batch, computed on the host and passed by value.
struct TreeParams {
  int32_t num_trees;
  int32_t W;
  int32_t rows_per_branch;
  int32_t total_branches;
  int32_t num_tiles;
  int32_t row_base[SPECOPD_MAX_TREES + 1];     // first packed row of each tree
  int32_t trunk_len[SPECOPD_MAX_TREES];
  int32_t prompt_len[SPECOPD_MAX_TREES];
  int32_t branch_base[SPECOPD_MAX_TREES + 1];  // first global branch id of each tree
  int32_t tile_base[SPECOPD_MAX_TREES + 1];    // first query tile of each tree
};

cudaError_t launch_tree_mask(const TreeParams& p, const int32_t* anchors, int32_t* pos, int32_t* trunk_limit,
                             int32_t* branch_of, uint64_t* anc_bits, int32_t* pred_rows, int32_t* cu_rows,
                             specopd_tile_meta* tile_meta, int32_t* status, cudaStream_t stream);

cudaError_t launch_rope(const void* q, const void* k, void* q_out, void* k_out, specopd_dtype dtype, int64_t N,
                        int Hq, int Hkv, int d, const int32_t* pos, float theta, cudaStream_t stream);

struct AttnArgs {
  const void* q;  // rotated
  const void* k;  // rotated
  const void* v;
  void* out;
  int64_t N;
  int Hq, Hkv, d;
  float scale;
  const int32_t* pos;
  const int32_t* trunk_limit;
  const uint64_t* anc_bits;
  const specopd_tile_meta* meta;
  int64_t num_tiles;
  int32_t* status;
};

// Indexer-group selection read by the tcgen05 kernel's sparse mode: per
// (row, KV head) `words` uint32 words, bit m set iff complete group m of the
// row's history is selected; g a multiple of 64.
struct SparseSel {
  const uint32_t* mask;
  int words;
  int g;
};
// tcgen05 kernel: bf16, d = 128; sparse mode when sel is non-null.
cudaError_t launch_tree_attention_sm100(const AttnArgs& a, cudaStream_t stream, const SparseSel* sel = nullptr);
// SIMT kernel: fp32 or bf16, d multiple of 32 up to 256.
cudaError_t launch_tree_attention_simt(const AttnArgs& a, specopd_dtype dtype, cudaStream_t stream);

struct OverlapArgs {
  const void* draft;
  const void* teacher;
  int64_t ld_draft, ld_teacher;
  int64_t rows, V;
  // one launch computes the statistics of rows [row_begin, row_end) and the
  // gradient of rows [grad_begin, grad_end) (an empty range: no gradient);
  // per-row and per-branch outputs are indexed by the global row
  int64_t row_begin, row_end;
  int64_t grad_begin, grad_end;
  // outputs of the statistics pass
  float* alpha;
  float* q_less;     // nullable
  float* lse_draft;  // nullable (natural log)
  float* lse_teacher;
  // fused path (all null in the unfused entry point)
  uint8_t* mbits;    // [rows, mbits_ld] strict-less bits
  int64_t mbits_ld;
  float* lz2;        // [rows] draft normaliser, log2 units
  float* ql;         // [rows] q_less
  float* g;          // [rows] dL/dalpha
  uint32_t* branch_cnt;  // [num_branches + 2], zero on entry: arrivals per branch, branches done,
                         // gradient units claimed
  double* branch_sum;    // [num_branches]
  float* loss;
  int W;
  int64_t num_branches;
  double inv_count;
  // gradient output (fused path)
  float* grad;
  int64_t ld_grad;
  int32_t* status;
};

// Every argument check of specopd_tv_overlap_e2e except its workspace (api.cu).
int check_overlap_e2e_args(const void* draft, const void* teacher, specopd_dtype dtype, int64_t rows, int64_t V,
                           int64_t ld_draft, int64_t ld_teacher, int64_t num_branches, int W, double count,
                           const float* alpha, const float* loss, const float* grad_draft, int64_t ld_grad,
                           const int32_t* status);

cudaError_t launch_tv_stats(const OverlapArgs& a, specopd_dtype dtype, cudaStream_t stream);
// bf16 kernels (tv_bf16.cu); launch_tv_stats routes bf16 here
cudaError_t launch_tv_stats_bf16(const OverlapArgs& a, cudaStream_t stream);
// bf16 statistics + gradient in one cooperative launch (the only bf16 gradient path)
cudaError_t launch_tv_fused_bf16(OverlapArgs a, cudaStream_t stream);
cudaError_t launch_tv_grad(const OverlapArgs& a, specopd_dtype dtype, cudaStream_t stream);
cudaError_t launch_e2e_loss(const float* alpha, int64_t num_branches, int W, double inv_count, float* loss,
                            float* grad_alpha, cudaStream_t stream);

// Short causal convolution along each row's history (tree_conv.cu).
cudaError_t launch_tree_conv(const void* x, void* out, specopd_dtype dtype, int64_t N, int C, const float* w,
                             const float* bias, int Kw, int silu, const int32_t* pos, const int32_t* trunk_limit,
                             const int32_t* cu_rows, int num_trees, cudaStream_t stream);

// Gated DeltaNet over a proposal tree with indexed state replay (gdn.cu).
struct GdnArgs {
  const void* q;        // [N, H, 128] bf16
  const void* k;        // [N, H, 128] bf16
  const void* v;        // [N, H, 128] bf16
  const float* alpha;   // [N, H]
  const float* beta;    // [N, H]
  float* out;           // [N, H, 128] fp32
  int H;
  const int32_t* anchors;  // device [total branches], zero-based within the tree
  float* ckpt;             // [sum_t T_t / 64][H][128][128] fp32 checkpoints
  float* chunk_data;       // per trunk chunk and head: the chunked form's data (gdn.cu)
  int32_t* status;
  TreeParams tp;
  int32_t ck_off[SPECOPD_MAX_TREES];      // first checkpoint of each tree (set by the launcher)
  int32_t ch_off[SPECOPD_MAX_TREES + 1];  // first trunk chunk of each tree (set by the launcher)
};
size_t gdn_checkpoint_floats(const TreeParams& tp, int H);
size_t gdn_chunk_floats(const TreeParams& tp, int H);
cudaError_t launch_gdn_tree(GdnArgs g, cudaStream_t stream);

// Sparse attention with branch-consistent indexer groups (sparse_attn.cu).
constexpr int kSpMaxGroups = 1024;  // complete groups a row may score
constexpr int kSpMaxTopk = 64;
struct SparseArgs {
  const void* q;        // [N, Hq, 128] bf16
  const void* k;        // [N, Hkv, 128] bf16
  const void* v;        // [N, Hkv, 128] bf16
  const void* qi;       // [N, Hkv, di] bf16 indexer queries
  const void* ki;       // [N, Hkv, di] bf16 indexer keys
  void* out;            // [N, Hq, 128] bf16
  void* rq;             // workspace: rotated q
  void* rk;             // workspace: rotated k
  float* gkey;          // workspace: per tree [Hkv][di][trunk groups of the tree] fp32
  float* bkey;          // workspace: [branches][bslots][Hkv][di] fp32, keys of groups holding branch tokens
  int bslots;           // rows_per_branch / g + 1: groups holding branch tokens per branch, at most
  int64_t N;
  int Hq, Hkv, di, g, topk;
  float theta, scale, scale_log2;  // softmax scale and scale * log2(e)
  const int32_t* pos;      // [N] semantic positions (specopd_build_tree_mask)
  const int32_t* trunk_limit;            // [N] (specopd_build_tree_mask)
  const uint64_t* anc_bits;              // [N]
  const specopd_tile_meta* meta;         // [num_tiles]
  int64_t num_tiles;
  const int32_t* anchors;  // [total branches]
  int32_t* sel_list;       // workspace: [N][Hkv][topk] chosen groups, ascending, -1 padded
  uint32_t* sel_mask;      // workspace: [N][Hkv][sel_words] bit m = group m chosen
  int sel_words;
  int32_t* sel_out;        // nullable caller copy of sel_list
  int32_t* status;
  TreeParams tp;
  int32_t gk_off[SPECOPD_MAX_TREES + 1];  // first trunk group of each tree (set by the launcher)
};
size_t sparse_group_keys(const TreeParams& tp, int g);
// slots per branch for the keys of complete groups that hold branch tokens
inline int sparse_branch_slots(const TreeParams& tp, int g) { return tp.rows_per_branch / g + 1; }
int sparse_selection_words(const TreeParams& tp, int g);
cudaError_t launch_sparse_attention(SparseArgs s, cudaStream_t stream);

// Overlap statistics from hidden states and LM heads (lm_head_sm100.cu).
struct LmHeadArgs {
  const void* h_draft;    // [rows, Hd] bf16
  const void* w_draft;    // [V, Hd] bf16
  const void* h_teacher;  // [rows, Ht] bf16
  const void* w_teacher;  // [V, Ht] bf16
  int64_t rows, V;
  int Hd, Ht;
  int64_t num_branches;
  int W;
  double inv_count;
  float* alpha;         // nullable: workspace then
  float* q_less;        // nullable
  float* lse_draft;     // nullable (natural log)
  float* lse_teacher;   // nullable
  float* loss;
  float* grad_alpha;    // nullable
  float* grad_draft;    // nullable: [rows, ld_grad] dL/dz
  int64_t ld_grad;
  void* workspace;
  int32_t* status;
};
struct LmHeadLayout {
  int64_t n_tiles;
  size_t part_a, part_b, lz2, lt2, alpha, q_less, g, bits, total;
};
LmHeadLayout lm_head_layout(int64_t rows, int64_t V);
cudaError_t launch_lm_head_overlap(const LmHeadArgs& a, cudaStream_t stream);
// one phase over a vocabulary shard (lm_head_sm100.cu): 0 stats, 1 alpha/q_less shares, 2 dL/dz
cudaError_t launch_lm_head_phase(LmHeadArgs a, int phase, const float* lz2, const float* lt2, const float* q_less,
                                 const float* g, float* out1, float* out2, cudaStream_t stream);
// parts [nparts][n] combined in part order: mode 0 sum, mode 1 base-2 log-sum-exp
cudaError_t launch_merge_parts(const float* parts, int nparts, int64_t n, int mode, float* out, cudaStream_t stream);

}  // namespace specopd
