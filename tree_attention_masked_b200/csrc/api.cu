// C ABI of the library (include/specopd.h): host-side validation, workspace
// carving and kernel launches.  Nothing here allocates or synchronises.
#include <cmath>
#include <cstring>

#include "internal.h"

using namespace specopd;

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Validate a tree description and fill the per-tree layout.  Returns a status.
int tree_params(const specopd_tree_desc* d, TreeParams* p) {
  if (!d || !d->trunk_len || !d->prompt_len || !d->num_branches) return SPECOPD_ERR_ARG;
  if (d->num_trees < 1 || d->num_trees > SPECOPD_MAX_TREES) return SPECOPD_ERR_ARG;
  if (d->W < 1 || d->W > SPECOPD_MAX_W) return SPECOPD_ERR_ARG;
  if (d->pack_terminal != 0 && d->pack_terminal != 1) return SPECOPD_ERR_ARG;
  std::memset(p, 0, sizeof(*p));
  p->num_trees = d->num_trees;
  p->W = d->W;
  p->rows_per_branch = d->pack_terminal ? d->W : d->W - 1;
  long long rows = 0, branches = 0, tiles = 0;
  for (int t = 0; t < d->num_trees; ++t) {
    const long long T = d->trunk_len[t], P = d->prompt_len[t], B = d->num_branches[t];
    if (T < 1 || P < 0 || P > T - 1 || B < 0) return SPECOPD_ERR_ARG;
    const long long n = T + B * p->rows_per_branch;
    p->row_base[t] = (int32_t)rows;
    p->trunk_len[t] = (int32_t)T;
    p->prompt_len[t] = (int32_t)P;
    p->branch_base[t] = (int32_t)branches;
    p->tile_base[t] = (int32_t)tiles;
    rows += n;
    branches += B;
    tiles += (n + SPECOPD_TILE_ROWS - 1) / SPECOPD_TILE_ROWS;
    if (rows > (1LL << 30) || branches * d->W > (1LL << 30)) return SPECOPD_ERR_SHAPE;
  }
  p->row_base[d->num_trees] = (int32_t)rows;
  p->branch_base[d->num_trees] = (int32_t)branches;
  p->tile_base[d->num_trees] = (int32_t)tiles;
  p->total_branches = (int32_t)branches;
  p->num_tiles = (int32_t)tiles;
  return SPECOPD_OK;
}

inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? SPECOPD_OK : SPECOPD_ERR_CUDA; }

size_t elem_size(specopd_dtype dt) { return dt == SPECOPD_BF16 ? 2 : 4; }

struct OverlapLayout {
  size_t mbits, lz2, ql, g, counters, bsum, total;
  size_t counters_bytes;
  int64_t mbits_ld;
};

// Workspace of the fused overlap pass (all regions 256-byte aligned):
//   mbits     [rows][mbits_ld]  one bit per logit, [q < p]
//   lz2, ql, g [rows]           draft normaliser (base 2), q_less, dL/dalpha
//   counters  branch arrivals [nb] + branches done [1] + gradient units claimed [1]
//   bsum      [nb] doubles      each branch's share of L
OverlapLayout overlap_layout(int64_t rows, int64_t V, int64_t nb) {
  OverlapLayout L;
  L.mbits_ld = ((V + 7) / 8 + 15) / 16 * 16;
  size_t off = 0;
  L.mbits = off;
  off = align_up(off + (size_t)rows * L.mbits_ld);
  L.lz2 = off;
  off = align_up(off + (size_t)rows * 4);
  L.ql = off;
  off = align_up(off + (size_t)rows * 4);
  L.g = off;
  off = align_up(off + (size_t)rows * 4);
  L.counters = off;
  L.counters_bytes = (size_t)(nb + 2) * 4;
  off = align_up(off + L.counters_bytes);
  L.bsum = off;
  off = align_up(off + (size_t)nb * 8);
  L.total = off;
  return L;
}

}  // namespace

extern "C" {

int64_t specopd_tree_packed_rows(const specopd_tree_desc* desc) {
  TreeParams p;
  const int s = tree_params(desc, &p);
  return s != SPECOPD_OK ? s : (int64_t)p.row_base[p.num_trees];
}

int64_t specopd_tree_num_tiles(const specopd_tree_desc* desc) {
  TreeParams p;
  const int s = tree_params(desc, &p);
  return s != SPECOPD_OK ? s : (int64_t)p.num_tiles;
}

int64_t specopd_tree_num_predictions(const specopd_tree_desc* desc) {
  TreeParams p;
  const int s = tree_params(desc, &p);
  return s != SPECOPD_OK ? s : (int64_t)p.total_branches * p.W;
}

int specopd_build_tree_mask(const specopd_tree_desc* desc, int32_t* pos, int32_t* trunk_limit,
                            int32_t* branch_of, uint64_t* anc_bits, int32_t* pred_rows, int32_t* cu_rows,
                            specopd_tile_meta* tile_meta, int32_t* status, specopd_stream_t stream) {
  TreeParams local;
  const int s = tree_params(desc, &local);
  if (s != SPECOPD_OK) return s;
  if (!pos || !trunk_limit || !branch_of || !anc_bits || !cu_rows || !tile_meta || !status) return SPECOPD_ERR_ARG;
  if (local.total_branches > 0 && (!desc->anchors || !pred_rows)) return SPECOPD_ERR_ARG;
  return cuda_status(launch_tree_mask(local, desc->anchors, pos, trunk_limit, branch_of, anc_bits, pred_rows,
                                      cu_rows, tile_meta, status, reinterpret_cast<cudaStream_t>(stream)));
}

int specopd_rope(const void* q, const void* k, void* q_out, void* k_out, specopd_dtype dtype, int64_t N, int Hq,
                 int Hkv, int d, const int32_t* pos, float theta, specopd_stream_t stream) {
  if (dtype != SPECOPD_F32 && dtype != SPECOPD_BF16) return SPECOPD_ERR_DTYPE;
  if (N < 0 || Hq < 0 || Hkv < 0 || Hq + Hkv < 1 || d < 4 || d > 256 || d % 4) return SPECOPD_ERR_SHAPE;
  if (N > 0 && (!pos || (Hq > 0 && (!q || !q_out)) || (Hkv > 0 && (!k || !k_out)))) return SPECOPD_ERR_ARG;
  if (!(theta > 0.f) || !std::isfinite(theta)) return SPECOPD_ERR_ARG;
  return cuda_status(
      launch_rope(q, k, q_out, k_out, dtype, N, Hq, Hkv, d, pos, theta, reinterpret_cast<cudaStream_t>(stream)));
}

size_t specopd_attention_workspace_bytes(specopd_dtype dtype, int64_t N, int Hq, int Hkv, int d) {
  if (N <= 0 || Hq < 1 || Hkv < 1 || d < 1) return 0;
  const size_t e = elem_size(dtype);
  return align_up((size_t)N * Hq * d * e) + align_up((size_t)N * Hkv * d * e);
}

int specopd_tree_attention(const void* q, const void* k, const void* v, void* out, specopd_dtype dtype,
                           int64_t N, int Hq, int Hkv, int d, float rope_theta, float softmax_scale,
                           const int32_t* pos, const int32_t* trunk_limit, const uint64_t* anc_bits,
                           const specopd_tile_meta* tile_meta, int64_t num_tiles, void* workspace,
                           size_t workspace_bytes, int32_t* status, specopd_stream_t stream) {
  if (dtype != SPECOPD_F32 && dtype != SPECOPD_BF16) return SPECOPD_ERR_DTYPE;
  if (N < 0 || num_tiles < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv) return SPECOPD_ERR_SHAPE;
  if (d < 32 || d > 256 || d % 32) return SPECOPD_ERR_SHAPE;
  if (N == 0) return SPECOPD_OK;
  if (num_tiles > N) return SPECOPD_ERR_SHAPE;  // every tile holds at least one row
  if (num_tiles == 0) return SPECOPD_OK;
  if (!q || !k || !v || !out || !pos || !trunk_limit || !anc_bits || !tile_meta || !status) return SPECOPD_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return SPECOPD_ERR_ALIGN;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const void* qr = q;
  const void* kr = k;
  if (rope_theta > 0.f) {
    if (!std::isfinite(rope_theta)) return SPECOPD_ERR_ARG;
    const size_t need = specopd_attention_workspace_bytes(dtype, N, Hq, Hkv, d);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) % kAlign))
      return SPECOPD_ERR_WORKSPACE;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    void* qo = ws;
    void* ko = ws + align_up((size_t)N * Hq * d * elem_size(dtype));
    const int rs = specopd_rope(q, k, qo, ko, dtype, N, Hq, Hkv, d, pos, rope_theta, stream);
    if (rs != SPECOPD_OK) return rs;
    qr = qo;
    kr = ko;
  }
  AttnArgs a;
  a.q = qr;
  a.k = kr;
  a.v = v;
  a.out = out;
  a.N = N;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.d = d;
  a.scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)d);
  a.pos = pos;
  a.trunk_limit = trunk_limit;
  a.anc_bits = anc_bits;
  a.meta = tile_meta;
  a.num_tiles = num_tiles;
  a.status = status;
  if (dtype == SPECOPD_BF16 && d == 128) return cuda_status(launch_tree_attention_sm100(a, st));
  return cuda_status(launch_tree_attention_simt(a, dtype, st));
}

size_t specopd_overlap_workspace_bytes(int64_t rows, int64_t V, int64_t num_branches) {
  if (rows < 0 || V < 1 || num_branches < 0) return 0;
  return overlap_layout(rows, V, num_branches).total;
}

static int check_logits(const void* draft, const void* teacher, specopd_dtype dtype, int64_t rows, int64_t V,
                        int64_t ld_draft, int64_t ld_teacher) {
  if (dtype != SPECOPD_F32 && dtype != SPECOPD_BF16) return SPECOPD_ERR_DTYPE;
  if (rows < 0 || V < 1 || ld_draft < V || ld_teacher < V) return SPECOPD_ERR_SHAPE;
  if (V > (1LL << 20)) return SPECOPD_ERR_SHAPE;
  if (rows > 0 && (!draft || !teacher)) return SPECOPD_ERR_ARG;
  const size_t e = elem_size(dtype);
  if (!aligned16(draft) || !aligned16(teacher) || (ld_draft * e) % 16 || (ld_teacher * e) % 16)
    return SPECOPD_ERR_ALIGN;
  return SPECOPD_OK;
}

int specopd_tv_overlap(const void* draft, const void* teacher, specopd_dtype dtype, int64_t rows, int64_t V,
                       int64_t ld_draft, int64_t ld_teacher, float* alpha, float* q_less, float* lse_draft,
                       float* lse_teacher, int32_t* status, specopd_stream_t stream) {
  const int c = check_logits(draft, teacher, dtype, rows, V, ld_draft, ld_teacher);
  if (c != SPECOPD_OK) return c;
  if (rows == 0) return SPECOPD_OK;
  if (!alpha || !status) return SPECOPD_ERR_ARG;
  OverlapArgs a;
  std::memset(&a, 0, sizeof(a));
  a.draft = draft;
  a.teacher = teacher;
  a.ld_draft = ld_draft;
  a.ld_teacher = ld_teacher;
  a.rows = rows;
  a.V = V;
  a.row_begin = 0;
  a.row_end = rows;
  a.alpha = alpha;
  a.q_less = q_less;
  a.lse_draft = lse_draft;
  a.lse_teacher = lse_teacher;
  a.status = status;
  return cuda_status(launch_tv_stats(a, dtype, reinterpret_cast<cudaStream_t>(stream)));
}

int specopd_e2e_tv_loss(const float* alpha, int64_t num_branches, int W, double count, float* loss,
                        float* grad_alpha, specopd_stream_t stream) {
  if (num_branches < 0 || W < 1 || W > SPECOPD_MAX_W) return SPECOPD_ERR_SHAPE;
  if (!loss || (num_branches > 0 && !alpha)) return SPECOPD_ERR_ARG;
  if (!(count <= 0.0) && !std::isfinite(count)) return SPECOPD_ERR_ARG;
  const double n = count > 0.0 ? count : (double)num_branches * W;
  const double inv = n > 0.0 ? 1.0 / n : 0.0;
  return cuda_status(
      launch_e2e_loss(alpha, num_branches, W, inv, loss, grad_alpha, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"

// Every check of specopd_tv_overlap_e2e's arguments except the workspace.
int specopd::check_overlap_e2e_args(const void* draft, const void* teacher, specopd_dtype dtype, int64_t rows,
                                    int64_t V, int64_t ld_draft, int64_t ld_teacher, int64_t num_branches, int W,
                                    double count, const float* alpha, const float* loss, const float* grad_draft,
                                    int64_t ld_grad, const int32_t* status) {
  const int c = check_logits(draft, teacher, dtype, rows, V, ld_draft, ld_teacher);
  if (c != SPECOPD_OK) return c;
  if (W < 1 || W > SPECOPD_MAX_W || num_branches < 0 || rows != num_branches * W) return SPECOPD_ERR_SHAPE;
  if (!loss || !status) return SPECOPD_ERR_ARG;
  if (!(count <= 0.0) && !std::isfinite(count)) return SPECOPD_ERR_ARG;
  if (rows == 0) return SPECOPD_OK;
  if (!alpha) return SPECOPD_ERR_ARG;
  if (grad_draft && (ld_grad < V || !aligned16(grad_draft) || (ld_grad * 4) % 16)) return SPECOPD_ERR_ALIGN;
  return SPECOPD_OK;
}

extern "C" {

int specopd_tv_overlap_e2e(const void* draft, const void* teacher, specopd_dtype dtype, int64_t rows, int64_t V,
                           int64_t ld_draft, int64_t ld_teacher, int64_t num_branches, int W, double count,
                           float* alpha, float* loss, float* grad_draft, int64_t ld_grad, void* workspace,
                           size_t workspace_bytes, int32_t* status, specopd_stream_t stream) {
  const int c = check_overlap_e2e_args(draft, teacher, dtype, rows, V, ld_draft, ld_teacher, num_branches, W, count,
                                       alpha, loss, grad_draft, ld_grad, status);
  if (c != SPECOPD_OK) return c;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (rows == 0) return cuda_status(cudaMemsetAsync(loss, 0, sizeof(float), st));
  const OverlapLayout L = overlap_layout(rows, V, num_branches);
  if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) % kAlign))
    return SPECOPD_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const double n = count > 0.0 ? count : (double)rows;
  OverlapArgs a;
  std::memset(&a, 0, sizeof(a));
  a.draft = draft;
  a.teacher = teacher;
  a.ld_draft = ld_draft;
  a.ld_teacher = ld_teacher;
  a.rows = rows;
  a.V = V;
  a.row_begin = 0;
  a.row_end = rows;
  a.alpha = alpha;
  a.mbits = grad_draft ? ws + L.mbits : nullptr;
  a.mbits_ld = L.mbits_ld;
  a.lz2 = reinterpret_cast<float*>(ws + L.lz2);
  a.ql = reinterpret_cast<float*>(ws + L.ql);
  a.g = reinterpret_cast<float*>(ws + L.g);
  uint32_t* counters = reinterpret_cast<uint32_t*>(ws + L.counters);
  a.branch_cnt = counters;  // [nb] arrivals per branch, [1] branches done, [1] gradient units claimed
  a.branch_sum = reinterpret_cast<double*>(ws + L.bsum);
  a.loss = loss;
  a.W = W;
  a.num_branches = num_branches;
  a.inv_count = 1.0 / n;
  a.grad = grad_draft;
  a.ld_grad = ld_grad;
  a.status = status;
  cudaError_t e = cudaMemsetAsync(counters, 0, L.counters_bytes, st);
  if (e != cudaSuccess) return SPECOPD_ERR_CUDA;
  if (dtype == SPECOPD_BF16 && grad_draft) {
    e = launch_tv_fused_bf16(a, st);
    return e == cudaSuccess ? SPECOPD_OK : SPECOPD_ERR_CUDA;
  }
  e = launch_tv_stats(a, dtype, st);
  if (e != cudaSuccess) return SPECOPD_ERR_CUDA;
  if (grad_draft) {
    a.grad_begin = 0;
    a.grad_end = rows;
    e = launch_tv_grad(a, dtype, st);
    if (e != cudaSuccess) return SPECOPD_ERR_CUDA;
  }
  return SPECOPD_OK;
}

int specopd_diag_overlap_wait_timeout(const void* draft, const void* teacher, int64_t rows, int64_t V,
                                      int64_t ld_draft, int64_t ld_teacher, int64_t num_branches, int W,
                                      float* grad_draft, int64_t ld_grad, void* workspace, size_t workspace_bytes,
                                      int32_t* status, specopd_stream_t stream) {
  const int c = check_logits(draft, teacher, SPECOPD_BF16, rows, V, ld_draft, ld_teacher);
  if (c != SPECOPD_OK) return c;
  if (W < 1 || W > SPECOPD_MAX_W || num_branches < 1 || rows != num_branches * W) return SPECOPD_ERR_SHAPE;
  if (!status || !grad_draft) return SPECOPD_ERR_ARG;
  if (ld_grad < V || !aligned16(grad_draft) || (ld_grad * 4) % 16) return SPECOPD_ERR_ALIGN;
  const OverlapLayout L = overlap_layout(rows, V, num_branches);
  if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) % kAlign))
    return SPECOPD_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  OverlapArgs a;
  std::memset(&a, 0, sizeof(a));
  a.draft = draft;
  a.teacher = teacher;
  a.ld_draft = ld_draft;
  a.ld_teacher = ld_teacher;
  a.rows = rows;
  a.V = V;
  a.row_begin = 0;  // no statistics rows: no branch is ever published
  a.row_end = 0;
  a.grad_begin = 0;
  a.grad_end = rows;
  a.mbits = ws + L.mbits;
  a.mbits_ld = L.mbits_ld;
  a.lz2 = reinterpret_cast<float*>(ws + L.lz2);
  a.ql = reinterpret_cast<float*>(ws + L.ql);
  a.g = reinterpret_cast<float*>(ws + L.g);
  a.branch_cnt = reinterpret_cast<uint32_t*>(ws + L.counters);
  a.branch_sum = reinterpret_cast<double*>(ws + L.bsum);
  a.W = W;
  a.num_branches = num_branches;
  a.inv_count = 1.0 / (double)rows;
  a.grad = grad_draft;
  a.ld_grad = ld_grad;
  a.status = status;
  if (cudaMemsetAsync(a.branch_cnt, 0, L.counters_bytes, st) != cudaSuccess) return SPECOPD_ERR_CUDA;
  return cuda_status(launch_tv_stats_bf16(a, st));
}

int specopd_tree_causal_conv(const void* x, void* out, specopd_dtype dtype, int64_t N, int C, const float* weight,
                             const float* bias, int Kw, int silu, const int32_t* pos, const int32_t* trunk_limit,
                             const int32_t* cu_rows, int num_trees, specopd_stream_t stream) {
  if (dtype != SPECOPD_F32 && dtype != SPECOPD_BF16) return SPECOPD_ERR_DTYPE;
  const int vec = dtype == SPECOPD_BF16 ? 8 : 4;
  if (N < 0 || N > (1LL << 30) || C < 1 || C % vec || C > (1 << 24) || Kw < 1 || Kw > 8) return SPECOPD_ERR_SHAPE;
  if (num_trees < 1 || num_trees > SPECOPD_MAX_TREES || (silu != 0 && silu != 1)) return SPECOPD_ERR_ARG;
  if (N == 0) return SPECOPD_OK;
  if (!x || !out || !weight || !pos || !trunk_limit || !cu_rows) return SPECOPD_ERR_ARG;
  if (!aligned16(x) || !aligned16(out) || (reinterpret_cast<uintptr_t>(weight) & 3) ||
      (reinterpret_cast<uintptr_t>(bias) & 3))
    return SPECOPD_ERR_ALIGN;
  return cuda_status(launch_tree_conv(x, out, dtype, N, C, weight, bias, Kw, silu, pos, trunk_limit, cu_rows,
                                      num_trees, reinterpret_cast<cudaStream_t>(stream)));
}

size_t specopd_gdn_workspace_bytes(const specopd_tree_desc* desc, int H) {
  TreeParams p;
  if (tree_params(desc, &p) != SPECOPD_OK || H < 1) return 0;
  return align_up(gdn_checkpoint_floats(p, H) * sizeof(float)) + align_up(gdn_chunk_floats(p, H) * sizeof(float));
}

int specopd_gdn_tree(const specopd_tree_desc* desc, const void* q, const void* k, const void* v,
                     const float* alpha, const float* beta, float* out, int64_t N, int H, int dk, int dv,
                     void* workspace, size_t workspace_bytes, int32_t* status, specopd_stream_t stream) {
  GdnArgs g;
  const int s = tree_params(desc, &g.tp);
  if (s != SPECOPD_OK) return s;
  if (dk != 128 || dv != 128 || H < 1 || H > 1024) return SPECOPD_ERR_SHAPE;
  if (N != (int64_t)g.tp.row_base[g.tp.num_trees]) return SPECOPD_ERR_SHAPE;
  if (!q || !k || !v || !alpha || !beta || !out || !status) return SPECOPD_ERR_ARG;
  if (g.tp.total_branches > 0 && !desc->anchors) return SPECOPD_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || (reinterpret_cast<uintptr_t>(alpha) & 3) ||
      (reinterpret_cast<uintptr_t>(beta) & 3))
    return SPECOPD_ERR_ALIGN;
  const size_t ck_bytes = align_up(gdn_checkpoint_floats(g.tp, H) * sizeof(float));
  const size_t need = ck_bytes + align_up(gdn_chunk_floats(g.tp, H) * sizeof(float));
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) % kAlign))
    return SPECOPD_ERR_WORKSPACE;
  g.q = q;
  g.k = k;
  g.v = v;
  g.alpha = alpha;
  g.beta = beta;
  g.out = out;
  g.H = H;
  g.anchors = desc->anchors;
  g.ckpt = static_cast<float*>(workspace);
  g.chunk_data = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + ck_bytes);
  g.status = status;
  return cuda_status(launch_gdn_tree(g, reinterpret_cast<cudaStream_t>(stream)));
}

// Sparse attention workspace (all regions 256-byte aligned): rotated Q [N][Hq][128]
// and K [N][Hkv][128] bf16, trunk group keys [groups][Hkv][di] fp32, the keys of
// the groups holding branch tokens [branches][slots][Hkv][di] fp32, the chosen
// groups [N][Hkv][topk] int32 and the selection words [N][Hkv][words] uint32.
struct SparseLayout {
  size_t rk, gk, bk, list, mask, total;
  int words;
};

static SparseLayout sparse_layout(const TreeParams& p, int Hq, int Hkv, int di, int g, int topk) {
  const int64_t N = p.row_base[p.num_trees];
  SparseLayout L;
  L.words = sparse_selection_words(p, g);
  L.rk = align_up((size_t)N * Hq * 128 * 2);
  L.gk = L.rk + align_up((size_t)N * Hkv * 128 * 2);
  L.bk = L.gk + align_up(sparse_group_keys(p, g) * Hkv * di * sizeof(float));
  L.list = L.bk + align_up((size_t)p.total_branches * sparse_branch_slots(p, g) * Hkv * di * sizeof(float));
  L.mask = L.list + align_up((size_t)N * Hkv * topk * sizeof(int32_t));
  L.total = L.mask + align_up((size_t)N * Hkv * L.words * sizeof(uint32_t));
  return L;
}

size_t specopd_sparse_workspace_bytes(const specopd_tree_desc* desc, int Hq, int Hkv, int di, int g, int topk) {
  TreeParams p;
  if (tree_params(desc, &p) != SPECOPD_OK || Hq < 1 || Hkv < 1 || di < 1 || g < 1 || topk < 1) return 0;
  return sparse_layout(p, Hq, Hkv, di, g, topk).total;
}

int specopd_sparse_tree_attention(const specopd_tree_desc* desc, const void* q, const void* k, const void* v,
                                  const void* qi, const void* ki, void* out, int64_t N, int Hq, int Hkv, int d,
                                  int di, int g, int topk, float rope_theta, float softmax_scale, const int32_t* pos,
                                  const int32_t* trunk_limit, const uint64_t* anc_bits,
                                  const specopd_tile_meta* tile_meta, int64_t num_tiles, int32_t* selected,
                                  void* workspace, size_t workspace_bytes, int32_t* status,
                                  specopd_stream_t stream) {
  SparseArgs a;
  const int st = tree_params(desc, &a.tp);
  if (st != SPECOPD_OK) return st;
  if (d != 128 || Hq < 1 || Hkv < 1 || Hq % Hkv || di < 1 || di > 256 || g < 1 || topk < 1 ||
      topk > kSpMaxTopk)
    return SPECOPD_ERR_SHAPE;
  if (N != (int64_t)a.tp.row_base[a.tp.num_trees] || num_tiles != a.tp.num_tiles) return SPECOPD_ERR_SHAPE;
  for (int t = 0; t < a.tp.num_trees; ++t)  // every row's complete groups must fit the score buffer
    if ((a.tp.trunk_len[t] + a.tp.rows_per_branch) / g > kSpMaxGroups) return SPECOPD_ERR_SHAPE;
  if (!q || !k || !v || !qi || !ki || !out || !pos || !trunk_limit || !anc_bits || !tile_meta || !status)
    return SPECOPD_ERR_ARG;
  if (a.tp.total_branches > 0 && !desc->anchors) return SPECOPD_ERR_ARG;
  if (!(rope_theta > 0.f) || !std::isfinite(rope_theta)) return SPECOPD_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return SPECOPD_ERR_ALIGN;
  const SparseLayout L = sparse_layout(a.tp, Hq, Hkv, di, g, topk);
  if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) % kAlign))
    return SPECOPD_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.q = q;
  a.k = k;
  a.v = v;
  a.qi = qi;
  a.ki = ki;
  a.out = out;
  a.rq = ws;
  a.rk = ws + L.rk;
  a.gkey = reinterpret_cast<float*>(ws + L.gk);
  a.bkey = reinterpret_cast<float*>(ws + L.bk);
  a.bslots = sparse_branch_slots(a.tp, g);
  a.sel_list = reinterpret_cast<int32_t*>(ws + L.list);
  a.sel_mask = reinterpret_cast<uint32_t*>(ws + L.mask);
  a.sel_words = L.words;
  a.sel_out = selected;
  a.N = N;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.di = di;
  a.g = g;
  a.topk = topk;
  a.theta = rope_theta;
  a.scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)d);
  a.scale_log2 = a.scale * 1.4426950408889634f;
  a.pos = pos;
  a.trunk_limit = trunk_limit;
  a.anc_bits = anc_bits;
  a.meta = tile_meta;
  a.num_tiles = num_tiles;
  a.anchors = desc->anchors;
  a.status = status;
  return cuda_status(launch_sparse_attention(a, reinterpret_cast<cudaStream_t>(stream)));
}

size_t specopd_lm_head_workspace_bytes(int64_t rows, int64_t V) {
  if (rows < 0 || V < 1) return 0;
  return lm_head_layout(rows, V).total;
}

int specopd_lm_head_overlap(const void* h_draft, const void* head_draft, int Hd, const void* h_teacher,
                            const void* head_teacher, int Ht, int64_t rows, int64_t V, int64_t num_branches, int W,
                            double count, float* alpha, float* q_less, float* lse_draft, float* lse_teacher,
                            float* loss, float* grad_alpha, float* grad_draft, int64_t ld_grad, void* workspace,
                            size_t workspace_bytes, int32_t* status, specopd_stream_t stream) {
  if (W < 1 || W > SPECOPD_MAX_W || num_branches < 0 || rows != num_branches * W) return SPECOPD_ERR_SHAPE;
  if (V < 1 || V > (1LL << 31) - 256 || Hd < 64 || Ht < 64 || Hd % 64 || Ht % 64 || Hd > (1 << 20) ||
      Ht > (1 << 20) || rows > (1LL << 31) - 128)
    return SPECOPD_ERR_SHAPE;
  if (!loss || !status) return SPECOPD_ERR_ARG;
  if (!(count <= 0.0) && !std::isfinite(count)) return SPECOPD_ERR_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (rows == 0) return cuda_status(cudaMemsetAsync(loss, 0, sizeof(float), st));
  if (!h_draft || !head_draft || !h_teacher || !head_teacher) return SPECOPD_ERR_ARG;
  if (!aligned16(h_draft) || !aligned16(head_draft) || !aligned16(h_teacher) || !aligned16(head_teacher))
    return SPECOPD_ERR_ALIGN;
  if (grad_draft && (ld_grad < V || !aligned16(grad_draft) || (ld_grad * 4) % 16)) return SPECOPD_ERR_ALIGN;
  const LmHeadLayout L = lm_head_layout(rows, V);
  if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) % kAlign))
    return SPECOPD_ERR_WORKSPACE;
  const double n = count > 0.0 ? count : (double)rows;
  LmHeadArgs a;
  a.h_draft = h_draft;
  a.w_draft = head_draft;
  a.h_teacher = h_teacher;
  a.w_teacher = head_teacher;
  a.rows = rows;
  a.V = V;
  a.Hd = Hd;
  a.Ht = Ht;
  a.num_branches = num_branches;
  a.W = W;
  a.inv_count = 1.0 / n;
  a.alpha = alpha;
  a.q_less = q_less;
  a.lse_draft = lse_draft;
  a.lse_teacher = lse_teacher;
  a.loss = loss;
  a.grad_alpha = grad_alpha;
  a.grad_draft = grad_draft;
  a.ld_grad = ld_grad;
  a.workspace = workspace;
  a.status = status;
  return cuda_status(launch_lm_head_overlap(a, st));
}

int specopd_lm_head_shard_phase(int phase, const void* h_draft, const void* head_draft, int Hd, const void* h_teacher,
                                const void* head_teacher, int Ht, int64_t rows, int64_t V_shard, const float* lz2,
                                const float* lt2, const float* q_less, const float* grad_alpha, float* out1,
                                float* out2, int64_t ld_grad, void* workspace, size_t workspace_bytes,
                                int32_t* status, specopd_stream_t stream) {
  if (phase < 0 || phase > 2) return SPECOPD_ERR_ARG;
  if (rows < 0 || V_shard < 1 || V_shard > (1LL << 31) - 256 || Hd < 64 || Ht < 64 || Hd % 64 || Ht % 64 ||
      Hd > (1 << 20) || Ht > (1 << 20) || rows > (1LL << 31) - 128)
    return SPECOPD_ERR_SHAPE;
  if (!status) return SPECOPD_ERR_ARG;
  if (rows == 0) return SPECOPD_OK;
  if (!h_draft || !head_draft || !h_teacher || !head_teacher || !out1) return SPECOPD_ERR_ARG;
  if (phase <= 1 && !out2) return SPECOPD_ERR_ARG;
  if (phase >= 1 && !lz2) return SPECOPD_ERR_ARG;
  if (phase == 1 && !lt2) return SPECOPD_ERR_ARG;
  if (phase == 2 && (!q_less || !grad_alpha)) return SPECOPD_ERR_ARG;
  if (!aligned16(h_draft) || !aligned16(head_draft) || !aligned16(h_teacher) || !aligned16(head_teacher))
    return SPECOPD_ERR_ALIGN;
  if (phase == 2 && (ld_grad < V_shard || !aligned16(out1) || (ld_grad * 4) % 16)) return SPECOPD_ERR_ALIGN;
  const LmHeadLayout L = lm_head_layout(rows, V_shard);
  if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) % kAlign))
    return SPECOPD_ERR_WORKSPACE;
  LmHeadArgs a;
  std::memset(&a, 0, sizeof(a));
  a.h_draft = h_draft;
  a.w_draft = head_draft;
  a.h_teacher = h_teacher;
  a.w_teacher = head_teacher;
  a.rows = rows;
  a.V = V_shard;
  a.Hd = Hd;
  a.Ht = Ht;
  a.ld_grad = ld_grad;
  a.workspace = workspace;
  a.status = status;
  return cuda_status(launch_lm_head_phase(a, phase, lz2, lt2, q_less, grad_alpha, out1, out2,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

int specopd_merge_parts(const float* parts, int nparts, int64_t n, int mode, float* out, specopd_stream_t stream) {
  if (nparts < 1 || n < 0 || (mode != 0 && mode != 1)) return SPECOPD_ERR_ARG;
  if (n == 0) return SPECOPD_OK;
  if (!parts || !out) return SPECOPD_ERR_ARG;
  return cuda_status(launch_merge_parts(parts, nparts, n, mode, out, reinterpret_cast<cudaStream_t>(stream)));
}

const char* specopd_status_string(int status) {
  switch (status) {
    case SPECOPD_OK: return "ok";
    case SPECOPD_ERR_ARG: return "invalid argument";
    case SPECOPD_ERR_SHAPE: return "unsupported shape";
    case SPECOPD_ERR_DTYPE: return "unsupported dtype";
    case SPECOPD_ERR_CUDA: return "CUDA launch failed";
    case SPECOPD_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case SPECOPD_ERR_ALIGN: return "pointer or leading dimension not 16-byte aligned";
    default: return "unknown status";
  }
}

}  // extern "C"
