// Sparse attention with branch-consistent indexer groups over a proposal tree.
//
// SpecOPD (thelatestinai.com listing), Fig 4: every row reuses the complete
// trunk group keys; an incomplete boundary group stays in the row's causal
// tail; a group completed by branch tokens needs a branch-specific indexer
// group key; indexer queries select eligible complete groups with top-k, and
// attention reads the selected groups' keys and values plus the causal tail,
// which bypasses top-k.  Readings (the figure prints no formula): groups are
// g consecutive semantic positions of the row's own history (trunk through
// the anchor, then its branch); a complete group's key is the mean of its
// members' indexer keys; the score is the indexer query dotted with it; the
// k best per KV head are taken, ties to the earlier group.
//
//   sparse_gkey_kernel   -- the keys of every complete trunk group (shared by
//                           all rows of the tree): fp32 mean in position order;
//   sparse_bkey_kernel   -- the keys of the complete groups holding branch
//                           tokens, once per branch (members in position order);
//   sparse_select_kernel -- one warp per (row, KV head): scores of the row's
//                           complete groups (trunk keys from the table, one group
//                           per lane with a sequential FMA chain; the branch's
//                           keys with the lanes splitting a key's elements and
//                           a fixed shuffle tree summing the products), top-k by
//                           repeated warp argmax; it
//                           writes the chosen groups as an ascending list and
//                           as bits of the row's selection words;
//   attention            -- for g a multiple of 64, the tcgen05 tree-attention
//                           kernel in its sparse mode (tensor cores; every
//                           query head of the KV group shares the selection);
//                           otherwise sparse_attn_kernel, one warp per (row,
//                           KV head) with an fp32 online softmax over the
//                           chosen groups' members and the tail.
// Scores are fp32 sums and fused multiply-adds in a fixed order, so the
// selection is reproducible.
#include <cuda_bf16.h>

#include "internal.h"

namespace specopd {
namespace {

constexpr int kSpD = 128;             // head dim
constexpr int kSpWarps = 4;           // (row, KV head) items per CTA

struct RowPlace {
  int gb;           // global branch (branch rows)
  int t;            // tree
  long long base;   // first packed row of the tree
  long long bfirst; // first packed row of the branch (branch rows)
  int a;            // last trunk position of the history (the anchor; p itself for trunk rows)
  int p;            // the row's semantic position
};

__device__ __forceinline__ RowPlace place_row(const SparseArgs& s, long long r) {
  int lo = 0, hi = s.tp.num_trees - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) / 2;
    if (s.tp.row_base[mid] <= r) lo = mid; else hi = mid - 1;
  }
  const int t = lo;
  RowPlace x;
  x.t = t;
  x.base = s.tp.row_base[t];
  const int T = s.tp.trunk_len[t], P = s.tp.prompt_len[t], rpb = s.tp.rows_per_branch;
  const long long local = r - x.base;
  if (local < T) {
    x.p = (int)local;
    x.a = x.p;
    x.bfirst = 0;
    x.gb = -1;
  } else {
    const long long bl = (local - T) / rpb;
    const int i = (int)((local - T) % rpb);
    int a = s.anchors[s.tp.branch_base[t] + bl];
    a = a < P ? P : (a > T - 1 ? T - 1 : a);
    x.a = a;
    x.p = a + 1 + i;
    x.bfirst = x.base + T + bl * rpb;
    x.gb = s.tp.branch_base[t] + (int)bl;
  }
  return x;
}

__device__ __forceinline__ long long hist_row(const RowPlace& x, int q) {
  return q <= x.a ? x.base + q : x.bfirst + (q - x.a - 1);
}

__device__ __forceinline__ float ldbf(const __nv_bfloat16* p) { return __bfloat162float(*p); }

__global__ void sparse_gkey_kernel(const SparseArgs s) {
  const int gidx = blockIdx.x, kvh = blockIdx.y, e = threadIdx.x;
  if (e >= s.di) return;
  int t = 0;
  while (t + 1 < s.tp.num_trees && s.gk_off[t + 1] <= gidx) ++t;
  const int m = gidx - s.gk_off[t];
  const long long base = s.tp.row_base[t];
  const __nv_bfloat16* ki = static_cast<const __nv_bfloat16*>(s.ki);
  float sum = 0.f;
  for (int j = 0; j < s.g; ++j) sum += ldbf(ki + ((base + (long long)m * s.g + j) * s.Hkv + kvh) * s.di + e);
  // element-major per (tree, KV head): element e of group m at (kvh di + e) ng + m,
  // so that the lanes of the selection warp, one group each, read consecutive words
  const int ng = s.gk_off[t + 1] - s.gk_off[t];
  s.gkey[(long long)s.gk_off[t] * s.Hkv * s.di + ((long long)kvh * s.di + e) * ng + m] = sum / (float)s.g;
}

// Keys of the complete groups that hold branch tokens, once per (branch, slot,
// KV head): group m0 + slot with m0 = (a + 1) / g, members in position order
// (trunk rows up to the anchor, then the branch's rows), an fp32 sum divided by
// g; every row of the branch that sees the group complete shares its key.
__global__ void sparse_bkey_kernel(const SparseArgs s) {
  const int gb = blockIdx.x / s.bslots, slot = blockIdx.x % s.bslots, kvh = blockIdx.y, e = threadIdx.x;
  if (e >= s.di) return;
  int lo = 0, hi = s.tp.num_trees - 1;  // the tree holding global branch gb
  while (lo < hi) {
    const int mid = (lo + hi + 1) / 2;
    if (s.tp.branch_base[mid] <= gb) lo = mid; else hi = mid - 1;
  }
  const int t = lo;
  const int T = s.tp.trunk_len[t], P = s.tp.prompt_len[t], rpb = s.tp.rows_per_branch;
  int a = s.anchors[gb];
  a = a < P ? P : (a > T - 1 ? T - 1 : a);
  const int m = (a + 1) / s.g + slot;
  if ((long long)m * s.g + s.g - 1 > a + rpb) return;  // no row of the branch sees it complete
  const long long base = s.tp.row_base[t];
  const long long bfirst = base + T + (long long)(gb - s.tp.branch_base[t]) * rpb;
  const __nv_bfloat16* ki = static_cast<const __nv_bfloat16*>(s.ki);
  float sum = 0.f;
  for (int j = 0; j < s.g; ++j) {
    const int q = m * s.g + j;
    const long long row = q <= a ? base + q : bfirst + (q - a - 1);
    sum += ldbf(ki + (row * s.Hkv + kvh) * s.di + e);
  }
  s.bkey[(((long long)gb * s.bslots + slot) * s.Hkv + kvh) * s.di + e] = sum / (float)s.g;
}

__global__ void __launch_bounds__(32 * kSpWarps) sparse_select_kernel(const SparseArgs s) {
  __shared__ float score[kSpWarps][kSpMaxGroups];
  __shared__ int sel[kSpWarps][kSpMaxTopk];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long item = (long long)blockIdx.x * kSpWarps + w;
  if (item >= s.N * s.Hkv) return;
  const long long r = item / s.Hkv;
  const int kvh = (int)(item % s.Hkv);
  const RowPlace x = place_row(s, r);
  const int t = x.t;
  const int nc = (x.p + 1) / s.g;  // complete groups
  const __nv_bfloat16* qi = static_cast<const __nv_bfloat16*>(s.qi) + (r * s.Hkv + kvh) * s.di;

  // ---- indexer scores of the complete groups.  Groups wholly in the trunk
  // part of the history use the shared keys: one group per lane, a sequential
  // fp32 FMA chain over the di products in element order (the query from
  // shared memory).  A group holding branch tokens gets this branch's key:
  // the lanes split its elements (lane + 32 i), sum the members in position
  // order, and a fixed xor-shuffle tree sums the products.
  __shared__ __align__(16) float qsm[kSpWarps][256];
  for (int e = lane; e < s.di; e += 32) qsm[w][e] = ldbf(qi + e);
  __syncwarp();
  const int nct = min(nc, (x.a + 1) / s.g);  // complete groups inside the trunk part
  {
    const int ng = s.gk_off[t + 1] - s.gk_off[t];
    const float* gk0 = s.gkey + (long long)s.gk_off[t] * s.Hkv * s.di + (long long)kvh * s.di * ng;
    for (int m = lane; m < nct; m += 32) {
      const float* col = gk0 + m;  // element e of group m at col[e ng]
      float part = 0.f;
      int e = 0;
#pragma unroll 2
      for (; e + 4 <= s.di; e += 4) {
        const float4 q4 = *reinterpret_cast<const float4*>(&qsm[w][e]);
        part = fmaf(q4.x, col[0], part);
        part = fmaf(q4.y, col[ng], part);
        part = fmaf(q4.z, col[2 * ng], part);
        part = fmaf(q4.w, col[3 * ng], part);
        col += 4 * ng;
      }
      for (; e < s.di; ++e, col += ng) part = fmaf(qsm[w][e], *col, part);
      score[w][m] = part;
    }
  }
  constexpr int kQi = 8;  // di <= 256
  for (int m = nct; m < nc; ++m) {  // groups holding branch tokens: this branch's keys, formed once per branch
    const float* key = s.bkey + (((long long)x.gb * s.bslots + (m - nct)) * s.Hkv + kvh) * s.di;
    float part = 0.f;
#pragma unroll
    for (int i = 0; i < kQi; ++i)
      if (lane + 32 * i < s.di) part = fmaf(qsm[w][lane + 32 * i], key[lane + 32 * i], part);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    if (lane == 0) score[w][m] = part;
  }
  __syncwarp();

  // ---- top-k: repeated warp argmax (higher score, then lower index)
  const int K = nc < s.topk ? nc : s.topk;
  if (nc > s.topk) {
    for (int it = 0; it < K; ++it) {
      float bs = -INFINITY;
      int bm = 0x7fffffff;
      for (int m = lane; m < nc; m += 32) {
        const float v = score[w][m];
        if (v > bs || (v == bs && m < bm)) {
          bs = v;
          bm = m;
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float os = __shfl_xor_sync(0xffffffffu, bs, off);
        const int om = __shfl_xor_sync(0xffffffffu, bm, off);
        if (os > bs || (os == bs && om < bm)) {
          bs = os;
          bm = om;
        }
      }
      if (lane == 0) {
        sel[w][it] = bm;
        score[w][bm] = -INFINITY;
      }
      __syncwarp();
    }
    // groups in ascending order: every lane ranks the choices it holds (the
    // groups are distinct, so the ranks are a permutation)
    __syncwarp();
    const int v0 = lane < K ? sel[w][lane] : 0x7fffffff;
    const int v1 = lane + 32 < K ? sel[w][lane + 32] : 0x7fffffff;
    int r0 = 0, r1 = 0;
    for (int i = 0; i < K; ++i) {
      const int u = sel[w][i];
      r0 += u < v0 ? 1 : 0;
      r1 += u < v1 ? 1 : 0;
    }
    __syncwarp();
    if (lane < K) sel[w][r0] = v0;
    if (lane + 32 < K) sel[w][r1] = v1;
  } else if (lane == 0) {
    for (int i = 0; i < K; ++i) sel[w][i] = i;
  }
  __syncwarp();

  // ---- outputs: the ascending list (-1 past K) and the selection words
  int32_t* list = s.sel_list + item * s.topk;
  for (int i = lane; i < s.topk; i += 32) {
    const int v = i < K ? sel[w][i] : -1;
    list[i] = v;
    if (s.sel_out) s.sel_out[item * s.topk + i] = v;
  }
  uint32_t* words = s.sel_mask + item * s.sel_words;
  for (int wd = lane; wd < s.sel_words; wd += 32) {
    uint32_t bits = 0;
    for (int i = 0; i < K; ++i) {
      const int m = sel[w][i];
      if ((m >> 5) == wd) bits |= 1u << (m & 31);
    }
    words[wd] = bits;
  }
}

// fp32 SIMT attention over the chosen groups' members and the tail (group
// sizes that are not a multiple of 64).
__global__ void __launch_bounds__(32 * kSpWarps) sparse_attn_kernel(const SparseArgs s) {
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long item = (long long)blockIdx.x * kSpWarps + w;
  if (item >= s.N * s.Hkv) return;
  const long long r = item / s.Hkv;
  const int kvh = (int)(item % s.Hkv);
  const RowPlace x = place_row(s, r);
  const int nc = (x.p + 1) / s.g;
  const int tail0 = nc * s.g;
  const int K = nc < s.topk ? nc : s.topk;
  const int32_t* sel = s.sel_list + item * s.topk;
  const int ncols = K * s.g + (x.p + 1 - tail0);
  const __nv_bfloat16* rq = static_cast<const __nv_bfloat16*>(s.rq);
  const __nv_bfloat16* rk = static_cast<const __nv_bfloat16*>(s.rk);
  const __nv_bfloat16* vv = static_cast<const __nv_bfloat16*>(s.v);
  const int G = s.Hq / s.Hkv;
  for (int hh = 0; hh < G; ++hh) {
    const int h = kvh * G + hh;
    float qv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) qv[i] = ldbf(rq + (r * s.Hq + h) * kSpD + lane * 4 + i) * s.scale_log2;
    float mx = -INFINITY, l = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
    for (int c = 0; c < ncols; ++c) {
      const int q = c < K * s.g ? sel[c / s.g] * s.g + c % s.g : tail0 + (c - K * s.g);
      const long long col = hist_row(x, q);
      const __nv_bfloat16* kp = rk + (col * s.Hkv + kvh) * kSpD + lane * 4;
      float d = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) d = fmaf(qv[i], ldbf(kp + i), d);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
      const float mn = fmaxf(mx, d);
      const float corr = exp2f(mx - mn), pw = exp2f(d - mn);
      l = l * corr + pw;
      const __nv_bfloat16* vp = vv + (col * s.Hkv + kvh) * kSpD + lane * 4;
#pragma unroll
      for (int i = 0; i < 4; ++i) o[i] = fmaf(pw, ldbf(vp + i), o[i] * corr);
      mx = mn;
    }
    __nv_bfloat16* op = static_cast<__nv_bfloat16*>(s.out) + (r * s.Hq + h) * kSpD + lane * 4;
#pragma unroll
    for (int i = 0; i < 4; ++i) op[i] = __float2bfloat16(o[i] / l);
  }
}

}  // namespace

size_t sparse_group_keys(const TreeParams& tp, int g) {
  size_t n = 0;
  for (int t = 0; t < tp.num_trees; ++t) n += (size_t)(tp.trunk_len[t] / g);
  return n;
}

int sparse_selection_words(const TreeParams& tp, int g) {
  int most = 0;
  for (int t = 0; t < tp.num_trees; ++t) {
    const int n = (tp.trunk_len[t] + tp.rows_per_branch) / g;  // complete groups of the deepest row
    if (n > most) most = n;
  }
  return (most + 31) / 32 > 0 ? (most + 31) / 32 : 1;
}

cudaError_t launch_sparse_attention(SparseArgs s, cudaStream_t stream) {
  int off = 0;
  for (int t = 0; t < s.tp.num_trees; ++t) {
    s.gk_off[t] = off;
    off += s.tp.trunk_len[t] / s.g;
  }
  s.gk_off[s.tp.num_trees] = off;
  cudaError_t e = launch_rope(s.q, s.k, s.rq, s.rk, SPECOPD_BF16, s.N, s.Hq, s.Hkv, kSpD, s.pos, s.theta, stream);
  if (e != cudaSuccess) return e;
  if (off > 0) {
    sparse_gkey_kernel<<<dim3(off, s.Hkv), (s.di + 31) / 32 * 32, 0, stream>>>(s);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (s.tp.total_branches > 0 && s.tp.rows_per_branch > 0) {
    sparse_bkey_kernel<<<dim3(s.tp.total_branches * s.bslots, s.Hkv), (s.di + 31) / 32 * 32, 0, stream>>>(s);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const long long items = s.N * s.Hkv;
  const unsigned blocks = (unsigned)((items + kSpWarps - 1) / kSpWarps);
  sparse_select_kernel<<<blocks, 32 * kSpWarps, 0, stream>>>(s);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (s.g % 64 == 0) {
    AttnArgs a;
    a.q = s.rq;
    a.k = s.rk;
    a.v = s.v;
    a.out = s.out;
    a.N = s.N;
    a.Hq = s.Hq;
    a.Hkv = s.Hkv;
    a.d = kSpD;
    a.scale = s.scale;
    a.pos = s.pos;
    a.trunk_limit = s.trunk_limit;
    a.anc_bits = s.anc_bits;
    a.meta = s.meta;
    a.num_tiles = s.num_tiles;
    a.status = s.status;
    SparseSel sel{s.sel_mask, s.sel_words, s.g};
    return launch_tree_attention_sm100(a, stream, &sel);
  }
  sparse_attn_kernel<<<blocks, 32 * kSpWarps, 0, stream>>>(s);
  return cudaGetLastError();
}

}  // namespace specopd
