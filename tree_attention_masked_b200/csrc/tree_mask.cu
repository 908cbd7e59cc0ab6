// K1: proposal-tree packing and the compact tree mask.
//
// SpecOPD (thelatestinai.com listing), Fig 2 step 3 and Fig 3; daiwk.github.io
// write-up, section "Equations": trunk token j sits at position j and sees
// trunk tokens 0..j; sample y_{b,i} sits at semantic position a_b + i and sees
// trunk tokens 0..a_b plus y_{b,1..i}; the anchor row predicts y_{b,1} and the
// row of y_{b,i-1} predicts y_{b,i}.
//
// One CTA per 128-row query tile: each thread writes one row's fields and the
// CTA reduces the tile's column ranges for the attention kernel.  The same
// launch also writes the prediction rows (grid-stride over predictions).
#include <climits>

#include "internal.h"

namespace specopd {
namespace {

__device__ __forceinline__ int find_segment(const int32_t* base, int n, int x) {
  // largest t in [0, n) with base[t] <= x (base ascending)
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (base[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ int checked_anchor(const TreeParams& p, const int32_t* anchors, int tree, int gb,
                                              int32_t* status) {
  int a = anchors[gb];
  const int lo = p.prompt_len[tree], hi = p.trunk_len[tree] - 1;
  if (a < lo || a > hi) {
    atomicOr(reinterpret_cast<unsigned*>(status), SPECOPD_FLAG_ANCHOR);
    a = a < lo ? lo : hi;
  }
  return a;
}

__global__ void __launch_bounds__(128) tree_mask_kernel(const TreeParams p, const int32_t* __restrict__ anchors,
                                                        int32_t* __restrict__ pos, int32_t* __restrict__ trunk_limit,
                                                        int32_t* __restrict__ branch_of,
                                                        uint64_t* __restrict__ anc_bits,
                                                        int32_t* __restrict__ pred_rows,
                                                        int32_t* __restrict__ cu_rows,
                                                        specopd_tile_meta* __restrict__ tile_meta,
                                                        int32_t* __restrict__ status) {
  __shared__ int s_hi, s_full, s_blo, s_bhi;
  const int tid = threadIdx.x;

  if (blockIdx.x == 0) {
    for (int t = tid; t <= p.num_trees; t += blockDim.x) cu_rows[t] = p.row_base[t];
  }

  // ---- per-row fields and tile ranges
  const int tile = blockIdx.x;
  if (tile < p.num_tiles) {
    const int tree = find_segment(p.tile_base, p.num_trees, tile);
    const int base = p.row_base[tree];
    const int T = p.trunk_len[tree];
    const int row_start = base + (tile - p.tile_base[tree]) * SPECOPD_TILE_ROWS;
    const int row_end = min(p.row_base[tree + 1], row_start + SPECOPD_TILE_ROWS);
    if (tid == 0) {
      s_hi = INT_MIN;
      s_full = INT_MAX;
      s_blo = INT_MAX;
      s_bhi = INT_MIN;
    }
    __syncthreads();
    const int r = row_start + tid;
    if (r < row_end) {
      const int L = r - base;
      int ps, tl, bo;
      uint64_t bits;
      if (L < T) {
        ps = L;
        tl = L;
        bo = -1;
        bits = 0;
      } else {
        const int bl = (L - T) / p.rows_per_branch;
        const int i = (L - T) - bl * p.rows_per_branch + 1;  // 1-based sample index
        const int gb = p.branch_base[tree] + bl;
        const int a = checked_anchor(p, anchors, tree, gb, status);
        ps = a + i;
        tl = a;
        bo = gb;
        bits = (i >= 64) ? ~0ull : ((1ull << i) - 1ull);
        atomicMin(&s_blo, r - i + 1);
        atomicMax(&s_bhi, r + 1);
      }
      pos[r] = ps;
      trunk_limit[r] = tl;
      branch_of[r] = bo;
      anc_bits[r] = bits;
      atomicMax(&s_hi, base + tl + 1);
      atomicMin(&s_full, base + tl + 1);
    }
    __syncthreads();
    if (tid == 0) {
      specopd_tile_meta m;
      m.row_start = row_start;
      m.row_end = row_end;
      m.tree_base = base;
      m.trunk_hi = s_hi;
      m.trunk_full = s_full;
      if (s_bhi > s_blo) {
        m.br_lo = s_blo;
        m.br_hi = s_bhi;
      } else {
        m.br_lo = 0;
        m.br_hi = 0;
      }
      m.reserved = 0;
      tile_meta[tile] = m;
    }
  }

  // ---- prediction rows: (b, i) is read out at the parent of y_{b,i}
  const long long npred = (long long)p.total_branches * p.W;
  for (long long g = (long long)blockIdx.x * blockDim.x + tid; g < npred; g += (long long)gridDim.x * blockDim.x) {
    const int gb = (int)(g / p.W);
    const int i = (int)(g - (long long)gb * p.W) + 1;
    const int tree = find_segment(p.branch_base, p.num_trees, gb);
    const int base = p.row_base[tree];
    int row;
    if (i == 1) {
      row = base + checked_anchor(p, anchors, tree, gb, status);
    } else {
      const int bl = gb - p.branch_base[tree];
      row = base + p.trunk_len[tree] + bl * p.rows_per_branch + (i - 2);
    }
    pred_rows[g] = row;
  }
}

}  // namespace

cudaError_t launch_tree_mask(const TreeParams& p, const int32_t* anchors, int32_t* pos, int32_t* trunk_limit,
                             int32_t* branch_of, uint64_t* anc_bits, int32_t* pred_rows, int32_t* cu_rows,
                             specopd_tile_meta* tile_meta, int32_t* status, cudaStream_t stream) {
  const long long npred = (long long)p.total_branches * p.W;
  long long blocks = p.num_tiles;
  const long long pred_blocks = (npred + 127) / 128;
  if (pred_blocks > blocks) blocks = pred_blocks;
  if (blocks < 1) blocks = 1;
  tree_mask_kernel<<<(unsigned)blocks, 128, 0, stream>>>(p, anchors, pos, trunk_limit, branch_of, anc_bits,
                                                         pred_rows, cu_rows, tile_meta, status);
  return cudaGetLastError();
}

}  // namespace specopd
