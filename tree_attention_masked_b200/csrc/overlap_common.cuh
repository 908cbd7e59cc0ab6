// Device helpers shared by the overlap kernels: base-2 log-sum-exp merging
// and the per-row E2E-TV epilogue.
#pragma once
#include "internal.h"
#include "ptx.cuh"

namespace specopd {

// atomic add at GPU scope with acquire-release ordering: the caller's earlier
// writes are visible to whoever reads the new count, and writes released by
// earlier adders are visible to the caller
__device__ __forceinline__ unsigned atomic_add_acq_rel(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// load at GPU scope with acquire ordering: writes released before the value
// was stored are visible to the caller's later reads
__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// (m, s) pairs of a base-2 log-sum-exp: value = m + log2(s)
__device__ __forceinline__ void lse_merge(float& m, float& s, float m2, float s2) {
  const float mn = fmaxf(m, m2);
  if (mn == -INFINITY) return;
  s = s * ex2(m - mn) + s2 * ex2(m2 - mn);
  m = mn;
}

// Row results and the E2E-TV epilogue.  Called by one thread per row after
// the row's alpha and q_less are final: writes the per-row outputs, then the
// last row of the branch to arrive forms the branch's prefix products,
// dL/dalpha and its share of L, and the last branch forms L from the shares
// in branch order.
__device__ inline void row_epilogue(const OverlapArgs& a, long long row, float alpha, float qless, float lz2, float lt2) {
  a.alpha[row] = alpha;
  if (a.q_less) a.q_less[row] = qless;
  if (a.lse_draft) a.lse_draft[row] = lz2 * 0.6931471805599453f;
  if (a.lse_teacher) a.lse_teacher[row] = lt2 * 0.6931471805599453f;
  if (a.lz2) a.lz2[row] = lz2;
  if (a.ql) a.ql[row] = qless;
  if (!a.branch_cnt) return;
  const int W = a.W;
  const long long b = row / W;
  // release: this row's alpha precedes the count; acquire for the last row:
  // every other row's alpha is visible to it
  const unsigned old = atomic_add_acq_rel(&a.branch_cnt[b], 1u);
  if (old != (unsigned)(W - 1)) return;
  // the branch's alphas, fetched in batches of independent loads (one L2
  // round trip per batch instead of one per alpha)
  const float* al_b = a.alpha + b * W;
  float al[SPECOPD_MAX_W];
  for (int i0 = 0; i0 < W; i0 += 16) {
    float v[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) v[u] = (i0 + u < W) ? __ldcg(al_b + i0 + u) : 0.f;
#pragma unroll
    for (int u = 0; u < 16; ++u)
      if (i0 + u < W) al[i0 + u] = v[u];
  }
  double pre[SPECOPD_MAX_W + 1];
  pre[0] = 1.0;
  double share = 0.0;
  for (int i = 1; i <= W; ++i) {
    pre[i] = pre[i - 1] * (double)al[i - 1];
    share += pre[i];
  }
  // S_i = 1 + alpha_{i+1} S_{i+1}, S_W = 1; g_i = -(1/count) pre_{i-1} S_i
  double S = 1.0;
  for (int i = W; i >= 1; --i) {
    a.g[b * W + i - 1] = (float)(-a.inv_count * pre[i - 1] * S);
    S = 1.0 + (double)al[i - 1] * S;
  }
  // publish the branch's dL/dalpha: its count becomes W + 1 (release), which
  // gradient warps of the same launch wait for (acquire)
  atomic_add_acq_rel(&a.branch_cnt[b], 1u);
  a.branch_sum[b] = share;
  const unsigned done = atomic_add_acq_rel(&a.branch_cnt[a.num_branches], 1u);
  if (done != (unsigned)(a.num_branches - 1)) return;
  // the shares in branch order (the same additions, in the same order, as one
  // at a time), fetched in batches of independent loads
  double total = 0.0;
  for (long long k0 = 0; k0 < a.num_branches; k0 += 32) {
    double v[32];
#pragma unroll
    for (int u = 0; u < 32; ++u) v[u] = (k0 + u < a.num_branches) ? __ldcg(a.branch_sum + k0 + u) : 0.0;
#pragma unroll
    for (int u = 0; u < 32; ++u)
      if (k0 + u < a.num_branches) total += v[u];
  }
  *a.loss = (float)(1.0 - total * a.inv_count);
}

}  // namespace specopd
