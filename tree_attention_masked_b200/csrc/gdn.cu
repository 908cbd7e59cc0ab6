// Gated DeltaNet (GDN) linear attention over a proposal tree with indexed
// state replay.
//
// SpecOPD (thelatestinai.com listing), Fig 5: a shared trunk pass caches an
// fp32 GDN state at every C = 64 boundary; in the indexed recurrent kernel
// each CTA copies its state from the checkpoint at or before the branch's
// anchor, replays the cached trunk features up to the anchor (restoring the
// anchor state), then updates the state over the branch's tokens and reads it
// with each token's query; checkpoints stay immutable.  The recurrence (the
// pages name GDN and print no formula; the gated delta rule), per head with
// S in R^{dv x dk}:
//   S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,  o_t = S_t q_t,
// so row i of S evolves on its own:
//   u = S_i . k,  S_i <- alpha S_i + beta (v_i - alpha u) k,  o_i = S_i . q.
// Four threads own a row (32 of its 128 columns each, fp32 in registers) and
// join their partial dot products with two shuffles, in a fixed order.  Each
// token's features (k, q, v, alpha, beta) are staged kGdnDepth tokens ahead
// in a shared-memory ring with cp.async, so a step waits on the arithmetic
// and one CTA barrier rather than on a global load.
//
//   gdn_trunk_kernel  -- one CTA per (tree, head, 32 state rows): the trunk in order; writes
//                        every trunk row's output and the state after tokens
//                        64 j - 1 (the checkpoints);
//   gdn_branch_kernel -- one CTA per (branch, head, 32 state rows): the checkpoint at or
//                        before the anchor, replay to the anchor, then the
//                        branch's rows, writing their outputs.
#include <cuda_bf16.h>

#include "internal.h"

namespace specopd {
namespace {

constexpr int kGdnD = 128;            // dk = dv
constexpr int kGdnTpr = 4;            // threads per state row
constexpr int kGdnCols = kGdnD / kGdnTpr;
constexpr int kGdnRows = 32;           // state rows per CTA: a head's rows spread over kGdnD / kGdnRows CTAs
constexpr int kGdnThreads = kGdnRows * kGdnTpr;
constexpr int kGdnC = 64;             // checkpoint interval

// Features of one token and head in shared memory: k, q, v (bf16, 256 bytes
// each), alpha, beta.
constexpr int kGdnDepth = 16;                  // tokens in flight
constexpr int kGdnFeatBytes = 3 * kGdnD * 2 + 16;
struct GdnRing {
  alignas(16) uint8_t slot[kGdnDepth][kGdnFeatBytes];
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// token r's features of head h into a slot: 48 threads copy 16-byte pieces of
// k, q and v, two more copy alpha and beta
__device__ __forceinline__ void gdn_fetch(uint8_t* slot, const GdnArgs& g, long long r, int h) {
  const int t = threadIdx.x;
  const long long off = (r * g.H + h) * kGdnD;
  if (t < 48) {
    const int which = t >> 4, piece = t & 15;
    const void* src = static_cast<const uint8_t*>(which == 0 ? g.k : which == 1 ? g.q : g.v) + off * 2 + piece * 16;
    cp_async16(slot + which * kGdnD * 2 + piece * 16, src);
  } else if (t == 48) {
    cp_async4(slot + 3 * kGdnD * 2, g.alpha + r * g.H + h);
  } else if (t == 49) {
    cp_async4(slot + 3 * kGdnD * 2 + 4, g.beta + r * g.H + h);
  }
}

__device__ __forceinline__ void unpack16(const uint4 (&w)[kGdnCols / 8], float (&x)[kGdnCols]) {
#pragma unroll
  for (int i = 0; i < kGdnCols / 8; ++i) {
    const uint32_t u[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      x[8 * i + 2 * j] = __uint_as_float(u[j] << 16);
      x[8 * i + 2 * j + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
    }
  }
}

// one token from its slot: update this thread's 32 columns of row `row`,
// return o_row (valid in every thread of the row's quad)
__device__ __forceinline__ float gdn_step(float (&S)[kGdnCols], const uint8_t* slot, int row, int part) {
  uint4 kw[kGdnCols / 8], qw[kGdnCols / 8];
#pragma unroll
  for (int i = 0; i < kGdnCols / 8; ++i) {
    kw[i] = reinterpret_cast<const uint4*>(slot + part * kGdnCols * 2)[i];
    qw[i] = reinterpret_cast<const uint4*>(slot + kGdnD * 2 + part * kGdnCols * 2)[i];
  }
  float k[kGdnCols], q[kGdnCols];
  unpack16(kw, k);
  unpack16(qw, q);
  const float v = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(slot + 2 * kGdnD * 2)[row]);
  const float a = *reinterpret_cast<const float*>(slot + 3 * kGdnD * 2);
  const float b = *reinterpret_cast<const float*>(slot + 3 * kGdnD * 2 + 4);
  float u0 = 0.f, u1 = 0.f, u2 = 0.f, u3 = 0.f;
#pragma unroll
  for (int j = 0; j < kGdnCols; j += 4) {
    u0 = fmaf(S[j], k[j], u0);
    u1 = fmaf(S[j + 1], k[j + 1], u1);
    u2 = fmaf(S[j + 2], k[j + 2], u2);
    u3 = fmaf(S[j + 3], k[j + 3], u3);
  }
  float u = (u0 + u1) + (u2 + u3);
  u += __shfl_xor_sync(0xffffffffu, u, 1);
  u += __shfl_xor_sync(0xffffffffu, u, 2);
  const float c = b * (v - a * u);
  float o0 = 0.f, o1 = 0.f, o2 = 0.f, o3 = 0.f;
#pragma unroll
  for (int j = 0; j < kGdnCols; j += 4) {
    S[j] = fmaf(c, k[j], a * S[j]);
    S[j + 1] = fmaf(c, k[j + 1], a * S[j + 1]);
    S[j + 2] = fmaf(c, k[j + 2], a * S[j + 2]);
    S[j + 3] = fmaf(c, k[j + 3], a * S[j + 3]);
    o0 = fmaf(S[j], q[j], o0);
    o1 = fmaf(S[j + 1], q[j + 1], o1);
    o2 = fmaf(S[j + 2], q[j + 2], o2);
    o3 = fmaf(S[j + 3], q[j + 3], o3);
  }
  float o = (o0 + o1) + (o2 + o3);
  o += __shfl_xor_sync(0xffffffffu, o, 1);
  o += __shfl_xor_sync(0xffffffffu, o, 2);
  return o;
}

// rows r0 .. r1-1 (packed, consecutive) through the recurrence, their
// features staged kGdnDepth tokens ahead in the CTA's ring (one cp.async group
// per token; a slot is refilled only after every thread has passed the next
// step's barrier, so no thread still reads it); outputs of rows >= out_from
// written; with ck non-null a checkpoint after every row whose trunk position
// p has (p + 1) % C == 0.  Every thread of the CTA calls it with the same
// arguments.
__device__ __forceinline__ void gdn_run(float (&S)[kGdnCols], GdnRing* ring, const GdnArgs& g, int h, int row,
                                        int part, long long r0, long long r1, long long out_from, float* ck,
                                        long long ck_pos0) {
  if (r0 >= r1) return;
  __syncthreads();  // the ring may still be read by an earlier call
#pragma unroll 1
  for (int d = 0; d < kGdnDepth - 1; ++d) {
    if (r0 + d < r1) gdn_fetch(ring->slot[(r0 + d) % kGdnDepth], g, r0 + d, h);
    cp_async_commit();
  }
  for (long long r = r0; r < r1; ++r) {
    cp_async_wait<kGdnDepth - 2>();
    __syncthreads();
    const long long rn = r + kGdnDepth - 1;
    if (rn < r1) gdn_fetch(ring->slot[rn % kGdnDepth], g, rn, h);
    cp_async_commit();
    const float o = gdn_step(S, ring->slot[r % kGdnDepth], row, part);
    if (r >= out_from && part == 0) g.out[(r * g.H + h) * kGdnD + row] = o;
    if (ck) {
      const long long p = ck_pos0 + (r - r0);
      if ((p + 1) % kGdnC == 0) {
        float* dst = ck + ((p + 1) / kGdnC - 1) * (long long)g.H * kGdnD * kGdnD + row * kGdnD + part * kGdnCols;
#pragma unroll
        for (int j = 0; j < kGdnCols; j += 4)
          *reinterpret_cast<float4*>(dst + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
      }
    }
  }
  cp_async_wait<0>();
}

__global__ void __launch_bounds__(kGdnThreads) gdn_trunk_kernel(const GdnArgs g) {
  __shared__ GdnRing ring;
  const int t = blockIdx.x, h = blockIdx.y;
  const int row = blockIdx.z * kGdnRows + threadIdx.x / kGdnTpr, part = threadIdx.x % kGdnTpr;
  float S[kGdnCols];
#pragma unroll
  for (int j = 0; j < kGdnCols; ++j) S[j] = 0.f;
  // this tree's checkpoints, head h: [T / C][H][dv][dk] starting at ck_off[t]
  float* ck = g.ckpt + ((long long)g.ck_off[t] * g.H + h) * kGdnD * kGdnD;
  const long long base = g.tp.row_base[t];
  gdn_run(S, &ring, g, h, row, part, base, base + g.tp.trunk_len[t], base, ck, 0);
}

__global__ void __launch_bounds__(kGdnThreads) gdn_branch_kernel(const GdnArgs g) {
  __shared__ GdnRing ring;
  const int gb = blockIdx.x, h = blockIdx.y;
  const int row = blockIdx.z * kGdnRows + threadIdx.x / kGdnTpr, part = threadIdx.x % kGdnTpr;
  int lo = 0, hi = g.tp.num_trees - 1;  // the tree holding global branch gb
  while (lo < hi) {
    const int mid = (lo + hi + 1) / 2;
    if (g.tp.branch_base[mid] <= gb) lo = mid; else hi = mid - 1;
  }
  const int t = lo;
  const int T = g.tp.trunk_len[t], P = g.tp.prompt_len[t];
  int a = g.anchors[gb];
  if (a < P || a > T - 1) {
    if (threadIdx.x == 0) atomicOr(reinterpret_cast<unsigned*>(g.status), SPECOPD_FLAG_ANCHOR);
    a = a < P ? P : T - 1;
  }
  const long long base = g.tp.row_base[t];
  const int c = (a + 1) / kGdnC;  // checkpoints at or before the anchor
  float S[kGdnCols];
  if (c > 0) {
    const float* src = g.ckpt + ((long long)(g.ck_off[t] + c - 1) * g.H + h) * kGdnD * kGdnD + row * kGdnD +
                       part * kGdnCols;
#pragma unroll
    for (int j = 0; j < kGdnCols; j += 4) {
      const float4 x = *reinterpret_cast<const float4*>(src + j);
      S[j] = x.x;
      S[j + 1] = x.y;
      S[j + 2] = x.z;
      S[j + 3] = x.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < kGdnCols; ++j) S[j] = 0.f;
  }
  // replay the trunk from the checkpoint to the anchor (no outputs)
  gdn_run(S, &ring, g, h, row, part, base + (long long)c * kGdnC, base + a + 1, base + a + 1, nullptr, 0);
  // the branch's own rows
  const long long first = base + T + (long long)(gb - g.tp.branch_base[t]) * g.tp.rows_per_branch;
  gdn_run(S, &ring, g, h, row, part, first, first + g.tp.rows_per_branch, first, nullptr, 0);
}

}  // namespace

size_t gdn_checkpoint_floats(const TreeParams& tp, int H) {
  long long n = 0;
  for (int t = 0; t < tp.num_trees; ++t) n += tp.trunk_len[t] / kGdnC;
  return (size_t)n * H * kGdnD * kGdnD;
}

cudaError_t launch_gdn_tree(GdnArgs g, cudaStream_t stream) {
  if (g.tp.num_trees == 0) return cudaSuccess;
  int off = 0;
  for (int t = 0; t < g.tp.num_trees; ++t) {
    g.ck_off[t] = off;
    off += g.tp.trunk_len[t] / kGdnC;
  }
  gdn_trunk_kernel<<<dim3(g.tp.num_trees, g.H, kGdnD / kGdnRows), kGdnThreads, 0, stream>>>(g);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (g.tp.total_branches == 0) return cudaSuccess;
  gdn_branch_kernel<<<dim3(g.tp.total_branches, g.H, kGdnD / kGdnRows), kGdnThreads, 0, stream>>>(g);
  return cudaGetLastError();
}

}  // namespace specopd
