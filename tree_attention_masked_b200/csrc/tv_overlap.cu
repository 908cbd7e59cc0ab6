// K4/K5: full-vocabulary overlap, E2E-TV loss and its gradient -- the generic
// kernels, used for fp32 logits (bf16 logits take the kernels in tv_bf16.cu).
//
// daiwk.github.io write-up of SpecOPD, section "Equations":
//   alpha_{b,i} = sum_v min(q(v), p(v)),
//   L = 1 - (1/(B W)) sum_b sum_j prod_{i<=j} alpha_{b,i},
// samples and teacher fixed during differentiation, teacher mass outside the
// draft support kept.  Section "Inputs and code mapping": NaN padding marks
// inactive draft entries, the teacher must be finite, bf16 work promotes to fp32.
//
// Statistics kernel (one thread-block cluster per prediction row):
//   the row's V logits of draft and teacher are split over the C CTAs of the
//   cluster and bulk-copied (cp.async.bulk, no multicast) into shared memory,
//   where they stay for the whole row:
//   pass 1  online max/sum of both softmaxes in base 2 (one exp per element);
//           the C partials combine through distributed shared memory in rank
//           order, so every CTA holds identical normalisers;
//   pass 2  alpha = sum exp2(min(z2 - lz2, t2 - lt2)), q_less = the part where
//           the draft side is strictly smaller (one exp per element), and one
//           bit per element recording that comparison for the gradient pass.
//   The last row of a branch to finish (per-branch arrival counter) forms the
//   branch's prefix products, dL/dalpha (division-free: prefix products times
//   suffix sums) and its share of L; the last branch sums the shares in branch
//   order, so L is bitwise reproducible.
// Gradient kernel: streams the draft logits and the bits once more and writes
//   dL/dz = g q (bit - q_less), zero outside the draft support.
#include <cuda_bf16.h>

#include <type_traits>

#include "internal.h"
#include "overlap_common.cuh"
#include "ptx.cuh"

namespace specopd {
namespace {

constexpr int kStatThreads = 256;
constexpr int kChunkElems = 4096;
constexpr int kMaxChunks = 32;
constexpr float kLog2e = 1.4426950408889634f;

template <typename T>
struct Elem;
template <>
struct Elem<float> {
  // 8 consecutive values from 16-byte aligned shared/global memory
  __device__ static void load8(const float* p, float (&x)[8]) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    const float4 b = *reinterpret_cast<const float4*>(p + 4);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
  __device__ static float one(const float* p) { return *p; }
};
struct StatSmem {
  float part[8];      // this CTA's partials, read by the cluster
  float bcast[4];
  float warp_red[kStatThreads / 32][4];
  int bad;
  int abort_flag;
};

template <typename T>
__global__ void __launch_bounds__(kStatThreads) tv_stats_kernel(const OverlapArgs a, int C, int seg_len) {
  extern __shared__ __align__(128) uint8_t smem[];
  T* zb = reinterpret_cast<T*>(smem);
  T* tb = zb + seg_len;
  uint64_t* bars = reinterpret_cast<uint64_t*>(tb + seg_len);
  StatSmem* ss = reinterpret_cast<StatSmem*>(bars + kMaxChunks);

  const int tid = threadIdx.x;
  const int rank = (int)cluster_ctarank();
  const long long row = blockIdx.x / C;
  const long long s0 = (long long)rank * seg_len;
  const long long s1 = min((long long)a.V, s0 + seg_len);
  const int len = (int)max(0LL, s1 - s0);
  const T* zrow = static_cast<const T*>(a.draft) + row * a.ld_draft + s0;
  const T* trow = static_cast<const T*>(a.teacher) + row * a.ld_teacher + s0;
  const int nch = (len + kChunkElems - 1) / kChunkElems;
  // elements copied in bulk (whole 16-byte units); the rest are loaded directly
  const int bulk_len = (int)(((long long)len * sizeof(T)) / 16 * 16 / sizeof(T));

  if (tid == 0) {
    for (int c = 0; c < nch; ++c) mbar_init(&bars[c], 1);
    ss->bad = 0;
    ss->abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0) {
    for (int c = 0; c < nch; ++c) {
      const int e0 = c * kChunkElems;
      const int e1 = min(bulk_len, e0 + kChunkElems);
      const uint32_t bytes = e1 > e0 ? (uint32_t)((e1 - e0) * sizeof(T)) : 0u;
      if (bytes) {
        mbar_arrive_expect_tx(&bars[c], 2 * bytes);
        bulk_g2s(zb + e0, zrow + e0, bytes, &bars[c]);
        bulk_g2s(tb + e0, trow + e0, bytes, &bars[c]);
      } else {
        mbar_arrive(&bars[c]);
      }
    }
  }
  for (int e = bulk_len + tid; e < len; e += kStatThreads) {
    zb[e] = zrow[e];
    tb[e] = trow[e];
  }
  __syncthreads();

  // ---------------- pass 1: base-2 log-sum-exp of draft (active) and teacher
  float mz = -INFINITY, sz = 0.f, mt = -INFINITY, st = 0.f;
  int bad = 0;
  volatile int* abort_flag = &ss->abort_flag;
  for (int c = 0; c < nch; ++c) {
    if (!mbar_wait(&bars[c], 0, abort_flag)) break;
    const int e0 = c * kChunkElems;
    const int e1 = min(len, e0 + kChunkElems);
    float cz = -INFINITY, ct = -INFINITY;
    for (int g = e0 + tid * 8; g < e1; g += kStatThreads * 8) {
      float z[8], t[8];
      if (g + 8 <= e1) {
        Elem<T>::load8(zb + g, z);
        Elem<T>::load8(tb + g, t);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          z[i] = g + i < e1 ? Elem<T>::one(zb + g + i) : -INFINITY;
          t[i] = g + i < e1 ? Elem<T>::one(tb + g + i) : -INFINITY;
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (g + i >= e1) continue;
        if (!(fabsf(t[i]) < INFINITY)) bad = 1;              // NaN or inf teacher
        if (z[i] == INFINITY) bad = 1;
        if (z[i] == z[i] && z[i] != -INFINITY) cz = fmaxf(cz, z[i]);
        ct = fmaxf(ct, t[i]);
      }
    }
    // rescale the running sums once per chunk, then one exp per element
    const float nmz = fmaxf(mz, cz * kLog2e), nmt = fmaxf(mt, ct * kLog2e);
    if (nmz != -INFINITY) sz = (mz == -INFINITY) ? 0.f : sz * ex2(mz - nmz);
    if (nmt != -INFINITY) st = (mt == -INFINITY) ? 0.f : st * ex2(mt - nmt);
    mz = nmz;
    mt = nmt;
    for (int g = e0 + tid * 8; g < e1; g += kStatThreads * 8) {
      float z[8], t[8];
      const bool full = g + 8 <= e1;
      if (full) {
        Elem<T>::load8(zb + g, z);
        Elem<T>::load8(tb + g, t);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (!full) {
          if (g + i >= e1) continue;
          z[i] = Elem<T>::one(zb + g + i);
          t[i] = Elem<T>::one(tb + g + i);
        }
        if (z[i] == z[i] && fabsf(z[i]) != INFINITY) sz += ex2(fmaf(z[i], kLog2e, -mz));
        if (fabsf(t[i]) < INFINITY) st += ex2(fmaf(t[i], kLog2e, -mt));
      }
    }
  }
  // block reduce (fixed shuffle tree, then warps in order)
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    lse_merge(mz, sz, __shfl_xor_sync(0xffffffffu, mz, off), __shfl_xor_sync(0xffffffffu, sz, off));
    lse_merge(mt, st, __shfl_xor_sync(0xffffffffu, mt, off), __shfl_xor_sync(0xffffffffu, st, off));
  }
  if (bad) atomicOr(&ss->bad, 1);
  const int warp = tid >> 5, lane = tid & 31;
  if (lane == 0) {
    ss->warp_red[warp][0] = mz;
    ss->warp_red[warp][1] = sz;
    ss->warp_red[warp][2] = mt;
    ss->warp_red[warp][3] = st;
  }
  __syncthreads();
  if (tid == 0) {
    float m1 = -INFINITY, s1v = 0.f, m2 = -INFINITY, s2v = 0.f;
    for (int w = 0; w < kStatThreads / 32; ++w) {
      lse_merge(m1, s1v, ss->warp_red[w][0], ss->warp_red[w][1]);
      lse_merge(m2, s2v, ss->warp_red[w][2], ss->warp_red[w][3]);
    }
    ss->part[0] = m1;
    ss->part[1] = s1v;
    ss->part[2] = m2;
    ss->part[3] = s2v;
  }
  cluster_sync();
  if (tid == 0) {
    float m1 = -INFINITY, s1v = 0.f, m2 = -INFINITY, s2v = 0.f;
    const uint32_t base = smem_u32(&ss->part[0]);
    for (int q = 0; q < C; ++q) {
      const uint32_t ra = map_cluster(base, q);
      lse_merge(m1, s1v, ld_cluster_f32(ra), ld_cluster_f32(ra + 4));
      lse_merge(m2, s2v, ld_cluster_f32(ra + 8), ld_cluster_f32(ra + 12));
    }
    ss->bcast[0] = (s1v > 0.f) ? m1 + log2f(s1v) : -INFINITY;  // lz2 (-inf: empty support)
    ss->bcast[1] = m2 + log2f(s2v);                             // lt2
  }
  __syncthreads();
  const float lz2 = ss->bcast[0];
  const float lt2 = ss->bcast[1];

  // ---------------- pass 2: alpha, q_less and the strict-less bits
  float al = 0.f, ql = 0.f;
  uint8_t* mrow = a.mbits ? a.mbits + row * a.mbits_ld + s0 / 8 : nullptr;
  for (int g = tid * 8; g < len; g += kStatThreads * 8) {
    float z[8], t[8];
    const bool full = g + 8 <= len;
    if (full) {
      Elem<T>::load8(zb + g, z);
      Elem<T>::load8(tb + g, t);
    }
    uint32_t byte = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (!full) {
        if (g + i >= len) continue;
        z[i] = Elem<T>::one(zb + g + i);
        t[i] = Elem<T>::one(tb + g + i);
      }
      if (z[i] == z[i] && fabsf(z[i]) != INFINITY && lz2 != -INFINITY) {
        const float da = fmaf(z[i], kLog2e, -lz2);
        const float db = fmaf(t[i], kLog2e, -lt2);
        const float e = ex2(fminf(da, db));
        al += e;
        if (da < db) {
          ql += e;
          byte |= 1u << i;
        }
      }
    }
    if (mrow) mrow[g >> 3] = (uint8_t)byte;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    al += __shfl_xor_sync(0xffffffffu, al, off);
    ql += __shfl_xor_sync(0xffffffffu, ql, off);
  }
  if (lane == 0) {
    ss->warp_red[warp][0] = al;
    ss->warp_red[warp][1] = ql;
  }
  __syncthreads();
  if (tid == 0) {
    float x = 0.f, y = 0.f;
    for (int w = 0; w < kStatThreads / 32; ++w) {
      x += ss->warp_red[w][0];
      y += ss->warp_red[w][1];
    }
    ss->part[4] = x;
    ss->part[5] = y;
    ss->part[6] = (float)(ss->bad | (ss->abort_flag ? 2 : 0));
  }
  cluster_sync();
  if (rank == 0 && tid == 0) {
    float x = 0.f, y = 0.f;
    int flags = 0;
    const uint32_t base = smem_u32(&ss->part[0]);
    for (int q = 0; q < C; ++q) {
      const uint32_t ra = map_cluster(base, q);
      x += ld_cluster_f32(ra + 16);
      y += ld_cluster_f32(ra + 20);
      flags |= (int)ld_cluster_f32(ra + 24);
    }
    if (flags & 1) atomicOr(reinterpret_cast<unsigned*>(a.status), SPECOPD_FLAG_NONFINITE);
    if (flags & 2) atomicOr(reinterpret_cast<unsigned*>(a.status), SPECOPD_FLAG_TIMEOUT);
    row_epilogue(a, row, x, y, lz2, lt2);
  }
  // keep this CTA's shared memory alive until rank 0 has read it, and make
  // sure no bulk copy into it is still in flight (matters only after a timeout)
  if (tid == 0 && ss->abort_flag) {
    for (int c = 0; c < nch; ++c) {
      const long long t0 = clock64();
      while (!mbar_try_wait(&bars[c], 0) && clock64() - t0 < kWaitLimitCycles) {
      }
    }
  }
  cluster_sync();
}

// ---------------- gradient: dL/dz = g q (bit - q_less)
template <typename T>
__global__ void __launch_bounds__(256) tv_grad_kernel(const OverlapArgs a, int bx) {
  const long long row = blockIdx.x / bx;
  const int bxi = blockIdx.x - (int)(row * bx);
  const float L2 = a.lz2[row];
  const float Q = a.ql[row];
  const float G = a.g[row];
  const T* zrow = static_cast<const T*>(a.draft) + row * a.ld_draft;
  const uint8_t* mrow = a.mbits + row * a.mbits_ld;
  float* grow = a.grad + row * a.ld_grad;
  const long long groups = (a.V + 7) / 8;
  for (long long gi = (long long)bxi * blockDim.x + threadIdx.x; gi < groups; gi += (long long)bx * blockDim.x) {
    const long long e0 = gi * 8;
    const uint32_t byte = mrow[gi];
    float z[8], out[8];
    const bool full = e0 + 8 <= a.V;
    if (full) {
      Elem<T>::load8(zrow + e0, z);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) z[i] = e0 + i < a.V ? Elem<T>::one(zrow + e0 + i) : -INFINITY;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const bool active = z[i] == z[i] && fabsf(z[i]) != INFINITY && L2 != -INFINITY;
      const float q = active ? ex2(fmaf(z[i], kLog2e, -L2)) : 0.f;
      out[i] = G * q * ((float)((byte >> i) & 1u) - Q);
    }
    if (full) {
      __stcs(reinterpret_cast<float4*>(grow + e0), make_float4(out[0], out[1], out[2], out[3]));
      __stcs(reinterpret_cast<float4*>(grow + e0 + 4), make_float4(out[4], out[5], out[6], out[7]));
    } else {
      for (int i = 0; i < 8 && e0 + i < a.V; ++i) grow[e0 + i] = out[i];
    }
  }
}

// ---------------- unfused loss from alpha
__global__ void __launch_bounds__(1024) e2e_loss_kernel(const float* __restrict__ alpha, long long nb, int W,
                                                        double inv_count, float* loss, float* grad_alpha) {
  __shared__ double red[1024];
  double share = 0.0;
  for (long long b = threadIdx.x; b < nb; b += blockDim.x) {
    const float* al = alpha + b * W;
    double pre[SPECOPD_MAX_W + 1];
    pre[0] = 1.0;
    for (int i = 1; i <= W; ++i) {
      pre[i] = pre[i - 1] * (double)al[i - 1];
      share += pre[i];
    }
    if (grad_alpha) {
      double S = 1.0;
      for (int i = W; i >= 1; --i) {
        grad_alpha[b * W + i - 1] = (float)(-inv_count * pre[i - 1] * S);
        S = 1.0 + (double)al[i - 1] * S;
      }
    }
  }
  red[threadIdx.x] = share;
  __syncthreads();
  for (int s = blockDim.x / 2; s > 0; s >>= 1) {
    if ((int)threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) *loss = (nb == 0) ? 0.f : (float)(1.0 - red[0] * inv_count);
}

// Cluster size: the smallest C in {1,2,4,8,16} whose per-CTA share of the
// row (draft + teacher) fits `target` bytes, so several CTAs fit on an SM.
int pick_cluster(long long V, size_t elem, size_t extra, size_t target, int* seg_len, size_t* smem_bytes) {
  const int choices[5] = {1, 2, 4, 8, 16};
  for (int i = 0; i < 5; ++i) {
    const int C = choices[i];
    long long seg = (V + C - 1) / C;
    seg = (seg + 7) / 8 * 8;
    const size_t bytes = 2 * (size_t)seg * elem + kMaxChunks * 8 + extra + 128;
    if ((bytes <= target || C == 16) && seg <= (long long)kChunkElems * kMaxChunks) {
      if (bytes > 227 * 1024) return 0;
      *seg_len = (int)seg;
      *smem_bytes = bytes;
      return C;
    }
  }
  return 0;
}

template <typename K>
cudaError_t launch_cluster(K kernel, const OverlapArgs& a, int C, int seg_len, size_t smem, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (C > 8) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.rows * C), 1, 1);
  cfg.blockDim = dim3(kStatThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kernel, a, C, seg_len);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_stats_t(const OverlapArgs& a, cudaStream_t stream) {
  int seg_len = 0;
  size_t smem = 0;
  const int C = pick_cluster(a.V, sizeof(T), sizeof(StatSmem), 100 * 1024, &seg_len, &smem);
  if (C == 0) return cudaErrorInvalidValue;
  return launch_cluster(tv_stats_kernel<T>, a, C, seg_len, smem, stream);
}

template <typename T>
cudaError_t launch_grad_t(const OverlapArgs& a, cudaStream_t stream) {
  const long long groups = (a.V + 7) / 8;
  long long bx = (groups + 256 * 4 - 1) / (256 * 4);
  if (bx < 1) bx = 1;
  tv_grad_kernel<T><<<(unsigned)(bx * a.rows), 256, 0, stream>>>(a, (int)bx);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_tv_stats(const OverlapArgs& a, specopd_dtype dtype, cudaStream_t stream) {
  if (a.rows == 0) return cudaSuccess;
  return dtype == SPECOPD_BF16 ? launch_tv_stats_bf16(a, stream) : launch_stats_t<float>(a, stream);
}

// fp32 gradient (the bf16 gradient runs inside launch_tv_fused_bf16)
cudaError_t launch_tv_grad(const OverlapArgs& a, specopd_dtype dtype, cudaStream_t stream) {
  if (a.rows == 0) return cudaSuccess;
  return dtype == SPECOPD_BF16 ? cudaErrorInvalidValue : launch_grad_t<float>(a, stream);
}

cudaError_t launch_e2e_loss(const float* alpha, int64_t num_branches, int W, double inv_count, float* loss,
                            float* grad_alpha, cudaStream_t stream) {
  e2e_loss_kernel<<<1, 1024, 0, stream>>>(alpha, num_branches, W, inv_count, loss, grad_alpha);
  return cudaGetLastError();
}

}  // namespace specopd
