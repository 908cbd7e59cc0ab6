// K4/K5 for bf16 logits: per-row overlap statistics (cluster kernel) and the
// streaming gradient.
//
// daiwk.github.io write-up of SpecOPD, section "Equations": alpha = sum_v
// min(q(v), p(v)); L = 1 - (1/(B W)) sum_b sum_j prod_{i<=j} alpha_{b,i};
// teacher and samples fixed during differentiation; teacher mass outside the
// draft support kept.  Section "Inputs and code mapping": NaN padding marks
// inactive draft entries, the teacher must be finite, bf16 work promotes to fp32.
//
// Statistics: one thread-block cluster of C CTAs per prediction row, the row's
// draft and teacher logits split over the CTAs and bulk-copied (no multicast)
// into shared memory, where they stay for both passes.  The per-row latency
// (load -> pass 1 -> exchange -> pass 2 -> exchange) bounds the bandwidth
// (bytes in flight / latency), so the chain is kept short:
//   * copies are issued before the cluster start barrier, whose wait is
//     deferred until after pass 1;
//   * pass 1 is a single online base-2 (max, sum) pass over packed bf16x2
//     data as the copy chunks land;
//   * every CTA pushes its partials into the shared memory of the CTAs that
//     need them before a cluster barrier, so all reads after it are local and
//     CTAs other than rank 0 exit right after the second barrier;
//   * reductions use fixed shuffle trees, so every CTA derives bitwise
//     identical normalisers and the results are reproducible run to run.
// Gradient: dL/dz = g q ([q < p] - q_less) from the draft logits and the bits
// written by pass 2; every warp access is contiguous.
#include <cuda_bf16.h>

#include "internal.h"
#include "overlap_common.cuh"
#include "ptx.cuh"

namespace specopd {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kChunkElems = 4096;
constexpr int kMaxChunks = 32;
constexpr int kMaxCluster = 16;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kNegInf2 = 0xFF80FF80u;  // two bf16 -inf

__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bmin2_nan(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("min.NaN.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ bool nonfinite(float x) { return !(fabsf(x) < INFINITY); }

__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }
__device__ __forceinline__ void st_cluster_v4(uint32_t caddr, float a, float b, float c, float d) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(caddr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}
// try_wait that lets the hardware suspend the thread for up to `ns`
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const long long t0 = clock64();
  while (!mbar_try_wait_sleep(bar, parity, 20000u)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitLimitCycles) {
      *abort_flag = 1;
      return false;
    }
  }
  return true;
}

struct Smem {
  float lse_in[kMaxCluster][4];  // (mz, sz, mt, st) pushed by each CTA of the cluster, by rank
  float al_in[kMaxCluster][4];   // (alpha, q_less, flags) pushed to rank 0, by rank
  float red[kWarps][4];
  float bcast[2];
  int bad;
  int abort_flag;
};

__global__ void __launch_bounds__(kThreads) tv_stats_bf16_kernel(const OverlapArgs a, int C, int seg_len) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint32_t* zb = reinterpret_cast<uint32_t*>(smem);  // bf16 pairs
  uint32_t* tb = zb + seg_len / 2;
  uint64_t* bars = reinterpret_cast<uint64_t*>(tb + seg_len / 2);
  Smem* ss = reinterpret_cast<Smem*>(bars + kMaxChunks);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rank = (int)cluster_ctarank();
  const long long row = blockIdx.x / C;
  const long long s0 = (long long)rank * seg_len;
  const int len = (int)max(0LL, min((long long)a.V, s0 + seg_len) - s0);
  const int len8 = len & ~7;
  const int tail = len - len8;
  const int nch = (len8 + kChunkElems - 1) / kChunkElems;
  const __nv_bfloat16* zrow = static_cast<const __nv_bfloat16*>(a.draft) + row * a.ld_draft + s0;
  const __nv_bfloat16* trow = static_cast<const __nv_bfloat16*>(a.teacher) + row * a.ld_teacher + s0;

  if (tid == 0) {
    for (int c = 0; c < nch; ++c) mbar_init(&bars[c], 1);
    ss->bad = 0;
    ss->abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0) {
    for (int c = 0; c < nch; ++c) {
      const int e0 = c * kChunkElems, e1 = min(len8, e0 + kChunkElems);
      const uint32_t bytes = (uint32_t)(e1 - e0) * 2u;
      mbar_arrive_expect_tx(&bars[c], 2 * bytes);
      bulk_g2s(zb + e0 / 2, zrow + e0, bytes, &bars[c]);
      bulk_g2s(tb + e0 / 2, trow + e0, bytes, &bars[c]);
    }
  }
  cluster_arrive_relaxed();  // every CTA of the cluster has started (waited below)
  volatile int* abort_flag = &ss->abort_flag;

  // ---- pass 1: online base-2 log-sum-exp of draft (active) and teacher
  float mz = -INFINITY, sz = 0.f, mt = -INFINITY, st = 0.f;
  uint32_t tmn = 0u;  // NaN-aware running min of the teacher: NaN or -inf wins
  const float2 l2e = make_float2(kLog2e, kLog2e);
  for (int c = 0; c < nch; ++c) {
    if (!mbar_wait_sleep(&bars[c], 0, abort_flag)) break;
    const int g1 = min(len8, (c + 1) * kChunkElems) / 8;
    for (int g = c * (kChunkElems / 8) + tid; g < g1; g += kThreads) {
      const uint4 zw = reinterpret_cast<const uint4*>(zb)[g];
      const uint4 tw = reinterpret_cast<const uint4*>(tb)[g];
      const uint32_t zm = bmax2(bmax2(zw.x, zw.y), bmax2(zw.z, zw.w));
      const uint32_t tm = bmax2(bmax2(tw.x, tw.y), bmax2(tw.z, tw.w));
      tmn = bmin2_nan(tmn, bmin2_nan(bmin2_nan(tw.x, tw.y), bmin2_nan(tw.z, tw.w)));
      const float gz = fmaxf(bf_lo(zm), bf_hi(zm)) * kLog2e;
      const float gt = fmaxf(bf_lo(tm), bf_hi(tm)) * kLog2e;
      if (gz > mz) {
        sz *= ex2(mz - gz);
        mz = gz;
      }
      if (gt > mt) {
        st *= ex2(mt - gt);
        mt = gt;
      }
      const float mze = (mz == -INFINITY) ? 0.f : mz;
      const float2 nmz = make_float2(-mze, -mze), nmt = make_float2(-mt, -mt);
      const uint32_t zs[4] = {zw.x, zw.y, zw.z, zw.w};
      const uint32_t ts[4] = {tw.x, tw.y, tw.z, tw.w};
      float2 az = make_float2(0.f, 0.f), at = make_float2(0.f, 0.f);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t zc = bmax2(zs[k], kNegInf2);  // NaN (inactive) -> -inf -> adds 0
        const float2 ea = __ffma2_rn(make_float2(bf_lo(zc), bf_hi(zc)), l2e, nmz);
        const float2 eb = __ffma2_rn(make_float2(bf_lo(ts[k]), bf_hi(ts[k])), l2e, nmt);
        az = __fadd2_rn(az, make_float2(ex2(ea.x), ex2(ea.y)));
        at = __fadd2_rn(at, make_float2(ex2(eb.x), ex2(eb.y)));
      }
      sz += az.x + az.y;
      st += at.x + at.y;
    }
  }
  bool bad = nonfinite(bf_lo(tmn)) || nonfinite(bf_hi(tmn)) || mz == INFINITY || mt == INFINITY;
  float ztail = -INFINITY, ttail = 0.f;
  if (tid < tail) {  // fewer than 8 logits at the very end of the row
    ztail = __bfloat162float(zrow[len8 + tid]);
    ttail = __bfloat162float(trow[len8 + tid]);
    bad |= nonfinite(ttail) || ztail == INFINITY;
    if (ztail == ztail && ztail != -INFINITY) lse_merge(mz, sz, ztail * kLog2e, 1.f);
    lse_merge(mt, st, ttail * kLog2e, 1.f);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float om1 = __shfl_xor_sync(0xffffffffu, mz, off), os1 = __shfl_xor_sync(0xffffffffu, sz, off);
    const float om2 = __shfl_xor_sync(0xffffffffu, mt, off), os2 = __shfl_xor_sync(0xffffffffu, st, off);
    lse_merge(mz, sz, om1, os1);
    lse_merge(mt, st, om2, os2);
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) ss->bad = 1;
  if (lane == 0) {
    ss->red[warp][0] = mz;
    ss->red[warp][1] = sz;
    ss->red[warp][2] = mt;
    ss->red[warp][3] = st;
  }
  __syncthreads();
  cluster_wait();  // all CTAs have started: remote shared memory may be written
  if (warp == 0) {
    float m1 = -INFINITY, s1 = 0.f, m2 = -INFINITY, s2 = 0.f;
    if (lane < kWarps) {
      m1 = ss->red[lane][0];
      s1 = ss->red[lane][1];
      m2 = ss->red[lane][2];
      s2 = ss->red[lane][3];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float o1 = __shfl_xor_sync(0xffffffffu, m1, off), p1 = __shfl_xor_sync(0xffffffffu, s1, off);
      const float o2 = __shfl_xor_sync(0xffffffffu, m2, off), p2 = __shfl_xor_sync(0xffffffffu, s2, off);
      lse_merge(m1, s1, o1, p1);
      lse_merge(m2, s2, o2, p2);
    }
    // lane q pushes this CTA's partial into CTA q's slot for this rank
    if (lane < C) st_cluster_v4(map_cluster(smem_u32(&ss->lse_in[rank][0]), lane), m1, s1, m2, s2);
  }
  cluster_sync();
  if (warp == 0) {
    float m1 = -INFINITY, s1 = 0.f, m2 = -INFINITY, s2 = 0.f;
    if (lane < C) {
      m1 = ss->lse_in[lane][0];
      s1 = ss->lse_in[lane][1];
      m2 = ss->lse_in[lane][2];
      s2 = ss->lse_in[lane][3];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float o1 = __shfl_xor_sync(0xffffffffu, m1, off), p1 = __shfl_xor_sync(0xffffffffu, s1, off);
      const float o2 = __shfl_xor_sync(0xffffffffu, m2, off), p2 = __shfl_xor_sync(0xffffffffu, s2, off);
      lse_merge(m1, s1, o1, p1);
      lse_merge(m2, s2, o2, p2);
    }
    if (lane == 0) {
      ss->bcast[0] = (s1 > 0.f) ? m1 + log2f(s1) : -INFINITY;
      ss->bcast[1] = m2 + log2f(s2);
    }
  }
  __syncthreads();
  const float lz2 = ss->bcast[0];
  const float lt2 = ss->bcast[1];

  // ---- pass 2: alpha, q_less and the strict-less bits
  float2 acc_a = make_float2(0.f, 0.f), acc_q = make_float2(0.f, 0.f);
  uint8_t* mrow = a.mbits ? a.mbits + row * a.mbits_ld + s0 / 8 : nullptr;
  if (lz2 != -INFINITY) {
    const float2 nlz = make_float2(-lz2, -lz2), nlt = make_float2(-lt2, -lt2);
    for (int g = tid; g < len8 / 8; g += kThreads) {
      const uint4 zw = reinterpret_cast<const uint4*>(zb)[g];
      const uint4 tw = reinterpret_cast<const uint4*>(tb)[g];
      const uint32_t zs[4] = {zw.x, zw.y, zw.z, zw.w};
      const uint32_t ts[4] = {tw.x, tw.y, tw.z, tw.w};
      uint32_t byte = 0;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t zc = bmax2(zs[k], kNegInf2);
        const float2 da = __ffma2_rn(make_float2(bf_lo(zc), bf_hi(zc)), l2e, nlz);
        const float2 db = __ffma2_rn(make_float2(bf_lo(ts[k]), bf_hi(ts[k])), l2e, nlt);
        const float e0 = ex2(fminf(da.x, db.x)), e1 = ex2(fminf(da.y, db.y));
        const bool c0 = da.x < db.x, c1 = da.y < db.y;
        acc_a = __fadd2_rn(acc_a, make_float2(e0, e1));
        acc_q = __fadd2_rn(acc_q, make_float2(c0 ? e0 : 0.f, c1 ? e1 : 0.f));
        byte |= (c0 ? 1u : 0u) << (2 * k) | (c1 ? 1u : 0u) << (2 * k + 1);
      }
      if (mrow) mrow[g] = (uint8_t)byte;
    }
  }
  float al = acc_a.x + acc_a.y, ql = acc_q.x + acc_q.y;
  if (tail > 0 && warp == 0) {
    bool lt = false;
    if (tid < tail && lz2 != -INFINITY && ztail == ztail && ztail != -INFINITY) {
      const float da = fmaf(ztail, kLog2e, -lz2), db = fmaf(ttail, kLog2e, -lt2);
      const float e = ex2(fminf(da, db));
      lt = da < db;
      al += e;
      if (lt) ql += e;
    }
    const unsigned bits = __ballot_sync(0xffffffffu, lt) & ((1u << tail) - 1u);
    if (mrow && tid == 0) mrow[len8 / 8] = (uint8_t)bits;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    al += __shfl_xor_sync(0xffffffffu, al, off);
    ql += __shfl_xor_sync(0xffffffffu, ql, off);
  }
  if (lane == 0) {
    ss->red[warp][0] = al;
    ss->red[warp][1] = ql;
  }
  __syncthreads();
  if (warp == 0) {
    float x = (lane < kWarps) ? ss->red[lane][0] : 0.f;
    float y = (lane < kWarps) ? ss->red[lane][1] : 0.f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      x += __shfl_xor_sync(0xffffffffu, x, off);
      y += __shfl_xor_sync(0xffffffffu, y, off);
    }
    if (lane == 0) {
      const float flags = (float)((ss->bad ? 1 : 0) | (ss->abort_flag ? 2 : 0));
      st_cluster_v4(map_cluster(smem_u32(&ss->al_in[rank][0]), 0), x, y, flags, 0.f);
    }
  }
  // drain before this CTA may exit (copies only remain in flight after a timeout)
  if (tid == 0 && ss->abort_flag) {
    for (int c = 0; c < nch; ++c) {
      const long long t0 = clock64();
      while (!mbar_try_wait(&bars[c], 0) && clock64() - t0 < kWaitLimitCycles) {
      }
    }
  }
  cluster_sync();
  if (rank == 0 && warp == 0) {
    float x = 0.f, y = 0.f;
    int f = 0;
    if (lane < C) {
      x = ss->al_in[lane][0];
      y = ss->al_in[lane][1];
      f = (int)ss->al_in[lane][2];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      x += __shfl_xor_sync(0xffffffffu, x, off);
      y += __shfl_xor_sync(0xffffffffu, y, off);
      f |= __shfl_xor_sync(0xffffffffu, f, off);
    }
    if (lane == 0) {
      if (f & 1) atomicOr(reinterpret_cast<unsigned*>(a.status), SPECOPD_FLAG_NONFINITE);
      if (f & 2) atomicOr(reinterpret_cast<unsigned*>(a.status), SPECOPD_FLAG_TIMEOUT);
      if (lz2 == -INFINITY) x = y = 0.f;
      row_epilogue(a, row, x, y, lz2, lt2);
    }
  }
}

// ---------------- gradient
// A warp covers 512 consecutive logits per pass: lane l owns logits 4l..4l+3
// of each 128-logit step, so every load (8 bytes of draft logits, one byte of
// bits) and every store (16 bytes of gradient) is contiguous across the warp.
// The four steps' loads are all issued before any arithmetic.
constexpr int kGradThreads = 256;
constexpr int kGradSteps = 4;
constexpr int kGradElemsPerWarp = 128 * kGradSteps;

__global__ void __launch_bounds__(kGradThreads) tv_grad_bf16_kernel(const OverlapArgs a, int bx) {
  const long long row = blockIdx.x / bx;
  const int bxi = blockIdx.x - (int)(row * bx);
  const int lane = threadIdx.x & 31;
  const long long wbase = ((long long)bxi * (kGradThreads / 32) + (threadIdx.x >> 5)) * kGradElemsPerWarp;
  if (wbase >= a.V) return;
  const float L2 = a.lz2[row];
  const float Q = a.ql[row];
  const float G = a.g[row];
  const __nv_bfloat16* zrow = static_cast<const __nv_bfloat16*>(a.draft) + row * a.ld_draft;
  const uint8_t* mrow = a.mbits + row * a.mbits_ld;
  float* grow = a.grad + row * a.ld_grad;
  const bool live = L2 != -INFINITY;
  const float2 l2e = make_float2(kLog2e, kLog2e), nl = make_float2(live ? -L2 : 0.f, live ? -L2 : 0.f);
  if (wbase + kGradElemsPerWarp <= a.V) {
    uint2 zw[kGradSteps];
    uint32_t nib[kGradSteps];
#pragma unroll
    for (int v = 0; v < kGradSteps; ++v) {
      const long long e = wbase + v * 128 + 4 * lane;
      zw[v] = __ldcs(reinterpret_cast<const uint2*>(zrow + e));
      nib[v] = mrow[e >> 3];
    }
#pragma unroll
    for (int v = 0; v < kGradSteps; ++v) {
      const long long e = wbase + v * 128 + 4 * lane;
      const uint32_t bits = nib[v] >> ((lane & 1) * 4);
      const uint32_t z0 = bmax2(zw[v].x, kNegInf2), z1 = bmax2(zw[v].y, kNegInf2);  // inactive -> q = 0
      const float2 x0 = __ffma2_rn(make_float2(bf_lo(z0), bf_hi(z0)), l2e, nl);
      const float2 x1 = __ffma2_rn(make_float2(bf_lo(z1), bf_hi(z1)), l2e, nl);
      const float gg = live ? G : 0.f;
      float4 o;
      o.x = gg * ex2(x0.x) * ((float)(bits & 1u) - Q);
      o.y = gg * ex2(x0.y) * ((float)((bits >> 1) & 1u) - Q);
      o.z = gg * ex2(x1.x) * ((float)((bits >> 2) & 1u) - Q);
      o.w = gg * ex2(x1.y) * ((float)((bits >> 3) & 1u) - Q);
      __stcs(reinterpret_cast<float4*>(grow + e), o);
    }
  } else {
    for (long long e = wbase + lane; e < min((long long)a.V, wbase + kGradElemsPerWarp); e += 32) {
      const float z = __bfloat162float(zrow[e]);
      const bool active = live && z == z && fabsf(z) != INFINITY;
      const float q = active ? ex2(fmaf(z, kLog2e, -L2)) : 0.f;
      const uint32_t bit = (mrow[e >> 3] >> (e & 7)) & 1u;
      grow[e] = G * q * ((float)bit - Q);
    }
  }
}

}  // namespace

// Cluster size: the smallest C in {1,2,4,8,16} whose per-CTA share of the
// row (draft + teacher) fits about 48 KB, so four or five CTAs share an SM.
cudaError_t launch_tv_stats_bf16(const OverlapArgs& a, cudaStream_t stream) {
  if (a.rows == 0) return cudaSuccess;
  int C = 0;
  long long seg = 0;
  const int choices[5] = {1, 2, 4, 8, 16};
  for (int i = 0; i < 5 && !C; ++i) {
    seg = (a.V + choices[i] - 1) / choices[i];
    seg = (seg + 7) / 8 * 8;
    if (4 * seg <= 48 * 1024 || choices[i] == kMaxCluster) C = choices[i];
  }
  if (seg > (long long)kChunkElems * kMaxChunks) return cudaErrorInvalidValue;
  const size_t smem = (size_t)4 * seg + kMaxChunks * 8 + sizeof(Smem) + 128;
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(tv_stats_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (C > 8) {
    e = cudaFuncSetAttribute(tv_stats_bf16_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.rows * C), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, tv_stats_bf16_kernel, a, C, (int)seg);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_tv_grad_bf16(const OverlapArgs& a, cudaStream_t stream) {
  if (a.rows == 0) return cudaSuccess;
  const long long per_block = (long long)kGradElemsPerWarp * (kGradThreads / 32);
  const long long bx = (a.V + per_block - 1) / per_block;
  tv_grad_bf16_kernel<<<(unsigned)(bx * a.rows), kGradThreads, 0, stream>>>(a, (int)bx);
  return cudaGetLastError();
}

}  // namespace specopd
