// K4/K5 for bf16 logits: per-row overlap statistics (persistent ring kernel)
// and the streaming gradient.
//
// daiwk.github.io write-up of SpecOPD, section "Equations": alpha = sum_v
// min(q(v), p(v)); L = 1 - (1/(B W)) sum_b sum_j prod_{i<=j} alpha_{b,i};
// teacher and samples fixed during differentiation; teacher mass outside the
// draft support kept.  Section "Inputs and code mapping": NaN padding marks
// inactive draft entries, the teacher must be finite, bf16 work promotes to fp32.
//
// Statistics need two passes over a row (the normalisers before alpha).  A
// row's logits are read from HBM once: the second pass re-reads them while
// they are still in the L2 (one row in flight per SM is a small part of it),
// and every copy goes through a ring of shared-memory slots fed by one
// producer thread, so HBM reads run ahead of the arithmetic and through the
// reductions between the passes.  Gradient: dL/dz = g q ([q < p] - q_less)
// from the draft logits and the bits written by pass 2; every warp access is
// contiguous.
#include <cuda_bf16.h>

#include "internal.h"
#include "overlap_common.cuh"
#include "ptx.cuh"

namespace specopd {
namespace {

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

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// pass-1 update for the G 16-byte groups a thread owns in one chunk: one
// maximum over all of them, then the exponentials of every group against that
// single reference (independent, so they overlap).  Groups with valid[k]
// false hold -inf logits and do not enter the teacher finiteness check.
template <int G>
__device__ __forceinline__ void p1_chunk(const uint4 (&zw)[G], const uint4 (&tw)[G], const bool (&valid)[G], float& mz,
                                         float& sz, float& mt, float& st, uint32_t& tmn) {
  uint32_t zm = kNegInf2, tm = kNegInf2;
#pragma unroll
  for (int k = 0; k < G; ++k) {
    zm = bmax2(zm, bmax2(bmax2(zw[k].x, zw[k].y), bmax2(zw[k].z, zw[k].w)));
    tm = bmax2(tm, bmax2(bmax2(tw[k].x, tw[k].y), bmax2(tw[k].z, tw[k].w)));
    if (valid[k]) tmn = bmin2_nan(tmn, bmin2_nan(bmin2_nan(tw[k].x, tw[k].y), bmin2_nan(tw[k].z, tw[k].w)));
  }
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
  const float mte = (mt == -INFINITY) ? 0.f : mt;
  const float2 l2e = make_float2(kLog2e, kLog2e);
  const float2 nmz = make_float2(-mze, -mze), nmt = make_float2(-mte, -mte);
  float2 az = make_float2(0.f, 0.f), at = make_float2(0.f, 0.f);
#pragma unroll
  for (int k = 0; k < G; ++k) {
    const uint32_t zs[4] = {zw[k].x, zw[k].y, zw[k].z, zw[k].w};
    const uint32_t ts[4] = {tw[k].x, tw[k].y, tw[k].z, tw[k].w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t zc = bmax2(zs[q], kNegInf2);  // NaN (inactive) -> -inf -> adds 0
      const float2 ea = __ffma2_rn(make_float2(bf_lo(zc), bf_hi(zc)), l2e, nmz);
      const float2 eb = __ffma2_rn(make_float2(bf_lo(ts[q]), bf_hi(ts[q])), l2e, nmt);
      az = __fadd2_rn(az, make_float2(ex2(ea.x), ex2(ea.y)));
      at = __fadd2_rn(at, make_float2(ex2(eb.x), ex2(eb.y)));
    }
  }
  sz += az.x + az.y;
  st += at.x + at.y;
}

// pass-2 update for 8 logit pairs: alpha and q_less shares, one byte of bits
__device__ __forceinline__ uint32_t p2_group(const uint4& zw, const uint4& tw, float2 nlz, float2 nlt, float2& acc_a,
                                             float2& acc_q) {
  const float2 l2e = make_float2(kLog2e, kLog2e);
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
  return byte;
}

// ---------------- statistics: persistent ring kernel
// One CTA owns one prediction row at a time (rows blockIdx.x, + gridDim.x,
// ...) and reads it twice through a ring of shared-memory slots:
//   pass 1 -- the row's draft and teacher logits from HBM (L2 policy
//             evict_last) into the online base-2 (max, sum) of both softmaxes;
//   pass 2 -- the same bytes again, an L2 hit (one row per SM is a small part
//             of the L2), for alpha, q_less and the [q < p] bits.
// Warp 0 is the producer and warp 1 the row epilogue.  The producer walks the
// chunk sequence P1(row), P2(row), P1(next row), ... and bulk-copies each
// chunk of draft and teacher logits into the next free slot (no multicast);
// the epilogue warp takes each row's results from a two-entry queue and runs
// the E2E-TV row epilogue.  The other warps consume the slots in the same
// order, so the copies run ahead through the reductions between the passes.  Per-row reductions use fixed shuffle trees
// (reproducible results).  All waits are bounded; the consumer warps always
// pass the same named barriers, whatever happened, so none can be left behind.
constexpr int kRProd = 64;                       // producer warp, epilogue warp
constexpr int kRCons = 512;                      // consumer threads (16 warps)
constexpr int kRThreads = kRProd + kRCons;
constexpr int kRWarps = kRCons / 32;
constexpr int kRChunk = 12288;                   // logits per chunk and array (3 groups per consumer)
constexpr int kRSlots = 4;                        // 4 x 48 KB ring
constexpr int kRGroups = kRChunk / 8;            // 16-byte groups per chunk and array
constexpr uint32_t kRSlotBytes = 2u * kRChunk * 2u;

struct RingCtl {
  uint64_t full[kRSlots];
  uint64_t empty[kRSlots];
  uint64_t epi_full[2];   // a row's results are queued for the epilogue lane
  uint64_t epi_empty[2];  // the epilogue lane has taken them
  float epi[2][4];        // (alpha, q_less, lz2, lt2) of the queued row
  int epi_bad[2];
  int abort_flag;
};

__device__ __forceinline__ void bulk_g2s_policy(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                                uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}
__device__ __forceinline__ void cons_bar() { asm volatile("bar.sync 1, %0;" ::"n"(kRCons) : "memory"); }

struct RingRed {
  float r1[kRWarps][4];  // pass-1 partials (mz, sz, mt, st) by consumer warp
  float r2[kRWarps][2];  // pass-2 partials (alpha, q_less)
  int bad[kRWarps];
};

__device__ __forceinline__ void ring_drain_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitLimitCycles) return;
  }
}

__global__ void __launch_bounds__(kRThreads, 1) tv_stats_bf16_ring_kernel(const OverlapArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* ring = smem;
  RingCtl* ctl = reinterpret_cast<RingCtl*>(ring + kRSlots * kRSlotBytes);
  RingRed* rr = reinterpret_cast<RingRed*>(ctl + 1);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int len8 = (int)(a.V & ~7LL);
  const int tail = (int)(a.V - len8);
  const int nch = (len8 + kRChunk - 1) / kRChunk;
  if (tid == 0) {
    for (int s = 0; s < kRSlots; ++s) {
      mbar_init(&ctl->full[s], 1);
      mbar_init(&ctl->empty[s], kRWarps);
    }
    for (int e = 0; e < 2; ++e) {
      mbar_init(&ctl->epi_full[e], 1);
      mbar_init(&ctl->epi_empty[e], 1);
    }
    ctl->abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  volatile int* abort_flag = &ctl->abort_flag;

  if (warp < kRProd / 32) {
    // ================= producer: chunk sequence P1(row), P2(row), P1(next row), ...
    if (warp == 0 && lane == 0) {
      const uint64_t pol_keep = l2_policy_evict_last();
      const uint64_t pol_drop = l2_policy_evict_first();
      long long n = 0;  // chunks issued
      bool ok = true;
      for (long long row = blockIdx.x; ok && row < a.rows; row += gridDim.x) {
        const __nv_bfloat16* zrow = static_cast<const __nv_bfloat16*>(a.draft) + row * a.ld_draft;
        const __nv_bfloat16* trow = static_cast<const __nv_bfloat16*>(a.teacher) + row * a.ld_teacher;
        for (int pass = 0; ok && pass < 2; ++pass) {
          for (int c = 0; c < nch; ++c, ++n) {
            const int slot = (int)(n % kRSlots);
            if (n >= kRSlots && !mbar_wait(&ctl->empty[slot], (uint32_t)((n / kRSlots) - 1) & 1u, abort_flag)) {
              ok = false;
              break;
            }
            const int e0 = c * kRChunk;
            const uint32_t bytes = (uint32_t)(min(len8, e0 + kRChunk) - e0) * 2u;
            uint8_t* dz = ring + slot * kRSlotBytes;
            mbar_arrive_expect_tx(&ctl->full[slot], 2u * bytes);
            bulk_g2s_policy(dz, zrow + e0, bytes, &ctl->full[slot], pass ? pol_drop : pol_keep);
            bulk_g2s_policy(dz + kRChunk * 2, trow + e0, bytes, &ctl->full[slot], pass ? pol_drop : pol_keep);
          }
        }
      }
      // every issued copy must land before the CTA may exit
      for (long long k = (n > kRSlots ? n - kRSlots : 0); k < n; ++k)
        ring_drain_wait(&ctl->full[k % kRSlots], (uint32_t)(k / kRSlots) & 1u);
      if (ctl->abort_flag) atomicOr(reinterpret_cast<unsigned*>(a.status), SPECOPD_FLAG_TIMEOUT);
    } else if (warp == 1 && lane == 0) {
      // ================= row epilogue in a warp of its own, off the
      // consumers' and the producer's paths (its atomics and the branch's
      // last-arriver loads are long round trips)
      int i = 0;
      for (long long row = blockIdx.x; row < a.rows; row += gridDim.x, ++i) {
        const int e = i & 1;
        if (!mbar_wait(&ctl->epi_full[e], (uint32_t)(i >> 1) & 1u, abort_flag)) break;
        const float x = ctl->epi[e][0], y = ctl->epi[e][1], lz2 = ctl->epi[e][2], lt2 = ctl->epi[e][3];
        const int bad = ctl->epi_bad[e];
        mbar_arrive(&ctl->epi_empty[e]);
        if (bad) atomicOr(reinterpret_cast<unsigned*>(a.status), SPECOPD_FLAG_NONFINITE);
        row_epilogue(a, row, x, y, lz2, lt2);
      }
    }
    return;
  }

  // ================= consumers (16 warps, three 16-byte groups of each array per chunk each)
  const int ct = tid - kRProd;
  const int cw = ct >> 5;
  long long n = 0;  // chunks consumed
  bool ok = true;   // uniform per warp; a failed wait only skips work, never a barrier
  long long irow = 0;  // rows of this CTA so far
  for (long long row = blockIdx.x; row < a.rows; row += gridDim.x, ++irow) {
    const __nv_bfloat16* zrow = static_cast<const __nv_bfloat16*>(a.draft) + row * a.ld_draft;
    const __nv_bfloat16* trow = static_cast<const __nv_bfloat16*>(a.teacher) + row * a.ld_teacher;

    // ---- pass 1
    float mz = -INFINITY, sz = 0.f, mt = -INFINITY, st = 0.f;
    uint32_t tmn = 0u;  // NaN-aware running min of the teacher: NaN or -inf wins
    for (int c = 0; c < nch; ++c, ++n) {
      const int slot = (int)(n % kRSlots);
      if (ok) ok = mbar_wait_warp(&ctl->full[slot], (uint32_t)(n / kRSlots) & 1u, abort_flag);
      if (ok) {
        const int ngc = (min(len8, (c + 1) * kRChunk) - c * kRChunk) / 8;
        const uint4* zs = reinterpret_cast<const uint4*>(ring + slot * kRSlotBytes);
        const uint4* ts = zs + kRGroups;
        constexpr int G = kRGroups / kRCons;
        uint4 zw[G], tw[G];
        bool valid[G];
#pragma unroll
        for (int k = 0; k < G; ++k) {
          valid[k] = ct + k * kRCons < ngc;
          zw[k] = valid[k] ? zs[ct + k * kRCons] : make_uint4(kNegInf2, kNegInf2, kNegInf2, kNegInf2);
          tw[k] = valid[k] ? ts[ct + k * kRCons] : make_uint4(kNegInf2, kNegInf2, kNegInf2, kNegInf2);
        }
        p1_chunk<G>(zw, tw, valid, mz, sz, mt, st, tmn);
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->empty[slot]);
      }
    }
    bool bad = nonfinite(bf_lo(tmn)) || nonfinite(bf_hi(tmn)) || mz == INFINITY || mt == INFINITY;
    float ztail = -INFINITY, ttail = 0.f;
    if (ct < tail) {  // fewer than 8 logits at the very end of the row
      ztail = __bfloat162float(zrow[len8 + ct]);
      ttail = __bfloat162float(trow[len8 + ct]);
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
    const bool wbad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
      rr->r1[cw][0] = mz;
      rr->r1[cw][1] = sz;
      rr->r1[cw][2] = mt;
      rr->r1[cw][3] = st;
      rr->bad[cw] = wbad ? 1 : 0;
    }
    cons_bar();
    // every warp merges the 16 partials with the same shuffle tree: identical bits
    float lz2, lt2;
    bool row_bad = false;
    {
      float m1 = -INFINITY, s1 = 0.f, m2 = -INFINITY, s2 = 0.f;
      if (lane < kRWarps) {
        m1 = rr->r1[lane][0];
        s1 = rr->r1[lane][1];
        m2 = rr->r1[lane][2];
        s2 = rr->r1[lane][3];
        row_bad = rr->bad[lane] != 0;
      }
      row_bad = __any_sync(0xffffffffu, row_bad);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float o1 = __shfl_xor_sync(0xffffffffu, m1, off), p1 = __shfl_xor_sync(0xffffffffu, s1, off);
        const float o2 = __shfl_xor_sync(0xffffffffu, m2, off), p2 = __shfl_xor_sync(0xffffffffu, s2, off);
        lse_merge(m1, s1, o1, p1);
        lse_merge(m2, s2, o2, p2);
      }
      lz2 = (s1 > 0.f) ? m1 + log2f(s1) : -INFINITY;
      lt2 = m2 + log2f(s2);
    }

    // ---- pass 2: alpha, q_less and the strict-less bits (L2 re-read)
    const bool live = lz2 != -INFINITY;
    const float2 nlz = make_float2(live ? -lz2 : 0.f, live ? -lz2 : 0.f), nlt = make_float2(-lt2, -lt2);
    float2 acc_a = make_float2(0.f, 0.f), acc_q = make_float2(0.f, 0.f);
    uint8_t* mrow = a.mbits ? a.mbits + row * a.mbits_ld : nullptr;
    for (int c = 0; c < nch; ++c, ++n) {
      const int slot = (int)(n % kRSlots);
      if (ok) ok = mbar_wait_warp(&ctl->full[slot], (uint32_t)(n / kRSlots) & 1u, abort_flag);
      if (ok) {
        const int ngc = (min(len8, (c + 1) * kRChunk) - c * kRChunk) / 8;
        const uint4* zs = reinterpret_cast<const uint4*>(ring + slot * kRSlotBytes);
        const uint4* ts = zs + kRGroups;
        uint8_t* mc = mrow ? mrow + (long long)c * kRGroups : nullptr;
        if (live) {
#pragma unroll
          for (int k = 0; k < kRGroups / kRCons; ++k) {
            const int g = ct + k * kRCons;
            if (g < ngc) {
              const uint32_t b0 = p2_group(zs[g], ts[g], nlz, nlt, acc_a, acc_q);
              if (mc) mc[g] = (uint8_t)b0;
            }
          }
        } else if (mc) {  // no active draft logit: q = 0 everywhere
          for (int g = ct; g < ngc; g += kRCons) mc[g] = 0;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->empty[slot]);
      }
    }
    float al = acc_a.x + acc_a.y, ql = acc_q.x + acc_q.y;
    if (tail > 0 && cw == 0) {
      bool lt = false;
      if (ct < tail && live && ztail == ztail && ztail != -INFINITY) {
        const float da = fmaf(ztail, kLog2e, -lz2), db = fmaf(ttail, kLog2e, -lt2);
        const float e = ex2(fminf(da, db));
        lt = da < db;
        al += e;
        if (lt) ql += e;
      }
      const unsigned bits = __ballot_sync(0xffffffffu, lt) & ((1u << tail) - 1u);
      if (mrow && ct == 0) mrow[len8 / 8] = (uint8_t)bits;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      al += __shfl_xor_sync(0xffffffffu, al, off);
      ql += __shfl_xor_sync(0xffffffffu, ql, off);
    }
    if (lane == 0) {
      rr->r2[cw][0] = al;
      rr->r2[cw][1] = ql;
    }
    cons_bar();
    if (cw == 0) {
      float x = (lane < kRWarps) ? rr->r2[lane][0] : 0.f;
      float y = (lane < kRWarps) ? rr->r2[lane][1] : 0.f;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        x += __shfl_xor_sync(0xffffffffu, x, off);
        y += __shfl_xor_sync(0xffffffffu, y, off);
      }
      if (lane == 0) {  // queue the row's results for the epilogue lane
        const int e = (int)(irow & 1);
        if (irow < 2 || mbar_wait(&ctl->epi_empty[e], (uint32_t)((irow >> 1) - 1) & 1u, abort_flag)) {
          ctl->epi[e][0] = live ? x : 0.f;
          ctl->epi[e][1] = live ? y : 0.f;
          ctl->epi[e][2] = lz2;
          ctl->epi[e][3] = lt2;
          ctl->epi_bad[e] = row_bad ? 1 : 0;
          mbar_arrive(&ctl->epi_full[e]);
        }
      }
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

// Persistent ring statistics kernel: one CTA per SM (192 KB of ring),
// at most one CTA per row.
cudaError_t launch_tv_stats_bf16(const OverlapArgs& a, cudaStream_t stream) {
  if (a.rows == 0) return cudaSuccess;
  if (a.V > 0x7fffffffLL - kRChunk) return cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const size_t smem = (size_t)kRSlots * kRSlotBytes + sizeof(RingCtl) + sizeof(RingRed);
  e = cudaFuncSetAttribute(tv_stats_bf16_ring_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long grid = a.rows < sms ? a.rows : sms;
  tv_stats_bf16_ring_kernel<<<(unsigned)grid, kRThreads, smem, stream>>>(a);
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
