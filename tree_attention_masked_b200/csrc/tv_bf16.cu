// K4/K5 for bf16 logits: per-row overlap statistics and the gradient with
// respect to the draft logits, in one persistent ring kernel.
//
// daiwk.github.io write-up of SpecOPD, section "Equations": alpha = sum_v
// min(q(v), p(v)); L = 1 - (1/(B W)) sum_b sum_j prod_{i<=j} alpha_{b,i};
// teacher and samples fixed during differentiation; teacher mass outside the
// draft support kept.  Section "Inputs and code mapping": NaN padding marks
// inactive draft entries, the teacher must be finite, bf16 work promotes to fp32.
//
// Statistics need two passes over a row (the normalisers before alpha).  A
// row's logits are read from HBM once: the second pass re-reads them from the
// L2, walking the row's chunks last to first (the chunks pass 1 read last are
// the likeliest still to be there), and every copy goes through a ring of
// shared-memory slots fed by one producer thread, so HBM reads run ahead of
// the arithmetic and through the reductions between the passes.  Gradient: dL/dz = g q ([q < p] - q_less)
// from the draft logits and the bits written by pass 2.  The statistics are
// bound by instruction issue and the gradient by HBM, so the same kernel runs
// both side by side: gradient warps on every SM stream the gradient of the
// rows whose branch is already finished while the consumer warps work on the
// next rows.
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
//   pass 2 -- the same bytes again, last chunk first, mostly L2 hits, for
//             alpha, q_less and the [q < p] bits.
// Warp 0 is the producer, warp 1 the row epilogue and warp 2 the gradient
// producer.  The producer walks the chunk sequence P1(row), P2(row), P1(next
// row), ... and bulk-copies each chunk of draft and teacher logits into the
// next free slot (no multicast); the epilogue warp takes each row's results
// from a two-entry queue and runs the E2E-TV row epilogue, which publishes a
// branch's dL/dalpha once its last row is in.  The 16 consumer warps consume
// the slots in the same order, so the copies run ahead through the reductions
// between the passes.  The 8 gradient warps stream the gradient of this CTA's
// rows once published (grad_producer / grad_consumer below).  Per-row
// reductions use fixed shuffle trees (reproducible results).  All waits are
// bounded; the consumer warps always pass the same named barriers, whatever
// happened, so none can be left behind.
constexpr int kRHead = 128;                      // warpgroup 0: producer warp, epilogue warp, 2 idle
constexpr int kRCons = 512;                      // consumer threads (16 warps, warpgroups 1-4)
constexpr int kRGradWarps = 8;                   // gradient warps (warpgroups 5-6)
constexpr int kGUnit = 8192;                     // logits per gradient stage
constexpr int kGStages = 4;
constexpr int kGParts = 4;                       // gradient units per row (claimed one at a time)
constexpr uint32_t kGStageBytes = kGUnit * 2 + kGUnit / 8;  // draft logits + bits
constexpr int kRThreads = kRHead + kRCons + 32 * kRGradWarps;
constexpr int kRWarps = kRCons / 32;
// registers per thread: 72 at launch (896 threads), then warpgroup 0 drops to
// 56, the gradient warpgroups to 48 and the consumers rise to 88
constexpr int kRRegLaunch = 72, kRRegHead = 56, kRRegCons = 88, kRRegGrad = 48;
static_assert(kRHead * kRRegHead + kRCons * kRRegCons + 32 * kRGradWarps * kRRegGrad <= kRThreads * kRRegLaunch,
              "register split exceeds the launch's registers");
constexpr int kRChunk = 12288;                   // logits per chunk and array (3 groups per consumer)
constexpr int kRSlots = 3;                        // 3 x 48 KB ring
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
// 16-byte store that skips L1 and enters L2 with the given eviction policy
// (evict_first for the gradient, so it does not push the statistics' pass-1
// rows out of the L2 before pass 2 re-reads them)
__device__ __forceinline__ void st_global_v4_policy(float* p, const float4& v, uint64_t pol) {
  asm volatile("st.global.L1::no_allocate.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "f"(v.x),
               "f"(v.y), "f"(v.z), "f"(v.w), "l"(pol)
               : "memory");
}
__device__ __forceinline__ void cons_bar() { asm volatile("bar.sync 1, %0;" ::"n"(kRCons) : "memory"); }

struct GradCtl {
  uint64_t full[kGStages];
  uint64_t empty[kGStages];
  float info[kGStages][4];  // (lz2, q_less, dL/dalpha) of the stage's row
  long long row[kGStages];  // the stage's row; -1: no more work
  int e0[kGStages];         // the stage's first logit
};

struct RingRed {
  float r1[kRWarps][4];  // pass-1 partials (mz, sz, mt, st) by consumer warp
  float r2[kRWarps][2];  // pass-2 partials (alpha, q_less)
  int bad[kRWarps];
};

// shared memory: ring slots | RingCtl | RingRed | GradCtl | gradient stages
constexpr size_t kRCtlOff = (size_t)kRSlots * kRSlotBytes;
constexpr size_t kRRedOff = kRCtlOff + sizeof(RingCtl);
constexpr size_t kGCtlOff = kRRedOff + sizeof(RingRed);
constexpr size_t kGBufOff = (kGCtlOff + sizeof(GradCtl) + 127) / 128 * 128;
constexpr size_t kRSmem = kGBufOff + (size_t)kGStages * kGStageBytes;
static_assert(kRSmem <= 232448, "ring kernel exceeds the shared memory of a CTA");

__device__ __forceinline__ void ring_drain_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitLimitCycles) return;
  }
}

__device__ void grad_producer(const OverlapArgs& a, GradCtl* gc, uint8_t* gbuf, volatile int* abort_flag);
__device__ void grad_consumer(const OverlapArgs& a, GradCtl* gc, const uint8_t* gbuf, volatile int* abort_flag, int gw,
                              int lane);

__global__ void __launch_bounds__(kRThreads, 1) tv_stats_bf16_ring_kernel(const OverlapArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* ring = smem;
  RingCtl* ctl = reinterpret_cast<RingCtl*>(smem + kRCtlOff);
  RingRed* rr = reinterpret_cast<RingRed*>(smem + kRRedOff);
  GradCtl* gc = reinterpret_cast<GradCtl*>(smem + kGCtlOff);
  uint8_t* gbuf = smem + kGBufOff;
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
    for (int g = 0; g < kGStages; ++g) {
      mbar_init(&gc->full[g], 1);
      mbar_init(&gc->empty[g], kRGradWarps);
    }
    ctl->abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  volatile int* abort_flag = &ctl->abort_flag;

  if (warp < kRHead / 32) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRRegHead));
    // ================= producer: chunk sequence P1(row), P2(row), P1(next row), ...
    if (warp == 0 && lane == 0) {
      const uint64_t pol_keep = l2_policy_evict_last();
      const uint64_t pol_drop = l2_policy_evict_first();
      long long n = 0;  // chunks issued
      bool ok = true;
      for (long long row = a.row_begin + blockIdx.x; ok && row < a.row_end; row += gridDim.x) {
        const __nv_bfloat16* zrow = static_cast<const __nv_bfloat16*>(a.draft) + row * a.ld_draft;
        const __nv_bfloat16* trow = static_cast<const __nv_bfloat16*>(a.teacher) + row * a.ld_teacher;
        for (int pass = 0; ok && pass < 2; ++pass) {
          for (int cc = 0; cc < nch; ++cc, ++n) {
            const int c = pass ? nch - 1 - cc : cc;  // pass 2 walks the row backwards
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
      for (long long row = a.row_begin + blockIdx.x; row < a.row_end; row += gridDim.x, ++i) {
        const int e = i & 1;
        if (!mbar_wait(&ctl->epi_full[e], (uint32_t)(i >> 1) & 1u, abort_flag)) break;
        const float x = ctl->epi[e][0], y = ctl->epi[e][1], lz2 = ctl->epi[e][2], lt2 = ctl->epi[e][3];
        const int bad = ctl->epi_bad[e];
        mbar_arrive(&ctl->epi_empty[e]);
        if (bad) atomicOr(reinterpret_cast<unsigned*>(a.status), SPECOPD_FLAG_NONFINITE);
        row_epilogue(a, row, x, y, lz2, lt2);
      }
    } else if (warp == 2 && lane == 0) {
      // ================= gradient producer: stages of finished rows
      grad_producer(a, gc, gbuf, abort_flag);
    }
    return;
  }

  if (warp >= (kRHead + kRCons) / 32) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRRegGrad));
    // ================= gradient of rows finished by an earlier launch
    grad_consumer(a, gc, gbuf, abort_flag, warp - (kRHead + kRCons) / 32, lane);
    return;
  }

  // ================= consumers (16 warps, three 16-byte groups of each array per chunk each)
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRRegCons));
  const int ct = tid - kRHead;
  const int cw = ct >> 5;
  long long n = 0;  // chunks consumed
  bool ok = true;   // uniform per warp; a failed wait only skips work, never a barrier
  long long irow = 0;  // rows of this CTA so far
  for (long long row = a.row_begin + blockIdx.x; row < a.row_end; row += gridDim.x, ++irow) {
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
    for (int cc = 0; cc < nch; ++cc, ++n) {
      const int c = nch - 1 - cc;  // the producer's order: last chunk first
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
// The ring kernel's gradient side.  The gradient of rows [grad_begin,
// grad_end) is cut into units of a quarter row (in row order) that the CTAs'
// gradient producers claim from a global counter, so whichever SM is free
// takes the next unit and the last branches' gradient spreads over the whole
// GPU.  A unit waits until its branch's dL/dalpha is published (count W + 1,
// set by the branch's last row in this launch); then one producer thread
// streams its draft logits and bits through kGStages stages of shared memory
// (bulk copies, L2 evict_first, no multicast), each tagged with its row and
// first logit, and the gradient warps write dL/dz = g q ([q < p] - q_less)
// with 16-byte stores hinted L2 evict_first.  The launch is cooperative: every
// CTA is resident and the statistics never wait for the gradient, so every
// wait ends.  All waits are bounded.
__device__ void grad_producer(const OverlapArgs& a, GradCtl* gc, uint8_t* gbuf, volatile int* abort_flag) {
  const uint64_t pol = l2_policy_evict_first();
  const long long nrows = a.grad_end - a.grad_begin;
  const long long per_row = (a.V + kGUnit - 1) / kGUnit;  // stages per row
  const long long per_unit = (per_row + kGParts - 1) / kGParts;
  const long long units = kGParts * nrows;
  unsigned* claim = a.branch_cnt + a.num_branches + 1;
  long long k = 0;  // stages issued
  bool ok = nrows > 0;
  long long u = ok ? (long long)atomicAdd(claim, 1u) : units;
  long long pub_b = -1, sc_row = -1;  // the last branch seen published, the row whose scalars are held
  float lz2 = 0.f, ql = 0.f, g = 0.f;
  while (ok && u < units) {
    const long long un = (long long)atomicAdd(claim, 1u);  // the next unit, claimed early
    const long long row = a.grad_begin + u / kGParts;
    const long long b = row / a.W;
    if (b != pub_b) {
      const unsigned* cnt = a.branch_cnt + b;
      const long long t0 = clock64();
      while (ld_acquire(cnt) != (unsigned)(a.W + 1)) {
        if (*abort_flag) {
          ok = false;
          break;
        }
        if (clock64() - t0 > kWaitLimitCycles) {
          *abort_flag = 1;
          atomicOr(reinterpret_cast<unsigned*>(a.status), SPECOPD_FLAG_TIMEOUT);
          ok = false;
          break;
        }
        __nanosleep(200);
      }
      if (!ok) break;
      pub_b = b;
      // the bits were stored through the generic proxy; the copies read them
      // through the async proxy
      asm volatile("fence.proxy.async.global;" ::: "memory");
    }
    if (row != sc_row) {
      lz2 = __ldcg(a.lz2 + row);
      ql = __ldcg(a.ql + row);
      g = __ldcg(a.g + row);
      sc_row = row;
    }
    const __nv_bfloat16* zrow = static_cast<const __nv_bfloat16*>(a.draft) + row * a.ld_draft;
    const uint8_t* mrow = a.mbits + row * a.mbits_ld;
    const long long s0 = (u % kGParts) * per_unit, s1 = min(per_row, s0 + per_unit);
    for (long long sidx = s0; sidx < s1; ++sidx, ++k) {
      const long long e0 = sidx * kGUnit;
      const int st = (int)(k % kGStages);
      if (k >= kGStages && !mbar_wait(&gc->empty[st], (uint32_t)((k / kGStages) - 1) & 1u, abort_flag)) {
        ok = false;
        break;
      }
      gc->info[st][0] = lz2;
      gc->info[st][1] = ql;
      gc->info[st][2] = g;
      gc->row[st] = row;
      gc->e0[st] = (int)e0;
      const int n = (int)min((long long)kGUnit, a.V - e0);
      const int nbk = n & ~127;  // bulk part: whole 128-logit steps
      uint8_t* dz = gbuf + st * kGStageBytes;
      if (nbk > 0) {
        mbar_arrive_expect_tx(&gc->full[st], (uint32_t)(nbk * 2 + nbk / 8));
        bulk_g2s_policy(dz, zrow + e0, (uint32_t)nbk * 2u, &gc->full[st], pol);
        bulk_g2s_policy(dz + kGUnit * 2, mrow + e0 / 8, (uint32_t)nbk / 8u, &gc->full[st], pol);
      } else {
        mbar_arrive(&gc->full[st]);
      }
    }
    u = un;
  }
  // tell the gradient warps there is no more work: a stage tagged row -1
  if (ok) {
    const int st = (int)(k % kGStages);
    if (k < kGStages || mbar_wait(&gc->empty[st], (uint32_t)((k / kGStages) - 1) & 1u, abort_flag)) {
      gc->row[st] = -1;
      mbar_arrive(&gc->full[st]);
      ++k;
    }
  }
  // every issued copy must land before the CTA may exit
  for (long long j = (k > kGStages ? k - kGStages : 0); j < k; ++j)
    ring_drain_wait(&gc->full[j % kGStages], (uint32_t)(j / kGStages) & 1u);
}

__device__ void grad_consumer(const OverlapArgs& a, GradCtl* gc, const uint8_t* gbuf, volatile int* abort_flag, int gw,
                              int lane) {
  if (a.grad_end <= a.grad_begin) return;
  const float2 l2e = make_float2(kLog2e, kLog2e);
  const uint64_t spol = l2_policy_evict_first();
  for (long long k = 0;; ++k) {
    const int st = (int)(k % kGStages);
    if (!mbar_wait_warp(&gc->full[st], (uint32_t)(k / kGStages) & 1u, abort_flag)) return;
    const long long row = gc->row[st];
    if (row < 0) return;
    const long long e0 = gc->e0[st];
    const float L2 = gc->info[st][0], Q = gc->info[st][1], G = gc->info[st][2];
    const __nv_bfloat16* zrow = static_cast<const __nv_bfloat16*>(a.draft) + row * a.ld_draft;
    const uint8_t* mrow = a.mbits + row * a.mbits_ld;
    float* grow = a.grad + row * a.ld_grad;
    const bool live = L2 != -INFINITY;
    const float gg = live ? G : 0.f;
    const float2 nl = make_float2(live ? -L2 : 0.f, live ? -L2 : 0.f);
    const float omq = 1.f - Q, zmq = 0.f - Q;  // [q < p] - q_less for bit 1 and bit 0
    const int n = (int)min((long long)kGUnit, a.V - e0);
    const int nbk = n & ~127;
    const uint8_t* sz = gbuf + st * kGStageBytes;
    const uint8_t* sb = sz + kGUnit * 2;
    for (int v = gw; v * 128 < nbk; v += kRGradWarps) {
      const int e = v * 128 + 4 * lane;
      const uint2 zw = *reinterpret_cast<const uint2*>(sz + 2 * e);
      const uint32_t bits = (uint32_t)sb[e >> 3] >> ((lane & 1) * 4);
      const uint32_t z0 = bmax2(zw.x, kNegInf2), z1 = bmax2(zw.y, kNegInf2);  // inactive -> q = 0
      const float2 x0 = __ffma2_rn(make_float2(bf_lo(z0), bf_hi(z0)), l2e, nl);
      const float2 x1 = __ffma2_rn(make_float2(bf_lo(z1), bf_hi(z1)), l2e, nl);
      float4 o;
      o.x = gg * ex2(x0.x) * ((bits & 1u) ? omq : zmq);
      o.y = gg * ex2(x0.y) * ((bits & 2u) ? omq : zmq);
      o.z = gg * ex2(x1.x) * ((bits & 4u) ? omq : zmq);
      o.w = gg * ex2(x1.y) * ((bits & 8u) ? omq : zmq);
      st_global_v4_policy(grow + e0 + e, o, spol);
    }
    if (gw == 0) {  // fewer than 128 logits at the end of the row: plain loads
      for (long long e = e0 + nbk + lane; e < e0 + n; e += 32) {
        const float z = __bfloat162float(zrow[e]);
        const bool active = live && z == z && fabsf(z) != INFINITY;
        const float q = active ? ex2(fmaf(z, kLog2e, -L2)) : 0.f;
        const uint32_t bit = (__ldcg(mrow + (e >> 3)) >> (e & 7)) & 1u;
        grow[e] = G * q * ((float)bit - Q);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&gc->empty[st]);
  }
}

}  // namespace

// Persistent ring kernel: one CTA per SM; statistics of rows [row_begin,
// row_end), at most one CTA per row, and, when rows [grad_begin, grad_end)
// are given, their gradient on every SM's gradient warps (a cooperative
// launch: the gradient warps wait for branches finished by other CTAs).
cudaError_t launch_tv_stats_bf16(const OverlapArgs& a, cudaStream_t stream) {
  const long long nrows = a.row_end - a.row_begin;
  const long long ngrad = a.grad_end - a.grad_begin;
  if (nrows <= 0 && ngrad <= 0) return cudaSuccess;
  if (a.V > 0x7fffffffLL - kRChunk) return cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  // setmaxnreg.inc waits until the warpgroups that gave registers back have
  // done so: the split must fit in what the launch allocates
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, tv_stats_bf16_ring_kernel);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kRRegLaunch) return cudaErrorInvalidConfiguration;
  const size_t smem = kRSmem;
  e = cudaFuncSetAttribute(tv_stats_bf16_ring_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long grid = (ngrad > 0 || nrows > sms) ? sms : nrows;
  if (ngrad <= 0) {
    tv_stats_bf16_ring_kernel<<<(unsigned)grid, kRThreads, smem, stream>>>(a);
    return cudaGetLastError();
  }
  // the gradient warps wait for branches finished by other CTAs: all CTAs
  // must be resident at once
  OverlapArgs arg = a;
  void* params[] = {&arg};
  return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(tv_stats_bf16_ring_kernel), dim3((unsigned)grid),
                                     dim3(kRThreads), params, smem, stream);
}

// Fused statistics + gradient in one cooperative launch: the consumer warps
// run the statistics row by row while the gradient warps of every SM stream
// the gradient of the rows whose branch is finished.
cudaError_t launch_tv_fused_bf16(OverlapArgs a, cudaStream_t stream) {
  if (a.rows <= 0) return cudaSuccess;
  a.row_begin = 0;
  a.row_end = a.rows;
  a.grad_begin = 0;
  a.grad_end = a.rows;
  return launch_tv_stats_bf16(a, stream);
}

}  // namespace specopd
