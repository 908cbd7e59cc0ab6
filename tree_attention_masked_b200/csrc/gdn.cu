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
// so row i of S evolves on its own.
//
// Everything runs in the chunked form of the rule (C = 64 tokens, the
// checkpoint interval): within a chunk with start state S0, cumulative decays
// g_t and update vectors U (S_t = alpha_t S_{t-1} + u_t k_t^T), the delta rule
// is the unit lower-triangular system
//   (I + A) U = diag(beta) (V - diag(g) K S0^T),  A_ti = beta_t (g_t/g_i) (k_t . k_i), i < t,
// and  O = diag(g) Q S0^T + (L o Q K^T) U,  S_C = g_C S0 + (diag(g_C/g) U)^T K.
// Four kernels, fp32 state and fp32 sums; the products run on the tensor
// cores (tcgen05, TMEM accumulators) with bf16 inputs exact and fp32 operands
// split into bf16 pairs (hi + lo), the triangular solves on fp32 FMAs:
//   gdn_prep_kernel   -- per (trunk chunk, head), in parallel: A, W = (I+A)^-1 diag(beta g) K and
//                        U' = (I+A)^-1 diag(beta) V (so U = U' - W S0^T), the decay-
//                        weighted Q K^T and the decay ratios;
//   gdn_scan_kernel   -- per (tree, head): the only sequential part, chunk by
//                        chunk: the checkpoint at each chunk start,
//                        U = U' - W S0^T, S <- g_C S + (diag(g_C/g) U)^T K;
//   gdn_out_kernel    -- per (trunk chunk, head, half of the columns), in parallel:
//                        the trunk rows' outputs;
//   gdn_branch_kernel -- per (branch, head), in parallel: the state after the
//                        anchor from the checkpoint of its chunk plus that chunk's
//                        first m + 1 update vectors (the indexed state replay of the
//                        figure, without a token-by-token pass), then the branch's
//                        own samples as one chunk from that state.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace specopd {
namespace {

constexpr int kGdnD = 128;            // dk = dv
constexpr int kGdnC = 64;             // checkpoint interval

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------- chunked trunk pass
// Per (trunk chunk, head) the workspace holds (fp32): W [64][128], U [64][128]
// (U' from phase A, then U from phase B), P [64][64], log2 decays [64], the
// chunk-end decay ratios g_n/g_t [64] and g_n (padded to 4): kGdnChunkFloats.
constexpr int kOffW = 0;
constexpr int kOffU = kOffW + kGdnD * kGdnC;
constexpr int kOffP = kOffU + kGdnC * kGdnD;
constexpr int kOffLg = kOffP + kGdnC * kGdnC;
constexpr int kOffCoef = kOffLg + kGdnC;
constexpr int kOffGn = kOffCoef + kGdnC;
constexpr int kGdnChunkFloats = kOffGn + 4;

__device__ __forceinline__ float* chunk_ptr(const GdnArgs& g, long long chunk, int h) {
  return g.chunk_data + (chunk * g.H + h) * (long long)kGdnChunkFloats;
}

// Phase A: one CTA per (trunk chunk of at most C tokens, head), 256 threads.  With the
// chunk's cumulative decays g_t = prod_{i<=t} alpha_i (as log2 g):
//   Gram [K; Q] K^T on the tensor cores (bf16 products are exact in fp32): one
//   M = 128, N = 64, K = 128 MMA group, the K panel serving as both operands;
//   A_ti = beta_t (g_t/g_i) (k_t . k_i), i < t;   P_ti = (g_t/g_i)(q_t . k_i), i <= t;
//   (I + A) X = B by forward substitution, one right-hand-side column per
//   thread in registers: B = diag(beta g) K gives W, B = diag(beta) V gives U'
//   (so a start state S0 gives the chunk's update vectors U = U' - W S0^T);
//   coef_t = g_n / g_t, the decay from token t to the chunk's end.
constexpr int kPrepThreads = 2 * kGdnD;
constexpr int kAsP = kGdnC + 4;  // padded row of A (16-byte aligned rows, 4 banks apart)
constexpr uint32_t kPanel = 128 * 128;  // [128 rows][64 bf16] 128-byte-swizzled panel, bytes

struct PrepSmem {
  uint8_t kq[2 * kPanel];  // rows 0..63: K, rows 64..127: Q (zero past n); K = 128 in two panels
  float As[kGdnC][kAsP];
  __nv_bfloat16 V[kGdnC][kGdnD];
  float lg_s[kGdnC], beta_s[kGdnC], bg_s[kGdnC];  // log2 g_t, beta_t, beta_t g_t
  uint64_t done;
  uint32_t tmem;
  int abort_flag;
};

// byte offset of element (r, k) of a [rows][128] bf16 operand in two 128-byte-swizzled panels
__device__ __forceinline__ uint32_t swz(int r, int j) { return (uint32_t)r * 128u + (uint32_t)((j ^ (r & 7)) << 4); }
__device__ __forceinline__ uint32_t swz_elem(int r, int k) {
  return (uint32_t)(k >> 6) * kPanel + swz(r, (k & 63) >> 3) + (uint32_t)(k & 7) * 2u;
}

__global__ void __launch_bounds__(kPrepThreads) gdn_prep_kernel(const GdnArgs g) {
  extern __shared__ uint8_t smem_raw[];
  PrepSmem& ps = *reinterpret_cast<PrepSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int chunk = blockIdx.x, h = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int t = 0;
  while (t + 1 < g.tp.num_trees && g.ch_off[t + 1] <= chunk) ++t;
  const int c = chunk - g.ch_off[t];
  const long long r0 = g.tp.row_base[t] + (long long)c * kGdnC;
  const int n = min(kGdnC, g.tp.trunk_len[t] - c * kGdnC);
  const __nv_bfloat16* kk = static_cast<const __nv_bfloat16*>(g.k);
  const __nv_bfloat16* qq = static_cast<const __nv_bfloat16*>(g.q);
  const __nv_bfloat16* vv = static_cast<const __nv_bfloat16*>(g.v);
  float* cd = chunk_ptr(g, chunk, h);
  if (tid == 0) {
    mbar_init(&ps.done, 1);
    ps.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&ps.tmem, 64);
    tmem_relinquish();
  }
  // 16 bytes of a token's k, q and v per step
#pragma unroll 2
  for (int idx = tid; idx < kGdnC * (kGdnD / 8); idx += kPrepThreads) {
    const int tt = idx >> 4, j = idx & 15;
    uint4 kw = make_uint4(0u, 0u, 0u, 0u), qw = kw, vw = kw;
    if (tt < n) {
      const long long off = ((r0 + tt) * g.H + h) * kGdnD + 8 * j;
      kw = *reinterpret_cast<const uint4*>(kk + off);
      qw = *reinterpret_cast<const uint4*>(qq + off);
      vw = *reinterpret_cast<const uint4*>(vv + off);
    }
    *reinterpret_cast<uint4*>(ps.kq + (j >> 3) * kPanel + swz(tt, j & 7)) = kw;
    *reinterpret_cast<uint4*>(ps.kq + (j >> 3) * kPanel + swz(kGdnC + tt, j & 7)) = qw;
    *reinterpret_cast<uint4*>(&ps.V[tt][8 * j]) = vw;
  }
  if (tid < kGdnC) {
    const bool in = tid < n;
    ps.lg_s[tid] = in ? log2f(g.alpha[(r0 + tid) * g.H + h]) : 0.f;
    ps.beta_s[tid] = in ? g.beta[(r0 + tid) * g.H + h] : 0.f;
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ps.tmem;
  if (tid == 0) {
    constexpr uint32_t idesc = idesc_bf16_f32(128, 64, false);
    const uint32_t base = smem_u32(ps.kq);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {  // K = 128 in steps of 16: panel ks / 4, 32 bytes per step
      const uint64_t d = smem_desc_sw128(base + (ks >> 2) * kPanel + (ks & 3) * 32, 16, 1024);
      mma_ss(tmem, d, d, idesc, ks > 0 ? 1u : 0u);  // B: the panel's first 64 rows (K)
    }
    mma_commit(&ps.done);
  }
  if (tid == 32)
    for (int tt = 1; tt < kGdnC; ++tt) ps.lg_s[tt] += ps.lg_s[tt - 1];
  __syncthreads();
  if (tid < kGdnC) ps.bg_s[tid] = ps.beta_s[tid] * exp2f(ps.lg_s[tid]);
  // TMEM lanes 0..63 hold K K^T (warps 0, 1), lanes 64..127 Q K^T (warps 2, 3)
  if (warp < 4) {
    if (mbar_wait_warp(&ps.done, 0, &ps.abort_flag)) {
      tc_fence_after();
      const int tt = (32 * warp + lane) & (kGdnC - 1);
      const bool qrow = warp >= 2;
      const float lgt = ps.lg_s[tt], bt = ps.beta_s[tt];
      float* prow = cd + kOffP + tt * kGdnC;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t v[32];
        tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + 32 * half, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          float o[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i = 32 * half + e + u;
            const float ratio = exp2f(lgt - ps.lg_s[i]);
            const float x = __uint_as_float(v[e + u]);
            o[u] = qrow ? ((i <= tt && tt < n) ? ratio * x : 0.f) : ((i < tt && tt < n) ? bt * ratio * x : 0.f);
          }
          const float4 o4 = make_float4(o[0], o[1], o[2], o[3]);
          if (qrow)
            *reinterpret_cast<float4*>(prow + 32 * half + e) = o4;
          else
            *reinterpret_cast<float4*>(&ps.As[tt][32 * half + e]) = o4;
        }
      }
    } else if (lane == 0) {
      atomicOr(reinterpret_cast<unsigned*>(g.status), SPECOPD_FLAG_TIMEOUT);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
  // forward substitution, column j of [W | U'] per thread, in registers
  const int j = tid;
  float X[kGdnC];
#pragma unroll
  for (int tt = 0; tt < kGdnC; ++tt) {
    if (tt >= n) {  // rows past n are zero (zero right-hand side, zero A)
      X[tt] = 0.f;
      continue;
    }
    const float b = j < kGdnD ? ps.bg_s[tt] * __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(ps.kq + swz_elem(tt, j)))
                              : ps.beta_s[tt] * __bfloat162float(ps.V[tt][j - kGdnD]);
    float a0 = b, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
    for (int i = 0; i + 3 < tt; i += 4) {
      const float4 av = *reinterpret_cast<const float4*>(&ps.As[tt][i]);
      a0 = fmaf(-av.x, X[i], a0);
      a1 = fmaf(-av.y, X[i + 1], a1);
      a2 = fmaf(-av.z, X[i + 2], a2);
      a3 = fmaf(-av.w, X[i + 3], a3);
    }
#pragma unroll
    for (int i = tt & ~3; i < tt; ++i) a0 = fmaf(-ps.As[tt][i], X[i], a0);
    X[tt] = (a0 + a1) + (a2 + a3);
  }
  if (j < kGdnD) {  // column j (key element j) of every token's W row
    float* dst = cd + kOffW + j;
#pragma unroll
    for (int tt = 0; tt < kGdnC; ++tt) dst[tt * kGdnD] = X[tt];
  } else {
    float* dst = cd + kOffU + (j - kGdnD);
#pragma unroll
    for (int tt = 0; tt < kGdnC; ++tt) dst[tt * kGdnD] = X[tt];
  }
  if (tid < kGdnC) {
    cd[kOffLg + tid] = ps.lg_s[tid];
    cd[kOffCoef + tid] = exp2f(ps.lg_s[n - 1] - ps.lg_s[tid]);
  }
  if (tid < 4) cd[kOffGn + tid] = tid == 0 ? exp2f(ps.lg_s[n - 1]) : 0.f;
}

// Phase B: the state scan, the only sequential part, on the tensor cores.  One
// CTA per (tree, head), 256 threads.  The state S (128 value rows x 128 key
// elements, fp32) lives in TMEM as an MMA accumulator (lane r = row r).  TMEM
// columns: S [0, 128), its bf16 split Shi [128, 192) and Slo [192, 256) (two
// bf16 per column), D = S W^T [256, 320), the split of (coef U)^T: Uhi
// [320, 352) and Ulo [352, 384).  Per chunk c of n tokens:
//   every warp, one state row per thread (warps 0-3 and 4-7 share the TMEM
//     lanes and take half of the columns each): store the checkpoint (the
//     state at the chunk start), split S into Shi + Slo, scale S in place by
//     g_n, the chunk's total decay, and take half of the row's U' column into
//     registers; all threads split the chunk's W into bf16 panels and
//     transpose K into a bf16 panel (exact);
//   MMA group 1 (A from TMEM):  D = Shi Whi^T + Shi Wlo^T + Slo Whi^T    (M 128, N 64, K 128);
//   meanwhile every thread prefetches the next chunk's W, U', K and decays
//     (cp.async) into a raw staging buffer;
//   every warp, half of the tokens: U = U' - D^T (stored for phases C and D),
//     then coef_t U_t split into Uhi + Ulo;
//   MMA group 2 (A from TMEM):  S += Uhi^T K + Ulo^T K                   (M 128, N 128, K 64).
// The fp32 operands enter as bf16 pairs x = hi + lo (about 16 mantissa bits;
// the dropped lo x lo term is about 2^-16 of a product); K is exact in bf16.
// Shared-memory operand panels are K-major with the 128-byte swizzle (16-byte
// chunk j of row r at chunk j ^ (r mod 8)).  Every wait is bounded.
constexpr int kScanThreads = 256;
constexpr uint32_t kHalfPanel = 64 * 128;  // [64 rows][64 bf16] swizzled panel, bytes
constexpr uint32_t kScS = 0, kScShi = 128, kScSlo = 192, kScD = 256, kScUhi = 320, kScUlo = 352;

struct ScanRaw {  // one chunk record's W, U', decays, and the chunk's K rows, as copied
  float w[kGdnC][kGdnD];
  float u[kGdnC][kGdnD];
  float coef[kGdnC + 4];  // g_n / g_t, then g_n
  __nv_bfloat16 k[kGdnC][kGdnD];
};
struct ScanSmem {
  float ct[kScanThreads / 32][32][33];                 // per warp: a 32 x 32 state tile on its way to the checkpoint
  uint8_t w_hi[2 * kHalfPanel], w_lo[2 * kHalfPanel];  // B of group 1: W rows (tokens), K = 128
  uint8_t kt[kPanel];                                  // B of group 2: K^T rows (key elements), K = 64 tokens
  ScanRaw raw;
  float coef[kGdnC];
  uint64_t bar1, bar2;
  uint32_t tmem;
  int abort_flag;
};

// eight fp32 values -> bf16 hi (rounded) and lo (rounded remainder), packed
__device__ __forceinline__ void split8(const float (&x)[8], uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    h[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
    l[i] = pack_bf16x2(x[2 * i] - __uint_as_float(h[i] << 16), x[2 * i + 1] - __uint_as_float(h[i] & 0xFFFF0000u));
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// chunk c's record (W, U', decays) and K rows into the raw buffer; K rows past
// the chunk's n tokens are zero-filled
__device__ __forceinline__ void scan_prefetch(ScanRaw& raw, const GdnArgs& g, int t, int h, int c, int tid) {
  const int T = g.tp.trunk_len[t];
  const int n = min(kGdnC, T - c * kGdnC);
  const float* cd = chunk_ptr(g, g.ch_off[t] + c, h);
  const __nv_bfloat16* kk = static_cast<const __nv_bfloat16*>(g.k);
  const long long r0 = g.tp.row_base[t] + (long long)c * kGdnC;
  float* wu = &raw.w[0][0];  // W and U' are adjacent in the record and in the buffer
  for (int i = tid; i < 2 * kGdnC * kGdnD / 4; i += kScanThreads) cp_async16(wu + 4 * i, cd + kOffW + 4 * i);
  for (int i = tid; i < (kGdnC + 4) / 4; i += kScanThreads) cp_async16(&raw.coef[4 * i], cd + kOffCoef + 4 * i);
  for (int i = tid; i < kGdnC * (kGdnD / 8); i += kScanThreads) {
    const int tt = i >> 4, j = i & 15;
    if (tt < n)
      cp_async16(&raw.k[tt][8 * j], kk + ((r0 + tt) * g.H + h) * kGdnD + 8 * j);
    else
      *reinterpret_cast<uint4*>(&raw.k[tt][8 * j]) = make_uint4(0u, 0u, 0u, 0u);
  }
  cp_async_commit();
}

__global__ void __launch_bounds__(kScanThreads, 1) gdn_scan_kernel(const GdnArgs g) {
  extern __shared__ uint8_t smem_raw[];
  ScanSmem& sm = *reinterpret_cast<ScanSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int t = blockIdx.x, h = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = g.tp.trunk_len[t];
  const int nch = (T + kGdnC - 1) / kGdnC;
  if (tid == 0) {
    mbar_init(&sm.bar1, 1);
    mbar_init(&sm.bar2, 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem, 512);
    tmem_relinquish();
  }
  if (nch > 0) scan_prefetch(sm.raw, g, t, h, 0, tid);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem;
  const int r = 32 * (warp & 3) + lane;  // state row r = TMEM lane r
  const int hc = warp >> 2;
  const uint32_t trow = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
  bool ok = true;
  // the warp's 32 state rows (TMEM lanes), 32 elements from column 32 q, of the
  // state after token C j - 1 into the checkpoint: transposed through shared
  // memory so that every store writes 128 contiguous bytes of one row
  auto store_ckpt_row = [&](int j, int q, const uint32_t (&v)[32]) {
    float (*tile)[33] = sm.ct[warp];
#pragma unroll
    for (int e = 0; e < 32; ++e) tile[lane][e] = __uint_as_float(v[e]);
    __syncwarp();
    float* dst = g.ckpt + ((long long)(g.ck_off[t] + j - 1) * g.H + h) * kGdnD * kGdnD +
                 (long long)(32 * (warp & 3)) * kGdnD + 32 * q + lane;
#pragma unroll 8
    for (int rr = 0; rr < 32; ++rr) dst[rr * kGdnD] = tile[rr][lane];
    __syncwarp();
  };
  for (int c = 0; c < nch; ++c) {
    const int n = min(kGdnC, T - c * kGdnC);
    float* cd = chunk_ptr(g, g.ch_off[t] + c, h);
    cp_async_wait<0>();
    __syncthreads();  // chunk c's raw data is in shared memory
    // every warp: state row r = TMEM lane r; warps 0-3 take the state's columns
    // 0..63 and tokens 0..31, warps 4-7 columns 64..127 and tokens 32..63
    float up[kGdnC / 2];  // U'[32 hc + i][r]
#pragma unroll
    for (int i = 0; i < kGdnC / 2; ++i) up[i] = sm.raw.u[32 * hc + i][r];
    if (c > 0 && ok) {
      // the state at the chunk start: checkpoint, bf16 split, scale by g_n in place
      const float gn = sm.raw.coef[kGdnC];
#pragma unroll 1
      for (int qq = 0; qq < 2; ++qq) {
        const int q = 2 * hc + qq;
        uint32_t v[32];
        tmem_ld32(trow + kScS + 32 * q, v);
        tmem_ld_wait();
        store_ckpt_row(c, q, v);
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float x0 = __uint_as_float(v[2 * e]), x1 = __uint_as_float(v[2 * e + 1]);
          hi[e] = pack_bf16x2(x0, x1);
          lo[e] = pack_bf16x2(x0 - __uint_as_float(hi[e] << 16), x1 - __uint_as_float(hi[e] & 0xFFFF0000u));
        }
        // 32 fp32 columns -> 16 bf16-pair columns of Shi and of Slo
        tmem_st16(trow + kScShi + 16 * q, hi);
        tmem_st16(trow + kScSlo + 16 * q, lo);
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(gn * __uint_as_float(v[e]));
        tmem_st32(trow + kScS + 32 * q, v);
      }
      tmem_st_wait();
    }
    if (c > 0) {  // W rows (tokens) split into bf16 pairs; rows past n are zero in the record
#pragma unroll 2
      for (int idx = tid; idx < kGdnC * 16; idx += kScanThreads) {
        const int tt = idx >> 4, j = idx & 15;
        const float4 a = *reinterpret_cast<const float4*>(&sm.raw.w[tt][8 * j]);
        const float4 b = *reinterpret_cast<const float4*>(&sm.raw.w[tt][8 * j + 4]);
        const float x[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        uint4 hi, lo;
        split8(x, hi, lo);
        const uint32_t off = (j >> 3) * kHalfPanel + swz(tt, j & 7);
        *reinterpret_cast<uint4*>(sm.w_hi + off) = hi;
        *reinterpret_cast<uint4*>(sm.w_lo + off) = lo;
      }
    }
    // K^T: row e, tokens 8 j .. 8 j + 7
    for (int idx = tid; idx < kGdnD * 8; idx += kScanThreads) {
      const int e = idx & 127, j = idx >> 7;
      uint32_t w[4];
#pragma unroll
      for (int p = 0; p < 4; ++p)
        w[p] = (uint32_t)__bfloat16_as_ushort(sm.raw.k[8 * j + 2 * p][e]) |
               ((uint32_t)__bfloat16_as_ushort(sm.raw.k[8 * j + 2 * p + 1][e]) << 16);
      *reinterpret_cast<uint4*>(sm.kt + swz(e, j)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    if (tid < kGdnC) sm.coef[tid] = tid < n ? sm.raw.coef[tid] : 0.f;
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (c > 0 && tid == 0) {
      constexpr uint32_t idesc1 = idesc_bf16_f32(128, 64, false);
      const uint32_t wh = smem_u32(sm.w_hi), wl = smem_u32(sm.w_lo);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t bo = (ks >> 2) * kHalfPanel + (ks & 3) * 32;
        const uint64_t b_hi = smem_desc_sw128(wh + bo, 16, 1024), b_lo = smem_desc_sw128(wl + bo, 16, 1024);
        mma_ts(tmem + kScD, tmem + kScShi + ks * 8, b_hi, idesc1, ks > 0 ? 1u : 0u);
        mma_ts(tmem + kScD, tmem + kScShi + ks * 8, b_lo, idesc1, 1u);
        mma_ts(tmem + kScD, tmem + kScSlo + ks * 8, b_hi, idesc1, 1u);
      }
      mma_commit(&sm.bar1);
    }
    // the raw buffer is consumed: fetch the next chunk during this one's MMAs
    if (c + 1 < nch) scan_prefetch(sm.raw, g, t, h, c + 1, tid);
    {
      // U = U' - (S W^T)^T for row r and this warp's 32 tokens, stored in place of
      // U'; coef_t U_t split for group 2
      if (c > 0) {
        ok = ok && mbar_wait_warp(&sm.bar1, (uint32_t)(c - 1) & 1u, &sm.abort_flag);
        tc_fence_after();
      }
      uint32_t v[32];
      if (c > 0 && ok) {
        tmem_ld32(trow + kScD + 32 * hc, v);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0u;
      }
      uint32_t hi[16], lo[16];
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        const int tt = 32 * hc + e;
        const float u0 = tt < n ? up[e] - __uint_as_float(v[e]) : 0.f;
        const float u1 = tt + 1 < n ? up[e + 1] - __uint_as_float(v[e + 1]) : 0.f;
        if (tt < n) cd[kOffU + tt * kGdnD + r] = u0;
        if (tt + 1 < n) cd[kOffU + (tt + 1) * kGdnD + r] = u1;
        const float c0 = sm.coef[tt] * u0, c1 = sm.coef[tt + 1] * u1;
        const uint32_t hh = pack_bf16x2(c0, c1);
        hi[e / 2] = hh;
        lo[e / 2] = pack_bf16x2(c0 - __uint_as_float(hh << 16), c1 - __uint_as_float(hh & 0xFFFF0000u));
      }
      tmem_st16(trow + kScUhi + 16 * hc, hi);
      tmem_st16(trow + kScUlo + 16 * hc, lo);
      tmem_st_wait();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
      constexpr uint32_t idesc2 = idesc_bf16_f32(128, 128, false);
      const uint32_t kb = smem_u32(sm.kt);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const uint64_t b = smem_desc_sw128(kb + ks * 32, 16, 1024);
        mma_ts(tmem + kScS, tmem + kScUhi + ks * 8, b, idesc2, (c > 0 || ks > 0) ? 1u : 0u);
        mma_ts(tmem + kScS, tmem + kScUlo + ks * 8, b, idesc2, 1u);
      }
      mma_commit(&sm.bar2);
    }
    // every thread: group 2 (and with it group 1) has finished with the panels and TMEM
    if (!mbar_wait_warp(&sm.bar2, (uint32_t)c & 1u, &sm.abort_flag)) ok = false;
    tc_fence_after();
  }
  cp_async_wait<0>();
  if (!ok && lane == 0) atomicOr(reinterpret_cast<unsigned*>(g.status), SPECOPD_FLAG_TIMEOUT);
  if (ok && T % kGdnC == 0 && nch > 0) {  // the state after the last token
#pragma unroll 1
    for (int q = 2 * hc; q < 2 * hc + 2; ++q) {
      uint32_t v[32];
      tmem_ld32(trow + kScS + 32 * q, v);
      tmem_ld_wait();
      store_ckpt_row(nch, q, v);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Phase C: outputs of the trunk rows on the tensor cores, one CTA per (chunk,
// head, half of the 128 value columns), 256 threads.  With S0 the state at
// the chunk start (zero, or its checkpoint):  O = diag(g) Q S0^T + P U.  Q is
// exact in bf16; S0, P and U are fp32 and enter the MMAs as bf16 pairs
// x = hi + lo (hi = bf16(x), lo = bf16(x - hi), together about 16 mantissa
// bits), so
//   Q S0^T = Q S0hi^T + Q S0lo^T,    P U = Phi Uhi + Phi Ulo + Plo Uhi
// (the dropped Plo Ulo term is about 2^-16 of P U), accumulated in fp32 in
// TMEM: R1 = Q S0^T (columns 0..63), R2 = P U (columns 64..127).  All threads
// stage the operands into K-major 128-byte-swizzled panels (8-row x 128-byte
// atoms, 16-byte chunk j of row r at chunk j ^ (r mod 8)), first Q and S0,
// then, once those MMAs are done, P and U in the same 64 KB (three CTAs share
// an SM); M is 128 with the rows past the chunk's 64 tokens zero.  One thread
// issues the MMAs (kind::f16, bf16 in, fp32 accumulate) and commits each
// group to an mbarrier; the warps that own TMEM lanes 0..63 form g_t R1 + R2.
constexpr int kOutThreads = 256;
struct OutTcSmem {
  // GEMM 1: Q (two panels, K = 128) | S0 rows of the half, hi and lo (two 64-row panels each)
  // GEMM 2: P hi, lo (one panel each, K = 64) | U^T rows of the half, hi and lo (one 64-row panel each)
  uint8_t buf[4 * kPanel];
  uint64_t done;
  uint32_t tmem;
  int abort_flag;
  float lg[kGdnC];
};
constexpr uint32_t kOutAq = 0, kOutBsHi = 2 * kPanel, kOutBsLo = 3 * kPanel;
constexpr uint32_t kOutApHi = 0, kOutApLo = kPanel, kOutBuHi = 2 * kPanel, kOutBuLo = 2 * kPanel + kHalfPanel;

__global__ void __launch_bounds__(kOutThreads) gdn_out_kernel(const GdnArgs g) {
  extern __shared__ uint8_t smem_raw[];
  OutTcSmem& sm = *reinterpret_cast<OutTcSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int chunk = blockIdx.x, h = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int v0 = blockIdx.z * 64;
  int t = 0;
  while (t + 1 < g.tp.num_trees && g.ch_off[t + 1] <= chunk) ++t;
  const int c = chunk - g.ch_off[t];
  const long long r0 = g.tp.row_base[t] + (long long)c * kGdnC;
  const int n = min(kGdnC, g.tp.trunk_len[t] - c * kGdnC);
  const __nv_bfloat16* qq = static_cast<const __nv_bfloat16*>(g.q);
  const float* cd = chunk_ptr(g, chunk, h);
  const float* S0 = c > 0 ? g.ckpt + ((long long)(g.ck_off[t] + c - 1) * g.H + h) * kGdnD * kGdnD : nullptr;
  uint8_t* buf = sm.buf;
  const uint32_t sb = smem_u32(buf);
  constexpr uint32_t idesc = idesc_bf16_f32(128, 64, false);
  if (tid == 0) {
    mbar_init(&sm.done, 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem, 128);
    tmem_relinquish();
  }
  if (tid < kGdnC) sm.lg[tid] = cd[kOffLg + tid];
  uint32_t phase = 0;
  bool ok = true;
  if (S0) {
    // ---- GEMM 1 operands: Q rows (rows >= n zero), S0 rows v0 .. v0 + 63
    for (int idx = tid; idx < 128 * 16; idx += kOutThreads) {
      const int r = idx >> 4, j = idx & 15;
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if (r < n) w = *reinterpret_cast<const uint4*>(qq + ((r0 + r) * g.H + h) * kGdnD + 8 * j);
      *reinterpret_cast<uint4*>(buf + kOutAq + (j >> 3) * kPanel + swz(r, j & 7)) = w;
    }
#pragma unroll 2
    for (int idx = tid; idx < 64 * 16; idx += kOutThreads) {
      const int v = idx >> 4, j = idx & 15;
      const float* src = S0 + (v0 + v) * kGdnD + 8 * j;
      const float4 a = *reinterpret_cast<const float4*>(src);
      const float4 b = *reinterpret_cast<const float4*>(src + 4);
      const float x[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      uint4 hi, lo;
      split8(x, hi, lo);
      const uint32_t off = (j >> 3) * kHalfPanel + swz(v, j & 7);
      *reinterpret_cast<uint4*>(buf + kOutBsHi + off) = hi;
      *reinterpret_cast<uint4*>(buf + kOutBsLo + off) = lo;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
      const uint32_t tmem = sm.tmem;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {  // K = 128 in steps of 16: panel ks / 4, 32 bytes per step
        const uint64_t a = smem_desc_sw128(sb + kOutAq + (ks >> 2) * kPanel + (ks & 3) * 32, 16, 1024);
        const uint32_t boff = (ks >> 2) * kHalfPanel + (ks & 3) * 32;
        mma_ss(tmem, a, smem_desc_sw128(sb + kOutBsHi + boff, 16, 1024), idesc, ks > 0 ? 1u : 0u);
        mma_ss(tmem, a, smem_desc_sw128(sb + kOutBsLo + boff, 16, 1024), idesc, 1u);
      }
      mma_commit(&sm.done);
    }
    // the buffer is reused: every thread waits for GEMM 1 to finish reading it
    ok = mbar_wait_warp(&sm.done, 0, &sm.abort_flag);
    tc_fence_after();
    phase = 1;
  }
  // ---- GEMM 2 operands: P rows (rows >= n zero), U^T rows v0 .. v0 + 63 (tokens >= n zero)
  for (int idx = tid; idx < 128 * 8; idx += kOutThreads) {
    const int r = idx >> 3, j = idx & 7;
    float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (r < n) {
      const float4 a = *reinterpret_cast<const float4*>(cd + kOffP + r * kGdnC + 8 * j);
      const float4 b = *reinterpret_cast<const float4*>(cd + kOffP + r * kGdnC + 8 * j + 4);
      x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    }
    uint4 hi, lo;
    split8(x, hi, lo);
    *reinterpret_cast<uint4*>(buf + kOutApHi + swz(r, j)) = hi;
    *reinterpret_cast<uint4*>(buf + kOutApLo + swz(r, j)) = lo;
  }
  for (int idx = tid; idx < 64 * 8; idx += kOutThreads) {
    const int v = idx & 63, j = idx >> 6;
    float x[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int i = 8 * j + q;
      x[q] = i < n ? cd[kOffU + i * kGdnD + v0 + v] : 0.f;
    }
    uint4 hi, lo;
    split8(x, hi, lo);
    *reinterpret_cast<uint4*>(buf + kOutBuHi + swz(v, j)) = hi;
    *reinterpret_cast<uint4*>(buf + kOutBuLo + swz(v, j)) = lo;
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem;
  if (tid == 0) {
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {  // K = 64
      const uint32_t off = ks * 32;
      const uint64_t ph = smem_desc_sw128(sb + kOutApHi + off, 16, 1024);
      const uint64_t pl = smem_desc_sw128(sb + kOutApLo + off, 16, 1024);
      const uint64_t uh = smem_desc_sw128(sb + kOutBuHi + off, 16, 1024);
      const uint64_t ul = smem_desc_sw128(sb + kOutBuLo + off, 16, 1024);
      mma_ss(tmem + 64, ph, uh, idesc, ks > 0 ? 1u : 0u);
      mma_ss(tmem + 64, ph, ul, idesc, 1u);
      mma_ss(tmem + 64, pl, uh, idesc, 1u);
    }
    mma_commit(&sm.done);
  }
  // ---- epilogue: warps 0, 1 (columns 0..31 of the half) and 4, 5 (32..63) own TMEM lanes 0..63
  if ((warp & 3) < 2) {
    if (ok && mbar_wait_warp(&sm.done, phase, &sm.abort_flag)) {
      tc_fence_after();
      const int row = 32 * (warp & 3) + lane;
      const int cb = warp >= 4 ? 32 : 0;
      const uint32_t ta = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
      uint32_t a[32], b[32];
      tmem_ld32(ta + 64 + cb, b);
      if (S0) tmem_ld32(ta + cb, a);
      tmem_ld_wait();
      if (row < n) {
        const float gt = exp2f(sm.lg[row]);
        float* orow = g.out + ((r0 + row) * g.H + h) * kGdnD + v0 + cb;
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          float4 o;
          o.x = S0 ? fmaf(gt, __uint_as_float(a[e]), __uint_as_float(b[e])) : __uint_as_float(b[e]);
          o.y = S0 ? fmaf(gt, __uint_as_float(a[e + 1]), __uint_as_float(b[e + 1])) : __uint_as_float(b[e + 1]);
          o.z = S0 ? fmaf(gt, __uint_as_float(a[e + 2]), __uint_as_float(b[e + 2])) : __uint_as_float(b[e + 2]);
          o.w = S0 ? fmaf(gt, __uint_as_float(a[e + 3]), __uint_as_float(b[e + 3])) : __uint_as_float(b[e + 3]);
          *reinterpret_cast<float4*>(orow + e) = o;
        }
      }
    } else if (lane == 0) {
      atomicOr(reinterpret_cast<unsigned*>(g.status), SPECOPD_FLAG_TIMEOUT);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// Phase D: branches on the tensor cores, one CTA per (branch, head), 256
// threads.  A branch's nb <= 64 samples form one chunk whose start state is
// S_a, the state after the anchor a (in trunk chunk c, m = a - C c), formed
// without a token-by-token replay (the indexed state replay of the figure):
//   S_a = g_m S_c + sum_{t<=m} (g_m/g_t) U_t k_t^T       (S_c: the chunk's checkpoint)
// then the chunked form from S_a, as for a trunk chunk:
//   Gram [K_b; Q_b] K_b^T -> A_b, P_b;   (I + A_b) [W_b | U'_b] = [diag(beta g) K_b | diag(beta) V_b];
//   U_b = U'_b - W_b S_a^T;    O_b = diag(g) Q_b S_a^T + P_b U_b.
// Products on the tensor cores (fp32 operands as bf16 pairs, bf16 inputs
// exact; token dimensions padded to 64), the triangular solve on fp32 FMAs
// (one column per thread, NMAX >= nb steps unrolled).  TMEM (256 columns):
// S_a [0, 128), then D1 = S_a W_b^T [0, 64) and D2 = S_a Q_b^T [64, 128); the
// Gram [128, 192) and (coef U)^T's split [192, 256), then S_a's split [128,
// 256), then U_b^T's split [128, 192) and D3 = U_b^T P_b^T [192, 256).
constexpr int kBrThreads = 256;
constexpr uint32_t kBrRA = 16 * 1024;  // K_c^T panel, then P_b panels
constexpr uint32_t kBrRB = 32 * 1024;  // [K_b; Q_b] panels
constexpr uint32_t kBrRC = 34 * 1024;  // V_b and A_b, then W_b panels

struct BranchSmem {
  uint8_t ra[kBrRA];
  uint8_t kq[kBrRB];
  uint8_t rc[kBrRC];
  float lgb[kGdnC], betab[kGdnC], bgb[kGdnC];  // the branch's log2 g_t, beta_t, beta_t g_t
  uint64_t bar;
  uint32_t tmem;
  int abort_flag;
};
constexpr uint32_t kBrKct = 0;                                      // region A, phase 0-1
constexpr uint32_t kBrPHi = 0, kBrPLo = kPanel / 2;                 // region A, phase 2-5
constexpr uint32_t kBrV = 0, kBrAs = kPanel;                        // region C, phase 0-2
constexpr uint32_t kBrWHi = 0, kBrWLo = kPanel;                     // region C, phase 2-3
static_assert(kPanel + kGdnC * kAsP * 4 <= kBrRC, "branch region C too small");

template <int NMAX>
__global__ void __launch_bounds__(kBrThreads, NMAX <= 32 ? 2 : 1) gdn_branch_kernel(const GdnArgs g) {
  extern __shared__ uint8_t smem_raw[];
  BranchSmem& sm = *reinterpret_cast<BranchSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int gb = blockIdx.x, h = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nb = g.tp.rows_per_branch;
  if (nb <= 0 || nb > NMAX) return;  // uniform (the launcher picks NMAX >= nb)
  int lo = 0, hi = g.tp.num_trees - 1;  // the tree holding global branch gb
  while (lo < hi) {
    const int mid = (lo + hi + 1) / 2;
    if (g.tp.branch_base[mid] <= gb) lo = mid; else hi = mid - 1;
  }
  const int t = lo;
  const int T = g.tp.trunk_len[t], Pl = g.tp.prompt_len[t];
  int a = g.anchors[gb];
  if (a < Pl || a > T - 1) {
    if (tid == 0) atomicOr(reinterpret_cast<unsigned*>(g.status), SPECOPD_FLAG_ANCHOR);
    a = a < Pl ? Pl : T - 1;
  }
  const long long base = g.tp.row_base[t];
  const int c = a / kGdnC, m = a - c * kGdnC;
  const long long first = base + T + (long long)(gb - g.tp.branch_base[t]) * nb;
  const float* cdc = chunk_ptr(g, g.ch_off[t] + c, h);
  const __nv_bfloat16* kk = static_cast<const __nv_bfloat16*>(g.k);
  const __nv_bfloat16* qq = static_cast<const __nv_bfloat16*>(g.q);
  const __nv_bfloat16* vv = static_cast<const __nv_bfloat16*>(g.v);
  uint8_t* ra = sm.ra;
  uint8_t* rc = sm.rc;
  if (tid == 0) {
    mbar_init(&sm.bar, 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem;
  const int r = 32 * (warp & 3) + lane;   // the TMEM lane (state row) this thread may access
  const int hc = warp >> 2;               // which half of the columns / tokens
  const uint32_t tl = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
  const float lgm = cdc[kOffLg + m];
  // ---- phase 0: staging
  {  // (coef U)^T row r, tokens 32 hc .. 32 hc + 31, split into TMEM [192, 256)
    uint32_t uh[16], ul[16];
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const int t0 = 32 * hc + e;
      const float x0 = t0 <= m ? exp2f(lgm - cdc[kOffLg + t0]) * cdc[kOffU + t0 * kGdnD + r] : 0.f;
      const float x1 = t0 + 1 <= m ? exp2f(lgm - cdc[kOffLg + t0 + 1]) * cdc[kOffU + (t0 + 1) * kGdnD + r] : 0.f;
      const uint32_t hh = pack_bf16x2(x0, x1);
      uh[e / 2] = hh;
      ul[e / 2] = pack_bf16x2(x0 - __uint_as_float(hh << 16), x1 - __uint_as_float(hh & 0xFFFF0000u));
    }
    tmem_st16(tl + 192 + 16 * hc, uh);
    tmem_st16(tl + 224 + 16 * hc, ul);
  }
  for (int idx = tid; idx < kGdnD * 8; idx += kBrThreads) {  // K_c^T: row e, tokens 8 j .. (exact)
    const int e = idx & 127, j = idx >> 7;
    uint32_t w[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int t0 = 8 * j + 2 * p;
      const long long rw = base + (long long)c * kGdnC + t0;
      const uint32_t l16 = t0 <= m ? __bfloat16_as_ushort(kk[(rw * g.H + h) * kGdnD + e]) : 0u;
      const uint32_t h16 = t0 + 1 <= m ? __bfloat16_as_ushort(kk[((rw + 1) * g.H + h) * kGdnD + e]) : 0u;
      w[p] = l16 | (h16 << 16);
    }
    *reinterpret_cast<uint4*>(ra + kBrKct + swz(e, j)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  for (int idx = tid; idx < kGdnC * 16; idx += kBrThreads) {  // K_b, Q_b, V_b rows (zero past nb)
    const int tt = idx >> 4, j = idx & 15;
    uint4 kw = make_uint4(0u, 0u, 0u, 0u), qw = kw, vw = kw;
    if (tt < nb) {
      const long long off = ((first + tt) * g.H + h) * kGdnD + 8 * j;
      kw = *reinterpret_cast<const uint4*>(kk + off);
      qw = *reinterpret_cast<const uint4*>(qq + off);
      vw = *reinterpret_cast<const uint4*>(vv + off);
    }
    *reinterpret_cast<uint4*>(sm.kq + (j >> 3) * kPanel + swz(tt, j & 7)) = kw;
    *reinterpret_cast<uint4*>(sm.kq + (j >> 3) * kPanel + swz(kGdnC + tt, j & 7)) = qw;
    if (tt < NMAX) *reinterpret_cast<uint4*>(rc + kBrV + (tt * kGdnD + 8 * j) * 2) = vw;
  }
  if (tid < kGdnC) {
    const bool in = tid < nb;
    sm.lgb[tid] = in ? log2f(g.alpha[(first + tid) * g.H + h]) : 0.f;
    sm.betab[tid] = in ? g.beta[(first + tid) * g.H + h] : 0.f;
  }
  if (c > 0) {  // g_m S_c into the accumulator: row r, columns 64 hc ..
    const float gm = exp2f(lgm);
    const float* src = g.ckpt + ((long long)(g.ck_off[t] + c - 1) * g.H + h) * kGdnD * kGdnD + r * kGdnD + 64 * hc;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      uint32_t v[32];
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        const float4 x = *reinterpret_cast<const float4*>(src + 32 * q + e);
        v[e] = __float_as_uint(gm * x.x);
        v[e + 1] = __float_as_uint(gm * x.y);
        v[e + 2] = __float_as_uint(gm * x.z);
        v[e + 3] = __float_as_uint(gm * x.w);
      }
      tmem_st32(tl + 64 * hc + 32 * q, v);
    }
  }
  tmem_st_wait();
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // ---- phase 1: S_a += (coef U)^T K_c (A from TMEM);  Gram [K_b; Q_b] K_b^T
  if (tid == 0) {
    constexpr uint32_t id128 = idesc_bf16_f32(128, 128, false), id64 = idesc_bf16_f32(128, 64, false);
    const uint32_t sra = smem_u32(ra), skq = smem_u32(sm.kq);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      const uint64_t b = smem_desc_sw128(sra + kBrKct + ks * 32, 16, 1024);
      mma_ts(tmem, tmem + 192 + ks * 8, b, id128, (c > 0 || ks > 0) ? 1u : 0u);
      mma_ts(tmem, tmem + 224 + ks * 8, b, id128, 1u);
    }
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const uint64_t d = smem_desc_sw128(skq + (ks >> 2) * kPanel + (ks & 3) * 32, 16, 1024);
      mma_ss(tmem + 128, d, d, id64, ks > 0 ? 1u : 0u);
    }
    mma_commit(&sm.bar);
  }
  if (tid == 32)
    for (int tt = 1; tt < kGdnC; ++tt) sm.lgb[tt] += sm.lgb[tt - 1];
  __syncthreads();
  if (tid < kGdnC) sm.bgb[tid] = sm.betab[tid] * exp2f(sm.lgb[tid]);
  bool ok = mbar_wait_warp(&sm.bar, 0, &sm.abort_flag);
  tc_fence_after();
  // ---- phase 2a: from the Gram (TMEM lanes 0..63: K_b K_b^T, 64..127: Q_b K_b^T),
  // A_b to shared memory and P_b straight into its bf16 panels (region A is free)
  float* As = reinterpret_cast<float*>(rc + kBrAs);
  if (warp < 4 && ok) {
    const int tt = r & (kGdnC - 1);
    const bool qrow = warp >= 2;
    const float lgt = sm.lgb[tt], bt = sm.betab[tt];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      uint32_t v[32];
      tmem_ld32(tl + 128 + 32 * half, v);
      tmem_ld_wait();
#pragma unroll
      for (int e8 = 0; e8 < 32; e8 += 8) {
        float o[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = 32 * half + e8 + u;
          const float ratio = exp2f(lgt - sm.lgb[i]);
          const float x = __uint_as_float(v[e8 + u]);
          o[u] = qrow ? ((i <= tt && tt < nb) ? ratio * x : 0.f) : ((i < tt && tt < nb) ? bt * ratio * x : 0.f);
        }
        if (qrow) {
          uint4 xh, xl;
          split8(o, xh, xl);
          const int j = (32 * half + e8) >> 3;
          *reinterpret_cast<uint4*>(ra + kBrPHi + swz(tt, j)) = xh;
          *reinterpret_cast<uint4*>(ra + kBrPLo + swz(tt, j)) = xl;
        } else if (tt < NMAX) {
          *reinterpret_cast<float4*>(As + tt * kAsP + 32 * half + e8) = make_float4(o[0], o[1], o[2], o[3]);
          *reinterpret_cast<float4*>(As + tt * kAsP + 32 * half + e8 + 4) = make_float4(o[4], o[5], o[6], o[7]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // ---- phase 2b: S_a's bf16 split into TMEM (row r, columns 64 hc ..); the solve
  if (ok) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      uint32_t v[32], sh[16], sl[16];
      tmem_ld32(tl + 64 * hc + 32 * q, v);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float x0 = __uint_as_float(v[2 * e]), x1 = __uint_as_float(v[2 * e + 1]);
        sh[e] = pack_bf16x2(x0, x1);
        sl[e] = pack_bf16x2(x0 - __uint_as_float(sh[e] << 16), x1 - __uint_as_float(sh[e] & 0xFFFF0000u));
      }
      tmem_st16(tl + 128 + 32 * hc + 16 * q, sh);
      tmem_st16(tl + 192 + 32 * hc + 16 * q, sl);
    }
    tmem_st_wait();
  }
  const int j = tid;  // column j of [W_b | U'_b]
  float X[NMAX];
#pragma unroll
  for (int tt = 0; tt < NMAX; ++tt) {
    if (tt >= nb) {
      X[tt] = 0.f;
      continue;
    }
    const float bv = j < kGdnD
                         ? sm.bgb[tt] * __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sm.kq + swz_elem(tt, j)))
                         : sm.betab[tt] * __bfloat162float(
                                              reinterpret_cast<const __nv_bfloat16*>(rc + kBrV)[tt * kGdnD + j - kGdnD]);
    float a0 = bv, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
    for (int i = 0; i + 3 < tt; i += 4) {
      const float4 av = *reinterpret_cast<const float4*>(As + tt * kAsP + i);
      a0 = fmaf(-av.x, X[i], a0);
      a1 = fmaf(-av.y, X[i + 1], a1);
      a2 = fmaf(-av.z, X[i + 2], a2);
      a3 = fmaf(-av.w, X[i + 3], a3);
    }
#pragma unroll
    for (int i = tt & ~3; i < tt; ++i) a0 = fmaf(-As[tt * kAsP + i], X[i], a0);
    X[tt] = (a0 + a1) + (a2 + a3);
  }
  __syncthreads();  // the solve is done with V_b and A_b
  // ---- phase 2c: W_b column j straight into its bf16 panels (rows = tokens, zero past NMAX)
  if (j < kGdnD) {
    __nv_bfloat16* wh = reinterpret_cast<__nv_bfloat16*>(rc + kBrWHi);
    __nv_bfloat16* wl = reinterpret_cast<__nv_bfloat16*>(rc + kBrWLo);
#pragma unroll
    for (int tt = 0; tt < kGdnC; ++tt) {
      const float x = tt < NMAX ? X[tt < NMAX ? tt : 0] : 0.f;
      const __nv_bfloat16 xh = __float2bfloat16_rn(x);
      const __nv_bfloat16 xl = __float2bfloat16_rn(x - __bfloat162float(xh));
      const uint32_t off = ((j >> 6) * kHalfPanel + swz(tt, (j & 63) >> 3) + (j & 7) * 2) / 2;
      wh[off] = xh;
      wl[off] = xl;
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // ---- phase 3: D1 = S_a W_b^T (3 MMAs per step), D2 = S_a Q_b^T (2 per step), A from TMEM
  if (tid == 0) {
    constexpr uint32_t id64 = idesc_bf16_f32(128, 64, false);
    const uint32_t src_ = smem_u32(rc), skq = smem_u32(sm.kq);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const uint32_t bo = (ks >> 2) * kHalfPanel + (ks & 3) * 32;
      const uint64_t wh = smem_desc_sw128(src_ + kBrWHi + bo, 16, 1024);
      const uint64_t wl = smem_desc_sw128(src_ + kBrWLo + bo, 16, 1024);
      const uint64_t bq = smem_desc_sw128(skq + (ks >> 2) * kPanel + kGdnC * 128 + (ks & 3) * 32, 16, 1024);
      const uint32_t ah = tmem + 128 + ks * 8, al = tmem + 192 + ks * 8;
      mma_ts(tmem, ah, wh, id64, ks > 0 ? 1u : 0u);
      mma_ts(tmem, ah, wl, id64, 1u);
      mma_ts(tmem, al, wh, id64, 1u);
      mma_ts(tmem + 64, ah, bq, id64, ks > 0 ? 1u : 0u);
      mma_ts(tmem + 64, al, bq, id64, 1u);
    }
    mma_commit(&sm.bar);
  }
  ok = mbar_wait_warp(&sm.bar, 1, &sm.abort_flag) && ok;
  tc_fence_after();
  // ---- phase 4: U_b = U'_b - D1^T (warps 4-7: U'_b column r is this thread's X), split into TMEM
  if (warp >= 4 && ok) {
    uint32_t uh[32], ul[32];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      uint32_t v[32];
      if (32 * q < NMAX) {
        tmem_ld32(tl + 32 * q, v);
        tmem_ld_wait();
      }
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        const int tt = 32 * q + e;
        const float u0 = (tt < NMAX && tt < nb) ? X[tt < NMAX ? tt : 0] - __uint_as_float(v[e]) : 0.f;
        const float u1 = (tt + 1 < NMAX && tt + 1 < nb) ? X[tt + 1 < NMAX ? tt + 1 : 0] - __uint_as_float(v[e + 1]) : 0.f;
        const uint32_t hh = pack_bf16x2(u0, u1);
        uh[16 * q + e / 2] = hh;
        ul[16 * q + e / 2] = pack_bf16x2(u0 - __uint_as_float(hh << 16), u1 - __uint_as_float(hh & 0xFFFF0000u));
      }
    }
    tmem_st32(tl + 128, uh);
    tmem_st32(tl + 160, ul);
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // ---- phase 5: D3 = U_b^T P_b^T (3 MMAs per step)
  if (tid == 0) {
    constexpr uint32_t id64 = idesc_bf16_f32(128, 64, false);
    const uint32_t sra = smem_u32(ra);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      const uint64_t ph = smem_desc_sw128(sra + kBrPHi + ks * 32, 16, 1024);
      const uint64_t pl = smem_desc_sw128(sra + kBrPLo + ks * 32, 16, 1024);
      const uint32_t ah = tmem + 128 + ks * 8, al = tmem + 160 + ks * 8;
      mma_ts(tmem + 192, ah, ph, id64, ks > 0 ? 1u : 0u);
      mma_ts(tmem + 192, ah, pl, id64, 1u);
      mma_ts(tmem + 192, al, ph, id64, 1u);
    }
    mma_commit(&sm.bar);
  }
  ok = mbar_wait_warp(&sm.bar, 0, &sm.abort_flag) && ok;
  tc_fence_after();
  // ---- phase 6: O_b[t][r] = g_t D2[r][t] + D3[r][t], tokens 32 hc ..
  if (ok) {
    if (32 * hc < nb) {
      uint32_t d2[32], d3[32];
      tmem_ld32(tl + 64 + 32 * hc, d2);
      tmem_ld32(tl + 192 + 32 * hc, d3);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int tt = 32 * hc + e;
        if (tt < nb)
          g.out[((first + tt) * g.H + h) * kGdnD + r] =
              fmaf(exp2f(sm.lgb[tt]), __uint_as_float(d2[e]), __uint_as_float(d3[e]));
      }
    }
  } else if (lane == 0) {
    atomicOr(reinterpret_cast<unsigned*>(g.status), SPECOPD_FLAG_TIMEOUT);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <int NMAX>
cudaError_t launch_branch(const GdnArgs& g, cudaStream_t stream) {
  const int smem = (int)sizeof(BranchSmem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(gdn_branch_kernel<NMAX>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  gdn_branch_kernel<NMAX><<<dim3(g.tp.total_branches, g.H), kBrThreads, smem, stream>>>(g);
  return cudaGetLastError();
}

}  // namespace

size_t gdn_checkpoint_floats(const TreeParams& tp, int H) {
  long long n = 0;
  for (int t = 0; t < tp.num_trees; ++t) n += tp.trunk_len[t] / kGdnC;
  return (size_t)n * H * kGdnD * kGdnD;
}

size_t gdn_chunk_floats(const TreeParams& tp, int H) {
  long long n = 0;
  for (int t = 0; t < tp.num_trees; ++t) n += (tp.trunk_len[t] + kGdnC - 1) / kGdnC;
  return (size_t)n * H * kGdnChunkFloats;
}

cudaError_t launch_gdn_tree(GdnArgs g, cudaStream_t stream) {
  if (g.tp.num_trees == 0) return cudaSuccess;
  int off = 0, coff = 0;
  for (int t = 0; t < g.tp.num_trees; ++t) {
    g.ck_off[t] = off;
    g.ch_off[t] = coff;
    off += g.tp.trunk_len[t] / kGdnC;
    coff += (g.tp.trunk_len[t] + kGdnC - 1) / kGdnC;
  }
  g.ch_off[g.tp.num_trees] = coff;
  cudaError_t e = cudaFuncSetAttribute(gdn_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sizeof(PrepSmem) + 1024);
  if (e != cudaSuccess) return e;
  gdn_prep_kernel<<<dim3(coff, g.H), kPrepThreads, sizeof(PrepSmem) + 1024, stream>>>(g);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(gdn_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(ScanSmem) + 1024);
  if (e != cudaSuccess) return e;
  gdn_scan_kernel<<<dim3(g.tp.num_trees, g.H), kScanThreads, sizeof(ScanSmem) + 1024, stream>>>(g);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(gdn_out_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(OutTcSmem) + 1024);
  if (e != cudaSuccess) return e;
  gdn_out_kernel<<<dim3(coff, g.H, 2), kOutThreads, sizeof(OutTcSmem) + 1024, stream>>>(g);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (g.tp.total_branches == 0) return cudaSuccess;
  // the branch kernel unrolls its triangular solve to the branch length
  const int nb = g.tp.rows_per_branch;
  if (nb <= 0) return cudaSuccess;
  return nb <= 16 ? launch_branch<16>(g, stream) : nb <= 32 ? launch_branch<32>(g, stream) : launch_branch<64>(g, stream);
}

}  // namespace specopd
