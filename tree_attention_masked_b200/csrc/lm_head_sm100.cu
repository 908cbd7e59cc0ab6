// Prediction logits from hidden states and a head, consumed tile by tile by
// the overlap statistics: the [rows, V] logits never reach HBM.
//
// daiwk.github.io write-up of SpecOPD, section "Inputs and code mapping":
// prediction_logits reads supplied hidden states and a supplied head (here
// logits = h W^T: no bias, temperature 1), and e2e_tv_loss consumes the
// same-history aligned logits of draft and teacher.  Section "Equations":
// alpha = sum_v min(q, p), L from prefix products of alpha.
//
// alpha needs the normalisers of both softmaxes first, so the logits are
// computed twice:
//   pass A -- every (128-row, 256-entry) tile of draft and teacher logits
//             into TMEM; the epilogue reduces each row's part of the tile to
//             a base-2 (max, sum) pair per softmax;
//   reduce  -- per row, the tile pairs merged in tile order: lz2, lt2;
//   pass B -- the same tiles again; the epilogue forms the row's share of
//             alpha = sum exp2(min(z2 - lz2, t2 - lt2)) and q_less;
//   reduce  -- per row, the shares summed in tile order: alpha, q_less;
// then the E2E-TV loss and dL/dalpha from alpha, and, when the caller asks for
// the gradient with respect to the draft logits,
//   pass C -- the draft tiles a third time; the epilogue writes
//             dL/dz = g q ([q < p] - q_less) from pass B's comparison bits.
//
// Tile kernel: a persistent grid, one CTA per SM, tiles dealt round-robin in
// vocabulary-major order (the row tiles of one head tile run together, so the
// head tile comes from HBM once and from L2 for the others).  Warp 0 issues
// TMA loads (2-D maps, 128-byte swizzle, no multicast) of [128 x 64] hidden
// and [256 x 64] head boxes into a 4-stage ring; one thread of warp 1 issues
// tcgen05.mma (kind::f16, M = 128, N = 256, K = 16) into TMEM columns
// [0, 256) for the draft and [256, 512) for the teacher; warps 4-7 (one
// TMEM lane quarter each, one row per thread) read the accumulators with
// tcgen05.ld.  Each accumulator half has its own full / empty barriers, so
// the epilogue of one half runs under the MMAs of the other.  All waits are
// bounded; a timeout raises SPECOPD_FLAG_TIMEOUT and every role winds down.
#include <cuda.h>
#include <cuda_bf16.h>

#include "internal.h"
#include "overlap_common.cuh"
#include "ptx.cuh"
#include "tmap.cuh"

namespace specopd {
namespace {

constexpr int kLBM = 128;   // rows per tile
constexpr int kLBN = 256;   // vocabulary entries per tile
constexpr int kLBK = 64;    // hidden elements per stage (one 128-byte swizzle row)
constexpr int kLStages = 4;
constexpr int kLThreads = 256;
constexpr uint32_t kLABytes = kLBM * kLBK * 2;  // 16 KB
constexpr uint32_t kLBBytes = kLBN * kLBK * 2;  // 32 KB
constexpr float kLLog2e = 1.4426950408889634f;

struct alignas(1024) LmSmem {
  uint8_t a[kLStages][kLABytes];
  uint8_t b[kLStages][kLBBytes];
  float out[4][32][33];   // pass C: a warp's 32 x 32 gradient block, transposed for coalesced stores
  uint64_t full[kLStages];
  uint64_t empty[kLStages];
  uint64_t acc_full[2];   // MMAs of the draft / teacher half done
  uint64_t acc_empty[2];  // the epilogue has read the half
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

struct LmParams {
  int64_t rows, V;
  int Hd, Ht;
  int m_tiles, n_tiles;
  float4* part_a;        // [n_tiles][rows]: (mz, sz, mt, st), base 2
  float2* part_b;        // [n_tiles][rows]: (alpha share, q_less share)
  const float* lz2;      // [rows] draft normaliser, base 2 (passes B, C)
  const float* lt2;      // [rows] teacher normaliser, base 2 (pass B)
  uint32_t* bits;        // [n_words][rows]: bit i of word w = [q < p] at entry 32 w + i (pass B
                         // writes it when non-null; pass C reads it)
  int64_t n_words;       // ceil(V / 32)
  const float* ql;       // [rows] q_less (pass C)
  const float* g;        // [rows] dL/dalpha (pass C)
  float* grad;           // [rows, ld_grad] dL/dz (pass C)
  int64_t ld_grad;
  int32_t* status;
};

__device__ __forceinline__ void lm_drain_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitLimitCycles) return;
  }
}

template <int PASS>
__global__ void __launch_bounds__(kLThreads, 1)
    lm_head_tile_kernel(const __grid_constant__ CUtensorMap tm_hd, const __grid_constant__ CUtensorMap tm_wd,
                        const __grid_constant__ CUtensorMap tm_ht, const __grid_constant__ CUtensorMap tm_wt,
                        const LmParams p) {
  extern __shared__ uint8_t smem_raw[];
  LmSmem* sm = reinterpret_cast<LmSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long total = (long long)p.m_tiles * p.n_tiles;
  constexpr int kHalves = PASS == 2 ? 1 : 2;  // pass C forms the draft logits only

  if (threadIdx.x == 0) {
    for (int s = 0; s < kLStages; ++s) {
      mbar_init(&sm->full[s], 1);
      mbar_init(&sm->empty[s], 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&sm->acc_full[h], 1);
      mbar_init(&sm->acc_empty[h], 4);
    }
    mbar_init(&sm->mma_done, 1);
    sm->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 2) {
    tmem_alloc(&sm->tmem_base, 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    prefetch_tmap(&tm_hd);
    prefetch_tmap(&tm_wd);
    prefetch_tmap(&tm_ht);
    prefetch_tmap(&tm_wt);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;
  volatile int* abort_flag = &sm->abort_flag;

  if (warp == 0) {
    // ================= TMA producer
    if (lane == 0) {
      long long it = 0;
      bool ok = true;
      for (long long tau = blockIdx.x; ok && tau < total; tau += gridDim.x) {
        const int m = (int)(tau % p.m_tiles), n = (int)(tau / p.m_tiles);
        for (int h = 0; ok && h < kHalves; ++h) {
          const CUtensorMap* ta = h ? &tm_ht : &tm_hd;
          const CUtensorMap* tb = h ? &tm_wt : &tm_wd;
          const int nk = (h ? p.Ht : p.Hd) / kLBK;
          for (int kb = 0; kb < nk; ++kb, ++it) {
            const int s = (int)(it % kLStages);
            if (it >= kLStages && !mbar_wait(&sm->empty[s], (uint32_t)((it / kLStages) - 1) & 1u, abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&sm->full[s], kLABytes + kLBBytes);
            tma_load_2d(sm->a[s], ta, kb * kLBK, m * kLBM, &sm->full[s]);
            tma_load_2d(sm->b[s], tb, kb * kLBK, n * kLBN, &sm->full[s]);
          }
        }
      }
      // every issued copy must land before the CTA may exit
      for (long long j = (it > kLStages ? it - kLStages : 0); j < it; ++j)
        lm_drain_wait(&sm->full[j % kLStages], (uint32_t)(j / kLStages) & 1u);
    }
  } else if (warp == 1) {
    // ================= MMA issuer (one thread)
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kLBM, kLBN, false);
      long long it = 0;
      int k = 0;  // tiles of this CTA so far
      bool ok = true;
      for (long long tau = blockIdx.x; ok && tau < total; tau += gridDim.x, ++k) {
        for (int mdl = 0; ok && mdl < kHalves; ++mdl) {
          // TMEM half: the model's own in passes A and B; in pass C (draft
          // only) the halves alternate between tiles, so the epilogue of one
          // tile runs under the MMAs of the next
          const int h = PASS == 2 ? (k & 1) : mdl;
          const int use = PASS == 2 ? (k >> 1) : k;  // earlier uses of half h
          if (use > 0 && !mbar_wait(&sm->acc_empty[h], (uint32_t)(use - 1) & 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int nk = (mdl ? p.Ht : p.Hd) / kLBK;
          for (int kb = 0; kb < nk; ++kb, ++it) {
            const int s = (int)(it % kLStages);
            if (!mbar_wait(&sm->full[s], (uint32_t)(it / kLStages) & 1u, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t ab = smem_u32(sm->a[s]), bb = smem_u32(sm->b[s]);
#pragma unroll
            for (int ks = 0; ks < kLBK / 16; ++ks)
              mma_ss(tmem + h * kLBN, smem_desc_sw128(ab + ks * 32, 16, 1024),
                     smem_desc_sw128(bb + ks * 32, 16, 1024), idesc, (kb > 0 || ks > 0) ? 1u : 0u);
            mma_commit(&sm->empty[s]);
          }
          if (ok) mma_commit(&sm->acc_full[h]);
        }
      }
      // all MMAs must finish before TMEM and shared memory are released
      mma_commit(&sm->mma_done);
      lm_drain_wait(&sm->mma_done, 0);
    }
  } else if (warp >= 4) {
    // ================= epilogue: one row per thread, TMEM lanes 32 (warp % 4) + lane
    const int q4 = warp & 3;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    const int r_in = q4 * 32 + lane;
    int k = 0;
    bool ok = true;
    for (long long tau = blockIdx.x; ok && tau < total; tau += gridDim.x, ++k) {
      const int m = (int)(tau % p.m_tiles), n = (int)(tau / p.m_tiles);
      const long long row = (long long)m * kLBM + r_in;
      const long long col0 = (long long)n * kLBN;
      const int ncols = (int)min((long long)kLBN, p.V - col0);
      if (PASS == 0) {
        float part[4];
        for (int h = 0; h < 2; ++h) {
          if (!mbar_wait_warp(&sm->acc_full[h], (uint32_t)k & 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          float mx = -INFINITY, sum = 0.f;
          for (int c = 0; c * 32 < ncols; ++c) {
            uint32_t r[32];
            tmem_ld32(tmem + lane_base + h * kLBN + c * 32, r);
            tmem_ld_wait();
            const int nv = min(32, ncols - c * 32);
            float cm = -INFINITY;
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (i < nv) cm = fmaxf(cm, __uint_as_float(r[i]) * kLLog2e);
            float cs = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (i < nv) cs += ex2(fmaf(__uint_as_float(r[i]), kLLog2e, -cm));
            lse_merge(mx, sum, cm, cs);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm->acc_empty[h]);
          part[2 * h] = mx;
          part[2 * h + 1] = sum;
        }
        if (ok && row < p.rows)
          p.part_a[(long long)n * p.rows + row] = make_float4(part[0], part[1], part[2], part[3]);
      } else if (PASS == 2) {
        // dL/dz = g q ([q < p] - q_less) from the draft logits and pass B's bits
        const int hb = k & 1;  // the TMEM half this tile went to
        if (!mbar_wait_warp(&sm->acc_full[hb], (uint32_t)(k >> 1) & 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const bool live_row = row < p.rows;
        const float lz = live_row ? p.lz2[row] : 0.f;
        const float G = live_row ? p.g[row] : 0.f;
        const float Q = live_row ? p.ql[row] : 0.f;
        const float omq = 1.f - Q, zmq = 0.f - Q;
        float(*blk)[33] = sm->out[q4];
        const long long row0 = (long long)m * kLBM + q4 * 32;  // the warp's first row
        for (int c = 0; c * 32 < ncols; ++c) {
          uint32_t rz[32];
          tmem_ld32(tmem + lane_base + hb * kLBN + c * 32, rz);
          const uint32_t word = live_row ? p.bits[((long long)n * (kLBN / 32) + c) * p.rows + row] : 0u;
          tmem_ld_wait();
          const int nv = min(32, ncols - c * 32);
          // lane = row: each lane fills its row of the block ...
#pragma unroll
          for (int i = 0; i < 32; ++i)
            blk[lane][i] = G * ex2(fmaf(__uint_as_float(rz[i]), kLLog2e, -lz)) * (((word >> i) & 1u) ? omq : zmq);
          __syncwarp();
          // ... then the warp stores it row by row: 32 consecutive floats per store
          float* gcol = p.grad + col0 + c * 32 + lane;
          for (int r = 0; r < 32; ++r)
            if (row0 + r < p.rows && lane < nv) __stcs(gcol + (row0 + r) * p.ld_grad, blk[r][lane]);
          __syncwarp();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm->acc_empty[hb]);
      } else {
        if (!mbar_wait_warp(&sm->acc_full[0], (uint32_t)k & 1u, abort_flag) ||
            !mbar_wait_warp(&sm->acc_full[1], (uint32_t)k & 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float lz = row < p.rows ? p.lz2[row] : 0.f;
        const float lt = row < p.rows ? p.lt2[row] : 0.f;
        float al = 0.f, ql = 0.f;
        for (int c = 0; c * 32 < ncols; ++c) {
          uint32_t rz[32], rt[32];
          tmem_ld32(tmem + lane_base + c * 32, rz);
          tmem_ld32(tmem + lane_base + kLBN + c * 32, rt);
          tmem_ld_wait();
          const int nv = min(32, ncols - c * 32);
          uint32_t word = 0;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if (i < nv) {
              const float da = fmaf(__uint_as_float(rz[i]), kLLog2e, -lz);
              const float db = fmaf(__uint_as_float(rt[i]), kLLog2e, -lt);
              const float e = ex2(fminf(da, db));
              al += e;
              if (da < db) {
                ql += e;
                word |= 1u << i;
              }
            }
          }
          if (p.bits && row < p.rows) p.bits[((long long)n * (kLBN / 32) + c) * p.rows + row] = word;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&sm->acc_empty[0]);
          mbar_arrive(&sm->acc_empty[1]);
        }
        if (row < p.rows) p.part_b[(long long)n * p.rows + row] = make_float2(al, ql);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && sm->abort_flag) atomicOr(reinterpret_cast<unsigned*>(p.status), SPECOPD_FLAG_TIMEOUT);
}

// Per row (one warp), the tile pairs of pass A merged in a fixed order: lane
// l takes tiles l, l + 32, ... in turn, then a fixed shuffle tree joins the
// lanes.  Outputs: base-2 normalisers, natural ones for the caller, and the
// non-finite check (a NaN or infinite logit leaves a non-finite pair).
__global__ void lm_reduce_a_kernel(const float4* __restrict__ part, int n_tiles, int64_t rows, float* lz2,
                                   float* lt2, float* lse_draft, float* lse_teacher, int32_t* status) {
  const long long row = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float mz = -INFINITY, sz = 0.f, mt = -INFINITY, st = 0.f;
  bool bad = false;
  for (int n = lane; n < n_tiles; n += 32) {
    const float4 v = part[(long long)n * rows + row];
    bad |= !(fabsf(v.x) < INFINITY) || !(fabsf(v.y) < INFINITY) || !(fabsf(v.z) < INFINITY) ||
           !(fabsf(v.w) < INFINITY);
    lse_merge(mz, sz, v.x, v.y);
    lse_merge(mt, st, v.z, v.w);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float om = __shfl_xor_sync(0xffffffffu, mz, off), os = __shfl_xor_sync(0xffffffffu, sz, off);
    const float pm = __shfl_xor_sync(0xffffffffu, mt, off), ps = __shfl_xor_sync(0xffffffffu, st, off);
    lse_merge(mz, sz, om, os);
    lse_merge(mt, st, pm, ps);
  }
  bad = __any_sync(0xffffffffu, bad);
  if (lane != 0) return;
  const float a = mz + log2f(sz), b = mt + log2f(st);
  lz2[row] = a;
  lt2[row] = b;
  if (lse_draft) lse_draft[row] = a * 0.6931471805599453f;
  if (lse_teacher) lse_teacher[row] = b * 0.6931471805599453f;
  if (bad) atomicOr(reinterpret_cast<unsigned*>(status), SPECOPD_FLAG_NONFINITE);
}

// Per row (one warp), pass B's shares summed in the same fixed order.
__global__ void lm_reduce_b_kernel(const float2* __restrict__ part, int n_tiles, int64_t rows, float* alpha,
                                   float* q_less) {
  const long long row = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float a = 0.f, q = 0.f;
  for (int n = lane; n < n_tiles; n += 32) {
    const float2 v = part[(long long)n * rows + row];
    a += v.x;
    q += v.y;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, off);
    q += __shfl_xor_sync(0xffffffffu, q, off);
  }
  if (lane != 0) return;
  alpha[row] = a;
  if (q_less) q_less[row] = q;
}

// [rows, H] bf16, row-major -> 2-D map, box [64 elements][box_rows rows], 128-byte swizzle
bool make_map_2d(CUtensorMap* tm, const void* ptr, int64_t rows, int H, int box_rows) {
  TensorMapEncodeFn enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)H, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)H * 2};
  cuuint32_t box[2] = {(cuuint32_t)kLBK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

LmHeadLayout lm_head_layout(int64_t rows, int64_t V) {
  LmHeadLayout L;
  L.n_tiles = (V + kLBN - 1) / kLBN;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = (off + bytes + 255) / 256 * 256;
    return at;
  };
  L.part_a = take((size_t)L.n_tiles * rows * sizeof(float4));
  L.part_b = take((size_t)L.n_tiles * rows * sizeof(float2));
  L.lz2 = take((size_t)rows * 4);
  L.lt2 = take((size_t)rows * 4);
  L.alpha = take((size_t)rows * 4);
  L.q_less = take((size_t)rows * 4);
  L.g = take((size_t)rows * 4);
  L.bits = take((size_t)L.n_tiles * (kLBN / 32) * rows * 4);
  L.total = off;
  return L;
}

// Tensor maps and kernel parameters shared by the fused call and the shard phases.
static cudaError_t lm_setup(const LmHeadArgs& a, CUtensorMap* thd, CUtensorMap* twd, CUtensorMap* tht,
                            CUtensorMap* twt, LmParams* pp, unsigned* grid, size_t* smem) {
  if (!make_map_2d(thd, a.h_draft, a.rows, a.Hd, kLBM) || !make_map_2d(twd, a.w_draft, a.V, a.Hd, kLBN) ||
      !make_map_2d(tht, a.h_teacher, a.rows, a.Ht, kLBM) || !make_map_2d(twt, a.w_teacher, a.V, a.Ht, kLBN))
    return cudaErrorInvalidValue;
  const LmHeadLayout L = lm_head_layout(a.rows, a.V);
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  LmParams& p = *pp;
  p.rows = a.rows;
  p.V = a.V;
  p.Hd = a.Hd;
  p.Ht = a.Ht;
  p.m_tiles = (int)((a.rows + kLBM - 1) / kLBM);
  p.n_tiles = (int)L.n_tiles;
  p.part_a = reinterpret_cast<float4*>(ws + L.part_a);
  p.part_b = reinterpret_cast<float2*>(ws + L.part_b);
  p.lz2 = reinterpret_cast<float*>(ws + L.lz2);
  p.lt2 = reinterpret_cast<float*>(ws + L.lt2);
  p.n_words = L.n_tiles * (kLBN / 32);
  p.bits = a.grad_draft ? reinterpret_cast<uint32_t*>(ws + L.bits) : nullptr;
  p.ql = a.q_less ? a.q_less : reinterpret_cast<float*>(ws + L.q_less);
  p.g = a.grad_alpha ? a.grad_alpha : reinterpret_cast<float*>(ws + L.g);
  p.grad = a.grad_draft;
  p.ld_grad = a.ld_grad;
  p.status = a.status;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  *smem = sizeof(LmSmem) + 1024;
  e = cudaFuncSetAttribute(lm_head_tile_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)*smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(lm_head_tile_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)*smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(lm_head_tile_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)*smem);
  if (e != cudaSuccess) return e;
  const long long total = (long long)p.m_tiles * p.n_tiles;
  *grid = (unsigned)(total < sms ? total : sms);
  return cudaSuccess;
}

cudaError_t launch_lm_head_overlap(const LmHeadArgs& a, cudaStream_t stream) {
  if (a.rows <= 0) return cudaSuccess;
  CUtensorMap thd, twd, tht, twt;
  LmParams p;
  unsigned grid;
  size_t smem;
  cudaError_t e = lm_setup(a, &thd, &twd, &tht, &twt, &p, &grid, &smem);
  if (e != cudaSuccess) return e;
  const LmHeadLayout L = lm_head_layout(a.rows, a.V);
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  float* lz2 = const_cast<float*>(p.lz2);
  float* lt2 = const_cast<float*>(p.lt2);
  float* q_less = const_cast<float*>(p.ql);
  float* g = const_cast<float*>(p.g);
  const unsigned rb = (unsigned)((a.rows + 7) / 8);  // one warp per row, 8 per block
  lm_head_tile_kernel<0><<<grid, kLThreads, smem, stream>>>(thd, twd, tht, twt, p);
  lm_reduce_a_kernel<<<rb, 256, 0, stream>>>(p.part_a, p.n_tiles, a.rows, lz2, lt2, a.lse_draft, a.lse_teacher,
                                               a.status);
  lm_head_tile_kernel<1><<<grid, kLThreads, smem, stream>>>(thd, twd, tht, twt, p);
  float* alpha = a.alpha ? a.alpha : reinterpret_cast<float*>(ws + L.alpha);
  lm_reduce_b_kernel<<<rb, 256, 0, stream>>>(p.part_b, p.n_tiles, a.rows, alpha, q_less);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_e2e_loss(alpha, a.num_branches, a.W, a.inv_count, a.loss, g, stream);
  if (e != cudaSuccess || !a.grad_draft) return e;
  // pass C: the draft logits once more, now with dL/dalpha known, into dL/dz
  lm_head_tile_kernel<2><<<grid, kLThreads, smem, stream>>>(thd, twd, tht, twt, p);
  return cudaGetLastError();
}

// One phase over a vocabulary shard (the heads' rows [0, a.V) of the shard):
//   phase 0 -- pass A + merge: out1/out2 = the shard's base-2 log-sum-exps of
//              draft / teacher logits per row;
//   phase 1 -- pass B with the global normalisers lz2, lt2 + merge: out1/out2
//              = the shard's alpha / q_less shares; the [q < p] bits stay in
//              the workspace for phase 2;
//   phase 2 -- pass C with the global lz2, q_less and dL/dalpha: dL/dz of the
//              shard's columns into a.grad_draft.
cudaError_t launch_lm_head_phase(LmHeadArgs a, int phase, const float* lz2, const float* lt2, const float* q_less,
                                 const float* g, float* out1, float* out2, cudaStream_t stream) {
  if (a.rows <= 0) return cudaSuccess;
  CUtensorMap thd, twd, tht, twt;
  LmParams p;
  unsigned grid;
  size_t smem;
  cudaError_t e = lm_setup(a, &thd, &twd, &tht, &twt, &p, &grid, &smem);
  if (e != cudaSuccess) return e;
  // the [q < p] bits: written by phase 1, read by phase 2 (same workspace)
  p.bits = phase >= 1
               ? reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(a.workspace) + lm_head_layout(a.rows, a.V).bits)
               : nullptr;
  const unsigned rb = (unsigned)((a.rows + 7) / 8);
  if (phase == 0) {
    lm_head_tile_kernel<0><<<grid, kLThreads, smem, stream>>>(thd, twd, tht, twt, p);
    lm_reduce_a_kernel<<<rb, 256, 0, stream>>>(p.part_a, p.n_tiles, a.rows, out1, out2, nullptr, nullptr,
                                                 a.status);
  } else if (phase == 1) {
    p.lz2 = lz2;
    p.lt2 = lt2;
    lm_head_tile_kernel<1><<<grid, kLThreads, smem, stream>>>(thd, twd, tht, twt, p);
    lm_reduce_b_kernel<<<rb, 256, 0, stream>>>(p.part_b, p.n_tiles, a.rows, out1, out2);
  } else {
    p.lz2 = lz2;
    p.ql = q_less;
    p.g = g;
    p.grad = out1;
    lm_head_tile_kernel<2><<<grid, kLThreads, smem, stream>>>(thd, twd, tht, twt, p);
  }
  return cudaGetLastError();
}

namespace {
// out[i] = the parts' values at i combined in part order: a sum (mode 0) or
// a base-2 log-sum-exp (mode 1: max, then the sum of 2^(x - max)).
__global__ void merge_parts_kernel(const float* __restrict__ parts, int nparts, int64_t n, int mode, float* out) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  if (mode == 0) {
    float acc = 0.f;
    for (int k = 0; k < nparts; ++k) acc += parts[(long long)k * n + i];
    out[i] = acc;
    return;
  }
  float m = -INFINITY;
  for (int k = 0; k < nparts; ++k) m = fmaxf(m, parts[(long long)k * n + i]);
  if (m == -INFINITY || m != m || m == INFINITY) {  // no entry, or a non-finite part: pass it on
    out[i] = m;
    return;
  }
  float acc = 0.f;
  for (int k = 0; k < nparts; ++k) acc += ex2(parts[(long long)k * n + i] - m);
  out[i] = m + log2f(acc);
}
}  // namespace

cudaError_t launch_merge_parts(const float* parts, int nparts, int64_t n, int mode, float* out, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  merge_parts_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(parts, nparts, n, mode, out);
  return cudaGetLastError();
}

}  // namespace specopd
