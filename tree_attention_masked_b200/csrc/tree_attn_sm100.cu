// K3: tree-masked GQA attention on the 5th-generation tensor cores (sm_100a).
//
// SpecOPD listing, Fig 3: one packed pass scores every row of a proposal tree;
// packed queries share the trunk's keys and values while each row attends only
// to itself and its ancestors.  The pages give no kernel; this design is new:
//
//  * a CTA owns two (query tile, query head) slots that read the same KV
//    head (GQA), so every K/V tile it loads feeds both: two heads of one
//    128-row tile, or -- for the last head of an odd group size G -- that
//    head on two neighbouring tiles of one tree, so that no CTA runs with a
//    single head (its second softmax warpgroup would idle and each K/V load
//    would feed half the MMA work);
//  * the columns it visits are the trunk span [tree_base, trunk_hi)
//    followed by the branch span [br_lo, br_hi) of its tile(s) (from the mask
//    builder; for two tiles their union, masked per row); column blocks
//    outside them are never loaded.  Trunk blocks below `trunk_full` are seen
//    by every row and skip masking entirely;
//  * warp 0 issues TMA tile loads (no multicast) into a 4-slot K/V ring,
//    one thread of warp 1 issues tcgen05.mma: S = Q K^T into TMEM, then
//    O += P V with P read straight from TMEM;
//  * warps 4-7 and 8-11 (one warpgroup per query head) own one query row per
//    thread, with 216 registers each (the TMA/MMA warpgroup gives up its
//    share): they read S from TMEM, mask, run the online softmax in base 2,
//    write P (bf16) back over S, and rescale O in TMEM only when the running
//    maximum grows by more than 2^8 (the stale maximum is exact: the same
//    reference enters numerator and denominator);
//  * TMEM: S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512) fp32 columns;
//    P_t occupies the first 64 columns of S_t as packed bf16 pairs.
//
// Sparse mode (the listing's Fig 4: attention reads the selected indexer
// groups plus the causal tail) runs the same pipeline with one more per-row
// filter: a column of the row's history is kept only when its semantic
// position lies in the row's causal tail or in a complete group the indexer
// selected for the row and KV head (bit m of the row's selection words).  With
// the group size g a multiple of 64, each 64-column half of a trunk block lies
// in one group, so the filter costs one flag per half-block; branch columns
// are filtered once per row into the row's ancestor bits.
//
// All waits are bounded (see ptx.cuh); a wait that gives up sets
// SPECOPD_FLAG_TIMEOUT, and the CTA drains its copies and MMAs, frees TMEM
// and returns.
#include <cuda.h>
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"
#include "tmap.cuh"

namespace specopd {
namespace {

constexpr int kBM = 128;             // query rows per tile
constexpr int kBN = 128;             // key columns per block
constexpr int kHD = 128;             // head dim
constexpr int kSlots = 4;            // K/V ring slots
constexpr int kBoxBytes = 128 * 64 * 2;   // one [128 rows][64 elems] swizzled box
constexpr int kTileBytes = 2 * kBoxBytes; // [128][128] bf16
constexpr int kThreads = 384;
constexpr float kRescaleLog2 = 8.0f;

struct __align__(1024) Smem {
  uint8_t q[2][kTileBytes];
  uint8_t kv[kSlots][kTileBytes];
  uint64_t q_full;
  uint64_t kv_full[kSlots];
  uint64_t kv_empty[kSlots];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_done[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

struct Params {
  __nv_bfloat16* out;
  const int32_t* pos;
  const int32_t* trunk_limit;
  const uint64_t* anc_bits;
  const specopd_tile_meta* meta;
  int num_tiles;
  int Hq, Hkv, G, pairs;  // pairs = G / 2 head pairs per tile
  int items_per_pair;     // work items per pair of tiles (2k, 2k+1)
  float scale_log2;
  int32_t* status;
  // sparse mode only: per (row, KV head) sel_words words, bit m set iff
  // complete group m of the row's history is selected; g % 64 == 0
  const uint32_t* sel_mask;
  int sel_words;
  int g;
};

__device__ __forceinline__ bool group_selected(const uint32_t* w, int m) { return (w[m >> 5] >> (m & 31)) & 1u; }

// bounded wait used only to drain in-flight work before exit: ignores the
// abort flag, still gives up after the time limit.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitLimitCycles) return;
  }
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ int block_col(const specopd_tile_meta& m, int n_trunk, int j) {
  return j < n_trunk ? m.tree_base + j * kBN : m.br_lo + (j - n_trunk) * kBN;
}

template <bool kSparse>
__global__ void __launch_bounds__(kThreads, 1)
    tree_attn_sm100_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem* sm = reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item.  Tiles are taken in pairs (2k, 2k+1), the latest rows (the
  // costliest) first.  Per pair: for each of its two tiles, KV head and head
  // pair an item with two heads of that tile; for odd G, per KV head one item
  // with head G-1 on both tiles (when they belong to the same tree; else one
  // single-slot item per tile).  Items with nothing to do return at once.
  int tile_s[2], head_s[2], nq;
  {
    const int w = blockIdx.x;
    const int k = (p.num_tiles + 1) / 2 - 1 - w / p.items_per_pair;
    const int r = w % p.items_per_pair;
    const int n_two = 2 * p.Hkv * p.pairs;
    if (r < n_two) {
      const int sub = r / (p.Hkv * p.pairs);
      const int rem = r % (p.Hkv * p.pairs);
      const int h = (rem / p.pairs) * p.G + 2 * (rem % p.pairs);
      tile_s[0] = tile_s[1] = 2 * k + 1 - sub;
      head_s[0] = h;
      head_s[1] = h + 1;
      nq = 2;
    } else {
      const int sub = (r - n_two) / p.Hkv;
      const int h = ((r - n_two) % p.Hkv) * p.G + p.G - 1;
      const bool has1 = 2 * k + 1 < p.num_tiles;
      const bool same = has1 && p.meta[2 * k].tree_base == p.meta[2 * k + 1].tree_base;
      head_s[0] = head_s[1] = h;
      tile_s[0] = 2 * k + sub;
      tile_s[1] = 2 * k + 1;
      nq = same ? (sub == 0 ? 2 : 0) : 1;
    }
    if (tile_s[0] >= p.num_tiles) nq = 0;
  }
  if (nq == 0) return;  // uniform over the CTA, before any barrier or TMEM use
  // column spans: the union over the CTA's tiles (each slot's rows mask per row)
  specopd_tile_meta m = p.meta[tile_s[0]];
  if (nq == 2 && tile_s[1] != tile_s[0]) {
    const specopd_tile_meta m1 = p.meta[tile_s[1]];
    m.trunk_hi = max(m.trunk_hi, m1.trunk_hi);
    m.trunk_full = min(m.trunk_full, m1.trunk_full);
    if (m1.br_hi > m1.br_lo) {
      if (m.br_hi > m.br_lo) {
        m.br_lo = min(m.br_lo, m1.br_lo);
        m.br_hi = max(m.br_hi, m1.br_hi);
      } else {
        m.br_lo = m1.br_lo;
        m.br_hi = m1.br_hi;
      }
    }
  }
  const int n_trunk = (m.trunk_hi - m.tree_base + kBN - 1) / kBN;
  const int n_br = (m.br_hi > m.br_lo) ? (m.br_hi - m.br_lo + kBN - 1) / kBN : 0;
  const int nblk = n_trunk + n_br;
  const int kvh = head_s[0] / p.G;

  if (threadIdx.x == 0) {
    mbar_init(&sm->q_full, 1);
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&sm->kv_full[s], 1);
      mbar_init(&sm->kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&sm->s_full[t], 1);
      mbar_init(&sm->p_full[t], 128);
      mbar_init(&sm->o_done[t], 1);
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
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;
  volatile int* abort_flag = &sm->abort_flag;

  // Registers: the TMA/MMA warpgroup needs few, the two softmax warpgroups
  // (a query row of 128 scores per thread) many; 128 x 72 + 256 x 216 equals
  // the 384 x 168 the block is launched with.
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 72;");
    if (warp == 0) {
    // ================= TMA producer
    if (lane == 0) {
      mbar_arrive_expect_tx(&sm->q_full, nq * kTileBytes);
      for (int t = 0; t < nq; ++t) {
        const int row0 = p.meta[tile_s[t]].row_start;
        for (int hx = 0; hx < 2; ++hx)
          tma_load_3d(sm->q[t] + hx * kBoxBytes, &tmQ, hx * 64, head_s[t], row0, &sm->q_full);
      }
      int last_n[kSlots] = {-1, -1, -1, -1};
      for (int n = 0; n < 2 * nblk; ++n) {
        const int slot = n % kSlots;
        if (n >= kSlots && !mbar_wait(&sm->kv_empty[slot], ((n / kSlots) - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(&sm->kv_full[slot], kTileBytes);
        const int c0 = block_col(m, n_trunk, n >> 1);
        const CUtensorMap* tm = (n & 1) ? &tmV : &tmK;
        tma_load_3d(sm->kv[slot], tm, 0, kvh, c0, &sm->kv_full[slot]);
        tma_load_3d(sm->kv[slot] + kBoxBytes, tm, 64, kvh, c0, &sm->kv_full[slot]);
        last_n[slot] = n;
      }
      // every issued copy must land before the CTA may exit
      drain_wait(&sm->q_full, 0);
      for (int s = 0; s < kSlots; ++s)
        if (last_n[s] >= 0) drain_wait(&sm->kv_full[s], (last_n[s] / kSlots) & 1);
    }
    } else if (warp == 1) {
    // ================= MMA issuer (one thread)
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, kHD, true);
      auto issue_s = [&](int j, int t) {
        const uint32_t kb = smem_u32(sm->kv[(2 * j) % kSlots]);
        const uint32_t qb = smem_u32(sm->q[t]);
#pragma unroll
        for (int s = 0; s < kHD / 16; ++s) {
          const uint32_t off = (s >> 2) * kBoxBytes + (s & 3) * 32;
          mma_ss(tmem + t * 128, smem_desc_sw128(qb + off, 16, 1024), smem_desc_sw128(kb + off, 16, 1024),
                 idesc_qk, s > 0);
        }
        mma_commit(&sm->s_full[t]);
      };
      auto issue_pv = [&](int j, int t) {
        const uint32_t vb = smem_u32(sm->kv[(2 * j + 1) % kSlots]);
#pragma unroll
        for (int s = 0; s < kBN / 16; ++s) {
          mma_ts(tmem + 256 + t * 128, tmem + t * 128 + s * 8, smem_desc_sw128(vb + s * 2048, kBoxBytes, 1024),
                 idesc_pv, (j > 0 || s > 0) ? 1u : 0u);
        }
        mma_commit(&sm->o_done[t]);
      };
      bool ok = mbar_wait(&sm->q_full, 0, abort_flag);
      if (ok) ok = mbar_wait(&sm->kv_full[0], 0, abort_flag);
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < nq; ++t) issue_s(0, t);
        mma_commit(&sm->kv_empty[0]);
      }
      for (int j = 0; ok && j < nblk; ++j) {
        const int nv = 2 * j + 1;
        if (!mbar_wait(&sm->kv_full[nv % kSlots], (nv / kSlots) & 1, abort_flag)) break;
        const bool next = j + 1 < nblk;
        const int nk = 2 * (j + 1);
        for (int t = 0; t < nq; ++t) {
          if (!mbar_wait(&sm->p_full[t], j & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_pv(j, t);
          if (next) {
            if (t == 0 && !mbar_wait(&sm->kv_full[nk % kSlots], (nk / kSlots) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            issue_s(j + 1, t);
          }
        }
        if (!ok) break;
        mma_commit(&sm->kv_empty[nv % kSlots]);
        if (next) mma_commit(&sm->kv_empty[nk % kSlots]);
      }
      // all MMAs must finish before TMEM and shared memory are released
      mma_commit(&sm->mma_done);
      drain_wait(&sm->mma_done, 0);
    }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 216;");
    // ================= softmax: one warpgroup per query head, one row per thread
    const int t = (warp - 4) >> 2;
    if (t < nq) {
      const int quad = warp & 3;
      const int rloc = quad * 32 + lane;
      const int r = p.meta[tile_s[t]].row_start + rloc;
      const bool valid = r < p.meta[tile_s[t]].row_end;
      int lim = m.tree_base, bstart = 0;
      uint64_t bits = 0;
      int tail0 = 0;                  // sparse: first position of the causal tail
      const uint32_t* selw = nullptr;  // sparse: the row's selection words
      if (valid) {
        const int tl = p.trunk_limit[r];
        const int prow = p.pos[r];
        lim = m.tree_base + tl;
        bstart = r - (prow - tl) + 1;
        bits = p.anc_bits[r];
        if (kSparse) {
          tail0 = (prow + 1) / p.g * p.g;
          selw = p.sel_mask + ((long long)r * p.Hkv + kvh) * p.sel_words;
          // branch sample k (position tl + k) stays visible only if its group is selected or in the tail
          uint64_t keep = 0;
          for (int k = 1; k <= prow - tl; ++k) {
            const int q = tl + k;
            if (q >= tail0 || group_selected(selw, q / p.g)) keep |= 1ull << (k - 1);
          }
          bits &= keep;
        }
      }
      const uint32_t trow = tmem + ((uint32_t)(quad * 32) << 16);
      const uint32_t s_col = t * 128;
      const uint32_t o_col = 256 + t * 128;
      float m_use = -INFINITY;
      float l = 0.f;
      bool ok = true;
      for (int j = 0; j < nblk; ++j) {
        if (!mbar_wait_warp(&sm->s_full[t], j & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[128];
        tmem_ld32(trow + s_col + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(trow + s_col + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_ld32(trow + s_col + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
        tmem_ld32(trow + s_col + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
        tmem_ld_wait();
        float* s = reinterpret_cast<float*>(sr);
        const int c0 = block_col(m, n_trunk, j);
        const bool trunk = j < n_trunk;
        if (kSparse && trunk) {
          // positions of this block: c0 - tree_base + [0, 128); a half below the
          // tail lies in one complete group (g % 64 == 0, blocks 128-aligned)
          const int q0 = c0 - m.tree_base;
          if (!(q0 >= tail0 || group_selected(selw, q0 / p.g))) {
#pragma unroll
            for (int e = 0; e < 64; ++e) s[e] = -INFINITY;
          }
          if (!(q0 + 64 >= tail0 || group_selected(selw, (q0 + 64) / p.g))) {
#pragma unroll
            for (int e = 64; e < 128; ++e) s[e] = -INFINITY;
          }
        }
        if (!(trunk && c0 + kBN <= m.trunk_full)) {
          if (trunk) {
#pragma unroll
            for (int e = 0; e < 128; ++e)
              if (c0 + e > lim) s[e] = -INFINITY;
          } else {
#pragma unroll
            for (int e = 0; e < 128; ++e) {
              const unsigned off = (unsigned)(c0 + e - bstart);
              const bool vis = off < 64u && ((bits >> off) & 1ull);
              if (!vis) s[e] = -INFINITY;
            }
          }
        }
        float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
        for (int e = 4; e < 128; e += 8) {
          mx0 = fmax3(mx0, s[e], s[e + 1]);
          mx1 = fmax3(mx1, s[e + 2], s[e + 3]);
          mx2 = fmax3(mx2, s[e + 4], s[e + 5]);
          mx3 = fmax3(mx3, s[e + 6], s[e + 7]);
        }
        const float mx = fmax3(fmaxf(mx0, mx1), mx2, mx3);
        const float m_new = fmaxf(m_use, mx * p.scale_log2);
        float corr = 1.f;
        bool rescale = false;
        // (a fully masked block before any visible column leaves m_use at -inf)
        if ((m_use == -INFINITY && m_new != -INFINITY) || m_new > m_use + kRescaleLog2) {
          corr = ex2(m_use - m_new);
          m_use = m_new;
          rescale = j > 0;
        }
        const float m_eff = (m_use == -INFINITY) ? 0.f : m_use;
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
        const float2 nm2 = make_float2(-m_eff, -m_eff);
        float2 acc[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) acc[a] = make_float2(0.f, 0.f);
        uint32_t pk[64];
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          const float2 x = __ffma2_rn(make_float2(s[2 * e], s[2 * e + 1]), sc2, nm2);
          const float2 pe = make_float2(ex2(x.x), ex2(x.y));
          acc[e & 3] = __fadd2_rn(acc[e & 3], pe);
          pk[e] = pack_bf16x2(pe.x, pe.y);
        }
        acc[0] = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
        l = l * corr + (acc[0].x + acc[0].y);
        tmem_st32(trow + s_col + 0, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
        tmem_st32(trow + s_col + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
        tmem_st_wait();
        if (__any_sync(0xffffffffu, rescale)) {
          // O may be touched only after the previous P.V has finished
          if (!mbar_wait_warp(&sm->o_done[t], (j - 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t orr[32];
            tmem_ld32(trow + o_col + c * 32, orr);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * corr);
            tmem_st32(trow + o_col + c * 32, orr);
          }
          tmem_st_wait();
        }
        tc_fence_before();
        mbar_arrive(&sm->p_full[t]);
      }
      if (ok && mbar_wait_warp(&sm->o_done[t], (nblk - 1) & 1, abort_flag)) {
        tc_fence_after();
        const float inv = 1.f / l;
        __nv_bfloat16* orow = p.out + ((long long)r * p.Hq + head_s[t]) * kHD;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t orr[32];
          tmem_ld32(trow + o_col + c * 32, orr);
          tmem_ld_wait();
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(orr[2 * e]) * inv, __uint_as_float(orr[2 * e + 1]) * inv);
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
        }
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

// ------------------------------------------------------------------ host side
// [N, H, 128] bf16 -> 3-D map, box [64 elems][1 head][128 rows], 128-byte swizzle
bool make_map(CUtensorMap* tm, const void* ptr, int64_t N, int H) {
  TensorMapEncodeFn enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kHD, (cuuint64_t)H, (cuuint64_t)N};
  cuuint64_t strides[2] = {(cuuint64_t)kHD * 2, (cuuint64_t)H * kHD * 2};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_tree_attention_sm100(const AttnArgs& a, cudaStream_t stream, const SparseSel* sel) {
  if (a.num_tiles == 0) return cudaSuccess;
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, a.q, a.N, a.Hq) || !make_map(&tk, a.k, a.N, a.Hkv) || !make_map(&tv, a.v, a.N, a.Hkv))
    return cudaErrorInvalidValue;
  Params p;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.pos = a.pos;
  p.trunk_limit = a.trunk_limit;
  p.anc_bits = a.anc_bits;
  p.meta = a.meta;
  p.num_tiles = (int)a.num_tiles;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.G = a.Hq / a.Hkv;
  p.pairs = p.G / 2;
  p.items_per_pair = p.Hkv * (2 * p.pairs + 2 * (p.G & 1));
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.status = a.status;
  p.sel_mask = sel ? sel->mask : nullptr;
  p.sel_words = sel ? sel->words : 0;
  p.g = sel ? sel->g : 0;
  const size_t smem = sizeof(Smem) + 1024;
  auto kern = sel ? tree_attn_sm100_kernel<true> : tree_attn_sm100_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long grid = (long long)((a.num_tiles + 1) / 2) * p.items_per_pair;
  kern<<<(unsigned)grid, kThreads, smem, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace specopd
