// K3f: tree-masked GQA attention on the CUDA cores (fp32 arithmetic).
//
// The same operation as the tcgen05 kernel (SpecOPD listing, Fig 3: each row
// attends to itself and its ancestors), for inputs the tensor-core kernel does
// not take: fp32 Q/K/V (whose tolerance rules out TF32 tensor-core products)
// and bf16 heads with d != 128.
//
// One warp per (row, query head); lane l holds elements [l*DPL, (l+1)*DPL) of
// the rotated query.  The warp walks exactly the visible columns -- the trunk
// prefix up to the row's trunk limit, then the set bits of its ancestor mask --
// with an online softmax in base 2.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace specopd {
namespace {

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

template <typename T, int DPL>
__global__ void __launch_bounds__(128) tree_attn_simt_kernel(const AttnArgs a, float scale_log2) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int tile = blockIdx.x;
  const int h = blockIdx.y;
  const int d = a.d;
  const int G = a.Hq / a.Hkv;
  const int kvh = h / G;
  const specopd_tile_meta m = a.meta[tile];
  const T* Q = static_cast<const T*>(a.q);
  const T* K = static_cast<const T*>(a.k);
  const T* Vv = static_cast<const T*>(a.v);
  T* O = static_cast<T*>(a.out);

  for (int r = m.row_start + warp; r < m.row_end; r += 4) {
    const int tl = a.trunk_limit[r];
    const int lim = m.tree_base + tl;
    const int i = a.pos[r] - tl;          // sample index on a branch, 0 on the trunk
    const int bstart = r - i + 1;         // row of y_{b,1}
    const uint64_t bits = a.anc_bits[r];
    float qv[DPL], acc[DPL];
    const T* qrow = Q + ((long long)r * a.Hq + h) * d + lane * DPL;
#pragma unroll
    for (int e = 0; e < DPL; ++e) {
      qv[e] = to_f(qrow[e]);
      acc[e] = 0.f;
    }
    float mrun = -INFINITY, l = 0.f;
    auto visit = [&](int c) {
      const T* krow = K + ((long long)c * a.Hkv + kvh) * d + lane * DPL;
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < DPL; ++e) dot = fmaf(qv[e], to_f(krow[e]), dot);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
      const float s = dot * scale_log2;
      const float mnew = fmaxf(mrun, s);
      const float corr = ex2(mrun - mnew);
      const float p = ex2(s - mnew);
      l = l * corr + p;
      const T* vrow = Vv + ((long long)c * a.Hkv + kvh) * d + lane * DPL;
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] = fmaf(p, to_f(vrow[e]), acc[e] * corr);
      mrun = mnew;
    };
    for (int c = m.tree_base; c <= lim; ++c) visit(c);
    uint64_t b = bits;
    while (b) {
      const int k = __ffsll((long long)b) - 1;
      b &= b - 1;
      visit(bstart + k);
    }
    const float inv = 1.f / l;
    T* orow = O + ((long long)r * a.Hq + h) * d + lane * DPL;
#pragma unroll
    for (int e = 0; e < DPL; ++e) orow[e] = from_f<T>(acc[e] * inv);
  }
}

template <typename T>
cudaError_t launch_t(const AttnArgs& a, cudaStream_t stream) {
  const float scale_log2 = a.scale * 1.4426950408889634f;
  dim3 grid((unsigned)a.num_tiles, (unsigned)a.Hq);
  switch (a.d / 32) {
    case 1: tree_attn_simt_kernel<T, 1><<<grid, 128, 0, stream>>>(a, scale_log2); break;
    case 2: tree_attn_simt_kernel<T, 2><<<grid, 128, 0, stream>>>(a, scale_log2); break;
    case 3: tree_attn_simt_kernel<T, 3><<<grid, 128, 0, stream>>>(a, scale_log2); break;
    case 4: tree_attn_simt_kernel<T, 4><<<grid, 128, 0, stream>>>(a, scale_log2); break;
    case 5: tree_attn_simt_kernel<T, 5><<<grid, 128, 0, stream>>>(a, scale_log2); break;
    case 6: tree_attn_simt_kernel<T, 6><<<grid, 128, 0, stream>>>(a, scale_log2); break;
    case 7: tree_attn_simt_kernel<T, 7><<<grid, 128, 0, stream>>>(a, scale_log2); break;
    case 8: tree_attn_simt_kernel<T, 8><<<grid, 128, 0, stream>>>(a, scale_log2); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_tree_attention_simt(const AttnArgs& a, specopd_dtype dtype, cudaStream_t stream) {
  if (a.num_tiles == 0) return cudaSuccess;
  return dtype == SPECOPD_BF16 ? launch_t<__nv_bfloat16>(a, stream) : launch_t<float>(a, stream);
}

}  // namespace specopd
