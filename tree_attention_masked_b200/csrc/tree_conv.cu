// K9: short causal convolution along each packed row's own history.
//
// SpecOPD (thelatestinai.com listing), Fig 5: in the GDN branch path the
// causal convolution follows branch ancestry -- a branch token's window holds
// its own history (the trunk through its anchor, then its branch's earlier
// samples), not its packed neighbours.  Reading (the figure prints no
// formula): a depthwise causal convolution of width Kw,
//   out[r, c] = act(bias[c] + sum_{j<Kw} weight[c, j] x[h_j(r), c]),
// h_j(r) the row j steps back in r's history (zero before its start), act the
// identity or SiLU.
//
// HBM-bound: one thread per (row, 16-byte group of channels).  The history
// rows of a row follow from the mask builder's fields: with p = pos[r] and
// a = trunk_limit[r], the row's own branch samples are the i = p - a packed
// rows ending at r (none on the trunk), and lag L >= i reads trunk token
// a - (L - i) of the row's tree.  fp32 arithmetic, output in the input dtype.
#include <cuda_bf16.h>

#include "internal.h"

namespace specopd {
namespace {

constexpr int kConvThreads = 256;

template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int n = 8;
  __device__ static void load(const __nv_bfloat16* p, float* v) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __device__ static void store(__nv_bfloat16* p, const float* v) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
      w[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
  }
};
template <>
struct Vec<float> {
  static constexpr int n = 4;
  __device__ static void load(const float* p, float* v) {
    const float4 u = *reinterpret_cast<const float4*>(p);
    v[0] = u.x;
    v[1] = u.y;
    v[2] = u.z;
    v[3] = u.w;
  }
  __device__ static void store(float* p, const float* v) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};

template <typename T>
__global__ void __launch_bounds__(kConvThreads) tree_conv_kernel(const T* __restrict__ x, T* __restrict__ out,
                                                                 int64_t N, int C, const float* __restrict__ w,
                                                                 const float* __restrict__ bias, int Kw, int silu,
                                                                 const int32_t* __restrict__ pos,
                                                                 const int32_t* __restrict__ trunk_limit,
                                                                 const int32_t* __restrict__ cu_rows, int num_trees) {
  constexpr int V = Vec<T>::n;
  const int groups = C / V;
  const long long idx = (long long)blockIdx.x * kConvThreads + threadIdx.x;
  if (idx >= N * groups) return;
  const long long r = idx / groups;
  const int c0 = (int)(idx % groups) * V;
  // the row's tree: last tree whose first row is <= r
  int lo = 0, hi = num_trees - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) / 2;
    if (cu_rows[mid] <= r) lo = mid; else hi = mid - 1;
  }
  const long long base = cu_rows[lo];
  const int a = trunk_limit[r];
  const int own = pos[r] - a;  // the row's branch samples up to itself (0 on the trunk)
  float acc[V];
#pragma unroll
  for (int e = 0; e < V; ++e) acc[e] = bias ? bias[c0 + e] : 0.f;
  for (int L = 0; L < Kw; ++L) {
    long long src;
    if (L < own) {
      src = r - L;
    } else {
      const int j = a - (L - own);
      if (j < 0) break;  // before the start of the history: zero
      src = base + j;
    }
    float xv[V];
    Vec<T>::load(x + src * C + c0, xv);
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = fmaf(w[(c0 + e) * Kw + L], xv[e], acc[e]);
  }
  if (silu) {
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = acc[e] / (1.f + __expf(-acc[e]));
  }
  Vec<T>::store(out + r * C + c0, acc);
}

}  // namespace

cudaError_t launch_tree_conv(const void* x, void* out, specopd_dtype dtype, int64_t N, int C, const float* w,
                             const float* bias, int Kw, int silu, const int32_t* pos, const int32_t* trunk_limit,
                             const int32_t* cu_rows, int num_trees, cudaStream_t stream) {
  const int V = dtype == SPECOPD_BF16 ? 8 : 4;
  const long long items = N * (long long)(C / V);
  if (items == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((items + kConvThreads - 1) / kConvThreads);
  if (dtype == SPECOPD_BF16)
    tree_conv_kernel<__nv_bfloat16><<<grid, kConvThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(x), static_cast<__nv_bfloat16*>(out), N, C, w, bias, Kw, silu, pos,
        trunk_limit, cu_rows, num_trees);
  else
    tree_conv_kernel<float><<<grid, kConvThreads, 0, stream>>>(static_cast<const float*>(x),
                                                               static_cast<float*>(out), N, C, w, bias, Kw, silu,
                                                               pos, trunk_limit, cu_rows, num_trees);
  return cudaGetLastError();
}

}  // namespace specopd
