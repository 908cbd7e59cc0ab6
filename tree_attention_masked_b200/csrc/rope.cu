// K2: rotate-half rotary embedding of Q and K at semantic positions.
//
// daiwk.github.io write-up of SpecOPD, section "Equations": branch token
// y_{b,i} takes position a_b + i, not its packed offset.  Element k of a head
// pairs with element k + d/2 and both rotate by pos * theta^(-2k/d).
//
// One CTA per packed row.  The d/2 angles are formed in fp64 and reduced to
// fp32 cos/sin once per row; every head of the row then reuses them.  Each
// thread rotates two adjacent frequency pairs of one head (vector loads).
#include <cuda_bf16.h>

#include "internal.h"

namespace specopd {
namespace {

template <typename T>
struct Vec2;
template <>
struct Vec2<float> {
  using type = float2;
  __device__ static float2 to_f(float2 v) { return v; }
  __device__ static float2 from_f(float2 v) { return v; }
};
template <>
struct Vec2<__nv_bfloat16> {
  using type = __nv_bfloat162;
  __device__ static float2 to_f(__nv_bfloat162 v) { return __bfloat1622float2(v); }
  __device__ static __nv_bfloat162 from_f(float2 v) { return __float22bfloat162_rn(v); }
};

template <typename T>
__global__ void __launch_bounds__(256) rope_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                   T* __restrict__ q_out, T* __restrict__ k_out, int Hq, int Hkv,
                                                   int d, const int32_t* __restrict__ pos, float theta) {
  using V2 = typename Vec2<T>::type;
  __shared__ float s_cos[128], s_sin[128];
  const long long r = blockIdx.x;
  const int half = d >> 1;
  const int p = pos[r];
  for (int j = threadIdx.x; j < half; j += blockDim.x) {
    const double inv_freq = pow((double)theta, -2.0 * (double)j / (double)d);
    double s, c;
    sincos((double)p * inv_freq, &s, &c);
    s_cos[j] = (float)c;
    s_sin[j] = (float)s;
  }
  __syncthreads();
  const int pairs = half >> 1;  // two frequencies per thread
  const int total = (Hq + Hkv) * pairs;
  for (int idx = threadIdx.x; idx < total; idx += blockDim.x) {
    const int h = idx / pairs;
    const int j = (idx - h * pairs) * 2;
    const T* src;
    T* dst;
    if (h < Hq) {
      src = q + (r * Hq + h) * d;
      dst = q_out + (r * Hq + h) * d;
    } else {
      src = k + (r * Hkv + (h - Hq)) * d;
      dst = k_out + (r * Hkv + (h - Hq)) * d;
    }
    const float2 x1 = Vec2<T>::to_f(*reinterpret_cast<const V2*>(src + j));
    const float2 x2 = Vec2<T>::to_f(*reinterpret_cast<const V2*>(src + j + half));
    const float c0 = s_cos[j], c1 = s_cos[j + 1], s0 = s_sin[j], s1 = s_sin[j + 1];
    float2 y1, y2;
    y1.x = x1.x * c0 - x2.x * s0;
    y1.y = x1.y * c1 - x2.y * s1;
    y2.x = x2.x * c0 + x1.x * s0;
    y2.y = x2.y * c1 + x1.y * s1;
    *reinterpret_cast<V2*>(dst + j) = Vec2<T>::from_f(y1);
    *reinterpret_cast<V2*>(dst + j + half) = Vec2<T>::from_f(y2);
  }
}


// Vectorised form for d a multiple of 16: each thread rotates 8 consecutive
// frequency pairs of one head with 16-byte loads and stores.
template <typename T>
struct Vec8;
template <>
struct Vec8<__nv_bfloat16> {
  __device__ static void load(const __nv_bfloat16* p, float (&x)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
  __device__ static void store(__nv_bfloat16* p, const float (&x)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 b = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
      w[i] = *reinterpret_cast<const uint32_t*>(&b);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
  }
};
template <>
struct Vec8<float> {
  __device__ static void load(const float* p, float (&x)[8]) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    const float4 b = *reinterpret_cast<const float4*>(p + 4);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
  __device__ static void store(float* p, const float (&x)[8]) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
    *reinterpret_cast<float4*>(p + 4) = make_float4(x[4], x[5], x[6], x[7]);
  }
};

template <typename T>
__global__ void __launch_bounds__(128) rope_vec_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                       T* __restrict__ q_out, T* __restrict__ k_out, int Hq,
                                                       int Hkv, int d, const int32_t* __restrict__ pos,
                                                       float theta) {
  __shared__ float s_cos[128], s_sin[128];
  const long long r = blockIdx.x;
  const int half = d >> 1;
  const int p = pos[r];
  for (int j = threadIdx.x; j < half; j += blockDim.x) {
    const double inv_freq = pow((double)theta, -2.0 * (double)j / (double)d);
    double s, c;
    sincos((double)p * inv_freq, &s, &c);
    s_cos[j] = (float)c;
    s_sin[j] = (float)s;
  }
  __syncthreads();
  const int per_head = half / 8;
  const int total = (Hq + Hkv) * per_head;
  for (int idx = threadIdx.x; idx < total; idx += blockDim.x) {
    const int h = idx / per_head;
    const int j = (idx - h * per_head) * 8;
    const T* src;
    T* dst;
    if (h < Hq) {
      src = q + (r * Hq + h) * d;
      dst = q_out + (r * Hq + h) * d;
    } else {
      src = k + (r * Hkv + (h - Hq)) * d;
      dst = k_out + (r * Hkv + (h - Hq)) * d;
    }
    float x1[8], x2[8], y1[8], y2[8];
    Vec8<T>::load(src + j, x1);
    Vec8<T>::load(src + j + half, x2);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float c = s_cos[j + i], s = s_sin[j + i];
      y1[i] = x1[i] * c - x2[i] * s;
      y2[i] = x2[i] * c + x1[i] * s;
    }
    Vec8<T>::store(dst + j, y1);
    Vec8<T>::store(dst + j + half, y2);
  }
}

}  // namespace

cudaError_t launch_rope(const void* q, const void* k, void* q_out, void* k_out, specopd_dtype dtype, int64_t N,
                        int Hq, int Hkv, int d, const int32_t* pos, float theta, cudaStream_t stream) {
  if (N == 0) return cudaSuccess;
  const unsigned grid = (unsigned)N;
  if (d % 16 == 0) {
    if (dtype == SPECOPD_BF16)
      rope_vec_kernel<__nv_bfloat16><<<grid, 128, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
          static_cast<__nv_bfloat16*>(q_out), static_cast<__nv_bfloat16*>(k_out), Hq, Hkv, d, pos, theta);
    else
      rope_vec_kernel<float><<<grid, 128, 0, stream>>>(static_cast<const float*>(q), static_cast<const float*>(k),
                                                       static_cast<float*>(q_out), static_cast<float*>(k_out), Hq,
                                                       Hkv, d, pos, theta);
    return cudaGetLastError();
  }
  if (dtype == SPECOPD_BF16) {
    rope_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<__nv_bfloat16*>(q_out), static_cast<__nv_bfloat16*>(k_out), Hq, Hkv, d, pos, theta);
  } else {
    rope_kernel<float><<<grid, 256, 0, stream>>>(static_cast<const float*>(q), static_cast<const float*>(k),
                                                 static_cast<float*>(q_out), static_cast<float*>(k_out), Hq, Hkv,
                                                 d, pos, theta);
  }
  return cudaGetLastError();
}

}  // namespace specopd
