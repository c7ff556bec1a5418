// One recurrent decode step for every (b, h):
//   S <- gamma S + psi(k) v^T,  Z <- gamma Z + psi(k),
//   o  = psi(q) S / (psi(q) . Z + eps)   or   psi(q) S
// ("Linear Attention and Retentive Networks ...", "The Recurrent Dual" and
// "B. Recurrent Representation").  One CTA per (b, h); thread j owns value column j and
// streams the state column S[:, j] (coalesced across threads), so each state element is
// read and written exactly once.  The step is memory-bound: 8 dk dv bytes of state
// traffic per (b, h).

#include <cuda_bf16.h>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace la {
namespace {

constexpr int kDecThreads = 256;

template <typename T>
__device__ __forceinline__ float ld_f(const T* p, long long i);
template <>
__device__ __forceinline__ float ld_f<float>(const float* p, long long i) { return p[i]; }
template <>
__device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16* p, long long i) {
  return __bfloat162float(p[i]);
}
template <typename T>
__device__ __forceinline__ void st_f(T* p, long long i, float x);
template <>
__device__ __forceinline__ void st_f<float>(float* p, long long i, float x) { p[i] = x; }
template <>
__device__ __forceinline__ void st_f<__nv_bfloat16>(__nv_bfloat16* p, long long i, float x) {
  p[i] = __float2bfloat16_rn(x);
}

template <typename T, int FM, bool DECAY, bool NORM>
__global__ void __launch_bounds__(kDecThreads)
decode_step(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
            T* __restrict__ out, float* __restrict__ S, float* __restrict__ Z, int H, int dk,
            int dv, float eps, GammaTable gt) {
  __shared__ float sq[256], sk[256];
  __shared__ float red[kDecThreads / 32];
  const int bh = blockIdx.x;
  const float g = DECAY ? gt.g[bh % H] : 1.f;
  for (int i = threadIdx.x; i < dk; i += blockDim.x) {
    sq[i] = feature<FM>(ld_f(q, static_cast<long long>(bh) * dk + i));
    sk[i] = feature<FM>(ld_f(k, static_cast<long long>(bh) * dk + i));
  }
  __syncthreads();

  float den_part = 0.f;
  if (NORM) {
    for (int i = threadIdx.x; i < dk; i += blockDim.x) {
      const long long zi = static_cast<long long>(bh) * dk + i;
      const float z = fmaf(g, Z[zi], sk[i]);
      Z[zi] = z;
      den_part = fmaf(sq[i], z, den_part);
    }
  } else if (Z) {
    for (int i = threadIdx.x; i < dk; i += blockDim.x) {
      const long long zi = static_cast<long long>(bh) * dk + i;
      Z[zi] = fmaf(g, Z[zi], sk[i]);
    }
  }
  float den = 0.f;
  if (NORM) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den_part += __shfl_xor_sync(0xffffffffu, den_part, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = den_part;
    __syncthreads();
    for (int w = 0; w < kDecThreads / 32; ++w) den += red[w];
  }

  float* Sb = S + static_cast<long long>(bh) * dk * dv;
  for (int j = threadIdx.x; j < dv; j += blockDim.x) {
    const float vj = ld_f(v, static_cast<long long>(bh) * dv + j);
    float acc = 0.f;
    for (int i = 0; i < dk; ++i) {
      const long long e = static_cast<long long>(i) * dv + j;
      const float s = fmaf(sk[i], vj, g * Sb[e]);
      Sb[e] = s;
      acc = fmaf(sq[i], s, acc);
    }
    if (NORM) acc = acc / (den + eps);
    st_f(out, static_cast<long long>(bh) * dv + j, acc);
  }
}

template <typename T, int FM, bool DECAY, bool NORM>
cudaError_t go(const void* q, const void* k, const void* v, void* out, float* S, float* Z,
               int BH, int H, int dk, int dv, float eps, const GammaTable& gt, cudaStream_t s) {
  decode_step<T, FM, DECAY, NORM><<<BH, kDecThreads, 0, s>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v),
      static_cast<T*>(out), S, Z, H, dk, dv, eps, gt);
  return cudaGetLastError();
}

template <typename T>
cudaError_t dispatch(const void* q, const void* k, const void* v, void* out, float* S,
                     float* Z, int BH, int H, int dk, int dv, Flags f, const GammaTable& gt,
                     float eps, cudaStream_t s) {
  if (f.fm == 1) {
    if (f.decay) {
      if (f.norm) return go<T, 1, true, true>(q, k, v, out, S, Z, BH, H, dk, dv, eps, gt, s);
      return go<T, 1, true, false>(q, k, v, out, S, Z, BH, H, dk, dv, eps, gt, s);
    }
    if (f.norm) return go<T, 1, false, true>(q, k, v, out, S, Z, BH, H, dk, dv, eps, gt, s);
    return go<T, 1, false, false>(q, k, v, out, S, Z, BH, H, dk, dv, eps, gt, s);
  }
  if (f.decay) return go<T, 0, true, false>(q, k, v, out, S, Z, BH, H, dk, dv, eps, gt, s);
  return go<T, 0, false, false>(q, k, v, out, S, Z, BH, H, dk, dv, eps, gt, s);
}

}  // namespace

cudaError_t launch_decode(const void* q, const void* k, const void* v, void* out, float* S,
                          float* Z, int BH, int H, int dk, int dv, int dtype, Flags f,
                          const GammaTable& gt, float eps, int* /*err*/, cudaStream_t s) {
  if (dtype == kF32) return dispatch<float>(q, k, v, out, S, Z, BH, H, dk, dv, f, gt, eps, s);
  return dispatch<__nv_bfloat16>(q, k, v, out, S, Z, BH, H, dk, dv, f, gt, eps, s);
}

}  // namespace la
