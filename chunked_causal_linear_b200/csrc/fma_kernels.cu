// CUDA-core fp32 FMA kernels for K1 and K3 (float32 inputs, and bf16 inputs whose shape
// the tensor-core kernels do not cover).  One CTA per (b*H + h, chunk).  Everything is
// computed in float32 with fused multiply-adds; shared memory holds one chunk.
//
// K1 computes the chunk summaries
//   S_loc = sum_j Xi_j psi(k_j) v_j^T,  Z_loc = sum_j Xi_j psi(k_j),  Xi_j = gamma^(L-1-j)
// ("Log-Depth Chunked Linear-Attention Scan", "Formulas"; the decay weights follow the
// chunkwise retention form, "Linear Attention and Retentive Networks ...", "C. Chunkwise
// Recurrent Representation", read so that it equals the recurrent form).  Padded
// positions j >= L contribute zero ("Implementation notes").
//
// K3 evaluates, for each valid position i of the chunk,
//   num_i = Theta_i psi(q_i) P_c + sum_{j<=i} gamma^(i-j) (psi(q_i).psi(k_j)) v_j
//   den_i = Theta_i psi(q_i) ZP_c + sum_{j<=i} gamma^(i-j) (psi(q_i).psi(k_j))
//   o_i   = num_i / (den_i + eps)  or  num_i,      Theta_i = gamma^(i+1),
// where (P_c, ZP_c) is the exclusive prefix that K2 left in the chunk's record.  The
// intra-chunk part is computed here rather than handed over from K1 (both are exact).

#include <cuda_bf16.h>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace la {
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

constexpr int kFmaThreads = 256;

template <typename Tin, int FM, bool DECAY, bool NORM>
__global__ void __launch_bounds__(kFmaThreads)
k1_fma(const Tin* __restrict__ k, const Tin* __restrict__ v, PrefillParams p, GammaTable gt) {
  extern __shared__ float smem[];
  const int dk = p.dk, dv = p.dv, C = p.C;
  float* sK = smem;            // [C][dk], psi(k) * Xi, zero past the chunk end
  float* sV = sK + C * dk;     // [C][dv]
  const long long item = blockIdx.x;
  const int c = static_cast<int>(item % p.NC);
  const int bh = static_cast<int>(item / p.NC);
  const long long t0 = static_cast<long long>(c) * C;
  const int L = chunk_len(p, c);
  const float g = DECAY ? gt.g[bh % p.H] : 1.f;

  const Tin* kb = k + (static_cast<long long>(bh) * p.T + t0) * dk;
  const Tin* vb = v + (static_cast<long long>(bh) * p.T + t0) * dv;
  for (int e = threadIdx.x; e < C * dk; e += blockDim.x) {
    const int t = e / dk;
    float x = 0.f;
    if (t < L) {
      const float w = DECAY ? powf(g, static_cast<float>(L - 1 - t)) : 1.f;
      x = feature<FM>(to_f(kb[e])) * w;
    }
    sK[e] = x;
  }
  for (int e = threadIdx.x; e < C * dv; e += blockDim.x) {
    const int t = e / dv;
    sV[e] = t < L ? to_f(vb[e]) : 0.f;
  }
  __syncthreads();

  // The record holds S^T: element (j, i) = sum_t K'[t][i] V[t][j] at j * dk + i.
  float* rec = p.rec + (static_cast<long long>(bh) * p.NC + c) * p.R;
  for (int e = threadIdx.x; e < dk * dv; e += blockDim.x) {
    const int j = e / dk, i = e % dk;
    float acc = 0.f;
    for (int t = 0; t < C; ++t) acc = fmaf(sK[t * dk + i], sV[t * dv + j], acc);
    rec[e] = acc;
  }
  if (NORM) {
    for (int i = threadIdx.x; i < dk; i += blockDim.x) {
      float acc = 0.f;
      for (int t = 0; t < C; ++t) acc += sK[t * dk + i];
      rec[dk * dv + i] = acc;
    }
  }
}

template <typename Tin, typename Tout, int FM, bool DECAY, bool NORM>
__global__ void __launch_bounds__(kFmaThreads)
k3_fma(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
       Tout* __restrict__ out, PrefillParams p, GammaTable gt) {
  extern __shared__ float smem[];
  const int dk = p.dk, dv = p.dv, C = p.C;
  // Rows of dk + 1 and C + 1 floats: the loops below read one row per lane (sK, sP, and sQ,
  // sA in the denominators), and a stride of a multiple of 32 words would put every lane
  // on the same bank.
  const int ldk = dk + 1, lc = C + 1;
  float* sQ = smem;             // [C][ldk] psi(q)
  float* sK = sQ + C * ldk;     // [C][ldk] psi(k), zero past the chunk end
  float* sV = sK + C * ldk;     // [C][dv]
  float* sP = sV + C * dv;      // [dv][ldk] exclusive prefix state, transposed as stored
  float* sZP = sP + dv * ldk;   // [dk]
  float* sA = sZP + dk;         // [C][lc] masked, decayed scores
  float* sDen = sA + C * lc;    // [C]
  float* sTh = sDen + C;        // [C] Theta_i

  const long long item = blockIdx.x;
  const int c = static_cast<int>(item % p.NC);
  // Chunk 0 has a prefix too when the sequence continues from an initial state.
  const bool pre = c > 0 || p.has_init;
  const int bh = static_cast<int>(item / p.NC);
  const long long t0 = static_cast<long long>(c) * C;
  const int L = chunk_len(p, c);
  const float g = DECAY ? gt.g[bh % p.H] : 1.f;

  const Tin* qb = q + (static_cast<long long>(bh) * p.T + t0) * dk;
  const Tin* kb = k + (static_cast<long long>(bh) * p.T + t0) * dk;
  const Tin* vb = v + (static_cast<long long>(bh) * p.T + t0) * dv;
  for (int e = threadIdx.x; e < C * dk; e += blockDim.x) {
    const int t = e / dk, col = e % dk;
    const bool ok = t < L;
    sQ[t * ldk + col] = ok ? feature<FM>(to_f(qb[e])) : 0.f;
    sK[t * ldk + col] = ok ? feature<FM>(to_f(kb[e])) : 0.f;
  }
  for (int e = threadIdx.x; e < C * dv; e += blockDim.x) sV[e] = e / dv < L ? to_f(vb[e]) : 0.f;
  const float* rec = p.rec + (static_cast<long long>(bh) * p.NC + c) * p.R;
  for (int e = threadIdx.x; e < dk * dv; e += blockDim.x)
    sP[(e / dk) * ldk + e % dk] = pre ? rec[e] : 0.f;
  if (NORM)
    for (int i = threadIdx.x; i < dk; i += blockDim.x) sZP[i] = pre ? rec[dk * dv + i] : 0.f;
  for (int i = threadIdx.x; i < C; i += blockDim.x)
    sTh[i] = DECAY ? powf(g, static_cast<float>(i + 1)) : 1.f;
  __syncthreads();

  for (int e = threadIdx.x; e < C * C; e += blockDim.x) {
    const int i = e / C, j = e % C;
    float a = 0.f;
    if (j <= i && i < L) {
      for (int kk = 0; kk < dk; ++kk) a = fmaf(sQ[i * ldk + kk], sK[j * ldk + kk], a);
      // gamma^(i-j) from the Theta table: sTh[d - 1] = gamma^d, and gamma^0 = 1.
      if (DECAY && j < i) a *= sTh[i - j - 1];
    }
    sA[i * lc + j] = a;
  }
  __syncthreads();
  if (NORM) {
    for (int i = threadIdx.x; i < C; i += blockDim.x) {
      float inter = 0.f, loc = 0.f;
      for (int kk = 0; kk < dk; ++kk) inter = fmaf(sQ[i * ldk + kk], sZP[kk], inter);
      for (int j = 0; j <= i; ++j) loc += sA[i * lc + j];
      sDen[i] = fmaf(sTh[i], inter, loc) + p.eps;
    }
    __syncthreads();
  }
  Tout* ob = out + (static_cast<long long>(bh) * p.T + t0) * dv;
  for (int e = threadIdx.x; e < C * dv; e += blockDim.x) {
    const int i = e / dv, j = e % dv;
    if (i >= L) continue;
    float inter = 0.f, loc = 0.f;
    if (pre)
      for (int kk = 0; kk < dk; ++kk) inter = fmaf(sQ[i * ldk + kk], sP[j * ldk + kk], inter);
    for (int t = 0; t <= i; ++t) loc = fmaf(sA[i * lc + t], sV[t * dv + j], loc);
    float o = fmaf(sTh[i], inter, loc);
    if (NORM) o = o / sDen[i];
    ob[e] = from_f<Tout>(o);
  }
}

size_t k1_fma_smem(const PrefillParams& p) {
  return sizeof(float) * static_cast<size_t>(p.C) * (p.dk + p.dv);
}
size_t k3_fma_smem(const PrefillParams& p) {
  const size_t C = p.C, dk = p.dk, dv = p.dv;
  return sizeof(float) * (2 * C * (dk + 1) + C * dv + dv * (dk + 1) + dk + C * (C + 1) + 2 * C);
}

template <typename Kern>
cudaError_t set_smem(Kern kern, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(bytes));
}

template <typename Tin, int FM, bool DECAY, bool NORM>
cudaError_t k1_fma_go(const PrefillParams& p, const GammaTable& gt, const void* k,
                      const void* v, cudaStream_t s) {
  auto kern = k1_fma<Tin, FM, DECAY, NORM>;
  const size_t sm = k1_fma_smem(p);
  cudaError_t e = set_smem(kern, sm);
  if (e != cudaSuccess) return e;
  const long long grid = static_cast<long long>(p.BH) * p.NC;
  kern<<<static_cast<unsigned>(grid), kFmaThreads, sm, s>>>(
      static_cast<const Tin*>(k), static_cast<const Tin*>(v), p, gt);
  return cudaGetLastError();
}

template <typename Tin, typename Tout, int FM, bool DECAY, bool NORM>
cudaError_t k3_fma_go(const PrefillParams& p, const GammaTable& gt, const void* q,
                      const void* k, const void* v, void* out, cudaStream_t s) {
  auto kern = k3_fma<Tin, Tout, FM, DECAY, NORM>;
  const size_t sm = k3_fma_smem(p);
  cudaError_t e = set_smem(kern, sm);
  if (e != cudaSuccess) return e;
  const long long grid = static_cast<long long>(p.BH) * p.NC;
  kern<<<static_cast<unsigned>(grid), kFmaThreads, sm, s>>>(
      static_cast<const Tin*>(q), static_cast<const Tin*>(k), static_cast<const Tin*>(v),
      static_cast<Tout*>(out), p, gt);
  return cudaGetLastError();
}

// (fm, decay, norm) -> instantiation.  normalize with the identity map is rejected by the
// API before it gets here.
#define LA_DISPATCH_FLAGS(f, CALL)                                  \
  do {                                                              \
    if (f.fm == 1) {                                                \
      if (f.decay) {                                                \
        if (f.norm) return CALL(1, true, true);                     \
        return CALL(1, true, false);                                \
      }                                                             \
      if (f.norm) return CALL(1, false, true);                      \
      return CALL(1, false, false);                                 \
    }                                                               \
    if (f.decay) return CALL(0, true, false);                       \
    return CALL(0, false, false);                                   \
  } while (0)

}  // namespace

cudaError_t launch_k1_fma(const PrefillParams& p, const GammaTable& gt, const void* k,
                          const void* v, int dtype, Flags f, cudaStream_t s) {
  if (dtype == kF32) {
#define CALL(FM, D, N) k1_fma_go<float, FM, D, N>(p, gt, k, v, s)
    LA_DISPATCH_FLAGS(f, CALL);
#undef CALL
  } else {
#define CALL(FM, D, N) k1_fma_go<__nv_bfloat16, FM, D, N>(p, gt, k, v, s)
    LA_DISPATCH_FLAGS(f, CALL);
#undef CALL
  }
}

cudaError_t launch_k3_fma(const PrefillParams& p, const GammaTable& gt, const void* q,
                          const void* k, const void* v, void* out, int dtype, Flags f,
                          cudaStream_t s) {
  if (dtype == kF32) {
#define CALL(FM, D, N) k3_fma_go<float, float, FM, D, N>(p, gt, q, k, v, out, s)
    LA_DISPATCH_FLAGS(f, CALL);
#undef CALL
  } else if (f.out_f32) {
#define CALL(FM, D, N) k3_fma_go<__nv_bfloat16, float, FM, D, N>(p, gt, q, k, v, out, s)
    LA_DISPATCH_FLAGS(f, CALL);
#undef CALL
  } else {
#define CALL(FM, D, N) k3_fma_go<__nv_bfloat16, __nv_bfloat16, FM, D, N>(p, gt, q, k, v, out, s)
    LA_DISPATCH_FLAGS(f, CALL);
#undef CALL
  }
}

}  // namespace la
