// One recurrent decode step for every (b, h):
//   S <- gamma S + psi(k) v^T,  Z <- gamma Z + psi(k),
//   o  = psi(q) S / (psi(q) . Z + eps)   or   psi(q) S
// ("Linear Attention and Retentive Networks ...", "The Recurrent Dual" and
// "B. Recurrent Representation").  The step is memory-bound: each state element is read
// and written once, 8 dk dv bytes of state traffic per (b, h).
//
// decode_tiles (dk a multiple of 16 up to 128, dv a multiple of 4 up to 256, 16-byte
// aligned tensors): the state of one (b, h) is cut into tiles of 16 or 64 rows (key
// features), one CTA each, and those CTAs form one thread-block cluster.  A thread streams
// float4 columns of its rows (every row is contiguous), so a step is one wave of
// independent 16-byte loads over the whole GPU.  Each CTA reduces psi(q) . S over its rows
// in shared memory; the cluster then adds the tiles' partial outputs (and denominators)
// through distributed shared memory in a fixed order, each CTA finishing a share of the
// value features.  No atomics and no scratch memory: the result does not depend on timing.
// decode_step (any dk, dv up to 256): one CTA per (b, h), thread j streams state column j.

#include <cooperative_groups.h>
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

constexpr int kTileRows = 16;
constexpr int kTileThreads = 256;

// Four consecutive values as float (bf16: one 8-byte load; float: one 16-byte load).
__device__ __forceinline__ float4 ld4(const float* p, long long i) {
  return *reinterpret_cast<const float4*>(p + i);
}
__device__ __forceinline__ float4 ld4(const __nv_bfloat16* p, long long i) {
  const uint2 u = *reinterpret_cast<const uint2*>(p + i);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ void st4(float* p, long long i, float4 x) {
  *reinterpret_cast<float4*>(p + i) = x;
}
__device__ __forceinline__ void st4(__nv_bfloat16* p, long long i, float4 x) {
  __nv_bfloat162 a = __floats2bfloat162_rn(x.x, x.y), b = __floats2bfloat162_rn(x.z, x.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p + i) = u;
}

// RPT: rows per thread, at least ceil(TR / row lanes).  It is a template argument so that
// the state registers are only the rows a thread really holds (at TR = 64 and dv = 128, 8
// float4 instead of 16: 64 registers instead of ~110, four CTAs per SM instead of two).
template <typename T, int FM, bool DECAY, bool NORM, int TR, int RPT>
__global__ void __launch_bounds__(kTileThreads)
decode_tiles(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
             T* __restrict__ out, float* __restrict__ S, float* __restrict__ Z, int H, int dk,
             int dv, float eps, GammaTable gt) {
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  __shared__ float sq[TR], sk[TR];
  __shared__ float4 sAcc[kTileThreads];
  __shared__ float4 sPart[64];  // this tile's partial psi(q) . S, dv / 4 float4
  __shared__ float sDen;
  const int nt = static_cast<int>(cl.num_blocks());
  const int rank = static_cast<int>(cl.block_rank());
  const int bh = blockIdx.x / nt;
  const int i0 = rank * TR;
  const int tid = threadIdx.x;
  const float g = DECAY ? gt.g[bh % H] : 1.f;

  // The tile's state rows first (they depend on nothing else): thread (row lane rl,
  // float4 column c4) loads rows rl, rl + lanes, ... of the tile.
  const int dv4 = dv / 4;
  const int lanes = kTileThreads / dv4;  // row lanes (>= 4)
  const int c4 = tid % dv4, rl = tid / dv4;
  const bool active = rl < lanes && rl < TR;
  constexpr int kMax = RPT;  // rows per thread: RPT * lanes >= TR
  float* Sb = S + (static_cast<long long>(bh) * dk + i0) * dv + 4 * c4;
  float4 s[kMax];
  if (active) {
#pragma unroll
    for (int m = 0; m < kMax; ++m) {
      const int r = rl + m * lanes;
      if (r < TR) s[m] = *reinterpret_cast<const float4*>(Sb + static_cast<long long>(r) * dv);
    }
  }
  float4 vj = make_float4(0.f, 0.f, 0.f, 0.f);
  if (active) vj = ld4(v, static_cast<long long>(bh) * dv + 4 * c4);

  if (tid < 32 * ((TR + 31) / 32)) {
    // Rows i0 .. i0 + TR - 1: psi(q), psi(k), the Z update and this tile's psi(q) . Z.
    float part = 0.f;
    if (tid < TR) {
      const long long i = static_cast<long long>(bh) * dk + i0 + tid;
      const float fq = feature<FM>(static_cast<float>(q[i]));
      const float fk = feature<FM>(static_cast<float>(k[i]));
      sq[tid] = fq;
      sk[tid] = fk;
      if (Z) {
        const float z = fmaf(g, Z[i], fk);
        Z[i] = z;
        part = fq * z;
      }
    }
    if (NORM) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
      if ((tid & 31) == 0) sAcc[tid >> 5].x = part;  // per-warp sums, read below
    }
  }
  __syncthreads();
  if (NORM && tid == 0) {
    float d = 0.f;
    for (int w = 0; w < (TR + 31) / 32; ++w) d += sAcc[w].x;
    sDen = d;
  }
  __syncthreads();

  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (active) {
#pragma unroll
    for (int m = 0; m < kMax; ++m) {
      const int r = rl + m * lanes;
      if (r < TR) {
        const float a = sk[r], b = sq[r];
        float4 x = s[m];
        x.x = fmaf(a, vj.x, g * x.x);
        x.y = fmaf(a, vj.y, g * x.y);
        x.z = fmaf(a, vj.z, g * x.z);
        x.w = fmaf(a, vj.w, g * x.w);
        *reinterpret_cast<float4*>(Sb + static_cast<long long>(r) * dv) = x;
        acc.x = fmaf(b, x.x, acc.x);
        acc.y = fmaf(b, x.y, acc.y);
        acc.z = fmaf(b, x.z, acc.z);
        acc.w = fmaf(b, x.w, acc.w);
      }
    }
  }
  sAcc[tid] = acc;
  __syncthreads();
  if (tid < dv4) {
    float4 t = sAcc[tid];
    for (int r = 1; r < lanes && r < TR; ++r) {
      const float4 u = sAcc[r * dv4 + tid];
      t.x += u.x;
      t.y += u.y;
      t.z += u.z;
      t.w += u.w;
    }
    sPart[tid] = t;
  }
  cl.sync();
  // Value features c4 = rank, rank + nt, ...: the tiles' partials added in rank order.
  for (int c = rank + nt * tid; c < dv4; c += nt * kTileThreads) {
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    float den = 0.f;
    for (int j = 0; j < nt; ++j) {
      const float4 u = *cl.map_shared_rank(&sPart[c], j);
      o.x += u.x;
      o.y += u.y;
      o.z += u.z;
      o.w += u.w;
      if (NORM) den += *cl.map_shared_rank(&sDen, j);
    }
    if (NORM) {
      const float d = den + eps;
      o.x /= d;
      o.y /= d;
      o.z /= d;
      o.w /= d;
    }
    st4(out, static_cast<long long>(bh) * dv + 4 * c, o);
  }
  cl.sync();  // no CTA leaves while another still reads its shared memory
}

// Rows per CTA: 64 (four tiles in flight per thread pair of rows: 8 loads of 16 bytes per
// thread at dv = 128) when that still gives every SM two CTAs, else 16.
int tile_rows(long long BH, int dk) {
  if (dk % 64 == 0 && BH * (dk / 64) >= 2 * 148) return 64;
  return 16;
}

bool tiles_ok(const void* q, const void* k, const void* v, const void* out, const float* S,
              const float* Z, int dk, int dv) {
  auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  return dk % kTileRows == 0 && dk <= 8 * kTileRows && dv % 4 == 0 && dv <= 256 && a16(q) &&
         a16(k) && a16(v) && a16(out) && a16(S) && a16(Z);
}

template <typename T, int FM, bool DECAY, bool NORM, int TR, int RPT>
cudaError_t go_tiles_r(const void* q, const void* k, const void* v, void* out, float* S,
                       float* Z, int BH, int H, int dk, int dv, float eps, const GammaTable& gt,
                       cudaStream_t s) {
  const int nt = dk / TR;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(BH) * nt);
  cfg.blockDim = dim3(kTileThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = nt;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_tiles<T, FM, DECAY, NORM, TR, RPT>, static_cast<const T*>(q),
                            static_cast<const T*>(k), static_cast<const T*>(v),
                            static_cast<T*>(out), S, Z, H, dk, dv, eps, gt);
}

template <typename T, int FM, bool DECAY, bool NORM>
cudaError_t go_tiles(const void* q, const void* k, const void* v, void* out, float* S, float* Z,
                     int BH, int H, int dk, int dv, float eps, const GammaTable& gt,
                     cudaStream_t s) {
  // Row lanes = threads / (dv / 4) >= 4 (dv <= 256); each thread takes ceil(TR / lanes) rows.
  const int lanes = kTileThreads / (dv / 4);
  if (tile_rows(BH, dk) == 64) {
    const int rpt = (64 + lanes - 1) / lanes;
    if (rpt <= 4)
      return go_tiles_r<T, FM, DECAY, NORM, 64, 4>(q, k, v, out, S, Z, BH, H, dk, dv, eps, gt, s);
    if (rpt <= 8)
      return go_tiles_r<T, FM, DECAY, NORM, 64, 8>(q, k, v, out, S, Z, BH, H, dk, dv, eps, gt, s);
    return go_tiles_r<T, FM, DECAY, NORM, 64, 16>(q, k, v, out, S, Z, BH, H, dk, dv, eps, gt, s);
  }
  return go_tiles_r<T, FM, DECAY, NORM, 16, 4>(q, k, v, out, S, Z, BH, H, dk, dv, eps, gt, s);
}

template <typename T, int FM, bool DECAY, bool NORM>
cudaError_t go(const void* q, const void* k, const void* v, void* out, float* S, float* Z,
               int BH, int H, int dk, int dv, float eps, const GammaTable& gt, cudaStream_t s) {
  if (tiles_ok(q, k, v, out, S, Z, dk, dv))
    return go_tiles<T, FM, DECAY, NORM>(q, k, v, out, S, Z, BH, H, dk, dv, eps, gt, s);
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
