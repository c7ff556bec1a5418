// Gated linear attention: the data-dependent decay of "Linear Attention and Retentive
// Networks ..." (Gated Linear Attention (GLA) and Hardware-Software Co-Design):
//     S_t = (alpha_t 1^T) (.) S_{t-1} + k_t^T v_t,      o_t = q_t S_t,
// alpha_t a per-token, per-key-feature gate in [0, 1].  The scan page's three kernels with
// the decayed monoid generalised from a scalar to a diagonal: a chunk scales what came before
// it by a_c = prod_{j in c} alpha_j (a dk-vector), so (a1, S1) + (a2, S2) = (a1 a2,
// diag(a2) S1 + S2) ("Log-Depth Chunked Linear-Attention Scan", Formulas, with the decay of
// "C. Chunkwise Recurrent Representation" made per feature).  Within a chunk, with
// L_j = sum_{r<=j} log alpha_r (per feature, from the chunk start):
//   K1  S_loc = sum_j (k_j (.) e^(L_last - L_j)) v_j^T,   a_c = e^(L_last)
//   K2  P_c = the exclusive prefix of (a_c, S_loc) over chunks (a carry per state element)
//   K3  o_j = (q_j (.) e^(L_j)) P_c + sum_{i<=j} (sum_f q_j[f] k_i[f] e^(L_j[f] - L_i[f])) v_i
// The kernels form these as powers of two of cumulative log2 gates, every exponent <= 0,
// so nothing overflows whatever the gates (a gate below 2^-126 counts as 2^-126).  Two paths:
//   Tensor cores (default for bf16, C = 64, dk in {64, 128}, dv = 128; gla_seg.cu): the
//     segmented arrangement on tcgen05 with hi / lo split factored operands.  Chunks whose
//     gates are too small for the factored scores are flagged there, and gla_k3 in fix-up
//     mode adds their exact intra-chunk part.
//   CUDA cores (every other shape, or kernel_path LA_PATH_FMA; gla_k1, gla_k2, gla_k3):
//     exact in float32 for any gates.  K3's scores factor as (q (.) 2^L) . (k (.) 2^-L) when
//     the chunk's logs stay >= -100 (plain dot products), else take one exponential per
//     (pair, feature).

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "../../include/linattn.h"
#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace la {
namespace {

// The intra-chunk weights factor into q 2^(L) and k 2^(-L) while L >= -kGlaFactorBound.
constexpr float kGlaFactorBound = 100.f;
constexpr int kGlaThreads = 512;  // 16 warps: one or two CTAs per SM, latency hidden by warps

struct GlaParams {
  int BH;
  long long T;
  int dk, dv, C;
  int NC;        // chunks
  int L_last;    // tokens in the last chunk
  int R;         // floats per record: S [dk][dv] then a [dk]
  const void* q;
  const void* k;
  const void* v;
  const float* alpha;
  void* out;
  bool in_f32, out_f32;
  float* rec;    // [BH][NC][R]
  const float* S_init;
  float* S_final;
  // Fix-up mode of gla_k3: [BH][NC] flags; only flagged chunks run, they compute the
  // intra-chunk part alone and add it to `out` (which holds the prefix part).
  const unsigned char* steep;
};

__device__ __forceinline__ int chunk_len(const GlaParams& p, int c) {
  return c == p.NC - 1 ? p.L_last : p.C;
}

// Loads rows [t0, t0 + L) of a [T, d] slice into sm[r * lds + f] as float32 (rows >= L zero),
// eight elements per access (d is a multiple of 8): 16-byte loads of bf16, two of float32.
__device__ __forceinline__ void load_rows(float* sm, int lds, const void* g, bool f32,
                                          long long base, int d, int C, int L) {
  const int g8 = d / 8;
  for (int e = threadIdx.x; e < C * g8; e += blockDim.x) {
    const int r = e / g8, f = (e - r * g8) * 8;
    float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (r < L) {
      const long long i = base + static_cast<long long>(r) * d + f;
      if (f32) {
        const float4 a = *reinterpret_cast<const float4*>(static_cast<const float*>(g) + i);
        const float4 b = *reinterpret_cast<const float4*>(static_cast<const float*>(g) + i + 4);
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
        x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
      } else {
        const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(g) + i);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          __nv_bfloat162 h;
          std::memcpy(&h, &w[k], 4);
          const float2 v = __bfloat1622float2(h);
          x[2 * k] = v.x;
          x[2 * k + 1] = v.y;
        }
      }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) sm[r * lds + f + k] = x[k];
  }
}

// The gates of rows [t0, t0 + L) into sm[r * lds + f] (rows >= L: 1), float4 loads.
__device__ __forceinline__ void load_gates(float* sm, int lds, const float* g, long long base,
                                           int d, int C, int L) {
  const int g4 = d / 4;
  for (int e = threadIdx.x; e < C * g4; e += blockDim.x) {
    const int r = e / g4, f = (e - r * g4) * 4;
    const float4 a = r < L ? *reinterpret_cast<const float4*>(g + base + static_cast<long long>(r) * d + f)
                           : make_float4(1.f, 1.f, 1.f, 1.f);
    sm[r * lds + f] = a.x;
    sm[r * lds + f + 1] = a.y;
    sm[r * lds + f + 2] = a.z;
    sm[r * lds + f + 3] = a.w;
  }
}

// Cumulative log2 of the gates down each feature column (sm holds the gates on entry).  A
// gate below 2^-126 counts as 2^-126, so that sums stay finite (a zero gate would give
// -inf - -inf); whatever passes through it is then below 2^-126 of its size.
__device__ __forceinline__ void cum_log2(float* sm, int lds, int d, int L) {
  for (int f = threadIdx.x; f < d; f += blockDim.x) {
    float acc = 0.f;
    for (int r = 0; r < L; ++r) {
      acc += fmaxf(log2f(sm[r * lds + f]), -126.f);
      sm[r * lds + f] = acc;
    }
  }
}

// K1: one CTA per (b*H + h, chunk): the chunk's summary and decay vector.
constexpr int kGlaThreads1 = 256;  // K1: two CTAs per SM (8 x 8 tiles, 94 registers)

__global__ void __launch_bounds__(kGlaThreads1) gla_k1(GlaParams p) {
  extern __shared__ float sm[];
  const int bh = static_cast<int>(blockIdx.x / p.NC), c = static_cast<int>(blockIdx.x % p.NC);
  const int C = p.C, dk = p.dk, dv = p.dv, L = chunk_len(p, c);
  float* sK = sm;            // [C][dk]
  float* sA = sK + C * dk;   // [C][dk]: gates, then cumulative log2
  float* sV = sA + C * dk;   // [C][dv]
  const long long t0 = static_cast<long long>(c) * C;
  load_rows(sK, dk, p.k, p.in_f32, (static_cast<long long>(bh) * p.T + t0) * dk, dk, C, L);
  load_rows(sV, dv, p.v, p.in_f32, (static_cast<long long>(bh) * p.T + t0) * dv, dv, C, L);
  load_gates(sA, dk, p.alpha, (static_cast<long long>(bh) * p.T + t0) * dk, dk, C, L);
  __syncthreads();
  cum_log2(sA, dk, dk, L);
  __syncthreads();
  float* rec = p.rec + (static_cast<long long>(bh) * p.NC + c) * p.R;
  // k_j (.) 2^(L_last - L_j), in place; the chunk's decay vector a_c = 2^(L_last).
  for (int e = threadIdx.x; e < C * dk; e += blockDim.x) {
    const int r = e / dk, f = e - r * dk;
    sK[e] = r < L ? sK[e] * exp2f(sA[(L - 1) * dk + f] - sA[e]) : 0.f;
  }
  for (int f = threadIdx.x; f < dk; f += blockDim.x) rec[dk * dv + f] = exp2f(sA[(L - 1) * dk + f]);
  __syncthreads();
  // S[f][e] = sum_j K'[j][f] v[j][e]: an 8 x 8 tile of (f, e) per thread.
  const int tiles_e = dv / 8, tiles = (dk / 8) * tiles_e;
  for (int tile = threadIdx.x; tile < tiles; tile += blockDim.x) {
    const int f0 = (tile / tiles_e) * 8, e0 = (tile % tiles_e) * 8;
    float acc[8][8] = {};
    for (int j = 0; j < L; ++j) {
      const float4 a0 = *reinterpret_cast<const float4*>(sK + j * dk + f0);
      const float4 a1 = *reinterpret_cast<const float4*>(sK + j * dk + f0 + 4);
      const float4 b0 = *reinterpret_cast<const float4*>(sV + j * dv + e0);
      const float4 b1 = *reinterpret_cast<const float4*>(sV + j * dv + e0 + 4);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int w = 0; w < 8; ++w) acc[u][w] = fmaf(av[u], bv[w], acc[u][w]);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int w = 0; w < 8; w += 4)
        *reinterpret_cast<float4*>(rec + (f0 + u) * dv + e0 + w) =
            make_float4(acc[u][w], acc[u][w + 1], acc[u][w + 2], acc[u][w + 3]);
  }
}

// K2: the exclusive prefix over chunks, one thread per float4 column of the state: record c
// receives the state before chunk c, then P <- a_c (.) P + S_c (row f scaled by a_c[f]).
__global__ void gla_k2(GlaParams p) {
  const long long n4 = static_cast<long long>(p.dk) * p.dv / 4;
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long long>(p.BH) * n4) return;
  const long long bh = idx / n4, col = idx - bh * n4;
  const int f = static_cast<int>(col * 4 / p.dv);
  float4 P = p.S_init ? reinterpret_cast<const float4*>(p.S_init + bh * p.dk * p.dv)[col]
                      : make_float4(0.f, 0.f, 0.f, 0.f);
  float* base = p.rec + bh * p.NC * p.R;
  constexpr int kB = 8;  // chunks whose records are loaded before the carry walks them
  for (int c0 = 0; c0 < p.NC; c0 += kB) {
    float4 x[kB];
    float a[kB];
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      if (c0 + u >= p.NC) break;
      const long long r = static_cast<long long>(c0 + u) * p.R;
      x[u] = reinterpret_cast<const float4*>(base + r)[col];
      a[u] = base[r + p.dk * p.dv + f];
    }
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      if (c0 + u >= p.NC) break;
      reinterpret_cast<float4*>(base + static_cast<long long>(c0 + u) * p.R)[col] = P;
      P = make_float4(fmaf(a[u], P.x, x[u].x), fmaf(a[u], P.y, x[u].y), fmaf(a[u], P.z, x[u].z),
                      fmaf(a[u], P.w, x[u].w));
    }
  }
  if (p.S_final) reinterpret_cast<float4*>(p.S_final + bh * p.dk * p.dv)[col] = P;
}

// K3: one CTA per (b*H + h, chunk): the intra-chunk part with per-feature gate ratios and
// the prefix read out through the gates' running products.
__device__ __forceinline__ void gla_k3_chunk(const GlaParams& p, int id) {
  extern __shared__ float sm[];
  const bool fix = p.steep != nullptr;
  const int bh = id / p.NC, c = id % p.NC;
  const int C = p.C, dk = p.dk, dv = p.dv, L = chunk_len(p, c);
  const int lk = dk + 1;       // padded rows: threads of a warp read different rows
  float* sQ = sm;              // [C][lk]
  float* sK = sQ + C * lk;     // [C][lk]
  float* sL = sK + C * lk;     // [C][lk]: gates, then cumulative log2
  float* sV = sL + C * lk;     // [C][dv]
  float* sP = sV + C * dv;     // [dk][dv]
  float* sS = sP + dk * dv;    // [C][C] scores
  const long long t0 = static_cast<long long>(c) * C;
  const long long rq = (static_cast<long long>(bh) * p.T + t0) * dk;
  load_rows(sQ, lk, p.q, p.in_f32, rq, dk, C, L);
  load_rows(sK, lk, p.k, p.in_f32, rq, dk, C, L);
  load_rows(sV, dv, p.v, p.in_f32, (static_cast<long long>(bh) * p.T + t0) * dv, dv, C, L);
  load_gates(sL, lk, p.alpha, rq, dk, C, L);
  if (!fix) {
    const float4* P4 =
        reinterpret_cast<const float4*>(p.rec + (static_cast<long long>(bh) * p.NC + c) * p.R);
    for (int e = threadIdx.x; e < dk * dv / 4; e += blockDim.x)
      reinterpret_cast<float4*>(sP)[e] = P4[e];
  }
  __syncthreads();
  cum_log2(sL, lk, dk, L);
  __syncthreads();
  // Scores A[j][i] = sum_f q_j[f] k_i[f] 2^(L_j[f] - L_i[f]) for i <= j (0 above the diagonal).
  // When every L of the chunk is >= -kGlaFactorBound (the usual case), the weight factors
  // exactly: q~_j = q_j 2^(L_j) and k~_i = k_i 2^(-L_i) stay within 2^kGlaFactorBound of q, k,
  // and A = q~ k~^T is a plain product.  Otherwise (gates small enough for 2^(-L) to overflow)
  // each (pair, feature) takes its own exponential, whose exponent is <= 0.
  __shared__ int s_wide;
  if (threadIdx.x == 0) s_wide = 0;
  for (int e = threadIdx.x; e < C * C; e += blockDim.x) {
    const int j = e / C, i = e - j * C;
    if (i > j) sS[e] = 0.f;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < L * dk; e += blockDim.x) {
    const int r = e / dk, f = e - r * dk;
    if (sL[r * lk + f] < -kGlaFactorBound) s_wide = 1;  // every writer stores 1
  }
  __syncthreads();
  const int npairs = C * (C + 1) / 2;
  if (!s_wide) {
    for (int e = threadIdx.x; e < C * dk; e += blockDim.x) {
      const int r = e / dk, f = e - r * dk;
      const float x = sL[r * lk + f];
      sQ[r * lk + f] = r < L ? sQ[r * lk + f] * exp2f(x) : 0.f;
      sK[r * lk + f] = r < L ? sK[r * lk + f] * exp2f(-x) : 0.f;
    }
    __syncthreads();
    // 2 x 2 blocks of pairs over the lower triangle, numbered row by row.
    const int h = C / 2, nblk = h * (h + 1) / 2;
    for (int e = threadIdx.x; e < nblk; e += blockDim.x) {
      int bj = static_cast<int>((sqrtf(8.f * e + 1.f) - 1.f) * 0.5f);
      while (bj * (bj + 1) / 2 > e) --bj;
      while ((bj + 1) * (bj + 2) / 2 <= e) ++bj;
      const int j = 2 * bj, i = 2 * (e - bj * (bj + 1) / 2);
      const float* q0 = sQ + j * lk;
      const float* k0 = sK + i * lk;
      float a00 = 0.f, a01 = 0.f, a10 = 0.f, a11 = 0.f;
      for (int f = 0; f < dk; ++f) {
        const float x0 = q0[f], x1 = q0[lk + f], y0 = k0[f], y1 = k0[lk + f];
        a00 = fmaf(x0, y0, a00);
        a01 = fmaf(x0, y1, a01);
        a10 = fmaf(x1, y0, a10);
        a11 = fmaf(x1, y1, a11);
      }
      sS[j * C + i] = a00;
      if (i + 1 <= j) sS[j * C + i + 1] = a01;  // above the diagonal stays zero
      sS[(j + 1) * C + i] = a10;
      sS[(j + 1) * C + i + 1] = a11;
    }
  } else {
    for (int e = threadIdx.x; e < npairs; e += blockDim.x) {
      int j = static_cast<int>((sqrtf(8.f * e + 1.f) - 1.f) * 0.5f);
      while (j * (j + 1) / 2 > e) --j;           // guard the float root at row boundaries
      while ((j + 1) * (j + 2) / 2 <= e) ++j;
      const int i = e - j * (j + 1) / 2;
      float a = 0.f;
      if (j < L) {
        const float* qj = sQ + j * lk;
        const float* ki = sK + i * lk;
        const float* Lj = sL + j * lk;
        const float* Li = sL + i * lk;
        for (int f = 0; f < dk; ++f) a = fmaf(qj[f] * ki[f], exp2f(Lj[f] - Li[f]), a);
      }
      sS[j * C + i] = a;
    }
    __syncthreads();
    // q_j (.) 2^(L_j) for the prefix, in place.
    for (int e = threadIdx.x; e < C * dk; e += blockDim.x) {
      const int r = e / dk, f = e - r * dk;
      sQ[r * lk + f] *= exp2f(sL[r * lk + f]);
    }
  }
  __syncthreads();
  // o[j][e] = sum_f q~[j][f] P[f][e] + sum_{i<=j} A[j][i] v[i][e]: a 4 x 4 tile per thread.
  const int tiles_e = dv / 4, tiles = (C / 4) * tiles_e;
  for (int tile = threadIdx.x; tile < tiles; tile += blockDim.x) {
    const int j0 = (tile / tiles_e) * 4, e0 = (tile % tiles_e) * 4;
    float acc[4][4] = {};
    for (int f = 0; f < (fix ? 0 : dk); ++f) {
      float a[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) a[u] = sQ[(j0 + u) * lk + f];
      const float4 b = *reinterpret_cast<const float4*>(sP + f * dv + e0);
      const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) acc[u][w] = fmaf(a[u], bv[w], acc[u][w]);
    }
    for (int i = 0; i <= j0 + 3 && i < C; ++i) {
      float a[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) a[u] = sS[(j0 + u) * C + i];
      const float4 b = *reinterpret_cast<const float4*>(sV + i * dv + e0);
      const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) acc[u][w] = fmaf(a[u], bv[w], acc[u][w]);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (j0 + u >= L) continue;
      const long long o = (static_cast<long long>(bh) * p.T + t0 + j0 + u) * dv + e0;
      if (p.out_f32) {
        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + o);
        if (fix) {
          const float4 x = *dst;
          acc[u][0] += x.x;
          acc[u][1] += x.y;
          acc[u][2] += x.z;
          acc[u][3] += x.w;
        }
        *dst = make_float4(acc[u][0], acc[u][1], acc[u][2], acc[u][3]);
      } else {
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + o;
#pragma unroll
        for (int w = 0; w < 4; ++w)
          dst[w] = __float2bfloat16_rn(fix ? acc[u][w] + __bfloat162float(dst[w]) : acc[u][w]);
      }
    }
  }
}

// One CTA per chunk; in fix-up mode a grid of a few CTAs per SM walks every chunk and
// takes the flagged ones (usually none), so that the common case costs one short launch.
__global__ void __launch_bounds__(kGlaThreads) gla_k3(GlaParams p) {
  if (!p.steep) {
    gla_k3_chunk(p, static_cast<int>(blockIdx.x));
    return;
  }
  // The flags of kGlaThreads chunks at a time, read by all threads at once.
  __shared__ unsigned char s_flag[kGlaThreads];
  const int n = p.BH * p.NC;
  for (int b0 = static_cast<int>(blockIdx.x) * kGlaThreads; b0 < n;
       b0 += static_cast<int>(gridDim.x) * kGlaThreads) {
    const int my = b0 + static_cast<int>(threadIdx.x);
    const unsigned char f = my < n ? p.steep[my] : 0;
    s_flag[threadIdx.x] = f;
    if (!__syncthreads_or(f)) continue;
    for (int j = 0; j < kGlaThreads && b0 + j < n; ++j) {
      if (!s_flag[j]) continue;  // the same j for every thread of the CTA
      gla_k3_chunk(p, b0 + j);
      __syncthreads();  // the next flagged chunk reuses shared memory
    }
    __syncthreads();  // s_flag is rewritten next round
  }
}

size_t gla_smem_k1(int C, int dk, int dv) { return static_cast<size_t>(C) * (2 * dk + dv) * 4; }
size_t gla_smem_k3(int C, int dk, int dv) {
  return (static_cast<size_t>(C) * (3 * (dk + 1) + dv) + static_cast<size_t>(dk) * dv +
          static_cast<size_t>(C) * C) * 4;
}

bool gla_dims_ok(int d) { return d >= 8 && d <= 128 && d % 8 == 0; }

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool overlaps(const void* a, size_t an, const void* b, size_t bn) {
  if (!a || !b || an == 0 || bn == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + bn && b0 < a0 + an;
}

// Workspace of either path: one record of dk*dv + dk floats per chunk (the CUDA-core path's
// chunk records; the tensor-core path's segment records, at most one per chunk), then one
// byte per chunk (the tensor-core path's fix-up flags).
struct GlaLayout {
  size_t rec, flags, total;
};
GlaLayout gla_layout(int B, int H, long long T, int dk, int dv, int C) {
  GlaLayout l{};
  if (B <= 0 || H <= 0 || T <= 0 || C <= 0) return l;
  const size_t BH = static_cast<size_t>(B) * H, NC = static_cast<size_t>((T + C - 1) / C);
  l.rec = 0;
  l.flags = align256(BH * NC * (static_cast<size_t>(dk) * dv + dk) * 4);
  l.total = l.flags + align256(BH * NC);
  return l;
}

size_t gla_ws(int B, int H, long long T, int dk, int dv, int C) {
  return gla_layout(B, H, T, dk, dv, C).total;
}

bool gla_tc_shape(const la_gla_args& a) {
  return a.dtype == LA_DTYPE_BF16 && a.C == 64 && (a.dk == 64 || a.dk == 128) && a.dv == 128 &&
         a.T < (1LL << 31);
}

bool gla_device_sm100() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return false;
  return major == 10;
}

int gla_validate(const la_gla_args& a) {
  if (a.B < 0 || a.H < 0 || a.T < 0 || a.dk <= 0 || a.dv <= 0 || a.C <= 0)
    return LA_ERR_INVALID_ARGUMENT;
  if (a.dtype != LA_DTYPE_BF16 && a.dtype != LA_DTYPE_F32) return LA_ERR_INVALID_ARGUMENT;
  if (a.out_dtype != LA_OUT_AS_INPUT && a.out_dtype != LA_OUT_F32) return LA_ERR_INVALID_ARGUMENT;
  if (!gla_dims_ok(a.dk) || !gla_dims_ok(a.dv) || !(a.C == 16 || a.C == 32 || a.C == 64))
    return LA_ERR_UNSUPPORTED;
  if (a.kernel_path < LA_PATH_AUTO || a.kernel_path > LA_PATH_FMA) return LA_ERR_INVALID_ARGUMENT;
  if (a.kernel_path == LA_PATH_TENSOR_CORE && !gla_tc_shape(a)) return LA_ERR_UNSUPPORTED;
  if (a.segment_chunks < 0 || a.segment_chunks > 1024) return LA_ERR_INVALID_ARGUMENT;
  const long long BH = static_cast<long long>(a.B) * a.H;
  const long long NC = a.T > 0 ? (a.T + a.C - 1) / a.C : 0;
  if (BH * NC > (1LL << 31) - 1) return LA_ERR_UNSUPPORTED;
  if (a.workspace && (reinterpret_cast<uintptr_t>(a.workspace) & 255u)) return LA_ERR_INVALID_ARGUMENT;
  if (!aligned16(a.S_init) || !aligned16(a.S_final)) return LA_ERR_INVALID_ARGUMENT;
  if (BH > 0 && a.T > 0) {
    if (!a.q || !a.k || !a.v || !a.alpha || !a.out) return LA_ERR_INVALID_ARGUMENT;
    if (!aligned16(a.q) || !aligned16(a.k) || !aligned16(a.v) || !aligned16(a.alpha) ||
        !aligned16(a.out))
      return LA_ERR_INVALID_ARGUMENT;
    const size_t e = a.dtype == LA_DTYPE_F32 ? 4 : 2;
    const size_t eo = (a.dtype == LA_DTYPE_F32 || a.out_dtype == LA_OUT_F32) ? 4 : 2;
    const size_t nk = static_cast<size_t>(BH) * a.T * a.dk, nv = static_cast<size_t>(BH) * a.T * a.dv;
    if (overlaps(a.out, nv * eo, a.q, nk * e) || overlaps(a.out, nv * eo, a.k, nk * e) ||
        overlaps(a.out, nv * eo, a.v, nv * e) || overlaps(a.out, nv * eo, a.alpha, nk * 4))
      return LA_ERR_INVALID_ARGUMENT;
  }
  return LA_OK;
}

int gla_prefill(const la_gla_args& a, Recorder* rec) {
  int st = gla_validate(a);
  if (st != LA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(a.stream);
  const long long BH = static_cast<long long>(a.B) * a.H;
  if (BH == 0) return LA_OK;
  const size_t state_bytes = static_cast<size_t>(BH) * a.dk * a.dv * 4;
  if (a.T == 0) {
    if (!a.S_final) return LA_OK;
    const cudaError_t e = a.S_init ? cudaMemcpyAsync(a.S_final, a.S_init, state_bytes,
                                                     cudaMemcpyDeviceToDevice, s)
                                   : cudaMemsetAsync(a.S_final, 0, state_bytes, s);
    return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
  }
  const size_t need = gla_ws(a.B, a.H, a.T, a.dk, a.dv, a.C);
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  bool owned = false;
  if (ws) {
    if (a.workspace_bytes < need) return LA_ERR_INVALID_ARGUMENT;
  } else {
    if (workspace_alloc(reinterpret_cast<void**>(&ws), need, s) != cudaSuccess) {
      cudaGetLastError();
      return LA_ERR_OUT_OF_MEMORY;
    }
    owned = true;
  }
  GlaParams p;
  p.BH = static_cast<int>(BH);
  p.T = a.T;
  p.dk = a.dk;
  p.dv = a.dv;
  p.C = a.C;
  p.NC = static_cast<int>((a.T + a.C - 1) / a.C);
  p.L_last = static_cast<int>(a.T - static_cast<long long>(p.NC - 1) * a.C);
  p.R = a.dk * a.dv + a.dk;
  p.q = a.q;
  p.k = a.k;
  p.v = a.v;
  p.alpha = a.alpha;
  p.out = a.out;
  p.in_f32 = a.dtype == LA_DTYPE_F32;
  p.out_f32 = p.in_f32 || a.out_dtype == LA_OUT_F32;
  p.rec = reinterpret_cast<float*>(ws);
  p.S_init = a.S_init;
  p.S_final = a.S_final;
  p.steep = nullptr;

  const bool tc = a.kernel_path != LA_PATH_FMA && gla_tc_shape(a) && gla_device_sm100();
  if (a.kernel_path == LA_PATH_TENSOR_CORE && !tc) {
    if (owned) cudaFreeAsync(ws, s);
    return LA_ERR_UNSUPPORTED;
  }
  if (tc) {
    const GlaLayout l = gla_layout(a.B, a.H, a.T, a.dk, a.dv, a.C);
    GlaSegParams sp{};
    sp.BH = p.BH;
    sp.T = a.T;
    sp.dk = a.dk;
    sp.NC = p.NC;
    sp.L_last = p.L_last;
    sp.Lseg = a.segment_chunks > 0 ? std::min(a.segment_chunks, p.NC)
                                   : default_segment_chunks(BH, p.NC);
    sp.NS = (p.NC + sp.Lseg - 1) / sp.Lseg;
    sp.R = p.R;
    sp.srec = reinterpret_cast<float*>(ws + l.rec);
    sp.out = a.out;
    sp.steep = ws + l.flags;
    sp.has_init = a.S_init != nullptr;
    sp.err = device_error_word();
    const uint64_t T = static_cast<uint64_t>(a.T), BHu = static_cast<uint64_t>(BH);
    const uint64_t dk = a.dk, dv = a.dv;
    GlaSegMaps m;
    const bool ok =
        make_tile_map(&m.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.q, dk, T, BHu, dk * 2, T * dk * 2,
                      64, 64) &&
        make_tile_map(&m.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.k, dk, T, BHu, dk * 2, T * dk * 2,
                      64, 64) &&
        make_tile_map(&m.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.v, dv, T, BHu, dv * 2, T * dv * 2,
                      64, 64) &&
        make_plain_map(&m.a, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.alpha, dk, T, BHu, dk * 4,
                       T * dk * 4, static_cast<uint32_t>(dk), 64) &&
        make_tile_map(&m.rec, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, sp.srec, dk, dv,
                      BHu * static_cast<uint64_t>(sp.NS), dk * 4, static_cast<uint64_t>(p.R) * 4,
                      32, static_cast<uint32_t>(dv));
    cudaError_t e = ok ? cudaSuccess : cudaErrorInvalidValue;
    if (e == cudaSuccess) e = launch_gla_seg(sp, m, a.S_init, a.S_final, p.out_f32, s, rec);
    // The exact intra-chunk part of the chunks the tensor-core combine flagged.
    if (e == cudaSuccess) {
      const size_t s3 = gla_smem_k3(a.C, a.dk, a.dv);
      e = cudaFuncSetAttribute(gla_k3, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(s3));
      GlaParams pf = p;
      pf.steep = sp.steep;
      if (e == cudaSuccess) {
        if (rec) rec->mark(s, "gla_fixup");
        const long long nf = std::min<long long>((BH * p.NC + kGlaThreads - 1) / kGlaThreads, 2 * 148);
        gla_k3<<<static_cast<unsigned>(nf), kGlaThreads, s3, s>>>(pf);
        e = cudaGetLastError();
      }
    }
    if (rec) rec->mark(s);
    if (owned) {
      const cudaError_t e2 = cudaFreeAsync(ws, s);
      if (e == cudaSuccess) e = e2;
    }
    return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
  }

  const size_t s1 = gla_smem_k1(a.C, a.dk, a.dv), s3 = gla_smem_k3(a.C, a.dk, a.dv);
  cudaError_t e = cudaFuncSetAttribute(gla_k1, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(s1));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gla_k3, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(s3));
  const unsigned grid = static_cast<unsigned>(BH * p.NC);
  if (e == cudaSuccess) {
    if (rec) rec->mark(s, "gla_k1");
    gla_k1<<<grid, kGlaThreads1, s1, s>>>(p);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) {
    const long long n = BH * a.dk * a.dv / 4;
    if (rec) rec->mark(s, "gla_k2");
    gla_k2<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(p);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) {
    if (rec) rec->mark(s, "gla_k3");
    gla_k3<<<grid, kGlaThreads, s3, s>>>(p);
    e = cudaGetLastError();
  }
  if (rec) rec->mark(s);
  if (owned) {
    const cudaError_t e2 = cudaFreeAsync(ws, s);
    if (e == cudaSuccess) e = e2;
  }
  return e == cudaSuccess ? LA_OK
                          : (e == cudaErrorMemoryAllocation ? LA_ERR_OUT_OF_MEMORY : LA_ERR_CUDA);
}

}  // namespace
}  // namespace la

extern "C" int lin_attn_gla_prefill(const la_gla_args* args) {
  if (!args) return LA_ERR_INVALID_ARGUMENT;
  return la::gla_prefill(*args, nullptr);
}

extern "C" size_t lin_attn_gla_workspace_bytes(int B, int H, long long T, int dk, int dv, int C) {
  return la::gla_ws(B, H, T, dk, dv, C);
}

extern "C" int lin_attn_gla_prefill_timed(const la_gla_args* args, float* kernel_ms,
                                          int max_kernels, int* n_kernels) {
  if (!args || !kernel_ms || !n_kernels || max_kernels < 1) return LA_ERR_INVALID_ARGUMENT;
  *n_kernels = 0;
  constexpr int kEv = 8;
  cudaEvent_t ev[kEv];
  const char* label[kEv] = {nullptr};
  for (int i = 0; i < kEv; ++i)
    if (cudaEventCreate(&ev[i]) != cudaSuccess) {
      for (int j = 0; j < i; ++j) cudaEventDestroy(ev[j]);
      return LA_ERR_CUDA;
    }
  la::Recorder rec;
  rec.ev = ev;
  rec.label = label;
  rec.cap = kEv;
  int st = la::gla_prefill(*args, &rec);
  if (st == LA_OK && cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(args->stream)) != cudaSuccess)
    st = LA_ERR_CUDA;
  if (st == LA_OK) {
    int nk = 0;
    for (int i = 0; i + 1 < rec.n && nk < max_kernels; ++i) {
      float ms = 0.f;
      cudaEventElapsedTime(&ms, ev[i], ev[i + 1]);
      kernel_ms[nk++] = ms;
    }
    *n_kernels = nk;
  }
  for (int i = 0; i < kEv; ++i) cudaEventDestroy(ev[i]);
  return st;
}
