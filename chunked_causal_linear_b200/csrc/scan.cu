// K2: exclusive associative scan of the chunk records across chunks.
//
// Each record column is an independent scan over the chunk axis with the element
// (a_c, x_c), a_c = gamma^(L_c) and x_c the chunk summary, and the combine
//   (a1, x1) + (a2, x2) = (a1 a2, a2 x1 + x2)
// which is the scan page's monoid (S1 + S2, Z1 + Z2) when gamma = 1 ("Log-Depth Chunked
// Linear-Attention Scan", "Formulas" and "Mathematical statement"), extended with the
// retention decay ("Linear Attention and Retentive Networks ...", "C. Chunkwise
// Recurrent Representation": S_i = gamma^B S_{i-1} + chunk term).  The scan is exclusive:
// after K2, record c holds P_c, the state before chunk c, and P_0 = 0.  The inclusive
// total (the state after the last token) goes to S_final / Z_final.
//
// Log-depth mode ("Implementation notes": a Blelloch or Hillis-Steele scan) splits the
// chunk axis into G <= 32 segments of Ls chunks (when Ls = 1, i.e. at most 32 elements,
// k2_scan_totals alone scans the records in place):
//   k2_reduce       one pass over the records: each segment's aggregate (parallel over
//                   segments and columns);
//   k2_scan_totals  Hillis-Steele scan of the G segment aggregates, ceil(log2 G) rounds
//                   in shared memory, giving each segment's exclusive prefix;
//   k2_downsweep    second pass: each segment re-scans its chunks from its prefix and
//                   writes P_c in place.
// Sequential mode (comparison only) carries the state through every chunk in order.
// Both modes read and write float4 columns; a warp touches 512 contiguous bytes of a
// record per step.
// A caller-given state before token 0 (S_init, Z_init) is the scan's first element: the
// exclusive prefix of chunk 0 is that state, and every later prefix carries it decayed by
// gamma^(tokens before the chunk) -- the same monoid with one more element in front.

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace la {
namespace {

constexpr int kScanThreads = 128;
constexpr int kUnroll = 8;

__device__ __forceinline__ float4 axpy4(float a, float4 x, float4 y) {
  return make_float4(fmaf(a, x.x, y.x), fmaf(a, x.y, y.y), fmaf(a, x.z, y.z), fmaf(a, x.w, y.w));
}

// Record column `col` of S^T (j = col / dk, i = col % dk) goes to S_final[i][j].
__device__ __forceinline__ void write_final1(const PrefillParams& p, int bh, int col, float x) {
  const int dkdv = p.dk * p.dv;
  if (col < dkdv) {
    if (p.S_final) {
      const int j = col / p.dk, i = col % p.dk;
      p.S_final[static_cast<long long>(bh) * dkdv + static_cast<long long>(i) * p.dv + j] = x;
    }
  } else if (p.Z_final) {
    p.Z_final[static_cast<long long>(bh) * p.dk + (col - dkdv)] = x;
  }
}

__device__ __forceinline__ void write_final(const PrefillParams& p, int bh, int col, float4 v) {
  write_final1(p, bh, col, v.x);
  write_final1(p, bh, col + 1, v.y);
  write_final1(p, bh, col + 2, v.z);
  write_final1(p, bh, col + 3, v.w);
}

// The initial state of record column `col` (same mapping as write_final1); zero without one.
__device__ __forceinline__ float read_init1(const PrefillParams& p, int bh, int col) {
  const int dkdv = p.dk * p.dv;
  if (col < dkdv) {
    if (!p.S_init) return 0.f;
    const int j = col / p.dk, i = col % p.dk;
    return p.S_init[static_cast<long long>(bh) * dkdv + static_cast<long long>(i) * p.dv + j];
  }
  return p.Z_init ? p.Z_init[static_cast<long long>(bh) * p.dk + (col - dkdv)] : 0.f;
}

__device__ __forceinline__ float4 read_init(const PrefillParams& p, int bh, int col) {
  return make_float4(read_init1(p, bh, col), read_init1(p, bh, col + 1), read_init1(p, bh, col + 2),
                     read_init1(p, bh, col + 3));
}

// In-place exclusive carry over chunks [cbeg, cend) of one float4 column: record c
// receives the carry before chunk c, then carry <- a_c carry + x_c.  The next batch of
// loads is issued before the current batch is stored, so a thread always has loads in
// flight (in-place read-then-write streams reach copy bandwidth only this way).
template <bool DECAY>
__device__ __forceinline__ float4 carry_in_place(float4* base, long long stride, int cbeg,
                                                 int cend, int last, float gC, float aL,
                                                 float4 carry) {
  float4 x[kUnroll], y[kUnroll];
#pragma unroll
  for (int u = 0; u < kUnroll; ++u)
    if (cbeg + u < cend) x[u] = base[static_cast<long long>(cbeg + u) * stride];
  for (int c0 = cbeg; c0 < cend; c0 += kUnroll) {
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (c0 + kUnroll + u < cend) y[u] = base[static_cast<long long>(c0 + kUnroll + u) * stride];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (c0 + u < cend) {
        base[static_cast<long long>(c0 + u) * stride] = carry;
        const float a = DECAY ? (c0 + u == last ? aL : gC) : 1.f;
        carry = axpy4(a, carry, x[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) x[u] = y[u];
  }
  return carry;
}

// Sequential carry: one thread per float4 column, loop over all chunks.
template <bool DECAY>
__global__ void __launch_bounds__(kScanThreads) k2_sequential(PrefillParams p, GammaTable gt) {
  const int R4 = p.R / 4;
  const int nblk = (R4 + kScanThreads - 1) / kScanThreads;
  const int bh = blockIdx.x / nblk;
  const int col4 = (blockIdx.x % nblk) * kScanThreads + threadIdx.x;
  if (col4 >= R4) return;
  const float g = DECAY ? gt.g[bh % p.H] : 1.f;
  const float gC = DECAY ? powf(g, static_cast<float>(p.C)) : 1.f;
  const float aL = DECAY ? powf(g, static_cast<float>(p.L_last)) : 1.f;
  float4* base = reinterpret_cast<float4*>(p.rec + static_cast<long long>(bh) * p.NC * p.R) + col4;
  const float4 carry = carry_in_place<DECAY>(base, R4, 0, p.NC, p.NC - 1, gC, aL,
                                             read_init(p, bh, col4 * 4));
  write_final(p, bh, col4 * 4, carry);
}

// Segment aggregates: grid = (column blocks) x G x BH.
template <bool DECAY>
__global__ void __launch_bounds__(kScanThreads) k2_reduce(PrefillParams p, GammaTable gt) {
  const int R4 = p.R / 4;
  const int nblk = (R4 + kScanThreads - 1) / kScanThreads;
  const int cb = blockIdx.x % nblk;
  const int s = (blockIdx.x / nblk) % p.G;
  const int bh = blockIdx.x / (nblk * p.G);
  const int col4 = cb * kScanThreads + threadIdx.x;
  if (col4 >= R4) return;
  const float g = DECAY ? gt.g[bh % p.H] : 1.f;
  const float gC = DECAY ? powf(g, static_cast<float>(p.C)) : 1.f;
  const float aL = DECAY ? powf(g, static_cast<float>(p.L_last)) : 1.f;
  const int cbeg = s * p.Ls;
  const int cend = min(p.NC, cbeg + p.Ls);
  const float4* base =
      reinterpret_cast<const float4*>(p.rec + static_cast<long long>(bh) * p.NC * p.R) + col4;
  float4 agg = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int c0 = cbeg; c0 < cend; c0 += kUnroll) {
    float4 x[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (c0 + u < cend) x[u] = base[static_cast<long long>(c0 + u) * R4];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (c0 + u < cend) agg = axpy4(DECAY ? (c0 + u == p.NC - 1 ? aL : gC) : 1.f, agg, x[u]);
  }
  reinterpret_cast<float4*>(p.tot + (static_cast<long long>(bh) * p.G + s) * p.R)[col4] = agg;
}

// Hillis-Steele scan of the segment aggregates.  Block (32 float4 columns) x (32
// segments); ceil(log2 G) rounds in shared memory.
template <bool DECAY>
__global__ void __launch_bounds__(1024) k2_scan_totals(PrefillParams p, GammaTable gt) {
  __shared__ float4 sX[32][33];
  __shared__ float sA[32];
  const int R4 = p.R / 4;
  const int ncb = (R4 + 31) / 32;
  const int bh = blockIdx.x / ncb;
  const int col4 = (blockIdx.x % ncb) * 32 + threadIdx.x;
  const int s = threadIdx.y;
  const bool live = s < p.G && col4 < R4;
  const float g = DECAY ? gt.g[bh % p.H] : 1.f;

  // Segment decay: product of its chunks' decays.
  float a = 1.f;
  if (DECAY && s < p.G) {
    const int cbeg = s * p.Ls;
    const int cend = min(p.NC, cbeg + p.Ls);
    const float tokens = static_cast<float>(cend == p.NC
                                                ? static_cast<long long>(cend - cbeg - 1) * p.C + p.L_last
                                                : static_cast<long long>(cend - cbeg) * p.C);
    a = powf(g, tokens);
  }
  float4* tot = reinterpret_cast<float4*>(p.tot + static_cast<long long>(bh) * p.G * p.R);
  float4 x = live ? tot[static_cast<long long>(s) * R4 + col4] : make_float4(0.f, 0.f, 0.f, 0.f);

  for (int d = 1; d < p.G; d <<= 1) {
    sX[s][threadIdx.x] = x;
    if (threadIdx.x == 0) sA[s] = a;
    __syncthreads();
    if (s >= d) {
      x = axpy4(a, sX[s - d][threadIdx.x], x);
      a = sA[s - d] * a;
    }
    __syncthreads();
  }
  // `a` is now the product of the decays of segments 0 .. s: the initial state reaches
  // the end of segment s scaled by it.
  const float4 init = (p.S_init || p.Z_init) && live ? read_init(p, bh, col4 * 4)
                                                      : make_float4(0.f, 0.f, 0.f, 0.f);
  x = axpy4(a, init, x);
  // Inclusive -> exclusive.
  sX[s][threadIdx.x] = x;
  __syncthreads();
  if (live) {
    tot[static_cast<long long>(s) * R4 + col4] = s > 0 ? sX[s - 1][threadIdx.x] : init;
    if (s == p.G - 1) write_final(p, bh, col4 * 4, x);
  }
}

// Second pass: each segment writes its chunks' exclusive prefixes in place.
template <bool DECAY>
__global__ void __launch_bounds__(kScanThreads) k2_downsweep(PrefillParams p, GammaTable gt) {
  const int R4 = p.R / 4;
  const int nblk = (R4 + kScanThreads - 1) / kScanThreads;
  const int cb = blockIdx.x % nblk;
  const int s = (blockIdx.x / nblk) % p.G;
  const int bh = blockIdx.x / (nblk * p.G);
  const int col4 = cb * kScanThreads + threadIdx.x;
  if (col4 >= R4) return;
  const float g = DECAY ? gt.g[bh % p.H] : 1.f;
  const float gC = DECAY ? powf(g, static_cast<float>(p.C)) : 1.f;
  const float aL = DECAY ? powf(g, static_cast<float>(p.L_last)) : 1.f;
  const int cbeg = s * p.Ls;
  const int cend = min(p.NC, cbeg + p.Ls);
  float4* base = reinterpret_cast<float4*>(p.rec + static_cast<long long>(bh) * p.NC * p.R) + col4;
  const float4 carry =
      reinterpret_cast<const float4*>(p.tot + (static_cast<long long>(bh) * p.G + s) * p.R)[col4];
  carry_in_place<DECAY>(base, R4, cbeg, cend, p.NC - 1, gC, aL, carry);
}

template <bool DECAY>
cudaError_t go(const PrefillParams& p, const GammaTable& gt, int mode, cudaStream_t s,
               Recorder* rec) {
  const int R4 = p.R / 4;
  const long long nblk = (R4 + kScanThreads - 1) / kScanThreads;
  if (mode == 1) {
    if (rec) rec->mark(s, "k2_sequential");
    k2_sequential<DECAY><<<static_cast<unsigned>(nblk * p.BH), kScanThreads, 0, s>>>(p, gt);
    return cudaGetLastError();
  }
  const long long grid = nblk * p.G * p.BH;
  const long long ncb = (R4 + 31) / 32;
  if (p.Ls == 1) {
    // Every segment is one element: the Hillis-Steele scan alone, in place on the records.
    PrefillParams q = p;
    q.tot = p.rec;
    if (rec) rec->mark(s, "k2_scan_totals");
    k2_scan_totals<DECAY><<<static_cast<unsigned>(ncb * p.BH), dim3(32, 32), 0, s>>>(q, gt);
    return cudaGetLastError();
  }
  if (rec) rec->mark(s, "k2_reduce");
  k2_reduce<DECAY><<<static_cast<unsigned>(grid), kScanThreads, 0, s>>>(p, gt);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (rec) rec->mark(s, "k2_scan_totals");
  k2_scan_totals<DECAY><<<static_cast<unsigned>(ncb * p.BH), dim3(32, 32), 0, s>>>(p, gt);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (rec) rec->mark(s, "k2_downsweep");
  k2_downsweep<DECAY><<<static_cast<unsigned>(grid), kScanThreads, 0, s>>>(p, gt);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_k2(const PrefillParams& p, const GammaTable& gt, int mode, Flags f,
                      cudaStream_t s, Recorder* rec) {
  return f.decay ? go<true>(p, gt, mode, s, rec) : go<false>(p, gt, mode, s, rec);
}

}  // namespace la
