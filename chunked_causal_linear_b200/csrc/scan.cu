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
// Log-depth mode ("Implementation notes": a Blelloch or Hillis-Steele scan; "Verification":
// ceil(log2 N_C) rounds) is a work-efficient blocked scan (Brent's arrangement of
// Hillis-Steele).  One CTA of 1024 threads takes up to 2048 elements of the chunk axis, split
// over NG <= 128 groups of E <= 16 consecutive elements, and a slab of 1024 / NG float4
// columns (128 contiguous bytes of every record or more), one thread per (group, column):
//   k2_block_scan   pass 1: each thread folds its E elements (E dependent steps);
//                   Hillis-Steele over the NG group folds in shared memory (log2 NG
//                   rounds); pass 2: each thread re-reads its elements (from L2: a CTA's
//                   slab is at most 256 KB) and writes their exclusive prefixes in place
//                   (E steps).  Depth 2E + log2 NG, e.g. 16 + 7 + 16 at N_C = 2048; the
//                   records cross HBM once each way, as in the sequential carry.
// Beyond 2048 elements one level more: segments of Ls >= 16 chunks, G = ceil(N_C / Ls)
// <= 2048 of them:
//   k2_reduce       each segment's fold (Ls steps, parallel over segments and columns);
//   k2_block_scan   the scan above over the G segment folds, giving each segment's
//                   exclusive prefix;
//   k2_downsweep    each segment re-scans its chunks from its prefix, in place (Ls steps).
// Depth 2 Ls + 2E + log2 NG (55 at N_C = 16384).
// Sequential mode (comparison only) carries the state through every chunk in order
// (depth N_C).  Every mode reads and writes float4 columns.
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
constexpr int kBlockThreads = 1024;  // block-scan CTA, groups of one element
constexpr int kBlockThreadsU = 512;  // block-scan CTA, longer groups (two per SM)
constexpr int kMaxGroups = 128;      // groups per block-scan CTA (slab of at least 4 float4)

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
template <bool DECAY, int U = kUnroll>
__device__ __forceinline__ float4 carry_in_place(float4* base, long long stride, int cbeg,
                                                 int cend, int last, float gC, float aL,
                                                 float4 carry) {
  float4 x[U], y[U];
#pragma unroll
  for (int u = 0; u < U; ++u)
    if (cbeg + u < cend) x[u] = base[static_cast<long long>(cbeg + u) * stride];
  for (int c0 = cbeg; c0 < cend; c0 += U) {
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (c0 + U + u < cend) y[u] = base[static_cast<long long>(c0 + U + u) * stride];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (c0 + u < cend) {
        base[static_cast<long long>(c0 + u) * stride] = carry;
        const float a = DECAY ? (c0 + u == last ? aL : gC) : 1.f;
        carry = axpy4(a, carry, x[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) x[u] = y[u];
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

// Blocked scan of N = p.NC elements, in place, one CTA of NT threads per (b*H + h, slab of
// W = NT / NG float4 columns); NG groups of E consecutive elements (NG a power of two,
// NG * E >= N).
// U: loads in flight per thread (pass 1 U, pass 2 U / 2): 8 for longer groups (NT = 512,
// 64 registers, two CTAs per SM, so that one CTA's loads overlap the other's barrier rounds
// and second pass; one CTA of 1024 threads per SM left HBM idle during them), 1 for groups
// of one element (NT = 1024, 32 registers, two CTAs per SM).
template <bool DECAY, int U, int NT>
__global__ void __launch_bounds__(NT, 2)
k2_block_scan(PrefillParams p, GammaTable gt, int NG, int E) {
  __shared__ float4 sX[NT];
  __shared__ float sA[NT];
  __shared__ float sG[2];
  const int kSlab = NT / NG;  // W
  const int R4 = p.R / 4;
  const int nslab = (R4 + kSlab - 1) / kSlab;
  const int bh = blockIdx.x / nslab;
  const int c8 = threadIdx.x % kSlab;
  const int col4 = (blockIdx.x % nslab) * kSlab + c8;
  const int gi = threadIdx.x / kSlab;
  const bool live = col4 < R4;
  // The element decays gamma^C and gamma^(L_last), once per CTA.
  if (DECAY && threadIdx.x == 0) {
    const float g = gt.g[bh % p.H];
    sG[0] = powf(g, static_cast<float>(p.C));
    sG[1] = powf(g, static_cast<float>(p.L_last));
  }
  if (DECAY) __syncthreads();
  const float gC = DECAY ? sG[0] : 1.f;
  const float aL = DECAY ? sG[1] : 1.f;
  const int e0 = min(p.NC, gi * E);
  const int e1 = min(p.NC, e0 + E);
  float4* base = reinterpret_cast<float4*>(p.rec + static_cast<long long>(bh) * p.NC * p.R) + col4;

  // Pass 1: this group's fold, agg = sum_e (decay after e within the group) x_e, and the
  // group's decay A, the product of its elements' decays.
  float4 agg = make_float4(0.f, 0.f, 0.f, 0.f);
  float A = 1.f;
  if (U == 1) {
    // One element per group: it stays in registers for pass 2.
    if (live && e0 < e1) {
      agg = base[static_cast<long long>(e0) * R4];
      A = DECAY ? (e0 == p.NC - 1 ? aL : gC) : 1.f;
    }
  } else if (live) {
    for (int c0 = e0; c0 < e1; c0 += U) {
      float4 x[U];
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (c0 + u < e1) x[u] = base[static_cast<long long>(c0 + u) * R4];
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (c0 + u < e1) {
          const float a = DECAY ? (c0 + u == p.NC - 1 ? aL : gC) : 1.f;
          agg = axpy4(a, agg, x[u]);
          A *= a;
        }
    }
  }
  const float4 x_own = agg;  // the group's own fold and decay (U == 1: the element itself)
  const float a_own = A;
  // Hillis-Steele over the groups: after round r, group gi holds the fold of groups
  // gi - 2^(r+1) + 1 .. gi, and A their decay.
  for (int d = 1; d < NG; d <<= 1) {
    sX[gi * kSlab + c8] = agg;
    if (c8 == 0) sA[gi] = A;
    __syncthreads();
    if (gi >= d) {
      agg = axpy4(A, sX[(gi - d) * kSlab + c8], agg);
      A *= sA[gi - d];
    }
    __syncthreads();
  }
  // Inclusive -> exclusive over groups; the initial state enters with the decay of every
  // group before this one.
  sX[gi * kSlab + c8] = agg;
  if (c8 == 0) sA[gi] = A;
  __syncthreads();
  if (!live || e0 >= e1) return;
  const float4 init = p.has_init ? read_init(p, bh, col4 * 4) : make_float4(0.f, 0.f, 0.f, 0.f);
  float4 carry = init;
  if (gi > 0) carry = axpy4(sA[gi - 1], init, sX[(gi - 1) * kSlab + c8]);
  if (U == 1) {
    // The element's exclusive prefix; the state after it is a carry + x.
    base[static_cast<long long>(e0) * R4] = carry;
    if (e1 == p.NC) write_final(p, bh, col4 * 4, axpy4(a_own, carry, x_own));
    return;
  }
  // Pass 2: exclusive prefixes of this group's elements, in place (re-read from L2, so
  // four loads in flight suffice and keep the thread within 64 registers).
  carry = carry_in_place<DECAY, (U > 1 ? U / 2 : 1)>(base, R4, e0, e1, p.NC - 1, gC, aL, carry);
  if (e1 == p.NC) write_final(p, bh, col4 * 4, carry);
}

// The blocked scan for at most 32 elements (the segmented arrangement's usual case): lanes
// in runs of `seg` (the element count rounded up to a power of two), one run per (b*h,
// kWarpScanCols float4 columns), lane e of a run holding element e; Hillis-Steele over the
// run by shuffles (log2 seg rounds, as the blocked scan's group rounds at one element per
// group) and no CTA-wide barrier, so every warp keeps its loads in flight on its own.
// Lanes past the last element hold the identity (decay 1, state 0).
constexpr int kWarpScanCols = 4;
constexpr int kWarpScanThreads = 256;

template <bool DECAY>
__global__ void __launch_bounds__(kWarpScanThreads) k2_warp_scan(PrefillParams p, GammaTable gt,
                                                                 int seg) {
  const int lane = threadIdx.x & 31;
  const int e = lane & (seg - 1);
  const int runs = 32 / seg;
  const long long wid = (static_cast<long long>(blockIdx.x) * kWarpScanThreads + threadIdx.x) >> 5;
  const int R4 = p.R / 4;
  const long long nblk = (R4 + kWarpScanCols - 1) / kWarpScanCols;
  if (wid * runs >= nblk * p.BH) return;  // (whole warps)
  const long long blk = wid * runs + lane / seg;
  const bool in = blk < nblk * p.BH;
  const int bh = in ? static_cast<int>(blk / nblk) : 0;
  const int c0 = in ? static_cast<int>(blk % nblk) * kWarpScanCols : 0;
  float gC = 1.f, aL = 1.f;
  if (DECAY) {
    const float g = gt.g[bh % p.H];
    gC = powf(g, static_cast<float>(p.C));
    aL = powf(g, static_cast<float>(p.L_last));
  }
  const bool el = in && e < p.NC;
  float4* base = reinterpret_cast<float4*>(p.rec + static_cast<long long>(bh) * p.NC * p.R) +
                 static_cast<long long>(e) * R4 + c0;
  float4 x[kWarpScanCols];
#pragma unroll
  for (int u = 0; u < kWarpScanCols; ++u)
    x[u] = el && c0 + u < R4 ? base[u] : make_float4(0.f, 0.f, 0.f, 0.f);
  float A = el && DECAY ? (e == p.NC - 1 ? aL : gC) : 1.f;
  // Inclusive: (A, x) of elements 0..e under (a1, x1) (+) (a2, x2) = (a1 a2, a2 x1 + x2).
  for (int d = 1; d < seg; d <<= 1) {
    const float Ap = __shfl_up_sync(0xffffffffu, A, d, seg);
#pragma unroll
    for (int u = 0; u < kWarpScanCols; ++u) {
      float4 xp;
      xp.x = __shfl_up_sync(0xffffffffu, x[u].x, d, seg);
      xp.y = __shfl_up_sync(0xffffffffu, x[u].y, d, seg);
      xp.z = __shfl_up_sync(0xffffffffu, x[u].z, d, seg);
      xp.w = __shfl_up_sync(0xffffffffu, x[u].w, d, seg);
      if (e >= d) x[u] = axpy4(A, xp, x[u]);
    }
    if (e >= d) A *= Ap;
  }
  // Exclusive: element e's prefix is (A, x) of elements 0..e-1 applied to the initial state.
  const float Ae = __shfl_up_sync(0xffffffffu, A, 1, seg);
#pragma unroll
  for (int u = 0; u < kWarpScanCols; ++u) {
    const bool live = c0 + u < R4;
    const float4 init = el && live && p.has_init ? read_init(p, bh, (c0 + u) * 4)
                                                 : make_float4(0.f, 0.f, 0.f, 0.f);
    float4 xe;
    xe.x = __shfl_up_sync(0xffffffffu, x[u].x, 1, seg);
    xe.y = __shfl_up_sync(0xffffffffu, x[u].y, 1, seg);
    xe.z = __shfl_up_sync(0xffffffffu, x[u].z, 1, seg);
    xe.w = __shfl_up_sync(0xffffffffu, x[u].w, 1, seg);
    if (el && live) {
      base[u] = e == 0 ? init : axpy4(Ae, init, xe);
      if (e == p.NC - 1) write_final(p, bh, (c0 + u) * 4, axpy4(A, init, x[u]));
    }
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
cudaError_t block_scan(const PrefillParams& p, const GammaTable& gt, cudaStream_t s,
                       Recorder* rec) {
  if (p.NC <= 32) {
    if (rec) rec->mark(s, "k2_warp_scan");
    int seg = 1;
    while (seg < p.NC) seg <<= 1;
    const long long runs =
        static_cast<long long>((p.R / 4 + kWarpScanCols - 1) / kWarpScanCols) * p.BH;
    const long long warps = (runs + 32 / seg - 1) / (32 / seg);
    const long long blocks = (warps * 32 + kWarpScanThreads - 1) / kWarpScanThreads;
    k2_warp_scan<DECAY><<<static_cast<unsigned>(blocks), kWarpScanThreads, 0, s>>>(p, gt, seg);
    return cudaGetLastError();
  }
  if (rec) rec->mark(s, "k2_block_scan");
  const ScanPlan bp = scan_plan(p.NC);  // p.NC <= kScanBlockElems: a single block level
  const int R4 = p.R / 4;
  const int nt = bp.E == 1 ? kBlockThreads : kBlockThreadsU;
  const int W = nt / bp.NG;
  const long long nslab = (R4 + W - 1) / W;
  const unsigned grid = static_cast<unsigned>(nslab * p.BH);
  if (bp.E == 1)
    k2_block_scan<DECAY, 1, kBlockThreads><<<grid, kBlockThreads, 0, s>>>(p, gt, bp.NG, bp.E);
  else
    k2_block_scan<DECAY, kUnroll, kBlockThreadsU><<<grid, kBlockThreadsU, 0, s>>>(p, gt, bp.NG, bp.E);
  return cudaGetLastError();
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
  if (p.NC <= kScanBlockElems) {
    // One block level: the blocked scan alone, in place on the records.
    return block_scan<DECAY>(p, gt, s, rec);
  }
  // Two levels: segment folds, the blocked scan over them, the per-segment sweep.
  const ScanPlan plan = scan_plan(p.NC);
  if (plan.Ls != p.Ls || plan.G != p.G) return cudaErrorInvalidValue;
  const long long grid = nblk * p.G * p.BH;
  if (rec) rec->mark(s, "k2_reduce");
  k2_reduce<DECAY><<<static_cast<unsigned>(grid), kScanThreads, 0, s>>>(p, gt);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // The scan over segments: one element per segment, each of Ls chunks (the last one
  // holding what is left).
  PrefillParams q = p;
  q.rec = p.tot;
  q.NC = p.G;
  q.C = p.C * p.Ls;
  q.L_last = static_cast<int>(p.T - static_cast<long long>(p.G - 1) * p.Ls * p.C);
  e = block_scan<DECAY>(q, gt, s, rec);
  if (e != cudaSuccess) return e;
  if (rec) rec->mark(s, "k2_downsweep");
  k2_downsweep<DECAY><<<static_cast<unsigned>(grid), kScanThreads, 0, s>>>(p, gt);
  return cudaGetLastError();
}

}  // namespace

ScanPlan scan_plan(long long n) {
  ScanPlan pl;
  if (n <= 0) return pl;
  long long m = n;  // elements of the block level
  if (n > kScanBlockElems) {
    long long ls = (n + kScanBlockElems - 1) / kScanBlockElems;
    if (ls < kScanMinSegment) ls = kScanMinSegment;
    pl.Ls = static_cast<int>(ls);
    pl.G = static_cast<int>((n + ls - 1) / ls);
    m = pl.G;
  } else {
    pl.Ls = static_cast<int>(n);
    pl.G = 1;
  }
  int ng = 1, lg = 0;
  while (ng < m && ng < kMaxGroups) {
    ng <<= 1;
    ++lg;
  }
  pl.NG = ng;
  pl.E = static_cast<int>((m + ng - 1) / ng);
  pl.depth = 2LL * pl.E + lg + (n > kScanBlockElems ? 2LL * pl.Ls : 0);
  return pl;
}

cudaError_t launch_k2(const PrefillParams& p, const GammaTable& gt, int mode, Flags f,
                      cudaStream_t s, Recorder* rec) {
  return f.decay ? go<true>(p, gt, mode, s, rec) : go<false>(p, gt, mode, s, rec);
}

}  // namespace la
