// Segmented variant of the prefill: the chunk axis is cut into segments of Lseg chunks.
//
//   K1s  one CTA per (b*H + h, segment): loops over the segment's chunks (double-buffered
//        TMA) and accumulates the segment total  T_s = sum_tau gamma^(len_s - 1 - tau)
//        psi(k_tau) v_tau^T  (and Z_s) in one TMEM accumulator.  Only one record per
//        segment reaches HBM.
//   K2   the same exclusive scan as the chunked variant, run over segments (each segment
//        is one scan element with decay gamma^(len_s)).
//   K3s  one CTA per segment: starts from the segment's exclusive prefix and walks its
//        chunks in order.  For each chunk it combines the intra-chunk part with the
//        carried prefix P (exactly K3's arithmetic), then advances the prefix in TMEM,
//        P <- gamma^(L_c) P + V^T (Xi .* psi(K)), with one more MMA chain.
//
// This is the hierarchical form of the scan page's method ("Log-Depth Chunked
// Linear-Attention Scan": the associative combine of chunk summaries, here first inside a
// segment, sequentially, then across segments, log-depth) with the intra-chunk state
// passing of fused chunk kernels ("Linear Attention and Retentive Networks ...",
// "FlashLinearAttention: I/O-Aware GPU Kernels").  Per-chunk summaries never go to HBM:
// HBM traffic is q, k, v read (k, v twice), the output written, and one record per
// segment.
//
// Layout of K3s (dv = 128): the prefix lives in TMEM as P^T (lane j = value feature,
// column i = key feature, float32).  Each chunk it is split into bf16 hi + lo and stored
// back into TMEM as the A operand of  X^T = P^T psi(Q)^T  (M = dv = 128, N = 64 tokens).
// The local part is computed transposed as well, N^T = V^T A^T, so the epilogue reads
// output columns (token t) per lane (feature j).  Precision: the same hi/lo splits as the
// chunked kernels (tc_kernels.cu).

#include <cuda_bf16.h>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace la {
namespace {

constexpr int kC = 64;
constexpr int kThreads = 256;  // 8 warps: two warps per TMEM lane quarter share its columns
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

__device__ __forceinline__ void unpack8(uint4 raw, float (&x)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __bfloat1622float2(h[e]);
    x[2 * e] = f.x;
    x[2 * e + 1] = f.y;
  }
}

__device__ __forceinline__ uint4 pack8(const float (&x)[8]) {
  uint4 raw;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
  for (int e = 0; e < 4; ++e) h[e] = __floats2bfloat162_rn(x[2 * e], x[2 * e + 1]);
  return raw;
}

__device__ __forceinline__ void split8(const float (&x)[8], uint4& hi, uint4& lo) {
  hi = pack8(x);
  float h[8], r[8];
  unpack8(hi, h);
#pragma unroll
  for (int e = 0; e < 8; ++e) r[e] = x[e] - h[e];
  lo = pack8(r);
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Uniform bounded wait: every thread waits; if any gave up the whole CTA reports and
// leaves (after freeing its TMEM).
#define LA_WAIT_OR_LEAVE(bar, parity, code, tmem, ncols)          \
  do {                                                            \
    const bool ok_ = mbar_wait((bar), (parity));                  \
    if (__syncthreads_or(!ok_)) {                                 \
      if (threadIdx.x == 0) report_error(sp.err, (code));         \
      if ((threadIdx.x >> 5) == 0) tmem_dealloc((tmem), (ncols)); \
      return;                                                     \
    }                                                             \
  } while (0)

// ---------------------------------------------------------------------------------------
// K1s

template <int DK, int DV>
struct K1sSmem {
  static constexpr uint32_t kK = DK * kC * 2;
  static constexpr uint32_t kV = DV * kC * 2;
  static constexpr uint32_t kStage = kK + kV;
  static constexpr uint32_t kIn = 2 * kStage + kK;  // two stages + the lo tile of K'
  static constexpr uint32_t kS = DK * DV * 4;       // staging of T_s^T, aliases the inputs
  static constexpr uint32_t kRegion = kIn > kS ? kIn : kS;
  static constexpr uint32_t kTotal = kRegion + kWarps * DK * 4 + 64 + 1024;
};

template <int DK, int DV, int FM, bool DECAY, bool NORM>
__global__ void __launch_bounds__(kThreads, 1)
k1_seg(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
       const __grid_constant__ CUtensorMap tm_srec, SegParams sp, GammaTable gt) {
  using L_ = K1sSmem<DK, DV>;
  constexpr bool kSplit = FM == 1 || DECAY;
  constexpr uint32_t kTmemCols = DK;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1024(smem_raw);
  uint8_t* sKl = base + 2 * L_::kStage;
  uint8_t* sS = base;
  float* sZ = reinterpret_cast<float*>(base + L_::kRegion);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sZ + kWarps * DK);  // tma[2], mma
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3);

  if (error_pending(sp.err)) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int seg = static_cast<int>(blockIdx.x % sp.NS);
  const int bh = static_cast<int>(blockIdx.x / sp.NS);
  const int cb = seg * sp.Lseg;
  const int ce = min(sp.NC, cb + sp.Lseg);
  const int n = ce - cb;
  const long long tok0 = static_cast<long long>(cb) * kC;
  const long long tok1 = min(sp.T, static_cast<long long>(ce) * kC);
  const int seg_tokens = static_cast<int>(tok1 - tok0);
  const float g = DECAY ? gt.g[bh % sp.H] : 1.f;

  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    mbar_init(&bars[2], 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_srec);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto issue_load = [&](int i) {
    uint8_t* sK = base + (i & 1) * L_::kStage;
    uint8_t* sV = sK + L_::kK;
    const int t0 = (cb + i) * kC;
    mbar_arrive_expect_tx(&bars[i & 1], L_::kK + L_::kV);
#pragma unroll
    for (int b = 0; b < DK / 64; ++b) tma_load_3d(sK + b * kC * 128, &tm_k, &bars[i & 1], b * 64, t0, bh);
#pragma unroll
    for (int b = 0; b < DV / 64; ++b) tma_load_3d(sV + b * kC * 128, &tm_v, &bars[i & 1], b * 64, t0, bh);
  };
  if (tid == 0) issue_load(0);

  constexpr int NCC = DK / 8;
  constexpr int RG = kThreads / NCC;
  const int cc = tid % NCC, rg = tid / NCC;
  float zacc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) zacc[e] = 0.f;

  for (int i = 0; i < n; ++i) {
    const int c = cb + i;
    const int L = chunk_len(sp, c);
    uint8_t* sK = base + (i & 1) * L_::kStage;
    uint8_t* sV = sK + L_::kK;
    if (i >= 1) LA_WAIT_OR_LEAVE(&bars[2], (i - 1) & 1, kErrMmaTimeout, tmem, kTmemCols);
    if (tid == 0 && i + 1 < n) issue_load(i + 1);
    LA_WAIT_OR_LEAVE(&bars[i & 1], (i >> 1) & 1, kErrTmaTimeout, tmem, kTmemCols);

    if constexpr (kSplit || NORM) {
      const uint32_t boff = (cc / 8) * (kC * 128);
      for (int r = rg; r < kC; r += RG) {
        const uint32_t off = boff + sw128_offset(r, cc % 8);
        const int tau = i * kC + r;  // token within the segment
        const float w = r < L ? (DECAY ? powf(g, static_cast<float>(seg_tokens - 1 - tau)) : 1.f) : 0.f;
        float x[8];
        unpack8(*reinterpret_cast<const uint4*>(sK + off), x);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          x[e] = feature<FM>(x[e]) * w;
          zacc[e] += x[e];
        }
        if constexpr (kSplit) {
          uint4 hi, lo;
          split8(x, hi, lo);
          *reinterpret_cast<uint4*>(sK + off) = hi;
          *reinterpret_cast<uint4*>(sKl + off) = lo;
        }
      }
    }
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idesc = instr_desc(kFmtBF16, kFmtBF16, kMNMajor, kMNMajor, DV, DK);
      const uint32_t aK = smem_u32(sK), aKl = smem_u32(sKl), aV = smem_u32(sV);
#pragma unroll
      for (int kk = 0; kk < kC / 16; ++kk) {
        const uint64_t da = smem_desc_sw128(aV + kk * 2048, kC * 128, 1024);
        mma_bf16_ss(tmem, da, smem_desc_sw128(aK + kk * 2048, kC * 128, 1024), idesc,
                    (i > 0 || kk > 0) ? 1u : 0u);
        if constexpr (kSplit)
          mma_bf16_ss(tmem, da, smem_desc_sw128(aKl + kk * 2048, kC * 128, 1024), idesc, 1u);
      }
      mma_commit(&bars[2]);
    }
  }
  LA_WAIT_OR_LEAVE(&bars[2], (n - 1) & 1, kErrMmaTimeout, tmem, kTmemCols);
  tc_fence_after();

  float* srec = sp.srec + (static_cast<long long>(bh) * sp.NS + seg) * sp.R;
  if constexpr (NORM) {
#pragma unroll
    for (int e = 0; e < 8; ++e)
#pragma unroll
      for (int o = NCC; o < 32; o <<= 1) zacc[e] += __shfl_xor_sync(0xffffffffu, zacc[e], o);
    if (lane < NCC)
#pragma unroll
      for (int e = 0; e < 8; ++e) sZ[warp * DK + cc * 8 + e] = zacc[e];
    __syncthreads();
    if (tid < DK) {
      float z = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) z += sZ[w * DK + tid];
      srec[DK * DV + tid] = z;
    }
  }

  // Epilogue: warps w and w + 4 read the same TMEM lanes, each half of the columns.
  const int quarter = warp & 3, half = warp >> 2;
  const int row = DV == 128 ? quarter * 32 + lane : quarter * 16 + lane;
  const bool valid = DV == 128 || lane < 16;
  const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
#pragma unroll
  for (int q4 = half * (DK / 64); q4 < (half + 1) * (DK / 64); ++q4) {
    float r[32];
    tmem_ld32(tmem + lane_base + q4 * 32, r);
    tmem_ld_wait();
    if (valid) {
      uint8_t* box = sS + q4 * (DV * 128);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        *reinterpret_cast<float4*>(box + sw128_offset(row, q)) =
            make_float4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
#pragma unroll
    for (int q4 = 0; q4 < DK / 32; ++q4)
      tma_store_3d(&tm_srec, sS + q4 * (DV * 128), q4 * 32, 0, bh * sp.NS + seg);
    bulk_commit();
    bulk_wait_read_all();
  }
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------------------
// K3s (dv = 128), warp-specialised.
//
// 416 threads in three roles that hand work over through mbarriers, so that the
// transform of chunk i + 1 overlaps the MMAs and epilogues of chunk i:
//   warps 0-3  transform: psi on the staged Q, K (bf16 hi / lo operand tiles, double
//              buffered), Xi .* psi(K), psi(q).ZP and the Z update; then the prefix
//              operand: P^T from TMEM -> bf16 hi / lo into TMEM, and P scaled by gamma^L.
//   warps 4-11 epilogue (two warps per TMEM lane quarter, each half of the columns):
//              masks and decays the scores into A (hi / lo), then combines
//              o = Theta X + N (/ den) and stores the chunk's output tile with TMA.
//   warp 12    control (one thread): TMA loads two chunks ahead and every tcgen05.mma;
//              the next chunk's scores are issued before the current chunk's local
//              product has finished.
// Warp w reads TMEM lanes 32 (w % 4) .. + 31.  Accumulators (TMEM columns): scores
// [0, 64), X (two buffers) [64, 128) and [448, 512), N [128, 192), P [192, 192 + dk),
// P hi / lo after it.  Each is released by an mbarrier once its readers are done.

constexpr int kThreads3 = 416;

template <int DK, int FM, bool DECAY, bool OUTF32>
struct K3sSmem {
  static constexpr int DV = 128;
  static constexpr uint32_t kQ = DK * kC * 2;
  static constexpr uint32_t kK = DK * kC * 2;
  static constexpr uint32_t kV = DV * kC * 2;
  static constexpr uint32_t kStage = kQ + kK + kV;
  static constexpr uint32_t kLo = FM == 1 ? kQ + kK : 0;  // lo tiles of psi(Q), psi(K)
  static constexpr uint32_t kKpp = DECAY ? 2 * kK : 0;    // Xi .* psi(K), hi + lo
  static constexpr uint32_t kA = kC * kC * 2;
  static constexpr uint32_t kO = kC * DV * (OUTF32 ? 4 : 2);
  static constexpr uint32_t kSmallFloats = 5 * DK + 10 * kC;
  static constexpr uint32_t kTotal =
      2 * kStage + 2 * kLo + 2 * kKpp + 2 * kA + kO + kSmallFloats * 4 + 16 * 8 + 1024;
};

template <int DK, int FM, bool DECAY, bool NORM, bool OUTF32>
__global__ void __launch_bounds__(kThreads3, 1)
k3_seg(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_out,
       SegParams sp, GammaTable gt) {
  constexpr int DV = 128;
  using L_ = K3sSmem<DK, FM, DECAY, OUTF32>;
  constexpr bool kSplitQK = FM == 1;
  constexpr uint32_t kTmemCols = 512;
  constexpr uint32_t kColS = 0, kColN = 128, kColP = 192;
  constexpr uint32_t kColPH = kColP + DK, kColPL = kColPH + DK / 2;
  constexpr uint32_t kColX[2] = {64, 448};
  static_assert(kColPL + DK / 2 <= 448, "TMEM budget");
  static_assert(L_::kTotal <= 232448, "shared memory budget");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1024(smem_raw);
  uint8_t* sLo = base + 2 * L_::kStage;      // [2] x (Q lo, K lo)
  uint8_t* sKpp = sLo + 2 * L_::kLo;         // [2] x (hi, lo)
  uint8_t* sAh = sKpp + 2 * L_::kKpp;
  uint8_t* sAl = sAh + L_::kA;
  uint8_t* sO = sAl + L_::kA;
  float* sZP = reinterpret_cast<float*>(sO + L_::kO);
  float* sZpart = sZP + DK;        // [4][DK]
  float* sDenX = sZpart + 4 * DK;  // [2][kC]
  float* sDen = sDenX + 2 * kC;
  float* sTh = sDen + kC;
  float* sPow = sTh + kC;
  float* sXi = sPow + kC;          // [2][kC]
  float* sDenPart = sXi + 2 * kC;  // [2][kC]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sDenPart + 2 * kC);
  uint64_t* full = bars;           // [2]
  uint64_t* ops = bars + 2;        // [2]
  uint64_t* pready = bars + 4;
  uint64_t* sfree = bars + 5;
  uint64_t* xfree = bars + 6;      // [2]
  uint64_t* aready = bars + 8;
  uint64_t* sdone = bars + 9;
  uint64_t* statedone = bars + 10;
  uint64_t* ndone = bars + 11;
  uint64_t* drain = bars + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 13);

  if (error_pending(sp.err)) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int seg = static_cast<int>(blockIdx.x % sp.NS);
  const int bh = static_cast<int>(blockIdx.x / sp.NS);
  const int cb = seg * sp.Lseg;
  const int ce = min(sp.NC, cb + sp.Lseg);
  const int n = ce - cb;
  const float g = DECAY ? gt.g[bh % sp.H] : 1.f;
  const float* srec = sp.srec + (static_cast<long long>(bh) * sp.NS + seg) * sp.R;

  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&full[b], 1);
      mbar_init(&ops[b], 128);
    }
    mbar_init(pready, 128);
    mbar_init(sfree, 256);
    mbar_init(&xfree[0], 256);
    mbar_init(&xfree[1], 256);
    mbar_init(aready, 256);
    mbar_init(sdone, 1);
    mbar_init(statedone, 1);
    mbar_init(ndone, 1);
    mbar_init(drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_out);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (tid < kC) {
    sTh[tid] = DECAY ? powf(g, static_cast<float>(tid + 1)) : 1.f;
    sPow[tid] = DECAY ? powf(g, static_cast<float>(tid)) : 1.f;
  }
  if constexpr (NORM) {
    if (tid < DK) sZP[tid] = srec[DK * DV + tid];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  bool failed = false;

  // A wait that runs out marks its thread failed, and a failed thread waits no more:
  // the transform and epilogue roles still walk through their named barriers (on
  // meaningless data, stored only in bounds) so that no thread of a role is left behind,
  // and the control thread drains what it has issued before TMEM is freed.
  auto wait = [&](uint64_t* bar, uint32_t parity, int code) -> bool {
    if (failed) return false;
    if (mbar_wait(bar, parity)) return true;
    report_error(sp.err, code);
    failed = true;
    return false;
  };

  if (warp < 4) {
    // ------------------------------------------------------------------ transform
    const int tw = tid;
    {  // the segment's exclusive prefix, P^T row tw, into TMEM
      const float4* src = reinterpret_cast<const float4*>(srec + static_cast<long long>(tw) * DK);
#pragma unroll
      for (int q4 = 0; q4 < DK / 32; ++q4) {
        uint32_t u[32];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float4 f = src[q4 * 8 + e];
          u[4 * e] = __float_as_uint(f.x);
          u[4 * e + 1] = __float_as_uint(f.y);
          u[4 * e + 2] = __float_as_uint(f.z);
          u[4 * e + 3] = __float_as_uint(f.w);
        }
        tmem_st32(tmem + lane_base + kColP + q4 * 32, u);
      }
      tmem_st_wait();
    }
    constexpr int NCC = DK / 8;
    constexpr int RG = 128 / NCC;
    const int cc = tw % NCC, rg = tw / NCC;
    for (int i = 0; i < n; ++i) {
      const int s = i & 1;
      const int L = chunk_len(sp, cb + i);
      const bool last = i == n - 1;
      uint8_t* sQ = base + s * L_::kStage;
      uint8_t* sK = sQ + L_::kQ;
      uint8_t* sQl = sLo + s * L_::kLo;
      uint8_t* sKl = sQl + L_::kQ;
      uint8_t* sKph = sKpp + s * L_::kKpp;
      uint8_t* sKpl = sKph + L_::kK;
      float* xi = sXi + s * kC;
      if (tw < kC) xi[tw] = tw < L ? (DECAY ? powf(g, static_cast<float>(L - 1 - tw)) : 1.f) : 0.f;
      wait(&full[s], (i >> 1) & 1, kErrTmaTimeout);
      named_barrier(1, 128);

      float zacc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) zacc[e] = 0.f;
      const uint32_t boff = (cc / 8) * (kC * 128);
      float zp[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) zp[e] = NORM ? sZP[cc * 8 + e] : 0.f;
      for (int r = rg; r < kC; r += RG) {
        const uint32_t off = boff + sw128_offset(r, cc % 8);
        if constexpr (kSplitQK || DECAY || NORM) {
          float x[8];
          unpack8(*reinterpret_cast<const uint4*>(sK + off), x);
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = r < L ? feature<FM>(x[e]) : 0.f;
          if constexpr (kSplitQK) {
            uint4 hi, lo;
            split8(x, hi, lo);
            *reinterpret_cast<uint4*>(sK + off) = hi;
            *reinterpret_cast<uint4*>(sKl + off) = lo;
          }
          const float w = xi[r];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            x[e] *= w;
            zacc[e] += x[e];
          }
          if constexpr (DECAY) {
            uint4 hi, lo;
            split8(x, hi, lo);
            *reinterpret_cast<uint4*>(sKph + off) = hi;
            *reinterpret_cast<uint4*>(sKpl + off) = lo;
          }
        }
        if constexpr (kSplitQK || NORM) {
          float x[8];
          unpack8(*reinterpret_cast<const uint4*>(sQ + off), x);
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = feature<FM>(x[e]);
          if constexpr (kSplitQK) {
            uint4 hi, lo;
            split8(x, hi, lo);
            *reinterpret_cast<uint4*>(sQ + off) = hi;
            *reinterpret_cast<uint4*>(sQl + off) = lo;
          }
          if constexpr (NORM) {
            float part = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) part = fmaf(x[e], zp[e], part);
#pragma unroll
            for (int o = NCC / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
            if (cc == 0) sDenX[s * kC + r] = part;
          }
        }
      }
      fence_async_smem();
      mbar_arrive(&ops[s]);

      const float a_c = DECAY ? powf(g, static_cast<float>(L)) : 1.f;
      if constexpr (NORM) {
#pragma unroll
        for (int e = 0; e < 8; ++e)
#pragma unroll
          for (int o = NCC; o < 32; o <<= 1) zacc[e] += __shfl_xor_sync(0xffffffffu, zacc[e], o);
        if (lane < NCC)
#pragma unroll
          for (int e = 0; e < 8; ++e) sZpart[warp * DK + cc * 8 + e] = zacc[e];
        named_barrier(1, 128);
        if (tw < DK)
          sZP[tw] = fmaf(a_c, sZP[tw],
                         sZpart[tw] + sZpart[DK + tw] + sZpart[2 * DK + tw] + sZpart[3 * DK + tw]);
      }

      // Prefix operand for chunk i (the state after chunk i - 1).
      if (i > 0) wait(statedone, (i - 1) & 1, kErrMmaTimeout);
      tc_fence_after();
#pragma unroll
      for (int q4 = 0; q4 < DK / 32; ++q4) {
        float rr[32];
        tmem_ld32(tmem + lane_base + kColP + q4 * 32, rr);
        tmem_ld_wait();
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const __nv_bfloat162 h = __floats2bfloat162_rn(rr[2 * e], rr[2 * e + 1]);
          const float2 hf = __bfloat1622float2(h);
          hi[e] = *reinterpret_cast<const uint32_t*>(&h);
          lo[e] = pack2(rr[2 * e] - hf.x, rr[2 * e + 1] - hf.y);
        }
        tmem_st16(tmem + lane_base + kColPH + q4 * 16, hi);
        tmem_st16(tmem + lane_base + kColPL + q4 * 16, lo);
        if constexpr (DECAY) {
          if (!last) {
            uint32_t u[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(rr[e] * a_c);
            tmem_st32(tmem + lane_base + kColP + q4 * 32, u);
          }
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(pready);
    }
  } else if (warp < 12) {
    // ------------------------------------------------------------------ epilogue
    const int tw = tid - 128;
    const int quarter = warp & 3, half = (warp - 4) >> 2;
    for (int i = 0; i < n; ++i) {
      const int s = i & 1;
      const int t0 = (cb + i) * kC;
      const bool has_prefix = !(seg == 0 && i == 0);
      wait(sdone, i & 1, kErrMmaTimeout);
      wait(&ops[s], (i >> 1) & 1, kErrMmaTimeout);
      tc_fence_after();
      {
        // Rows 16 quarter .. + 15 (lanes 0-15), keys 32 half .. + 31.
        const int row = quarter * 16 + lane;
        float sc[32];
        tmem_ld32(tmem + lane_base + kColS + 32 * half, sc);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(sfree);
        if (lane < 16) {
          float den_loc = 0.f;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float a[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int j = 32 * half + q * 8 + e;
              a[e] = j <= row ? sc[q * 8 + e] * sPow[row - j] : 0.f;
              den_loc += a[e];
            }
            uint4 hi, lo;
            split8(a, hi, lo);
            *reinterpret_cast<uint4*>(sAh + sw128_offset(row, 4 * half + q)) = hi;
            *reinterpret_cast<uint4*>(sAl + sw128_offset(row, 4 * half + q)) = lo;
          }
          if constexpr (NORM) sDenPart[half * kC + row] = den_loc;
        }
      }
      // psi(q).ZP of this chunk is read before A is handed over: once N(i) is done the
      // stage (and its sDenX slot) is refilled with chunk i + 2.
      const float denx = NORM && has_prefix && tw < kC ? sDenX[s * kC + tw] : 0.f;
      fence_async_smem();
      mbar_arrive(aready);
      if constexpr (NORM) {
        named_barrier(2, 256);
        if (tw < kC) sDen[tw] = fmaf(sTh[tw], denx, sDenPart[tw] + sDenPart[kC + tw]) + sp.eps;
      }

      wait(ndone, i & 1, kErrMmaTimeout);
      tc_fence_after();
      // Column j (value feature), tokens 32 half .. + 31.
      float xo[32], no[32];
      if (has_prefix) tmem_ld32(tmem + lane_base + kColX[s] + 32 * half, xo);
      tmem_ld32(tmem + lane_base + kColN + 32 * half, no);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&xfree[s]);
      if (tw == 0) bulk_wait_read_all();  // the previous tile has left the staging buffer
      named_barrier(2, 256);
      const int j = quarter * 32 + lane;
#pragma unroll
      for (int tt = 0; tt < kC / 2; ++tt) {
        const int t = 32 * half + tt;
        float o = has_prefix ? fmaf(sTh[t], xo[tt], no[tt]) : no[tt];
        if constexpr (NORM) o = o / sDen[t];
        if constexpr (OUTF32) {
          *reinterpret_cast<float*>(sO + (j / 32) * (kC * 128) + sw128_offset(t, (j % 32) / 4) +
                                    (j % 4) * 4) = o;
        } else {
          *reinterpret_cast<__nv_bfloat16*>(sO + (j / 64) * (kC * 128) +
                                            sw128_offset(t, (j % 64) / 8) + (j % 8) * 2) =
              __float2bfloat16_rn(o);
        }
      }
      fence_async_smem();
      named_barrier(2, 256);
      if (tw == 0) {
        constexpr int kOutCols = OUTF32 ? 32 : 64;
#pragma unroll
        for (int b = 0; b < DV / kOutCols; ++b)
          tma_store_3d(&tm_out, sO + b * (kC * 128), b * kOutCols, t0, bh);
        bulk_commit();
      }
    }
    if (tw == 0) bulk_wait_read_all();
  } else if (lane == 0) {
    // ------------------------------------------------------------------ control
    auto issue_load = [&](int i) {
      uint8_t* sQ = base + (i & 1) * L_::kStage;
      uint8_t* sK = sQ + L_::kQ;
      uint8_t* sV = sK + L_::kK;
      const int t0 = (cb + i) * kC;
      mbar_arrive_expect_tx(&full[i & 1], L_::kStage);
#pragma unroll
      for (int b = 0; b < DK / 64; ++b) {
        tma_load_3d(sQ + b * kC * 128, &tm_q, &full[i & 1], b * 64, t0, bh);
        tma_load_3d(sK + b * kC * 128, &tm_k, &full[i & 1], b * 64, t0, bh);
      }
#pragma unroll
      for (int b = 0; b < DV / 64; ++b) tma_load_3d(sV + b * kC * 128, &tm_v, &full[i & 1], b * 64, t0, bh);
    };
    auto issue_scores = [&](int i) -> bool {
      const int s = i & 1;
      uint8_t* sQ = base + s * L_::kStage;
      const uint32_t aQ = smem_u32(sQ), aK = aQ + L_::kQ;
      const uint32_t aQl = smem_u32(sLo + s * L_::kLo), aKl = aQl + L_::kQ;
      if (!wait(&ops[s], (i >> 1) & 1, kErrMmaTimeout)) return false;
      if (i > 0 && !wait(sfree, (i - 1) & 1, kErrMmaTimeout)) return false;
      tc_fence_after();
      constexpr uint32_t ids = instr_desc(kFmtBF16, kFmtBF16, kKMajor, kKMajor, 64, 64);
#pragma unroll
      for (int kk = 0; kk < DK / 16; ++kk) {
        const uint32_t off = (kk / 4) * (kC * 128) + (kk % 4) * 32;
        const uint64_t qh = smem_desc_sw128(aQ + off, 16, 1024);
        const uint64_t kh = smem_desc_sw128(aK + off, 16, 1024);
        mma_bf16_ss(tmem + kColS, qh, kh, ids, kk > 0 ? 1u : 0u);
        if constexpr (kSplitQK) {
          mma_bf16_ss(tmem + kColS, qh, smem_desc_sw128(aKl + off, 16, 1024), ids, 1u);
          mma_bf16_ss(tmem + kColS, smem_desc_sw128(aQl + off, 16, 1024), kh, ids, 1u);
        }
      }
      mma_commit(sdone);
      return true;
    };
    int loads = 0;
    issue_load(loads++);
    if (n > 1) issue_load(loads++);
    issue_scores(0);
    for (int i = 0; i < n && !failed; ++i) {
      const int s = i & 1;
      const bool last = i == n - 1;
      const bool has_prefix = !(seg == 0 && i == 0);
      uint8_t* sQ = base + s * L_::kStage;
      const uint32_t aQ = smem_u32(sQ), aK = aQ + L_::kQ, aV = aK + L_::kK;
      const uint32_t aQl = smem_u32(sLo + s * L_::kLo), aKl = aQl + L_::kQ;
      const uint32_t aKph = smem_u32(sKpp + s * L_::kKpp), aKpl = aKph + L_::kK;

      // X(i) = P^T psi(Q)^T and the prefix update with chunk i.
      if (!wait(pready, i & 1, kErrMmaTimeout)) break;
      if (i > 1 && !wait(&xfree[s], ((i - 2) >> 1) & 1, kErrMmaTimeout)) break;
      tc_fence_after();
      if (has_prefix) {
        constexpr uint32_t idx = instr_desc(kFmtBF16, kFmtBF16, kKMajor, kKMajor, 128, 64);
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
          const uint32_t off = (kk / 4) * (kC * 128) + (kk % 4) * 32;
          const uint64_t qh = smem_desc_sw128(aQ + off, 16, 1024);
          mma_bf16_ts(tmem + kColX[s], tmem + kColPH + kk * 8, qh, idx, kk > 0 ? 1u : 0u);
          mma_bf16_ts(tmem + kColX[s], tmem + kColPL + kk * 8, qh, idx, 1u);
          if constexpr (kSplitQK)
            mma_bf16_ts(tmem + kColX[s], tmem + kColPH + kk * 8,
                        smem_desc_sw128(aQl + off, 16, 1024), idx, 1u);
        }
      }
      if (!last) {
        constexpr uint32_t idp = instr_desc(kFmtBF16, kFmtBF16, kMNMajor, kMNMajor, 128, DK);
        const uint32_t bh_ = DECAY ? aKph : aK;
        const uint32_t bl_ = DECAY ? aKpl : aKl;
#pragma unroll
        for (int kk = 0; kk < kC / 16; ++kk) {
          const uint64_t da = smem_desc_sw128(aV + kk * 2048, kC * 128, 1024);
          mma_bf16_ss(tmem + kColP, da, smem_desc_sw128(bh_ + kk * 2048, kC * 128, 1024), idp, 1u);
          if constexpr (kSplitQK || DECAY)
            mma_bf16_ss(tmem + kColP, da, smem_desc_sw128(bl_ + kk * 2048, kC * 128, 1024), idp, 1u);
        }
      }
      mma_commit(statedone);

      // N(i) = V^T A^T.
      if (!wait(aready, i & 1, kErrMmaTimeout)) break;
      tc_fence_after();
      constexpr uint32_t idn = instr_desc(kFmtBF16, kFmtBF16, kMNMajor, kKMajor, 128, 64);
      const uint32_t aAh = smem_u32(sAh), aAl = smem_u32(sAl);
#pragma unroll
      for (int kk = 0; kk < kC / 16; ++kk) {
        const uint64_t da = smem_desc_sw128(aV + kk * 2048, kC * 128, 1024);
        mma_bf16_ss(tmem + kColN, da, smem_desc_sw128(aAh + kk * 32, 16, 1024), idn,
                    kk > 0 ? 1u : 0u);
        mma_bf16_ss(tmem + kColN, da, smem_desc_sw128(aAl + kk * 32, 16, 1024), idn, 1u);
      }
      mma_commit(ndone);

      // The next chunk's scores go in behind N(i); the stage of chunk i is refilled with
      // chunk i + 2 once all of chunk i's MMAs are done.
      if (i + 1 < n && !issue_scores(i + 1)) break;
      if (i + 2 < n) {
        if (!wait(ndone, i & 1, kErrMmaTimeout)) break;
        issue_load(loads++);
      }
    }
    if (failed) {
      // Let the issued MMAs finish and the last two loads land before TMEM and shared
      // memory are given up; both waits are bounded.
      mma_commit(drain);
      mbar_wait(drain, 0);
      for (int j = max(0, loads - 2); j < loads; ++j) mbar_wait(&full[j & 1], (j >> 1) & 1);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------------------
// Launchers

template <typename Kern>
cudaError_t set_smem(Kern kern, uint32_t bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(bytes));
}

template <int DK, int DV, int FM, bool DECAY, bool NORM>
cudaError_t k1s_go(const SegParams& sp, const GammaTable& gt, const TcMaps& m, Flags,
                   cudaStream_t s) {
  auto kern = k1_seg<DK, DV, FM, DECAY, NORM>;
  const uint32_t sm = K1sSmem<DK, DV>::kTotal;
  cudaError_t e = set_smem(kern, sm);
  if (e != cudaSuccess) return e;
  const long long grid = static_cast<long long>(sp.BH) * sp.NS;
  kern<<<static_cast<unsigned>(grid), kThreads, sm, s>>>(m.k, m.v, m.rec, sp, gt);
  return cudaGetLastError();
}

template <int DK, int FM, bool DECAY, bool NORM, bool OUTF32>
cudaError_t k3s_go_o(const SegParams& sp, const GammaTable& gt, const TcMaps& m, cudaStream_t s) {
  auto kern = k3_seg<DK, FM, DECAY, NORM, OUTF32>;
  const uint32_t sm = K3sSmem<DK, FM, DECAY, OUTF32>::kTotal;
  cudaError_t e = set_smem(kern, sm);
  if (e != cudaSuccess) return e;
  const long long grid = static_cast<long long>(sp.BH) * sp.NS;
  kern<<<static_cast<unsigned>(grid), kThreads3, sm, s>>>(m.q, m.k, m.v, m.out, sp, gt);
  return cudaGetLastError();
}

template <int DK, int DV, int FM, bool DECAY, bool NORM>
cudaError_t k3s_go(const SegParams& sp, const GammaTable& gt, const TcMaps& m, Flags f,
                   cudaStream_t s) {
  static_assert(DV == 128, "the segmented combine needs dv = 128");
  if constexpr (FM == 1 && DECAY) {
    return cudaErrorInvalidValue;  // excluded by seg_supported (shared memory budget)
  } else {
    return f.out_f32 ? k3s_go_o<DK, FM, DECAY, NORM, true>(sp, gt, m, s)
                     : k3s_go_o<DK, FM, DECAY, NORM, false>(sp, gt, m, s);
  }
}

#define LA_SEG_FLAGS(DK, DV, GO)                                          \
  do {                                                                    \
    if (f.fm == 1) {                                                      \
      if (f.decay) {                                                      \
        if (f.norm) return GO<DK, DV, 1, true, true>(sp, gt, m, f, s);    \
        return GO<DK, DV, 1, true, false>(sp, gt, m, f, s);               \
      }                                                                   \
      if (f.norm) return GO<DK, DV, 1, false, true>(sp, gt, m, f, s);     \
      return GO<DK, DV, 1, false, false>(sp, gt, m, f, s);                \
    }                                                                     \
    if (f.decay) return GO<DK, DV, 0, true, false>(sp, gt, m, f, s);      \
    return GO<DK, DV, 0, false, false>(sp, gt, m, f, s);                  \
  } while (0)

}  // namespace

bool seg_supported(int dk, int dv, int C, int fm, bool decay) {
  // ELU+1 with decay needs both the psi lo tiles and the decayed key tiles double
  // buffered, which does not fit in shared memory next to the two stages.
  return C == kC && (dk == 64 || dk == 128) && dv == 128 && !(fm == 1 && decay);
}

cudaError_t launch_k1_seg(const SegParams& sp, const GammaTable& gt, const TcMaps& m, Flags f,
                          cudaStream_t s) {
  if (sp.dk == 64 && sp.dv == 128) LA_SEG_FLAGS(64, 128, k1s_go);
  if (sp.dk == 128 && sp.dv == 128) LA_SEG_FLAGS(128, 128, k1s_go);
  return cudaErrorInvalidValue;
}

cudaError_t launch_k3_seg(const SegParams& sp, const GammaTable& gt, const TcMaps& m, Flags f,
                          cudaStream_t s) {
  if (sp.dk == 64 && sp.dv == 128) LA_SEG_FLAGS(64, 128, k3s_go);
  if (sp.dk == 128 && sp.dv == 128) LA_SEG_FLAGS(128, 128, k3s_go);
  return cudaErrorInvalidValue;
}

}  // namespace la
