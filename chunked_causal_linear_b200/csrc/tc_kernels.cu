// Tensor-core K1 and K3 for bf16 inputs on sm_100a: TMA-staged tiles, tcgen05.mma with
// float32 accumulators in TMEM, TMEM -> register epilogues, TMA stores.  One CTA of 128
// threads per (b*H + h, chunk of C = 64 tokens).  dk, dv in {64, 128}.
//
// Precision.  Every operand that is not already an exact bf16 value (psi(q), psi(k) for
// the ELU+1 map, Xi psi(k), the masked scores, the float32 prefix state) is split into
// two bf16 values, x = hi + lo with hi = bf16(x) and lo = bf16(x - hi), and each product
// is accumulated as hi*hi + hi*lo + lo*hi (or hi*y + lo*y when the other side is exact).
// That keeps every product within about 2^-16 of its float32 value, so the outputs
// carry float32-level error: the normalised form's outputs shrink like 1/sqrt(t) over a
// long sequence while its first tokens stay O(|v|), and plain bf16 operands would
// exceed 2e-2 of the outputs' rms there.  The MMAs are a small share of the time next to
// the HBM traffic.
//
// Shared-memory tiles use the 128-byte swizzle that TMA writes; a tile is a stack of
// blocks of 128-byte rows (a bf16 tile of R rows x d columns is d/64 blocks of R rows, a
// float32 tile d/32 blocks).  The MMA descriptors read them K-major (a row's columns are
// the contraction) or MN-major (the rows are the contraction).
//
// K1 (chunk summaries, "Log-Depth Chunked Linear-Attention Scan", "Formulas"):
//   K' = Xi .* psi(K), zero past the chunk end; S_loc^T = V^T K'  [dv x dk]
//   (M = dv, N = dk, K = C; both operands MN-major), stored transposed so that K3 reads
//   the prefix state K-major; Z_loc = column sums of K' in float32 on CUDA cores.
// K3 (combine, same page, "Implementation notes"; decay weights from "Linear Attention
// and Retentive Networks ...", "C. Chunkwise Recurrent Representation"):
//   scores  D_S = psi(Q) psi(K)^T                      M = 64, N = 64, K = dk
//   mask    A_ij = D_S[i][j] gamma^(i-j) for j <= i, else 0
//   inter   D_X = psi(Q) P_c   (P_c arrives as P_c^T) M = 64, N = dv, K = dk
//   local   D_N = A V                                  M = 64, N = dv, K = C
//   output  o_i = Theta_i D_X[i] + D_N[i], divided by Theta_i psi(q_i).ZP_c +
//           sum_j A_ij + eps in the normalised form; Theta_i = gamma^(i+1).
// With M = 64 the accumulator rows live in TMEM lanes 0-15 of each 32-lane quarter
// (row r -> lane (r % 16) + 32 (r / 16)); in the epilogues warp w, lanes 0-15 own rows
// 16w .. 16w + 15.

#include <cuda_bf16.h>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace la {
namespace {

constexpr int kC = 64;
constexpr int kTcThreads = 128;

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

// x -> (bf16(x), bf16(x - bf16(x))), eight values at a time.
__device__ __forceinline__ void split8(const float (&x)[8], uint4& hi, uint4& lo) {
  hi = pack8(x);
  float h[8], r[8];
  unpack8(hi, h);
#pragma unroll
  for (int e = 0; e < 8; ++e) r[e] = x[e] - h[e];
  lo = pack8(r);
}

// ---------------------------------------------------------------------------------------
// K1

template <int DK, int DV>
struct K1Smem {
  static constexpr uint32_t kK = DK * kC * 2;   // one bf16 K' tile (hi or lo)
  static constexpr uint32_t kV = DV * kC * 2;
  static constexpr uint32_t kS = DK * DV * 4;   // float32 staging of S^T
  static constexpr uint32_t kIn = 2 * kK + kV;
  static constexpr uint32_t kRegion = kIn > kS ? kIn : kS;  // staging aliases the inputs
  static constexpr uint32_t kTotal = kRegion + 4 * DK * 4 + kC * 4 + 64 + 1024;
};

template <int DK, int DV, int FM, bool DECAY, bool NORM>
__global__ void __launch_bounds__(kTcThreads, 1)
k1_tc(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
      const __grid_constant__ CUtensorMap tm_rec, PrefillParams p, GammaTable gt) {
  using L_ = K1Smem<DK, DV>;
  constexpr bool kSplit = FM == 1 || DECAY;  // K' is not an exact bf16 value
  constexpr uint32_t kTmemCols = DK;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sKh = align1024(smem_raw);
  uint8_t* sKl = sKh + L_::kK;
  uint8_t* sV = sKl + L_::kK;
  uint8_t* sS = sKh;  // staging, written after the MMAs have read K' and V
  float* sZ = reinterpret_cast<float*>(sKh + L_::kRegion);
  float* sXi = sZ + 4 * DK;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sXi + kC);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);

  if (error_pending(p.err)) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = static_cast<int>(blockIdx.x % p.NC);
  const int bh = static_cast<int>(blockIdx.x / p.NC);
  const int t0 = c * kC;
  const int L = chunk_len(p, c);
  const float g = DECAY ? gt.g[bh % p.H] : 1.f;

  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_rec);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (tid < kC) sXi[tid] = tid < L ? (DECAY ? powf(g, static_cast<float>(L - 1 - tid)) : 1.f) : 0.f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (tid == 0) {
    mbar_arrive_expect_tx(&bars[0], L_::kK + L_::kV);
#pragma unroll
    for (int b = 0; b < DK / 64; ++b) tma_load_3d(sKh + b * kC * 128, &tm_k, &bars[0], b * 64, t0, bh);
#pragma unroll
    for (int b = 0; b < DV / 64; ++b) tma_load_3d(sV + b * kC * 128, &tm_v, &bars[0], b * 64, t0, bh);
  }
  bool ok = mbar_wait(&bars[0], 0);
  if (__syncthreads_or(!ok)) {
    if (tid == 0) report_error(p.err, kErrTmaTimeout);
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
    return;
  }

  // K' = Xi .* psi(K) in float32, split into bf16 hi (in place) and lo; column sums of
  // the float32 values for Z_loc.
  constexpr int NCC = DK / 8;  // 16-byte chunks per row
  constexpr int RG = kTcThreads / NCC;
  const int cc = tid % NCC, rg = tid / NCC;
  float zacc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) zacc[e] = 0.f;
  if constexpr (kSplit || NORM) {
    const uint32_t boff = (cc / 8) * (kC * 128);
    for (int r = rg; r < kC; r += RG) {
      const uint32_t off = boff + sw128_offset(r, cc % 8);
      float x[8];
      unpack8(*reinterpret_cast<const uint4*>(sKh + off), x);
      const float w = sXi[r];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        x[e] = feature<FM>(x[e]) * w;
        zacc[e] += x[e];
      }
      if constexpr (kSplit) {
        uint4 hi, lo;
        split8(x, hi, lo);
        *reinterpret_cast<uint4*>(sKh + off) = hi;
        *reinterpret_cast<uint4*>(sKl + off) = lo;
      }
    }
  }
  if constexpr (NORM) {
#pragma unroll
    for (int e = 0; e < 8; ++e)
#pragma unroll
      for (int o = NCC; o < 32; o <<= 1) zacc[e] += __shfl_xor_sync(0xffffffffu, zacc[e], o);
    if (lane < NCC)
#pragma unroll
      for (int e = 0; e < 8; ++e) sZ[warp * DK + cc * 8 + e] = zacc[e];
  }
  fence_async_smem();
  __syncthreads();

  if (tid == 0) {
    tc_fence_after();
    // D[j][i] = sum_t V[t][j] K'[t][i]: A = V^T (M = dv), B = K' (N = dk), K = tokens.
    constexpr uint32_t idesc = instr_desc(kFmtBF16, kFmtBF16, kMNMajor, kMNMajor, DV, DK);
    const uint32_t aKh = smem_u32(sKh), aKl = smem_u32(sKl), aV = smem_u32(sV);
#pragma unroll
    for (int kk = 0; kk < kC / 16; ++kk) {
      const uint64_t da = smem_desc_sw128(aV + kk * 2048, kC * 128, 1024);
      mma_bf16_ss(tmem, da, smem_desc_sw128(aKh + kk * 2048, kC * 128, 1024), idesc,
                  kk > 0 ? 1u : 0u);
      if constexpr (kSplit)
        mma_bf16_ss(tmem, da, smem_desc_sw128(aKl + kk * 2048, kC * 128, 1024), idesc, 1u);
    }
    mma_commit(&bars[1]);
  }
  float* rec = p.rec + (static_cast<long long>(bh) * p.NC + c) * p.R;
  if constexpr (NORM) {
    if (tid < DK) rec[DK * DV + tid] = sZ[tid] + sZ[DK + tid] + sZ[2 * DK + tid] + sZ[3 * DK + tid];
  }

  ok = mbar_wait(&bars[1], 0);
  if (__syncthreads_or(!ok)) {
    if (tid == 0) report_error(p.err, kErrMmaTimeout);
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
    return;
  }
  tc_fence_after();

  // Epilogue: TMEM rows (dv index) -> swizzled float32 staging (dk/32 boxes of dv rows)
  // -> TMA store into the chunk's record.
  const int row = DV == 128 ? warp * 32 + lane : warp * 16 + lane;
  const bool valid = DV == 128 || lane < 16;
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
#pragma unroll
  for (int cb = 0; cb < DK / 32; ++cb) {
    float r[32];
    tmem_ld32(tmem + lane_base + cb * 32, r);
    tmem_ld_wait();
    if (valid) {
      uint8_t* box = sS + cb * (DV * 128);
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
    for (int cb = 0; cb < DK / 32; ++cb)
      tma_store_3d(&tm_rec, sS + cb * (DV * 128), cb * 32, 0, bh * p.NC + c);
    bulk_commit();
    bulk_wait_read_all();
  }
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------------------
// K3

template <int DK, int DV, bool OUTF32>
struct K3Smem {
  static constexpr uint32_t kQ = DK * kC * 2;   // one bf16 psi(Q) tile (hi or lo)
  static constexpr uint32_t kK = DK * kC * 2;   // one bf16 psi(K) tile (hi or lo)
  static constexpr uint32_t kV = DV * kC * 2;
  static constexpr uint32_t kP = DK * DV * 4;   // float32 P^T, then bf16 hi + lo in place
  static constexpr uint32_t kA = kC * kC * 2;   // one bf16 score tile (hi or lo)
  static constexpr uint32_t kO = kC * DV * (OUTF32 ? 4 : 2);  // staging, aliases psi(Q), psi(K)
  static_assert(kO <= 2 * kQ + 2 * kK, "output staging must fit in the psi(Q), psi(K) tiles");
  static constexpr uint32_t kSmall = (DK + 4 * kC) * 4 + 64;
  static constexpr uint32_t kTotal = 2 * kQ + 2 * kK + kV + kP + 2 * kA + kSmall + 1024;
};

template <int DK, int DV, int FM, bool DECAY, bool NORM, bool OUTF32>
__global__ void __launch_bounds__(kTcThreads, 1)
k3_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_out,
      const __grid_constant__ CUtensorMap tm_rec, PrefillParams p, GammaTable gt) {
  using L_ = K3Smem<DK, DV, OUTF32>;
  constexpr bool kSplitQK = FM == 1;     // psi(q), psi(k) are not exact bf16 values
  constexpr uint32_t kTmemCols = 512;
  constexpr uint32_t kColX = 64;         // inter-chunk accumulator
  constexpr uint32_t kColN = 64 + DV;    // local accumulator
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sQh = align1024(smem_raw);
  uint8_t* sQl = sQh + L_::kQ;
  uint8_t* sKh = sQl + L_::kQ;
  uint8_t* sKl = sKh + L_::kK;
  uint8_t* sV = sKl + L_::kK;
  uint8_t* sP = sV + L_::kV;
  uint8_t* sPh = sP;
  uint8_t* sPl = sP + DK * DV * 2;
  uint8_t* sAh = sP + L_::kP;
  uint8_t* sAl = sAh + L_::kA;
  uint8_t* sO = sQh;  // written after every MMA that reads psi(Q) and psi(K) is done
  float* sZP = reinterpret_cast<float*>(sAl + L_::kA);
  float* sDenX = sZP + DK;   // psi(q_i) . ZP_c
  float* sDen = sDenX + kC;  // full denominator
  float* sTh = sDen + kC;
  float* sPow = sTh + kC;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sPow + kC);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);

  if (error_pending(p.err)) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = static_cast<int>(blockIdx.x % p.NC);
  // Chunk 0 has a prefix too when the sequence continues from an initial state.
  const bool pre = c > 0 || p.has_init;
  const int bh = static_cast<int>(blockIdx.x / p.NC);
  const int t0 = c * kC;
  const int L = chunk_len(p, c);
  const float g = DECAY ? gt.g[bh % p.H] : 1.f;
  const float* rec = p.rec + (static_cast<long long>(bh) * p.NC + c) * p.R;

  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_out);
    tma_prefetch_desc(&tm_rec);
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
    if (tid < DK) sZP[tid] = pre ? rec[DK * DV + tid] : 0.f;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (tid == 0) {
    mbar_arrive_expect_tx(&bars[0], L_::kQ + L_::kK + L_::kV + (pre ? L_::kP : 0u));
#pragma unroll
    for (int b = 0; b < DK / 64; ++b) {
      tma_load_3d(sQh + b * kC * 128, &tm_q, &bars[0], b * 64, t0, bh);
      tma_load_3d(sKh + b * kC * 128, &tm_k, &bars[0], b * 64, t0, bh);
    }
#pragma unroll
    for (int b = 0; b < DV / 64; ++b) tma_load_3d(sV + b * kC * 128, &tm_v, &bars[0], b * 64, t0, bh);
    if (pre) {
#pragma unroll
      for (int b = 0; b < DK / 32; ++b)
        tma_load_3d(sP + b * (DV * 128), &tm_rec, &bars[0], b * 32, 0, bh * p.NC + c);
    }
  }
  bool ok = mbar_wait(&bars[0], 0);
  if (__syncthreads_or(!ok)) {
    if (tid == 0) report_error(p.err, kErrTmaTimeout);
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
    return;
  }

  // psi on Q and K (K zero past the chunk end), split into bf16 hi (in place) and lo;
  // psi(q_i) . ZP_c in float32 for the denominator.
  {
    constexpr int NCC = DK / 8;
    constexpr int RG = kTcThreads / NCC;
    const int cc = tid % NCC, rg = tid / NCC;
    const uint32_t boff = (cc / 8) * (kC * 128);
    float zp[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) zp[e] = NORM ? sZP[cc * 8 + e] : 0.f;
    for (int r = rg; r < kC; r += RG) {
      const uint32_t off = boff + sw128_offset(r, cc % 8);
      if constexpr (kSplitQK) {
        float x[8];
        unpack8(*reinterpret_cast<const uint4*>(sKh + off), x);
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = r < L ? feature<FM>(x[e]) : 0.f;
        uint4 hi, lo;
        split8(x, hi, lo);
        *reinterpret_cast<uint4*>(sKh + off) = hi;
        *reinterpret_cast<uint4*>(sKl + off) = lo;
      }
      float x[8];
      unpack8(*reinterpret_cast<const uint4*>(sQh + off), x);
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = feature<FM>(x[e]);
      if constexpr (kSplitQK) {
        uint4 hi, lo;
        split8(x, hi, lo);
        *reinterpret_cast<uint4*>(sQh + off) = hi;
        *reinterpret_cast<uint4*>(sQl + off) = lo;
      }
      if constexpr (NORM) {
        float part = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) part = fmaf(x[e], zp[e], part);
#pragma unroll
        for (int o = NCC / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (cc == 0) sDenX[r] = part;
      }
    }
  }
  fence_async_smem();
  __syncthreads();

  const uint32_t aQh = smem_u32(sQh), aQl = smem_u32(sQl);
  if (tid == 0) {
    tc_fence_after();
    constexpr uint32_t idesc = instr_desc(kFmtBF16, kFmtBF16, kKMajor, kKMajor, 64, 64);
    const uint32_t aKh = smem_u32(sKh), aKl = smem_u32(sKl);
#pragma unroll
    for (int kk = 0; kk < DK / 16; ++kk) {
      const uint32_t off = (kk / 4) * (kC * 128) + (kk % 4) * 32;
      const uint64_t qh = smem_desc_sw128(aQh + off, 16, 1024);
      const uint64_t kh = smem_desc_sw128(aKh + off, 16, 1024);
      mma_bf16_ss(tmem, qh, kh, idesc, kk > 0 ? 1u : 0u);
      if constexpr (kSplitQK) {
        mma_bf16_ss(tmem, qh, smem_desc_sw128(aKl + off, 16, 1024), idesc, 1u);
        mma_bf16_ss(tmem, smem_desc_sw128(aQl + off, 16, 1024), kh, idesc, 1u);
      }
    }
    mma_commit(&bars[1]);
  }

  // Prefix state P_c^T: float32 -> bf16 hi + lo, in place (all values are read into
  // registers before any is overwritten).
  if (pre) {
    constexpr int NF = DK * DV / kTcThreads;  // floats per thread
    const int j = tid % DV;
    const int c0 = (tid / DV) * NF;
    float v[NF];
#pragma unroll
    for (int u = 0; u < NF / 4; ++u) {
      const int col = c0 + 4 * u;
      const float4 f = *reinterpret_cast<const float4*>(
          sP + (col / 32) * (DV * 128) + sw128_offset(j, (col % 32) / 4));
      v[4 * u] = f.x;
      v[4 * u + 1] = f.y;
      v[4 * u + 2] = f.z;
      v[4 * u + 3] = f.w;
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < NF / 8; ++u) {
      const int col = c0 + 8 * u;
      float x[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = v[8 * u + e];
      uint4 hi, lo;
      split8(x, hi, lo);
      const uint32_t off = (col / 64) * (DV * 128) + sw128_offset(j, (col % 64) / 8);
      *reinterpret_cast<uint4*>(sPh + off) = hi;
      *reinterpret_cast<uint4*>(sPl + off) = lo;
    }
    fence_async_smem();
  }
  __syncthreads();

  if (tid == 0 && pre) {
    tc_fence_after();
    constexpr uint32_t idx = instr_desc(kFmtBF16, kFmtBF16, kKMajor, kKMajor, 64, DV);
    const uint32_t aPh = smem_u32(sPh), aPl = smem_u32(sPl);
#pragma unroll
    for (int kk = 0; kk < DK / 16; ++kk) {
      const uint32_t offa = (kk / 4) * (kC * 128) + (kk % 4) * 32;
      const uint32_t offb = (kk / 4) * (DV * 128) + (kk % 4) * 32;
      const uint64_t qh = smem_desc_sw128(aQh + offa, 16, 1024);
      const uint64_t ph = smem_desc_sw128(aPh + offb, 16, 1024);
      mma_bf16_ss(tmem + kColX, qh, ph, idx, kk > 0 ? 1u : 0u);
      mma_bf16_ss(tmem + kColX, qh, smem_desc_sw128(aPl + offb, 16, 1024), idx, 1u);
      if constexpr (kSplitQK)
        mma_bf16_ss(tmem + kColX, smem_desc_sw128(aQl + offa, 16, 1024), ph, idx, 1u);
    }
  }

  ok = mbar_wait(&bars[1], 0);
  if (__syncthreads_or(!ok)) {
    if (tid == 0) report_error(p.err, kErrMmaTimeout);
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
    return;
  }
  tc_fence_after();

  const int row = warp * 16 + lane;
  const bool valid = lane < 16;
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
  {
    // Causal mask and decay on the scores, split into bf16 hi + lo operands for A V.
    float s[64];
    tmem_ld32(tmem + lane_base + 0, *reinterpret_cast<float(*)[32]>(&s[0]));
    tmem_ld32(tmem + lane_base + 32, *reinterpret_cast<float(*)[32]>(&s[32]));
    tmem_ld_wait();
    if (valid) {
      float den_loc = 0.f;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        float a[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int j = q * 8 + e;
          a[e] = j <= row ? s[j] * sPow[row - j] : 0.f;
          den_loc += a[e];
        }
        uint4 hi, lo;
        split8(a, hi, lo);
        *reinterpret_cast<uint4*>(sAh + sw128_offset(row, q)) = hi;
        *reinterpret_cast<uint4*>(sAl + sw128_offset(row, q)) = lo;
      }
      if constexpr (NORM) sDen[row] = fmaf(sTh[row], sDenX[row], den_loc) + p.eps;
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();

  if (tid == 0) {
    tc_fence_after();
    constexpr uint32_t idv = instr_desc(kFmtBF16, kFmtBF16, kKMajor, kMNMajor, 64, DV);
    const uint32_t aAh = smem_u32(sAh), aAl = smem_u32(sAl), aV = smem_u32(sV);
#pragma unroll
    for (int kk = 0; kk < kC / 16; ++kk) {
      const uint64_t dv_ = smem_desc_sw128(aV + kk * 2048, kC * 128, 1024);
      mma_bf16_ss(tmem + kColN, smem_desc_sw128(aAh + kk * 32, 16, 1024), dv_, idv,
                  kk > 0 ? 1u : 0u);
      mma_bf16_ss(tmem + kColN, smem_desc_sw128(aAl + kk * 32, 16, 1024), dv_, idv, 1u);
    }
    mma_commit(&bars[1]);
  }
  ok = mbar_wait(&bars[1], 1);
  if (__syncthreads_or(!ok)) {
    if (tid == 0) report_error(p.err, kErrMmaTimeout);
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
    return;
  }
  tc_fence_after();

  {
    const float den = NORM && valid ? sDen[row] : 1.f;
    const float th = valid ? sTh[row] : 0.f;
#pragma unroll
    for (int cb = 0; cb < DV / 32; ++cb) {
      float xo[32], no[32];
      tmem_ld32(tmem + lane_base + kColX + cb * 32, xo);
      tmem_ld32(tmem + lane_base + kColN + cb * 32, no);
      tmem_ld_wait();
      if (valid) {
        float o[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float num = pre ? fmaf(th, xo[e], no[e]) : no[e];
          o[e] = NORM ? num / den : num;
        }
        if constexpr (OUTF32) {
          uint8_t* ob = sO + cb * (kC * 128);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4*>(ob + sw128_offset(row, q)) =
                make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
        } else {
          uint8_t* ob = sO + (cb / 2) * (kC * 128);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float y[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) y[e] = o[8 * q + e];
            *reinterpret_cast<uint4*>(ob + sw128_offset(row, (cb % 2) * 4 + q)) = pack8(y);
          }
        }
      }
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    constexpr int kOutCols = OUTF32 ? 32 : 64;  // columns per 128-byte staging row
#pragma unroll
    for (int b = 0; b < DV / kOutCols; ++b)
      tma_store_3d(&tm_out, sO + b * (kC * 128), b * kOutCols, t0, bh);
    bulk_commit();
    bulk_wait_read_all();
  }
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
cudaError_t k1_go(const PrefillParams& p, const GammaTable& gt, const TcMaps& m, Flags,
                  cudaStream_t s) {
  auto kern = k1_tc<DK, DV, FM, DECAY, NORM>;
  const uint32_t sm = K1Smem<DK, DV>::kTotal;
  cudaError_t e = set_smem(kern, sm);
  if (e != cudaSuccess) return e;
  const long long grid = static_cast<long long>(p.BH) * p.NC;
  kern<<<static_cast<unsigned>(grid), kTcThreads, sm, s>>>(m.k, m.v, m.rec, p, gt);
  return cudaGetLastError();
}

template <int DK, int DV, int FM, bool DECAY, bool NORM, bool OUTF32>
cudaError_t k3_go_o(const PrefillParams& p, const GammaTable& gt, const TcMaps& m, cudaStream_t s) {
  auto kern = k3_tc<DK, DV, FM, DECAY, NORM, OUTF32>;
  const uint32_t sm = K3Smem<DK, DV, OUTF32>::kTotal;
  cudaError_t e = set_smem(kern, sm);
  if (e != cudaSuccess) return e;
  const long long grid = static_cast<long long>(p.BH) * p.NC;
  kern<<<static_cast<unsigned>(grid), kTcThreads, sm, s>>>(m.q, m.k, m.v, m.out, m.rec, p, gt);
  return cudaGetLastError();
}

template <int DK, int DV, int FM, bool DECAY, bool NORM>
cudaError_t k3_go(const PrefillParams& p, const GammaTable& gt, const TcMaps& m, Flags f,
                  cudaStream_t s) {
  return f.out_f32 ? k3_go_o<DK, DV, FM, DECAY, NORM, true>(p, gt, m, s)
                   : k3_go_o<DK, DV, FM, DECAY, NORM, false>(p, gt, m, s);
}

#define LA_TC_FLAGS(DK, DV, GO)                                          \
  do {                                                                   \
    if (f.fm == 1) {                                                     \
      if (f.decay) {                                                     \
        if (f.norm) return GO<DK, DV, 1, true, true>(p, gt, m, f, s);    \
        return GO<DK, DV, 1, true, false>(p, gt, m, f, s);               \
      }                                                                  \
      if (f.norm) return GO<DK, DV, 1, false, true>(p, gt, m, f, s);     \
      return GO<DK, DV, 1, false, false>(p, gt, m, f, s);                \
    }                                                                    \
    if (f.decay) return GO<DK, DV, 0, true, false>(p, gt, m, f, s);      \
    return GO<DK, DV, 0, false, false>(p, gt, m, f, s);                  \
  } while (0)

#define LA_TC_SHAPES(GO)                                                 \
  do {                                                                   \
    if (p.dk == 64 && p.dv == 64) LA_TC_FLAGS(64, 64, GO);               \
    if (p.dk == 64 && p.dv == 128) LA_TC_FLAGS(64, 128, GO);             \
    if (p.dk == 128 && p.dv == 64) LA_TC_FLAGS(128, 64, GO);             \
    if (p.dk == 128 && p.dv == 128) LA_TC_FLAGS(128, 128, GO);           \
    return cudaErrorInvalidValue;                                        \
  } while (0)

}  // namespace

cudaError_t launch_k1_tc(const PrefillParams& p, const GammaTable& gt, const TcMaps& m,
                         Flags f, cudaStream_t s) {
  if (p.C != kC) return cudaErrorInvalidValue;
  LA_TC_SHAPES(k1_go);
}

cudaError_t launch_k3_tc(const PrefillParams& p, const GammaTable& gt, const TcMaps& m,
                         Flags f, cudaStream_t s) {
  if (p.C != kC) return cudaErrorInvalidValue;
  LA_TC_SHAPES(k3_go);
}

}  // namespace la
