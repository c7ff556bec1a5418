// Gated linear attention on the tensor cores, in the segmented arrangement.
//
// The recurrence of "Linear Attention and Retentive Networks ..." (Gated Linear Attention
// (GLA) and Hardware-Software Co-Design),  S_t = (alpha_t 1^T) (.) S_{t-1} + k_t^T v_t,
// o_t = q_t S_t,  with a gate alpha_t[f] in [0, 1] per token and key feature.  Write
// l_t = log2 alpha_t (a gate below 2^-126 counts as 2^-126) and, inside a chunk of 64
// tokens, L_t = sum of l over the chunk's tokens up to t (per feature).  The weight with
// which token i reaches token j >= i is 2^(L_j - L_i) per feature, so
//   o_j = (q_j (.) 2^(L_j)) P_c + sum_{i<=j} [sum_f q_j[f] 2^(L_j[f]) k_i[f] 2^(-L_i[f])] v_i
//   P_{c+1} = diag(2^(L_last)) P_c + sum_i (k_i (.) 2^(L_last - L_i)) v_i^T,
// the scan page's three kernels with the decayed monoid made per feature
// ("Log-Depth Chunked Linear-Attention Scan", Formulas: (a1, S1) + (a2, S2) = (a1 a2,
// diag(a2) S1 + S2)).  The scores and both state products are dense: tcgen05 MMAs on
// factored operands, each split into bf16 hi + lo (about 16 bits, like the retention
// kernels), so the only rounding beyond float32 accumulation is ~2^-16 per product.
//
// Renormalised window.  The kernels carry a per-feature window offset W (<= 0): the TMEM
// state holds P~ with P = diag(2^W) P~, and a chunk whose exponents keep every factor within
// 2^60 uses  q~_j = q_j (.) 2^(W + L_j)  (<= 1) and  k~_i = k_i (.) 2^(-(W + L_i))  (<= 2^60)
// for the scores, the prefix product and the state update alike, with no pass over the
// state.  A chunk that would leave that range first rebases (P~ <- diag(2^W) P~, W <- 0, one
// TMEM pass); if even its own exponents leave the range (gates averaging below ~0.5 over the
// chunk), its state update uses k_i (.) 2^(L_last - L_i) (<= 1) on the state scaled by
// 2^(L_last) in that pass, and its intra-chunk scores are left to an exact CUDA-core pass
// (gla_k3 in fix-up mode), flagged per chunk.
//
//   gla_k1_seg  per (b*H + h, segment): the segment's fold S_s = sum_i (k_i (.) 2^(A_end -
//               A_i)) v_i^T (A the cumulative log over the segment) and its decay
//               a_s = 2^(A_end), both into one record (S_s^T, then a_s).
//   gla_scan    exclusive scan of the segment records with per-feature decays (a blocked
//               Hillis-Steele scan, like the prefill's K2), from S_init; writes S_final.
//   gla_k3_seg  per segment: walks its chunks from the segment's prefix, carrying P~ in
//               TMEM: scores, prefix product, state update, output.

#include <cuda_bf16.h>

#include "../../include/linattn.h"
#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"
#include "tile_util.cuh"

namespace la {
namespace {

constexpr int kC = 64;
constexpr float kWin = 60.f;  // factors stay within 2^kWin
constexpr int kXf = 256;      // transform threads (8 warps)

// ---------------------------------------------------------------------------------------
// Shared per-chunk gate work of both kernels (the 256 transform threads).

// Cumulative log2 gates down each feature column of the chunk's gate tile (float32,
// row-major [64][DK], in place).  Rows at or past the chunk's length count as gate 1.
// Thread tw owns feature tw % DK and a quarter or half of the rows; parts are joined
// through sTot.  On return (after a barrier among the transform threads) sLc[f] holds the
// chunk's total and the tile holds L.
template <int DK>
__device__ __forceinline__ void chunk_cumlog(float* sA, float* sTot, float* sLc, int tw, int L,
                                             bool rev_unused) {
  (void)rev_unused;
  constexpr int NP = kXf / DK;  // parts per feature
  constexpr int RP = kC / NP;   // rows per part
  const int f = tw % DK, part = tw / DK;
  // All of the part's gates first, then their logarithms (independent, so they overlap;
  // taken unconditionally and selected: a padding row reads as zero), then the running
  // sum in registers; the tile is written once, with the earlier parts' total added.
  float l[RP];
#pragma unroll
  for (int j = 0; j < RP; ++j) l[j] = sA[(part * RP + j) * DK + f];
#pragma unroll
  for (int j = 0; j < RP; ++j) {
    // Gates below 2^-126 read as zero and clamp to -126, as they would unflushed.
    const float lg = log2_approx(l[j]);
    l[j] = part * RP + j < L ? fmaxf(lg, -126.f) : 0.f;
  }
  float acc = 0.f;
#pragma unroll
  for (int j = 0; j < RP; ++j) {
    acc += l[j];
    l[j] = acc;
  }
  sTot[part * DK + f] = acc;
  named_barrier(1, kXf);
  float off = 0.f;
#pragma unroll
  for (int p = 0; p < NP; ++p)
    if (p < part) off += sTot[p * DK + f];
#pragma unroll
  for (int j = 0; j < RP; ++j) sA[(part * RP + j) * DK + f] = l[j] + off;
  if (part == NP - 1) sLc[f] = acc + off;
  named_barrier(1, kXf);
}

// Chunk modes.
enum : int { kModeWindow = 0, kModeRebase = 1, kModeSteep = 2 };

// Decides the chunk's mode from the window offsets sW and the chunk totals sLc, and sets the
// per-feature exponent bases: the q operand takes 2^(bq + L), the k operand 2^(bk - L).
// sScale receives the per-feature factor a rebase applies to the carried state (2^W), and
// sScale2 the one it applies after the prefix product (1, or 2^(L_last) in a steep chunk);
// sW is advanced to the window offset after the chunk.  Returns the mode (same in every
// thread).  Uses sRed[16].
template <int DK>
__device__ __forceinline__ int chunk_mode(float* sW, const float* sLc, float* sBq, float* sBk,
                                          float* sScale, float* sScale2, float* sRed, int tw,
                                          int warp, int lane) {
  float m1 = 0.f, m2 = 0.f;  // min over features of W + Lc, and of Lc
  if (tw < DK) {
    m1 = sW[tw] + sLc[tw];
    m2 = sLc[tw];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    m1 = fminf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
    m2 = fminf(m2, __shfl_xor_sync(0xffffffffu, m2, o));
  }
  if (lane == 0) {
    sRed[warp] = m1;
    sRed[8 + warp] = m2;
  }
  named_barrier(1, kXf);
  float w1 = 0.f, w2 = 0.f;
#pragma unroll
  for (int w = 0; w < DK / 32; ++w) {
    w1 = fminf(w1, sRed[w]);
    w2 = fminf(w2, sRed[8 + w]);
  }
  const int mode = w1 >= -kWin ? kModeWindow : (w2 >= -kWin ? kModeRebase : kModeSteep);
  if (tw < DK) {
    const float W = sW[tw], Lc = sLc[tw];
    if (mode == kModeWindow) {
      sBq[tw] = W;
      sBk[tw] = -W;
      sScale[tw] = 1.f;
      sScale2[tw] = 1.f;
      sW[tw] = W + Lc;
    } else if (mode == kModeRebase) {
      sBq[tw] = 0.f;
      sBk[tw] = 0.f;
      sScale[tw] = exp2f(W);
      sScale2[tw] = 1.f;
      sW[tw] = Lc;
    } else {
      sBq[tw] = 0.f;
      sBk[tw] = Lc;
      sScale[tw] = exp2f(W);
      sScale2[tw] = exp2f(Lc);
      sW[tw] = 0.f;
    }
  }
  named_barrier(1, kXf);
  return mode;
}

// The factored operand of one 128B-swizzled bf16 tile (q or k): x (.) 2^(base + sign * L) for
// rows < L (zero past them), split into bf16 hi, written in place, and lo, returned in `lo`
// (kRows x uint4) for factor_tile_store_lo once every thread has read the gate tile.
// Thread (cc, rg): 8 consecutive features of rows rg, rg + RG, ...
template <int DK>
struct FactorShape {
  static constexpr int NCC = DK / 8;
  static constexpr int RG = kXf / NCC;
  static constexpr int kRows = kC / RG;
};

template <int DK, int SIGN>
__device__ __forceinline__ void factor_tile(uint8_t* tile, const float* sA, const float* sBase,
                                            int tw, int L,
                                            uint4 (&lo)[FactorShape<DK>::kRows]) {
  constexpr int NCC = FactorShape<DK>::NCC;
  constexpr int RG = FactorShape<DK>::RG;
  constexpr int kRows = FactorShape<DK>::kRows;
  const int cc = tw % NCC, rg = tw / NCC;
  const uint32_t boff = (cc / 8) * (kC * 128);
  float base[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) base[e] = sBase[cc * 8 + e];
  uint4 raw[kRows];
#pragma unroll
  for (int k = 0; k < kRows; ++k)
    raw[k] = *reinterpret_cast<const uint4*>(tile + boff + sw128_offset(rg + k * RG, cc % 8));
#pragma unroll
  for (int k = 0; k < kRows; ++k) {
    const int r = rg + k * RG;
    const float4 l0 = *reinterpret_cast<const float4*>(sA + r * DK + cc * 8);
    const float4 l1 = *reinterpret_cast<const float4*>(sA + r * DK + cc * 8 + 4);
    const float lv[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
    float x[8];
    unpack8(raw[k], x);
#pragma unroll
    for (int e = 0; e < 8; ++e)
      x[e] = r < L ? x[e] * exp2_approx(base[e] + static_cast<float>(SIGN) * lv[e]) : 0.f;
    uint4 hi;
    split8(x, hi, lo[k]);
    *reinterpret_cast<uint4*>(tile + boff + sw128_offset(r, cc % 8)) = hi;
  }
}

// The lo halves of factor_tile, into a tile of the same layout.
template <int DK>
__device__ __forceinline__ void factor_tile_store_lo(uint8_t* lo_tile, int tw,
                                                     const uint4 (&lo)[FactorShape<DK>::kRows]) {
  constexpr int NCC = FactorShape<DK>::NCC;
  constexpr int RG = FactorShape<DK>::RG;
  constexpr int kRows = FactorShape<DK>::kRows;
  const int cc = tw % NCC, rg = tw / NCC;
  const uint32_t boff = (cc / 8) * (kC * 128);
#pragma unroll
  for (int k = 0; k < kRows; ++k)
    *reinterpret_cast<uint4*>(lo_tile + boff + sw128_offset(rg + k * RG, cc % 8)) = lo[k];
}

// ---------------------------------------------------------------------------------------
// gla_k1_seg: one CTA per (b*H + h, segment), 320 threads.
//   warps 0-7  transform: cumulative log gates, the chunk's mode, the key operand
//              (hi in place, lo over the gate tile once every thread has read it); a rebase
//              scales the accumulator in TMEM (after the previous chunk's MMAs); at the end
//              the epilogue applies 2^W and stores the record.
//   warp 8     producer: TMA loads of K, V, alpha into a three-stage ring.
//   warp 9     MMA issuer: V^T K' into one TMEM accumulator (M = dv = 128, N = DK).

constexpr int kThreadsK1 = 320;
constexpr int kStagesK1 = 3;

template <int DK>
struct GK1Smem {
  static constexpr uint32_t kK = DK * kC * 2;
  static constexpr uint32_t kV = 128 * kC * 2;
  static constexpr uint32_t kG = kC * DK * 4;
  // K (hi in place), V, the gate tile (cumulative logs, then the lo half of K)
  static constexpr uint32_t kStage = kK + kV + kG;
  static constexpr uint32_t kIn = kStagesK1 * kStage;
  static constexpr uint32_t kS = DK * 128 * 4;  // staging of S^T, aliases the inputs
  static constexpr uint32_t kRegion = kIn > kS ? kIn : kS;
  static constexpr uint32_t kSmall = (6 * DK + kXf + 16) * 4;
  static constexpr uint32_t kBars = 3 * kStagesK1 + 2;
  static constexpr uint32_t kTotal = kRegion + kSmall + (kBars + 1) * 8 + 1024;
};

template <int DK>
__global__ void __launch_bounds__(kThreadsK1, 1)
gla_k1_seg(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
           const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_srec,
           GlaSegParams sp) {
  constexpr int DV = 128;
  using L_ = GK1Smem<DK>;
  static_assert(L_::kTotal <= 232448, "shared memory budget");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1024(smem_raw);
  uint8_t* sS = base;
  float* sW = reinterpret_cast<float*>(base + L_::kRegion);  // [DK] window offset
  float* sLc = sW + DK;       // [DK] chunk total
  float* sBq = sLc + DK;      // [DK] (unused by K1)
  float* sBk = sBq + DK;      // [DK]
  float* sScale = sBk + DK;   // [DK]
  float* sScale2 = sScale + DK;
  float* sTot = sScale2 + DK;  // [kXf]: the cumulative-log parts
  float* sRed = sTot + kXf;     // [16]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sRed + 16);
  uint64_t* full = bars;                   // [kStagesK1]
  uint64_t* ops = bars + kStagesK1;        // [kStagesK1], 256 arrivals
  uint64_t* empty = bars + 2 * kStagesK1;  // [kStagesK1], MMA commits
  uint64_t* accdone = bars + 3 * kStagesK1;     // each chunk's MMAs
  uint64_t* done = bars + 3 * kStagesK1 + 1;    // the segment's last MMA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + L_::kBars);

  if (error_pending(sp.err)) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int seg = static_cast<int>(blockIdx.x % sp.NS);
  const int bh = static_cast<int>(blockIdx.x / sp.NS);
  const int cb = seg * sp.Lseg;
  const int ce = min(sp.NC, cb + sp.Lseg);
  const int n = ce - cb;

  if (tid == 0) {
    for (int b = 0; b < kStagesK1; ++b) {
      mbar_init(&full[b], 1);
      mbar_init(&ops[b], kXf);
      mbar_init(&empty[b], 1);
    }
    mbar_init(accdone, 1);
    mbar_init(done, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_srec);
  }
  if (tid < DK) sW[tid] = 0.f;
  if (warp == 0) {
    tmem_alloc(tmem_slot, DK);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool failed = false;
  auto wait = [&](uint64_t* bar, uint32_t parity, int code) -> bool {
    if (failed) return false;
    if (mbar_wait(bar, parity)) return true;
    report_error(sp.err, code);
    failed = true;
    return false;
  };

  if (warp < 8) {
    // ------------------------------------------------------------------ transform
    const int tw = tid;
    float seg_log = 0.f;  // thread tw < DK: the segment's total log2 decay of feature tw
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    for (int i = 0; i < n; ++i) {
      const int st = i % kStagesK1;
      const int L = chunk_len(sp, cb + i);
      uint8_t* sK = base + st * L_::kStage;
      uint8_t* sKl = sK + L_::kK + L_::kV;  // the gate tile, reused for the lo half of K
      float* sA = reinterpret_cast<float*>(sKl);
      wait(&full[st], (i / kStagesK1) & 1, kErrTmaTimeout);
      chunk_cumlog<DK>(sA, sTot, sLc, tw, L, false);
      const int mode = chunk_mode<DK>(sW, sLc, sBq, sBk, sScale, sScale2, sRed, tw, warp, lane);
      if (tw < DK) seg_log += sLc[tw];
      // The previous chunk's MMAs (waited every chunk, so that the barrier is never more
      // than one phase ahead; they were issued before this chunk's gates were processed).
      if (i > 0) wait(accdone, (i - 1) & 1, kErrMmaTimeout);
      if (mode != kModeWindow && i > 0) {
        // Rebase: the accumulator (lane = value feature, column = key feature) times
        // 2^W (and 2^(L_last) in a steep chunk).
        tc_fence_after();
        const uint32_t c0 = static_cast<uint32_t>(warp >> 2) * (DK / 2);
#pragma unroll
        for (int q4 = 0; q4 < DK / 64; ++q4) {
          const uint32_t col = c0 + q4 * 32;
          float r[32];
          tmem_ld32(tmem + lane_base + col, r);
          tmem_ld_wait();
          uint32_t u[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(r[e] * sScale[col + e] * sScale2[col + e]);
          tmem_st32(tmem + lane_base + col, u);
        }
        tmem_st_wait();
        tc_fence_before();
      }
      uint4 klo[FactorShape<DK>::kRows];
      factor_tile<DK, -1>(sK, sA, sBk, tw, L, klo);
      named_barrier(1, kXf);  // every thread has read the gate tile
      factor_tile_store_lo<DK>(sKl, tw, klo);
      fence_async_smem();
      mbar_arrive(&ops[st]);
    }
    // The record: S~^T scaled per key feature by 2^W (the window offset after the last
    // chunk), then the segment's decay vector.
    wait(done, 0, kErrMmaTimeout);
    tc_fence_after();
    named_barrier(1, kXf);  // every transform thread is past its last use of the stages
    const int quarter = warp & 3, half = warp >> 2;
    const int row = quarter * 32 + lane;
#pragma unroll
    for (int q4 = half * (DK / 64); q4 < (half + 1) * (DK / 64); ++q4) {
      float r[32];
      tmem_ld32(tmem + lane_base + q4 * 32, r);
      tmem_ld_wait();
      uint8_t* box = sS + q4 * (DV * 128);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int c = q4 * 32 + 4 * q;
        *reinterpret_cast<float4*>(box + sw128_offset(row, q)) =
            make_float4(r[4 * q] * exp2f(sW[c]), r[4 * q + 1] * exp2f(sW[c + 1]),
                        r[4 * q + 2] * exp2f(sW[c + 2]), r[4 * q + 3] * exp2f(sW[c + 3]));
      }
    }
    float* srec = sp.srec + (static_cast<long long>(bh) * sp.NS + seg) * sp.R;
    if (tw < DK) srec[DK * DV + tw] = exp2f(seg_log);
    fence_async_smem();
    tc_fence_before();
    named_barrier(1, kXf);
    if (tid == 0) {
#pragma unroll
      for (int q4 = 0; q4 < DK / 32; ++q4)
        tma_store_3d(&tm_srec, sS + q4 * (DV * 128), q4 * 32, 0, bh * sp.NS + seg);
      bulk_commit();
      bulk_wait_read_all();
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      int loads = 0;
      for (int i = 0; i < n; ++i) {
        const int st = i % kStagesK1;
        if (i >= kStagesK1 && !wait(&empty[st], ((i / kStagesK1) - 1) & 1, kErrMmaTimeout)) break;
        uint8_t* sK = base + st * L_::kStage;
        uint8_t* sV = sK + L_::kK;
        uint8_t* sA = sV + L_::kV;
        const int t0 = (cb + i) * kC;
        mbar_arrive_expect_tx(&full[st], L_::kK + L_::kV + L_::kG);
#pragma unroll
        for (int b = 0; b < DK / 64; ++b) tma_load_3d(sK + b * kC * 128, &tm_k, &full[st], b * 64, t0, bh);
#pragma unroll
        for (int b = 0; b < DV / 64; ++b) tma_load_3d(sV + b * kC * 128, &tm_v, &full[st], b * 64, t0, bh);
        tma_load_3d(sA, &tm_a, &full[st], 0, t0, bh);
        ++loads;
      }
      for (int j = max(0, loads - kStagesK1); j < loads; ++j)
        mbar_wait(&full[j % kStagesK1], (j / kStagesK1) & 1);
    }
  } else if (lane == 0) {
    // ------------------------------------------------------------------ MMA issuer
    const uint32_t a0 = smem_u32(base);
    const uint64_t dK = smem_desc_sw128(a0, kC * 128, 1024);                  // MN-major
    const uint64_t dV = smem_desc_sw128(a0 + L_::kK, kC * 128, 1024);
    const uint64_t dKl = smem_desc_sw128(a0 + L_::kK + L_::kV, kC * 128, 1024);
    constexpr uint32_t kStageD = L_::kStage >> 4;
    constexpr uint32_t idesc = instr_desc(kFmtBF16, kFmtBF16, kMNMajor, kMNMajor, DV, DK);
    for (int i = 0; i < n && !failed; ++i) {
      const int st = i % kStagesK1;
      if (!wait(&ops[st], (i / kStagesK1) & 1, kErrMmaTimeout)) break;
      tc_fence_after();
      const uint64_t k = dK + st * kStageD, v = dV + st * kStageD, kl = dKl + st * kStageD;
#pragma unroll
      for (int kk = 0; kk < kC / 16; ++kk) {
        mma_bf16_ss(tmem, desc_at(v, kk * 2048), desc_at(k, kk * 2048), idesc,
                    (i > 0 || kk > 0) ? 1u : 0u);
        mma_bf16_ss(tmem, desc_at(v, kk * 2048), desc_at(kl, kk * 2048), idesc, 1u);
      }
      mma_commit(&empty[st]);
      mma_commit(accdone);
    }
    mma_commit(done);
    if (failed) mbar_wait(done, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, DK);
}


// ---------------------------------------------------------------------------------------
// gla_k3_seg: one CTA per (b*H + h, segment), 576 threads, the roles of the prefill's
// segmented combine:
//   warps 0-7   transform: cumulative log gates, the chunk's mode, the factored q~ and k~
//               (hi in place over the staged tiles, lo over the stage's gate tile once every
//               thread has read it); then the prefix operand:
//               P~ from TMEM -> (rebase: times 2^W) -> bf16 hi / lo into TMEM, and on a
//               rebase the state written back for the chunk's update.
//   warps 8-15  epilogue: causal mask of the scores into A (hi / lo), then o = X + N,
//               written straight to global memory.
//   warp 16     producer: TMA loads of Q, K, V and the gates into a two-stage ring.
//   warp 17     MMA issuer: scores q~ k~^T, X = P~^T q~^T, P~ += V^T k~, N = V^T A^T.
// TMEM columns: scores [0, 64), X [64, 128) and [448, 512), N [128, 192), P~ [192, 192 + DK),
// its bf16 hi / lo after it.

constexpr int kThreadsK3 = 576;
constexpr int kEp = 256;  // epilogue threads, warps 8-15

template <int DK>
struct GK3Smem {
  static constexpr int DV = 128;
  static constexpr uint32_t kQ = DK * kC * 2;
  static constexpr uint32_t kK = DK * kC * 2;
  static constexpr uint32_t kV = DV * kC * 2;
  static constexpr uint32_t kG = kC * DK * 4;
  // Q, K (hi in place), V, the gate tile (cumulative logs, then the lo halves of q~ and k~:
  // kG = kQ + kK)
  static constexpr uint32_t kStage = kQ + kK + kV + kG;
  static_assert(kG == kQ + kK, "the lo tiles fill the gate tile");
  static constexpr uint32_t kA = kC * kC * 2;
  static constexpr uint32_t kSmallFloats = 8 * DK + kXf + 16 + 4;
  static constexpr uint32_t kBars = 15;
  static constexpr uint32_t kTotal = 2 * kStage + 2 * kA + kSmallFloats * 4 + (kBars + 1) * 8 + 1024;
};

template <int DK, bool OUTF32>
__global__ void __launch_bounds__(kThreadsK3, 1)
gla_k3_seg(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
           const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_a,
           GlaSegParams sp) {
  constexpr int DV = 128;
  using L_ = GK3Smem<DK>;
  constexpr uint32_t kTmemCols = 512;
  constexpr uint32_t kColS = 0, kColN = 128, kColP = 192;
  constexpr uint32_t kColPH = kColP + DK, kColPL = kColPH + DK / 2;
  constexpr uint32_t kColX[2] = {64, 448};
  static_assert(kColPL + DK / 2 <= 448, "TMEM budget");
  static_assert(L_::kTotal <= 232448, "shared memory budget");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1024(smem_raw);
  uint8_t* sAh = base + 2 * L_::kStage;
  uint8_t* sAl = sAh + L_::kA;
  float* sW = reinterpret_cast<float*>(sAl + L_::kA);
  float* sLc = sW + DK;
  float* sBq = sLc + DK;
  float* sBk = sBq + DK;
  float* sScale = sBk + DK;         // [2][DK], by stage: read by the epilogue's prefix split
  float* sScale2 = sScale + 2 * DK;  // [2][DK]
  float* sTot = sScale2 + 2 * DK;    // [kXf]: the cumulative-log parts
  float* sRed = sTot + kXf;     // [16]
  int* sMode = reinterpret_cast<int*>(sRed + 16);  // [2], per stage
  uint64_t* bars = reinterpret_cast<uint64_t*>(sMode + 4);
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
  uint64_t* empty = bars + 13;     // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + L_::kBars);

  if (error_pending(sp.err)) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int seg = static_cast<int>(blockIdx.x % sp.NS);
  const int bh = static_cast<int>(blockIdx.x / sp.NS);
  const int cb = seg * sp.Lseg;
  const int ce = min(sp.NC, cb + sp.Lseg);
  const int n = ce - cb;
  const float* srec = sp.srec + (static_cast<long long>(bh) * sp.NS + seg) * sp.R;

  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&full[b], 1);
      mbar_init(&ops[b], kXf);
      mbar_init(&xfree[b], kEp);
      mbar_init(&empty[b], 1);
    }
    mbar_init(pready, kXf);
    mbar_init(sfree, kEp);
    mbar_init(aready, kEp);
    mbar_init(sdone, 1);
    mbar_init(statedone, 1);
    mbar_init(ndone, 1);
    mbar_init(drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_a);
  }
  if (tid < DK) sW[tid] = 0.f;
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  bool failed = false;
  auto wait = [&](uint64_t* bar, uint32_t parity, int code) -> bool {
    if (failed) return false;
    if (mbar_wait(bar, parity)) return true;
    report_error(sp.err, code);
    failed = true;
    return false;
  };

  // The prefix operand of the X MMA, prepared by the epilogue warps between their score and
  // output phases (the transform warps, whose gate pass sets the pace, keep only the chunk's
  // operands): warp w covers TMEM lanes 32 (w % 4) .. + 31 and key features
  // kHalf (w / 4 % 2) .. + kHalf - 1.
  constexpr int kHalf = DK / 2;
  const uint32_t pcol = static_cast<uint32_t>((warp >> 2) & 1) * kHalf;
  auto load_prefix = [&]() {  // the segment's exclusive prefix: row (lane) of P^T
    const int row = (warp & 3) * 32 + lane;
    const float4* src = reinterpret_cast<const float4*>(srec + static_cast<long long>(row) * DK + pcol);
#pragma unroll
    for (int q4 = 0; q4 < kHalf / 32; ++q4) {
      uint32_t u[32];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float4 f = src[q4 * 8 + e];
        u[4 * e] = __float_as_uint(f.x);
        u[4 * e + 1] = __float_as_uint(f.y);
        u[4 * e + 2] = __float_as_uint(f.z);
        u[4 * e + 3] = __float_as_uint(f.w);
      }
      tmem_st32(tmem + lane_base + kColP + pcol + q4 * 32, u);
    }
    tmem_st_wait();
  };
  // Prefix operand for chunk i (the state after chunk i - 1, final once statedone(i - 1)
  // completed; the chunk's mode and scales are set once ops of its stage completed):
  // P = P~ 2^W on a rebase (and, for the chunk's update, times 2^(L_last) in a steep chunk);
  // P~ itself inside a window.  16 columns at a time, inside the epilogue's register budget.
  auto split_prefix = [&](int i) {
    const int st = i & 1;
    const bool last = i == n - 1;
    const bool rebase = sMode[st] != kModeWindow;
    const float* scale = sScale + st * DK;
    const float* scale2 = sScale2 + st * DK;
#pragma unroll 2
    for (int q = 0; q < kHalf / 16; ++q) {
      const uint32_t col = pcol + q * 16;
      float rr[16];
      tmem_ld16(tmem + lane_base + kColP + col, rr);
      tmem_ld_wait();
      if (rebase) {
#pragma unroll
        for (int e = 0; e < 16; ++e) rr[e] *= scale[col + e];
      }
      uint32_t hi[8], lo[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(rr[2 * e], rr[2 * e + 1]);
        const float2 hf = __bfloat1622float2(h);
        hi[e] = *reinterpret_cast<const uint32_t*>(&h);
        lo[e] = pack2(rr[2 * e] - hf.x, rr[2 * e + 1] - hf.y);
      }
      tmem_st8(tmem + lane_base + kColPH + col / 2, hi);
      tmem_st8(tmem + lane_base + kColPL + col / 2, lo);
      if (rebase && !last) {
        uint32_t u[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) u[e] = __float_as_uint(rr[e] * scale2[col + e]);
        tmem_st16(tmem + lane_base + kColP + col, u);
      }
    }
    tmem_st_wait();
    tc_fence_before();
    mbar_arrive(pready);
  };

  if (warp < 8) {
    // ------------------------------------------------------------------ transform
    const int tw = tid;
    for (int i = 0; i < n; ++i) {
      const int s = i & 1;
      const int L = chunk_len(sp, cb + i);
      uint8_t* sQ = base + s * L_::kStage;
      uint8_t* sK = sQ + L_::kQ;
      uint8_t* sQl = sK + L_::kK + L_::kV;  // the gate tile, reused for the lo halves
      uint8_t* sKl = sQl + L_::kQ;
      float* sA = reinterpret_cast<float*>(sQl);
      wait(&full[s], (i >> 1) & 1, kErrTmaTimeout);
      chunk_cumlog<DK>(sA, sTot, sLc, tw, L, false);
      const int mode = chunk_mode<DK>(sW, sLc, sBq, sBk, sScale + s * DK, sScale2 + s * DK, sRed,
                                      tw, warp, lane);
      if (tw == 0) sMode[s] = mode;
      {
        uint4 qlo[FactorShape<DK>::kRows], klo[FactorShape<DK>::kRows];
        factor_tile<DK, 1>(sQ, sA, sBq, tw, L, qlo);
        factor_tile<DK, -1>(sK, sA, sBk, tw, L, klo);
        named_barrier(1, kXf);  // every thread has read the gate tile
        factor_tile_store_lo<DK>(sQl, tw, qlo);
        factor_tile_store_lo<DK>(sKl, tw, klo);
      }
      fence_async_smem();
      mbar_arrive(&ops[s]);
    }
  } else if (warp < 16) {
    // ------------------------------------------------------------------ epilogue
    const int tw = tid - kXf;
    const int quarter = warp & 3, half = (warp - 8) >> 2;
    const int j = quarter * 32 + lane;  // value feature of this thread's output column
    load_prefix();
    wait(&ops[0], 0, kErrMmaTimeout);  // chunk 0's mode and scales
    split_prefix(0);
    for (int i = 0; i < n; ++i) {
      const int s = i & 1;
      const long long t0 = static_cast<long long>(cb + i) * kC;
      const int L = chunk_len(sp, cb + i);
      const bool has_prefix = !(seg == 0 && i == 0) || sp.has_init;
      wait(sdone, i & 1, kErrMmaTimeout);
      wait(&ops[s], (i >> 1) & 1, kErrMmaTimeout);
      tc_fence_after();
      const int mode = sMode[s];
      {
        const int row = quarter * 16 + (lane & 15);
        const int kb = 32 * half + 16 * (lane >> 4);
        uint4 hi[2], lo[2];
        if (mode != kModeSteep) {
          float sc[16];
          tmem_ld16x2_x16(tmem + lane_base + kColS + 32 * half, sc);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            float a[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) a[e] = row >= kb + q * 8 + e ? sc[q * 8 + e] : 0.f;
            split8(a, hi[q], lo[q]);
          }
        } else {
          hi[0] = hi[1] = lo[0] = lo[1] = make_uint4(0u, 0u, 0u, 0u);
        }
        tc_fence_before();
        mbar_arrive(sfree);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          *reinterpret_cast<uint4*>(sAh + sw128_offset(row, kb / 8 + q)) = hi[q];
          *reinterpret_cast<uint4*>(sAl + sw128_offset(row, kb / 8 + q)) = lo[q];
        }
      }
      fence_async_smem();
      mbar_arrive(aready);
      if (tw == 0) sp.steep[static_cast<long long>(bh) * sp.NC + cb + i] = mode == kModeSteep ? 1 : 0;

      // The next chunk's prefix operand, while N(i) runs.
      if (i + 1 < n) {
        wait(statedone, i & 1, kErrMmaTimeout);
        wait(&ops[(i + 1) & 1], ((i + 1) >> 1) & 1, kErrMmaTimeout);
        tc_fence_after();
        split_prefix(i + 1);
      }

      wait(ndone, i & 1, kErrMmaTimeout);
      tc_fence_after();
      float xo[32], no[32];
      if (has_prefix) tmem_ld32(tmem + lane_base + kColX[s] + 32 * half, xo);
      tmem_ld32(tmem + lane_base + kColN + 32 * half, no);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&xfree[s]);
      if (has_prefix) {
#pragma unroll
        for (int e = 0; e < 32; ++e) no[e] += xo[e];
      }
      const long long row0 = static_cast<long long>(bh) * sp.T + t0 + 32 * half;
      const int t_hi = min(32, L - 32 * half);
#pragma unroll
      for (int tt = 0; tt < 32; ++tt) {
        if (tt < t_hi) {
          const long long idx = (row0 + tt) * DV + j;
          if constexpr (OUTF32)
            __stcs(static_cast<float*>(sp.out) + idx, no[tt]);
          else
            static_cast<__nv_bfloat16*>(sp.out)[idx] = __float2bfloat16_rn(no[tt]);
        }
      }
    }
  } else if (warp == 16) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      int loads = 0;
      for (int i = 0; i < n; ++i) {
        if (i >= 2 && !wait(&empty[i & 1], ((i - 2) >> 1) & 1, kErrMmaTimeout)) break;
        uint8_t* sQ = base + (i & 1) * L_::kStage;
        uint8_t* sK = sQ + L_::kQ;
        uint8_t* sV = sK + L_::kK;
        uint8_t* sA = sV + L_::kV;
        const int t0 = (cb + i) * kC;
        mbar_arrive_expect_tx(&full[i & 1], L_::kStage);
#pragma unroll
        for (int b = 0; b < DK / 64; ++b) {
          tma_load_3d(sQ + b * kC * 128, &tm_q, &full[i & 1], b * 64, t0, bh);
          tma_load_3d(sK + b * kC * 128, &tm_k, &full[i & 1], b * 64, t0, bh);
        }
#pragma unroll
        for (int b = 0; b < DV / 64; ++b)
          tma_load_3d(sV + b * kC * 128, &tm_v, &full[i & 1], b * 64, t0, bh);
        tma_load_3d(sA, &tm_a, &full[i & 1], 0, t0, bh);
        ++loads;
      }
      for (int jl = max(0, loads - 2); jl < loads; ++jl) mbar_wait(&full[jl & 1], (jl >> 1) & 1);
    }
  } else if (lane == 0) {
    // ------------------------------------------------------------------ MMA issuer
    const uint32_t a0 = smem_u32(base);
    const uint64_t dQk = smem_desc_sw128(a0, 16, 1024);                          // q~, K-major
    const uint64_t dKk = smem_desc_sw128(a0 + L_::kQ, 16, 1024);                 // k~, K-major
    const uint64_t dKm = smem_desc_sw128(a0 + L_::kQ, kC * 128, 1024);           // k~, MN-major
    const uint64_t dVm = smem_desc_sw128(a0 + L_::kQ + L_::kK, kC * 128, 1024);  // V, MN-major
    const uint32_t lo0 = a0 + L_::kQ + L_::kK + L_::kV;  // stage 0's gate tile: q~ lo, k~ lo
    const uint64_t dQlk = smem_desc_sw128(lo0, 16, 1024);
    const uint64_t dKlk = smem_desc_sw128(lo0 + L_::kQ, 16, 1024);
    const uint64_t dKlm = smem_desc_sw128(lo0 + L_::kQ, kC * 128, 1024);
    const uint64_t dAh = smem_desc_sw128(smem_u32(sAh), 16, 1024);
    const uint64_t dAl = smem_desc_sw128(smem_u32(sAl), 16, 1024);
    constexpr uint32_t kStageD = L_::kStage >> 4, kLoD = kStageD;

    auto issue_scores = [&](int i) -> bool {
      const int s = i & 1;
      const uint64_t q = dQk + s * kStageD, k = dKk + s * kStageD;
      const uint64_t ql = dQlk + s * kLoD, kl = dKlk + s * kLoD;
      if (!wait(&ops[s], (i >> 1) & 1, kErrMmaTimeout)) return false;
      if (i > 0 && !wait(sfree, (i - 1) & 1, kErrMmaTimeout)) return false;
      tc_fence_after();
      if (sMode[s] != kModeSteep) {
        constexpr uint32_t ids = instr_desc(kFmtBF16, kFmtBF16, kKMajor, kKMajor, 64, 64);
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
          const uint32_t off = (kk / 4) * (kC * 128) + (kk % 4) * 32;
          mma_bf16_ss(tmem + kColS, desc_at(q, off), desc_at(k, off), ids, kk > 0 ? 1u : 0u);
          mma_bf16_ss(tmem + kColS, desc_at(q, off), desc_at(kl, off), ids, 1u);
          mma_bf16_ss(tmem + kColS, desc_at(ql, off), desc_at(k, off), ids, 1u);
        }
      }
      mma_commit(sdone);
      return true;
    };
    issue_scores(0);
    for (int i = 0; i < n && !failed; ++i) {
      const int s = i & 1;
      const bool last = i == n - 1;
      const bool has_prefix = !(seg == 0 && i == 0) || sp.has_init;
      const uint64_t q = dQk + s * kStageD, ql = dQlk + s * kLoD;
      const uint64_t v = dVm + s * kStageD;

      // X(i) = P^T q~^T and the state update with chunk i.
      if (!wait(pready, i & 1, kErrMmaTimeout)) break;
      if (i > 1 && !wait(&xfree[s], ((i - 2) >> 1) & 1, kErrMmaTimeout)) break;
      tc_fence_after();
      if (has_prefix) {
        constexpr uint32_t idx = instr_desc(kFmtBF16, kFmtBF16, kKMajor, kKMajor, 128, 64);
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
          const uint32_t off = (kk / 4) * (kC * 128) + (kk % 4) * 32;
          mma_bf16_ts(tmem + kColX[s], tmem + kColPH + kk * 8, desc_at(q, off), idx,
                      kk > 0 ? 1u : 0u);
          mma_bf16_ts(tmem + kColX[s], tmem + kColPL + kk * 8, desc_at(q, off), idx, 1u);
          mma_bf16_ts(tmem + kColX[s], tmem + kColPH + kk * 8, desc_at(ql, off), idx, 1u);
        }
      }
      if (!last) {
        constexpr uint32_t idp = instr_desc(kFmtBF16, kFmtBF16, kMNMajor, kMNMajor, 128, DK);
        const uint64_t bh_ = dKm + s * kStageD;
        const uint64_t bl_ = dKlm + s * kLoD;
#pragma unroll
        for (int kk = 0; kk < kC / 16; ++kk) {
          mma_bf16_ss(tmem + kColP, desc_at(v, kk * 2048), desc_at(bh_, kk * 2048), idp, 1u);
          mma_bf16_ss(tmem + kColP, desc_at(v, kk * 2048), desc_at(bl_, kk * 2048), idp, 1u);
        }
      }
      mma_commit(statedone);

      // N(i) = V^T A^T.
      if (!wait(aready, i & 1, kErrMmaTimeout)) break;
      tc_fence_after();
      constexpr uint32_t idn = instr_desc(kFmtBF16, kFmtBF16, kMNMajor, kKMajor, 128, 64);
#pragma unroll
      for (int kk = 0; kk < kC / 16; ++kk) {
        mma_bf16_ss(tmem + kColN, desc_at(v, kk * 2048), desc_at(dAh, kk * 32), idn,
                    kk > 0 ? 1u : 0u);
        mma_bf16_ss(tmem + kColN, desc_at(v, kk * 2048), desc_at(dAl, kk * 32), idn, 1u);
      }
      mma_commit(ndone);
      mma_commit(&empty[s]);

      if (i + 1 < n && !issue_scores(i + 1)) break;
    }
    if (failed) {
      mma_commit(drain);
      mbar_wait(drain, 0);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------------------
// gla_scan: exclusive scan of the segment records over segments, in place, with the
// per-feature decays a_s (the records' tails).  Column col of S^T (j = col / dk, key feature
// i = col % dk) is scaled by a_s[i].  The blocked arrangement of the prefill's K2: one CTA of
// 1024 threads per (b*H + h, slab of 1024 / NG float4 columns), NG groups of E consecutive
// segments: fold each group, Hillis-Steele over the group folds, re-scan each group.

constexpr int kScanThreadsG = 1024;

__device__ __forceinline__ float4 fma4(float4 a, float4 x, float4 y) {
  return make_float4(fmaf(a.x, x.x, y.x), fmaf(a.y, x.y, y.y), fmaf(a.z, x.z, y.z),
                     fmaf(a.w, x.w, y.w));
}
__device__ __forceinline__ float4 mul4(float4 a, float4 b) {
  return make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w);
}

__global__ void __launch_bounds__(kScanThreadsG, 1)
gla_scan(GlaSegParams sp, const float* S_init, float* S_final, int NG, int E) {
  __shared__ float4 sX[kScanThreadsG];
  __shared__ float4 sA[kScanThreadsG];
  constexpr int DV = 128;
  const int W = kScanThreadsG / NG;
  const int R4 = sp.dk * DV / 4;  // scanned float4 columns: the S^T part of a record
  const int nslab = (R4 + W - 1) / W;
  const int bh = blockIdx.x / nslab;
  const int c = threadIdx.x % W;
  const int col4 = (blockIdx.x % nslab) * W + c;
  const int gi = threadIdx.x / W;
  const bool live = col4 < R4;
  const int N = sp.NS;
  const int e0 = min(N, gi * E), e1 = min(N, e0 + E);
  const int i0 = (4 * col4) % sp.dk, jv = (4 * col4) / sp.dk;
  float* base = sp.srec + static_cast<long long>(bh) * N * sp.R;
  const long long tail = static_cast<long long>(sp.dk) * DV + i0;

  float4 agg = make_float4(0.f, 0.f, 0.f, 0.f), A = make_float4(1.f, 1.f, 1.f, 1.f);
  if (live) {
    for (int e = e0; e < e1; ++e) {
      const float* r = base + static_cast<long long>(e) * sp.R;
      const float4 x = reinterpret_cast<const float4*>(r)[col4];
      const float4 a = *reinterpret_cast<const float4*>(r + tail);
      agg = fma4(a, agg, x);
      A = mul4(A, a);
    }
  }
  for (int d = 1; d < NG; d <<= 1) {
    sX[threadIdx.x] = agg;
    sA[threadIdx.x] = A;
    __syncthreads();
    if (gi >= d) {
      agg = fma4(A, sX[threadIdx.x - d * W], agg);
      A = mul4(A, sA[threadIdx.x - d * W]);
    }
    __syncthreads();
  }
  sX[threadIdx.x] = agg;
  sA[threadIdx.x] = A;
  __syncthreads();
  if (!live || e0 >= e1) return;
  const long long sbase = static_cast<long long>(bh) * sp.dk * DV;
  float4 init = make_float4(0.f, 0.f, 0.f, 0.f);
  if (S_init)
    init = make_float4(S_init[sbase + static_cast<long long>(i0) * DV + jv],
                       S_init[sbase + static_cast<long long>(i0 + 1) * DV + jv],
                       S_init[sbase + static_cast<long long>(i0 + 2) * DV + jv],
                       S_init[sbase + static_cast<long long>(i0 + 3) * DV + jv]);
  float4 carry = init;
  if (gi > 0) carry = fma4(sA[threadIdx.x - W], init, sX[threadIdx.x - W]);
  for (int e = e0; e < e1; ++e) {
    float* r = base + static_cast<long long>(e) * sp.R;
    const float4 x = reinterpret_cast<const float4*>(r)[col4];
    const float4 a = *reinterpret_cast<const float4*>(r + tail);
    reinterpret_cast<float4*>(r)[col4] = carry;
    carry = fma4(a, carry, x);
  }
  if (e1 == N && S_final) {
    S_final[sbase + static_cast<long long>(i0) * DV + jv] = carry.x;
    S_final[sbase + static_cast<long long>(i0 + 1) * DV + jv] = carry.y;
    S_final[sbase + static_cast<long long>(i0 + 2) * DV + jv] = carry.z;
    S_final[sbase + static_cast<long long>(i0 + 3) * DV + jv] = carry.w;
  }
}

template <typename Kern>
cudaError_t set_smem_g(Kern kern, uint32_t bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(bytes));
}

template <int DK>
cudaError_t gla_seg_go(const GlaSegParams& sp, const GlaSegMaps& m, const float* S_init,
                       float* S_final, bool out_f32, cudaStream_t s, Recorder* rec) {
  const unsigned grid = static_cast<unsigned>(static_cast<long long>(sp.BH) * sp.NS);
  {
    auto kern = gla_k1_seg<DK>;
    const uint32_t sm = GK1Smem<DK>::kTotal;
    cudaError_t e = set_smem_g(kern, sm);
    if (e != cudaSuccess) return e;
    if (rec) rec->mark(s, "gla_k1_seg");
    kern<<<grid, kThreadsK1, sm, s>>>(m.k, m.v, m.a, m.rec, sp);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  {
    const ScanPlan pl = scan_plan(sp.NS);
    // One block level over all segments (E grows past 16 only beyond 2048 segments).
    int ng = pl.G == 1 ? pl.NG : 128;
    const int E = (sp.NS + ng - 1) / ng;
    const int W = kScanThreadsG / ng;
    const long long nslab = (static_cast<long long>(DK) * 128 / 4 + W - 1) / W;
    if (rec) rec->mark(s, "gla_scan");
    gla_scan<<<static_cast<unsigned>(nslab * sp.BH), kScanThreadsG, 0, s>>>(sp, S_init, S_final,
                                                                           ng, E);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (out_f32) {
    auto kern = gla_k3_seg<DK, true>;
    const uint32_t sm = GK3Smem<DK>::kTotal;
    cudaError_t e = set_smem_g(kern, sm);
    if (e != cudaSuccess) return e;
    if (rec) rec->mark(s, "gla_k3_seg");
    kern<<<grid, kThreadsK3, sm, s>>>(m.q, m.k, m.v, m.a, sp);
  } else {
    auto kern = gla_k3_seg<DK, false>;
    const uint32_t sm = GK3Smem<DK>::kTotal;
    cudaError_t e = set_smem_g(kern, sm);
    if (e != cudaSuccess) return e;
    if (rec) rec->mark(s, "gla_k3_seg");
    kern<<<grid, kThreadsK3, sm, s>>>(m.q, m.k, m.v, m.a, sp);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gla_seg(const GlaSegParams& sp, const GlaSegMaps& m, const float* S_init,
                           float* S_final, bool out_f32, cudaStream_t s, Recorder* rec) {
  if (sp.dk == 64) return gla_seg_go<64>(sp, m, S_init, S_final, out_f32, s, rec);
  if (sp.dk == 128) return gla_seg_go<128>(sp, m, S_init, S_final, out_f32, s, rec);
  return cudaErrorInvalidValue;
}

}  // namespace la
