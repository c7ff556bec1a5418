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
#include "tile_util.cuh"

namespace la {
namespace {

constexpr int kC = 64;
constexpr int kThreads = 256;  // 8 warps: two warps per TMEM lane quarter share its columns
constexpr int kWarps = kThreads / 32;

// ---------------------------------------------------------------------------------------
// K1s, warp-specialised: one CTA per (b*H + h, segment).
//   warps 0-7  transform: psi, the segment-relative weights gamma^(len_s - 1 - tau), the
//              hi / lo split of the weighted keys (hi in place, lo beside the stage) and the
//              Z column sums, chunk by chunk with no CTA-wide barrier; at the end, the
//              epilogue (TMEM -> swizzled staging -> one TMA store of the record).
//   warp 8     producer (one thread): TMA loads of K, V into a four-stage ring, a stage
//              refilled as soon as the MMAs reading it are done.
//   warp 9     MMA issuer (one thread): V^T K' into one TMEM accumulator for the segment.
// One CTA per SM (about 200 KB of shared memory at d = 128): four chunks of loads in
// flight per SM cover the memory latency, and 1024 CTAs make nearly seven even waves.

constexpr int kThreads1 = 320;
constexpr int kStages1 = 4;

template <int DK, int DV>
struct K1sSmem {
  static constexpr uint32_t kK = DK * kC * 2;
  static constexpr uint32_t kV = DV * kC * 2;
  static constexpr uint32_t kStage = kK + kV + kK;  // K (hi in place), V, lo tile of K'
  static constexpr uint32_t kIn = kStages1 * kStage;
  static constexpr uint32_t kS = DK * DV * 4;       // staging of T_s^T, aliases the inputs
  static constexpr uint32_t kRegion = kIn > kS ? kIn : kS;
  static constexpr uint32_t kBars = 3 * kStages1 + 1;
  static constexpr uint32_t kTotal = kRegion + kWarps * DK * 4 + (kBars + 1) * 8 + 1024;
};

template <int DK, int DV, int FM, bool DECAY, bool NORM>
__global__ void __launch_bounds__(kThreads1, 1)
k1_seg(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
       const __grid_constant__ CUtensorMap tm_srec, SegParams sp, GammaTable gt) {
  using L_ = K1sSmem<DK, DV>;
  constexpr bool kSplit = FM == 1 || DECAY;
  constexpr uint32_t kTmemCols = DK;
  static_assert(L_::kTotal <= 232448, "shared memory budget");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1024(smem_raw);
  uint8_t* sS = base;
  float* sZ = reinterpret_cast<float*>(base + L_::kRegion);           // [8][DK]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sZ + kWarps * DK);
  uint64_t* full = bars;                  // [kStages1]
  uint64_t* ops = bars + kStages1;        // [kStages1], 256 arrivals
  uint64_t* empty = bars + 2 * kStages1;  // [kStages1], MMA commits
  uint64_t* done = bars + 3 * kStages1;   // the segment's last MMA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + L_::kBars);

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
    for (int b = 0; b < kStages1; ++b) {
      mbar_init(&full[b], 1);
      mbar_init(&ops[b], kThreads);
      mbar_init(&empty[b], 1);
    }
    mbar_init(done, 1);
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
  bool failed = false;
  // A wait that runs out marks its thread failed; a failed thread waits no more, so every
  // role reaches the end (the transform warps walk on over meaningless data, in bounds).
  auto wait = [&](uint64_t* bar, uint32_t parity, int code) -> bool {
    if (failed) return false;
    if (mbar_wait(bar, parity)) return true;
    report_error(sp.err, code);
    failed = true;
    return false;
  };

  constexpr int NCC = DK / 8;
  constexpr int RG = kThreads / NCC;
  constexpr int kRows = kC / RG;
  if (warp < kWarps) {
    // ------------------------------------------------------------------ transform
    const int cc = tid % NCC, rg = tid / NCC;
    float zacc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) zacc[e] = 0.f;
    // The weight of the token at chunk position p of chunk i is gamma^(len_s - 1 - 64 i - p);
    // tile row r holds position p = r, or p = 63 - r when the sequence runs in reverse
    // (the tile is loaded in memory order).  For gamma >= 1/2 it is formed as a per-chunk
    // factor times gamma^(-r) (<= 2^63) or gamma^r; smaller gamma takes one powf per row,
    // since gamma^(-r) would overflow.
    const bool rev = sp.reverse;
    const bool factored = DECAY && g >= 0.5f;
    float ginv[kRows];
#pragma unroll
    for (int k = 0; k < kRows; ++k)
      ginv[k] = factored ? powf(g, (rev ? 1.f : -1.f) * static_cast<float>(rg + k * RG)) : 1.f;
    for (int i = 0; i < n; ++i) {
      const int st = i % kStages1;
      const int L = chunk_len(sp, cb + i);
      uint8_t* sK = base + st * L_::kStage;
      uint8_t* sKl = sK + L_::kK + L_::kV;
      wait(&full[st], (i / kStages1) & 1, kErrTmaTimeout);
      if constexpr (kSplit || NORM) {
        const int e0 = rev ? seg_tokens - kC - i * kC : seg_tokens - 1 - i * kC;
        const float wb = factored ? powf(g, static_cast<float>(e0)) : 1.f;
        const uint32_t boff = (cc / 8) * (kC * 128);
        uint4 raw[kRows];
#pragma unroll
        for (int k = 0; k < kRows; ++k)
          raw[k] = *reinterpret_cast<const uint4*>(sK + boff + sw128_offset(rg + k * RG, cc % 8));
#pragma unroll
        for (int k = 0; k < kRows; ++k) {
          const int r = rg + k * RG;
          float w = 0.f;
          if ((rev ? kC - 1 - r : r) < L) {
            if (!DECAY) w = 1.f;
            else if (factored) w = wb * ginv[k];
            else w = powf(g, static_cast<float>(rev ? e0 + r : e0 - r));
          }
          float x[8];
          unpack8(raw[k], x);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            x[e] = feature<FM>(x[e]) * w;
            zacc[e] += x[e];
          }
          if constexpr (kSplit) {
            uint4 hi, lo;
            split8(x, hi, lo);
            const uint32_t off = boff + sw128_offset(r, cc % 8);
            *reinterpret_cast<uint4*>(sK + off) = hi;
            *reinterpret_cast<uint4*>(sKl + off) = lo;
          }
        }
        fence_async_smem();
      }
      mbar_arrive(&ops[st]);
    }

    // Z of the segment: column sums over this CTA's threads.
    float* srec = sp.srec + (static_cast<long long>(bh) * sp.NS + seg) * sp.R;
    if constexpr (NORM) {
#pragma unroll
      for (int e = 0; e < 8; ++e)
#pragma unroll
        for (int o = NCC; o < 32; o <<= 1) zacc[e] += __shfl_xor_sync(0xffffffffu, zacc[e], o);
      if (lane < NCC)
#pragma unroll
        for (int e = 0; e < 8; ++e) sZ[warp * DK + cc * 8 + e] = zacc[e];
      named_barrier(1, kThreads);
      if (tid < DK) {
        float z = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) z += sZ[w * DK + tid];
        srec[DK * DV + tid] = z;
      }
    }

    // Epilogue: warps w and w + 4 read the same TMEM lanes, each half of the columns.  The
    // staging aliases the load stages: every load has been consumed and every MMA is done.
    wait(done, 0, kErrMmaTimeout);
    tc_fence_after();
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
    named_barrier(1, kThreads);
    if (tid == 0) {
#pragma unroll
      for (int q4 = 0; q4 < DK / 32; ++q4)
        tma_store_3d(&tm_srec, sS + q4 * (DV * 128), q4 * 32, 0, bh * sp.NS + seg);
      bulk_commit();
      bulk_wait_read_all();
    }
  } else if (warp == kWarps) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      int loads = 0;
      for (int i = 0; i < n; ++i) {
        const int st = i % kStages1;
        if (i >= kStages1 && !wait(&empty[st], ((i / kStages1) - 1) & 1, kErrMmaTimeout)) break;
        uint8_t* sK = base + st * L_::kStage;
        uint8_t* sV = sK + L_::kK;
        // In reverse the chunk's tile starts 64 (c + 1) tokens before the end; the ragged
        // last chunk starts at a negative row, which the load fills with zeros.
        const int t0 = sp.reverse ? static_cast<int>(sp.T) - (cb + i + 1) * kC : (cb + i) * kC;
        mbar_arrive_expect_tx(&full[st], L_::kK + L_::kV);
#pragma unroll
        for (int b = 0; b < DK / 64; ++b) tma_load_3d(sK + b * kC * 128, &tm_k, &full[st], b * 64, t0, bh);
#pragma unroll
        for (int b = 0; b < DV / 64; ++b) tma_load_3d(sV + b * kC * 128, &tm_v, &full[st], b * 64, t0, bh);
        ++loads;
      }
      // Every issued load has landed before the stages are reused as staging (bounded).
      for (int j = max(0, loads - kStages1); j < loads; ++j)
        mbar_wait(&full[j % kStages1], (j / kStages1) & 1);
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
      const int st = i % kStages1;
      if (!wait(&ops[st], (i / kStages1) & 1, kErrMmaTimeout)) break;
      tc_fence_after();
      const uint64_t k = dK + st * kStageD, v = dV + st * kStageD, kl = dKl + st * kStageD;
#pragma unroll
      for (int kk = 0; kk < kC / 16; ++kk) {
        mma_bf16_ss(tmem, desc_at(v, kk * 2048), desc_at(k, kk * 2048), idesc,
                    (i > 0 || kk > 0) ? 1u : 0u);
        if constexpr (kSplit)
          mma_bf16_ss(tmem, desc_at(v, kk * 2048), desc_at(kl, kk * 2048), idesc, 1u);
      }
      mma_commit(&empty[st]);
    }
    // The transform warps read the accumulator once this lands (also after a failure,
    // so that no MMA is in flight when TMEM is given up).
    mma_commit(done);
    if (failed) mbar_wait(done, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------------------
// K3s (dv = 128), warp-specialised.
//
// 576 threads in four roles that hand work over through mbarriers, so that the
// transform of chunk i + 1 overlaps the MMAs and epilogues of chunk i:
//   warps 0-7   transform (two warps per TMEM lane quarter, each half of the key features):
//               psi on the staged Q, K (bf16 hi / lo operand tiles, double buffered),
//               Xi .* psi(K), psi(q).ZP and the Z update; then the prefix operand: P^T
//               from TMEM -> bf16 hi / lo into TMEM, and P scaled by gamma^L.
//   warps 8-15  epilogue (two warps per TMEM lane quarter, each half of the columns):
//               masks and decays the scores into A (hi / lo), then combines
//               o = Theta X + N (/ den) and writes it straight to global memory (a warp
//               stores 32 consecutive value features of one token per instruction).
//   warp 16     producer (one thread): TMA loads of Q, K, V into a two-stage ring; a
//               stage is refilled as soon as the last MMA reading it (N of its chunk) is done.
//   warp 17     MMA issuer (one thread): every tcgen05.mma.  Shared-memory descriptors are
//               built once per stage; each k-step only adds a constant offset, so the
//               tensor pipe, not the issuing thread, sets the pace.
// Warp w reads TMEM lanes 32 (w % 4) .. + 31.  Accumulators (TMEM columns): scores
// [0, 64) ([0, 128) for psi = ELU+1: the hi-key and lo-key halves side by side), then X,
// N (64 each), P (dk) and P hi / lo; a second X buffer at [448, 512) where that is free.
// Each is released by an mbarrier once its readers are done.

constexpr int kThreads3 = 576;
constexpr int kXfThreads = 256;  // transform warps 0-7
constexpr int kEpThreads = 256;  // epilogue warps 8-15

template <int DK, int FM, bool DECAY, bool OUTF32>
struct K3sSmem {
  static constexpr int DV = 128;
  static constexpr uint32_t kQ = DK * kC * 2;
  static constexpr uint32_t kK = DK * kC * 2;
  // A stage's K region: for psi = ELU+1 the hi and lo tiles of psi(K) interleaved per
  // 64-feature block (hi block b, then its lo block), so that [hi; lo] is one 128-row
  // operand of the scores MMA.
  static constexpr uint32_t kKBlk = FM == 1 ? 2 * kC * 128 : kC * 128;
  static constexpr uint32_t kKs = FM == 1 ? 2 * kK : kK;
  static constexpr uint32_t kV = DV * kC * 2;
  static constexpr uint32_t kStage = kQ + kKs + kV;
  static constexpr uint32_t kLo = FM == 1 ? kQ : 0;  // lo tile of psi(Q)
  static constexpr uint32_t kKpp = DECAY ? 2 * kK : 0;    // Xi .* psi(K), hi + lo
  static constexpr uint32_t kA = kC * kC * 2;
  static constexpr uint32_t kQf = FM == 0 ? kC * DK * 4 : 0;  // float32 copy of Q (tf32 X)
  static constexpr uint32_t kSmallFloats = 9 * DK + 9 * kC + 40;
  static constexpr uint32_t kBars = 15;
  static constexpr uint32_t kTotal =
      2 * kStage + 2 * kLo + 2 * kKpp + 2 * kA + kQf + kSmallFloats * 4 + (kBars + 1) * 8 + 1024;
};


template <int DK, int FM, bool DECAY, bool NORM, bool OUTF32, bool REV, int DVR>
__global__ void __launch_bounds__(kThreads3, 1)
k3_seg(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
       const __grid_constant__ CUtensorMap tm_v, SegParams sp, GammaTable gt) {
  // The MMAs run at dv = 128 (value features on the 128 TMEM lanes); a problem with
  // DVR = 64 value features leaves the upper half of the V tile zero, so its lanes of the
  // prefix, X and N stay zero and are never stored.
  constexpr int DV = 128;
  static_assert(DVR == 64 || DVR == 128, "value features");
  using L_ = K3sSmem<DK, FM, DECAY, OUTF32>;
  constexpr bool kSplitQK = FM == 1;
  // The unnormalised identity-map forward reads the prefix for X straight from its TMEM
  // accumulator as a tf32 operand (Q copied to float32, exact for bf16 inputs), instead of
  // splitting it into bf16 hi / lo every chunk: no per-chunk pass over the state.  tf32
  // keeps 10 mantissa bits of P (error ~2^-11 relative per term, about 3e-3 of rms(o) at
  // the largest of 10^8 outputs); the normalised form (whose bound is far tighter relative
  // to its outputs, see the precision notes) and the backward's reversed passes keep the
  // split, and so do the backward's passes (sp.tf32_prefix false: their sums cancel) and
  // heads decaying faster than gamma ~ 0.52 (no renormalised window).
  constexpr bool kTf32X = FM == 0 && !NORM && !REV;
  constexpr uint32_t kTmemCols = 512;
  constexpr uint32_t kSCols = kSplitQK ? 128 : 64;
  constexpr uint32_t kColS = 0, kColX0 = kSCols, kColN = kColX0 + 64, kColP = kColN + 64;
  constexpr uint32_t kColPH = kColP + DK, kColPL = kColPH + DK / 2;
  static_assert(kColPL + DK / 2 <= kTmemCols, "TMEM budget");
  static_assert(L_::kTotal <= 232448, "shared memory budget");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1024(smem_raw);
  uint8_t* sLo = base + 2 * L_::kStage;      // [2] x Q lo
  uint8_t* sKpp = sLo + 2 * L_::kLo;         // [2] x (hi, lo)
  uint8_t* sAh = sKpp + 2 * L_::kKpp;
  uint8_t* sAl = sAh + L_::kA;
  uint8_t* sQf = sAl + L_::kA;  // float32 copy of the chunk's Q (tf32 prefix product)
  float* sZP = reinterpret_cast<float*>(sQf + L_::kQf);
  float* sZpart = sZP + DK;        // [8][DK]
  float* sDenX = sZpart + 8 * DK;  // [2][kC]
  float* sDen = sDenX + 2 * kC;
  float* sTh = sDen + kC;
  float* sPow = sTh + kC;
  float* sXi = sPow + kC;          // [2][kC]
  float* sDenPart = sXi + 2 * kC;  // [2][kC]
  float* sCw = sDenPart + 2 * kC;  // [17] gamma^(64 m)
  float* sCwInv = sCw + 20;        // [17] gamma^(-64 m)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sCwInv + 20);
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
  const float g = DECAY ? gt.g[bh % sp.H] : 1.f;
  const float* srec = sp.srec + (static_cast<long long>(bh) * sp.NS + seg) * sp.R;

  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&full[b], 1);
      mbar_init(&ops[b], kXfThreads);
      mbar_init(&xfree[b], kEpThreads);
      mbar_init(&empty[b], 1);
    }
    mbar_init(pready, kXfThreads);
    mbar_init(sfree, kEpThreads);
    mbar_init(aready, kEpThreads);
    mbar_init(sdone, 1);
    mbar_init(statedone, 1);
    mbar_init(ndone, 1);
    mbar_init(drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  // Tile row r holds chunk position p = r, or p = 63 - r in reverse (the tile is loaded in
  // memory order); sTh is indexed by tile row, sPow by position difference.  The direction
  // is a template parameter: the causal kernel carries no trace of the reverse one.
  // Decayed prefix kept as P = c P~ (TMEM holds P~): within a window of W chunks the
  // state update adds V^T (Xi .* psi(K)) / c, the epilogue scales X by c, and only the
  // window's first chunk rescales P~ in TMEM, instead of every chunk writing gamma^L P
  // back.  c = gamma^(64 m) m chunks into the window; W keeps 1 / c <= 2^60.  Heads with
  // gamma < ~0.52 (and gamma = 0) keep W = 1: P itself, decayed every chunk.
  int W = 1;
  if constexpr (DECAY) {
    if (g > 0.f) {
      const float lg = -log2f(g);
      W = lg > 0.f ? static_cast<int>(fminf(16.f, 60.f / (64.f * lg))) : 16;
    }
    if (W < 2) W = 1;
  }
  const bool renorm = W >= 2;
  constexpr bool rev = REV;
  if (tid < kC) {
    sTh[tid] = DECAY ? powf(g, static_cast<float>((rev ? kC - 1 - tid : tid) + 1)) : 1.f;
    sPow[tid] = DECAY ? powf(g, static_cast<float>(tid)) : 1.f;
  }
  // Window factors gamma^(64 m) and their inverses (m <= W <= 16), so that no role needs a
  // power per chunk.
  if (DECAY && renorm && tid >= kC && tid < kC + 17) {
    const int m = tid - kC;
    sCw[m] = powf(g, static_cast<float>(kC * m));
    sCwInv[m] = powf(g, -static_cast<float>(kC * m));
  }
  const float g64 = DECAY ? powf(g, static_cast<float>(kC)) : 1.f;
  if constexpr (NORM) {
    if (tid < DK) sZP[tid] = srec[DK * DVR + tid];
  }
  if constexpr (DVR < DV) {
    // The V tiles' upper 64 value features: zero once, never loaded.
    for (int e = tid; e < 2 * (kC * 128 / 16); e += kThreads3) {
      const int st = e / (kC * 128 / 16), o = e % (kC * 128 / 16);
      reinterpret_cast<uint4*>(base + st * L_::kStage + L_::kQ + L_::kKs + kC * 128)[o] =
          make_uint4(0u, 0u, 0u, 0u);
    }
    fence_async_smem();
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
  // and the MMA issuer drains what it has issued before TMEM is freed.
  auto wait = [&](uint64_t* bar, uint32_t parity, int code) -> bool {
    if (failed) return false;
    if (mbar_wait(bar, parity)) return true;
    report_error(sp.err, code);
    failed = true;
    return false;
  };

  // The tf32 prefix product (see kTf32X) where the state needs no per-chunk pass.
  const bool tf32x = kTf32X && sp.tf32_prefix && (!DECAY || renorm);
  // X is double-buffered where [448, 512) is free of P hi / lo (the tf32 product does not
  // use them); otherwise X(i) waits until the epilogue has read X(i - 1).
  const bool x2 = tf32x || kColPL + DK / 2 <= 448;
  const uint32_t col_x1 = x2 ? 448u : kColX0;
  auto col_x = [&](int st) -> uint32_t { return st ? col_x1 : kColX0; };

  // The prefix operand of the X MMA is prepared by the transform warps for the tf32 product
  // (a float32 copy of Q) and by the epilogue warps otherwise (P split into bf16 hi / lo in
  // TMEM), which leaves the transform warps, whose psi pass sets the pace of the feature-
  // mapped forms, the chunk's operands alone.  Either role covers the 128 TMEM lanes with
  // its 8 warps: lanes 32 (warp % 4) .. + 31, key features kHalf (warp / 4 % 2) .. + kHalf - 1.
  constexpr int kHalf = DK / 2;
  const uint32_t pcol = static_cast<uint32_t>((warp >> 2) & 1) * kHalf;
  // The segment's exclusive prefix into TMEM: row (lane) of P^T, this thread's half.
  auto load_prefix = [&]() {
    const int row = (warp & 3) * 32 + lane;
    const float4* src = reinterpret_cast<const float4*>(srec + static_cast<long long>(row) * DK + pcol);
#pragma unroll
    for (int q4 = 0; q4 < kHalf / 32; ++q4) {
      uint32_t u[32];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float4 f = row < DVR ? src[q4 * 8 + e] : make_float4(0.f, 0.f, 0.f, 0.f);
        u[4 * e] = __float_as_uint(f.x);
        u[4 * e + 1] = __float_as_uint(f.y);
        u[4 * e + 2] = __float_as_uint(f.z);
        u[4 * e + 3] = __float_as_uint(f.w);
      }
      tmem_st32(tmem + lane_base + kColP + pcol + q4 * 32, u);
    }
    tmem_st_wait();
  };
  // Prefix operand for chunk i (the state after chunk i - 1, in TMEM once statedone(i - 1)
  // completed), this thread's half of the key features: a window's first chunk turns P~
  // back into P (c = gamma^(64 W) since the last one), then P goes to bf16 hi / lo, and a
  // head without a window pre-decays P by gamma^L for the state update of chunk i.
  auto split_prefix = [&](int i) {
    const bool rescale = renorm && i > 0 && i % W == 0;
    const float c_w = rescale ? sCw[W] : 1.f;
    const int L = chunk_len(sp, cb + i);
    const float a_c = DECAY ? (L == kC ? g64 : powf(g, static_cast<float>(L))) : 1.f;
    const bool decay_now = DECAY && !renorm && i != n - 1;
    // 16 columns at a time: this runs in the epilogue warps between the score and output
    // phases, inside their register budget.
#pragma unroll 2
    for (int q = 0; q < kHalf / 16; ++q) {
      const uint32_t col = pcol + q * 16;
      float rr[16];
      tmem_ld16(tmem + lane_base + kColP + col, rr);
      tmem_ld_wait();
      if (rescale) {
        uint32_t u[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          rr[e] *= c_w;
          u[e] = __float_as_uint(rr[e]);
        }
        tmem_st16(tmem + lane_base + kColP + col, u);
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
      if (decay_now) {
        uint32_t u[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) u[e] = __float_as_uint(rr[e] * a_c);
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
    if (tf32x) load_prefix();
    constexpr int NCC = DK / 8;
    constexpr int RG = kXfThreads / NCC;
    constexpr int kRows = kC / RG;
    const int cc = tw % NCC, rg = tw / NCC;
    for (int i = 0; i < n; ++i) {
      const int s = i & 1;
      const int L = chunk_len(sp, cb + i);
      uint8_t* sQ = base + s * L_::kStage;
      uint8_t* sK = sQ + L_::kQ;
      uint8_t* sQl = sLo + s * L_::kLo;
      uint8_t* sKph = sKpp + s * L_::kKpp;
      uint8_t* sKpl = sKph + L_::kK;
      float* xi = sXi + s * kC;
      if (tw < kC) {
        const int p = rev ? kC - 1 - tw : tw;
        xi[tw] = p < L ? (DECAY ? sPow[L - 1 - p] * (renorm ? sCwInv[i % W + 1] : 1.f) : 1.f)
                       : 0.f;
      }
      wait(&full[s], (i >> 1) & 1, kErrTmaTimeout);
      named_barrier(1, kXfThreads);

      float zacc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) zacc[e] = 0.f;
      const uint32_t boff = (cc / 8) * (kC * 128);
      const uint32_t boffK = (cc / 8) * L_::kKBlk;
      float zp[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) zp[e] = NORM ? sZP[cc * 8 + e] : 0.f;
      // Every shared load of this thread's rows first, then the arithmetic and stores
      // (a load issued after a store to shared memory waits for it).
      uint4 kraw[kRows], qraw[kRows];
      float wr[kRows];
#pragma unroll
      for (int k = 0; k < kRows; ++k) {
        const int r = rg + k * RG;
        const uint32_t off = boff + sw128_offset(r, cc % 8);
        if constexpr (kSplitQK || DECAY || NORM) {
          kraw[k] = *reinterpret_cast<const uint4*>(sK + boffK + sw128_offset(r, cc % 8));
          wr[k] = xi[r];
        }
        if constexpr (kSplitQK || NORM) qraw[k] = *reinterpret_cast<const uint4*>(sQ + off);
      }
#pragma unroll
      for (int k = 0; k < kRows; ++k) {
        const int r = rg + k * RG;
        const uint32_t off = boff + sw128_offset(r, cc % 8);
        if constexpr (kSplitQK || DECAY || NORM) {
          float x[8];
          unpack8(kraw[k], x);
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = (rev ? kC - 1 - r : r) < L ? feature<FM>(x[e]) : 0.f;
          if constexpr (kSplitQK) {
            uint4 hi, lo;
            split8(x, hi, lo);
            const uint32_t offK = boffK + sw128_offset(r, cc % 8);
            *reinterpret_cast<uint4*>(sK + offK) = hi;
            *reinterpret_cast<uint4*>(sK + offK + kC * 128) = lo;
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            x[e] *= wr[k];
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
          unpack8(qraw[k], x);
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

      // gamma^L: Theta of the chunk's last token for a full chunk.
      const float a_c = DECAY ? (L == kC ? g64 : powf(g, static_cast<float>(L))) : 1.f;
      if constexpr (NORM) {
#pragma unroll
        for (int e = 0; e < 8; ++e)
#pragma unroll
          for (int o = NCC; o < 32; o <<= 1) zacc[e] += __shfl_xor_sync(0xffffffffu, zacc[e], o);
        if (lane < NCC)
#pragma unroll
          for (int e = 0; e < 8; ++e) sZpart[warp * DK + cc * 8 + e] = zacc[e];
        named_barrier(1, kXfThreads);
        if (tw < DK) {
          float zs = 0.f;
#pragma unroll
          for (int w = 0; w < 8; ++w) zs += sZpart[w * DK + tw];
          sZP[tw] = fmaf(a_c, sZP[tw], zs);
        }
      }

      if (tf32x) {
        // tf32 prefix product: X reads P~ in place.  A window's first chunk turns P~ back
        // into P first; then the chunk's Q goes to float32 (K-major, 128-byte swizzle, 32
        // features per row) once the previous chunk's X has read the copy.
        if (i > 0) wait(statedone, (i - 1) & 1, kErrMmaTimeout);
        tc_fence_after();
        if (DECAY && i > 0 && i % W == 0) {
          const float c_w = sCw[W];
#pragma unroll
          for (int q4 = 0; q4 < kHalf / 32; ++q4) {
            const uint32_t col = pcol + q4 * 32;
            float rr[32];
            tmem_ld32(tmem + lane_base + kColP + col, rr);
            tmem_ld_wait();
            uint32_t u[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(rr[e] * c_w);
            tmem_st32(tmem + lane_base + kColP + col, u);
          }
          tmem_st_wait();
        }
        for (int e = tw; e < kC * DK / 8; e += kXfThreads) {
          const int r = e / (DK / 8), c8 = e % (DK / 8);
          const uint4 raw =
              *reinterpret_cast<const uint4*>(sQ + (c8 / 8) * (kC * 128) + sw128_offset(r, c8 % 8));
          float x[8];
          unpack8(raw, x);
          const int f0 = c8 * 8;
          uint8_t* dst = sQf + (f0 / 32) * (kC * 128);
          *reinterpret_cast<float4*>(dst + sw128_offset(r, (f0 % 32) / 4)) =
              make_float4(x[0], x[1], x[2], x[3]);
          *reinterpret_cast<float4*>(dst + sw128_offset(r, (f0 % 32) / 4 + 1)) =
              make_float4(x[4], x[5], x[6], x[7]);
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(pready);
      }
    }
  } else if (warp < 16) {
    // ------------------------------------------------------------------ epilogue
    const int tw = tid - kXfThreads;
    const int quarter = warp & 3, half = (warp - 8) >> 2;
    const int j = quarter * 32 + lane;  // value feature of this thread's output column
    if (!tf32x) {
      load_prefix();
      split_prefix(0);
    }
    for (int i = 0; i < n; ++i) {
      const int s = i & 1;
      const long long t0 = rev ? sp.T - static_cast<long long>(cb + i + 1) * kC
                               : static_cast<long long>(cb + i) * kC;
      const int L = chunk_len(sp, cb + i);
      const bool has_prefix = !(seg == 0 && i == 0) || sp.has_init;
      wait(sdone, i & 1, kErrMmaTimeout);
      wait(&ops[s], (i >> 1) & 1, kErrMmaTimeout);
      tc_fence_after();
      {
        // Row 16 quarter + (lane % 16), keys kb .. kb + 15 with kb = 32 half + 16 (lane / 16):
        // the 64-row score tile sits in lanes 0-15 of each quarter, and the 16-lane load
        // gives both halves of the warp a share of its columns.
        const int row = quarter * 16 + (lane & 15);
        const int kb = 32 * half + 16 * (lane >> 4);
        float sc[16];
        tmem_ld16x2_x16(tmem + lane_base + kColS + 32 * half, sc);
        if constexpr (kSplitQK) {  // the lo-key half
          float sl[16];
          tmem_ld16x2_x16(tmem + lane_base + kColS + 64 + 32 * half, sl);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; ++e) sc[e] += sl[e];
        }
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(sfree);
        // gamma^(row - key), zero above the diagonal; all loads before the stores.
        float den_loc = 0.f;
        uint4 hi[2], lo[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          float a[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int d = rev ? kb + q * 8 + e - row : row - kb - q * 8 - e;
            a[e] = d >= 0 ? (DECAY ? sc[q * 8 + e] * sPow[d] : sc[q * 8 + e]) : 0.f;
            den_loc += a[e];
          }
          split8(a, hi[q], lo[q]);
        }
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          *reinterpret_cast<uint4*>(sAh + sw128_offset(row, kb / 8 + q)) = hi[q];
          *reinterpret_cast<uint4*>(sAl + sw128_offset(row, kb / 8 + q)) = lo[q];
        }
        if constexpr (NORM) {
          den_loc += __shfl_xor_sync(0xffffffffu, den_loc, 16);
          if (lane < 16) sDenPart[half * kC + row] = den_loc;
        }
      }
      fence_async_smem();
      if constexpr (NORM) {
        // psi(q).ZP of this chunk is read before A is handed over: once N(i) is done
        // the stage (and its sDenX slot) is refilled with chunk i + 2.
        named_barrier(2, kEpThreads);
        if (tw < kC) {
          const float den_loc = sDenPart[tw] + sDenPart[kC + tw];
          // The reciprocal, so that the 32 outputs of a thread take multiplications.
          // (The fast reciprocal: ~2 ulp, far below the split operands' 2^-16; the
          // denominator is a positive sum of bounded scores, never near 2^126.)
          sDen[tw] = __fdividef(1.f, (has_prefix ? fmaf(sTh[tw], sDenX[s * kC + tw], den_loc) : den_loc) + sp.eps);
        }
      }
      mbar_arrive(aready);

      // The next chunk's prefix operand, while N(i) runs: X(i) and the state update with
      // chunk i are done once statedone(i) completes.
      if (!tf32x && i + 1 < n) {
        wait(statedone, i & 1, kErrMmaTimeout);
        tc_fence_after();
        split_prefix(i + 1);
      }

      wait(ndone, i & 1, kErrMmaTimeout);
      tc_fence_after();
      // Column j (value feature), tokens 32 half .. + 31.
      float xo[32], no[32];
      if (has_prefix) tmem_ld32(tmem + lane_base + col_x(s) + 32 * half, xo);
      tmem_ld32(tmem + lane_base + kColN + 32 * half, no);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&xfree[s]);
      if constexpr (NORM) named_barrier(2, kEpThreads);  // sDen of this chunk
      // Theta (and den) of this warp's 32 tokens as float4 broadcasts, all before the
      // first global store.
      if (has_prefix) {
        // X was computed from P~: the chunk's Theta carries the window factor c.
        const float c = renorm ? sCw[i % W] : 1.f;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 th = *reinterpret_cast<const float4*>(sTh + 32 * half + 4 * q);
          no[4 * q] = fmaf(th.x * c, xo[4 * q], no[4 * q]);
          no[4 * q + 1] = fmaf(th.y * c, xo[4 * q + 1], no[4 * q + 1]);
          no[4 * q + 2] = fmaf(th.z * c, xo[4 * q + 2], no[4 * q + 2]);
          no[4 * q + 3] = fmaf(th.w * c, xo[4 * q + 3], no[4 * q + 3]);
        }
      }
      if constexpr (NORM) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 dn = *reinterpret_cast<const float4*>(sDen + 32 * half + 4 * q);
          no[4 * q] *= dn.x;
          no[4 * q + 1] *= dn.y;
          no[4 * q + 2] *= dn.z;
          no[4 * q + 3] *= dn.w;
        }
      }
      const long long row0 = static_cast<long long>(bh) * sp.T + t0 + 32 * half;
      // Tokens of this half inside the sequence: tile rows [t_lo, t_hi).
      const int t_lo = rev ? max(0, kC - L - 32 * half) : 0;
      const int t_hi = rev ? 32 : min(32, L - 32 * half);
#pragma unroll
      for (int tt = 0; tt < 32; ++tt) {
        if (tt >= t_lo && tt < t_hi && j < DVR) {
          const long long idx = (row0 + tt) * DVR + j;
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
        // Stage i & 1 is free once N(i - 2), the last MMA reading it, is done.
        if (i >= 2 && !wait(&empty[i & 1], ((i - 2) >> 1) & 1, kErrMmaTimeout)) break;
        uint8_t* sQ = base + (i & 1) * L_::kStage;
        uint8_t* sK = sQ + L_::kQ;
        uint8_t* sV = sK + L_::kKs;
        const int t0 = rev ? static_cast<int>(sp.T) - (cb + i + 1) * kC : (cb + i) * kC;
        mbar_arrive_expect_tx(&full[i & 1], L_::kQ + L_::kK + DVR * kC * 2);
#pragma unroll
        for (int b = 0; b < DK / 64; ++b) {
          tma_load_3d(sQ + b * kC * 128, &tm_q, &full[i & 1], b * 64, t0, bh);
          tma_load_3d(sK + b * L_::kKBlk, &tm_k, &full[i & 1], b * 64, t0, bh);
        }
#pragma unroll
        for (int b = 0; b < DVR / 64; ++b)
          tma_load_3d(sV + b * kC * 128, &tm_v, &full[i & 1], b * 64, t0, bh);
        ++loads;
      }
      // The last two loads have landed before shared memory is given up (in a run
      // without failures they were consumed already; the waits are bounded).
      for (int jl = max(0, loads - 2); jl < loads; ++jl) mbar_wait(&full[jl & 1], (jl >> 1) & 1);
    }
  } else if (lane == 0) {
    // ------------------------------------------------------------------ MMA issuer
    // Descriptors of stage 0 (K-major: 128-byte rows, 1024-byte groups of eight; MN-major:
    // 128-byte atoms, kC * 128 bytes apart); stage 1 is kStage bytes further on.
    const uint32_t a0 = smem_u32(base);
    const uint64_t dQk = smem_desc_sw128(a0, 16, 1024);                       // Q, K-major
    const uint64_t dKk = smem_desc_sw128(a0 + L_::kQ, 16, 1024);                // K, K-major
    const uint64_t dKm = smem_desc_sw128(a0 + L_::kQ, L_::kKBlk, 1024);         // K, MN-major
    const uint64_t dKlm = smem_desc_sw128(a0 + L_::kQ + kC * 128, L_::kKBlk, 1024);  // K lo
    const uint64_t dVm = smem_desc_sw128(a0 + L_::kQ + L_::kKs, kC * 128, 1024);  // V, MN-major
    const uint32_t lo0 = smem_u32(sLo), kp0 = smem_u32(sKpp);
    const uint64_t dQlk = smem_desc_sw128(lo0, 16, 1024);
    const uint64_t dKhm = smem_desc_sw128(kp0, kC * 128, 1024);
    const uint64_t dKpm = smem_desc_sw128(kp0 + L_::kK, kC * 128, 1024);
    const uint64_t dAh = smem_desc_sw128(smem_u32(sAh), 16, 1024);
    const uint64_t dAl = smem_desc_sw128(smem_u32(sAl), 16, 1024);
    const uint64_t dQf = smem_desc_sw128(smem_u32(sQf), 16, 1024);  // float32 Q, K-major
    constexpr uint32_t kStageD = L_::kStage >> 4, kLoD = L_::kLo >> 4, kKppD = L_::kKpp >> 4;

    auto issue_scores = [&](int i) -> bool {
      const int s = i & 1;
      const uint64_t q = dQk + s * kStageD, k = dKk + s * kStageD;
      const uint64_t ql = dQlk + s * kLoD;
      if (!wait(&ops[s], (i >> 1) & 1, kErrMmaTimeout)) return false;
      if (i > 0 && !wait(sfree, (i - 1) & 1, kErrMmaTimeout)) return false;
      tc_fence_after();
      constexpr uint32_t ids = instr_desc(kFmtBF16, kFmtBF16, kKMajor, kKMajor, 64, 64);
      // psi = ELU+1: psi(Q)_hi [psi(K)_hi; psi(K)_lo]^T as one N = 128 MMA (the hi-key
      // and lo-key scores side by side, summed by the epilogue), plus psi(Q)_lo psi(K)_hi^T
      // into the hi-key half: two MMAs per 16 features instead of three (an MMA costs
      // about as much at N = 128 as at N = 64).
      constexpr uint32_t ids2 = instr_desc(kFmtBF16, kFmtBF16, kKMajor, kKMajor, 64, 128);
#pragma unroll
      for (int kk = 0; kk < DK / 16; ++kk) {
        const uint32_t off = (kk / 4) * (kC * 128) + (kk % 4) * 32;
        const uint32_t offk = (kk / 4) * L_::kKBlk + (kk % 4) * 32;
        if constexpr (kSplitQK) {
          mma_bf16_ss(tmem + kColS, desc_at(q, off), desc_at(k, offk), ids2, kk > 0 ? 1u : 0u);
          mma_bf16_ss(tmem + kColS, desc_at(ql, off), desc_at(k, offk), ids, 1u);
        } else {
          mma_bf16_ss(tmem + kColS, desc_at(q, off), desc_at(k, offk), ids, kk > 0 ? 1u : 0u);
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

      // X(i) = P^T psi(Q)^T and the prefix update with chunk i.
      if (!wait(pready, i & 1, kErrMmaTimeout)) break;
      if (x2) {
        if (i > 1 && !wait(&xfree[s], ((i - 2) >> 1) & 1, kErrMmaTimeout)) break;
      } else if (i > 0 && !wait(&xfree[s ^ 1], ((i - 1) >> 1) & 1, kErrMmaTimeout)) {
        break;
      }
      tc_fence_after();
      if (tf32x) {
        if (has_prefix) {
          constexpr uint32_t idt = instr_desc(kFmtTF32, kFmtTF32, kKMajor, kKMajor, 128, 64);
#pragma unroll
          for (int kk = 0; kk < DK / 8; ++kk) {
            const uint32_t off = (kk / 4) * (kC * 128) + (kk % 4) * 32;
            mma_tf32_ts(tmem + col_x(s), tmem + kColP + kk * 8, desc_at(dQf, off), idt,
                        kk > 0 ? 1u : 0u);
          }
        }
      } else if (has_prefix) {
        constexpr uint32_t idx = instr_desc(kFmtBF16, kFmtBF16, kKMajor, kKMajor, 128, 64);
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
          const uint32_t off = (kk / 4) * (kC * 128) + (kk % 4) * 32;
          mma_bf16_ts(tmem + col_x(s), tmem + kColPH + kk * 8, desc_at(q, off), idx,
                      kk > 0 ? 1u : 0u);
          mma_bf16_ts(tmem + col_x(s), tmem + kColPL + kk * 8, desc_at(q, off), idx, 1u);
          if constexpr (kSplitQK)
            mma_bf16_ts(tmem + col_x(s), tmem + kColPH + kk * 8, desc_at(ql, off), idx, 1u);
        }
      }
      if (!last) {
        constexpr uint32_t idp = instr_desc(kFmtBF16, kFmtBF16, kMNMajor, kMNMajor, 128, DK);
        const uint64_t bh_ = DECAY ? dKhm + s * kKppD : dKm + s * kStageD;
        const uint64_t bl_ = DECAY ? dKpm + s * kKppD : dKlm + s * kStageD;
#pragma unroll
        for (int kk = 0; kk < kC / 16; ++kk) {
          mma_bf16_ss(tmem + kColP, desc_at(v, kk * 2048), desc_at(bh_, kk * 2048), idp, 1u);
          if constexpr (kSplitQK || DECAY)
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

      // The next chunk's scores go in right behind N(i).
      if (i + 1 < n && !issue_scores(i + 1)) break;
    }
    if (failed) {
      // Let the issued MMAs finish before TMEM is given up (bounded).
      mma_commit(drain);
      mbar_wait(drain, 0);
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
  kern<<<static_cast<unsigned>(grid), kThreads1, sm, s>>>(m.k, m.v, m.rec, sp, gt);
  return cudaGetLastError();
}

template <int DK, int FM, bool DECAY, bool NORM, bool OUTF32, bool REV>
cudaError_t k3s_go_r(const SegParams& sp, const GammaTable& gt, const TcMaps& m, cudaStream_t s) {
  auto kern = sp.dv == 64 ? k3_seg<DK, FM, DECAY, NORM, OUTF32, REV, 64>
                          : k3_seg<DK, FM, DECAY, NORM, OUTF32, REV, 128>;
  const uint32_t sm = K3sSmem<DK, FM, DECAY, OUTF32>::kTotal;
  cudaError_t e = set_smem(kern, sm);
  if (e != cudaSuccess) return e;
  const long long grid = static_cast<long long>(sp.BH) * sp.NS;
  kern<<<static_cast<unsigned>(grid), kThreads3, sm, s>>>(m.q, m.k, m.v, sp, gt);
  return cudaGetLastError();
}

template <int DK, int FM, bool DECAY, bool NORM, bool OUTF32>
cudaError_t k3s_go_o(const SegParams& sp, const GammaTable& gt, const TcMaps& m, cudaStream_t s) {
  return sp.reverse ? k3s_go_r<DK, FM, DECAY, NORM, OUTF32, true>(sp, gt, m, s)
                    : k3s_go_r<DK, FM, DECAY, NORM, OUTF32, false>(sp, gt, m, s);
}

template <int DK, int DV, int FM, bool DECAY, bool NORM>
cudaError_t k3s_go(const SegParams& sp, const GammaTable& gt, const TcMaps& m, Flags f,
                   cudaStream_t s) {
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
  return C == kC && (dk == 64 || dk == 128) && (dv == 64 || dv == 128) && !(fm == 1 && decay);
}

cudaError_t launch_k1_seg(const SegParams& sp, const GammaTable& gt, const TcMaps& m, Flags f,
                          cudaStream_t s) {
  if (sp.dk == 64 && sp.dv == 128) LA_SEG_FLAGS(64, 128, k1s_go);
  if (sp.dk == 128 && sp.dv == 128) LA_SEG_FLAGS(128, 128, k1s_go);
  if (sp.dk == 64 && sp.dv == 64) LA_SEG_FLAGS(64, 64, k1s_go);
  if (sp.dk == 128 && sp.dv == 64) LA_SEG_FLAGS(128, 64, k1s_go);
  return cudaErrorInvalidValue;
}

cudaError_t launch_k3_seg(const SegParams& sp, const GammaTable& gt, const TcMaps& m, Flags f,
                          cudaStream_t s) {
  // k3s_go_r picks the kernel for sp.dv (64 or 128); the MMA geometry is the same.
  if (sp.dk == 64 && (sp.dv == 128 || sp.dv == 64)) LA_SEG_FLAGS(64, 128, k3s_go);
  if (sp.dk == 128 && (sp.dv == 128 || sp.dv == 64)) LA_SEG_FLAGS(128, 128, k3s_go);
  return cudaErrorInvalidValue;
}

}  // namespace la
