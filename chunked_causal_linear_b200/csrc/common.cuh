// Launch parameters and index helpers shared by every kernel of the prefill path.
#pragma once

#include <cstdint>

namespace la {

constexpr int kMaxHeads = 1024;

// Per-head decays, passed by value in the launch parameters (gamma_h = 1 when absent).
struct GammaTable {
  float g[kMaxHeads];
};

// One prefill problem.  The chunk summaries live in `rec`: one record of R floats per
// (b*H + h, chunk), holding S transposed (dv x dk, row-major: element (j, i) = S[i][j]
// at j*dk + i) followed by Z (dk floats) when the normalised form is requested
// (R = dk*dv + dk), else S^T alone (R = dk*dv).  Storing S^T makes the prefix state a
// K-major operand of the tensor-core product psi(Q) P in K3.
struct PrefillParams {
  int BH;          // B * H
  int H;
  long long T;
  int dk, dv, C;
  int NC;          // number of chunks, ceil(T / C)
  int L_last;      // valid tokens in the last chunk
  int R;           // floats per chunk record
  float eps;       // added to the denominator of the normalised form
  float* rec;      // [BH, NC, R] chunk summaries, turned into exclusive prefixes by K2
  float* tot;      // [BH, G, R] segment totals / segment prefixes (log-depth scan only)
  float* S_final;  // [BH, dk, dv] or nullptr
  float* Z_final;  // [BH, dk] or nullptr
  const float* S_init;  // [BH, dk, dv] state before token 0, or nullptr (zero)
  const float* Z_init;  // [BH, dk] or nullptr (zero)
  bool has_init;   // chunk 0 has a (nonzero) prefix: S_init or Z_init given
  int Ls;          // chunks per scan segment
  int G;           // number of scan segments, ceil(NC / Ls) (<= 32)
  int* err;        // device error word
};

__device__ __forceinline__ int chunk_len(const PrefillParams& p, int c) {
  return c == p.NC - 1 ? p.L_last : p.C;
}

// The segmented variant: chunks grouped into segments of Lseg chunks; one record per
// segment (same record layout as the chunk records).
struct SegParams {
  int BH;
  int H;
  long long T;
  int dk, dv, C;
  int NC;          // chunks
  int L_last;      // valid tokens in the last chunk
  int Lseg;        // chunks per segment
  int NS;          // segments per (b, h)
  int R;           // floats per record
  float eps;
  float* srec;     // [BH, NS, R] segment totals, turned into exclusive prefixes by K2
  void* out;       // [BH, T, dv] output, bf16 or fp32
  bool has_init;   // segment 0 starts from a given state (its prefix is not zero)
  bool reverse;    // the sequence runs from token T - 1 down to token 0: chunk c covers
                   // tokens [T - 64 (c + 1), T - 64 c), its position p is token T-64c-1-p
  bool tf32_prefix;  // the identity-map, unnormalised combine may read the prefix as tf32
  int* err;
};

__device__ __forceinline__ int chunk_len(const SegParams& p, int c) {
  return c == p.NC - 1 ? p.L_last : p.C;
}

// Gated linear attention on the tensor cores (segmented, dv = 128): one record per segment,
// R = dk * dv + dk floats: the segment's fold S^T (dv rows of dk), then its decay vector.
struct GlaSegParams {
  int BH;
  long long T;
  int dk;
  int NC;          // chunks of 64 tokens
  int L_last;      // valid tokens in the last chunk
  int Lseg;        // chunks per segment
  int NS;          // segments per (b, h)
  int R;           // floats per record
  float* srec;     // [BH, NS, R]: segment folds, turned into exclusive prefixes by the scan
  void* out;       // [BH, T, 128], bf16 or fp32
  unsigned char* steep;  // [BH, NC]: 1 where the chunk's intra part is left to the fix-up
  bool has_init;   // segment 0 starts from a given state
  int* err;
};

__device__ __forceinline__ int chunk_len(const GlaSegParams& p, int c) {
  return c == p.NC - 1 ? p.L_last : 64;
}

}  // namespace la
