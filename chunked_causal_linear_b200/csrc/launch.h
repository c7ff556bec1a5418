// Host-side launchers for the prefill and decode kernels (internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/linattn.h"
#include "common.cuh"

namespace la {

// The argument checks of the prefill alone: LA_OK when prefill_with_args(a) would launch.
int check_prefill_args(const la_prefill_args& a);

// The device error word of the current device (every kernel receives it).
int* device_error_word();

// Workspace allocation of every entry point that allocates (cudaMallocAsync on the
// stream).  With the environment variable LA_FAULT_INJECT=alloc it fails without
// allocating, so that callers' handling of LA_ERR_OUT_OF_MEMORY can be tested.
cudaError_t workspace_alloc(void** p, size_t bytes, cudaStream_t s);

// A 3D tiled TMA map (d0 innermost) with the 128-byte swizzle, as the prefill's kernels use.
bool make_tile_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t d0,
                   uint64_t d1, uint64_t d2, uint64_t stride1, uint64_t stride2, uint32_t box0,
                   uint32_t box1);

enum Dtype : int { kBF16 = 0, kF32 = 1 };

struct Flags {
  int fm;       // 0 identity, 1 elu+1
  bool decay;
  bool norm;
  bool out_f32; // float32 output (bf16 inputs only; float32 inputs always write float32)
};

// Optional per-kernel timing: when set, every launcher records the next event on the
// stream just before each of its kernel launches, labelled with the kernel's name, and the
// prefill records an unlabelled event after its last kernel.  Interval i (event i to
// event i + 1) is the kernel `label[i]`; an unlabelled interval holds no kernel.
struct Recorder {
  cudaEvent_t* ev = nullptr;
  const char** label = nullptr;
  int n = 0;
  int cap = 0;
  void mark(cudaStream_t s, const char* name = nullptr) {
    if (ev && n < cap) {
      if (label) label[n] = name;
      cudaEventRecord(ev[n++], s);
    }
  }
};

// The full prefill of lin_attn_prefill_ex (validation, workspace, launches), optionally
// recording an event before every kernel.
// exact_prefix: keep the bf16 hi / lo split of the carried prefix in the combine even where
// the forward reads it as tf32 (the backward's passes, whose sums cancel).
int prefill_with_args(const la_prefill_args& a, Recorder* rec = nullptr,
                      bool exact_prefix = false);

// CUDA-core fp32 FMA kernels (any supported shape, float32 or bf16 inputs).
cudaError_t launch_k1_fma(const PrefillParams& p, const GammaTable& gt, const void* k,
                          const void* v, int dtype, Flags f, cudaStream_t s);
cudaError_t launch_k3_fma(const PrefillParams& p, const GammaTable& gt, const void* q,
                          const void* k, const void* v, void* out, int dtype, Flags f,
                          cudaStream_t s);

// The log-depth K2's shape for n scan elements: up to kScanBlockElems elements one blocked
// scan (NG groups of E elements, Hillis-Steele over the groups); beyond that G segments of
// Ls >= kScanMinSegment elements, their folds scanned by the blocked scan.  `depth` is the
// longest chain of dependent combine steps: 2E + log2 NG (+ 2 Ls with segments).
constexpr long long kScanBlockElems = 2048;
constexpr long long kScanMinSegment = 16;
struct ScanPlan {
  int Ls = 1;  // elements per segment (n itself with one level)
  int G = 1;   // segments (1 with one level)
  int NG = 1;  // groups of the blocked scan (a power of two, <= 128)
  int E = 0;   // elements per group
  long long depth = 0;
};
ScanPlan scan_plan(long long n);

// K2: scan of the chunk records (mode 0 log-depth, 1 sequential carry).
cudaError_t launch_k2(const PrefillParams& p, const GammaTable& gt, int mode, Flags f,
                      cudaStream_t s, Recorder* rec = nullptr);

// Tensor-core (tcgen05/TMEM, TMA) kernels for bf16 inputs, dk, dv in {64, 128}, C = 64.
struct TcMaps {
  CUtensorMap q, k, v, out, rec;
};
cudaError_t launch_k1_tc(const PrefillParams& p, const GammaTable& gt, const TcMaps& m,
                         Flags f, cudaStream_t s);
cudaError_t launch_k3_tc(const PrefillParams& p, const GammaTable& gt, const TcMaps& m,
                         Flags f, cudaStream_t s);

// Segmented variant (seg_kernels.cu): K1s writes one record per segment, K3s walks a
// segment's chunks carrying the prefix in TMEM.  bf16 inputs, C = 64, dk in {64, 128},
// dv = 128, and not the ELU+1 map together with decay.
bool seg_supported(int dk, int dv, int C, int fm, bool decay);
cudaError_t launch_k1_seg(const SegParams& sp, const GammaTable& gt, const TcMaps& m, Flags f,
                          cudaStream_t s);
cudaError_t launch_k3_seg(const SegParams& sp, const GammaTable& gt, const TcMaps& m, Flags f,
                          cudaStream_t s);

// Gated linear attention on the tensor cores, segmented (gla_seg.cu): bf16 q, k, v,
// float32 gates, C = 64, dk in {64, 128}, dv = 128.  K1 (segment folds), the scan over
// segments (writes S_final), K3 (the combine; flags the chunks whose intra part the
// CUDA-core fix-up must add).
struct GlaSegMaps {
  CUtensorMap q, k, v, a, rec;
};
cudaError_t launch_gla_seg(const GlaSegParams& sp, const GlaSegMaps& m, const float* S_init,
                           float* S_final, bool out_f32, cudaStream_t s, Recorder* rec);

// A 3D tiled TMA map without swizzle (d0 innermost), for float32 gate tiles.
bool make_plain_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t d0,
                    uint64_t d1, uint64_t d2, uint64_t stride1, uint64_t stride2, uint32_t box0,
                    uint32_t box1);

// Chunks per segment chosen automatically for BH heads of NC chunks (about four segments
// per SM, at most 64 chunks each).
int default_segment_chunks(long long BH, int NC);

// One recurrent decode step for every (b, h).
cudaError_t launch_decode(const void* q, const void* k, const void* v, void* out, float* S,
                          float* Z, int BH, int H, int dk, int dv, int dtype, Flags f,
                          const GammaTable& gt, float eps, int* err, cudaStream_t s);

}  // namespace la
