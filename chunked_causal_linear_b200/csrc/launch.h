// Host-side launchers for the prefill and decode kernels (internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/linattn.h"
#include "common.cuh"

namespace la {

// The full prefill of lin_attn_prefill_ex (validation, workspace, launches).
int prefill_with_args(const la_prefill_args& a);

enum Dtype : int { kBF16 = 0, kF32 = 1 };

struct Flags {
  int fm;       // 0 identity, 1 elu+1
  bool decay;
  bool norm;
  bool out_f32; // float32 output (bf16 inputs only; float32 inputs always write float32)
};

// Optional per-kernel timing: when set, every launcher records the next event on the
// stream just before each of its kernel launches.
struct Recorder {
  cudaEvent_t* ev = nullptr;
  int n = 0;
  int cap = 0;
  void mark(cudaStream_t s) {
    if (ev && n < cap) cudaEventRecord(ev[n++], s);
  }
};

// CUDA-core fp32 FMA kernels (any supported shape, float32 or bf16 inputs).
cudaError_t launch_k1_fma(const PrefillParams& p, const GammaTable& gt, const void* k,
                          const void* v, int dtype, Flags f, cudaStream_t s);
cudaError_t launch_k3_fma(const PrefillParams& p, const GammaTable& gt, const void* q,
                          const void* k, const void* v, void* out, int dtype, Flags f,
                          cudaStream_t s);

// K2: scan of the chunk records (mode 0 log-depth over segments, 1 sequential carry).
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

// One recurrent decode step for every (b, h).
cudaError_t launch_decode(const void* q, const void* k, const void* v, void* out, float* S,
                          float* Z, int BH, int H, int dk, int dv, int dtype, Flags f,
                          const GammaTable& gt, float eps, int* err, cudaStream_t s);

}  // namespace la
