// Incoming state of one part of a sequence split into consecutive parts: the scan page's
// monoid ("Log-Depth Chunked Linear-Attention Scan", Formulas: (S1, Z1) + (S2, Z2) =
// (S1 + S2, Z1 + Z2)) with the retention decay ("Linear Attention and Retentive Networks
// ...", C. Chunkwise Recurrent Representation: a part of L tokens scales what came before
// it by gamma^L), folded over whole parts in order.  One thread per state element.

#include <cuda_runtime.h>

#include <cmath>

#include "../../include/linattn.h"
#include "common.cuh"

namespace la {
namespace {

constexpr int kMaxParts = 64;

struct PartTokens {
  long long t[kMaxParts];
};

__global__ void combine_states(const float* __restrict__ parts, long long part_stride,
                               int upto, int per_head, int H, long long n, GammaTable gt,
                               PartTokens pt, bool decay, float* __restrict__ out) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= n) return;
  const int h = static_cast<int>((idx / per_head) % H);
  const float g = gt.g[h];
  float P = 0.f;
  for (int j = 0; j < upto; ++j) {
    const float a = decay ? powf(g, static_cast<float>(pt.t[j])) : 1.f;
    P = fmaf(a, P, parts[static_cast<long long>(j) * part_stride + idx]);
  }
  out[idx] = P;
}

}  // namespace
}  // namespace la

extern "C" int lin_attn_combine_states(const float* S_parts, const float* Z_parts, int parts,
                                       int upto, const long long* part_tokens, int B, int H,
                                       int dk, int dv, const float* gamma, float* S_out,
                                       float* Z_out, la_stream_t stream) {
  using namespace la;
  if (B < 0 || H < 0 || dk <= 0 || dv <= 0 || parts < 0 || upto < 0 || upto > parts)
    return LA_ERR_INVALID_ARGUMENT;
  if (parts > kMaxParts || H > kMaxHeads) return LA_ERR_UNSUPPORTED;
  const long long BH = static_cast<long long>(B) * H;
  if (BH == 0) return LA_OK;
  if (!S_parts || !S_out || (Z_out && !Z_parts) || (parts > 0 && !part_tokens))
    return LA_ERR_INVALID_ARGUMENT;
  PartTokens pt{};
  for (int j = 0; j < parts; ++j) {
    if (part_tokens[j] < 0) return LA_ERR_INVALID_ARGUMENT;
    pt.t[j] = part_tokens[j];
  }
  GammaTable gt;
  for (int h = 0; h < kMaxHeads; ++h) gt.g[h] = 1.f;
  if (gamma)
    for (int h = 0; h < H; ++h) {
      if (!(gamma[h] >= 0.f && gamma[h] <= 1.f)) return LA_ERR_INVALID_ARGUMENT;
      gt.g[h] = gamma[h];
    }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long nS = BH * dk * dv, nZ = BH * dk;
  combine_states<<<static_cast<unsigned>((nS + 255) / 256), 256, 0, s>>>(
      S_parts, nS, upto, dk * dv, H, nS, gt, pt, gamma != nullptr, S_out);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess && Z_out) {
    combine_states<<<static_cast<unsigned>((nZ + 255) / 256), 256, 0, s>>>(
        Z_parts, nZ, upto, dk, H, nZ, gt, pt, gamma != nullptr, Z_out);
    e = cudaGetLastError();
  }
  return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}
