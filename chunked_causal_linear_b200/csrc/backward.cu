// Backward pass of the unnormalised form: the gradients of "Linear Attention and Retentive
// Networks ..." (B. Recurrent Representation, with S_{-1} = S_init) written as three
// causal linear attentions, each computed by the library's own prefill.
//
// With G_t = dL/dS_t (G_t = psi(q_t) do_t^T + gamma G_{t+1}, G_{T-1} holding dS_final):
//   dpsi(q)_t = S_t do_t       = sum_{s<=t} gamma^(t-s) (do_t . v_s) psi(k_s)
//                                + gamma^(t+1) S_init^T-readout
//       -> the prefill of (q', k', v') = (do, v, psi(k)) with the identity map and
//          S'_init = S_init^T;
//   dv_s        = G_s^T psi(k_s) = sum_{t>=s} gamma^(t-s) (psi(k_s) . psi(q_t)) do_t
//                                  + gamma^(T-1-s) dS_final^T psi(k_s)
//       -> on the time-reversed sequence (sigma = T-1-s) the prefill of (k, q, do) with
//          the model's map, S'_init = dS_final / gamma (its readout weight gamma^(sigma+1)
//          then gives gamma^sigma); its final state is G_0;
//   dpsi(k)_s   = G_s v_s      -> reversed, the prefill of (v, do, psi(q)) with the
//          identity map and S'_init = dS_final^T / gamma;
//   dS_init     = gamma G_0.
// The element-wise kernels here reverse time, apply psi and psi', and fold in the
// dS_final terms of heads whose decay is too small to divide by.

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "../../include/linattn.h"
#include "common.cuh"
#include "launch.h"

namespace la {
namespace {

// Heads with gamma below this take the dS_final terms from fix_small_decay (terms
// gamma^sigma, sigma >= 3, are below 2^-60 of the sigma = 0 term and are dropped).
constexpr float kSmallDecay = 0x1p-20f;
constexpr int kSmallDecayTerms = 3;
constexpr int kMaxJobs = 8;

__device__ __forceinline__ float psi(float x, int fm) {
  return fm == LA_FM_ELU1 ? (x > 0.f ? x + 1.f : expf(x)) : x;
}
__device__ __forceinline__ float psi_prime(float x, int fm) {
  return fm == LA_FM_ELU1 ? (x > 0.f ? 1.f : expf(x)) : 1.f;
}

// Four consecutive elements of a bf16 or float32 row.
__device__ __forceinline__ float4 load4(const void* base, long long idx, bool f32) {
  if (f32) return __ldcs(reinterpret_cast<const float4*>(static_cast<const float*>(base) + idx));
  const uint2 u = __ldcs(reinterpret_cast<const uint2*>(
      static_cast<const __nv_bfloat16*>(base) + idx));
  __nv_bfloat162 a, b;
  std::memcpy(&a, &u.x, 4);
  std::memcpy(&b, &u.y, 4);
  const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
  return make_float4(fa.x, fa.y, fb.x, fb.y);
}
__device__ __forceinline__ void store4(void* base, long long idx, float4 x, bool f32) {
  if (f32) {
    __stcs(reinterpret_cast<float4*>(static_cast<float*>(base) + idx), x);
    return;
  }
  const __nv_bfloat162 a = __float22bfloat162_rn(make_float2(x.x, x.y));
  const __nv_bfloat162 b = __float22bfloat162_rn(make_float2(x.z, x.w));
  uint2 u;
  std::memcpy(&u.x, &a, 4);
  std::memcpy(&u.y, &b, 4);
  __stcs(reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(base) + idx), u);
}

// dst[bh, t'] = (f(src[bh, t] + src2[bh, t]) rs[bh, t] + src3[bh, t]) g(x[bh, t']) for rows
// of d elements, where t' = T-1-t when `flip`, else t; f = psi when `fm_src` is ELU+1,
// g = psi' of x when `x` is given (absent terms drop out).  With `lo`, dst2 also receives
// the part of the value that bf16 rounding drops (value - bf16(value), itself rounded to
// bf16): a bf16 hi + lo pair carries psi to about 16 bits, like the split operands of the
// prefill's own kernels.
struct RowJob {
  const void* src;
  const void* src2;  // added to src (same type), or nullptr
  const void* src3;  // added after the row scale, or nullptr
  const float* rs;   // per-row scale of (src + src2), indexed by the source row, or nullptr
  void* dst;
  void* dst2;        // with `lo`: the value's bf16 residual goes here, the value to dst
  const void* x;     // multiplier input (same layout as dst, type of the inputs) or nullptr
  int d;
  int fm_src;        // la_feature_map applied to src
  int fm_x;          // la_feature_map whose derivative multiplies by x
  bool flip, lo;
  bool src_f32, dst_f32, x_f32;
};
struct RowJobs {
  RowJob j[kMaxJobs];
};

// Eight consecutive elements (or four, for rows of 4 (mod 8) elements) of a bf16 or float32
// row.
template <int W>
struct Vec {
  float v[W];
};
template <int W>
__device__ __forceinline__ Vec<W> loadw(const void* base, long long idx, bool f32) {
  Vec<W> r;
  if constexpr (W == 4) {
    const float4 a = load4(base, idx, f32);
    r.v[0] = a.x; r.v[1] = a.y; r.v[2] = a.z; r.v[3] = a.w;
  } else if (f32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + idx);
    const float4 a = __ldcs(p), b = __ldcs(p + 1);
    r.v[0] = a.x; r.v[1] = a.y; r.v[2] = a.z; r.v[3] = a.w;
    r.v[4] = b.x; r.v[5] = b.y; r.v[6] = b.z; r.v[7] = b.w;
  } else {
    const uint4 u = __ldcs(reinterpret_cast<const uint4*>(
        static_cast<const __nv_bfloat16*>(base) + idx));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      __nv_bfloat162 h;
      std::memcpy(&h, &w[e], 4);
      const float2 f = __bfloat1622float2(h);
      r.v[2 * e] = f.x;
      r.v[2 * e + 1] = f.y;
    }
  }
  return r;
}
template <int W>
__device__ __forceinline__ void storew(void* base, long long idx, const Vec<W>& x, bool f32) {
  if constexpr (W == 4) {
    store4(base, idx, make_float4(x.v[0], x.v[1], x.v[2], x.v[3]), f32);
  } else if (f32) {
    float4* p = reinterpret_cast<float4*>(static_cast<float*>(base) + idx);
    __stcs(p, make_float4(x.v[0], x.v[1], x.v[2], x.v[3]));
    __stcs(p + 1, make_float4(x.v[4], x.v[5], x.v[6], x.v[7]));
  } else {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 h = __float22bfloat162_rn(make_float2(x.v[2 * e], x.v[2 * e + 1]));
      std::memcpy(&w[e], &h, 4);
    }
    __stcs(reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(base) + idx),
           make_uint4(w[0], w[1], w[2], w[3]));
  }
}

// One group of W elements per thread over a grid that covers the job (a memory-bound
// element-wise pass wants every SM full of threads, each with its loads in flight, rather
// than a few threads looping); blockIdx.y selects the job.  32-bit index arithmetic.
template <int W>
__device__ __forceinline__ void row_job_group(const RowJob& J, unsigned T, unsigned g) {
  const unsigned gpr = static_cast<unsigned>(J.d / W);
  const unsigned row = g / gpr, col = (g - row * gpr) * W;
  const unsigned bh = row / T, t = row - bh * T;
  const unsigned drow = J.flip ? bh * T + (T - 1 - t) : row;
  const long long si = static_cast<long long>(row) * J.d + col;
  const long long di = static_cast<long long>(drow) * J.d + col;
  Vec<W> a = loadw<W>(J.src, si, J.src_f32), b{}, c{}, x{};
  if (J.src2) b = loadw<W>(J.src2, si, J.src_f32);
  if (J.src3) c = loadw<W>(J.src3, si, J.src_f32);
  const bool dx = J.x && J.fm_x == LA_FM_ELU1;
  if (dx) x = loadw<W>(J.x, di, J.x_f32);
  const float r = J.rs ? J.rs[row] : 1.f;
#pragma unroll
  for (int e = 0; e < W; ++e) {
    float v = a.v[e];
    if (J.src2) v += b.v[e];
    if (J.fm_src == LA_FM_ELU1) v = psi(v, 1);
    v *= r;
    if (J.src3) v += c.v[e];
    if (dx) v *= psi_prime(x.v[e], 1);
    a.v[e] = v;
    if (J.lo) b.v[e] = v - __bfloat162float(__float2bfloat16_rn(v));
  }
  storew<W>(J.dst, di, a, J.dst_f32);
  if (J.lo) storew<W>(J.dst2, di, b, J.dst_f32);
}

__global__ void __launch_bounds__(256) row_jobs(RowJobs jobs, unsigned T, unsigned rows) {
  const RowJob& J = jobs.j[blockIdx.y];
  const unsigned g = blockIdx.x * blockDim.x + threadIdx.x;
  if (J.d % 8 == 0) {
    if (g < rows * static_cast<unsigned>(J.d / 8)) row_job_group<8>(J, T, g);
  } else if (g < rows * static_cast<unsigned>(J.d / 4)) {
    row_job_group<4>(J, T, g);
  }
}

// ---------------------------------------------------------------------------------------
// Decayed vector scans of the normalised form's gradient: y_t = gamma y_{t-1} + x_t over the
// tokens of each (b, h) in scan order (t = 0 .. T-1, or T-1 .. 0 in reverse), x_t a
// d-vector (d <= 128):
//   mode 0 (forward)  x_t = psi(k_t), with gamma Z_init folded into the first element: y_t
//                     is the normaliser Z_t.  Per token the walk forms the denominator
//                     d_t = psi(q_t) . Z_t + eps, and from A_t = S_t do_t (the grad_q
//                     pass's output, computed before the walk): do_t . n_t = psi(q_t) . A_t,
//                     dd_t = -(do_t . n_t) / d_t^2, grad_q_t = psi'(q_t) (A_t / d_t +
//                     dd_t Z_t), 1 / d_t and dn_t = do_t / d_t (the grad_v pass's value).
//   mode 1 (reverse)  x_t = dd_t psi(q_t), with grad_Z_final folded into the first
//                     element (token T-1, no decay): y_t is g_t, part of dpsi(k_t); the
//                     walk writes it and grad_Z_init = gamma g_0.
// Three launches: each segment's decayed total (one warp per segment of Ls tokens), the
// exclusive scan over segments (one thread per (b, h, feature)), and the walk from each
// segment's prefix.  Lane l holds features 4l .. 4l + 3.
struct VecScan {
  int BH, H;
  long long T;
  int d, dv;        // features of x (dk) and of do / o / dn (dv)
  int Ls, NS;       // tokens per segment, segments per (b, h)
  int mode;         // 0 or 1 (see above)
  int fm;
  bool in_f32;      // q, k, grad_out (and dn) are float32, else bf16
  const void* x;    // k (mode 0) or q (mode 1)
  const void* q;    // mode 0: psi(q) for the denominator
  const void* dout;       // mode 0
  const float* A;         // mode 0: S_t do_t [BH, T, d], and its lo pass (or nullptr)
  const float* A_lo;
  void* grad_q;           // mode 0: [BH, T, d], float32 or bf16
  bool gq_f32;
  float eps;
  const float* init;      // Z_init (mode 0) or grad_Z_final (mode 1), [BH, d], or nullptr
  float* tot;             // [BH, NS, d]: segment totals, then exclusive prefixes
  float* dd;              // [BH, T]: written by mode 0, read by mode 1
  float* inv_den;         // mode 0: [BH, T], 1 / d_t
  void* dn;               // mode 0: [BH, T, dv] in the input type
  void* dn_lo;            // mode 0: bf16 inputs: the residual dn - bf16(dn), else nullptr
  bool dn_rev;            // mode 0: write dn's rows in reversed order
  float* y_out;           // mode 1: g_t [BH, T, d]
  bool y_rev;             // mode 1: write row T-1-t instead of t
  float* init_grad;       // mode 1: grad_Z_init [BH, d] or nullptr
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// x_t for this lane's four features; `pos` is the scan position of token t.
__device__ __forceinline__ float4 vs_x(const VecScan& p, long long bh, long long t, long long pos,
                                       int col, float g) {
  float4 a = load4(p.x, (bh * p.T + t) * p.d + col, p.in_f32);
  a = make_float4(psi(a.x, p.fm), psi(a.y, p.fm), psi(a.z, p.fm), psi(a.w, p.fm));
  if (p.mode == 1) {
    const float w = p.dd[bh * p.T + t];
    a = make_float4(a.x * w, a.y * w, a.z * w, a.w * w);
  }
  if (pos == 0 && p.init) {
    const float4 z = *reinterpret_cast<const float4*>(p.init + bh * p.d + col);
    const float w = p.mode == 0 ? g : 1.f;
    a = make_float4(fmaf(w, z.x, a.x), fmaf(w, z.y, a.y), fmaf(w, z.z, a.z), fmaf(w, z.w, a.w));
  }
  return a;
}

__global__ void __launch_bounds__(128) vs_totals(VecScan p, GammaTable gt) {
  const long long wid = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= static_cast<long long>(p.BH) * p.NS) return;
  const long long bh = wid / p.NS;
  const int seg = static_cast<int>(wid - bh * p.NS);
  const float g = gt.g[bh % p.H];
  const int col = 4 * lane;
  if (col >= p.d) return;
  const long long p0 = static_cast<long long>(seg) * p.Ls, p1 = min(p.T, p0 + p.Ls);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (long long pos = p0; pos < p1; ++pos) {
    const long long t = p.mode == 1 ? p.T - 1 - pos : pos;
    const float4 x = vs_x(p, bh, t, pos, col, g);
    acc = make_float4(fmaf(g, acc.x, x.x), fmaf(g, acc.y, x.y), fmaf(g, acc.z, x.z),
                      fmaf(g, acc.w, x.w));
  }
  *reinterpret_cast<float4*>(p.tot + (bh * p.NS + seg) * p.d + col) = acc;
}

// Exclusive prefixes of the segment totals: one warp per (b, h) and four features, lane i
// holding segment s0 + i of a block of 32; a decayed Hillis-Steele scan in registers
// (every segment but the last spans Ls tokens, so each step's decay is gamma^(Ls * off)),
// the block's total carried into the next block.
__global__ void __launch_bounds__(128) vs_prefix(VecScan p, GammaTable gt) {
  const long long wid = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int groups = (p.d + 3) / 4;
  if (wid >= static_cast<long long>(p.BH) * groups) return;
  const long long bh = wid / groups;
  const int col = 4 * static_cast<int>(wid - bh * groups);
  const float g = gt.g[bh % p.H];
  const float aL = powf(g, static_cast<float>(p.Ls));
  float4 carry = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < p.NS; s0 += 32) {
    const int sg = s0 + lane;
    float4* e = reinterpret_cast<float4*>(p.tot + (bh * p.NS + sg) * p.d + col);
    float4 x = sg < p.NS ? *e : make_float4(0.f, 0.f, 0.f, 0.f);
    float a = aL;  // gamma^(Ls * off)
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float4 y = make_float4(__shfl_up_sync(0xffffffffu, x.x, off),
                                   __shfl_up_sync(0xffffffffu, x.y, off),
                                   __shfl_up_sync(0xffffffffu, x.z, off),
                                   __shfl_up_sync(0xffffffffu, x.w, off));
      if (lane >= off)
        x = make_float4(fmaf(a, y.x, x.x), fmaf(a, y.y, x.y), fmaf(a, y.z, x.z), fmaf(a, y.w, x.w));
      a *= a;
    }
    // Inclusive over the block from the carry: x + aL^(lane + 1) carry; exclusive: the
    // previous lane's, or the carry itself for lane 0.
    const float w = powf(aL, static_cast<float>(lane + 1));
    const float4 inc = make_float4(fmaf(w, carry.x, x.x), fmaf(w, carry.y, x.y),
                                   fmaf(w, carry.z, x.z), fmaf(w, carry.w, x.w));
    float4 exc = make_float4(__shfl_up_sync(0xffffffffu, inc.x, 1),
                             __shfl_up_sync(0xffffffffu, inc.y, 1),
                             __shfl_up_sync(0xffffffffu, inc.z, 1),
                             __shfl_up_sync(0xffffffffu, inc.w, 1));
    if (lane == 0) exc = carry;
    if (sg < p.NS) *e = exc;
    carry = make_float4(__shfl_sync(0xffffffffu, inc.x, 31), __shfl_sync(0xffffffffu, inc.y, 31),
                        __shfl_sync(0xffffffffu, inc.z, 31), __shfl_sync(0xffffffffu, inc.w, 31));
  }
}

__global__ void __launch_bounds__(128) vs_walk(VecScan p, GammaTable gt) {
  const long long wid = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= static_cast<long long>(p.BH) * p.NS) return;
  const long long bh = wid / p.NS;
  const int seg = static_cast<int>(wid - bh * p.NS);
  const float g = gt.g[bh % p.H];
  const int col = 4 * lane, vcol = 4 * lane;
  const bool fx = col < p.d, fv = vcol < p.dv;
  const long long p0 = static_cast<long long>(seg) * p.Ls, p1 = min(p.T, p0 + p.Ls);
  float4 acc = fx ? *reinterpret_cast<const float4*>(p.tot + (bh * p.NS + seg) * p.d + col)
                  : make_float4(0.f, 0.f, 0.f, 0.f);
  for (long long pos = p0; pos < p1; ++pos) {
    const long long t = p.mode == 1 ? p.T - 1 - pos : pos;
    const long long row = bh * p.T + t;
    if (fx) {
      const float4 x = vs_x(p, bh, t, pos, col, g);
      acc = make_float4(fmaf(g, acc.x, x.x), fmaf(g, acc.y, x.y), fmaf(g, acc.z, x.z),
                        fmaf(g, acc.w, x.w));
    }
    if (p.mode == 0) {
      float part = 0.f, part_n = 0.f;
      float4 xq = make_float4(0.f, 0.f, 0.f, 0.f), A = xq;
      if (fx) {
        xq = load4(p.q, row * p.d + col, p.in_f32);
        const float4 fq = make_float4(psi(xq.x, p.fm), psi(xq.y, p.fm), psi(xq.z, p.fm),
                                      psi(xq.w, p.fm));
        A = __ldcs(reinterpret_cast<const float4*>(p.A + row * p.d + col));
        if (p.A_lo) {
          const float4 b = __ldcs(reinterpret_cast<const float4*>(p.A_lo + row * p.d + col));
          A = make_float4(A.x + b.x, A.y + b.y, A.z + b.z, A.w + b.w);
        }
        part = fq.x * acc.x + fq.y * acc.y + fq.z * acc.z + fq.w * acc.w;
        part_n = fq.x * A.x + fq.y * A.y + fq.z * A.z + fq.w * A.w;
      }
      const float den = warp_sum(part) + p.eps;
      const float r = 1.f / den;
      const float ddt = -warp_sum(part_n) * r * r;
      float4 dov = make_float4(0.f, 0.f, 0.f, 0.f);
      if (fv) dov = load4(p.dout, row * p.dv + vcol, p.in_f32);
      if (fv) {
        const float4 dn = make_float4(dov.x * r, dov.y * r, dov.z * r, dov.w * r);
        const long long drow = p.dn_rev ? bh * p.T + (p.T - 1 - t) : row;
        store4(p.dn, drow * p.dv + vcol, dn, p.in_f32);
        if (p.dn_lo) {
          auto rest = [](float x) { return x - __bfloat162float(__float2bfloat16_rn(x)); };
          store4(p.dn_lo, drow * p.dv + vcol,
                 make_float4(rest(dn.x), rest(dn.y), rest(dn.z), rest(dn.w)), false);
        }
      }
      if (lane == 0) {
        p.dd[row] = ddt;
        p.inv_den[row] = r;
      }
      if (fx) {  // dpsi(q_t) = A_t / d_t + dd_t Z_t, times psi'(q_t)
        const float4 gq = make_float4(fmaf(A.x, r, ddt * acc.x) * psi_prime(xq.x, p.fm),
                                      fmaf(A.y, r, ddt * acc.y) * psi_prime(xq.y, p.fm),
                                      fmaf(A.z, r, ddt * acc.z) * psi_prime(xq.z, p.fm),
                                      fmaf(A.w, r, ddt * acc.w) * psi_prime(xq.w, p.fm));
        store4(p.grad_q, row * p.d + col, gq, p.gq_f32);
      }
    } else if (fx) {
      const long long wrow = p.y_rev ? bh * p.T + (p.T - 1 - t) : row;
      __stcs(reinterpret_cast<float4*>(p.y_out + wrow * p.d + col), acc);
    }
  }
  if (p.mode == 1 && p.init_grad && fx && p1 == p.T && p0 < p1)  // the segment ending at token 0
    *reinterpret_cast<float4*>(p.init_grad + bh * p.d + col) =
        make_float4(g * acc.x, g * acc.y, g * acc.z, g * acc.w);
}

cudaError_t launch_vec_scan(const VecScan& p, const GammaTable& gt, cudaStream_t s) {
  const long long warps = static_cast<long long>(p.BH) * p.NS;
  const unsigned wb = static_cast<unsigned>((warps + 3) / 4);
  vs_totals<<<wb, 128, 0, s>>>(p, gt);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long pw = static_cast<long long>(p.BH) * ((p.d + 3) / 4);  // warps
  vs_prefix<<<static_cast<unsigned>((pw + 3) / 4), 128, 0, s>>>(p, gt);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  vs_walk<<<wb, 128, 0, s>>>(p, gt);
  return cudaGetLastError();
}

// dst[bh] = scale_h * (transpose ? src[bh]^T : src[bh]) for [rows x cols] float32
// matrices (dst is rows x cols; src is cols x rows when transposing).  scale_h is 1 / gamma_h
// (0 for heads below kSmallDecay) when `inverse_decay`, else 1.
__global__ void prep_state(const float* __restrict__ src, float* __restrict__ dst, int rows,
                           int cols, bool transpose, bool inverse_decay, int H, long long n,
                           GammaTable gt) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= n) return;
  const long long per = static_cast<long long>(rows) * cols;
  const long long bh = idx / per;
  const int e = static_cast<int>(idx - bh * per), r = e / cols, c = e - r * cols;
  float s = 1.f;
  if (inverse_decay) {
    const float g = gt.g[bh % H];
    s = g >= kSmallDecay ? 1.f / g : 0.f;
  }
  dst[idx] = s * src[bh * per + (transpose ? static_cast<long long>(c) * rows + r : e)];
}

// dS_init = gamma_h * G_0 (+ gamma_h^T dS_final for heads below kSmallDecay, whose G_0 lacks
// the dS_final term), in place on G_0.
__global__ void finish_state(float* __restrict__ G0, const float* __restrict__ dS_final, int per,
                             int H, long long n, long long T, GammaTable gt) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= n) return;
  const float g = gt.g[(idx / per) % H];
  float x = g * G0[idx];
  if (dS_final && g < kSmallDecay) {
    // gamma^T with T >= 1; for gamma = 0 only T = 0 would survive, and T = 0 never runs.
    const float gT = T == 1 ? g : (g == 0.f ? 0.f : exp2f(static_cast<float>(T) * log2f(g)));
    x = fmaf(gT, dS_final[idx], x);
  }
  G0[idx] = x;
}

// For heads below kSmallDecay: the terms gamma^sigma dS_final v and gamma^sigma
// dS_final^T psi(k) of the reversed rows sigma < 3 (tokens T-1-sigma), added to the
// float32 outputs of the reversed passes (Wk: dpsi(k) [T, dk]; Wv: dv [T, dv]; rows in
// reversed order unless `in_order`).  One block per (b, h); threads cover the dk + dv
// output columns.
__global__ void fix_small_decay(const float* __restrict__ dS_final, const void* k,
                                const void* v, float* __restrict__ Wk, float* __restrict__ Wv,
                                int dk, int dv, int H, long long T, int fm, bool in_f32,
                                bool in_order, GammaTable gt) {
  const long long bh = blockIdx.x;
  const float g = gt.g[bh % H];
  if (g >= kSmallDecay) return;
  const float* dS = dS_final + bh * dk * dv;
  float w = 1.f;
  for (int sg = 0; sg < kSmallDecayTerms && sg < T; ++sg) {
    const long long t = bh * T + (T - 1 - sg);  // the original row of reversed row sg
    const long long w_row = in_order ? t : bh * T + sg;  // its row in Wk / Wv
    for (int c = threadIdx.x; c < dk + dv; c += blockDim.x) {
      float acc = 0.f;
      if (c < dk) {  // (dS v_t)_c
        for (int j = 0; j < dv; ++j) {
          const long long e = t * dv + j;
          const float vj = in_f32 ? static_cast<const float*>(v)[e]
                                  : __bfloat162float(static_cast<const __nv_bfloat16*>(v)[e]);
          acc = fmaf(dS[c * dv + j], vj, acc);
        }
        Wk[w_row * dk + c] += w * acc;
      } else {  // (dS^T psi(k_t))_j
        const int j = c - dk;
        for (int i = 0; i < dk; ++i) {
          const long long e = t * dk + i;
          const float ki = in_f32 ? static_cast<const float*>(k)[e]
                                  : __bfloat162float(static_cast<const __nv_bfloat16*>(k)[e]);
          acc = fmaf(dS[i * dv + j], psi(ki, fm), acc);
        }
        Wv[w_row * dv + j] += w * acc;
      }
    }
    w *= g;
  }
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, size_t an, const void* b, size_t bn) {
  if (!a || !b || an == 0 || bn == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + bn && b0 < a0 + an;
}

bool has_small_decay(const la_backward_args& a) {
  if (!a.gamma || !a.grad_S_final) return false;
  for (int h = 0; h < a.H; ++h)
    if (a.gamma[h] < kSmallDecay) return true;
  return false;
}

// Segments of the normaliser scans: about 32 warps per SM in all, at least 64 tokens each.
void vec_segments(size_t BH, size_t T, int* Ls, int* NS) {
  if (BH == 0 || T == 0) {
    *Ls = 1;
    *NS = 0;
    return;
  }
  const size_t want = std::max<size_t>(1, (148 * 32 + BH - 1) / BH);
  const size_t most = (T + 63) / 64;
  const size_t ns = std::min(want, most);
  const size_t ls = (T + ns - 1) / ns;
  *Ls = static_cast<int>(ls);
  *NS = static_cast<int>((T + ls - 1) / ls);
}

// Whether the two reversed passes run on the segmented kernels in reverse mode (reading
// the inputs and writing the outputs in memory order) rather than on reversed copies.  A
// pure function of the arguments: bf16 inputs, C = 64, dk = dv = 128, a tensor-core
// algorithm that may be segmented, and not ELU+1 with a decay (whose model-map pass has no
// segmented kernel).
bool native_reverse(const la_backward_args& a) {
  return a.dtype == LA_DTYPE_BF16 && a.C == 64 && a.dk == 128 && a.dv == 128 &&
         a.algorithm != LA_ALGO_CHUNKED && a.kernel_path != LA_PATH_FMA &&
         !(a.feature_map == LA_FM_ELU1 && a.gamma != nullptr) && a.T < (1LL << 31);
}

// Workspace of one backward call.
//   Reversed copies (only without native reverse), type `dtype`: kr, qr [T, dk], dor,
//   vr [T, dv].
//   ELU+1: psi(q) for the dpsi(k) pass (reversed without native reverse) and psi(k) in
//   order [T, dk], each with its bf16 residual (lo) when the inputs are bf16.
//   Outputs of the reversed passes Wk [T, dk], Wv [T, dv] where they cannot go straight to
//   grad_k / grad_v: always without native reverse (float32 when multiplied by psi' or
//   corrected, else the output type); with it, float32 and only where psi', the
//   small-decay terms or the normalised form's lo pass still apply.  ELU+1: the grad_q
//   pass's float32 output Wq [T, dk] and the lo passes' float32 outputs.
//   Three [dk x dv] states per (b, h), then the prefill workspace.
struct BwdLayout {
  size_t kr, qr, dor, vr, pq, pk, pq_lo, pk_lo, Wk, Wv, Wq, Wk_lo, Wq_lo, SA, SB, SC;
  size_t dn, dn_lo, Wv_lo, dd, inv_den, Wkg, vtot, pw, total;
  int Ls, NS;  // the normaliser scans' segments
  bool native, elu, split, fix, wk, wv, w_f32, norm;
};

BwdLayout bwd_layout(const la_backward_args& a) {
  BwdLayout l{};
  const size_t BH = static_cast<size_t>(a.B > 0 ? a.B : 0) * (a.H > 0 ? a.H : 0);
  const size_t T = static_cast<size_t>(a.T > 0 ? a.T : 0);
  const size_t e = a.dtype == LA_DTYPE_F32 ? 4 : 2;
  const bool out_f32 = a.dtype == LA_DTYPE_F32 || a.out_dtype == LA_OUT_F32;
  l.native = native_reverse(a);
  l.norm = a.normalize != 0;
  l.elu = a.feature_map == LA_FM_ELU1;
  l.split = l.elu && a.dtype == LA_DTYPE_BF16;
  l.fix = has_small_decay(a);
  l.wk = !l.native || l.elu || l.fix;
  l.wv = !l.native || l.fix || a.normalize;
  l.w_f32 = l.native || out_f32 || l.elu || l.fix;
  const size_t ew = l.w_f32 ? 4 : 2;
  const size_t nk = BH * T * a.dk, nv = BH * T * a.dv, ns = BH * a.dk * a.dv * 4;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  const bool flip = !l.native;
  l.kr = take(flip ? nk * e : 0);
  l.qr = take(flip ? nk * e : 0);
  l.dor = take(flip ? nv * e : 0);
  l.vr = take(flip ? nv * e : 0);
  l.pq = take(l.elu ? nk * e : 0);
  l.pk = take(l.elu ? nk * e : 0);
  l.pq_lo = take(l.split ? nk * e : 0);
  l.pk_lo = take(l.split ? nk * e : 0);
  l.Wk = take(l.wk ? nk * ew : 0);
  l.Wv = take(l.wv ? nv * ew : 0);
  l.Wq = take(l.elu ? nk * 4 : 0);
  l.Wk_lo = take(l.split ? nk * 4 : 0);
  l.Wq_lo = take(l.split ? nk * 4 : 0);
  l.SA = take(a.S_init ? ns : 0);
  l.SB = take(a.grad_S_final ? ns : 0);
  l.SC = take(a.grad_S_final ? ns : 0);
  // The normalised form: dn = do / d as hi / lo (reversed without native reverse), the lo
  // pass's output of grad_v, dd, 1 / d, the g term of dpsi(k), and the scans' segment
  // records.
  vec_segments(BH, T, &l.Ls, &l.NS);
  l.dn = take(l.norm ? nv * e : 0);
  l.dn_lo = take(l.norm && l.split ? nv * e : 0);
  l.Wv_lo = take(l.norm && l.split ? nv * 4 : 0);
  l.dd = take(l.norm ? BH * T * 4 : 0);
  l.inv_den = take(l.norm ? BH * T * 4 : 0);
  l.Wkg = take(l.norm ? nk * 4 : 0);
  l.vtot = take(l.norm ? BH * static_cast<size_t>(l.NS) * a.dk * 4 : 0);
  l.pw = off;
  off += lin_attn_prefill_workspace_bytes(a.B, a.H, a.T, a.dk, a.dv, a.C, 0);
  l.total = off;
  return l;
}

// The prefill arguments of one pass; q, k, v, out and the states are filled in by the
// caller.
la_prefill_args pass_args(const la_backward_args& a, int dk, int dv, int fm, int out_dtype) {
  la_prefill_args p;
  std::memset(&p, 0, sizeof(p));
  p.B = a.B;
  p.H = a.H;
  p.T = a.T;
  p.dk = dk;
  p.dv = dv;
  p.C = a.C;
  p.feature_map = fm;
  p.gamma = a.gamma;
  p.normalize = 0;
  p.eps = 0.f;
  p.dtype = a.dtype;
  p.out_dtype = out_dtype;
  p.scan_mode = a.scan_mode;
  p.kernel_path = a.kernel_path;
  p.algorithm = a.algorithm;
  p.segment_chunks = a.segment_chunks;
  p.stream = a.stream;
  return p;
}

int validate(const la_backward_args& a) {
  if (a.B < 0 || a.H < 0 || a.T < 0 || a.dk <= 0 || a.dv <= 0 || a.C <= 0)
    return LA_ERR_INVALID_ARGUMENT;
  if (a.dtype != LA_DTYPE_BF16 && a.dtype != LA_DTYPE_F32) return LA_ERR_INVALID_ARGUMENT;
  if (a.out_dtype != LA_OUT_AS_INPUT && a.out_dtype != LA_OUT_F32) return LA_ERR_INVALID_ARGUMENT;
  if (a.feature_map != LA_FM_IDENTITY && a.feature_map != LA_FM_ELU1) return LA_ERR_INVALID_ARGUMENT;
  if (a.gamma && a.H > kMaxHeads) return LA_ERR_UNSUPPORTED;
  if (a.gamma)
    for (int h = 0; h < a.H; ++h)
      if (!(a.gamma[h] >= 0.f && a.gamma[h] <= 1.f)) return LA_ERR_INVALID_ARGUMENT;
  if (a.workspace && (reinterpret_cast<uintptr_t>(a.workspace) & 255u) != 0)
    return LA_ERR_INVALID_ARGUMENT;
  for (const void* p : {static_cast<const void*>(a.S_init), static_cast<const void*>(a.grad_S_final),
                        static_cast<const void*>(a.grad_S_init), static_cast<const void*>(a.Z_init),
                        static_cast<const void*>(a.grad_Z_final),
                        static_cast<const void*>(a.grad_Z_init)})
    if (!aligned16(p)) return LA_ERR_INVALID_ARGUMENT;
  if (a.normalize != 0 && a.normalize != 1) return LA_ERR_INVALID_ARGUMENT;
  if (a.normalize && a.feature_map != LA_FM_ELU1) return LA_ERR_INVALID_ARGUMENT;
  if (!(a.eps >= 0.f) || !std::isfinite(a.eps)) return LA_ERR_INVALID_ARGUMENT;
  // The three passes' shapes and options, checked as the prefill will check them (as
  // states-only calls, so that no output buffer is needed; q stands for every input).
  const long long BH = static_cast<long long>(a.B) * a.H;
  const bool empty = BH == 0 || a.T == 0;
  // The element-wise kernels index rows and groups of four elements in 32 bits.
  if (!empty && (BH * a.T >= (1LL << 31) || BH * a.T * (std::max(a.dk, a.dv) / 4) >= (1LL << 31)))
    return LA_ERR_UNSUPPORTED;
  const int fms[3] = {LA_FM_IDENTITY, a.feature_map, LA_FM_IDENTITY};
  const int dks[3] = {a.dv, a.dk, a.dv}, dvs[3] = {a.dk, a.dv, a.dk};
  const bool native = native_reverse(a);
  for (int i = 0; i < 3; ++i) {
    la_prefill_args p = pass_args(a, dks[i], dvs[i], fms[i], LA_OUT_F32);
    p.q = p.k = p.v = empty ? nullptr : a.q;
    p.states_only = 1;
    p.reverse = native && i > 0;
    const int st = check_prefill_args(p);
    if (st != LA_OK) return st;
  }
  if (!empty) {
    const void* in[4] = {a.q, a.k, a.v, a.grad_out};
    void* out[3] = {a.grad_q, a.grad_k, a.grad_v};
    for (const void* p : in)
      if (!p || !aligned16(p)) return LA_ERR_INVALID_ARGUMENT;
    for (const void* p : out)
      if (!p || !aligned16(p)) return LA_ERR_INVALID_ARGUMENT;
    const size_t e = a.dtype == LA_DTYPE_F32 ? 4 : 2;
    const size_t eo = (a.dtype == LA_DTYPE_F32 || a.out_dtype == LA_OUT_F32) ? 4 : 2;
    const size_t nk = static_cast<size_t>(BH) * a.T * a.dk, nv = static_cast<size_t>(BH) * a.T * a.dv;
    const size_t in_n[4] = {nk * e, nk * e, nv * e, nv * e};
    const size_t out_n[3] = {nk * eo, nk * eo, nv * eo};
    for (int o = 0; o < 3; ++o) {
      for (int i = 0; i < 4; ++i)
        if (overlaps(out[o], out_n[o], in[i], in_n[i])) return LA_ERR_INVALID_ARGUMENT;
      for (int o2 = o + 1; o2 < 3; ++o2)
        if (overlaps(out[o], out_n[o], out[o2], out_n[o2])) return LA_ERR_INVALID_ARGUMENT;
    }
  }
  return LA_OK;
}

cudaError_t launch_rows(const RowJobs& jobs, int n, long long BH, long long T, cudaStream_t s,
                        Recorder* rec, const char* name) {
  if (n == 0) return cudaSuccess;
  long long groups = 0;
  for (int i = 0; i < n; ++i)
    groups = std::max(groups, BH * T * (jobs.j[i].d / (jobs.j[i].d % 8 == 0 ? 8 : 4)));
  // The kernel indexes groups and elements' rows in 32 bits.
  if (groups >= (1LL << 31) || BH * T >= (1LL << 31)) return cudaErrorInvalidValue;
  const long long blocks = std::max(1LL, (groups + 255) / 256);
  if (rec) rec->mark(s, name);
  row_jobs<<<dim3(static_cast<unsigned>(blocks), n), 256, 0, s>>>(
      jobs, static_cast<unsigned>(T), static_cast<unsigned>(BH * T));
  return cudaGetLastError();
}

int backward(const la_backward_args& a, Recorder* rec = nullptr) {
  int st = validate(a);
  if (st != LA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(a.stream);
  const long long BH = static_cast<long long>(a.B) * a.H;
  if (BH == 0) return LA_OK;
  const size_t state_bytes = static_cast<size_t>(BH) * a.dk * a.dv * 4;
  if (a.T == 0) {
    // No tokens: S_final = S_init and Z_final = Z_init, so the gradients pass through.
    auto pass = [&](float* dst, const float* src, size_t bytes) {
      if (!dst) return cudaSuccess;
      return src ? cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, s)
                 : cudaMemsetAsync(dst, 0, bytes, s);
    };
    cudaError_t e = pass(a.grad_S_init, a.grad_S_final, state_bytes);
    if (e == cudaSuccess && a.normalize)
      e = pass(a.grad_Z_init, a.grad_Z_final, static_cast<size_t>(BH) * a.dk * 4);
    return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
  }

  GammaTable gt;
  for (int h = 0; h < kMaxHeads; ++h) gt.g[h] = 1.f;
  if (a.gamma)
    for (int h = 0; h < a.H; ++h) gt.g[h] = a.gamma[h];

  const BwdLayout l = bwd_layout(a);
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  bool owned = false;
  if (ws) {
    if (a.workspace_bytes < l.total) return LA_ERR_INVALID_ARGUMENT;
  } else {
    if (workspace_alloc(reinterpret_cast<void**>(&ws), l.total, s) != cudaSuccess) {
      cudaGetLastError();
      return LA_ERR_OUT_OF_MEMORY;
    }
    owned = true;
  }
  auto at = [&](size_t off) { return static_cast<void*>(ws + off); };
  const bool in_f32 = a.dtype == LA_DTYPE_F32;
  const bool out_f32 = in_f32 || a.out_dtype == LA_OUT_F32;
  const bool elu = a.feature_map == LA_FM_ELU1;
  const long long T = a.T;

  // Inputs of the passes: reversed copies unless the reversed passes run natively; for
  // ELU+1, psi(q) (reversed likewise) and psi(k) in order, as hi / lo pairs for bf16.
  auto job = [](RowJobs& J, int& n, const void* src, const void* src2, void* dst, const void* x,
                int d, int fm_src, int fm_x, bool flip, bool lo, bool sf, bool df, bool xf,
                const void* src3 = nullptr, const float* rs = nullptr, void* dst2 = nullptr) {
    J.j[n++] = RowJob{src, src2, src3, rs, dst, dst2, x, d, fm_src, fm_x, flip, lo, sf, df, xf};
  };
  RowJobs pre{};
  int np = 0;
  const bool f = in_f32, rv = !l.native;
  if (rv) {
    job(pre, np, a.k, nullptr, at(l.kr), nullptr, a.dk, LA_FM_IDENTITY, 0, true, false, f, f, f);
    job(pre, np, a.q, nullptr, at(l.qr), nullptr, a.dk, LA_FM_IDENTITY, 0, true, false, f, f, f);
    job(pre, np, a.grad_out, nullptr, at(l.dor), nullptr, a.dv, LA_FM_IDENTITY, 0, true, false,
        f, f, f);
    job(pre, np, a.v, nullptr, at(l.vr), nullptr, a.dv, LA_FM_IDENTITY, 0, true, false, f, f, f);
  }
  // (The normalised form's psi(q) is scaled by 1 / d_t, known only after its scan.)
  if (elu) {  // one job writes psi and, for bf16, its lo half
    const bool sp = l.split;
    if (!l.norm)
      job(pre, np, a.q, nullptr, at(l.pq), nullptr, a.dk, LA_FM_ELU1, 0, rv, sp, f, f, f,
          nullptr, nullptr, sp ? at(l.pq_lo) : nullptr);
    job(pre, np, a.k, nullptr, at(l.pk), nullptr, a.dk, LA_FM_ELU1, 0, false, sp, f, f, f,
        nullptr, nullptr, sp ? at(l.pk_lo) : nullptr);
  }
  cudaError_t e = launch_rows(pre, np, BH, T, s, rec, "bwd_reverse_inputs");

  // Initial states of the three passes.
  float* SA = a.S_init ? static_cast<float*>(at(l.SA)) : nullptr;
  float* SB = a.grad_S_final ? static_cast<float*>(at(l.SB)) : nullptr;
  float* SC = a.grad_S_final ? static_cast<float*>(at(l.SC)) : nullptr;
  const long long ns = BH * a.dk * a.dv;
  const unsigned sblocks = static_cast<unsigned>((ns + 255) / 256);
  if (rec && (SA || SB)) rec->mark(s, "bwd_prep_states");
  if (e == cudaSuccess && SA) {
    prep_state<<<sblocks, 256, 0, s>>>(a.S_init, SA, a.dv, a.dk, true, false, a.H, ns, gt);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess && SB) {
    prep_state<<<sblocks, 256, 0, s>>>(a.grad_S_final, SB, a.dk, a.dv, false, a.gamma != nullptr,
                                       a.H, ns, gt);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess && SC) {
    prep_state<<<sblocks, 256, 0, s>>>(a.grad_S_final, SC, a.dv, a.dk, true, a.gamma != nullptr,
                                       a.H, ns, gt);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) st = LA_ERR_CUDA;

  auto run = [&](la_prefill_args p) {
    if (st != LA_OK) return;
    p.workspace = at(l.pw);
    p.workspace_bytes = l.total - l.pw;
    const int r = prefill_with_args(p, rec, /*exact_prefix=*/true);
    if (r != LA_OK) st = r == LA_ERR_INVALID_ARGUMENT || r == LA_ERR_UNSUPPORTED ? LA_ERR_INTERNAL : r;
  };
  // grad_q (or, for ELU+1, dpsi(q) in float32): (do, v, psi(k)) in order, identity map;
  // linear in psi(k), so the lo half of a split psi(k) is a second pass from a zero state.
  {
    la_prefill_args p = pass_args(a, a.dv, a.dk, LA_FM_IDENTITY, elu ? LA_OUT_F32 : a.out_dtype);
    p.q = a.grad_out;
    p.k = a.v;
    p.v = elu ? at(l.pk) : a.k;
    p.out = elu ? at(l.Wq) : a.grad_q;
    p.S_init = SA;
    run(p);
    if (l.split) {
      p.v = at(l.pk_lo);
      p.out = at(l.Wq_lo);
      p.S_init = nullptr;
      run(p);
    }
  }
  // The normalised form: Z_t by a forward scan whose walk forms d_t, dd_t, dn_t and grad_q.
  // The two terms of dpsi(q_t) (A_t / d_t and Z_t dd_t) nearly cancel, and so do the two of
  // dpsi(k_s) (G_s v_s and g_s): both are sums of psi terms weighted by (v_s - o_t) . do_t
  // / d_t.  So nothing that meets such a cancellation passes through a bf16 rounding of
  // dn_t or of the output: the grad_q pass runs on do (A_t = S_t do_t) and the walk takes
  // do_t . n_t = psi(q_t) . A_t from it, both in float32; the dpsi(k) pass runs on do with
  // the value psi(q_t) / d_t (split hi / lo).  The grad_v pass takes dn_t as its value,
  // split into bf16 hi and lo: its largest entries come from the first tokens, where d_t
  // is small, and would carry dn's rounding whole.
  VecScan vs{};
  if (l.norm) {
    vs.BH = static_cast<int>(BH);
    vs.H = a.H;
    vs.T = T;
    vs.d = a.dk;
    vs.dv = a.dv;
    vs.Ls = l.Ls;
    vs.NS = l.NS;
    vs.fm = a.feature_map;
    vs.in_f32 = in_f32;
    vs.q = a.q;
    vs.dout = a.grad_out;
    vs.A = static_cast<const float*>(at(l.Wq));
    vs.A_lo = l.split ? static_cast<const float*>(at(l.Wq_lo)) : nullptr;
    vs.grad_q = a.grad_q;
    vs.gq_f32 = out_f32;
    vs.eps = a.eps;
    vs.tot = static_cast<float*>(at(l.vtot));
    vs.dd = static_cast<float*>(at(l.dd));
    vs.inv_den = static_cast<float*>(at(l.inv_den));
    vs.dn = at(l.dn);
    vs.dn_lo = l.split ? at(l.dn_lo) : nullptr;
    vs.dn_rev = rv;
    VecScan z = vs;
    z.mode = 0;
    z.x = a.k;
    z.init = a.Z_init;
    if (st == LA_OK && e == cudaSuccess) {
      if (rec) rec->mark(s, "bwd_z_scan");
      e = launch_vec_scan(z, gt, s);
      // psi(q_t) / d_t (reversed without native reverse), hi / lo for bf16.
      RowJobs pq{};
      int n = 0;
      const float* rs = static_cast<const float*>(at(l.inv_den));
      job(pq, n, a.q, nullptr, at(l.pq), nullptr, a.dk, LA_FM_ELU1, 0, rv, l.split, f, f, f,
          nullptr, rs, l.split ? at(l.pq_lo) : nullptr);
      if (e == cudaSuccess) e = launch_rows(pq, n, BH, T, s, rec, "bwd_scaled_psi_q");
      if (e != cudaSuccess) st = LA_ERR_CUDA;
    }
  }

  // grad_v: (k, q, do) in reverse time with the model's map; final state G_0.
  const int w_dtype = l.w_f32 ? LA_OUT_F32 : LA_OUT_AS_INPUT;
  {
    la_prefill_args p = pass_args(a, a.dk, a.dv, a.feature_map, l.wv ? w_dtype : a.out_dtype);
    p.reverse = l.native;
    p.q = rv ? at(l.kr) : a.k;
    p.k = rv ? at(l.qr) : a.q;
    p.v = l.norm ? at(l.dn) : (rv ? at(l.dor) : a.grad_out);
    p.out = l.wv ? at(l.Wv) : a.grad_v;
    p.S_init = SB;
    p.S_final = a.grad_S_init;
    run(p);
    if (l.norm && l.split) {  // the lo half of dn (linear in the value, from a zero state)
      p.v = at(l.dn_lo);
      p.out = at(l.Wv_lo);
      p.S_init = nullptr;
      p.S_final = nullptr;
      run(p);
    }
  }
  // dpsi(k): (v, do, psi(q)) in reverse time, identity map (lo half as for grad_q).
  {
    la_prefill_args p = pass_args(a, a.dv, a.dk, LA_FM_IDENTITY, l.wk ? w_dtype : a.out_dtype);
    p.reverse = l.native;
    p.q = rv ? at(l.vr) : a.v;
    p.k = rv ? at(l.dor) : a.grad_out;
    p.v = elu ? at(l.pq) : (rv ? at(l.qr) : a.q);
    p.out = l.wk ? at(l.Wk) : a.grad_k;
    p.S_init = SC;
    run(p);
    if (l.split) {
      p.v = at(l.pq_lo);
      p.out = at(l.Wk_lo);
      p.S_init = nullptr;
      run(p);
    }
  }
  e = cudaSuccess;
  // The normalised form: g_t = sum_{s >= t} gamma^(s-t) dd_s psi(q_s) (+ the final
  // normaliser's gradient), part of dpsi(k_t), by a reverse scan; grad_Z_init = gamma g_0.
  if (st == LA_OK && l.norm) {
    VecScan gs = vs;
    gs.mode = 1;
    gs.x = a.q;
    gs.init = a.grad_Z_final;
    gs.y_out = static_cast<float*>(at(l.Wkg));
    gs.y_rev = rv;
    gs.init_grad = a.grad_Z_init;
    if (rec) rec->mark(s, "bwd_g_scan");
    e = launch_vec_scan(gs, gt, s);
  }
  if (st == LA_OK && e == cudaSuccess && l.fix) {
    if (rec) rec->mark(s, "bwd_fix_small_decay");
    fix_small_decay<<<static_cast<unsigned>(BH), 128, 0, s>>>(
        a.grad_S_final, a.k, a.v, static_cast<float*>(at(l.Wk)), static_cast<float*>(at(l.Wv)),
        a.dk, a.dv, a.H, T, a.feature_map, in_f32, l.native, gt);
    e = cudaGetLastError();
  }
  if (st == LA_OK && e == cudaSuccess && a.grad_S_init && a.gamma) {
    if (rec) rec->mark(s, "bwd_finish_state");
    finish_state<<<sblocks, 256, 0, s>>>(a.grad_S_init, a.grad_S_final, a.dk * a.dv, a.H, ns, T,
                                         gt);
    e = cudaGetLastError();
  }
  // The gradients in forward time (reversed back unless the passes ran natively), with
  // psi' where the map has one.
  if (st == LA_OK && e == cudaSuccess) {
    RowJobs post{};
    int n = 0;
    const bool wf = l.w_f32;
    if (l.wv)
      job(post, n, at(l.Wv), l.norm && l.split ? at(l.Wv_lo) : nullptr, a.grad_v, nullptr, a.dv,
          LA_FM_IDENTITY, 0, rv, false, wf, out_f32, f);
    if (l.wk)
      job(post, n, at(l.Wk), l.split ? at(l.Wk_lo) : nullptr, a.grad_k, a.k, a.dk,
          LA_FM_IDENTITY, a.feature_map, rv, false, wf, out_f32, f,
          l.norm ? at(l.Wkg) : nullptr);
    if (elu && !l.norm)  // grad_q = psi'(q) .* dpsi(q) (the normalised walk wrote it)
      job(post, n, at(l.Wq), l.split ? at(l.Wq_lo) : nullptr, a.grad_q, a.q, a.dk,
          LA_FM_IDENTITY, a.feature_map, false, false, true, out_f32, f);
    e = launch_rows(post, n, BH, T, s, rec, "bwd_reverse_outputs");
  }
  if (rec) rec->mark(s);
  if (e != cudaSuccess && st == LA_OK) st = LA_ERR_CUDA;
  if (owned) {
    const cudaError_t e2 = cudaFreeAsync(ws, s);
    if (e2 != cudaSuccess && st == LA_OK) st = LA_ERR_CUDA;
  }
  return st;
}

}  // namespace
}  // namespace la

extern "C" int lin_attn_backward(const la_backward_args* args) {
  if (!args) return LA_ERR_INVALID_ARGUMENT;
  return la::backward(*args);
}

extern "C" int lin_attn_backward_timed(const la_backward_args* args, float* kernel_ms,
                                       const char** kernel_names, int max_kernels,
                                       int* n_kernels) {
  if (!args || !kernel_ms || !kernel_names || !n_kernels || max_kernels < 1)
    return LA_ERR_INVALID_ARGUMENT;
  *n_kernels = 0;
  constexpr int kMaxEvents = 48;
  cudaEvent_t ev[kMaxEvents];
  const char* label[kMaxEvents] = {nullptr};
  int created = 0;
  for (; created < kMaxEvents; ++created)
    if (cudaEventCreate(&ev[created]) != cudaSuccess) break;
  if (created < kMaxEvents) {
    for (int i = 0; i < created; ++i) cudaEventDestroy(ev[i]);
    return LA_ERR_CUDA;
  }
  la::Recorder rec;
  rec.ev = ev;
  rec.label = label;
  rec.cap = kMaxEvents;
  int st = la::backward(*args, &rec);
  if (st == LA_OK && cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(args->stream)) !=
                         cudaSuccess)
    st = LA_ERR_CUDA;
  if (st == LA_OK) {
    int nk = 0;
    for (int i = 0; i + 1 < rec.n && nk < max_kernels; ++i) {
      if (!label[i]) continue;  // the gap between two passes
      float ms = 0.f;
      cudaEventElapsedTime(&ms, ev[i], ev[i + 1]);
      kernel_ms[nk] = ms;
      kernel_names[nk] = label[i];
      ++nk;
    }
    *n_kernels = nk;
  }
  for (int i = 0; i < kMaxEvents; ++i) cudaEventDestroy(ev[i]);
  return st;
}

extern "C" size_t lin_attn_backward_workspace_bytes(const la_backward_args* args) {
  if (!args || args->B <= 0 || args->H <= 0 || args->T <= 0) return 0;
  return la::bwd_layout(*args).total;
}
