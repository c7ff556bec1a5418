// C ABI of the library: argument validation, workspace layout, TMA tensor maps, and the
// K1 -> K2 -> K3 launch sequence on the caller's stream.  See include/linattn.h for the
// contract of every entry point.

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/linattn.h"
#include "common.cuh"
#include "launch.h"

namespace la {

// Device error word; every kernel receives its address.
__device__ int g_error_word = 0;

namespace {

constexpr int kVersion = 1 * 10000 + 1 * 100 + 0;

struct Layout {
  long long BH = 0;
  int NC = 0, L_last = 0, R = 0, Ls = 1, G = 1;
  size_t rec_off = 0, rec_bytes = 0, tot_off = 0, tot_bytes = 0, total = 0;
};

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

Layout make_layout(int B, int H, long long T, int dk, int dv, int C, int normalize) {
  Layout l;
  l.BH = static_cast<long long>(B) * H;
  if (l.BH <= 0 || T <= 0 || C <= 0) return l;
  const long long nc = (T + C - 1) / C;
  l.NC = static_cast<int>(nc);
  l.L_last = static_cast<int>(T - (nc - 1) * C);
  l.R = dk * dv + (normalize ? dk : 0);
  const ScanPlan sp = scan_plan(nc);
  l.Ls = sp.Ls;
  l.G = sp.G;
  l.rec_off = 0;
  l.rec_bytes = align256(static_cast<size_t>(l.BH) * nc * l.R * sizeof(float));
  l.tot_off = l.rec_off + l.rec_bytes;
  // Segment folds of the two-level scan.  Sized for min(2048, ceil(NC / 16)) segments, a
  // bound on the segment count of any scan of at most NC elements, so that the segmented
  // algorithm's scan over its (fewer) segment records fits in the same space.
  const long long gmax = nc > kScanBlockElems
                             ? std::min<long long>(kScanBlockElems, (nc + kScanMinSegment - 1) / kScanMinSegment)
                             : 0;
  l.tot_bytes = align256(static_cast<size_t>(l.BH) * gmax * l.R * sizeof(float));
  l.total = l.tot_off + l.tot_bytes;
  return l;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, size_t an, const void* b, size_t bn) {
  if (!a || !b || an == 0 || bn == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + bn && b0 < a0 + an;
}

bool dim_ok_fma(int d) { return d >= 4 && d <= 128 && d % 4 == 0; }
bool chunk_ok_fma(int C) { return C == 16 || C == 32 || C == 64; }
bool dim_ok_tc(int d) { return d == 64 || d == 128; }

// Address of the device error word on the current device.  Looked up on every call and
// not cached: after cudaDeviceReset the module is loaded again and the word may move.
int* error_word_ptr() {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_error_word) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return static_cast<int*>(ptr);
}

bool device_is_sm100() {
  static std::mutex mu;
  static int cache[64] = {0};  // 0 unknown, 1 yes, 2 no
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == 0) {
    int major = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cache[dev] = major == 10 ? 1 : 2;
  }
  return cache[dev] == 1;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// A 3D tiled map (d0 innermost) with the 128-byte swizzle and zero fill out of bounds.
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1,
              uint64_t d2, uint64_t stride1, uint64_t stride2, uint32_t box0, uint32_t box1) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {stride1, stride2};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int check_gamma(const float* gamma, int H, GammaTable* gt) {
  for (int h = 0; h < kMaxHeads; ++h) gt->g[h] = 1.f;
  if (!gamma) return LA_OK;
  if (H > kMaxHeads) return LA_ERR_UNSUPPORTED;
  for (int h = 0; h < H; ++h) {
    const float g = gamma[h];
    if (!(g >= 0.f && g <= 1.f)) return LA_ERR_INVALID_ARGUMENT;  // also rejects NaN
    gt->g[h] = g;
  }
  return LA_OK;
}

enum class Path { kFma, kTensorCore, kSegmented };

// Validates `a` and picks the kernel path.  Touches no CUDA state except the device
// capability query, which happens only for non-empty problems.
int validate(const la_prefill_args& a, Path* path) {
  if (a.B < 0 || a.H < 0 || a.T < 0 || a.dk <= 0 || a.dv <= 0 || a.C <= 0)
    return LA_ERR_INVALID_ARGUMENT;
  if (a.dtype != LA_DTYPE_BF16 && a.dtype != LA_DTYPE_F32) return LA_ERR_INVALID_ARGUMENT;
  if (a.feature_map != LA_FM_IDENTITY && a.feature_map != LA_FM_ELU1) return LA_ERR_INVALID_ARGUMENT;
  if (a.scan_mode != LA_SCAN_LOGDEPTH && a.scan_mode != LA_SCAN_SEQUENTIAL)
    return LA_ERR_INVALID_ARGUMENT;
  if (a.kernel_path < LA_PATH_AUTO || a.kernel_path > LA_PATH_FMA) return LA_ERR_INVALID_ARGUMENT;
  if (a.out_dtype != LA_OUT_AS_INPUT && a.out_dtype != LA_OUT_F32) return LA_ERR_INVALID_ARGUMENT;
  if (a.algorithm < LA_ALGO_AUTO || a.algorithm > LA_ALGO_SEGMENTED) return LA_ERR_INVALID_ARGUMENT;
  if (a.segment_chunks < 0 || a.segment_chunks > 1024) return LA_ERR_INVALID_ARGUMENT;
  if (a.states_only != 0 && a.states_only != 1) return LA_ERR_INVALID_ARGUMENT;
  if (a.reverse != 0 && a.reverse != 1) return LA_ERR_INVALID_ARGUMENT;
  if ((reinterpret_cast<uintptr_t>(a.S_init) & 3u) || (reinterpret_cast<uintptr_t>(a.Z_init) & 3u))
    return LA_ERR_INVALID_ARGUMENT;
  if (a.normalize && a.feature_map == LA_FM_IDENTITY) return LA_ERR_INVALID_ARGUMENT;
  if (!(a.eps >= 0.f) || !std::isfinite(a.eps)) return LA_ERR_INVALID_ARGUMENT;
  if (a.gamma && a.H > kMaxHeads) return LA_ERR_UNSUPPORTED;

  if (!dim_ok_fma(a.dk) || !dim_ok_fma(a.dv) || !chunk_ok_fma(a.C)) return LA_ERR_UNSUPPORTED;
  const long long BH = static_cast<long long>(a.B) * a.H;
  const long long NC = a.T > 0 ? (a.T + a.C - 1) / a.C : 0;
  if (BH > (1LL << 31) - 1 || BH * NC > (1LL << 31) - 1) return LA_ERR_UNSUPPORTED;
  const int dmax = a.dk > a.dv ? a.dk : a.dv;
  if (BH > 0 && a.T > 0 && BH * a.T > (1LL << 62) / dmax) return LA_ERR_UNSUPPORTED;

  const bool tc_shape = a.dtype == LA_DTYPE_BF16 && dim_ok_tc(a.dk) && dim_ok_tc(a.dv) &&
                        a.C == 64 && a.T < (1LL << 31);
  if (a.kernel_path == LA_PATH_TENSOR_CORE && !tc_shape) return LA_ERR_UNSUPPORTED;
  const bool seg_ok = seg_supported(a.dk, a.dv, a.C, a.feature_map, a.gamma != nullptr);
  if (a.algorithm == LA_ALGO_SEGMENTED && (!tc_shape || a.kernel_path == LA_PATH_FMA || !seg_ok))
    return LA_ERR_UNSUPPORTED;

  const bool empty = BH == 0 || a.T == 0;
  if (!empty) {
    const bool want_out = !a.states_only;
    if (!a.q || !a.k || !a.v || (want_out && !a.out)) return LA_ERR_INVALID_ARGUMENT;
    if (!aligned16(a.q) || !aligned16(a.k) || !aligned16(a.v) || (a.out && !aligned16(a.out)))
      return LA_ERR_INVALID_ARGUMENT;
    const size_t e = a.dtype == LA_DTYPE_F32 ? 4 : 2;
    const size_t eo = (a.dtype == LA_DTYPE_F32 || a.out_dtype == LA_OUT_F32) ? 4 : 2;
    const size_t nq = static_cast<size_t>(BH) * a.T * a.dk * e;
    const size_t nv = static_cast<size_t>(BH) * a.T * a.dv * e;
    const size_t no = static_cast<size_t>(BH) * a.T * a.dv * eo;
    if (a.out && (overlaps(a.out, no, a.q, nq) || overlaps(a.out, no, a.k, nq) ||
                  overlaps(a.out, no, a.v, nv)))
      return LA_ERR_INVALID_ARGUMENT;
  }
  if ((a.S_final && !aligned16(a.S_final)) || (a.Z_final && !aligned16(a.Z_final)))
    return LA_ERR_INVALID_ARGUMENT;
  if (a.workspace && (reinterpret_cast<uintptr_t>(a.workspace) & 255u) != 0)
    return LA_ERR_INVALID_ARGUMENT;

  *path = Path::kFma;
  if (!empty && a.kernel_path != LA_PATH_FMA && tc_shape) {
    if (device_is_sm100()) {
      *path = Path::kTensorCore;
    } else if (a.kernel_path == LA_PATH_TENSOR_CORE || a.algorithm == LA_ALGO_SEGMENTED) {
      return LA_ERR_UNSUPPORTED;
    }
  }
  if (*path == Path::kTensorCore && a.algorithm != LA_ALGO_CHUNKED && seg_ok)
    *path = Path::kSegmented;
  if (a.reverse && !empty && *path != Path::kSegmented) return LA_ERR_UNSUPPORTED;
  return LA_OK;
}

// Chunks per segment for the segmented algorithm.  The base choice gives every SM about four
// segments of at most 64 chunks.  A segment's CTA pays a pipeline fill and drain of about
// four chunks' work (~12 us against ~2.4 us per chunk on retention_128k), and CTAs run in
// waves of one per SM, so the time goes roughly as waves x (4 + chunks per segment).  The
// model overstates partial last waves, so a longer segment is taken only where it predicts
// at least 25 % less time than the base choice: small problems, where the base choice leaves
// many short segments in many waves (norm_b4h16: 6 -> 32 chunks, k3_seg 0.099 -> 0.088 ms
// measured; ragged_b2h32 keeps 27, which measured best among 27-64).
int segment_chunks(long long BH, int NC) {
  const int cap = NC < 64 ? (NC < 1 ? 1 : NC) : 64;
  long long l0 = BH * NC / (4LL * 148);
  if (l0 < 1) l0 = 1;
  if (l0 > cap) l0 = cap;
  auto cost = [&](long long l) {
    const long long ctas = BH * ((NC + l - 1) / l);
    return static_cast<double>((ctas + 147) / 148) * (4.0 + static_cast<double>(l));
  };
  const double c0 = cost(l0);
  long long best = l0;
  double cb = c0;
  for (long long l = 1; l <= cap; ++l) {
    const double c = cost(l);
    if (c < cb) {
      cb = c;
      best = l;
    }
  }
  return static_cast<int>(cb <= 0.75 * c0 ? best : l0);
}

int to_status(cudaError_t e) {
  if (e == cudaSuccess) return LA_OK;
  if (e == cudaErrorMemoryAllocation) return LA_ERR_OUT_OF_MEMORY;
  return LA_ERR_CUDA;
}

int prefill(const la_prefill_args& a, Recorder* rec = nullptr, bool exact_prefix = false) {
  Path path;
  int st = validate(a, &path);
  if (st != LA_OK) return st;
  GammaTable gt;
  st = check_gamma(a.gamma, a.H, &gt);
  if (st != LA_OK) return st;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(a.stream);
  const long long BH = static_cast<long long>(a.B) * a.H;
  if (BH == 0) return LA_OK;
  if (a.T == 0) {
    // No tokens: the final state is the initial one (or zero).
    auto put = [&](float* dst, const float* init, size_t bytes) -> bool {
      if (!dst) return true;
      if (!init) return cudaMemsetAsync(dst, 0, bytes, s) == cudaSuccess;
      if (init == dst) return true;
      return cudaMemcpyAsync(dst, init, bytes, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    };
    if (!put(a.S_final, a.S_init, static_cast<size_t>(BH) * a.dk * a.dv * 4)) return LA_ERR_CUDA;
    if (a.normalize && !put(a.Z_final, a.Z_init, static_cast<size_t>(BH) * a.dk * 4))
      return LA_ERR_CUDA;
    return LA_OK;
  }

  const Layout l = make_layout(a.B, a.H, a.T, a.dk, a.dv, a.C, a.normalize);
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  bool owned = false;
  if (ws) {
    if (a.workspace_bytes < l.total) return LA_ERR_INVALID_ARGUMENT;
  } else {
    cudaError_t e = workspace_alloc(reinterpret_cast<void**>(&ws), l.total, s);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return LA_ERR_OUT_OF_MEMORY;
    }
    owned = true;
  }

  PrefillParams p;
  p.BH = static_cast<int>(BH);
  p.H = a.H;
  p.T = a.T;
  p.dk = a.dk;
  p.dv = a.dv;
  p.C = a.C;
  p.NC = l.NC;
  p.L_last = l.L_last;
  p.R = l.R;
  p.eps = a.eps;
  p.rec = reinterpret_cast<float*>(ws + l.rec_off);
  p.tot = reinterpret_cast<float*>(ws + l.tot_off);
  p.S_final = a.S_final;
  p.Z_final = a.normalize ? a.Z_final : nullptr;
  p.S_init = a.S_init;
  p.Z_init = a.normalize ? a.Z_init : nullptr;
  p.has_init = p.S_init != nullptr || p.Z_init != nullptr;
  p.Ls = l.Ls;
  p.G = l.G;
  p.err = error_word_ptr();
  const bool out_f32 = a.dtype == LA_DTYPE_F32 || a.out_dtype == LA_OUT_F32;
  Flags f{a.feature_map, a.gamma != nullptr, a.normalize != 0, out_f32};

  cudaError_t e = cudaSuccess;
  if (path == Path::kSegmented) {
    // Segments of Lseg chunks; one record per segment at the start of the workspace,
    // then the scan's totals over segments.
    const int Lseg = a.segment_chunks > 0 ? a.segment_chunks : segment_chunks(BH, l.NC);
    const int NS = (l.NC + Lseg - 1) / Lseg;
    SegParams sp;
    sp.BH = p.BH;
    sp.H = p.H;
    sp.T = p.T;
    sp.dk = p.dk;
    sp.dv = p.dv;
    sp.C = p.C;
    sp.NC = l.NC;
    sp.L_last = l.L_last;
    sp.Lseg = Lseg;
    sp.NS = NS;
    sp.R = l.R;
    sp.eps = a.eps;
    sp.srec = reinterpret_cast<float*>(ws);
    sp.out = a.out;
    sp.has_init = p.has_init;
    sp.reverse = a.reverse != 0;
    sp.tf32_prefix = !exact_prefix;
    sp.err = p.err;
    const size_t srec_bytes = align256(static_cast<size_t>(BH) * NS * l.R * sizeof(float));
    PrefillParams ps = p;  // the scan over segments: one scan element per segment
    ps.NC = NS;
    ps.C = Lseg * a.C;
    ps.L_last = static_cast<int>(a.T - static_cast<long long>(NS - 1) * Lseg * a.C);
    ps.rec = sp.srec;
    ps.tot = reinterpret_cast<float*>(ws + srec_bytes);
    const ScanPlan spl = scan_plan(NS);
    ps.Ls = spl.Ls;
    ps.G = spl.G;
    TcMaps m;
    const uint64_t T = static_cast<uint64_t>(a.T);
    bool ok = make_map(&m.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.q, a.dk, T, BH, a.dk * 2ull,
                       T * a.dk * 2ull, 64, 64) &&
              make_map(&m.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.k, a.dk, T, BH, a.dk * 2ull,
                       T * a.dk * 2ull, 64, 64) &&
              make_map(&m.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.v, a.dv, T, BH, a.dv * 2ull,
                       T * a.dv * 2ull, 64, 64) &&
              make_map(&m.rec, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, sp.srec, a.dk, a.dv,
                       static_cast<uint64_t>(BH) * NS, a.dk * 4ull, l.R * 4ull, 32,
                       static_cast<uint32_t>(a.dv));
    if (!ok) {
      e = cudaErrorInvalidValue;
    } else {
      if (rec) rec->mark(s, "k1_seg");
      e = launch_k1_seg(sp, gt, m, f, s);
      if (e == cudaSuccess) e = launch_k2(ps, gt, a.scan_mode, f, s, rec);
      if (rec && !a.states_only) rec->mark(s, "k3_seg");
      if (e == cudaSuccess && !a.states_only) e = launch_k3_seg(sp, gt, m, f, s);
    }
  } else if (path == Path::kTensorCore) {
    TcMaps m;
    const uint64_t T = static_cast<uint64_t>(a.T);
    bool ok = make_map(&m.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.q, a.dk, T, BH, a.dk * 2ull,
                       T * a.dk * 2ull, 64, 64) &&
              make_map(&m.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.k, a.dk, T, BH, a.dk * 2ull,
                       T * a.dk * 2ull, 64, 64) &&
              make_map(&m.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.v, a.dv, T, BH, a.dv * 2ull,
                       T * a.dv * 2ull, 64, 64) &&
              (a.states_only ||
               (out_f32 ? make_map(&m.out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.out, a.dv, T, BH,
                                   a.dv * 4ull, T * a.dv * 4ull, 32, 64)
                        : make_map(&m.out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.out, a.dv, T, BH,
                                   a.dv * 2ull, T * a.dv * 2ull, 64, 64))) &&
              make_map(&m.rec, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, p.rec, a.dk, a.dv,
                       static_cast<uint64_t>(BH) * l.NC, a.dk * 4ull, l.R * 4ull, 32,
                       static_cast<uint32_t>(a.dv));
    if (!ok) {
      e = cudaErrorInvalidValue;
    } else {
      if (rec) rec->mark(s, "k1_tc");
      e = launch_k1_tc(p, gt, m, f, s);
      if (e == cudaSuccess) e = launch_k2(p, gt, a.scan_mode, f, s, rec);
      if (rec && !a.states_only) rec->mark(s, "k3_tc");
      if (e == cudaSuccess && !a.states_only) e = launch_k3_tc(p, gt, m, f, s);
    }
  } else {
    if (rec) rec->mark(s, "k1_fma");
    e = launch_k1_fma(p, gt, a.k, a.v, a.dtype, f, s);
    if (e == cudaSuccess) e = launch_k2(p, gt, a.scan_mode, f, s, rec);
    if (rec && !a.states_only) rec->mark(s, "k3_fma");
    if (e == cudaSuccess && !a.states_only)
      e = launch_k3_fma(p, gt, a.q, a.k, a.v, a.out, a.dtype, f, s);
  }
  if (rec) rec->mark(s);  // end of the last kernel (an unnamed mark)
  if (owned) {
    cudaError_t e2 = cudaFreeAsync(ws, s);
    if (e == cudaSuccess) e = e2;
  }
  return to_status(e);
}

la_prefill_args basic_args(const void* q, const void* k, const void* v, void* out,
                           float* S_final, float* Z_final, int B, int H, long long T, int dk,
                           int dv, int C, int feature_map, const float* gamma, int normalize,
                           la_stream_t stream, int dtype) {
  la_prefill_args a;
  std::memset(&a, 0, sizeof(a));
  a.q = q;
  a.k = k;
  a.v = v;
  a.out = out;
  a.S_final = S_final;
  a.Z_final = Z_final;
  a.B = B;
  a.H = H;
  a.T = T;
  a.dk = dk;
  a.dv = dv;
  a.C = C;
  a.feature_map = feature_map;
  a.gamma = gamma;
  a.normalize = normalize;
  a.eps = 0.f;
  a.dtype = dtype;
  a.out_dtype = LA_OUT_AS_INPUT;
  a.scan_mode = LA_SCAN_LOGDEPTH;
  a.kernel_path = dtype == LA_DTYPE_F32 ? LA_PATH_FMA : LA_PATH_AUTO;
  a.stream = stream;
  return a;
}

// Device buffer layout of lin_attn_prefill_host: q, k, v, out, S, Z, then the workspace.
struct HostLayout {
  size_t q, k, v, out, S, Z, ws, total;
};

HostLayout host_layout(const la_prefill_args& a) {
  HostLayout h{};
  const size_t BH = static_cast<size_t>(a.B) * a.H;
  const size_t e = a.dtype == LA_DTYPE_F32 ? 4 : 2;
  const size_t eo = (a.dtype == LA_DTYPE_F32 || a.out_dtype == LA_OUT_F32) ? 4 : 2;
  const size_t T = static_cast<size_t>(a.T > 0 ? a.T : 0);
  size_t off = 0;
  h.q = off; off = align256(off + BH * T * a.dk * e);
  h.k = off; off = align256(off + BH * T * a.dk * e);
  h.v = off; off = align256(off + BH * T * a.dv * e);
  h.out = off; off = align256(off + BH * T * a.dv * eo);
  h.S = off; off = align256(off + BH * a.dk * a.dv * 4);
  h.Z = off; off = align256(off + BH * a.dk * 4);
  h.ws = off;
  off += make_layout(a.B, a.H, a.T, a.dk, a.dv, a.C, a.normalize).total;
  h.total = off;
  return h;
}

}  // namespace

int prefill_with_args(const la_prefill_args& a, Recorder* rec, bool exact_prefix) {
  return prefill(a, rec, exact_prefix);
}

int* device_error_word() { return error_word_ptr(); }

cudaError_t workspace_alloc(void** p, size_t bytes, cudaStream_t s) {
  const char* inj = std::getenv("LA_FAULT_INJECT");
  if (inj && std::strcmp(inj, "alloc") == 0) return cudaErrorMemoryAllocation;
  return cudaMallocAsync(p, bytes, s);
}

bool make_plain_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t d0,
                    uint64_t d1, uint64_t d2, uint64_t stride1, uint64_t stride2, uint32_t box0,
                    uint32_t box1) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {stride1, stride2};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int default_segment_chunks(long long BH, int NC) { return segment_chunks(BH, NC); }

bool make_tile_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t d0,
                   uint64_t d1, uint64_t d2, uint64_t stride1, uint64_t stride2, uint32_t box0,
                   uint32_t box1) {
  return make_map(m, dt, base, d0, d1, d2, stride1, stride2, box0, box1);
}

int check_prefill_args(const la_prefill_args& a) {
  Path path;
  const int st = validate(a, &path);
  if (st != LA_OK) return st;
  GammaTable gt;
  return check_gamma(a.gamma, a.H, &gt);
}

}  // namespace la

extern "C" {

int lin_attn_prefill(const void* q, const void* k, const void* v, void* out, float* S_final,
                     float* Z_final, int B, int H, long long T, int dk, int dv, int C,
                     int feature_map, const float* gamma, int normalize, la_stream_t stream) {
  const la_prefill_args a = la::basic_args(q, k, v, out, S_final, Z_final, B, H, T, dk, dv, C,
                                           feature_map, gamma, normalize, stream, LA_DTYPE_BF16);
  return la::prefill(a);
}

int lin_attn_prefill_f32(const float* q, const float* k, const float* v, float* out,
                         float* S_final, float* Z_final, int B, int H, long long T, int dk,
                         int dv, int C, int feature_map, const float* gamma, int normalize,
                         la_stream_t stream) {
  const la_prefill_args a = la::basic_args(q, k, v, out, S_final, Z_final, B, H, T, dk, dv, C,
                                           feature_map, gamma, normalize, stream, LA_DTYPE_F32);
  return la::prefill(a);
}

size_t lin_attn_prefill_workspace_bytes(int B, int H, long long T, int dk, int dv, int C,
                                        int normalize) {
  if (B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0 || C <= 0) return 0;
  return la::make_layout(B, H, T, dk, dv, C, normalize).total;
}

int lin_attn_prefill_ex(const la_prefill_args* args) {
  if (!args) return LA_ERR_INVALID_ARGUMENT;
  return la::prefill(*args);
}

int lin_attn_prefill_timed(const la_prefill_args* args, float* kernel_ms, int max_kernels,
                           int* n_kernels) {
  if (!args || !kernel_ms || !n_kernels || max_kernels < 1) return LA_ERR_INVALID_ARGUMENT;
  *n_kernels = 0;
  constexpr int kMaxEvents = 8;
  cudaEvent_t ev[kMaxEvents];
  int created = 0;
  for (; created < kMaxEvents; ++created)
    if (cudaEventCreate(&ev[created]) != cudaSuccess) break;
  if (created < kMaxEvents) {
    for (int i = 0; i < created; ++i) cudaEventDestroy(ev[i]);
    return LA_ERR_CUDA;
  }
  la::Recorder rec;
  rec.ev = ev;
  rec.cap = kMaxEvents;
  int st = la::prefill(*args, &rec);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(args->stream);
  if (st == LA_OK && cudaStreamSynchronize(s) != cudaSuccess) st = LA_ERR_CUDA;
  if (st == LA_OK) {
    const int nk = rec.n - 1;
    for (int i = 0; i < nk && i < max_kernels; ++i) {
      float ms = 0.f;
      cudaEventElapsedTime(&ms, ev[i], ev[i + 1]);
      kernel_ms[i] = ms;
    }
    *n_kernels = nk < 0 ? 0 : nk;
  }
  for (int i = 0; i < kMaxEvents; ++i) cudaEventDestroy(ev[i]);
  return st;
}

size_t lin_attn_prefill_host_buffer_bytes(const la_prefill_args* a) {
  if (!a || a->B < 0 || a->H < 0 || a->T < 0 || a->dk <= 0 || a->dv <= 0 || a->C <= 0) return 0;
  return la::host_layout(*a).total;
}

int lin_attn_prefill_host(const la_prefill_args* host_args, void* device_buffer,
                          size_t device_buffer_bytes) {
  if (!host_args) return LA_ERR_INVALID_ARGUMENT;
  const la_prefill_args& h = *host_args;
  la::Path path;
  int st = la::validate(h, &path);
  if (st != LA_OK) return st;
  const la::HostLayout hl = la::host_layout(h);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(h.stream);
  uint8_t* buf = static_cast<uint8_t*>(device_buffer);
  bool owned = false;
  if (buf) {
    if (device_buffer_bytes < hl.total || (reinterpret_cast<uintptr_t>(buf) & 255u))
      return LA_ERR_INVALID_ARGUMENT;
  } else {
    if (la::workspace_alloc(reinterpret_cast<void**>(&buf), hl.total, s) != cudaSuccess) {
      cudaGetLastError();
      return LA_ERR_OUT_OF_MEMORY;
    }
    owned = true;
  }
  const size_t BH = static_cast<size_t>(h.B) * h.H;
  const size_t e = h.dtype == LA_DTYPE_F32 ? 4 : 2;
  const size_t eo = (h.dtype == LA_DTYPE_F32 || h.out_dtype == LA_OUT_F32) ? 4 : 2;
  const size_t T = static_cast<size_t>(h.T);
  // Per (b, h) pair: bytes of q (= k), v, out, S and Z.  Pairs are contiguous in every
  // tensor, so a group of heads of one batch row is one byte range of each.
  const size_t pq = T * h.dk * e, pv = T * h.dv * e, po = T * h.dv * eo;
  const size_t pS = static_cast<size_t>(h.dk) * h.dv * 4, pZ = static_cast<size_t>(h.dk) * 4;
  // Groups of at least 32 MB of input (at most 16 groups): group g + 1 is copied in while
  // group g runs and group g - 1 is copied out, so the two copy directions overlap.
  const size_t in_bytes = BH * (2 * pq + pv);
  const int groups_target = static_cast<int>(std::min<size_t>(16, in_bytes >> 25));
  const int hpg = groups_target > 1 && BH > 1
                      ? std::max(1, static_cast<int>((BH + groups_target - 1) / groups_target))
                      : h.H;
  const int heads_per_group = std::min(hpg, h.H);
  cudaError_t err = cudaSuccess;
  cudaStream_t sc[2] = {nullptr, nullptr};  // copy-in, copy-out (compute runs on s)
  cudaEvent_t ev_start = nullptr;
  const bool pipelined = groups_target > 1 && BH > 1;
  if (pipelined && BH > 0 && T > 0) {
    for (auto& x : sc)
      if (err == cudaSuccess) err = cudaStreamCreateWithFlags(&x, cudaStreamNonBlocking);
    if (err == cudaSuccess) err = cudaEventCreateWithFlags(&ev_start, cudaEventDisableTiming);
    if (err == cudaSuccess) err = cudaEventRecord(ev_start, s);  // caller's prior work
    if (err == cudaSuccess) err = cudaStreamWaitEvent(sc[0], ev_start, 0);
    for (int b = 0; b < h.B && err == cudaSuccess && st == LA_OK; ++b) {
      for (int h0 = 0; h0 < h.H && err == cudaSuccess && st == LA_OK; h0 += heads_per_group) {
        const int hn = std::min(heads_per_group, h.H - h0);
        const size_t bh0 = static_cast<size_t>(b) * h.H + h0;
        auto src = [](const void* p, size_t off) { return static_cast<const uint8_t*>(p) + off; };
        err = cudaMemcpyAsync(buf + hl.q + bh0 * pq, src(h.q, bh0 * pq), hn * pq,
                              cudaMemcpyHostToDevice, sc[0]);
        if (err == cudaSuccess)
          err = cudaMemcpyAsync(buf + hl.k + bh0 * pq, src(h.k, bh0 * pq), hn * pq,
                                cudaMemcpyHostToDevice, sc[0]);
        if (err == cudaSuccess)
          err = cudaMemcpyAsync(buf + hl.v + bh0 * pv, src(h.v, bh0 * pv), hn * pv,
                                cudaMemcpyHostToDevice, sc[0]);
        if (err == cudaSuccess && h.S_init)
          err = cudaMemcpyAsync(buf + hl.S + bh0 * pS, src(h.S_init, bh0 * pS), hn * pS,
                                cudaMemcpyHostToDevice, sc[0]);
        if (err == cudaSuccess && h.Z_init && h.normalize)
          err = cudaMemcpyAsync(buf + hl.Z + bh0 * pZ, src(h.Z_init, bh0 * pZ), hn * pZ,
                                cudaMemcpyHostToDevice, sc[0]);
        cudaEvent_t ev_in = nullptr, ev_done = nullptr;
        if (err == cudaSuccess) err = cudaEventCreateWithFlags(&ev_in, cudaEventDisableTiming);
        if (err == cudaSuccess) err = cudaEventCreateWithFlags(&ev_done, cudaEventDisableTiming);
        if (err == cudaSuccess) err = cudaEventRecord(ev_in, sc[0]);
        if (err == cudaSuccess) err = cudaStreamWaitEvent(s, ev_in, 0);
        la_prefill_args d = h;
        d.B = 1;
        d.H = hn;
        d.gamma = h.gamma ? h.gamma + h0 : nullptr;
        d.q = buf + hl.q + bh0 * pq;
        d.k = buf + hl.k + bh0 * pq;
        d.v = buf + hl.v + bh0 * pv;
        d.out = buf + hl.out + bh0 * po;
        d.S_final = h.S_final ? reinterpret_cast<float*>(buf + hl.S + bh0 * pS) : nullptr;
        d.Z_final = h.Z_final ? reinterpret_cast<float*>(buf + hl.Z + bh0 * pZ) : nullptr;
        d.S_init = h.S_init ? reinterpret_cast<float*>(buf + hl.S + bh0 * pS) : nullptr;
        d.Z_init = h.Z_init ? reinterpret_cast<float*>(buf + hl.Z + bh0 * pZ) : nullptr;
        d.workspace = buf + hl.ws;  // one group at a time on the compute stream
        d.workspace_bytes = hl.total - hl.ws;
        d.stream = s;
        if (err == cudaSuccess) st = la::prefill(d);
        if (err == cudaSuccess && st == LA_OK) err = cudaEventRecord(ev_done, s);
        if (err == cudaSuccess && st == LA_OK) err = cudaStreamWaitEvent(sc[1], ev_done, 0);
        if (err == cudaSuccess && st == LA_OK && h.out && !h.states_only)
          err = cudaMemcpyAsync(static_cast<uint8_t*>(h.out) + bh0 * po, d.out, hn * po,
                                cudaMemcpyDeviceToHost, sc[1]);
        if (err == cudaSuccess && st == LA_OK && h.S_final)
          err = cudaMemcpyAsync(reinterpret_cast<uint8_t*>(h.S_final) + bh0 * pS, d.S_final,
                                hn * pS, cudaMemcpyDeviceToHost, sc[1]);
        if (err == cudaSuccess && st == LA_OK && h.Z_final && h.normalize)
          err = cudaMemcpyAsync(reinterpret_cast<uint8_t*>(h.Z_final) + bh0 * pZ, d.Z_final,
                                hn * pZ, cudaMemcpyDeviceToHost, sc[1]);
        // Events may be destroyed once recorded; the waits already made keep their order.
        if (ev_in) cudaEventDestroy(ev_in);
        if (ev_done) cudaEventDestroy(ev_done);
      }
    }
    // Every copy has finished before the buffer is released and the call returns.
    for (auto& x : sc)
      if (x) {
        const cudaError_t se = cudaStreamSynchronize(x);
        if (err == cudaSuccess) err = se;
        cudaStreamDestroy(x);
      }
    if (ev_start) cudaEventDestroy(ev_start);
  } else {
    const size_t nq = BH * pq, nv = BH * pv, no = BH * po;
    if (nq) err = cudaMemcpyAsync(buf + hl.q, h.q, nq, cudaMemcpyHostToDevice, s);
    if (err == cudaSuccess && nq) err = cudaMemcpyAsync(buf + hl.k, h.k, nq, cudaMemcpyHostToDevice, s);
    if (err == cudaSuccess && nv) err = cudaMemcpyAsync(buf + hl.v, h.v, nv, cudaMemcpyHostToDevice, s);
    if (err == cudaSuccess && h.S_init)
      err = cudaMemcpyAsync(buf + hl.S, h.S_init, BH * pS, cudaMemcpyHostToDevice, s);
    if (err == cudaSuccess && h.Z_init && h.normalize)
      err = cudaMemcpyAsync(buf + hl.Z, h.Z_init, BH * pZ, cudaMemcpyHostToDevice, s);
    la_prefill_args d = h;
    d.q = buf + hl.q;
    d.k = buf + hl.k;
    d.v = buf + hl.v;
    d.out = buf + hl.out;
    d.S_final = h.S_final ? reinterpret_cast<float*>(buf + hl.S) : nullptr;
    d.Z_final = h.Z_final ? reinterpret_cast<float*>(buf + hl.Z) : nullptr;
    d.S_init = h.S_init ? reinterpret_cast<float*>(buf + hl.S) : nullptr;
    d.Z_init = h.Z_init ? reinterpret_cast<float*>(buf + hl.Z) : nullptr;
    d.workspace = buf + hl.ws;
    d.workspace_bytes = hl.total - hl.ws;
    if (err == cudaSuccess) st = la::prefill(d);
    if (err == cudaSuccess && st == LA_OK) {
      if (no && h.out && !h.states_only) err = cudaMemcpyAsync(h.out, d.out, no, cudaMemcpyDeviceToHost, s);
      if (err == cudaSuccess && h.S_final)
        err = cudaMemcpyAsync(h.S_final, d.S_final, BH * pS, cudaMemcpyDeviceToHost, s);
      if (err == cudaSuccess && h.Z_final && h.normalize)
        err = cudaMemcpyAsync(h.Z_final, d.Z_final, BH * pZ, cudaMemcpyDeviceToHost, s);
    }
  }
  if (owned) cudaFreeAsync(buf, s);
  const cudaError_t se = cudaStreamSynchronize(s);
  if (err == cudaSuccess) err = se;
  if (st != LA_OK) return st;
  return la::to_status(err);
}

int lin_attn_decode_step(const void* q, const void* k, const void* v, void* out, float* S,
                         float* Z, int B, int H, int dk, int dv, int feature_map,
                         const float* gamma, int normalize, la_stream_t stream);

static int decode_common(const void* q, const void* k, const void* v, void* out, float* S,
                         float* Z, int B, int H, int dk, int dv, int feature_map,
                         const float* gamma, int normalize, la_stream_t stream, int dtype) {
  if (B < 0 || H < 0 || dk <= 0 || dv <= 0) return LA_ERR_INVALID_ARGUMENT;
  if (feature_map != LA_FM_IDENTITY && feature_map != LA_FM_ELU1) return LA_ERR_INVALID_ARGUMENT;
  if (normalize && feature_map == LA_FM_IDENTITY) return LA_ERR_INVALID_ARGUMENT;
  if (dk > 256 || dv > 256) return LA_ERR_UNSUPPORTED;
  const long long BH = static_cast<long long>(B) * H;
  if (BH == 0) return LA_OK;
  if (BH > (1LL << 31) - 1) return LA_ERR_UNSUPPORTED;
  if (!q || !k || !v || !out || !S || (normalize && !Z)) return LA_ERR_INVALID_ARGUMENT;
  la::GammaTable gt;
  int st = la::check_gamma(gamma, H, &gt);
  if (st != LA_OK) return st;
  la::Flags f{feature_map, gamma != nullptr, normalize != 0, dtype == la::kF32};
  const cudaError_t e = la::launch_decode(q, k, v, out, S, Z, static_cast<int>(BH), H, dk, dv,
                                          dtype, f, gt, 0.f, la::error_word_ptr(),
                                          reinterpret_cast<cudaStream_t>(stream));
  return la::to_status(e);
}

int lin_attn_decode_step(const void* q, const void* k, const void* v, void* out, float* S,
                         float* Z, int B, int H, int dk, int dv, int feature_map,
                         const float* gamma, int normalize, la_stream_t stream) {
  return decode_common(q, k, v, out, S, Z, B, H, dk, dv, feature_map, gamma, normalize, stream,
                       la::kBF16);
}

int lin_attn_decode_step_f32(const float* q, const float* k, const float* v, float* out,
                             float* S, float* Z, int B, int H, int dk, int dv, int feature_map,
                             const float* gamma, int normalize, la_stream_t stream) {
  return decode_common(q, k, v, out, S, Z, B, H, dk, dv, feature_map, gamma, normalize, stream,
                       la::kF32);
}

int lin_attn_device_error(int* code) {
  if (!code) return LA_ERR_INVALID_ARGUMENT;
  *code = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return LA_ERR_CUDA;
  int zero = 0;
  e = cudaMemcpyFromSymbol(code, la::g_error_word, sizeof(int));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(la::g_error_word, &zero, sizeof(int));
  return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

const char* lin_attn_status_string(int status) {
  switch (status) {
    case LA_OK: return "LA_OK";
    case LA_ERR_INVALID_ARGUMENT: return "LA_ERR_INVALID_ARGUMENT";
    case LA_ERR_UNSUPPORTED: return "LA_ERR_UNSUPPORTED";
    case LA_ERR_OUT_OF_MEMORY: return "LA_ERR_OUT_OF_MEMORY";
    case LA_ERR_CUDA: return "LA_ERR_CUDA";
    case LA_ERR_INTERNAL: return "LA_ERR_INTERNAL";
    default: return "LA_ERR_UNKNOWN";
  }
}

int lin_attn_scan_plan(long long n, int scan_mode, int* segment_len, int* segments,
                       int* groups, int* per_group, long long* depth) {
  if (n < 1 || (scan_mode != LA_SCAN_LOGDEPTH && scan_mode != LA_SCAN_SEQUENTIAL))
    return LA_ERR_INVALID_ARGUMENT;
  la::ScanPlan pl = la::scan_plan(n);
  if (scan_mode == LA_SCAN_SEQUENTIAL) {
    pl.Ls = static_cast<int>(n > (1LL << 31) - 1 ? (1LL << 31) - 1 : n);
    pl.G = 1;
    pl.NG = 1;
    pl.E = pl.Ls;
    pl.depth = n;
  }
  if (segment_len) *segment_len = pl.Ls;
  if (segments) *segments = pl.G;
  if (groups) *groups = pl.NG;
  if (per_group) *per_group = pl.E;
  if (depth) *depth = pl.depth;
  return LA_OK;
}

int lin_attn_version(void) { return la::kVersion; }

}  // extern "C"
