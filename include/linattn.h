/*
 * linattn.h -- C ABI of the chunked causal linear-attention library for NVIDIA B200
 * (sm_100a).
 *
 * What the library computes
 * -------------------------
 * For every (batch b, head h) and every token t < T:
 *
 *     S_t = gamma_h * S_{t-1} + psi(k_t) v_t^T        (dk x dv, float32 state)
 *     Z_t = gamma_h * Z_{t-1} + psi(k_t)              (dk)
 *     o_t = psi(q_t) S_t / (psi(q_t) . Z_t + eps)     (normalised form), or
 *     o_t = psi(q_t) S_t                              (unnormalised form)
 *
 * with S_{-1} = 0, Z_{-1} = 0, psi = ELU+1 (x + 1 for x > 0, e^x otherwise) or the
 * identity, and gamma_h = 1 when no decay is given.  Sources: "Log-Depth Chunked
 * Linear-Attention Scan", sections "Mathematical statement" (inclusive state and
 * normaliser sums) and "Implementation notes" (ratio with eps); "Linear Attention and
 * Retentive Networks: How Recurrent Duals and Chunkwise Tiling Eliminate the Quadratic
 * Bottleneck", sections "The Associative Property and Linear Kernel Formulation" (ELU+1
 * feature map), "The Recurrent Dual" and "B. Recurrent Representation" (per-head decay).
 *
 * How the prefill computes it (the scan page's three kernels):
 *   K1  per chunk of C tokens: psi, decay weights, and the chunk summaries
 *       S_loc = sum_j Xi_j psi(k_j) v_j^T,  Z_loc = sum_j Xi_j psi(k_j), Xi_j = gamma^(L-1-j)
 *       ("Formulas"; decay placement from "C. Chunkwise Recurrent Representation").
 *   K2  exclusive associative scan of the summaries across chunks
 *       ((a1,S1,Z1) + (a2,S2,Z2) = (a1 a2, a2 S1 + S2, a2 Z1 + Z2), a = gamma^L), either
 *       log-depth (a blocked Hillis-Steele scan, see lin_attn_scan_plan) or a sequential
 *       carry (comparison mode).
 *   K3  per chunk: the intra-chunk causal part (psi(Q) psi(K)^T masked with gamma^(i-j))
 *       plus Theta_i psi(q_i) P_c with the chunk's exclusive prefix P_c, Theta_i =
 *       gamma^(i+1), then the normalisation.
 * Positions past T in a padded last chunk contribute nothing and do not advance the
 * decay, so S_final is exactly S_{T-1}.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *   Layout   q, k: [B, H, T, dk]; v, out: [B, H, T, dv]; contiguous, row-major.
 *            S_final / S: [B, H, dk, dv] (row i = key feature, column j = value feature);
 *            Z_final / Z: [B, H, dk].  All float32 states.
 *   Memory   Tensor pointers are DEVICE pointers owned by the caller, except where an
 *            entry point says HOST.  The library never frees caller memory.  Every tensor
 *            pointer must be 16-byte aligned.
 *   gamma    HOST array of H float32 decays in [0, 1], or NULL for no decay.  It is read
 *            during the call and copied into the kernel launches (at most 1024 heads).
 *   stream   A CUDA stream (cudaStream_t / CUstream), or NULL for the legacy default.
 *   Async    Device entry points only enqueue work and return; errors raised by the
 *            kernels surface at the caller's next synchronisation.  No host sync.
 *   Errors   Arguments are validated before anything is enqueued; on a non-zero status
 *            nothing has been launched.
 *   Determinism  No atomics on the data path; results are bitwise reproducible for a
 *            fixed configuration.
 */
#ifndef LINATTN_H_
#define LINATTN_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream, declared here so the header needs no CUDA
 * include. */
typedef struct CUstream_st* la_stream_t;

typedef enum {
  LA_OK = 0,
  LA_ERR_INVALID_ARGUMENT = 1, /* NULL required pointer, negative size, gamma outside
                                  [0,1], normalize with the identity map, out aliasing an
                                  input, misaligned pointer, bad enum value */
  LA_ERR_UNSUPPORTED = 2,      /* shape outside the supported set (see below) */
  LA_ERR_OUT_OF_MEMORY = 3,    /* the library-side workspace could not be allocated */
  LA_ERR_CUDA = 4,             /* a CUDA runtime call or kernel launch failed */
  LA_ERR_INTERNAL = 5          /* a kernel reported a failed internal check */
} la_status;

typedef enum { LA_FM_IDENTITY = 0, LA_FM_ELU1 = 1 } la_feature_map;

typedef enum {
  LA_SCAN_LOGDEPTH = 0,   /* K2 as a blocked log-depth scan (lin_attn_scan_plan) */
  LA_SCAN_SEQUENTIAL = 1  /* K2 as one sequential carry over chunks (comparison only) */
} la_scan_mode;

typedef enum { LA_DTYPE_BF16 = 0, LA_DTYPE_F32 = 1 } la_dtype;

/* Element type of `out`: the input type, or float32 (exact-to-accumulator output for
 * bf16 inputs; the normalised form's outputs shrink with t, so bf16 output rounding can
 * dominate the error on long sequences). */
typedef enum { LA_OUT_AS_INPUT = 0, LA_OUT_F32 = 1 } la_out_dtype;

/*
 * How the chunk summaries are combined.
 *   LA_ALGO_CHUNKED    the scan page's three kernels as stated: K1 writes every chunk's
 *                      summary, K2 scans all of them, K3 reads each chunk's prefix once.
 *   LA_ALGO_SEGMENTED  the hierarchical form of the same scan: chunks are grouped into
 *                      segments; K1 writes one summary per segment, K2 scans segments,
 *                      and K3 walks each segment's chunks in order, carrying the prefix
 *                      on chip and advancing it with the chunk's own summary.  Same
 *                      results, about a third of the HBM traffic.  Tensor-core path
 *                      only: bf16 inputs, C = 64, dk in {64, 128}, dv = 128, and not the
 *                      ELU+1 map together with a decay.
 *   LA_ALGO_AUTO       segmented where supported, else chunked.
 */
typedef enum { LA_ALGO_AUTO = 0, LA_ALGO_CHUNKED = 1, LA_ALGO_SEGMENTED = 2 } la_algorithm;

typedef enum {
  LA_PATH_AUTO = 0,        /* tensor-core kernels where the shape allows, else FMA kernels */
  LA_PATH_TENSOR_CORE = 1, /* tcgen05/TMEM kernels only (LA_ERR_UNSUPPORTED otherwise) */
  LA_PATH_FMA = 2          /* CUDA-core fp32 FMA kernels for every step */
} la_kernel_path;

/*
 * Supported shapes.
 *   FMA path (float32 or bf16 inputs): dk, dv multiples of 4 in [4, 128], C in {16, 32, 64}.
 *   Tensor-core path (bf16 inputs only): dk, dv in {64, 128}, C = 64.
 * T may be any value >= 0 (a ragged last chunk is handled), B and H any value >= 0 with
 * B*H*T*max(dk,dv) < 2^62.
 */

/*
 * lin_attn_prefill -- bf16 inputs and output, float32 states; the whole K1 -> K2 -> K3
 * path on `stream`.
 *   q, k, v   DEVICE bf16, layout above; may be NULL only when B*H*T == 0.
 *   out       DEVICE bf16 [B,H,T,dv]; must not alias q, k or v.
 *   S_final   DEVICE float32 [B,H,dk,dv] or NULL (not written).  Final state S_{T-1}.
 *   Z_final   DEVICE float32 [B,H,dk] or NULL.  Written only when normalize != 0.
 *   C         chunk length.
 *   feature_map  la_feature_map.  normalize != 0 requires LA_FM_ELU1 (the identity map
 *             gives a denominator of indefinite sign).
 * Uses the log-depth scan, LA_ALGO_AUTO and eps = 0.  The workspace is allocated with
 * cudaMallocAsync / cudaFreeAsync on `stream` (LA_ERR_OUT_OF_MEMORY on failure; with
 * the environment variable LA_FAULT_INJECT=alloc every library-side allocation fails
 * this way without allocating, for testing callers' handling of it).
 * T == 0 zero-fills S_final / Z_final.  Returns a la_status.
 */
int lin_attn_prefill(const void* q, const void* k, const void* v, void* out,
                     float* S_final, float* Z_final, int B, int H, long long T, int dk,
                     int dv, int C, int feature_map, const float* gamma, int normalize,
                     la_stream_t stream);

/* lin_attn_prefill_f32 -- the same contract with float32 q, k, v and out; runs the
 * fp32 FMA kernels. */
int lin_attn_prefill_f32(const float* q, const float* k, const float* v, float* out,
                         float* S_final, float* Z_final, int B, int H, long long T, int dk,
                         int dv, int C, int feature_map, const float* gamma, int normalize,
                         la_stream_t stream);

/* Bytes of device workspace the prefill needs for this shape (chunk summaries and scan
 * segment totals), enough for either algorithm.  Pure host computation; 0 for an empty
 * problem. */
size_t lin_attn_prefill_workspace_bytes(int B, int H, long long T, int dk, int dv, int C,
                                        int normalize);

/* Every option of the prefill in one struct. */
typedef struct la_prefill_args {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  float* S_final;         /* may be NULL */
  float* Z_final;         /* may be NULL */
  int B, H;
  long long T;
  int dk, dv, C;
  int feature_map;        /* la_feature_map */
  const float* gamma;     /* HOST, H values, or NULL */
  int normalize;
  float eps;              /* added to the denominator of the normalised form (>= 0) */
  int dtype;              /* la_dtype of q, k and v */
  int out_dtype;          /* la_out_dtype of out */
  int scan_mode;          /* la_scan_mode */
  int kernel_path;        /* la_kernel_path */
  int algorithm;          /* la_algorithm */
  int segment_chunks;     /* chunks per segment for LA_ALGO_SEGMENTED (1..1024), or 0 to
                             choose automatically (a few segments per SM, at most 64) */
  void* workspace;        /* DEVICE, >= lin_attn_prefill_workspace_bytes(), 256-byte
                             aligned; NULL = allocate on the stream */
  size_t workspace_bytes;
  la_stream_t stream;
  /* The state before token 0, for a sequence that continues an earlier one: DEVICE
   * float32 in the layout of S_final / Z_final, or NULL for zero.  The scan takes it as
   * its first element (the scan page's monoid with one more element in front), so every
   * chunk's prefix carries it decayed by gamma^(tokens before the chunk) and S_final
   * includes gamma^T S_init.  May be the same memory as S_final / Z_final (each element
   * is read before it is written).  Z_init is used only when normalising. */
  const float* S_init;
  const float* Z_init;
  /* 1: compute only S_final / Z_final (the summaries and the scan, no output: `out` may
   * be NULL) -- the per-part totals of a sequence split across devices.  0: full prefill. */
  int states_only;
  /* 1: run the recurrence from token T-1 down to token 0 (the anti-causal direction):
   * out_t = psi(q_t) S'_t with S'_t = gamma S'_{t+1} + psi(k_t) v_t^T, S'_T = S_init, and
   * S_final = S'_0 -- the prefill of the time-reversed sequence, with every tensor kept
   * in its memory order.  Segmented algorithm only (LA_ERR_UNSUPPORTED otherwise).
   * 0: causal. */
  int reverse;
} la_prefill_args;

/* lin_attn_prefill_ex -- the prefill with every option of la_prefill_args.  A caller
 * workspace that is too small or misaligned gives LA_ERR_INVALID_ARGUMENT. */
int lin_attn_prefill_ex(const la_prefill_args* args);

/*
 * lin_attn_prefill_timed -- lin_attn_prefill_ex with a CUDA event recorded on the stream
 * before every kernel launch and after the last one; synchronises the stream and writes
 * each kernel's device duration (milliseconds, launch order) to kernel_ms[0 ..].
 * *n_kernels receives the number of kernels the prefill launched: K1, the scan's kernels
 * (3 for the log-depth scan over more than 2048 elements, 1 for at most 2048 elements or
 * for the sequential carry), K3.  For profiling;
 * the results are identical to lin_attn_prefill_ex.
 */
int lin_attn_prefill_timed(const la_prefill_args* args, float* kernel_ms, int max_kernels,
                           int* n_kernels);

/*
 * lin_attn_prefill_host -- the same computation with HOST buffers, for callers whose
 * data lives in host memory.  q, k, v, out, S_final, Z_final (and S_init, Z_init when
 * given) are HOST pointers (pinned
 * memory gives full copy bandwidth; pageable memory works).  `device_buffer` is DEVICE
 * memory of at least lin_attn_prefill_host_buffer_bytes() bytes used to stage the
 * tensors and the workspace, or NULL to allocate it on the stream.  Copies the inputs
 * to the device, runs the prefill, copies the results back and synchronises `stream`
 * before returning, so the host outputs are ready on LA_OK.  Problems of 64 MB of inputs
 * or more are processed in groups of heads (up to 16, each at least 32 MB) on two copy
 * streams of the library's own plus `stream`, so that the copies into the device, the
 * kernels and the copies back overlap; the work still starts after everything queued on
 * `stream` before the call.  Each (b, h) is computed exactly as by lin_attn_prefill_ex
 * whenever the segmented algorithm's segment length is fixed (segment_chunks > 0) or the
 * chunked algorithm runs.
 */
int lin_attn_prefill_host(const la_prefill_args* host_args, void* device_buffer,
                          size_t device_buffer_bytes);
size_t lin_attn_prefill_host_buffer_bytes(const la_prefill_args* host_args);

/*
 * lin_attn_combine_states -- the incoming state of one part of a sequence that is split
 * into consecutive parts (for example one part per device, each computing its part's
 * final state from a zero start with states_only = 1).  The scan page's monoid applied
 * to whole parts ("Log-Depth Chunked Linear-Attention Scan", Formulas; with the decay of
 * "Linear Attention and Retentive Networks ...", C. Chunkwise Recurrent Representation):
 *     P = 0;  for j < upto:  P = gamma_h^(part_tokens[j]) P + S_parts[j]
 * and likewise for Z.  P is part `upto`'s S_init (upto = parts gives the whole
 * sequence's final state).
 *   S_parts   DEVICE [parts, B, H, dk, dv] float32 (each part's final state)
 *   Z_parts   DEVICE [parts, B, H, dk] float32, or NULL (then Z_out is not written)
 *   part_tokens HOST [parts], tokens in each part (>= 0)
 *   gamma     HOST [H] decays in [0, 1], or NULL for none
 *   S_out     DEVICE [B, H, dk, dv]; Z_out DEVICE [B, H, dk] or NULL
 * 0 <= upto <= parts <= 64.  Asynchronous on `stream`.
 */
int lin_attn_combine_states(const float* S_parts, const float* Z_parts, int parts, int upto,
                            const long long* part_tokens, int B, int H, int dk, int dv,
                            const float* gamma, float* S_out, float* Z_out, la_stream_t stream);

/*
 * lin_attn_prefill_noalloc -- lin_attn_prefill_ex without any device allocation.  (No
 * passage of the pages corresponds to it; it exists for callers that cannot allocate.)
 *
 * Callers that must not allocate device memory while they run -- processes that
 * reserve a fixed memory budget at start-up, frameworks that route every allocation
 * through their own allocator, code that cannot recover from a failed allocation -- use
 * this entry point: the workspace is a fixed array inside the library's device image
 * (LA_NOALLOC_SCRATCH_BYTES bytes, held by every GPU that loads the library until the
 * process exits) instead of cudaMalloc / cudaMallocAsync memory.  args->workspace and
 * args->workspace_bytes are ignored; everything else is as in lin_attn_prefill_ex.
 *   - A problem whose workspace (lin_attn_prefill_workspace_bytes) exceeds
 *     LA_NOALLOC_SCRATCH_BYTES returns LA_ERR_UNSUPPORTED and launches nothing.
 *   - The first call on each device looks up the array's device address (with that
 *     device current) and keeps it; make that first call before any stream capture, and
 *     do not use this entry point across a reset of the device (cudaDeviceReset), which
 *     would leave the kept address stale.
 *   - Every call shares the array and it keeps the last call's contents; the kernels
 *     write all workspace bytes before reading them, so no clearing is needed.  Calls
 *     whose work overlaps on the GPU race on the array: serialise them.
 */
#define LA_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
int lin_attn_prefill_noalloc(const la_prefill_args* args);

/*
 * lin_attn_backward -- gradients of the unnormalised form (o_t = psi(q_t) S_t, any decay,
 * either feature map) for the loss L = sum(grad_out . out) + sum(grad_S_final . S_final).
 * The scan page asks for forward and backward latency ("Log-Depth Chunked
 * Linear-Attention Scan", Implementation notes); the gradients are those of the recurrent
 * form of "Linear Attention and Retentive Networks ..." (B. Recurrent Representation)
 * with S_{-1} = S_init.  With G_t = dL/dS_t accumulated backwards in time,
 *     G_t = psi(q_t) grad_out_t^T + gamma G_{t+1},  G_{T-1} includes grad_S_final,
 *     grad_q_t = psi'(q_t) .* (S_t grad_out_t),
 *     grad_k_t = psi'(k_t) .* (G_t v_t),   grad_v_t = G_t^T psi(k_t),
 *     grad_S_init = gamma G_0.
 * Each sum is itself a causal linear attention, so the library computes them with three
 * prefills (all their kernels, on the same workspace):
 *   grad_q  the prefill of (q, k, v) = (grad_out, v, psi(k)) under the identity map,
 *           started from S_init^T;
 *   grad_v  the prefill of (psi: k, q, grad_out) on the time-reversed sequence, started
 *           from grad_S_final / gamma (its final state is G_0);
 *   grad_k  the prefill of (v, grad_out, psi(q)) under the identity map on the
 *           time-reversed sequence, started from grad_S_final^T / gamma;
 * plus element-wise kernels that apply psi and psi' and fold in the grad_S_final terms
 * of heads whose decay is below 2^-20 (for those heads the division by gamma is replaced
 * by the exact first three terms, the rest being below 2^-60).  The two time-reversed
 * passes run as reverse-mode prefills (la_prefill_args.reverse) when bf16 inputs, C = 64,
 * dk = dv = 128 and not ELU+1 with a decay; otherwise on reversed copies of their inputs,
 * their outputs reversed back.  Under ELU+1 with bf16 inputs, psi(k) and psi(q) enter
 * two passes as the value operand; they are split into bf16 hi and lo halves and those
 * passes run once per half, so that psi keeps about 16 bits as in the forward kernels.
 * The normalised form (o_t = n_t / d_t, n_t = psi(q_t) S_t, d_t = psi(q_t) . Z_t + eps)
 * has, with dn_t = grad_out_t / d_t and dd_t = -(grad_out_t . n_t) / d_t^2,
 *     grad_q_t = psi'(q_t) .* (S_t dn_t + Z_t dd_t),
 *     grad_k_t = psi'(k_t) .* (G_t v_t + g_t),   grad_v_t = G_t^T psi(k_t),
 *     G_t = psi(q_t) dn_t^T + gamma G_{t+1},  g_t = psi(q_t) dd_t + gamma g_{t+1}
 *     (G_{T-1}, g_{T-1} include grad_S_final, grad_Z_final),
 *     grad_S_init = gamma G_0,   grad_Z_init = gamma g_0.
 * The same three prefills compute S_t grad_out_t, G_t v_t (with the value psi(q_t) / d_t)
 * and grad_v (with the value dn_t, as bf16 hi and lo halves); decayed vector scans over
 * the tokens add Z_t (forward: it also forms d_t, dd_t from psi(q_t) . S_t grad_out_t,
 * and grad_q) and g_t (reverse).
 *
 *   q, k, v, grad_out  DEVICE, the forward's inputs and dL/dout, type `dtype`,
 *                      [B,H,T,dk] / [B,H,T,dk] / [B,H,T,dv] / [B,H,T,dv].
 *   grad_q, grad_k, grad_v  DEVICE outputs, the shapes of q, k, v, type per out_dtype;
 *                      must not overlap any input or each other.
 *   S_init             DEVICE float32 [B,H,dk,dv], the forward's initial state, or NULL.
 *   grad_S_final       DEVICE float32 [B,H,dk,dv] or NULL (zero).
 *   grad_S_init        DEVICE float32 [B,H,dk,dv] output, or NULL (not computed).
 *   The other fields as in la_prefill_args; every pass uses `algorithm`, `kernel_path`,
 *   `scan_mode` and `segment_chunks`.  Supported shapes: those of the prefill for both
 *   (dk, dv) and (dv, dk), with B*H*T*max(dk, dv) / 4 < 2^31.  Workspace: lin_attn_backward_workspace_bytes(), or NULL to
 *   allocate on the stream.  Asynchronous; arguments are checked before any launch.
 */
typedef struct la_backward_args {
  const void* q;
  const void* k;
  const void* v;
  const void* grad_out;
  void* grad_q;
  void* grad_k;
  void* grad_v;
  const float* S_init;        /* may be NULL */
  const float* grad_S_final;  /* may be NULL */
  float* grad_S_init;         /* may be NULL */
  int B, H;
  long long T;
  int dk, dv, C;
  int feature_map;            /* la_feature_map */
  const float* gamma;         /* HOST, H values, or NULL */
  int dtype;                  /* la_dtype of q, k, v, grad_out */
  int out_dtype;              /* la_out_dtype of grad_q, grad_k, grad_v */
  int scan_mode;
  int kernel_path;
  int algorithm;
  int segment_chunks;
  void* workspace;            /* DEVICE, 256-byte aligned, or NULL */
  size_t workspace_bytes;
  la_stream_t stream;
  /* The normalised form (normalize = 1; requires LA_FM_ELU1): o_t = n_t / d_t with
   * n_t = psi(q_t) S_t, d_t = psi(q_t) . Z_t + eps (the forward's eps).  The forward's
   * output is not needed: n_t and d_t are recomputed.  Z_init: the forward's initial
   * normaliser or NULL; grad_Z_final: dL/dZ_final or NULL; grad_Z_init: output dL/dZ_init
   * or NULL (all float32 [B,H,dk]). */
  int normalize;
  float eps;
  const float* Z_init;
  const float* grad_Z_final;
  float* grad_Z_init;
} la_backward_args;

int lin_attn_backward(const la_backward_args* args);

/* lin_attn_backward_timed -- lin_attn_backward with a CUDA event recorded before every
 * kernel (or group of small kernels) and after the last; synchronises the stream and
 * writes each one's device duration (milliseconds, launch order) to kernel_ms[0 ..] and
 * its name to kernel_names[0 ..] (static strings owned by the library: the prefill
 * kernels' names, "bwd_reverse_inputs", "bwd_prep_states", "bwd_fix_small_decay",
 * "bwd_finish_state", "bwd_reverse_outputs").  *n_kernels receives the count.  For
 * profiling; the results are identical to lin_attn_backward. */
int lin_attn_backward_timed(const la_backward_args* args, float* kernel_ms,
                            const char** kernel_names, int max_kernels, int* n_kernels);

/* Device workspace of lin_attn_backward for these arguments (the reversed copies of the
 * inputs, the passes' float32 outputs, the prefill workspace).  Pure host computation. */
size_t lin_attn_backward_workspace_bytes(const la_backward_args* args);

/*
 * lin_attn_gla_prefill -- gated linear attention ("Linear Attention and Retentive Networks
 * ...", Gated Linear Attention (GLA) and Hardware-Software Co-Design): the data-dependent
 * decay
 *     S_t = (alpha_t 1^T) (.) S_{t-1} + k_t^T v_t,     o_t = q_t S_t,
 * S_{-1} = S_init (or zero), with a gate alpha_t[i] in [0, 1] per token and key feature
 * (no feature map, no normalisation, as on that page).  The scan page's three kernels with
 * the decayed monoid made per feature: (a1, S1) + (a2, S2) = (a1 a2, diag(a2) S1 + S2), a
 * the product of the gates.  Within a chunk the score for tokens i <= j weighs feature f by
 * prod_{i<r<=j} alpha_r[f], the prefix is read out through prod_{r<=j} alpha_r; gate
 * products are powers of two of cumulative log2 gates (a gate below 2^-126 counts as
 * 2^-126).  Two paths:
 *   Tensor cores (default for bf16 inputs, C = 64, dk in {64, 128}, dv = 128 on sm_100):
 *     the segmented arrangement.  Per segment of chunks a fold into (a_s, S_s), an exclusive
 *     scan over segments, then a combine that walks each segment's chunks carrying the state
 *     in TMEM.  The scores, the prefix product and the state update are tcgen05 MMAs on the
 *     factored operands q (.) 2^(W+L) and k (.) 2^-(W+L) (a per-feature window offset W keeps
 *     every factor within 2^60), each split into bf16 hi + lo, so products keep ~16 bits.
 *     Chunks whose gates fall so fast that their own factors would leave that range (an
 *     average gate below ~0.5 over the chunk in some feature) take an exact CUDA-core pass
 *     for their intra-chunk scores.  Exact to float32 accumulation for any gates.
 *   CUDA cores (every other shape, or kernel_path LA_PATH_FMA): per-chunk float32 kernels,
 *     exact for any gates.
 *   q, k      DEVICE [B,H,T,dk], v DEVICE [B,H,T,dv], bf16 or float32 per `dtype`
 *   alpha     DEVICE float32 [B,H,T,dk]
 *   out       DEVICE [B,H,T,dv], type per out_dtype; must not overlap the inputs
 *   S_init    DEVICE float32 [B,H,dk,dv] or NULL;  S_final DEVICE float32 or NULL
 * Shapes: dk, dv multiples of 8 in [8, 128]; C in {16, 32, 64}; T >= 0.  Workspace:
 * lin_attn_gla_workspace_bytes() (one record of dk*dv + dk floats and one byte per chunk),
 * or NULL to allocate on the stream.  Asynchronous; arguments are checked before any
 * launch.
 */
typedef struct la_gla_args {
  const void* q;
  const void* k;
  const void* v;
  const float* alpha;
  void* out;
  float* S_final;
  const float* S_init;
  int B, H;
  long long T;
  int dk, dv, C;
  int dtype;              /* la_dtype of q, k, v */
  int out_dtype;          /* la_out_dtype of out */
  void* workspace;        /* DEVICE, 256-byte aligned, or NULL */
  size_t workspace_bytes;
  la_stream_t stream;
  /* la_kernel_path.  LA_PATH_AUTO: the tensor cores where their shape rule holds, else the
   * CUDA cores.  LA_PATH_TENSOR_CORE: the tensor cores or LA_ERR_UNSUPPORTED.  LA_PATH_FMA:
   * the CUDA cores. */
  int kernel_path;
  /* Tensor-core path: chunks per segment, 0 to choose automatically (about four segments
   * per SM, at most 64 chunks); at most 1024. */
  int segment_chunks;
} la_gla_args;

int lin_attn_gla_prefill(const la_gla_args* args);
size_t lin_attn_gla_workspace_bytes(int B, int H, long long T, int dk, int dv, int C);
/* lin_attn_gla_prefill with a CUDA event around each of its kernels; synchronises the
 * stream and writes their durations (ms, launch order: K1, K2, K3 on the CUDA cores;
 * gla_k1_seg, gla_scan, gla_k3_seg, the fix-up on the tensor cores) to kernel_ms. */
int lin_attn_gla_prefill_timed(const la_gla_args* args, float* kernel_ms, int max_kernels,
                               int* n_kernels);

/*
 * lin_attn_decode_step -- one recurrent step for every (b, h), the O(1) decode that the
 * prefill's final states feed ("The Recurrent Dual"; "B. Recurrent Representation").
 *   q, k      DEVICE bf16 [B,H,dk]   v DEVICE bf16 [B,H,dv]   out DEVICE bf16 [B,H,dv]
 *   S, Z      DEVICE float32 [B,H,dk,dv] / [B,H,dk], updated IN PLACE:
 *             S <- gamma S + psi(k) v^T, Z <- gamma Z + psi(k); then
 *             out = psi(q) S / (psi(q) . Z) (normalize) or psi(q) S.
 *             Z may be NULL when normalize == 0.
 * Shapes: dk, dv in [1, 256].  One kernel launch, no workspace.
 */
int lin_attn_decode_step(const void* q, const void* k, const void* v, void* out, float* S,
                         float* Z, int B, int H, int dk, int dv, int feature_map,
                         const float* gamma, int normalize, la_stream_t stream);

/* lin_attn_decode_step_f32 -- the same with float32 q, k, v and out. */
int lin_attn_decode_step_f32(const float* q, const float* k, const float* v, float* out,
                             float* S, float* Z, int B, int H, int dk, int dv,
                             int feature_map, const float* gamma, int normalize,
                             la_stream_t stream);

/* Reads and clears the device-side error word that kernels set when an internal check
 * or a bounded wait fails (0 = none).  Synchronises the current device.  Codes: 1 a TMA
 * load never landed, 2 an MMA or a hand-off between warps never completed (each after
 * about two seconds), 3 an internal shape check failed, 4 gated attention: gates the
 * tensor-core kernels cannot factor, 5 the deliberate wait of lin_attn_check_wait_timeout
 * gave up.  While the word is set, the tensor-core kernels launched afterwards skip their
 * work (so one failure costs one bounded wait, not one per CTA). */
int lin_attn_device_error(int* code);

/*
 * lin_attn_check_wait_timeout -- exercises the failure detection above without faulting
 * anything (no passage of the pages corresponds to it; it is a diagnostic).  Launches one
 * small kernel on `stream` in which one thread waits, with a limit of timeout_us
 * microseconds, on an mbarrier that nothing arrives on; the wait gives up, and the kernel
 * records code 5 in the device error word and returns.  Read and clear it with
 * lin_attn_device_error.  timeout_us in [1, 10^6]; LA_ERR_INVALID_ARGUMENT otherwise.
 */
int lin_attn_check_wait_timeout(unsigned int timeout_us, la_stream_t stream);

/* A static, human-readable name for a la_status value. */
const char* lin_attn_status_string(int status);

/*
 * lin_attn_scan_plan -- the shape of K2 for a scan over n elements (chunks, or segments of
 * the segmented algorithm), without touching a device.  "Log-Depth Chunked Linear-Attention
 * Scan" (Implementation notes, Verification) asks for a Blelloch or Hillis-Steele scan in
 * ceil(log2 n) rounds.  The log-depth mode (scan_mode LA_SCAN_LOGDEPTH) arranges it the
 * work-efficient way: n <= 2048 elements are cut into *groups (a power of two, at most 128)
 * of *per_group consecutive elements; each thread folds its group, a Hillis-Steele scan
 * combines the group folds in log2(*groups) rounds, and each thread re-scans its group
 * from the result.  Beyond 2048 elements, *segments segments of *segment_len (>= 16)
 * elements are folded first and that scan runs over the segment folds.  *depth receives
 * the longest chain of dependent combine steps: 2 per_group + log2 groups (+ 2 segment_len
 * with segments); for scan_mode LA_SCAN_SEQUENTIAL it is n.  Any output pointer may be
 * NULL.  Returns LA_ERR_INVALID_ARGUMENT for n < 1 or an unknown mode.
 */
int lin_attn_scan_plan(long long n, int scan_mode, int* segment_len, int* segments,
                       int* groups, int* per_group, long long* depth);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int lin_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LINATTN_H_ */
