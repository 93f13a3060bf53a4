/*
 * m3ssd.h -- C ABI of libm3ssd, a B200-native (sm_100a) Mamba-3 SISO selective scan.
 *
 * The operation (sources, by page title and section):
 *   "TorchMamba" README, table "Models" (Mamba-3 SISO row) and "Math notes",
 *   paragraph "M3 SISO": the exponential-trapezoidal three-term recurrence
 *
 *       h_t = alpha_t h_{t-1} + beta_t Bbar_{t-1} x_{t-1}^T + gamma_t Bbar_t x_t^T
 *       y_t = Cbar_t^T h_t + D_h x_t
 *
 *   with alpha_t = exp(logdecay_t) and Bbar_t, Cbar_t equal to B_t, C_t rotated
 *   pairwise by the running data-dependent angle phi_t = angle0 + sum_{s<=t} theta_s
 *   (the "RoPE trick" for a complex state).  "VikramLex/mamba3-minimal",
 *   section "Two-SSD Decomposition": the beta term carries the previous step's
 *   B and x.  "TorchMamba" README, "Behavioral notes": lambda = 1 is the exact
 *   two-term path and theta absent is the real-only path; the Mamba-2 SSD scan
 *   is the lambda = 1, theta = 0 special case ("Reductions").
 *
 * Conventions fixed by this library where the pages are silent:
 *   - pair i is components (2i, 2i+1) and is rotated by theta index i;
 *   - R(phi) = [[cos phi, -sin phi], [sin phi, cos phi]] (counter-clockwise),
 *     applied to both B and C;
 *   - the running angle is inclusive: token t is rotated by phi_t, which
 *     already contains theta_t;
 *   - theta is taken as given (already multiplied by the step size);
 *   - head h reads B/C group g = h / (H / G);
 *   - h0 and hT are in the same absolute frame as Bbar (the cache frame);
 *   - angles written by the library (angleT, cache angle) are reduced to
 *     [-pi, pi] (the same rotation; it keeps fp32 angles precise over long runs).
 *
 * Layouts (row-major, contiguous, element strides implied by the shapes):
 *   X, Y        (b, L, H, P)    dtype x_dtype (fp32 or bf16)
 *   logdecay    (b, L, H)       fp32  (alpha = exp(logdecay))
 *   beta, gamma (b, L, H)       fp32
 *   B, C        (b, L, G, N)    dtype x_dtype
 *   theta       (b, L, H, N/2)  fp32
 *   D           (H)             fp32
 *   h0, hT      (b, H, N, P)    fp32
 *   cache:  angle (b, H, N/2), ssm (b, H, N, P), x_prev (b, H, P),
 *           b_prev (b, G, N) -- all fp32; b_prev holds B_{t-1} UNROTATED and
 *           is rotated at use by the stored angle phi_{t-1}.
 * Decode-step tensors drop the L axis.
 *
 * Ownership and execution: every pointer is a DEVICE pointer owned by the
 * caller.  The library allocates no memory, performs no host synchronisation
 * and enqueues all work on the given stream (a cudaStream_t passed as void*;
 * NULL is the legacy default stream).  Results are complete when the stream
 * reaches the enqueued work.  m3ssd_step is safe to capture in a CUDA graph.
 *
 * Errors: arguments are validated on the host before anything is enqueued;
 * a bad argument returns a status and enqueues nothing.  A launch failure
 * returns M3SSD_ERR_CUDA (the CUDA error is cleared).  Nothing aborts or traps.
 */
#ifndef M3SSD_H_
#define M3SSD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define M3SSD_ABI_VERSION 1

typedef enum {
  M3SSD_OK = 0,
  M3SSD_ERR_INVALID_ARG = 1,  /* NULL required pointer, odd N, H % G != 0, negative size, aliasing */
  M3SSD_ERR_UNSUPPORTED = 2,  /* valid request outside what this build implements (sizes, chunk, flags) */
  M3SSD_ERR_WORKSPACE = 3,    /* workspace smaller than m3ssd_fwd_workspace_size() or misaligned */
  M3SSD_ERR_CUDA = 4,         /* a CUDA launch failed */
  M3SSD_ERR_NONFINITE = 5,    /* m3ssd_nonfinite_outputs: a checked output held NaN or infinity */
  M3SSD_ERR_TIMEOUT = 6       /* reserved: a bounded device-side wait ran out */
} m3ssd_status;

typedef enum { M3SSD_F32 = 0, M3SSD_BF16 = 1 } m3ssd_dtype;

/* flags (m3ssd_dims.flags) */
/* M3SSD_CHECK_FINITE: after its kernels, m3ssd_fwd (and m3ssd_step,
 * m3ssd_mimo_fwd, m3ssd_mimo_step) scans the outputs it wrote -- Y and hT, or
 * y_t -- on the same stream for NaN or infinite values (from an input that was,
 * or from an intermediate that overflowed, e.g. a bf16 input beyond fp16's range
 * on the chunked path); m3ssd_nonfinite_outputs reports what the checks found.
 * It reads the outputs once more (about a fifth of the forward's bytes).  The
 * backward does not take the flag (M3SSD_ERR_UNSUPPORTED).  "Crate burn_mamba"
 * carries the same switch (DENY_NAN / DENY_INF). */
#define M3SSD_CHECK_FINITE 1u

typedef struct {
  int64_t batch;    /* b >= 0 */
  int64_t seqlen;   /* L >= 0 (ignored by m3ssd_step) */
  int64_t nheads;   /* H >= 1 */
  int64_t headdim;  /* P >= 1 */
  int64_t dstate;   /* N >= 2, even */
  int64_t ngroups;  /* G >= 1, H % G == 0 */
  int32_t chunk;    /* chunk length of the chunked forward: 0 = library choice (64),
                       64, or 128 / 256 (bf16, N = 128, P = 64 only; m3ssd_fwd) */
  int32_t x_dtype;  /* m3ssd_dtype of X, B, C, Y (and x_t, B_t, C_t, y_t) */
  uint32_t flags;   /* 0 or M3SSD_CHECK_FINITE */
  uint32_t reserved;/* must be 0 */
} m3ssd_dims;

/* Optional cache-shaped inputs and outputs of the forward, so that a forward
 * can start from a decode cache and hand one back (prefill -> decode).
 * Inputs may be NULL (read as zero); outputs may be NULL (not written).
 * angleT/xprevT may alias angle0/xprev0; bprevT must NOT alias bprev0
 * (several heads read a group's b_prev).  Note h0/hT live in m3ssd_fwd's own
 * arguments and may alias each other. */
typedef struct {
  const float* angle0;  /* (b, H, N/2): phi_{-1} */
  const float* xprev0;  /* (b, H, P):   x_{-1}   */
  const float* bprev0;  /* (b, G, N):   B_{-1}, unrotated */
  float* angleT;        /* (b, H, N/2): phi_{L-1} */
  float* xprevT;        /* (b, H, P):   x_{L-1} as fp32 */
  float* bprevT;        /* (b, G, N):   B_{L-1} as fp32, unrotated */
} m3ssd_fwd_extra;

typedef struct {
  float* angle;   /* (b, H, N/2) */
  float* ssm;     /* (b, H, N, P) */
  float* x_prev;  /* (b, H, P) */
  float* b_prev;  /* (b, G, N), unrotated */
} m3ssd_cache;

/* Bytes of device workspace m3ssd_fwd needs for these dims on the current
 * device: non-zero only when the chunked bf16 forward (N = 128, P = 64, chunk 0
 * or 64) splits each sequence into segments (see m3ssd_fwd), which depends on
 * batch, seqlen, nheads and the device's SM count, so query it on the device
 * that runs the call.  0 for invalid dims (m3ssd_fwd then reports the error)
 * and when no device is present. */
size_t m3ssd_fwd_workspace_size(const m3ssd_dims* dims);

/* The segment count and the chunks per segment that m3ssd_fwd would use for
 * batch x nheads sequences of seqlen tokens on a device with `sms` SMs
 * (*nseg = 1: no split).  Host arithmetic only; for tests and tuning.
 * M3SSD_ERR_INVALID_ARG for NULL outputs or negative sizes. */
m3ssd_status m3ssd_test_fwd_split_plan(int64_t batch, int64_t seqlen, int64_t nheads,
                                       int32_t sms, int32_t* nseg, int32_t* segc);

/*
 * Forward scan over a whole sequence ("TorchMamba" README, "Functional cores":
 * trap_rope_loop(X, logdecay, B, C, theta_dt, lam) -> (y, h)).
 *
 *   X, logdecay, gamma, B, C, Y : required when b*L > 0.
 *   beta   : NULL selects the exact two-term path (lambda = 1).
 *   theta  : NULL selects the real-only path (no rotation).
 *   D      : NULL means D = 0.
 *   h0     : NULL means a zero initial state.
 *   hT     : NULL means the final state is not written.
 *   extra  : NULL means no cache inputs/outputs (see m3ssd_fwd_extra).
 *   workspace, workspace_bytes : device scratch of at least
 *            m3ssd_fwd_workspace_size(dims) bytes, 256-byte aligned (may be
 *            NULL when that size is 0).
 *
 * Paths ("TorchMamba" README, "Math notes", M2: chunkwise intra-quadratic with
 * an inter-chunk carry):
 *   x_dtype = BF16, N = 128, P = 64, 16-byte aligned tensors: the chunked
 *     tensor-core forward (fp32 accumulation and state, fp16 operands converted
 *     from the bf16 inputs; X, B, C and their Gram products must stay inside
 *     fp16's range).  dims->chunk = 0 or 64 walks chunks of 64 rows (63 new
 *     tokens); 128 or 256 makes the intra-chunk quadratic form span 128 or 256
 *     rows (one CTA per SM instead of two).  With chunks of 64 rows and too few
     (b, h) sequences to fill the device (b*H at most two thirds of its SM
     count, at least 16 chunks), each sequence is cut into segments of at
     least 8 chunks: a pass builds every segment's state from a zero start
     and the linear recurrence links them (each segment's start state is the
     decayed previous start plus the previous segment's state, rotated to the
     absolute angle), then all segments run at once.  The result equals the
     unsplit walk up to fp32 rounding order; the workspace holds the segment
     states (64 KB per sequence and segment).
 *   x_dtype = F32, N = 128, P = 64, 16-byte aligned tensors: the chunked forward
 *     with every product on fp16 high and low operand parts (about 2^-22 of
 *     each term), chunk 0 or 64.
 *   every other valid request: the sequential fp32 forward (N <= 256,
 *     P <= 256, N*P <= 16384, else M3SSD_ERR_UNSUPPORTED); chunk 0 or 64.
 * A chunk of 128 or 256 outside the bf16 N = 128, P = 64 path returns
 * M3SSD_ERR_UNSUPPORTED.  Y is rounded once to x_dtype (round-to-nearest-even);
 * hT and the extra outputs are fp32.
 */
m3ssd_status m3ssd_fwd(const m3ssd_dims* dims, const void* X, const float* logdecay,
                       const float* beta, const float* gamma, const void* B, const void* C,
                       const float* theta, const float* D, const float* h0, void* Y, float* hT,
                       const m3ssd_fwd_extra* extra, void* workspace, size_t workspace_bytes,
                       void* stream);

/*
 * One decode step on a cache ("TorchMamba" README, "API reference": step(u_t,
 * cache) with Mamba3SisoCache(angle, ssm, x_prev, b_prev)):
 *   phi' = angle + theta_t;  Bbar_prev = R(angle) b_prev;  Bbar = R(phi') B_t;
 *   Cbar = R(phi') C_t;  ssm = alpha ssm + beta Bbar_prev x_prev^T + gamma Bbar x_t^T;
 *   y_t = Cbar^T ssm + D x_t;  then angle = phi', x_prev = x_t, b_prev = B_t.
 * x_t, y_t (b, H, P) and B_t, C_t (b, G, N) have dtype dims->x_dtype;
 * logdecay_t, beta_t, gamma_t (b, H) and theta_t (b, H, N/2) are fp32.
 * beta_t, theta_t, D may be NULL (zero).  dims->seqlen is ignored.
 * Limits: N <= 256, P <= 256, N*P <= 16384.  Capture-safe (no allocation, no sync).
 */
m3ssd_status m3ssd_step(const m3ssd_dims* dims, const void* x_t, const float* logdecay_t,
                        const float* beta_t, const float* gamma_t, const void* B_t,
                        const void* C_t, const float* theta_t, const float* D,
                        const m3ssd_cache* cache, void* y_t, void* stream);

/*
 * MIMO rank R forward ("TorchMamba" README, table "Models", row Mamba-3 MIMO:
 * a rank-R matmul update on a shared (N, P) state; "Functional cores":
 * mimo_loop with X (B,L,H,P,R) -> Y (B,L,H,P,R), h (B,H,N,P)):
 *   h_t = alpha_t h_{t-1} + beta_t sum_r Bbar_{t-1,r} x_{t-1,r}^T + gamma_t sum_r Bbar_{t,r} x_{t,r}^T
 *   y_{t,r} = Cbar_{t,r}^T h_t + D x_{t,r}
 * with every rank column of B and C rotated by the head's angle.  Layouts as
 * m3ssd_fwd with a trailing rank axis: X, Y (b, L, H, P, R); B, C
 * (b, L, G, N, R); extra->xprev0 / xprevT (b, H, P, R) and bprev0 / bprevT
 * (b, G, N, R); the state h0, hT stays (b, H, N, P).  1 <= rank <= 8, N <= 256,
 * P <= 256, N*P <= 16384 (else M3SSD_ERR_UNSUPPORTED).  Sequential fp32 state;
 * Y rounded once to x_dtype.  No workspace, no allocation, no synchronisation.
 */
m3ssd_status m3ssd_mimo_fwd(const m3ssd_dims* dims, int32_t rank, const void* X,
                            const float* logdecay, const float* beta, const float* gamma,
                            const void* B, const void* C, const float* theta, const float* D,
                            const float* h0, void* Y, float* hT, const m3ssd_fwd_extra* extra,
                            void* stream);

/*
 * One MIMO decode step on a cache whose x_prev is (b, H, P, R) and b_prev
 * (b, G, N, R) (angle and ssm as for m3ssd_step); x_t, y_t (b, H, P, R) and
 * B_t, C_t (b, G, N, R) have dtype dims->x_dtype.  Limits as m3ssd_mimo_fwd.
 * Two launches (the step, then b_prev <- B_t).  No allocation, no synchronisation.
 */
m3ssd_status m3ssd_mimo_step(const m3ssd_dims* dims, int32_t rank, const void* x_t,
                             const float* logdecay_t, const float* beta_t, const float* gamma_t,
                             const void* B_t, const void* C_t, const float* theta_t,
                             const float* D, const m3ssd_cache* cache, void* y_t, void* stream);

/* fp32 gradient outputs of m3ssd_bwd, each shaped like the matching input of
 * m3ssd_fwd (dB, dC, dbprev0 per group; dD per head).  dX, dlogdecay, dgamma,
 * dB, dC are required when b*L > 0; the others may be NULL (not written).  An
 * input passed to the forward as NULL is read as zero, and its gradient is the
 * derivative there. */
typedef struct {
  float* dX;         /* (b, L, H, P) */
  float* dlogdecay;  /* (b, L, H) */
  float* dbeta;      /* (b, L, H) */
  float* dgamma;     /* (b, L, H) */
  float* dB;         /* (b, L, G, N) */
  float* dC;         /* (b, L, G, N) */
  float* dtheta;     /* (b, L, H, N/2) */
  float* dD;         /* (H) */
  float* dh0;        /* (b, H, N, P) */
  float* dangle0;    /* (b, H, N/2) */
  float* dxprev0;    /* (b, H, P) */
  float* dbprev0;    /* (b, G, N) */
} m3ssd_bwd_grads;

/* Bytes of device workspace m3ssd_bwd needs for these dims (0 for invalid
 * dims, and for any flags, which the backward refuses); the size depends on
 * the path.  At N = 128, P = 64 it holds every
 * chunk-start state and angle (chunks of 63 tokens) and per-head shares of
 * the group-summed gradients: about 4 (b H ceil(L/63) (N P + N/2) +
 * 2 b L H N) bytes.  Other shapes keep a state checkpoint every 16 or 64
 * tokens, the states of one block per sequence and the same per-head (or
 * per-slice) shares. */
size_t m3ssd_bwd_workspace_size(const m3ssd_dims* dims);

/*
 * Backward of m3ssd_fwd: reverse-mode derivatives of the recurrence of the
 * "TorchMamba" README, "Math notes", M3 SISO.  Training through the scan is on
 * the pages: "mamba-rs" crate page, feature list (CUDA forward and backward
 * kernels); "TorchMamba" README, "Verification" (fp64 gradchecks per core).
 *
 * Takes the forward's inputs (same pointers, dtypes and NULL conventions;
 * extra supplies angle0, xprev0, bprev0 and its outputs are ignored), the
 * upstream gradients dY (b, L, H, P, dtype x_dtype) and dhT (b, H, N, P,
 * fp32, NULL = 0), and writes the fp32 gradients in *grads.  The cache outputs
 * angleT, xprevT and bprevT take no upstream gradient.
 *
 * The backward recomputes the forward.  At N = 128, P = 64 it works chunk by
 * chunk (one CTA per sequence: a forward pass stores the state and angle at
 * every chunk start, then each chunk's adjoint is a set of products, walking
 * the chunks in reverse): with bf16 X, B, C, dY (16-byte aligned, as theta)
 * the products run on the tensor cores with every fp32 operand split into a
 * bf16 high part and residual (about 2^-16 relative error per product term;
 * gradients within about 1e-3 of their RMS at L = 4096), otherwise in fp32.  At N = 128 with
 * another P a multiple of 16 it splits each sequence over P/16 CTAs of 16
 * state columns and sums the per-slice partials of the column-mixing
 * gradients afterwards; other shapes run one CTA per sequence token by
 * token.  Every sum (over slices, the heads of a group, the batch) runs in a
 * fixed order, so results are deterministic.  Limits as the sequential forward:
 * N <= 256, P <= 256, N*P <= 16384 (else M3SSD_ERR_UNSUPPORTED); dims->flags
 * must be 0 (else M3SSD_ERR_UNSUPPORTED).  workspace must hold
 * m3ssd_bwd_workspace_size(dims) bytes, 256-byte aligned (else
 * M3SSD_ERR_WORKSPACE); the size depends on the path.  No allocation, no
 * synchronisation.
 */
m3ssd_status m3ssd_bwd(const m3ssd_dims* dims, const void* X, const float* logdecay,
                       const float* beta, const float* gamma, const void* B, const void* C,
                       const float* theta, const float* D, const float* h0,
                       const m3ssd_fwd_extra* extra, const void* dY, const float* dhT,
                       const m3ssd_bwd_grads* grads, void* workspace, size_t workspace_bytes,
                       void* stream);

/*
 * m3ssd_bwd without a caller workspace, for callers that cannot allocate
 * device memory where they call the backward (code inside a CUDA graph
 * capture, or a runtime whose allocator may not be used from the launching
 * thread).  The scratch is a fixed 64 MiB device array inside the library,
 * reserved when its device code is loaded on a device and kept by every GPU
 * that loads the library until the process exits.  The pages have no
 * counterpart for this entry point; it is a convenience of this library.
 * Arguments and results are those of m3ssd_bwd.  Invalid dims return
 * m3ssd_bwd's status without touching the device; requests whose
 * m3ssd_bwd_workspace_size exceeds 64 MiB return M3SSD_ERR_UNSUPPORTED before
 * any device call.  The first call on a device (with that device current)
 * looks up the array's device address once (cudaGetSymbolAddress); make that
 * first call before any stream capture.  No call allocates.  Every call uses
 * the same array, which keeps the last call's contents, so calls that overlap
 * on the GPU race: issue them on one stream, or synchronise between streams.
 */
m3ssd_status m3ssd_bwd_noalloc(const m3ssd_dims* dims, const void* X, const float* logdecay,
                               const float* beta, const float* gamma, const void* B,
                               const void* C, const float* theta, const float* D,
                               const float* h0, const m3ssd_fwd_extra* extra, const void* dY,
                               const float* dhT, const m3ssd_bwd_grads* grads, void* stream);

/*
 * The Mamba-3 SISO block around the scan ("VikramLex/mamba3-minimal" README,
 * "Architecture", the Mamba3 SSM box; "TorchMamba" README, "API reference",
 * Mamba3SisoBlock with forward / prefill / step and its cache):
 *
 *   zx = u W_in^T                       in_proj, no bias
 *   [z | x | B | C | dt | lam | theta] = zx   (widths H P, H P, G N, G N, H, H, H N/2;
 *                                              heads outermost inside each part)
 *   Delta = softplus(dt + dt_bias), logdecay = -exp(A_log) Delta,
 *   lambda = sigmoid(lam), gamma = lambda Delta, beta = (1 - lambda) Delta exp(logdecay),
 *   theta_dt = Delta theta
 *   B'_h = B_g / sqrt(mean_n B_g^2 + eps) * B_norm_w + B_bias[h]   (QK-norm, then the
 *   C'_h likewise                                                   head-specific BC bias)
 *   y = scan(x, logdecay, beta, gamma, B', C', theta_dt, D)        (the SISO scan above,
 *                                                                    one B/C per head)
 *   out = (y * SiLU(z)) W_out^T          out_proj, no bias
 *
 * The projections are plain GEMMs on this library's tensor-core GEMM
 * (m3ssd_gemm_bf16: bf16 operands, fp32 accumulation, bf16 outputs); the rest
 * runs in this library's kernels too, the head biases inside the scan (added
 * in fp32 before the rotation).  u and out are bf16.  The block cache is an m3ssd_cache with
 * b_prev (b, G, N) holding the QK-normed group vector B_{t-1} (times its norm
 * weight, without the head bias) unrotated; the bias is added at use.
 */
typedef struct {
  int64_t batch;    /* b >= 0 */
  int64_t seqlen;   /* L >= 0 (ignored by m3ssd_block_step) */
  int64_t d_model;  /* >= 1, a multiple of 8 */
  int64_t nheads;   /* H >= 1 */
  int64_t headdim;  /* P >= 1, H * P a multiple of 8 */
  int64_t dstate;   /* N >= 2, even */
  int64_t ngroups;  /* G >= 1, H % G == 0 */
} m3ssd_block_dims;

typedef struct {
  const void* W_in;       /* (2HP + 2GN + 2H + H N/2, d_model) bf16, row-major */
  const void* W_out;      /* (d_model, H P) bf16, row-major */
  const float* dt_bias;   /* (H) */
  const float* A_log;     /* (H) */
  const float* D;         /* (H), may be NULL (zero) */
  const float* B_norm_w;  /* (N) */
  const float* C_norm_w;  /* (N) */
  const float* B_bias;    /* (H, N) */
  const float* C_bias;    /* (H, N) */
  float eps;              /* >= 0 */
} m3ssd_block_weights;

/* Bytes of device workspace m3ssd_block_fwd needs for these dims (with
 * seqlen = 1 it also covers m3ssd_block_step); 0 for invalid dims. */
size_t m3ssd_block_workspace_size(const m3ssd_block_dims* dims);

/*
 * Block forward over a sequence (Mamba3SisoBlock.forward; with cache_out it is
 * prefill).  u, out: (b, L, d_model) bf16.  cache_in (may be NULL: start from
 * zero) is the state the sequence continues from; cache_out (may be NULL) gets
 * the state after the last token and may be the same object as cache_in.
 * workspace: workspace_bytes >= m3ssd_block_workspace_size(dims), 256-byte
 * aligned, not read afterwards.  Errors as m3ssd_fwd.
 */
m3ssd_status m3ssd_block_fwd(const m3ssd_block_dims* dims, const m3ssd_block_weights* w,
                             const void* u, void* out, const m3ssd_cache* cache_in,
                             const m3ssd_cache* cache_out, void* workspace,
                             size_t workspace_bytes, void* stream);

/*
 * The block's projection GEMM ("VikramLex/mamba3-minimal" README,
 * "Architecture": in_proj and out_proj are plain linear maps), exported for
 * callers that compose the block themselves:
 *     D (M x N, row stride ldd elements) = A (M x K) W^T
 * A (M x K) and W (N x K): bf16, row-major (row stride K), 16-byte aligned,
 * K a multiple of 8; D: bf16, ldd >= N, 2-byte aligned (16-byte stores when D
 * is 16-byte aligned and ldd a multiple of 8).  fp32 accumulation on the
 * tensor cores, each output rounded once to bf16 (nearest even).  M, N, K up
 * to 2^31 - 1 with at most 2^31 - 1 output tiles of 128 x 256; M = 0 or N = 0
 * does nothing.  Other shapes or alignments: M3SSD_ERR_INVALID_ARG (or
 * M3SSD_ERR_CUDA for a tile count past that limit).  No allocation, no
 * synchronisation.
 */
m3ssd_status m3ssd_gemm_bf16(int64_t M, int64_t N, int64_t K, const void* A, const void* W,
                             void* D, int64_t ldd, void* stream);

/*
 * One decode step of the block (Mamba3SisoBlock.step): u_t, out_t (b, d_model)
 * bf16; cache (required) is advanced in place.  workspace as for
 * m3ssd_block_fwd with seqlen = 1.  Capturable in a CUDA graph.
 */
m3ssd_status m3ssd_block_step(const m3ssd_block_dims* dims, const m3ssd_block_weights* w,
                              const void* u_t, void* out_t, const m3ssd_cache* cache,
                              void* workspace, size_t workspace_bytes, void* stream);

/* Number of bounded device-side waits of the chunked forwards (SISO and
 * MIMO), the tensor-core backward and the projection GEMM that ran out since
 * the last call (a forward's CTA then stops and leaves its outputs unwritten;
 * the backward's and the GEMM's CTAs skip their remaining waits and leave their
 * outputs undefined); the count is then reset.  This call synchronises the current device
 * and must not be captured in a CUDA graph.  Returns M3SSD_ERR_INVALID_ARG for
 * a NULL pointer and M3SSD_ERR_CUDA if the device cannot be read. */
m3ssd_status m3ssd_device_wait_timeouts(uint32_t* count);

/*
 * Testing hooks for the failure path of the bounded device-side waits (no page
 * counterpart).  They copy to device variables synchronously, so they must not
 * be called while work of this library is in flight or being captured.
 *   m3ssd_test_set_wait_limit: the time limit of the chunked forward's bounded
 *     waits, in nanoseconds (0 restores the default of 2 s).
 *   m3ssd_test_drop_next_gram_signal: the next chunked forward that rotates
 *     (theta or angle0 given) and is not split into segments leaves out the
 *     completion signal of its first Gram product, so its compute warps'
 *     wait for it runs out: that launch counts one timeout in
 *     m3ssd_device_wait_timeouts and leaves its outputs undefined; the GPU
 *     context stays usable and later launches are unaffected.
 */
m3ssd_status m3ssd_test_set_wait_limit(uint64_t nanoseconds);
m3ssd_status m3ssd_test_drop_next_gram_signal(void);

/* The result of the M3SSD_CHECK_FINITE checks enqueued since the last call:
 * M3SSD_ERR_NONFINITE if any checked output held a NaN or an infinity, else
 * M3SSD_OK; the record is then cleared.  It synchronises the current device
 * and must not be captured in a CUDA graph; M3SSD_ERR_CUDA if the device
 * cannot be read. */
m3ssd_status m3ssd_nonfinite_outputs(void);

/* Static, human-readable name of a status. */
const char* m3ssd_status_string(m3ssd_status status);

/* M3SSD_ABI_VERSION of the loaded library. */
int m3ssd_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* M3SSD_H_ */
