// Internal launch interface shared by the C-ABI layer and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace m3ssd {

// Everything one forward launch needs; validated by the C-ABI layer.
struct FwdArgs {
  int64_t b, L, H, P, N, G;
  int chunk;
  bool bf16;  // X, B, C, Y are bf16 (else fp32)
  const void* X;
  const float* logdecay;
  const float* beta;   // nullable
  const float* gamma;
  const void* B;
  const void* C;
  const float* theta;  // nullable
  const float* D;      // nullable
  const float* h0;     // nullable
  void* Y;
  float* hT;           // nullable
  const float* angle0; // nullable
  const float* xprev0; // nullable
  const float* bprev0; // nullable
  float* angleT;       // nullable
  float* xprevT;       // nullable
  float* bprevT;       // nullable
  // Head-specific additive biases of B and C, (H, N) fp32, nullable: every use
  // of B (including the cache's bprev0) reads B + Bbias[h], likewise C.  Used by
  // the block (its QK-normed B, C per group plus a bias per head); the public
  // scan entry points leave them NULL.
  const float* Bbias;
  const float* Cbias;
  // Elements between consecutive tokens of X (0: H P, a dense (b, L, H, P)
  // tensor).  The block points X into its in_proj rows this way; only the
  // chunked kernel takes a stride (a multiple of 8).
  int64_t x_tok_stride;
  // The block's raw angle projection instead of theta (chunked kernel only):
  // theta(t, h, i) = Delta(t, h) theta16[t * theta16_tok_stride + h N/2 + i]
  // (bf16), with Delta = logdecay / -exp(A_log[h]) recovered from logdecay.
  const void* theta16;
  int64_t theta16_tok_stride;
  const float* A_log;
  // Sequence split of the chunked bf16 forward (0 or 1: one CTA walks each whole
  // sequence).  With nseg > 1, CTA (b h) nseg + k walks chunks [k segc,
  // min((k + 1) segc, chunks)) of sequence (b, h); segment k >= 1 starts from the
  // state hseg + ((b H + h)(nseg - 1) + k - 1) N P (fp32, (n, p)) and the angle
  // aseg + (same index) N / 2 that the segment pass and its combine step wrote,
  // and only the last segment writes hT and the cache outputs.
  int nseg, segc;
  const float* hseg;
  const float* aseg;
};

struct StepArgs {
  int64_t b, H, P, N, G;
  bool bf16;
  const void* x_t;
  const float* logdecay_t;
  const float* beta_t;   // nullable
  const float* gamma_t;
  const void* B_t;
  const void* C_t;
  const float* theta_t;  // nullable
  const float* D;        // nullable
  float* angle;
  float* ssm;
  float* x_prev;
  float* b_prev;
  void* y_t;
  const float* Bbias;  // nullable, as in FwdArgs
  const float* Cbias;  // nullable
};

// Everything one backward launch needs (gradients are fp32; the nullable
// outputs are not written when absent).
struct BwdArgs {
  int64_t b, L, H, P, N, G;
  bool bf16;  // X, B, C, dY are bf16 (else fp32)
  const void* X;
  const float* logdecay;
  const float* beta;    // nullable
  const float* gamma;
  const void* B;
  const void* C;
  const float* theta;   // nullable
  const float* D;       // nullable
  const float* h0;      // nullable
  const float* angle0;  // nullable
  const float* xprev0;  // nullable
  const float* bprev0;  // nullable
  const void* dY;
  const float* dhT;     // nullable
  float *dX, *dlogdecay, *dbeta, *dgamma, *dB, *dC, *dtheta, *dD, *dh0, *dangle0, *dxprev0,
      *dbprev0;
  void* workspace;      // bwd_workspace_bytes(...) bytes, 256-byte aligned
};

// Workspace of the sequential backward: state checkpoints, the states of one
// block per sequence, and per-head shares of the group-summed gradients.
size_t bwd_workspace_bytes(int64_t b, int64_t L, int64_t H, int64_t P, int64_t N);
cudaError_t launch_bwd_seq(const BwdArgs& a, cudaStream_t s);
// The backward with the state's columns split across CTAs (N = 128, P a
// multiple of 16): checkpoints and block states per (b, h, column slice), and
// per-slice partials of the column-summed gradients.
bool bwd_split_supported(int64_t N, int64_t P);
size_t bwd_split_workspace_bytes(int64_t b, int64_t L, int64_t H, int64_t P);
cudaError_t launch_bwd_split(const BwdArgs& a, cudaStream_t s);
// The chunked backward (N = 128, P = 64): one CTA per (b, h) walks chunks of 63
// tokens, forward for the chunk-start states, then in reverse; per-head shares
// of the group-summed gradients in the workspace.
bool bwd_chunk_supported(int64_t N, int64_t P);
// Workspace regions of the chunked backwards (byte offsets): chunk-start
// states (fp32, (p, n) per chunk) and angles, per-head dB and dC shares,
// per-head dbprev0 shares and per-(b, h) dD partials.
struct ChunkWs {
  size_t hs, phs, dBh, dCh, dbph, dDbh, total;
};
ChunkWs chunk_ws_layout(int64_t b, int64_t L, int64_t H);
// A 4-D TMA tensor map (d0 innermost) with a box of d0-extent `box0` by 64
// tokens; d2 (the token axis) is `tok` elements apart (0: dense, d0 d1).
bool encode_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1,
                uint64_t d2, uint64_t d3, uint64_t esz, uint32_t box0, CUtensorMapSwizzle sw,
                uint64_t tok = 0);

// Sums the per-head shares into dB, dC, dbprev0 and dD, in a fixed order.
cudaError_t launch_bwd_chunk_reduce(const BwdArgs& a, cudaStream_t s);
// The chunked backward on the tensor cores (bf16 X, B, C, dY; N = 128, P = 64;
// 16-byte aligned X, B, C, dY and theta); same workspace as the fp32 one.
bool bwd_tc_supported(const BwdArgs& a);
cudaError_t launch_bwd_tc(const BwdArgs& a, cudaStream_t s);
cudaError_t read_and_clear_bwd_wait_timeouts(unsigned int* count);
size_t bwd_chunk_workspace_bytes(int64_t b, int64_t L, int64_t H);
cudaError_t launch_bwd_chunk(const BwdArgs& a, cudaStream_t s);

// MIMO rank R (1..8): layouts as the SISO ones with a trailing rank axis on X,
// Y, B, C, x_prev, b_prev (and the extra cache inputs / outputs).
bool mimo_shape_ok(int64_t N, int64_t P, int64_t R);
cudaError_t launch_mimo_fwd(const FwdArgs& a, int64_t R, cudaStream_t s);
// Chunked bf16 tensor-core MIMO forward (N = 128, P = 64, R = 2, 4 or 8; 16-byte
// aligned X, B, C, Y, theta, h0, hT): 64 rows of (token, rank) per chunk.
bool fwd_chunk_mimo_supported(const FwdArgs& a, int64_t R);
cudaError_t launch_fwd_chunk_mimo(const FwdArgs& a, int64_t R, cudaStream_t s);
cudaError_t read_and_clear_mimo_wait_timeouts(unsigned int* count);
// The same for fp32 X, B, C, Y with fp16 high / low operand parts.
bool fwd_chunk_mimo32_supported(const FwdArgs& a, int64_t R);
cudaError_t launch_fwd_chunk_mimo32(const FwdArgs& a, int64_t R, cudaStream_t s);
cudaError_t read_and_clear_mimo32_wait_timeouts(unsigned int* count);
cudaError_t launch_mimo_step(const StepArgs& a, int64_t R, cudaStream_t s);

// Sequential fp32 forward: one CTA per (b, h), token by token.
cudaError_t launch_fwd_seq(const FwdArgs& a, cudaStream_t s);
// Chunked bf16 tensor-core forward (N = 128, P = 64).
cudaError_t launch_fwd_chunk(const FwdArgs& a, cudaStream_t s);
bool fwd_chunk_supported(const FwdArgs& a);
// Sequence split of that forward for launches with few (b, h) sequences: the
// number of segments a sequence is cut into (1: no split) and the chunks a
// segment holds, from the shape and the device's SM count; the workspace the
// split needs (0 without a split); and the split launch itself (the segment
// pass, the combine step and the chunked forward over every segment).
struct SplitPlan {
  int nseg, segc;
};
SplitPlan fwd_split_plan(int64_t b, int64_t L, int64_t H, int sms);
size_t fwd_split_workspace_bytes(int64_t b, int64_t H, const SplitPlan& p);
cudaError_t launch_fwd_split(const FwdArgs& a, const SplitPlan& p, void* workspace, cudaStream_t s);
cudaError_t read_and_clear_seg_wait_timeouts(unsigned int* count);
// SM count of the current device (0 when there is none).
int current_device_sms();
// Chunked fp32 forward on the tensor cores with fp16 high / low operand parts
// (fp32 X, B, C, Y; N = 128, P = 64; 16-byte aligned X, B, C, Y, theta, h0, hT).
// Chunked bf16 forward with chunks of 128 or 256 rows (FwdArgs::chunk), 64-row
// sub-tiles; same shapes and alignment as the 64-row kernel.
bool fwd_chunk_wide_supported(const FwdArgs& a);
cudaError_t launch_fwd_chunk_wide(const FwdArgs& a, cudaStream_t s);
cudaError_t read_and_clear_wide_wait_timeouts(unsigned int* count);
bool fwd_chunk32_supported(const FwdArgs& a);
cudaError_t launch_fwd_chunk32(const FwdArgs& a, cudaStream_t s);
cudaError_t read_and_clear_chunk32_wait_timeouts(unsigned int* count);
// Count of bounded device-side waits in the chunked forward that ran out since
// the last call; reading it synchronises the device and clears the count.
cudaError_t read_and_clear_wait_timeouts(unsigned int* count);
// Test settings of the chunked forward (synchronous copies to device symbols):
// the limit of its bounded waits (0 = 2 s), and a one-shot request that the
// next chunk walk drop its first Gram completion signal.
cudaError_t set_wait_limit_ns(unsigned long long ns);
cudaError_t request_dropped_gram_signal();
// The optional non-finite check: scans n elements (bf16 or fp32) at p on the
// stream and sets a device word when one is NaN or infinite; the host query
// reads and clears it (synchronising the device).
cudaError_t launch_nonfinite_check(const void* p, int64_t n, bool bf16, cudaStream_t s);
cudaError_t read_and_clear_nonfinite(unsigned int* flag);
// D (M x N, bf16, row stride ldd) = A (M x K) W^T on the tensor cores, with A
// (M x K) and W (N x K) bf16 row-major, 16-byte aligned, K a multiple of 8.
cudaError_t launch_gemm_bf16(int64_t M, int64_t N, int64_t K, const void* A, const void* W,
                             void* D, int64_t ldd, cudaStream_t s);
cudaError_t read_and_clear_gemm_wait_timeouts(unsigned int* count);
// Decode step (two launches: the state/outputs, then b_prev <- B_t).
cudaError_t launch_step(const StepArgs& a, cudaStream_t s);

}  // namespace m3ssd
