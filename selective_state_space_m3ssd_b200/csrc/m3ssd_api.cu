// C-ABI entry points of libm3ssd: host-side validation and dispatch.
//
// Nothing here computes a step of the scan; it checks arguments, picks the
// kernel path and enqueues the launches on the caller's stream.  No memory is
// allocated and no host synchronisation is performed.
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/m3ssd.h"
#include "internal.h"

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Validation shared by the forward and the step.
m3ssd_status check_dims(const m3ssd_dims* d) {
  if (!d) return M3SSD_ERR_INVALID_ARG;
  if (d->batch < 0 || d->seqlen < 0) return M3SSD_ERR_INVALID_ARG;
  if (d->nheads < 1 || d->headdim < 1 || d->ngroups < 1) return M3SSD_ERR_INVALID_ARG;
  if (d->dstate < 2 || d->dstate % 2 != 0) return M3SSD_ERR_INVALID_ARG;
  if (d->nheads % d->ngroups != 0) return M3SSD_ERR_INVALID_ARG;
  if (d->x_dtype != M3SSD_F32 && d->x_dtype != M3SSD_BF16) return M3SSD_ERR_INVALID_ARG;
  if (d->reserved != 0) return M3SSD_ERR_INVALID_ARG;
  if ((d->flags & ~(uint32_t)M3SSD_CHECK_FINITE) != 0) return M3SSD_ERR_UNSUPPORTED;
  if (d->batch * d->nheads > INT32_MAX) return M3SSD_ERR_UNSUPPORTED;
  return M3SSD_OK;
}

// Shapes every kernel of this build can take (the sequential and step paths
// keep an (N, P) fp32 state in one CTA's shared memory).
bool general_shape_ok(const m3ssd_dims* d) {
  return d->dstate <= 256 && d->headdim <= 256 && d->dstate * d->headdim <= 16384;
}

m3ssd_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return M3SSD_OK;
  (void)cudaGetLastError();
  return M3SSD_ERR_CUDA;
}

// Shapes whose chunked bf16 forward may be split along the sequence (the split
// itself depends on the batch, heads, length and the device's SM count).
bool split_candidate(const m3ssd_dims* d) {
  return d && check_dims(d) == M3SSD_OK && d->x_dtype == M3SSD_BF16 && d->dstate == 128 &&
         d->headdim == 64 && (d->chunk == 0 || d->chunk == 64);
}

}  // namespace

extern "C" {

int m3ssd_abi_version(void) { return M3SSD_ABI_VERSION; }

const char* m3ssd_status_string(m3ssd_status s) {
  switch (s) {
    case M3SSD_OK: return "ok";
    case M3SSD_ERR_INVALID_ARG: return "invalid argument";
    case M3SSD_ERR_UNSUPPORTED: return "unsupported request";
    case M3SSD_ERR_WORKSPACE: return "workspace too small or misaligned";
    case M3SSD_ERR_CUDA: return "CUDA launch failed";
    case M3SSD_ERR_NONFINITE: return "non-finite input";
    case M3SSD_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

m3ssd_status m3ssd_nonfinite_outputs(void) {
  unsigned int f = 0;
  const m3ssd_status st = from_cuda(m3ssd::read_and_clear_nonfinite(&f));
  if (st != M3SSD_OK) return st;
  return f ? M3SSD_ERR_NONFINITE : M3SSD_OK;
}

m3ssd_status m3ssd_device_wait_timeouts(uint32_t* count) {
  if (!count) return M3SSD_ERR_INVALID_ARG;
  unsigned int n = 0, nb = 0, nm = 0, ng = 0;
  m3ssd_status st = from_cuda(m3ssd::read_and_clear_wait_timeouts(&n));
  if (st == M3SSD_OK) st = from_cuda(m3ssd::read_and_clear_bwd_wait_timeouts(&nb));
  if (st == M3SSD_OK) st = from_cuda(m3ssd::read_and_clear_mimo_wait_timeouts(&nm));
  if (st == M3SSD_OK) st = from_cuda(m3ssd::read_and_clear_gemm_wait_timeouts(&ng));
  unsigned int n32 = 0, nw = 0;
  if (st == M3SSD_OK) st = from_cuda(m3ssd::read_and_clear_chunk32_wait_timeouts(&n32));
  if (st == M3SSD_OK) st = from_cuda(m3ssd::read_and_clear_wide_wait_timeouts(&nw));
  unsigned int nm32 = 0, ns = 0;
  if (st == M3SSD_OK) st = from_cuda(m3ssd::read_and_clear_mimo32_wait_timeouts(&nm32));
  if (st == M3SSD_OK) st = from_cuda(m3ssd::read_and_clear_seg_wait_timeouts(&ns));
  *count = n + nb + nm + ng + n32 + nw + nm32 + ns;
  return st;
}

m3ssd_status m3ssd_test_set_wait_limit(uint64_t nanoseconds) {
  return from_cuda(m3ssd::set_wait_limit_ns(nanoseconds));
}

m3ssd_status m3ssd_test_drop_next_gram_signal(void) {
  return from_cuda(m3ssd::request_dropped_gram_signal());
}

size_t m3ssd_fwd_workspace_size(const m3ssd_dims* dims) {
  if (!split_candidate(dims)) return 0;
  const m3ssd::SplitPlan p =
      m3ssd::fwd_split_plan(dims->batch, dims->seqlen, dims->nheads, m3ssd::current_device_sms());
  return m3ssd::fwd_split_workspace_bytes(dims->batch, dims->nheads, p);
}

m3ssd_status m3ssd_test_fwd_split_plan(int64_t batch, int64_t seqlen, int64_t nheads,
                                       int32_t sms, int32_t* nseg, int32_t* segc) {
  if (!nseg || !segc || batch < 0 || seqlen < 0 || nheads < 0 || sms < 0)
    return M3SSD_ERR_INVALID_ARG;
  const m3ssd::SplitPlan p = m3ssd::fwd_split_plan(batch, seqlen, nheads, sms);
  *nseg = p.nseg;
  *segc = p.segc;
  return M3SSD_OK;
}

m3ssd_status m3ssd_fwd(const m3ssd_dims* dims, const void* X, const float* logdecay,
                       const float* beta, const float* gamma, const void* B, const void* C,
                       const float* theta, const float* D, const float* h0, void* Y, float* hT,
                       const m3ssd_fwd_extra* extra, void* workspace, size_t workspace_bytes,
                       void* stream) {
  m3ssd_status st = check_dims(dims);
  if (st != M3SSD_OK) return st;
  if (dims->chunk != 0 && dims->chunk != 64 && dims->chunk != 128 && dims->chunk != 256)
    return M3SSD_ERR_UNSUPPORTED;

  const bool bf16 = dims->x_dtype == M3SSD_BF16;
  const uintptr_t esz = bf16 ? 2 : 4;
  const bool has_tokens = dims->batch * dims->seqlen > 0;
  if (has_tokens && (!X || !logdecay || !gamma || !B || !C || !Y)) return M3SSD_ERR_INVALID_ARG;
  if (!aligned(X, esz) || !aligned(B, esz) || !aligned(C, esz) || !aligned(Y, esz))
    return M3SSD_ERR_INVALID_ARG;
  const void* f32ptrs[] = {logdecay, beta, gamma, theta, D, h0, hT};
  for (const void* p : f32ptrs)
    if (!aligned(p, 4)) return M3SSD_ERR_INVALID_ARG;

  m3ssd::FwdArgs a{};
  a.b = dims->batch; a.L = dims->seqlen; a.H = dims->nheads; a.P = dims->headdim;
  a.N = dims->dstate; a.G = dims->ngroups; a.chunk = dims->chunk; a.bf16 = bf16;
  a.X = X; a.logdecay = logdecay; a.beta = beta; a.gamma = gamma; a.B = B; a.C = C;
  a.theta = theta; a.D = D; a.h0 = h0; a.Y = Y; a.hT = hT;
  if (extra) {
    if (extra->bprevT && extra->bprevT == extra->bprev0) return M3SSD_ERR_INVALID_ARG;
    const void* eptrs[] = {extra->angle0, extra->xprev0, extra->bprev0,
                           extra->angleT, extra->xprevT, extra->bprevT};
    for (const void* p : eptrs)
      if (!aligned(p, 4)) return M3SSD_ERR_INVALID_ARG;
    a.angle0 = extra->angle0; a.xprev0 = extra->xprev0; a.bprev0 = extra->bprev0;
    a.angleT = extra->angleT; a.xprevT = extra->xprevT; a.bprevT = extra->bprevT;
  }

  const size_t need = m3ssd_fwd_workspace_size(dims);
  if (workspace_bytes < need || (need > 0 && (!workspace || !aligned(workspace, 256))))
    return M3SSD_ERR_WORKSPACE;

  const bool chunked = m3ssd::fwd_chunk_supported(a);
  const m3ssd::SplitPlan plan =
      need > 0 ? m3ssd::fwd_split_plan(a.b, a.L, a.H, m3ssd::current_device_sms())
               : m3ssd::SplitPlan{1, 0};
  const bool split = chunked && plan.nseg > 1 &&
                     m3ssd::fwd_split_workspace_bytes(a.b, a.H, plan) <= workspace_bytes;
  const bool chunked32 = !chunked && m3ssd::fwd_chunk32_supported(a);
  const bool chunked_wide = m3ssd::fwd_chunk_wide_supported(a);
  // chunks longer than 64 rows exist only as the bf16 tensor-core kernel
  if ((dims->chunk == 128 || dims->chunk == 256) && !chunked_wide) return M3SSD_ERR_UNSUPPORTED;
  if (!chunked && !chunked32 && !chunked_wide && !general_shape_ok(dims))
    return M3SSD_ERR_UNSUPPORTED;
  if (dims->batch == 0) return M3SSD_OK;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = from_cuda(split          ? m3ssd::launch_fwd_split(a, plan, workspace, s)
                 : chunked      ? m3ssd::launch_fwd_chunk(a, s)
                 : chunked_wide ? m3ssd::launch_fwd_chunk_wide(a, s)
                 : chunked32    ? m3ssd::launch_fwd_chunk32(a, s)
                                : m3ssd::launch_fwd_seq(a, s));
  if (st == M3SSD_OK && (dims->flags & M3SSD_CHECK_FINITE)) {
    st = from_cuda(m3ssd::launch_nonfinite_check(
        Y, dims->batch * dims->seqlen * dims->nheads * dims->headdim, bf16, s));
    if (st == M3SSD_OK && hT)
      st = from_cuda(m3ssd::launch_nonfinite_check(
          hT, dims->batch * dims->nheads * dims->dstate * dims->headdim, false, s));
  }
  return st;
}

m3ssd_status m3ssd_mimo_fwd(const m3ssd_dims* dims, int32_t rank, const void* X,
                            const float* logdecay, const float* beta, const float* gamma,
                            const void* B, const void* C, const float* theta, const float* D,
                            const float* h0, void* Y, float* hT, const m3ssd_fwd_extra* extra,
                            void* stream) {
  m3ssd_status st = check_dims(dims);
  if (st != M3SSD_OK) return st;
  if (dims->chunk != 0) return M3SSD_ERR_UNSUPPORTED;
  if (rank < 1) return M3SSD_ERR_INVALID_ARG;
  if (!m3ssd::mimo_shape_ok(dims->dstate, dims->headdim, rank)) return M3SSD_ERR_UNSUPPORTED;
  const bool bf16 = dims->x_dtype == M3SSD_BF16;
  const uintptr_t esz = bf16 ? 2 : 4;
  if (dims->batch * dims->seqlen > 0 && (!X || !logdecay || !gamma || !B || !C || !Y))
    return M3SSD_ERR_INVALID_ARG;
  if (!aligned(X, esz) || !aligned(B, esz) || !aligned(C, esz) || !aligned(Y, esz))
    return M3SSD_ERR_INVALID_ARG;
  const void* f32ptrs[] = {logdecay, beta, gamma, theta, D, h0, hT};
  for (const void* p : f32ptrs)
    if (!aligned(p, 4)) return M3SSD_ERR_INVALID_ARG;
  m3ssd::FwdArgs a{};
  if (extra) {
    if (extra->bprevT && extra->bprevT == extra->bprev0) return M3SSD_ERR_INVALID_ARG;
    const void* eptrs[] = {extra->angle0, extra->xprev0, extra->bprev0,
                           extra->angleT, extra->xprevT, extra->bprevT};
    for (const void* p : eptrs)
      if (!aligned(p, 4)) return M3SSD_ERR_INVALID_ARG;
    a.angle0 = extra->angle0; a.xprev0 = extra->xprev0; a.bprev0 = extra->bprev0;
    a.angleT = extra->angleT; a.xprevT = extra->xprevT; a.bprevT = extra->bprevT;
  }
  if (dims->batch == 0) return M3SSD_OK;
  a.b = dims->batch; a.L = dims->seqlen; a.H = dims->nheads; a.P = dims->headdim;
  a.N = dims->dstate; a.G = dims->ngroups; a.bf16 = bf16;
  a.X = X; a.logdecay = logdecay; a.beta = beta; a.gamma = gamma; a.B = B; a.C = C;
  a.theta = theta; a.D = D; a.h0 = h0; a.Y = Y; a.hT = hT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  m3ssd_status rs = from_cuda(m3ssd::launch_mimo_fwd(a, rank, s));
  if (rs == M3SSD_OK && (dims->flags & M3SSD_CHECK_FINITE)) {
    rs = from_cuda(m3ssd::launch_nonfinite_check(
        Y, dims->batch * dims->seqlen * dims->nheads * dims->headdim * rank, bf16, s));
    if (rs == M3SSD_OK && hT)
      rs = from_cuda(m3ssd::launch_nonfinite_check(
          hT, dims->batch * dims->nheads * dims->dstate * dims->headdim, false, s));
  }
  return rs;
}

m3ssd_status m3ssd_mimo_step(const m3ssd_dims* dims, int32_t rank, const void* x_t,
                             const float* logdecay_t, const float* beta_t, const float* gamma_t,
                             const void* B_t, const void* C_t, const float* theta_t,
                             const float* D, const m3ssd_cache* cache, void* y_t, void* stream) {
  m3ssd_status st = check_dims(dims);
  if (st != M3SSD_OK) return st;
  if (rank < 1) return M3SSD_ERR_INVALID_ARG;
  if (!m3ssd::mimo_shape_ok(dims->dstate, dims->headdim, rank)) return M3SSD_ERR_UNSUPPORTED;
  if (!cache) return M3SSD_ERR_INVALID_ARG;
  const bool bf16 = dims->x_dtype == M3SSD_BF16;
  const uintptr_t esz = bf16 ? 2 : 4;
  if (dims->batch > 0) {
    if (!x_t || !logdecay_t || !gamma_t || !B_t || !C_t || !y_t) return M3SSD_ERR_INVALID_ARG;
    if (!cache->angle || !cache->ssm || !cache->x_prev || !cache->b_prev)
      return M3SSD_ERR_INVALID_ARG;
  }
  if (!aligned(x_t, esz) || !aligned(B_t, esz) || !aligned(C_t, esz) || !aligned(y_t, esz))
    return M3SSD_ERR_INVALID_ARG;
  const void* f32ptrs[] = {logdecay_t, beta_t, gamma_t, theta_t, D,
                           cache->angle, cache->ssm, cache->x_prev, cache->b_prev};
  for (const void* p : f32ptrs)
    if (!aligned(p, 4)) return M3SSD_ERR_INVALID_ARG;
  if (dims->batch == 0) return M3SSD_OK;
  m3ssd::StepArgs a{};
  a.b = dims->batch; a.H = dims->nheads; a.P = dims->headdim; a.N = dims->dstate;
  a.G = dims->ngroups; a.bf16 = bf16;
  a.x_t = x_t; a.logdecay_t = logdecay_t; a.beta_t = beta_t; a.gamma_t = gamma_t;
  a.B_t = B_t; a.C_t = C_t; a.theta_t = theta_t; a.D = D;
  a.angle = cache->angle; a.ssm = cache->ssm; a.x_prev = cache->x_prev; a.b_prev = cache->b_prev;
  a.y_t = y_t;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  m3ssd_status rs = from_cuda(m3ssd::launch_mimo_step(a, rank, s));
  if (rs == M3SSD_OK && (dims->flags & M3SSD_CHECK_FINITE))
    rs = from_cuda(m3ssd::launch_nonfinite_check(
        y_t, dims->batch * dims->nheads * dims->headdim * rank, bf16, s));
  return rs;
}

size_t m3ssd_bwd_workspace_size(const m3ssd_dims* dims) {
  // The backward takes no flags: a flagged request needs nothing (m3ssd_bwd
  // refuses it).
  if (check_dims(dims) != M3SSD_OK || !general_shape_ok(dims) || dims->flags != 0) return 0;
  if (m3ssd::bwd_chunk_supported(dims->dstate, dims->headdim))
    return m3ssd::bwd_chunk_workspace_bytes(dims->batch, dims->seqlen, dims->nheads);
  if (m3ssd::bwd_split_supported(dims->dstate, dims->headdim))
    return m3ssd::bwd_split_workspace_bytes(dims->batch, dims->seqlen, dims->nheads,
                                            dims->headdim);
  return m3ssd::bwd_workspace_bytes(dims->batch, dims->seqlen, dims->nheads, dims->headdim,
                                    dims->dstate);
}

m3ssd_status m3ssd_bwd(const m3ssd_dims* dims, const void* X, const float* logdecay,
                       const float* beta, const float* gamma, const void* B, const void* C,
                       const float* theta, const float* D, const float* h0,
                       const m3ssd_fwd_extra* extra, const void* dY, const float* dhT,
                       const m3ssd_bwd_grads* grads, void* workspace, size_t workspace_bytes,
                       void* stream) {
  m3ssd_status st = check_dims(dims);
  if (st != M3SSD_OK) return st;
  if (!general_shape_ok(dims) || dims->flags != 0) return M3SSD_ERR_UNSUPPORTED;
  if (!grads) return M3SSD_ERR_INVALID_ARG;
  const bool bf16 = dims->x_dtype == M3SSD_BF16;
  const uintptr_t esz = bf16 ? 2 : 4;
  if (dims->batch * dims->seqlen > 0 &&
      (!X || !logdecay || !gamma || !B || !C || !dY || !grads->dX || !grads->dlogdecay ||
       !grads->dgamma || !grads->dB || !grads->dC))
    return M3SSD_ERR_INVALID_ARG;
  if (!aligned(X, esz) || !aligned(B, esz) || !aligned(C, esz) || !aligned(dY, esz))
    return M3SSD_ERR_INVALID_ARG;
  const void* f32ptrs[] = {logdecay, beta, gamma, theta, D, h0, dhT, grads->dX, grads->dlogdecay,
                           grads->dbeta, grads->dgamma, grads->dB, grads->dC, grads->dtheta,
                           grads->dD, grads->dh0, grads->dangle0, grads->dxprev0, grads->dbprev0};
  for (const void* p : f32ptrs)
    if (!aligned(p, 4)) return M3SSD_ERR_INVALID_ARG;
  m3ssd::BwdArgs a{};
  if (extra) {
    const void* eptrs[] = {extra->angle0, extra->xprev0, extra->bprev0};
    for (const void* p : eptrs)
      if (!aligned(p, 4)) return M3SSD_ERR_INVALID_ARG;
    a.angle0 = extra->angle0; a.xprev0 = extra->xprev0; a.bprev0 = extra->bprev0;
  }
  const size_t need = m3ssd_bwd_workspace_size(dims);
  if (workspace_bytes < need || (need > 0 && (!workspace || !aligned(workspace, 256))))
    return M3SSD_ERR_WORKSPACE;
  if (dims->batch == 0) return M3SSD_OK;
  a.b = dims->batch; a.L = dims->seqlen; a.H = dims->nheads; a.P = dims->headdim;
  a.N = dims->dstate; a.G = dims->ngroups; a.bf16 = bf16;
  a.X = X; a.logdecay = logdecay; a.beta = beta; a.gamma = gamma; a.B = B; a.C = C;
  a.theta = theta; a.D = D; a.h0 = h0; a.dY = dY; a.dhT = dhT;
  a.dX = grads->dX; a.dlogdecay = grads->dlogdecay; a.dbeta = grads->dbeta;
  a.dgamma = grads->dgamma; a.dB = grads->dB; a.dC = grads->dC; a.dtheta = grads->dtheta;
  a.dD = grads->dD; a.dh0 = grads->dh0; a.dangle0 = grads->dangle0; a.dxprev0 = grads->dxprev0;
  a.dbprev0 = grads->dbprev0; a.workspace = workspace;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (m3ssd::bwd_chunk_supported(a.N, a.P))
    return from_cuda(m3ssd::bwd_tc_supported(a) ? m3ssd::launch_bwd_tc(a, s)
                                                : m3ssd::launch_bwd_chunk(a, s));
  return from_cuda(m3ssd::bwd_split_supported(a.N, a.P) ? m3ssd::launch_bwd_split(a, s)
                                                         : m3ssd::launch_bwd_seq(a, s));
}

m3ssd_status m3ssd_step(const m3ssd_dims* dims, const void* x_t, const float* logdecay_t,
                        const float* beta_t, const float* gamma_t, const void* B_t,
                        const void* C_t, const float* theta_t, const float* D,
                        const m3ssd_cache* cache, void* y_t, void* stream) {
  m3ssd_status st = check_dims(dims);
  if (st != M3SSD_OK) return st;
  if (!general_shape_ok(dims)) return M3SSD_ERR_UNSUPPORTED;
  if (!cache) return M3SSD_ERR_INVALID_ARG;
  const bool bf16 = dims->x_dtype == M3SSD_BF16;
  const uintptr_t esz = bf16 ? 2 : 4;
  if (dims->batch > 0) {
    if (!x_t || !logdecay_t || !gamma_t || !B_t || !C_t || !y_t) return M3SSD_ERR_INVALID_ARG;
    if (!cache->angle || !cache->ssm || !cache->x_prev || !cache->b_prev)
      return M3SSD_ERR_INVALID_ARG;
  }
  if (!aligned(x_t, esz) || !aligned(B_t, esz) || !aligned(C_t, esz) || !aligned(y_t, esz))
    return M3SSD_ERR_INVALID_ARG;
  const void* f32ptrs[] = {logdecay_t, beta_t, gamma_t, theta_t, D,
                           cache->angle, cache->ssm, cache->x_prev, cache->b_prev};
  for (const void* p : f32ptrs)
    if (!aligned(p, 4)) return M3SSD_ERR_INVALID_ARG;
  if (dims->batch == 0) return M3SSD_OK;

  m3ssd::StepArgs a{};
  a.b = dims->batch; a.H = dims->nheads; a.P = dims->headdim; a.N = dims->dstate;
  a.G = dims->ngroups; a.bf16 = bf16;
  a.x_t = x_t; a.logdecay_t = logdecay_t; a.beta_t = beta_t; a.gamma_t = gamma_t;
  a.B_t = B_t; a.C_t = C_t; a.theta_t = theta_t; a.D = D;
  a.angle = cache->angle; a.ssm = cache->ssm; a.x_prev = cache->x_prev; a.b_prev = cache->b_prev;
  a.y_t = y_t;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = from_cuda(m3ssd::launch_step(a, s));
  if (st == M3SSD_OK && (dims->flags & M3SSD_CHECK_FINITE))
    st = from_cuda(m3ssd::launch_nonfinite_check(
        y_t, dims->batch * dims->nheads * dims->headdim, bf16, s));
  return st;
}

}  // extern "C"
