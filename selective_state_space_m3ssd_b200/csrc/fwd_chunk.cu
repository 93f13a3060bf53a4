// Chunked bf16 forward of the Mamba-3 SISO scan on the sm_100a tensor cores
// (tcgen05 MMA, TMEM accumulators), for N = 128, P = 64.
//
// One CTA owns one (b, h) sequence and walks its chunks in order, keeping the
// fp32 state h on chip for the whole sequence (no chunk state goes to HBM).
//
// Chunk layout.  Chunk c has Q = 64 source rows: row 0 is the token just
// before the chunk (t0 - 1, the carry-in of the trapezoid's beta term) and rows
// 1..63 are the chunk's own tokens t0 .. t0+62 (t0 = 63 c).  With the chunk-local
// sums (row 0 has cs_0 = 0, psi_0 = 0)
//     cs_r = sum_{k=1..r} logdecay_k,   psi_r = sum_{k=1..r} theta_k,
// the rotated vectors are Bbar_r = R(Phi_c + psi_r) B_r and Cbar_r likewise, with
// Phi_c = phi_{t0-1} (reduced to [-pi, pi]) carried from chunk to chunk.  The recurrence ("TorchMamba"
// README, "Math notes", M3 SISO: h_t = alpha_t h_{t-1} + beta_t Bbar_{t-1} x_{t-1}^T
// + gamma_t Bbar_t x_t^T) unrolled over the chunk reads, for output rows r = 1..63,
//     y_r   = exp(cs_r) Cbar_r^T h + sum_{u<=r} W(r,u) (Cbar_r^T Bbar_u) x_u + D x_r
//     h_end = exp(cs_63) h + sum_u W(63,u) Bbar_u x_u^T
//     W(r,r) = gamma_r,   W(r,u<r) = exp(cs_r - cs_{u+1}) (gamma_u alpha_{u+1} + beta_{u+1}),
// with gamma_0 := 0 (row 0's own gamma term belongs to the previous chunk), so
// column u = 0 carries exactly the beta boundary term: the gamma and beta terms
// form one mask ("TorchMamba" README: "the parallel mask is L = 1SS @ band").
//
// Tensor-core work per chunk (tcgen05.mma kind::f16, bf16 in, fp32 in TMEM),
// issued by one thread in this order and tracked by four mbarriers (G done; S
// done; Y1 done; Y2 done) so each buffer is reused as soon as its last reader
// finishes:
//   G  = Cbar Bbar^T                 M=64  N=64 K=128   (TMEM cols   0..63)
//   S  = Bbar^T (W_end o X)          M=128 N=64 K=64    (TMEM cols 192..255)
//   Y1 = Cbar h 2^k                  M=64  N=64 K=128   (TMEM cols  64..127)
//   Y2 = (W o G) X                   M=64  N=64 K=64    (TMEM cols 128..191); in the
//        instances with the block's head biases the masked Gram is an fp16 high
//        part and residual (K=64 x2): there C'.B' is about N for every pair, so
//        M is large everywhere and its own rounding would otherwise dominate
// with fp16 operands: their 11 significant bits keep the large diagonal terms
// gamma_r (Cbar_r . Bbar_r) x_r within about 2^-12, where bf16 rotated
// operands gave 2^-9 of them.  X is converted exactly (bf16 values in fp16's
// normal range), and the fp16 copy of the state h is scaled by a power of two
// 2^k chosen from its largest element, so that it neither overflows nor loses
// precision to subnormals; the epilogue divides Y1 by 2^k.
// and y = exp(cs) 2^-k Y1 + Y2 + D x, h = exp(cs_63) h + S on the SIMT pipes, where the
// decay/angle cumsums, sincos, rotations and the mask also run.  Operand tiles
// live in shared memory in the 128-byte-swizzled canonical layouts: K-major rows
// of 128 B for Cbar, Bbar and the mask; MN-major 64-element atoms for X, h,
// W_end o X and Bbar as S's operand.  The inputs of a chunk (theta, B, C, X) arrive by TMA (4-D tensor
// maps over (inner, head or group, token, batch), so the carry-in row of the
// first chunk and the rows past the end are zero-filled by the hardware, and
// the 128-byte swizzle of the operand layouts is written by the copy itself).
// Two CTAs share an SM (about 100 KB of shared memory and 256 TMEM columns each).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <atomic>
#include <mutex>

#include "chunk_common.cuh"
#include "common.cuh"
#include "internal.h"
#include "tc5.cuh"

namespace m3ssd {

// Number of bounded device-side waits that ran out (read by the host query).
__device__ unsigned int g_chunk_wait_timeouts;
// The limit of the bounded waits of the testing instance of the kernel in
// nanoseconds (host-set between launches; 0: the default 2 s).  That instance
// runs only for a launch requested through request_dropped_gram_signal(): its
// first CTA leaves its first Gram product's completion signal out, so that the
// compute warps' bounded wait on it runs out (no fault, no hang).
__device__ unsigned long long g_wait_limit_ns;
// Host side: the next launch of the plain rotating instance runs the testing one.
std::atomic<bool> g_test_launch_requested{false};

namespace {

using namespace chunk;

constexpr int kCtrlWarp = 8;                 // the control warp
constexpr int kThreads = 32 * (kCtrlWarp + 1);  // 8 compute warps + 1 control warp
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColG = 0, kColY1 = 64, kColY2 = 128, kColS = 192;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // an mbarrier wait gives up after 2 s
constexpr uint32_t kIdescG = tc5::idesc_f16(64, 64, false, false);   // G
constexpr uint32_t kIdescY = tc5::idesc_f16(64, 64, false, true);    // Y1, Y2
constexpr uint32_t kIdescS = tc5::idesc_f16(128, 64, true, true);    // S

typedef __nv_bfloat16 bf16;

struct Smem {
  union {
    float theta[Q][NH];        // raw theta of the chunk (phase R1 only)
    struct {
      uint8_t wx[Q * 128];     // W_end o X in fp16 (phase R2 .. S MMA)
      uint8_t ml[Q * 128];     // the masked Gram's fp16 residual (bias instances, .. Y2)
    } t;
  } u;
  uint8_t B[2 * kAtom];        // raw B, then Bbar (fp16)
  uint8_t C[2 * kAtom];        // raw C, then Cbar (fp16)
  uint8_t X[2][Q * 128];       // X rows of chunks c, c+1 (row 0 = carry-in token), fp16 from R2
  uint8_t M[Q * 128];          // masked Gram W o G in fp16 (its residual: u.t.ml)
  uint8_t Hs[NS * 128];        // fp16 copy of h 2^k for the state-to-output product
  float hmax[8];               // per-warp max |h| (the scale k of Hs)
  ChunkParams prm[2];
  float segtot[8][NH];
  float Phi[NH];               // absolute angle at the chunk start, in [-pi, pi]
  float nPhi[NH];              // the same for the next chunk
  uint64_t mbar[4];            // G done; Y1 (and S) done; Y2 done; S done
  uint64_t lmbar;              // TMA loads of the next chunk
  uint32_t tmem;
  uint32_t err;
};
// two CTAs per SM: 228 KB of shared memory, 1 KB of it reserved per CTA, plus the
// 1 KB alignment slack of each CTA's dynamic block
static_assert(2 * (sizeof(Smem) + 1024 + 1024) <= 233472, "two CTAs per SM");

// Tensor maps of the chunk inputs, built on the host for each launch.
struct TmaMaps {
  CUtensorMap theta;  // fp32 (pair, head, token, batch), box 64 x 1 x 64 x 1, no swizzle
                      // (bf16 in the raw-angle variant)
  CUtensorMap B;      // bf16 (n, group, token, batch), box 64 x 1 x 64 x 1, 128-byte swizzle
  CUtensorMap C;      // same as B
  CUtensorMap X;      // bf16 (p, head, token, batch), box 64 x 1 x 64 x 1, 128-byte swizzle
};

template <bool ROT, bool BIAS, bool TH16, bool TEST, bool SEG>
__global__ void __launch_bounds__(kThreads, 2)
    fwd_chunk_kernel(FwdArgs a, const __grid_constant__ TmaMaps tm) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // operand tiles need a 1024-byte aligned shared-space address
  const uint32_t raw_addr = tc5::saddr(smem_raw);
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // the testing instance takes the host-set limit; the others keep the constant
  const uint64_t wait_ns = (TEST && g_wait_limit_ns) ? g_wait_limit_ns : kWaitLimitNs;
  // warps 0..7 compute; warp 8 (kCtrlWarp) issues the TMA copies and the tensor-core
  // products and prepares the next chunk's scalars
  const bool ctrl = warp == kCtrlWarp;
  const bool ctrl_lead = tid == kCtrlWarp * 32;
  const int64_t H = a.H, L = a.L, G = a.G;
  // CTA (b H + h) nseg + k walks segment k of sequence (b, h): chunks c_lo .. c_hi - 1
  // (the instances that never split keep the single-segment arithmetic constant)
  const int nseg = SEG ? a.nseg : 1;
  const int64_t bh = blockIdx.x / nseg;
  const int seg = (int)(blockIdx.x - bh * nseg);
  const int64_t b = bh / H, h = bh % H, g = h / (H / G);
  const int nCt = (int)((L + QT - 1) / QT);
  const int c_lo = nseg > 1 ? seg * a.segc : 0;
  const int c_hi = nseg > 1 ? min(c_lo + a.segc, nCt) : nCt;
  const bool seg_first = seg == 0, seg_last = seg == nseg - 1;
  // the start state and angle: the caller's for the first segment, else the
  // combine step's
  const int64_t su = bh * (nseg - 1) + seg - 1;
  const float* h0p = seg_first ? (a.h0 ? a.h0 + bh * NS * PD : nullptr) : a.hseg + su * NS * PD;
  const float* ang0 = seg_first ? (a.angle0 ? a.angle0 + bh * NH : nullptr) : a.aseg + su * NH;
  const bf16* Xg = static_cast<const bf16*>(a.X);
  const bf16* Bg = static_cast<const bf16*>(a.B);
  bf16* Yg = static_cast<bf16*>(a.Y);
  const float Dh = a.D ? a.D[h] : 0.f;
  const uint32_t aB = tc5::saddr(sm.B), aC = tc5::saddr(sm.C);
  const uint32_t aX0 = tc5::saddr(sm.X[0]);
  const uint32_t aM = tc5::saddr(sm.M), aH = tc5::saddr(sm.Hs);
  const uint32_t aWX = tc5::saddr(sm.u.t.wx);
  const uint32_t aT = tc5::saddr(&sm.u.theta[0][0]);

  bf16* const Y_seq = Yg + (b * L * H + h) * PD;
  const int64_t xstride_t = H * PD;  // Y elements per token
  const int64_t xtok = a.x_tok_stride ? a.x_tok_stride : H * PD;  // X elements per token
  // TMA issue (control thread): chunk c's rows start at token c*QT - 1
  const bool has_theta = (TH16 ? a.theta16 : static_cast<const void*>(a.theta)) != nullptr;  // ROT without theta: rotation by angle0 only
  const uint32_t chunk_bytes = (ROT && has_theta ? (TH16 ? 8192u : 16384u) : 0u) + 2u * 16384u + 8192u;
  // the raw-angle variant's 1 / A_h (Delta = logdecay / A_h)
  const float inv_a = TH16 ? -1.f / expf(a.A_log[h]) : 0.f;
  auto tma_theta = [&](int c) {
    tc5::tma_load_4d(aT, &tm.theta, &sm.lmbar, 0, (int)h, c * QT - 1, (int)b);
  };
  auto tma_bc = [&](int c, const CUtensorMap* map, uint32_t base) {
    tc5::tma_load_4d(base, map, &sm.lmbar, 0, (int)g, c * QT - 1, (int)b);
    tc5::tma_load_4d(base + kAtom, map, &sm.lmbar, 64, (int)g, c * QT - 1, (int)b);
  };
  auto tma_x = [&](int c) {
    tc5::tma_load_4d(aX0 + (uint32_t)(c & 1) * (Q * 128), &tm.X, &sm.lmbar, 0, (int)h, c * QT - 1,
                     (int)b);
  };

  // the control warp keeps logdecay / beta / gamma of rows lane and lane + 32 of
  // the next chunk in registers
  float pld[2], pbe[2], pga[2];
  auto load_params = [&](int c) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int r = lane + 32 * k;
      const int64_t t = (int64_t)c * QT - 1 + r;
      const bool ok = r > 0 && t < L;  // row 0 (carry-in) has a = gamma = beta = 0 here
      const int64_t idx = (b * L + (ok ? t : 0)) * H + h;
      pld[k] = ok ? a.logdecay[idx] : 0.f;
      pga[k] = ok ? a.gamma[idx] : 0.f;
      pbe[k] = (ok && a.beta) ? a.beta[idx] : 0.f;
    }
  };

  // ---- prologue -------------------------------------------------------------
  if (warp == 0) tc5::tmem_alloc(&sm.tmem, kTmemCols);
  if (ctrl_lead) {
    tc5::mbar_init(&sm.mbar[0], 1);
    tc5::mbar_init(&sm.mbar[1], 1);
    tc5::mbar_init(&sm.mbar[2], 1);
    tc5::mbar_init(&sm.mbar[3], 1);
    tc5::mbar_init(&sm.lmbar, 1);
    tc5::fence_mbar_init();
    sm.err = 0;
  }
  __syncthreads();  // mbarriers initialised
  if (ctrl_lead) {
    tc5::mbar_arrive_expect_tx(&sm.lmbar, chunk_bytes);
    if (ROT && has_theta) tma_theta(c_lo);
    tma_bc(c_lo, &tm.B, aB);
    tma_bc(c_lo, &tm.C, aC);
    tma_x(c_lo);
  }
  if (ctrl) {
    load_params(c_lo);
    chunk_params(sm.prm[c_lo & 1], pld, pbe, pga, lane, inv_a);
    if (c_lo + 1 < c_hi) load_params(c_lo + 1);
  }
  // row 0 of chunk 0 is the cache's previous token (the TMA zero-fills it; it is
  // patched once that copy has landed)
  const bool patch_row0 = seg_first && (a.bprev0 != nullptr || a.xprev0 != nullptr);
  const float bp0 = (patch_row0 && tid < NS && a.bprev0) ? a.bprev0[(b * G + g) * NS + tid] : 0.f;
  const float xp0 = (patch_row0 && tid < PD && a.xprev0) ? a.xprev0[bh * PD + tid] : 0.f;
  if (ROT && tid < NH) sm.Phi[tid] = wrap_angle(ang0 ? ang0[tid] : 0.f);

  // state fragment (compute warps): row n = 32 (warp % 4) + lane, columns cb .. cb + 31.
  // Between chunks the fp32 state lives in TMEM, in the columns of the state
  // product S: before chunk c it holds exp(cs_63(c)) h, and S accumulates onto it,
  // so the product leaves h after chunk c there; the registers hold it only while
  // its scaled fp16 copy and the next decay are applied.
  const int n_row = 32 * (warp & 3) + lane, cb = 32 * ((warp >> 2) & 1);
  float hs[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) hs[j] = 0.f;
  if (!ctrl && h0p) {
    const float4* src = reinterpret_cast<const float4*>(h0p + n_row * PD + cb);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 v = src[j];
      hs[4 * j] = v.x; hs[4 * j + 1] = v.y; hs[4 * j + 2] = v.z; hs[4 * j + 3] = v.w;
    }
  }
  // fp16 copy of h scaled by 2^kexp, kexp from the largest |h| of the CTA (compute
  // warps only; one named barrier)
  int kexp = 0;
  auto store_state_f16 = [&](const float (&hs)[32]) {
    float m4[4] = {0.f, 0.f, 0.f, 0.f};  // four independent chains
#pragma unroll
    for (int j = 0; j < 32; ++j) m4[j & 3] = fmaxf(m4[j & 3], fabsf(hs[j]));
    float m = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) sm.hmax[warp] = m;
    asm volatile("bar.sync 2, %0;" ::"n"(32 * kCtrlWarp) : "memory");
    m = sm.hmax[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) m = fmaxf(m, sm.hmax[w]);
    // m < 2^e, e = biased exponent - 126 for a normal m (a subnormal m reads as
    // e = -126, which the clamp maps to 100, as an exact frexp would)
    const int e = (int)((__float_as_uint(m) >> 23) & 0xffu) - 126;
    kexp = m > 0.f ? min(max(14 - e, -100), 100) : 0;
    const float sc = __uint_as_float((uint32_t)(127 + kexp) << 23);  // 2^kexp
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 v;
      v.x = pack_h2(sc * hs[8 * q + 0], sc * hs[8 * q + 1]);
      v.y = pack_h2(sc * hs[8 * q + 2], sc * hs[8 * q + 3]);
      v.z = pack_h2(sc * hs[8 * q + 4], sc * hs[8 * q + 5]);
      v.w = pack_h2(sc * hs[8 * q + 6], sc * hs[8 * q + 7]);
      *reinterpret_cast<uint4*>(sm.Hs + off1(n_row, cb + 8 * q)) = v;
    }
  };
  if (!ctrl) store_state_f16(hs);
  tc5::fence_proxy_async();
  tc5::fence_before_sync();
  __syncthreads();
  tc5::fence_after_sync();
  const uint32_t tmem = sm.tmem;
  // this warp's TMEM lane quarter (rows of the M=64 and M=128 accumulators)
  const uint32_t tlane = (uint32_t)(32 * (warp & 3)) << 16;
  // exp(cs_63) h for the first chunk's state product
  auto store_state_tmem = [&](const float (&hv)[32], float scale) {
    uint32_t w[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) w[j] = __float_as_uint(scale * hv[j]);
    tc5::st_32x32b_x32(tmem + tlane + kColS + (uint32_t)cb, w);
    tc5::wait_st();
  };
  if (!ctrl) store_state_tmem(hs, sm.prm[c_lo & 1].eE);
  // head biases of B and C for this thread's elements 4 lane .. 4 lane + 3 of a
  // row (real parts: elements 4 lane, 4 lane + 2; imaginary: 4 lane + 1, 4 lane + 3)
  const bool has_bbias = BIAS && a.Bbias != nullptr, has_cbias = BIAS && a.Cbias != nullptr;
  float2 bbr = make_float2(0.f, 0.f), bbi = bbr, cbr = bbr, cbi = bbr;
  if (has_bbias && !ctrl) {
    const float4 v = *reinterpret_cast<const float4*>(a.Bbias + h * NS + 4 * lane);
    bbr = make_float2(v.x, v.z);
    bbi = make_float2(v.y, v.w);
  }
  if (has_cbias && !ctrl) {
    const float4 v = *reinterpret_cast<const float4*>(a.Cbias + h * NS + 4 * lane);
    cbr = make_float2(v.x, v.z);
    cbi = make_float2(v.y, v.w);
  }

  // ---- chunk walk -------------------------------------------------------------
  for (int c = c_lo; c < c_hi; ++c) {
    const int64_t tbase = (int64_t)c * QT - 1;  // token of row 0
    const uint32_t par = (uint32_t)((c - c_lo) & 1);
    const ChunkParams& P = sm.prm[c & 1];
    const uint8_t* Xs = sm.X[c & 1];
    const uint32_t aX = aX0 + (uint32_t)(c & 1) * (Q * 128);
    if (tid == 0 && !tc5::mbar_wait(&sm.lmbar, par, wait_ns)) sm.err = 1;
    tc5::fence_before_sync();
    __syncthreads();  // S1: theta, B, C, X of this chunk are in shared memory; the
                      // previous chunk's accumulators and operands are consumed
    tc5::fence_after_sync();
    if (sm.err) {
      // let the copies and the previous chunk's products in flight land before
      // the CTA frees TMEM and exits (Y2 is that chunk's last commit; it covers
      // every product the control thread issued before it)
      (void)tc5::mbar_wait(&sm.lmbar, par, wait_ns);
      if (c > c_lo) (void)tc5::mbar_wait(&sm.mbar[2], par ^ 1u, wait_ns);
      break;
    }

    if (ctrl) {
      // ===================== control warp ======================================
      if (ctrl_lead && c + 1 < c_hi) {
        tc5::mbar_arrive_expect_tx(&sm.lmbar, chunk_bytes);
        tma_x(c + 1);
      }
      if (c + 1 < c_hi) {
        chunk_params(sm.prm[(c + 1) & 1], pld, pbe, pga, lane, inv_a);
        if (c + 2 < c_hi) load_params(c + 2);
      }
      // descriptors of the operand tiles: an offset inside a tile only adds
      // (offset >> 4) to the start-address field (shared addresses stay below 256 KB)
      const uint64_t dC = tc5::desc_sw128(aC, 16, 1024), dB = tc5::desc_sw128(aB, 16, 1024);
      const uint64_t dH = tc5::desc_sw128(aH, kAtom, 1024), dX = tc5::desc_sw128(aX, kAtom, 1024);
      const uint64_t dBm = tc5::desc_sw128(aB, kAtom, 1024), dWX = tc5::desc_sw128(aWX, kAtom, 1024);
      const uint64_t dM = tc5::desc_sw128(aM, 16, 1024);
      const uint64_t dMl = tc5::desc_sw128(tc5::saddr(sm.u.t.ml), 16, 1024);
      __syncthreads();  // S3: Cbar, Bbar, X, W_end o X ready
      if (ctrl_lead) {
        tc5::fence_after_sync();
        // G = Cbar Bbar^T (both K-major), K = 128 in 8 steps of 16
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint64_t ko = (uint64_t)(((j >> 2) * kAtom + (j & 3) * 32) >> 4);
          tc5::mma_bf16(tmem + kColG, dC + ko, dB + ko, kIdescG, j > 0);
        }
        // the testing instance's first CTA leaves its first Gram signal out
        if (!(TEST && c == c_lo && blockIdx.x == 0)) tc5::commit(&sm.mbar[0]);
        // S = Bbar^T (W_end o X) (A and B MN-major), K = 64 source rows
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint64_t kofs = (uint64_t)(j * (2048 >> 4));
          tc5::mma_bf16(tmem + kColS, dBm + kofs, dWX + kofs, kIdescS, true);
        }
        tc5::commit(&sm.mbar[3]);
        // Y1 = Cbar h (h MN-major: K = n, rows of 128 B)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint64_t ko = (uint64_t)(((j >> 2) * kAtom + (j & 3) * 32) >> 4);
          tc5::mma_bf16(tmem + kColY1, dC + ko, dH + (uint64_t)(j * (2048 >> 4)), kIdescY, j > 0);
        }
        tc5::commit(&sm.mbar[1]);
        // the Gram and S consume Bbar: refill it for the next chunk before joining S4
        if (c + 1 < c_hi) {
          if (!tc5::mbar_wait(&sm.mbar[3], par, wait_ns)) sm.err = 1;
          tma_bc(c + 1, &tm.B, aB);
        }
      }
      __syncthreads();  // S4: M ready
      if (ctrl_lead) {
        tc5::fence_after_sync();
        // Y2 = M X (with the block's biases: M in an fp16 high part and residual),
        // K = 64 source rows
#pragma unroll
        for (int j = 0; j < (BIAS ? 8 : 4); ++j)
          tc5::mma_bf16(tmem + kColY2, (j < 4 ? dM : dMl) + (uint64_t)((j & 3) * (32 >> 4)),
                        dX + (uint64_t)((j & 3) * (2048 >> 4)), kIdescY, j > 0);
        tc5::commit(&sm.mbar[2]);
        // Y1 and S consume Cbar and W_end o X (theta's space): refill them once
        // those products are done, after Y2 is on its way (in the bias instances
        // Y2 reads the mask's residual from theta's space too)
        if (c + 1 < c_hi) {
          if (!tc5::mbar_wait(&sm.mbar[BIAS ? 2 : 1], par, wait_ns)) sm.err = 1;
          tma_bc(c + 1, &tm.C, aC);
          if (ROT && has_theta) tma_theta(c + 1);
        }
      }
      continue;
    }

    // ===================== compute warps (0..7) ===================================
    if (c == 0 && patch_row0) {  // (the first segment's first chunk)
      if (tid < NS) *reinterpret_cast<bf16*>(sm.B + off2(0, tid)) = __float2bfloat16_rn(bp0);
      if (tid < PD) *reinterpret_cast<bf16*>(sm.X[0] + off1(0, tid)) = __float2bfloat16_rn(xp0);
    }

    // -- phase R1: chunk-local angle cumsum ------------------------------------
    // Thread (lane, warp) owns the adjacent pairs 2 lane, 2 lane + 1 (elements
    // 4 lane .. 4 lane + 3) in rows 8 warp .. 8 warp + 7; the two pairs travel
    // together in packed fp32 pairs.
    float2 psi[8];
    if (ROT) {
      float2 run = make_float2(0.f, 0.f);
      if (has_theta) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          if (warp > 0 || k > 0) {  // psi_0 = 0
            float2 th;
            if (TH16) {
              const uint32_t raw = reinterpret_cast<const uint32_t*>(&sm.u.theta[0][0])
                  [(8 * warp + k) * (NH / 2) + lane];
              const float dl = P.dl[8 * warp + k];
              th = __fmul2_rn(unpack_bf16(raw), make_float2(dl, dl));
            } else {
              th = *reinterpret_cast<const float2*>(&sm.u.theta[8 * warp + k][2 * lane]);
            }
            run = __fadd2_rn(run, th);
          }
          psi[k] = run;
        }
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) psi[k] = run;
      }
      *reinterpret_cast<float2*>(&sm.segtot[warp][2 * lane]) = run;
    }
    // S2 (compute warps only, so that the control warp's scalars for the next chunk
    // overlap phases R1 and R2): segment totals ready; theta no longer read
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kCtrlWarp) : "memory");

    // -- phase R2: rotation into the absolute frame; X and W_end o X in fp16 ------
    // The absolute angle of row r is Phi_c + psi_r with Phi_c kept in [-pi, pi];
    // its magnitude is bounded by pi plus one chunk's sum of theta, where the
    // hardware sincos keeps an absolute error of about 2^-21 + |angle| 2^-24.
    {
      float2 base = make_float2(0.f, 0.f);
      if (ROT) {
        base = *reinterpret_cast<const float2*>(&sm.Phi[2 * lane]);
#pragma unroll
        for (int s2 = 0; s2 < 7; ++s2)
          if (s2 < warp)
            base = __fadd2_rn(base, *reinterpret_cast<const float2*>(&sm.segtot[s2][2 * lane]));
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int r = 8 * warp + k;
        const uint32_t o = off2(r, 4 * lane);
        uint2* pb = reinterpret_cast<uint2*>(sm.B + o);
        uint2* pc = reinterpret_cast<uint2*>(sm.C + o);
        const uint2 bw2 = *pb, cw2 = *pc;
        float2 bre = make_float2(__uint_as_float(bw2.x << 16), __uint_as_float(bw2.y << 16));
        float2 bim = make_float2(__uint_as_float(bw2.x & 0xffff0000u),
                                 __uint_as_float(bw2.y & 0xffff0000u));
        float2 cre = make_float2(__uint_as_float(cw2.x << 16), __uint_as_float(cw2.y << 16));
        float2 cim = make_float2(__uint_as_float(cw2.x & 0xffff0000u),
                                 __uint_as_float(cw2.y & 0xffff0000u));
        if (has_bbias) {
          bre = __fadd2_rn(bre, bbr);
          bim = __fadd2_rn(bim, bbi);
        }
        if (has_cbias) {
          cre = __fadd2_rn(cre, cbr);
          cim = __fadd2_rn(cim, cbi);
        }
        if (ROT) {
          const float2 ang = __fadd2_rn(psi[k], base);
          float s0, c0, s1, c1;
          __sincosf(ang.x, &s0, &c0);
          __sincosf(ang.y, &s1, &c1);
          const float2 cr = make_float2(c0, c1), sr = make_float2(s0, s1);
          const float2 nsr = make_float2(-s0, -s1);
          const float2 bre2 = __ffma2_rn(nsr, bim, __fmul2_rn(cr, bre));
          const float2 bim2 = __ffma2_rn(cr, bim, __fmul2_rn(sr, bre));
          const float2 cre2 = __ffma2_rn(nsr, cim, __fmul2_rn(cr, cre));
          const float2 cim2 = __ffma2_rn(cr, cim, __fmul2_rn(sr, cre));
          bre = bre2; bim = bim2; cre = cre2; cim = cim2;
        }
        *pb = make_uint2(pack_h2(bre.x, bim.x), pack_h2(bre.y, bim.y));
        *pc = make_uint2(pack_h2(cre.x, cim.x), pack_h2(cre.y, cim.y));
      }
      {  // X of this chunk in fp16 (in place) and W_end o X: row tid / 4, 16 elements
        const int r = tid >> 2;
        const float we = P.wend[r];
        uint8_t* Xw = sm.X[c & 1];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int ch = 2 * (tid & 3) + q;
          const uint32_t o = (uint32_t)(r * 128 + ((ch ^ (r & 7)) << 4));
          uint4* px = reinterpret_cast<uint4*>(Xw + o);
          const uint4 xw = *px;
          const uint32_t w4[4] = {xw.x, xw.y, xw.z, xw.w};
          float xv[8];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            xv[2 * j] = __uint_as_float(w4[j] << 16);
            xv[2 * j + 1] = __uint_as_float(w4[j] & 0xffff0000u);
          }
          *px = make_uint4(pack_h2(xv[0], xv[1]), pack_h2(xv[2], xv[3]), pack_h2(xv[4], xv[5]),
                           pack_h2(xv[6], xv[7]));
          *reinterpret_cast<uint4*>(sm.u.t.wx + o) =
              make_uint4(pack_h2(we * xv[0], we * xv[1]), pack_h2(we * xv[2], we * xv[3]),
                         pack_h2(we * xv[4], we * xv[5]), pack_h2(we * xv[6], we * xv[7]));
        }
      }
      if (ROT && warp == 7) {
        const float2 pend = __fadd2_rn(psi[7], base);  // Phi_c + psi_63
        sm.nPhi[2 * lane] = wrap_angle(pend.x);
        sm.nPhi[2 * lane + 1] = wrap_angle(pend.y);
      }
    }
    tc5::fence_proxy_async();
    __syncthreads();  // S3: Cbar, Bbar, X, W_end o X ready
    if (ROT && tid >= 2 * NH && tid < 3 * NH) sm.Phi[tid - 2 * NH] = sm.nPhi[tid - 2 * NH];

    // -- phase G: masked Gram -> M (rows 16 (warp % 4) + .., columns cb + ..) -------
    {
      // the mask depends only on the chunk scalars: compute it while the Gram runs.
      // Row t = 16 (warp % 4) + lane/4 + 8 hf lies in 8-row block kr = t / 8; column
      // block kc = 2 q + warp / 4, so that every warp holds one of the two diagonal
      // blocks of its rows.  Below the diagonal blocks the weight factorises through
      // the decay at the block's first row (both factors at most 1); the diagonal
      // block takes the direct exponential; blocks with kc > kr are zero.
      const int cpar = warp >> 2;
      float wv[2][4][2];
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int t = 16 * (warp & 3) + (lane >> 2) + 8 * hf;
        const int kr = 2 * (warp & 3) + hf;
        const float et = P.et[t];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int kc = 2 * q + cpar;
          const int s0 = 8 * kc + 2 * (lane & 3);
          float w0 = 0.f, w1 = 0.f;
          if (kc < kr) {
            const float2 f = *reinterpret_cast<const float2*>(&P.fs[fs_index(kr, s0)]);
            w0 = et * f.x;
            w1 = et * f.y;
          } else if (kc == kr) {
            const float cst = P.cs2[t];
            if (s0 < t) w0 = ex2(cst - P.cs2[s0 + 1]) * P.cvec[s0];
            else if (s0 == t) w0 = P.gam[t];
            if (s0 + 1 < t) w1 = ex2(cst - P.cs2[s0 + 2]) * P.cvec[s0 + 1];
            else if (s0 + 1 == t) w1 = P.gam[t];
          }
          wv[hf][q][0] = w0;
          wv[hf][q][1] = w1;
        }
      }
      if (!tc5::mbar_wait(&sm.mbar[0], par, wait_ns)) sm.err = 1;
      tc5::fence_after_sync();
      uint32_t gr[4][4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        tc5::ld_16x256b_x1(tmem + tlane + kColG + (uint32_t)(8 * (2 * q + cpar)), gr[q]);
      tc5::wait_ld();
      // M = W o G in fp16 (with the block's biases: a high part and residual)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int t = 16 * (warp & 3) + (lane >> 2) + 8 * hf;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int s0 = 8 * (2 * q + cpar) + 2 * (lane & 3);
          const float m0 = __uint_as_float(gr[q][2 * hf]) * wv[hf][q][0];
          const float m1 = __uint_as_float(gr[q][2 * hf + 1]) * wv[hf][q][1];
          const uint32_t hi = pack_h2(m0, m1);
          const float2 hv = unpack_h2(hi);
          *reinterpret_cast<uint32_t*>(sm.M + off1(t, s0)) = hi;
          if (BIAS) *reinterpret_cast<uint32_t*>(sm.u.t.ml + off1(t, s0)) = pack_h2(m0 - hv.x, m1 - hv.y);
        }
      }
    }
    tc5::fence_proxy_async();
    tc5::fence_before_sync();
    __syncthreads();  // S4: M ready

    // -- phase S + Y: the state update, then the outputs ----------------------------
    // The state product and Y1 (which reads the fp16 state copy) were committed
    // before M X, so the state phase runs while M X is still in flight; the outputs
    // follow once it lands.
    {
      if (!tc5::mbar_wait(&sm.mbar[1], par, wait_ns)) sm.err = 1;  // G, S and Y1 done
      tc5::fence_after_sync();
      const float isc = __uint_as_float((uint32_t)(127 - kexp) << 23);  // Y1 used h 2^kexp
      // h after this chunk (the state product added S onto exp(cs_63) h)
      {
        uint32_t sv[32];
        tc5::ld_32x32b_x32(tmem + tlane + kColS + (uint32_t)cb, sv);
        tc5::wait_ld();
        tc5::reg_after_ld(sv);
        float hv[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) hv[j] = __uint_as_float(sv[j]);
        // every warp has read the previous maxima (the bar.sync of the last store
        // and this chunk's barriers lie between) before they are overwritten
        store_state_f16(hv);
        // the next chunk's product accumulates onto exp(cs_63 of that chunk) h; after
        // the last chunk TMEM keeps h itself for hT
        if (c + 1 < c_hi) store_state_tmem(hv, sm.prm[(c + 1) & 1].eE);
      }
      if (!tc5::mbar_wait(&sm.mbar[2], par, wait_ns)) sm.err = 1;  // M X done
      tc5::fence_after_sync();
      uint32_t y1[16], y2[16];
      tc5::ld_16x256b_x4(tmem + tlane + kColY1 + (uint32_t)cb, y1);
      tc5::ld_16x256b_x4(tmem + tlane + kColY2 + (uint32_t)cb, y2);
      tc5::wait_ld();
      tc5::reg_after_ld(y1);
      tc5::reg_after_ld(y2);
      const float2 D2 = make_float2(Dh, Dh);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int r = 16 * (warp & 3) + (lane >> 2) + 8 * hf;
        const int64_t t = tbase + r;
        if (r > 0 && t < L) {
          const float2 er2 = make_float2(P.ecs[r] * isc, P.ecs[r] * isc);
          bf16* yrow = Y_seq + t * xstride_t;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int p = cb + 8 * q + 2 * (lane & 3);
            const float2 xv = unpack_h2(*reinterpret_cast<const uint32_t*>(Xs + off1(r, p)));
            const float2 a1 = make_float2(__uint_as_float(y1[4 * q + 2 * hf]),
                                          __uint_as_float(y1[4 * q + 2 * hf + 1]));
            const float2 a2 = make_float2(__uint_as_float(y2[4 * q + 2 * hf]),
                                          __uint_as_float(y2[4 * q + 2 * hf + 1]));
            const float2 v = __ffma2_rn(D2, xv, __ffma2_rn(er2, a1, a2));
            *reinterpret_cast<uint32_t*>(yrow + p) = pack_bf16(v.x, v.y);
          }
        }
      }
    }
    tc5::fence_proxy_async();
  }

  // ---- outputs of the last token, TMEM release ---------------------------------
  if (sm.err) {
    if (tid == 0) atomicAdd(&g_chunk_wait_timeouts, 1u);
  } else if (!ctrl && seg_last) {
    if (a.hT) {
      uint32_t sv[32];
      tc5::ld_32x32b_x32(tmem + tlane + kColS + (uint32_t)cb, sv);
      tc5::wait_ld();
      tc5::reg_after_ld(sv);
      float4* dst = reinterpret_cast<float4*>(a.hT + (bh * NS + n_row) * PD + cb);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        dst[j] = make_float4(__uint_as_float(sv[4 * j]), __uint_as_float(sv[4 * j + 1]),
                             __uint_as_float(sv[4 * j + 2]), __uint_as_float(sv[4 * j + 3]));
    }
    if (a.angleT && tid < NH)
      a.angleT[bh * NH + tid] = ROT ? sm.Phi[tid] : (a.angle0 ? a.angle0[bh * NH + tid] : 0.f);
    if (a.xprevT && tid < PD)
      a.xprevT[bh * PD + tid] = __bfloat162float(Xg[(b * L + L - 1) * xtok + h * PD + tid]);
    if (a.bprevT && h % (H / G) == 0 && tid < NS)
      a.bprevT[(b * G + g) * NS + tid] =
          __bfloat162float(Bg[((b * L + L - 1) * G + g) * NS + tid]);
  }
  tc5::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc5::tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool encode_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1,
                uint64_t d2, uint64_t d3, uint64_t esz, uint32_t box0, CUtensorMapSwizzle sw,
                uint64_t tok) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
  if (!fn) return false;
  const cuuint64_t dims[4] = {d0, d1, d2, d3};
  const uint64_t ts = tok ? tok : d0 * d1;
  const cuuint64_t strides[3] = {d0 * esz, ts * esz, ts * d2 * esz};
  const cuuint32_t box[4] = {box0, 1, (cuuint32_t)Q, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, dt, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

template <bool ROT, bool BIAS, bool TH16, bool TEST = false, bool SEG = false>
cudaError_t launch_variant(const FwdArgs& a, cudaStream_t s) {
  TmaMaps tm;
  memset(&tm, 0, sizeof(tm));
  const uint64_t L = (uint64_t)a.L, b = (uint64_t)a.b, H = (uint64_t)a.H, G = (uint64_t)a.G;
  bool ok = encode_map(&tm.B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.B, NS, G, L, b, 2, 64,
                       CU_TENSOR_MAP_SWIZZLE_128B) &&
            encode_map(&tm.C, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.C, NS, G, L, b, 2, 64,
                       CU_TENSOR_MAP_SWIZZLE_128B) &&
            encode_map(&tm.X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.X, PD, H, L, b, 2, 64,
                       CU_TENSOR_MAP_SWIZZLE_128B, (uint64_t)a.x_tok_stride);
  if (ok && TH16 && a.theta16)
    ok = encode_map(&tm.theta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.theta16, NH, H, L, b, 2, NH,
                    CU_TENSOR_MAP_SWIZZLE_NONE, (uint64_t)a.theta16_tok_stride);
  else if (ok && a.theta)
    ok = encode_map(&tm.theta, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.theta, NH, H, L, b, 4, NH,
                    CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!ok) return cudaErrorInvalidValue;
  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(fwd_chunk_kernel<ROT, BIAS, TH16, TEST, SEG>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t nseg = SEG ? a.nseg : 1;
  fwd_chunk_kernel<ROT, BIAS, TH16, TEST, SEG><<<(unsigned)(a.b * a.H * nseg), kThreads, smem, s>>>(a, tm);
  return cudaGetLastError();
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

bool fwd_chunk_supported(const FwdArgs& a) {
  return a.bf16 && a.N == NS && a.P == PD && a.L > 0 && (a.chunk == 0 || a.chunk == Q) &&
         a.x_tok_stride % 8 == 0 && (a.x_tok_stride == 0 || a.x_tok_stride >= a.H * PD) &&
         (a.theta16 == nullptr ||
          (al16(a.theta16) && a.theta16_tok_stride % 8 == 0 && a.theta16_tok_stride >= a.H * NH)) &&
         al16(a.X) && al16(a.B) && al16(a.C) && al16(a.Y) && al16(a.theta) && al16(a.h0) &&
         al16(a.hT) && al16(a.logdecay) && al16(a.Bbias) && al16(a.Cbias);
}

cudaError_t launch_fwd_chunk(const FwdArgs& a, cudaStream_t s) {
  if (a.b * a.H == 0) return cudaSuccess;
  // the rotation phase also applies the head biases of B and C (its own variant,
  // so that the plain scan's kernel carries none of it)
  if (a.theta16 != nullptr) {  // the block's raw angle projection (biases alongside)
    if (a.theta != nullptr || a.A_log == nullptr) return cudaErrorInvalidValue;
    return launch_variant<true, true, true>(a, s);
  }
  if (a.Bbias != nullptr || a.Cbias != nullptr) return launch_variant<true, true, false>(a, s);
  if (a.nseg > 1) {  // the segments of a split sequence (the public scan only)
    if (a.hseg == nullptr || a.aseg == nullptr || a.segc < 1) return cudaErrorInvalidValue;
    if (a.theta != nullptr || a.angle0 != nullptr) return launch_variant<true, false, false, false, true>(a, s);
    return launch_variant<false, false, false, false, true>(a, s);
  }
  if (a.theta != nullptr || a.angle0 != nullptr) {
    if (g_test_launch_requested.exchange(false)) return launch_variant<true, false, false, true>(a, s);
    return launch_variant<true, false, false>(a, s);
  }
  return launch_variant<false, false, false>(a, s);
}

cudaError_t set_wait_limit_ns(unsigned long long ns) {
  return cudaMemcpyToSymbol(g_wait_limit_ns, &ns, sizeof(ns));
}

cudaError_t request_dropped_gram_signal() {
  g_test_launch_requested.store(true);
  return cudaSuccess;
}

cudaError_t read_and_clear_wait_timeouts(unsigned int* count) {
  const unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(count, g_chunk_wait_timeouts, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_chunk_wait_timeouts, &zero, sizeof(unsigned int));
}

}  // namespace m3ssd
