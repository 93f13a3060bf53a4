// Chunk-parallel bf16 forward of the Mamba-3 SISO scan on the sm_100a tensor
// cores (tcgen05 MMA, TMEM accumulators), for N = 128, P = 64.
//
// The recurrence ("TorchMamba" README, "Math notes", M3 SISO)
//     h_t = alpha_t h_{t-1} + beta_t Bbar_{t-1} x_{t-1}^T + gamma_t Bbar_t x_t^T,
//     y_t = Cbar_t^T h_t + D x_t,   Bbar_t = R(phi_t) B_t,  Cbar_t = R(phi_t) C_t,
// is cut into chunks of Q = 64 source rows: row 0 is the token just before the
// chunk (t0 - 1, the carry-in of the beta term) and rows 1..63 are the chunk's
// own tokens t0 .. t0 + 62 (t0 = 63 c).  Everything of a chunk is computed in
// the chunk's own rotation frame, whose origin is the absolute angle
// Phi_c = phi_{t0-1}: with the chunk-local sums (row 0 has cs_0 = psi_0 = 0)
//     cs_r = sum_{k=1..r} logdecay_k,   psi_r = sum_{k=1..r} theta_k,
// the local rotated vectors are Bt_r = R(psi_r) B_r, Ct_r = R(psi_r) C_r (so
// Bbar_r = R(Phi_c) Bt_r), and the state entering the chunk in that frame is
// ht_c = R(-Phi_c) h_{t0-1}.  Then, for the output rows r = 1..63,
//     y_r   = exp(cs_r) Ct_r^T ht_c + sum_{u<=r} W(r,u) (Ct_r . Bt_u) x_u + D x_r,
//     W(r,r) = gamma_r,  W(r,u<r) = exp(cs_r - cs_{u+1}) (gamma_u alpha_{u+1} + beta_{u+1})
// with gamma_0 := 0 (column u = 0 carries exactly the beta boundary term: the
// gamma and beta terms form one mask, "the parallel mask is L = 1SS @ band"),
// and the state carried to the next chunk, in its frame, is
//     ht_{c+1} = R(-Psi_c) (exp(cs_63) ht_c + S_c),   S_c = sum_u W(63,u) Bt_u x_u^T,
// Psi_c = psi_63 ("TorchMamba" README, "Math notes", M2: chunkwise
// intra-quadratic part plus a factored inter-chunk carry).  Only the carry
// (ht, and the absolute angle Phi for the final outputs) passes between
// chunks; the Gram, the mask, the intra-chunk outputs and S_c of every chunk
// are independent of all other chunks.
//
// Scheduling.  A work unit is one chunk of one (b, h) sequence.  Persistent
// CTAs take units from an atomic ticket in chunk-major order (all sequences'
// chunk 0, then chunk 1, ...), so a unit only ever waits for the carry of a
// unit with a smaller ticket, which is running or done: no unit waits on one
// that is not resident.  The carry ht_{c+1} (fp32, N x P) and Phi_{c+1} go to
// one of two ring slots per sequence in the workspace (they stay in L2); the
// producing CTA publishes it with a release store of the sequence's flag and
// the consuming CTA acquires the flag before reading it.  Several CTAs share
// an SM, so one unit's waits overlap the others' work.
//
// Tensor-core work per unit (kind::f16 with fp16 operands, fp32 in TMEM):
//   G  = Ct Bt^T          M=64  N=64 K=128   TMEM cols  0..63
//   S  = Bt^T (W_end o X) M=128 N=64 K=64    TMEM cols 64..127
//   Y2 = (W o G) X        M=64  N=64 K=64    TMEM cols  0..63 (after G is read)
//   Y1 = Ct ht 2^k        M=64  N=64 K=128   TMEM cols 64..127 (after S is read)
// fp16 operands (11 significant bits) keep the scan's own error near 2^-12 of
// the large diagonal terms, where bf16 operands gave 2^-9; ht is scaled by a
// power of two 2^k chosen from its largest element, so its fp16 copy neither
// overflows nor loses precision to subnormals.  The bf16 inputs X, B, C are
// converted exactly when their magnitudes lie in fp16's normal range
// [2^-14, 65504]; larger magnitudes overflow to infinity.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc5.cuh"

namespace m3ssd {

// Bounded device-side waits of the chunk-parallel forward that ran out.
__device__ unsigned int g_cp_wait_timeouts;

namespace {

constexpr int Q = 64;       // source rows per chunk (1 carry-in + 63 tokens)
constexpr int QT = Q - 1;   // tokens per chunk
constexpr int NS = 128;     // state size N
constexpr int PD = 64;      // head dim P
constexpr int NH = NS / 2;  // rotation pairs
constexpr uint32_t kTmemCols = 128;
constexpr uint32_t kColA = 0, kColB = 64;
constexpr uint32_t kAtom = Q * 128;               // one 64-element atom of a Q-row tile
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // a device-side wait gives up after 2 s
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kIdG = tc5::idesc_f16(64, 64, false, false);
constexpr uint32_t kIdY = tc5::idesc_f16(64, 64, false, true);
constexpr uint32_t kIdS = tc5::idesc_f16(128, 64, true, true);
// one ring slot: ht (N x P) and Phi (N/2)
constexpr int kSlotFloats = NS * PD + NH;
constexpr int kCompute = 256;               // 8 compute warps
constexpr int kCtaThreads = kCompute + 32;  // + the control warp

typedef __nv_bfloat16 bf16;

// Byte offset of element (r, n) in a Q-row tile of 128 elements a row, stored
// as two 64-element atoms of 128-byte rows with the 16-byte XOR swizzle.
__device__ __forceinline__ uint32_t off2(int r, int n) {
  return (uint32_t)((n >> 6) * kAtom + r * 128 + ((((n & 63) >> 3) ^ (r & 7)) << 4) +
                    ((n & 7) << 1));
}
// Byte offset of element (r, c) in a tile of 64 elements (128 B) a row.
__device__ __forceinline__ uint32_t off1(int r, int c) {
  return (uint32_t)(r * 128 + ((((c >> 3) ^ (r & 7))) << 4) + ((c & 7) << 1));
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// 2^x by the hardware approximation (relative error about 2^-22; flushes
// results below 2^-126 to zero).  The arguments are differences of fp32 decay
// sums, whose own rounding (about |cs| 2^-24) dominates that error.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned ld_volatile(const unsigned* p) {
  unsigned v;
  asm volatile("ld.volatile.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// 4-byte asynchronous global -> shared copy (completion: cp.async.wait_group).
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(tc5::saddr(dst)), "l"(src)
               : "memory");
}

// Per-chunk scalars: decay cumsum (log2 units), exp(cs), the mask coefficients
// gamma_u alpha_{u+1} + beta_{u+1}, the state weights W(63, u), gamma,
// exp(cs_t - cs_{8 floor(t/8)}), the below-diagonal factor table and exp(cs_63).
struct UnitParams {
  float cs2[Q];
  float ecs[Q];
  float cvec[Q];
  float wend[Q];
  float gam[Q];
  float et[Q];
  float fs[224];  // exp(cs_{8k} - cs_{s+1}) cvec_s for s < 8k, at fs_index(k, s)
  float csl[Q];   // decay sums within each 32-row half (log2 units)
  float half0;    // the first half's total
  float eE;
  float pad[2];
};

// Block row k = 1..7 of the factor table holds the 8k columns s < 8k, from 4k(k-1).
__host__ __device__ constexpr int fs_index(int k, int s) { return 4 * k * (k - 1) + s; }

struct CpMaps {
  CUtensorMap B;      // bf16 (n, group, token, batch), box 64 x 1 x 64 x 1, 128-byte swizzle
  CUtensorMap C;      // same as B
  CUtensorMap X;      // bf16 (p, head, token, batch), box 64 x 1 x 64 x 1, 128-byte swizzle
  CUtensorMap theta;  // fp32 (pair, head, token, batch), box 64 x 1 x 64 x 1, no swizzle
};

// The workspace: the ticket counter and the abort flag, one flag per sequence
// (the number of chunks whose carry has been published) and two ring slots of
// kSlotFloats per sequence.  The ticket, abort flag and sequence flags are
// cleared before every launch.
struct CpWs {
  unsigned long long* ticket;
  unsigned int* abort;
  unsigned int* flags;
  float* ring;
};

size_t header_bytes(int64_t S) { return (size_t)((64 + 4 * S + 255) / 256) * 256; }

// Shared memory of a CTA.  theta, B and phi are adjacent: once the angle sums
// and the products that read Bt are done, the three take the incoming carry
// (one ring slot, copied in one bulk copy).  WX takes the mask M once S is
// done, and X and WX take the fp16 copy of ht for Y1 once Y2 is done.
struct Smem {
  uint8_t TH[Q * NH * 4];  // raw theta of the unit (fp32); then carry in
  uint8_t B[2 * kAtom];    // raw B, then Bt (fp16); then carry in
  float phibuf[256];       // Phi of the carry in (padded to keep the tiles aligned)
  uint8_t C[2 * kAtom];    // raw C, then Ct (fp16)
  uint8_t X[Q * 128];      // raw X, then fp16; then ht (first half)
  uint8_t WX[Q * 128];     // W_end o X (fp16); then the mask M; then ht (second half)
  UnitParams prm;
  float raw[2][3][Q];      // logdecay, gamma, beta of a unit's rows, by unit parity
  float segtot[8][NH];
  float Psi[NH];
  float hmax[8];
  long long unit[2];       // the unit of each parity (total: no more units)
  // mbarriers: TMA inputs; the next unit's index (control -> compute warps 0,
  // 1); carry in; tensor-core products; compute warps -> control warp:
  // operands ready (2), mask ready (3), carry out stored (5), ht tile ready (6)
  uint64_t mbL, mbT, mbR, mbG, mbS, mbY2, mbY1, mb2, mb3, mb5, mb6;
  uint32_t tmem;
  uint32_t err;  // 1: a wait of this CTA timed out; 2: another CTA aborted the launch
};
static_assert(offsetof(Smem, B) == offsetof(Smem, TH) + Q * NH * 4, "carry in spans TH, B, phibuf");
static_assert(offsetof(Smem, phibuf) == offsetof(Smem, B) + 2 * kAtom, "carry in spans TH, B, phibuf");
static_assert(offsetof(Smem, WX) == offsetof(Smem, X) + Q * 128, "ht for Y1 spans X and WX");
static_assert(kSlotFloats * 4 <= Q * NH * 4 + 2 * kAtom + 256 * 4, "a ring slot fits the carry-in space");
static_assert(offsetof(Smem, C) % 1024 == 0 && offsetof(Smem, X) % 1024 == 0 &&
                  offsetof(Smem, WX) % 1024 == 0 && offsetof(Smem, B) % 1024 == 0,
              "operand tiles are 1024-byte aligned");

// Arrival of one compute warp on a compute -> control mbarrier (count 8).
__device__ __forceinline__ void warp_arrive(uint64_t* mb, int lane) {
  __syncwarp();
  if (lane == 0) tc5::mbar_arrive(mb);
}

template <bool ROT>
__global__ void __launch_bounds__(kCtaThreads, 3)
    fwd_cp_kernel(FwdArgs a, const __grid_constant__ CpMaps tm, CpWs ws, long long total,
                  int nC) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw_addr = tc5::saddr(smem_raw);
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t H = a.H, L = a.L, G = a.G, S = a.b * a.H;
  const uint32_t aTH = tc5::saddr(sm.TH), aB = tc5::saddr(sm.B), aC = tc5::saddr(sm.C);
  const uint32_t aX = tc5::saddr(sm.X), aWX = tc5::saddr(sm.WX);
  const uint32_t aM = aWX, aH = aX;  // ht for Y1 spans X and WX once Y2 is done
  constexpr uint32_t kUnitBytes = (uint32_t)(Q * NH * 4) + 2u * 16384u + 8192u;
  constexpr uint32_t kSlotBytes = (uint32_t)kSlotFloats * 4u;

  // decodes a unit: sequence s = b H + h, chunk c
  auto unit_of = [&](long long u, int64_t& s, int& c, int64_t& b, int64_t& h, int64_t& g) {
    s = u % S;
    c = (int)(u / S);
    b = s / H;
    h = s % H;
    g = h / (H / G);
  };
  // compute warps 0, 1: the raw chunk scalars of unit u (one row a thread) into
  // raw[p] by asynchronous copies; row 0 and rows past the end read as zeros
  auto stage_params = [&](long long u, uint32_t p) {
    int64_t s, b, h, g;
    int c;
    unit_of(u, s, c, b, h, g);
    const int r = tid;  // 0 .. 63
    const int64_t t = (int64_t)c * QT - 1 + r;
    if (r > 0 && t < L) {
      const int64_t idx = (b * L + t) * H + h;
      cp_async4(&sm.raw[p][0][r], a.logdecay + idx);
      cp_async4(&sm.raw[p][1][r], a.gamma + idx);
      if (a.beta) cp_async4(&sm.raw[p][2][r], a.beta + idx);
      else sm.raw[p][2][r] = 0.f;
    } else {
      sm.raw[p][0][r] = 0.f;
      sm.raw[p][1][r] = 0.f;
      sm.raw[p][2][r] = 0.f;
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  if (warp == 0) tc5::tmem_alloc(&sm.tmem, kTmemCols);
  if (tid == kCompute) {
    uint64_t* one[] = {&sm.mbL, &sm.mbT, &sm.mbR, &sm.mbG, &sm.mbS, &sm.mbY2, &sm.mbY1};
    for (uint64_t* m : one) tc5::mbar_init(m, 1);
    uint64_t* eight[] = {&sm.mb2, &sm.mb3, &sm.mb5, &sm.mb6};
    for (uint64_t* m : eight) tc5::mbar_init(m, 8);
    tc5::fence_mbar_init();
    sm.err = 0;
    sm.unit[0] = (long long)atomicAdd(ws.ticket, 1ull);
  }
  tc5::fence_before_sync();
  __syncthreads();
  tc5::fence_after_sync();
  const uint32_t tmem = sm.tmem;

  if (warp == 8) {
    // ===================== control warp ==========================================
    const bool lead = lane == 0;
    bool pendL = false, pendR = false;
    uint32_t rpar = 0;  // phase of mbR (completes only for units with c > 0)
    uint64_t* last_commit = nullptr;
    auto issue_loads = [&](long long u) {  // leader only
      if (u >= total) {
        tc5::mbar_arrive(&sm.mbL);  // no more units: wakes the compute warps
        return;
      }
      int64_t s, b, h, g;
      int c;
      unit_of(u, s, c, b, h, g);
      const int t0 = c * QT - 1;
      tc5::mbar_arrive_expect_tx(&sm.mbL, ROT ? kUnitBytes : kUnitBytes - (uint32_t)(Q * NH * 4));
      if (ROT) tc5::tma_load_4d(aTH, &tm.theta, &sm.mbL, 0, (int)h, t0, (int)b);
      tc5::tma_load_4d(aB, &tm.B, &sm.mbL, 0, (int)g, t0, (int)b);
      tc5::tma_load_4d(aB + kAtom, &tm.B, &sm.mbL, 64, (int)g, t0, (int)b);
      tc5::tma_load_4d(aC, &tm.C, &sm.mbL, 0, (int)g, t0, (int)b);
      tc5::tma_load_4d(aC + kAtom, &tm.C, &sm.mbL, 64, (int)g, t0, (int)b);
      tc5::tma_load_4d(aX, &tm.X, &sm.mbL, 0, (int)h, t0, (int)b);
      pendL = true;
    };
    long long u = sm.unit[0];
    if (lead) issue_loads(u);
    for (uint32_t i = 0; u < total; ++i) {
      const uint32_t par = i & 1u;
      int64_t s, b, h, g;
      int c;
      unit_of(u, s, c, b, h, g);
      const bool last = c + 1 == nC;
      bool fail = false;
      long long nx = total;
      if (lead) {
        // (A) operands ready: G = Ct Bt^T and S = Bt^T (W_end o X)
        if (!tc5::mbar_wait(&sm.mb2, par, kWaitLimitNs, &sm.err)) fail = true;
        else pendL = false;  // the compute warps waited for the loads before arriving
        if (!fail) {
          tc5::fence_after_sync();
          const uint64_t dC = tc5::desc_sw128(aC, 16, 1024), dB = tc5::desc_sw128(aB, 16, 1024);
          const uint64_t dBm = tc5::desc_sw128(aB, kAtom, 1024);
          const uint64_t dWX = tc5::desc_sw128(aWX, kAtom, 1024);
#pragma unroll
          for (int j = 0; j < 8; ++j) {  // K = n in 8 steps of 16
            const uint64_t ko = (uint64_t)(((j >> 2) * kAtom + (j & 3) * 32) >> 4);
            tc5::mma_bf16(tmem + kColA, dC + ko, dB + ko, kIdG, j > 0);
          }
          tc5::commit(&sm.mbG);
#pragma unroll
          for (int j = 0; j < 4; ++j) {  // K = rows in 4 steps of 16
            const uint64_t ko = (uint64_t)((j * 2048) >> 4);
            tc5::mma_bf16(tmem + kColB, dBm + ko, dWX + ko, kIdS, j > 0);
          }
          tc5::commit(&sm.mbS);
          last_commit = &sm.mbS;
        }
        // (B) mask ready -> Y2 = M X; carry published and Bt free -> carry copied in
        bool y2 = false, ring = c == 0 || fail, seen = c == 0;
        const uint64_t t0 = tc5::globaltimer_ns();
        uint32_t polls = 0;
        while (!fail && !(y2 && ring)) {
          if (!y2 && tc5::mbar_test(&sm.mb3, par)) {
            tc5::fence_after_sync();
            const uint64_t dM = tc5::desc_sw128(aM, 16, 1024), dX = tc5::desc_sw128(aX, kAtom, 1024);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tc5::mma_bf16(tmem + kColA, dM + (uint64_t)((j * 32) >> 4),
                            dX + (uint64_t)((j * 2048) >> 4), kIdY, j > 0);
            tc5::commit(&sm.mbY2);
            last_commit = &sm.mbY2;
            y2 = true;
          }
          if (!ring) {
            if (!seen) seen = ld_acquire(ws.flags + s) >= (unsigned)c;
            if (seen && tc5::mbar_test(&sm.mbS, par)) {
              tc5::fence_proxy_async_global();
              tc5::mbar_arrive_expect_tx(&sm.mbR, kSlotBytes);
              tc5::bulk_load(aTH, ws.ring + (s * 2 + (c & 1)) * (int64_t)kSlotFloats, kSlotBytes,
                             &sm.mbR);
              pendR = true;
              ring = true;
            }
          }
          if ((++polls & 31u) == 0) {
            if (tc5::globaltimer_ns() - t0 > kWaitLimitNs || sm.err) fail = true;
            else if (!seen && ld_volatile(ws.abort)) { fail = true; sm.err = 2; }
          }
        }
        // (C) this unit waits for nobody any more: take the next unit now (a unit
        // taken earlier would be held up by this unit's wait), prefetch its inputs
        // to L2 and hand it to compute warps 0, 1 for its chunk scalars
        if (!fail) {
          nx = (long long)atomicAdd(ws.ticket, 1ull);
          if (ld_volatile(ws.abort)) nx = total;
          if (nx < total) {
            int64_t s2, b2, h2, g2;
            int c2;
            unit_of(nx, s2, c2, b2, h2, g2);
            const int t2 = c2 > 0 ? c2 * QT - 1 : 0;  // a hint: kept in bounds
            if (ROT) tc5::tma_prefetch_4d(&tm.theta, 0, (int)h2, t2, (int)b2);
            tc5::tma_prefetch_4d(&tm.B, 0, (int)g2, t2, (int)b2);
            tc5::tma_prefetch_4d(&tm.B, 64, (int)g2, t2, (int)b2);
            tc5::tma_prefetch_4d(&tm.C, 0, (int)g2, t2, (int)b2);
            tc5::tma_prefetch_4d(&tm.C, 64, (int)g2, t2, (int)b2);
            tc5::tma_prefetch_4d(&tm.X, 0, (int)h2, t2, (int)b2);
          }
          sm.unit[par ^ 1u] = nx;
          tc5::mbar_arrive(&sm.mbT);
        }
        // (D) carry out stored: publish it (the chain's critical path), then
        // ht's fp16 tile ready: Y1 = Ct ht
        if (!fail && !tc5::mbar_wait(&sm.mb5, par, kWaitLimitNs, &sm.err)) fail = true;
        if (!fail && !last) st_release(ws.flags + s, (unsigned)(c + 1));
        if (!fail && !tc5::mbar_wait(&sm.mb6, par, kWaitLimitNs, &sm.err)) fail = true;
        if (!fail) {
          tc5::fence_after_sync();
          const uint64_t dC = tc5::desc_sw128(aC, 16, 1024), dH = tc5::desc_sw128(aH, kAtom, 1024);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint64_t ko = (uint64_t)(((j >> 2) * kAtom + (j & 3) * 32) >> 4);
            tc5::mma_bf16(tmem + kColB, dC + ko, dH + (uint64_t)((j * 2048) >> 4), kIdY, j > 0);
          }
          tc5::commit(&sm.mbY1);
          last_commit = &sm.mbY1;
        }
        // (E) every product of the unit done: the tiles take the next unit's inputs
        if (!fail) {
          if (!tc5::mbar_wait(&sm.mbY1, par, kWaitLimitNs, &sm.err)) fail = true;
          else last_commit = nullptr;
          if (c > 0) {  // the compute warps waited for the carry before arriving on mb5
            pendR = false;
            rpar ^= 1u;
          }
          if (!fail) issue_loads(nx);
        }
      }
      fail = __shfl_sync(0xffffffffu, fail ? 1 : 0, 0) != 0;
      if (fail) {
        if (lead && sm.err == 0) sm.err = 1;
        break;
      }
      u = __shfl_sync(0xffffffffu, nx, 0);
    }
    if (lead && sm.err) {
      if (sm.err == 1) {
        atomicAdd(&g_cp_wait_timeouts, 1u);
        atomicExch(ws.abort, 1u);
      }
      // let this CTA's copies and products in flight land before TMEM is freed:
      // waiting for both parities waits for whichever phase is still pending
      auto drain = [&](uint64_t* mb) {
        (void)tc5::mbar_wait(mb, 0, kWaitLimitNs);
        (void)tc5::mbar_wait(mb, 1, kWaitLimitNs);
      };
      if (pendL) drain(&sm.mbL);
      if (pendR) drain(&sm.mbR);
      if (last_commit) drain(last_commit);
    }
  } else {
    // ===================== compute warps ==========================================
    const uint32_t tq = (uint32_t)(32 * (warp & 3)) << 16;  // this warp's TMEM lane quarter
    const int nrow = 32 * (warp & 3) + lane, ccol = 32 * (warp >> 2);
    const int pair = nrow >> 1;
    uint32_t rpar = 0;
    // a wait that times out also stops the control warp (it waits on this CTA's flag)
    // Waiting threads sleep between probes, so that they leave the issue slots to
    // the other CTAs on the SM (eight warps spinning on a wait of a few
    // microseconds otherwise issue more instructions than the unit's work).
    auto cwait = [&](uint64_t* mb, uint32_t parity, uint32_t backoff_ns = 32) {
      const bool r = tc5::mbar_wait(mb, parity, kWaitLimitNs, &sm.err, backoff_ns);
      if (!r && sm.err == 0) sm.err = 1;
      return r;
    };
    if (warp < 2 && sm.unit[0] < total) stage_params(sm.unit[0], 0);
    UnitParams& P = sm.prm;
    for (uint32_t i = 0;; ++i) {
      const uint32_t par = i & 1u;
      bool ok = cwait(&sm.mbL, par, 128);
      if (tc5::bar_or(3, kCompute, !ok)) break;  // S0: every compute warp agrees
      const long long u = sm.unit[par];
      if (u >= total) break;
      int64_t s, b, h, g;
      int c;
      unit_of(u, s, c, b, h, g);
      const int64_t tbase = (int64_t)c * QT - 1;
      const bool last = c + 1 == nC;

      // ---- chunk-local inclusive angle sums (psi_0 = 0) from the theta tile; the
      // decay sums of each 32-row half (warps 0, 1, one row a lane) ---------------
      float2 psi[8];
      if (ROT) {
        float2 run = make_float2(0.f, 0.f);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          if (warp > 0 || k > 0)
            run = __fadd2_rn(run, *reinterpret_cast<const float2*>(sm.TH + (8 * warp + k) * 256 + 8 * lane));
          psi[k] = run;
        }
        *reinterpret_cast<float2*>(&sm.segtot[warp][2 * lane]) = run;
      }
      if (warp < 2) {
        asm volatile("cp.async.wait_group 0;" ::: "memory");  // this thread's raw scalars
        float v = sm.raw[par][0][tid] * kLog2e;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float w2 = __shfl_up_sync(0xffffffffu, v, o);
          if (lane >= o) v += w2;
        }
        P.csl[tid] = v;
        if (tid == 31) P.half0 = v;
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kCompute) : "memory");  // S1: segment totals, half sums
      float2 base = make_float2(0.f, 0.f);
      if (ROT) {
        for (int s2 = 0; s2 < warp; ++s2)
          base = __fadd2_rn(base, *reinterpret_cast<const float2*>(&sm.segtot[s2][2 * lane]));
        if (warp == 7) {
          const float2 tot = __fadd2_rn(base, psi[7]);
          sm.Psi[2 * lane] = tot.x;
          sm.Psi[2 * lane + 1] = tot.y;
        }
      }
      // ---- the chunk scalars: one row (tid < 64) or one factor-table entry a thread --
      {
        const float h0s = P.half0;
        auto csf = [&](int r) { return P.csl[r] + (r >= 32 ? h0s : 0.f); };
        const float(&rw)[3][Q] = sm.raw[par];
        auto cvf = [&](int r) {  // gamma_r alpha_{r+1} + beta_{r+1} (gamma_63 at r = 63)
          return r < Q - 1 ? rw[1][r] * ex2(rw[0][r + 1] * kLog2e) + rw[2][r + 1] : rw[1][r];
        };
        for (int idx = tid; idx < Q + 224; idx += kCompute) {
          if (idx < Q) {
          const int r = idx;
          const float cs = csf(r), cs_end = csf(Q - 1);
          const float cv = cvf(r);
          P.cs2[r] = cs;
          P.ecs[r] = ex2(cs);
          P.gam[r] = rw[1][r];
          P.et[r] = ex2(cs - csf(r & ~7));
          P.cvec[r] = cv;
          P.wend[r] = r < Q - 1 ? ex2(cs_end - csf(r + 1)) * cv : cv;
          if (r == 0) P.eE = ex2(cs_end);
          } else {
          const int j = idx - Q;
          int k = 1;
#pragma unroll
          for (int k2 = 2; k2 < 8; ++k2) k = j >= fs_index(k2, 0) ? k2 : k;
          const int s0 = j - fs_index(k, 0);
          P.fs[j] = ex2(csf(8 * k) - csf(s0 + 1)) * cvf(s0);
          }
        }
      }
      // ---- Bt, Ct in fp16 (chunk-local frame); row 0 of chunk 0 from the cache ---------
      {
        const bool row0_cache = c == 0 && warp == 0 && a.bprev0 != nullptr;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int r = 8 * warp + k;
          const uint32_t o = off2(r, 4 * lane);
          uint2* pb = reinterpret_cast<uint2*>(sm.B + o);
          uint2* pc = reinterpret_cast<uint2*>(sm.C + o);
          const uint2 bw = *pb, cw = *pc;
          float2 bre = make_float2(__uint_as_float(bw.x << 16), __uint_as_float(bw.y << 16));
          float2 bim = make_float2(__uint_as_float(bw.x & 0xffff0000u), __uint_as_float(bw.y & 0xffff0000u));
          float2 cre = make_float2(__uint_as_float(cw.x << 16), __uint_as_float(cw.y << 16));
          float2 cim = make_float2(__uint_as_float(cw.x & 0xffff0000u), __uint_as_float(cw.y & 0xffff0000u));
          if (k == 0 && row0_cache) {
            const float4 v = *reinterpret_cast<const float4*>(a.bprev0 + (b * G + g) * NS + 4 * lane);
            bre = make_float2(v.x, v.z);
            bim = make_float2(v.y, v.w);
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
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kCompute) : "memory");  // S1b: the chunk scalars
      // ---- X in fp16 and W_end o X; row 0 of chunk 0 from the cache --------------------
      {
        const int r = tid >> 2;
        const float we = P.wend[r];
        const bool row0_cache = c == 0 && r == 0 && a.xprev0 != nullptr;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int ch = 2 * (tid & 3) + q;
          const uint32_t o = (uint32_t)(r * 128 + ((ch ^ (r & 7)) << 4));
          uint4* px = reinterpret_cast<uint4*>(sm.X + o);
          const uint4 xw = *px;
          float xv[8];
          if (row0_cache) {
            const float* src = a.xprev0 + s * PD + 8 * ch;
#pragma unroll
            for (int j = 0; j < 8; ++j) xv[j] = src[j];
          } else {
            const uint32_t w4[4] = {xw.x, xw.y, xw.z, xw.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              xv[2 * j] = __uint_as_float(w4[j] << 16);
              xv[2 * j + 1] = __uint_as_float(w4[j] & 0xffff0000u);
            }
          }
          *px = make_uint4(pack_h2(xv[0], xv[1]), pack_h2(xv[2], xv[3]), pack_h2(xv[4], xv[5]),
                           pack_h2(xv[6], xv[7]));
          *reinterpret_cast<uint4*>(sm.WX + o) =
              make_uint4(pack_h2(we * xv[0], we * xv[1]), pack_h2(we * xv[2], we * xv[3]),
                         pack_h2(we * xv[4], we * xv[5]), pack_h2(we * xv[6], we * xv[7]));
        }
      }
      tc5::fence_proxy_async();
      tc5::fence_before_sync();
      warp_arrive(&sm.mb2, lane);  // -> G, S

      // ---- mask: M = W o G in fp16 (rows 16 (warp % 4) + .., column blocks of warp / 4) ---
      {
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
        ok = cwait(&sm.mbG, par) && ok;
        tc5::fence_after_sync();
        uint32_t gr[4][4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          tc5::ld_16x256b_x1(tmem + tq + kColA + (uint32_t)(8 * (2 * q + cpar)), gr[q]);
        tc5::wait_ld();
        uint32_t mv[2][4];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
#pragma unroll
          for (int q = 0; q < 4; ++q)
            mv[hf][q] = pack_h2(__uint_as_float(gr[q][2 * hf]) * wv[hf][q][0],
                                __uint_as_float(gr[q][2 * hf + 1]) * wv[hf][q][1]);
        // W_end o X is S's operand: the mask takes its space once S is done
        ok = cwait(&sm.mbS, par) && ok;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int t = 16 * (warp & 3) + (lane >> 2) + 8 * hf;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint32_t*>(sm.WX + off1(t, 8 * (2 * q + cpar) + 2 * (lane & 3))) =
                mv[hf][q];
        }
      }
      tc5::fence_proxy_async();
      tc5::fence_before_sync();
      warp_arrive(&sm.mb3, lane);  // -> Y2

      // ---- the carry: ht_c in; ht_{c+1} = R(-Psi_c) (exp(cs_63) ht_c + S_c) out -------
      // S_c (ready since the mask phase) is read before the carry is waited for
      uint32_t sv[32];
      tc5::ld_32x32b_x32(tmem + tq + kColB + (uint32_t)ccol, sv);
      tc5::wait_ld();
      const float psi_c = ROT ? sm.Psi[pair] : 0.f;
      float cp = 1.f, sp = 0.f;
      if (ROT) __sincosf(psi_c, &sp, &cp);
      const float sg = (nrow & 1) ? -sp : sp;  // R(-Psi): re' = c re + s im, im' = c im - s re
      float phi;  // Phi_c of this thread's pair
      float ca0 = 1.f, sa0 = 0.f;  // R(-angle0): h0 into the frame of chunk 0
      const float4* h0row = nullptr;
      if (c == 0) {
        phi = a.angle0 ? a.angle0[s * NH + pair] : 0.f;
        if (a.angle0) __sincosf(wrap_angle(phi), &sa0, &ca0);
        if (a.h0) h0row = reinterpret_cast<const float4*>(a.h0 + (s * NS + nrow) * PD + ccol);
      } else {
        ok = cwait(&sm.mbR, rpar) && ok;
        rpar ^= 1u;
        phi = sm.phibuf[pair];
      }
      const float sg0 = (nrow & 1) ? -sa0 : sa0;
      // eight elements of this thread's part of ht_c (columns ccol + 8 q ..)
      auto carry_in = [&](int q, float (&hq)[8]) {
        if (c == 0) {
          if (h0row) {
#pragma unroll
            for (int j2 = 0; j2 < 2; ++j2) {
              const float4 v = h0row[2 * q + j2];
              const float e4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const float o = __shfl_xor_sync(0xffffffffu, e4[k], 1);
                hq[4 * j2 + k] = fmaf(ca0, e4[k], sg0 * o);
              }
            }
          } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) hq[j] = 0.f;
          }
        } else {
          const float4* src = reinterpret_cast<const float4*>(sm.TH);
          const float4 v0 = src[(warp * 8 + 2 * q) * 32 + lane];
          const float4 v1 = src[(warp * 8 + 2 * q + 1) * 32 + lane];
          hq[0] = v0.x; hq[1] = v0.y; hq[2] = v0.z; hq[3] = v0.w;
          hq[4] = v1.x; hq[5] = v1.y; hq[6] = v1.z; hq[7] = v1.w;
        }
      };
      const float phi_next = wrap_angle(phi + psi_c);
      const float aE = P.eE;
      float cf = 1.f, sf = 0.f;  // R(Phi_{c+1}) for the final state
      if (last && (ROT || a.angle0)) __sincosf(phi_next, &sf, &cf);
      const float sgf = (nrow & 1) ? sf : -sf;  // R(+Phi): re' = c re - s im, im' = c im + s re
      float* slot_out = ws.ring + (s * 2 + ((c + 1) & 1)) * (int64_t)kSlotFloats;
      float hmx = 0.f;  // max |ht_c| of this thread
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float hq[8];
        carry_in(q, hq);
        float hn[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          hmx = fmaxf(hmx, fabsf(hq[j]));
          const float v = fmaf(aE, hq[j], __uint_as_float(sv[8 * q + j]));
          const float o = __shfl_xor_sync(0xffffffffu, v, 1);
          hn[j] = fmaf(cp, v, sg * o);
        }
        if (!last) {
          float4* dst = reinterpret_cast<float4*>(slot_out);
          __stcg(dst + (warp * 8 + 2 * q) * 32 + lane, make_float4(hn[0], hn[1], hn[2], hn[3]));
          __stcg(dst + (warp * 8 + 2 * q + 1) * 32 + lane, make_float4(hn[4], hn[5], hn[6], hn[7]));
        } else if (a.hT) {
          float ho[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float o = __shfl_xor_sync(0xffffffffu, hn[j], 1);
            ho[j] = fmaf(cf, hn[j], sgf * o);
          }
          float4* dst = reinterpret_cast<float4*>(a.hT + (s * NS + nrow) * PD + ccol + 8 * q);
          dst[0] = make_float4(ho[0], ho[1], ho[2], ho[3]);
          dst[1] = make_float4(ho[4], ho[5], ho[6], ho[7]);
        }
      }
      if ((nrow & 1) == 0 && ccol == 0) {
        if (!last) slot_out[NS * PD + pair] = phi_next;
        else if (a.angleT) a.angleT[s * NH + pair] = phi_next;
      }
      warp_arrive(&sm.mb5, lane);  // -> publish the carry
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) hmx = fmaxf(hmx, __shfl_xor_sync(0xffffffffu, hmx, o));
      if (lane == 0) sm.hmax[warp] = hmx;
      if (last) {
        const bf16* Xg = static_cast<const bf16*>(a.X);
        const bf16* Bg = static_cast<const bf16*>(a.B);
        if (a.xprevT && tid < PD)
          a.xprevT[s * PD + tid] = __bfloat162float(Xg[((b * L + L - 1) * H + h) * PD + tid]);
        if (a.bprevT && h % (H / G) == 0 && tid < NS)
          a.bprevT[(b * G + g) * NS + tid] = __bfloat162float(Bg[((b * L + L - 1) * G + g) * NS + tid]);
      }
      if (warp < 2) {  // the next unit's raw chunk scalars
        const bool okt = cwait(&sm.mbT, par, 64);
        const long long nx = sm.unit[par ^ 1u];
        if (okt && nx < total) stage_params(nx, par ^ 1u);
      }
      asm volatile("bar.sync 2, %0;" ::"n"(kCompute) : "memory");  // the maxima of ht_c
      // ---- ht_c 2^k in fp16 for Y1, k from the largest |ht_c| -------------------------
      int kexp = 0;
      {
        float m = sm.hmax[0];
#pragma unroll
        for (int w = 1; w < 8; ++w) m = fmaxf(m, sm.hmax[w]);
        if (m > 0.f) {
          int e;
          frexpf(m, &e);  // m < 2^e
          kexp = min(max(14 - e, -100), 100);
        }
        const float sc = ldexpf(1.f, kexp);
        // the tile takes the space of X and M: Y2 must be done
        ok = cwait(&sm.mbY2, par) && ok;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float hq[8];
          carry_in(q, hq);
          *reinterpret_cast<uint4*>(sm.X + nrow * 128 + (((ccol / 8 + q) ^ (nrow & 7)) << 4)) =
              make_uint4(pack_h2(sc * hq[0], sc * hq[1]), pack_h2(sc * hq[2], sc * hq[3]),
                         pack_h2(sc * hq[4], sc * hq[5]), pack_h2(sc * hq[6], sc * hq[7]));
        }
      }
      tc5::fence_proxy_async();
      tc5::fence_before_sync();
      warp_arrive(&sm.mb6, lane);  // -> Y1

      // ---- outputs: y = exp(cs) 2^-k Y1 + Y2 + D x, rounded to bf16 -------------------
      {
        const bf16* Xg = static_cast<const bf16*>(a.X);
        const float Dh = a.D ? a.D[h] : 0.f;
        uint32_t xr[2][4];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int r = 16 * (warp & 3) + (lane >> 2) + 8 * hf;
          const int64_t t = tbase + r;
          const bool valid = r > 0 && t < L;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            xr[hf][q] = valid ? __ldg(reinterpret_cast<const unsigned int*>(
                                    Xg + ((b * L + t) * H + h) * PD + ccol + 8 * q + 2 * (lane & 3)))
                              : 0u;
        }
        const bool ok2 = cwait(&sm.mbY1, par) && ok;
        tc5::fence_after_sync();
        uint32_t y1[16], y2[16];
        tc5::ld_16x256b_x4(tmem + tq + kColB + (uint32_t)ccol, y1);
        tc5::ld_16x256b_x4(tmem + tq + kColA + (uint32_t)ccol, y2);
        tc5::wait_ld();
        tc5::fence_before_sync();
        const float isc = ldexpf(1.f, -kexp);
        bf16* const Y_seq = static_cast<bf16*>(a.Y) + (b * L * H + h) * PD;
        if (ok2) {
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const int r = 16 * (warp & 3) + (lane >> 2) + 8 * hf;
            const int64_t t = tbase + r;
            if (r > 0 && t < L) {
              const float er = P.ecs[r] * isc;
              bf16* yrow = Y_seq + t * H * PD;
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int p = ccol + 8 * q + 2 * (lane & 3);
                const float x0 = __uint_as_float(xr[hf][q] << 16);
                const float x1 = __uint_as_float(xr[hf][q] & 0xffff0000u);
                const float v0 = fmaf(Dh, x0, fmaf(er, __uint_as_float(y1[4 * q + 2 * hf]),
                                                   __uint_as_float(y2[4 * q + 2 * hf])));
                const float v1 = fmaf(Dh, x1, fmaf(er, __uint_as_float(y1[4 * q + 2 * hf + 1]),
                                                   __uint_as_float(y2[4 * q + 2 * hf + 1])));
                *reinterpret_cast<uint32_t*>(yrow + p) = pack_bf16(v0, v1);
              }
            }
          }
        }
      }
    }
  }

  tc5::fence_before_sync();
  __syncthreads();
  if (warp == 0) tc5::tmem_dealloc(tmem, kTmemCols);
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

struct Occ {
  int nsm = 0, per_sm[2] = {0, 0};
};

}  // namespace

bool fwd_cp_shape_ok(const FwdArgs& a) {
  return a.bf16 && a.N == NS && a.P == PD && a.L > 0 && (a.chunk == 0 || a.chunk == Q);
}

bool fwd_cp_supported(const FwdArgs& a) {
  return fwd_cp_shape_ok(a) && a.x_tok_stride == 0 && a.theta16 == nullptr &&
         a.Bbias == nullptr && a.Cbias == nullptr && al16(a.X) && al16(a.B) && al16(a.C) &&
         al16(a.Y) && al16(a.theta) && al16(a.h0) && al16(a.hT) && al16(a.bprev0);
}

size_t fwd_cp_workspace_bytes(int64_t b, int64_t H) {
  const int64_t S = b * H;
  return header_bytes(S) + (size_t)S * 2 * kSlotFloats * sizeof(float);
}

cudaError_t launch_fwd_cp(const FwdArgs& a, void* workspace, cudaStream_t s) {
  const int64_t S = a.b * a.H;
  if (S == 0) return cudaSuccess;
  CpMaps tm;
  memset(&tm, 0, sizeof(tm));
  const uint64_t L = (uint64_t)a.L, b = (uint64_t)a.b, H = (uint64_t)a.H, G = (uint64_t)a.G;
  bool ok = encode_map(&tm.B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.B, NS, G, L, b, 2, 64,
                       CU_TENSOR_MAP_SWIZZLE_128B) &&
            encode_map(&tm.C, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.C, NS, G, L, b, 2, 64,
                       CU_TENSOR_MAP_SWIZZLE_128B) &&
            encode_map(&tm.X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.X, PD, H, L, b, 2, 64,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  if (ok && a.theta)
    ok = encode_map(&tm.theta, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.theta, NH, H, L, b, 4, NH,
                    CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!ok) return cudaErrorInvalidValue;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  CpWs ws;
  ws.ticket = reinterpret_cast<unsigned long long*>(w);
  ws.abort = reinterpret_cast<unsigned int*>(w + 8);
  ws.flags = reinterpret_cast<unsigned int*>(w + 64);
  ws.ring = reinterpret_cast<float*>(w + header_bytes(S));
  cudaError_t e = cudaMemsetAsync(w, 0, 64 + 4 * (size_t)S, s);
  if (e != cudaSuccess) return e;

  const int nC = (int)((a.L + QT - 1) / QT);
  const long long total = (long long)S * nC;
  const size_t smem = sizeof(Smem) + 1024;
  const bool rot = a.theta != nullptr;
  // CTAs per SM from registers, shared memory and TMEM (128 of the 512 columns
  // each), computed here: the runtime's occupancy query does not count several
  // CTAs per SM for this kernel although they run (measured).  More CTAs than
  // fit would only start later and find no units left.
  static Occ occ[16];
  static std::mutex mu;
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int per_sm = 0, nsm = 0;
  {
    std::lock_guard<std::mutex> lk(mu);
    Occ& o = occ[dev & 15];
    if (o.nsm == 0) {
      int smem_sm = 0, reserved = 0;
      cudaFuncAttributes fa[2];
      e = cudaFuncSetAttribute(fwd_cp_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(fwd_cp_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
      // several CTAs share an SM only if the SM is configured with the largest
      // shared-memory carveout; the default may size it for one CTA
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(fwd_cp_kernel<false>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(fwd_cp_kernel<true>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
      if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa[0], fwd_cp_kernel<false>);
      if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa[1], fwd_cp_kernel<true>);
      if (e == cudaSuccess) e = cudaDeviceGetAttribute(&o.nsm, cudaDevAttrMultiProcessorCount, dev);
      if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
      if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
      if (e != cudaSuccess) {
        o.nsm = 0;
        return e;
      }
      for (int v = 0; v < 2; ++v) {
        const int warps = kCtaThreads / 32;
        const int regs_warp = ((fa[v].numRegs * 32 + 255) / 256) * 256;
        int n = 65536 / (regs_warp * warps);
        n = std::min(n, smem_sm / (int)(smem + reserved));
        n = std::min(n, 512 / (int)kTmemCols);
        n = std::min(n, 2048 / kCtaThreads);
        o.per_sm[v] = std::max(n, 1);
      }
    }
    nsm = o.nsm;
    per_sm = o.per_sm[rot ? 1 : 0];
  }
  const long long grid = total < (long long)nsm * per_sm ? total : (long long)nsm * per_sm;
  if (rot)
    fwd_cp_kernel<true><<<(unsigned)grid, kCtaThreads, smem, s>>>(a, tm, ws, total, nC);
  else
    fwd_cp_kernel<false><<<(unsigned)grid, kCtaThreads, smem, s>>>(a, tm, ws, total, nC);
  return cudaGetLastError();
}

cudaError_t read_and_clear_cp_wait_timeouts(unsigned int* count) {
  const unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(count, g_cp_wait_timeouts, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_cp_wait_timeouts, &zero, sizeof(unsigned int));
}

}  // namespace m3ssd
