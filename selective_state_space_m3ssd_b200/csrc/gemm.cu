// Dense bf16 GEMM on the sm_100a tensor cores, for the block's two projections
// ("VikramLex/mamba3-minimal" README, "Architecture": in_proj and out_proj are
// plain linear maps):
//     D (M x N, bf16, row-major, row stride ldd) = A (M x K) W^T,
// with A (M x K) and W (N x K) bf16, row-major (both K-major operands), and
// fp32 accumulation in tensor memory.
//
// One persistent CTA per SM walks output tiles of (128 H) x 256, H = 1 or 2
// row halves.  When A is the larger operand (M > N) tile t covers row block
// t div nt and column block t mod nt: the CTAs in flight read a few A row
// blocks and every W panel, which stays in L2, so A streams from DRAM once;
// otherwise (row block t mod mt, column block t div mt) shares W panels the
// same way.  Warp roles:
//   warp 0   one thread issues the TMA copies of the A and W slices (64 of K
//            each, 128-byte swizzled) into a ring of stages;
//   warp 1   allocates the 512 TMEM columns; one thread issues the tcgen05
//            MMAs (M128 N256 K16, four per stage and half, every half reading
//            the stage's one W slice) and commits each stage back to the
//            producer;
//   warps 2 .. 4H+1  the epilogue: warp w reads TMEM lane quarter w mod 4 of
//            half (w - 2) / 4 (one output row a thread) 32 columns at a time,
//            rounds to bf16 into one of its two 2 KB staging blocks in shared
//            memory, and one lane writes the 32 x 32 block to D with a TMA
//            tensor store (an asynchronous bulk group).  Row-per-thread global
//            stores would touch 32 lines a warp instruction; with them the
//            output writes, not the products, set the kernel's rate (an
//            experiment that skipped the stores ran at 0.96 of the bf16 peak).
//            A thread first reads its whole row (256 columns) out of TMEM into
//            registers as bf16 and hands TMEM back, so the staging and the
//            stores drain while the next tile's products run.  Outputs whose
//            rows are not 16-byte aligned take plain stores instead.
// With H = 1 (four stages) the two 256-column accumulators alternate, so the
// epilogue of a tile overlaps the products of the next.  With H = 2 (three
// stages of 64 KB) the halves fill all 512 columns and the epilogue runs
// between tiles, but each K slice of W serves 256 rows: a third fewer operand
// bytes per product from L2, and the stages in flight cover twice the product
// time, which is what limits the single-half tile.  The host picks H per shape
// by how evenly the tiles fill the SMs.
// Every wait is bounded (2 s of %globaltimer); a wait that runs out sets a
// shared flag that ends the other roles' waits too, the MMA thread and the
// producer let their work in flight land, and the launch is counted in a
// device word the host query reads.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <cstddef>
#include <cstring>

#include "internal.h"
#include "tc5.cuh"

namespace m3ssd {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

__device__ unsigned int g_gemm_wait_timeouts;

namespace {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr uint32_t kABytes = BM * BK * 2;  // one half's A slice
constexpr uint32_t kWBytes = BN * BK * 2;
constexpr uint32_t kTmemCols = 2 * BN;
constexpr uint32_t kIdesc = tc5::idesc_bf16(BM, BN, false, false);
constexpr uint64_t kWaitLimitNs = 2000000000ull;

template <int H>
struct Cfg {
  static constexpr int STAGES = H == 1 ? 4 : 3;
  static constexpr int NACC = H == 1 ? 2 : 1;  // accumulators in flight
  static constexpr int EPI_WARPS = 4 * H;
  static constexpr int THREADS = 32 * (2 + EPI_WARPS);
};

constexpr uint32_t kStgBytes = 32 * 32 * 2;  // one warp's 32 x 32 bf16 output block

template <int H>
struct GSmem {
  static constexpr int S = Cfg<H>::STAGES;
  // every buffer a TMA copy reads or writes starts on a 1024-byte boundary (the
  // struct is placed at one, and each array before it is a multiple of 1024 bytes)
  uint8_t a[S][H * kABytes];
  uint8_t w[S][kWBytes];
  uint8_t stg[Cfg<H>::EPI_WARPS][2][kStgBytes];  // output staging, two blocks an epilogue warp
  uint64_t full[S];        // stage loaded (TMA bytes)
  uint64_t empty[S];       // stage consumed (MMA commit)
  uint64_t tfull[2];       // accumulator ready (MMA commit)
  uint64_t tempty[2];      // accumulator read (every epilogue warp)
  uint64_t drain;          // every product issued has finished
  uint32_t tmem;
  uint32_t err;
};

static_assert(sizeof(GSmem<1>) + 1024 <= 232448 && sizeof(GSmem<2>) + 1024 <= 232448,
              "one CTA's shared memory");
static_assert(offsetof(GSmem<1>, w) % 1024 == 0 && offsetof(GSmem<1>, stg) % 1024 == 0 &&
                  offsetof(GSmem<2>, w) % 1024 == 0 && offsetof(GSmem<2>, stg) % 1024 == 0,
              "TMA buffers on 1024-byte boundaries");

struct GMaps {
  CUtensorMap a;  // bf16 (K, M), box 64 x 128 H, 128-byte swizzle
  CUtensorMap w;  // bf16 (K, N), box 64 x 256, 128-byte swizzle
  CUtensorMap d;  // bf16 (N, M) with row stride ldd, box 32 x 32 (stores; when vec)
};

struct GArgs {
  int M, N, K;
  int64_t ldd;
  __nv_bfloat16* D;
  int mt, nt, nk;  // tiles along M and N, K slices
  bool vec;        // TMA stores (ldd % 8 == 0 and D 16-byte aligned)
  bool nfast;      // tile t = (row block t / nt, column block t % nt), else (t % mt, t / mt)
};

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <int H>
__global__ void __launch_bounds__(Cfg<H>::THREADS, 1)
    gemm_bf16_kernel(GArgs g, const __grid_constant__ GMaps tm) {
  constexpr int STAGES = Cfg<H>::STAGES, NACC = Cfg<H>::NACC;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw_addr = tc5::saddr(smem_raw);
  GSmem<H>& sm =
      *reinterpret_cast<GSmem<H>*>(smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = g.mt * g.nt;
  volatile uint32_t* err = &sm.err;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      tc5::mbar_init(&sm.full[s], 1);
      tc5::mbar_init(&sm.empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc5::mbar_init(&sm.tfull[i], 1);
      tc5::mbar_init(&sm.tempty[i], Cfg<H>::EPI_WARPS);
    }
    tc5::mbar_init(&sm.drain, 1);
    tc5::fence_mbar_init();
    sm.err = 0;
  }
  if (warp == 1) tc5::tmem_alloc(&sm.tmem, kTmemCols);
  tc5::fence_before_sync();
  __syncthreads();
  tc5::fence_after_sync();
  const uint32_t tmem = sm.tmem;

  if (warp == 0) {
    // ---- producer ---------------------------------------------------------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0;        // stages armed at least once (bit mask)
      uint32_t last_par = 0;     // parity of each stage's last arming (bit mask)
      for (int t = blockIdx.x; t < total && !*err; t += gridDim.x) {
        const int mb = g.nfast ? t / g.nt : t % g.mt, nb = g.nfast ? t % g.nt : t / g.mt;
        for (int kb = 0; kb < g.nk; ++kb) {
          if (!tc5::mbar_wait(&sm.empty[stage], phase ^ 1u, kWaitLimitNs, err)) {
            *err = 1;
            break;
          }
          tc5::mbar_arrive_expect_tx(&sm.full[stage], H * kABytes + kWBytes);
          tc5::tma_load_2d(tc5::saddr(sm.a[stage]), &tm.a, &sm.full[stage], kb * BK,
                           mb * (H * BM));
          tc5::tma_load_2d(tc5::saddr(sm.w[stage]), &tm.w, &sm.full[stage], kb * BK, nb * BN);
          armed |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // the copies issued last land before the CTA can exit
      for (int s = 0; s < STAGES; ++s)
        if (armed & (1u << s)) (void)tc5::mbar_wait(&sm.full[s], (last_par >> s) & 1u, kWaitLimitNs);
    }
  } else if (warp == 1) {
    // ---- MMA issue -----------------------------------------------------------------
    if (lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, aphase = 0;
      for (int t = blockIdx.x; t < total && !*err; t += gridDim.x) {
        if (!tc5::mbar_wait(&sm.tempty[acc], aphase ^ 1u, kWaitLimitNs, err)) {
          *err = 1;
          break;
        }
        tc5::fence_after_sync();
        const uint32_t d = tmem + (uint32_t)(acc * BN);  // half 1 (H = 2): columns 256 ..
        bool ok = true;
        for (int kb = 0; kb < g.nk; ++kb) {
          if (!tc5::mbar_wait(&sm.full[stage], phase, kWaitLimitNs, err)) {
            *err = 1;
            ok = false;
            break;
          }
          tc5::fence_after_sync();
          const uint64_t dw = tc5::desc_sw128(tc5::saddr(sm.w[stage]), 16, 1024);
#pragma unroll
          for (int hh = 0; hh < H; ++hh) {
            const uint64_t da = tc5::desc_sw128(tc5::saddr(sm.a[stage]) + hh * kABytes, 16, 1024);
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)  // +32 bytes a K step inside the swizzle atom
              tc5::mma_bf16(d + (uint32_t)(hh * BN), da + (uint64_t)(2 * k),
                            dw + (uint64_t)(2 * k), kIdesc, kb > 0 || k > 0);
          }
          tc5::commit(&sm.empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc5::commit(&sm.tfull[acc]);
        if (++acc == NACC) {
          acc = 0;
          aphase ^= 1u;
        }
      }
      // every product issued has finished before TMEM is released
      tc5::commit(&sm.drain);
      (void)tc5::mbar_wait(&sm.drain, 0, kWaitLimitNs);
    }
  } else {
    // ---- epilogue: TMEM lane quarter q = warp % 4 of half hh, one output row a thread
    const int q = warp & 3, hh = (warp - 2) >> 2;
    int acc = 0;
    uint32_t nst = 0;  // blocks staged by this warp (alternating staging blocks)
    uint32_t aphase = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x) {
      if (!tc5::mbar_wait(&sm.tfull[acc], aphase, kWaitLimitNs, err)) {
        *err = 1;
        break;
      }
      tc5::fence_after_sync();
      const int mb = g.nfast ? t / g.nt : t % g.mt, nb = g.nfast ? t % g.nt : t / g.mt;
      const int row = mb * (H * BM) + hh * BM + 32 * q + lane;
      const int col0 = nb * BN;
      __nv_bfloat16* const drow = g.D + (int64_t)row * g.ldd;
      const int nch = min(BN / 32, (g.N - col0 + 31) / 32);  // chunks with a valid column
      const uint32_t tbase = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)((acc + hh) * BN);
      if (g.vec) {
        // the thread's whole output row (256 columns) into registers as bf16, then
        // TMEM goes back to the MMA thread: the stores below drain while the next
        // tile's products run
        const int ew = warp - 2;
        const int row0 = mb * (H * BM) + hh * BM + 32 * q;
        uint32_t pk[BN / 32][16];
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          if (c < nch) {
#pragma unroll
            for (int hc = 0; hc < 2; ++hc) {  // 16 columns a load (fewer live registers)
              uint32_t v[16];
              tc5::ld_32x32b_x16(tbase + (uint32_t)(32 * c + 16 * hc), v);
              tc5::wait_ld();
              tc5::reg_after_ld(v);
#pragma unroll
              for (int j = 0; j < 8; ++j)
                pk[c][8 * hc + j] = pack2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
            }
          }
        }
        tc5::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc5::mbar_arrive(&sm.tempty[acc]);
        // stage each 32 x 32 block in shared memory and write it with a TMA store
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          if (c < nch) {
            uint8_t* const blk = sm.stg[ew][nst & 1];
            if (lane == 0) tc5::bulk_wait_group_read<1>();  // the block's previous store has read it
            __syncwarp();
            uint4* dst = reinterpret_cast<uint4*>(blk + lane * 64);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              dst[j] = make_uint4(pk[c][4 * j], pk[c][4 * j + 1], pk[c][4 * j + 2], pk[c][4 * j + 3]);
            tc5::fence_proxy_async();
            __syncwarp();
            if (lane == 0) {
              tc5::tma_store_2d(&tm.d, tc5::saddr(blk), col0 + 32 * c, row0);
              tc5::bulk_commit_group();
            }
            ++nst;
          }
        }
      } else {
        // plain stores, one row a thread
#pragma unroll 1
        for (int c = 0; c < nch; ++c) {
          const int col = col0 + 32 * c;
          uint32_t v[32];
          tc5::ld_32x32b_x32(tbase + (uint32_t)(32 * c), v);
          tc5::wait_ld();
          tc5::reg_after_ld(v);
          if (row < g.M) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (col + j < g.N) drow[col + j] = __float2bfloat16_rn(__uint_as_float(v[j]));
          }
        }
        tc5::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc5::mbar_arrive(&sm.tempty[acc]);
      }
      if (++acc == NACC) {
        acc = 0;
        aphase ^= 1u;
      }
    }
    if (lane == 0) tc5::bulk_wait_group<0>();  // every store of this warp has landed
    __syncwarp();
  }
  tc5::fence_before_sync();
  __syncthreads();
  tc5::fence_after_sync();
  if (warp == 1) tc5::tmem_dealloc(tmem, kTmemCols);
  if (threadIdx.x == 0 && sm.err) atomicAdd(&g_gemm_wait_timeouts, 1u);
}

bool encode_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_outer) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * 2};
  const cuuint32_t box[2] = {(cuuint32_t)BK, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// SMs of the current device (the grid is one persistent CTA per SM).
int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    return 148;
  }
  return n;
}

template <int H>
cudaError_t launch_h(const GArgs& g, const GMaps& tm, int grid, cudaStream_t s) {
  const size_t smem = sizeof(GSmem<H>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(gemm_bf16_kernel<H>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  gemm_bf16_kernel<H><<<grid, Cfg<H>::THREADS, smem, s>>>(g, tm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_bf16(int64_t M, int64_t N, int64_t K, const void* A, const void* W,
                             void* D, int64_t ldd, cudaStream_t s) {
  if (M == 0 || N == 0) return cudaSuccess;
  if (M < 0 || N < 0 || K < 1 || M > INT32_MAX || N > INT32_MAX || K > INT32_MAX || K % 8 != 0 ||
      ldd < N || (reinterpret_cast<uintptr_t>(A) & 15) || (reinterpret_cast<uintptr_t>(W) & 15) ||
      (reinterpret_cast<uintptr_t>(D) & 1))
    return cudaErrorInvalidValue;
  GMaps tm;
  memset(&tm, 0, sizeof(tm));
  // two row halves when their tiles fill at least 90 % of the SM rounds and
  // not much less evenly than single-half tiles
  const int64_t nt = (N + BN - 1) / BN, sms = sm_count();
  if (((M + BM - 1) / BM) * nt > INT32_MAX) return cudaErrorInvalidValue;  // tile index is an int
  const int64_t t1 = ((M + BM - 1) / BM) * nt, t2 = ((M + 2 * BM - 1) / (2 * BM)) * nt;
  const double f1 = (double)t1 / (double)(((t1 + sms - 1) / sms) * sms);
  const double f2 = (double)t2 / (double)(((t2 + sms - 1) / sms) * sms);
  const int H = (f2 >= 0.9 && f2 >= f1 - 0.05) ? 2 : 1;
  if (!encode_2d(&tm.a, A, (uint64_t)K, (uint64_t)M, (uint32_t)(H * BM)) ||
      !encode_2d(&tm.w, W, (uint64_t)K, (uint64_t)N, BN))
    return cudaErrorInvalidValue;
  GArgs g;
  g.M = (int)M;
  g.N = (int)N;
  g.K = (int)K;
  g.ldd = ldd;
  g.D = static_cast<__nv_bfloat16*>(D);
  g.mt = (int)((M + H * BM - 1) / (H * BM));
  g.nt = (int)nt;
  g.nk = (int)((K + BK - 1) / BK);
  g.vec = ldd % 8 == 0 && (reinterpret_cast<uintptr_t>(D) & 15) == 0;
  // the CTAs in flight share the panels of the smaller operand, which L2 keeps
  // while the larger one streams from DRAM once
  g.nfast = M > N;
  if (g.vec) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
    const cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)ldd * 2};
    const cuuint32_t box[2] = {32, 32};
    const cuuint32_t estr[2] = {1, 1};
    g.vec = fn && fn(&tm.d, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
                        CUDA_SUCCESS;
  }
  const int64_t tiles = (int64_t)g.mt * g.nt;
  const int grid = (int)(tiles < sms ? tiles : sms);
  return H == 2 ? launch_h<2>(g, tm, grid, s) : launch_h<1>(g, tm, grid, s);
}

cudaError_t read_and_clear_gemm_wait_timeouts(unsigned int* count) {
  const unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(count, g_gemm_wait_timeouts, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_gemm_wait_timeouts, &zero, sizeof(unsigned int));
}

}  // namespace m3ssd
