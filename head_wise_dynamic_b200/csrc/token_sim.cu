// Approximate DINO cosines of the token-wise heads on the tensor cores.
//
// SAF3R ("SAF3R: Dynamic Sparse Attention for Feed-Forward 3D Reconstruction Transformers"),
// section 4.1, "DINO Top-K Kernel": a patch query ranks, frame by frame, the patch tokens by the
// cosine of their DINO features.  All S*P queries against all S*P patch tokens is a dense
// contraction over the feature width, so it runs here as a tcgen05 GEMM: the unit features
// rounded to fp16 (K-major, 128-byte swizzle, staged by TMA), fp32 accumulators in TMEM, fp16
// scores written to a row-major [rows][ld] buffer.  The scores only pre-select: the ranking
// kernel recomputes exactly every candidate that the bound below cannot separate.
//
// Bound of |score - exact cosine of the fp32 unit vectors| (|u| = |w| = 1, dim <= 384):
//   fp16 operands: (2 * 2^-11 + 2^-22) * sum|u_i w_i| + 2^-25 * (sum|u_i| + sum|w_i|)
//                  <= 9.77e-4 + 1.2e-6
//   the tensor core's fp32 accumulation of <= 384 exact products (partial sums <= 1):
//                  taken as <= 384 * 2^-20 = 3.7e-4, i.e. at least 20 significant bits kept per
//                  addition, a margin of several bits over an fp32 adder
//   rounding the score to fp16 (|score| < 2): <= 2^-11 = 4.9e-4
//   total < 1.85e-3 < kTokScoreErr = 2e-3 (select.cu).
//
// One CTA per SM, persistent over 128 x 256 output tiles (contiguous runs of tiles, row-block
// major, so consecutive tiles reuse the same query rows from L2).  Warp 0 issues the TMA copies
// of one 64-feature slice of the 128 query rows and the 256 candidate rows per stage (4 stages);
// warp 1 allocates TMEM and issues 4 MMAs (K = 16) per stage from one elected lane into one of
// two 256-column accumulators; warps 2-5 (one TMEM lane quarter each, one thread per query row)
// convert a finished accumulator to fp16 and store it while the next tile accumulates.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "ptx.cuh"

namespace saf3r {

namespace {

constexpr int kSimStages = 4;
constexpr int kSimThreads = 192;
constexpr uint32_t kSimABytes = 128 * 128;  // 128 rows x 64 fp16
constexpr uint32_t kSimBBytes = 256 * 128;  // 256 rows x 64 fp16
constexpr uint32_t kSimStageBytes = kSimABytes + kSimBBytes;

struct __align__(1024) SimSmem {
  uint8_t a[kSimStages][kSimABytes];
  uint8_t b[kSimStages][kSimBBytes];
  uint64_t full[kSimStages];
  uint64_t empty[kSimStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drained;
  uint32_t tmem_base;
  int abort;
};

// Instruction descriptor of kind::f16 with fp16 A/B (format 0), fp32 accumulate, both K-major.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

struct TileRange {
  long long t0, t1;
};

__device__ __forceinline__ TileRange my_tiles(const TokenSimParams& p) {
  const long long total = static_cast<long long>(p.n_rb) * p.n_ct;
  TileRange r;
  r.t0 = total * blockIdx.x / gridDim.x;
  r.t1 = total * (blockIdx.x + 1) / gridDim.x;
  return r;
}

__device__ void sim_producer(const TokenSimParams& p, SimSmem& sm, const CUtensorMap& tm) {
  volatile int* abort = &sm.abort;
  tma_prefetch_desc(&tm);
  const TileRange tr = my_tiles(p);
  uint32_t it = 0;
  bool ok = true;
  for (long long t = tr.t0; ok && t < tr.t1; ++t) {
    const int rb = static_cast<int>(t / p.n_ct), ct = static_cast<int>(t - static_cast<long long>(rb) * p.n_ct);
    const int arow = p.r0 + rb * 128, brow = ct * 256;
    for (int kc = 0; kc < p.n_kc; ++kc, ++it) {
      const uint32_t st = it % kSimStages, ph = (it / kSimStages) & 1;
      if (it >= kSimStages && !mbar_wait(&sm.empty[st], ph ^ 1, abort, p.err, p.wait_budget, SAF3R_ERR_TIMEOUT)) {
        ok = false;
        break;
      }
      mbar_arrive_expect_tx(&sm.full[st], kSimStageBytes);
      tma_load_2d(sm.a[st], &tm, kc * 64, arow, &sm.full[st]);
      tma_load_2d(sm.b[st], &tm, kc * 64, brow, &sm.full[st]);
      tma_load_2d(sm.b[st] + kSimABytes, &tm, kc * 64, brow + 128, &sm.full[st]);
    }
  }
  // every copy issued must land before the CTA exits (bounded, ignores the abort flag)
  const long long drain = kDrainBudget;
  for (uint32_t c = (it > kSimStages ? it - kSimStages : 0); c < it; ++c)
    mbar_wait_drain(&sm.full[c % kSimStages], (c / kSimStages) & 1, drain);
}

__device__ void sim_mma(const TokenSimParams& p, SimSmem& sm, uint32_t tmem) {
  volatile int* abort = &sm.abort;
  constexpr uint32_t idesc = idesc_f16_f32(128, 256);
  const uint64_t da = smem_desc_sw128(smem_u32(sm.a[0]), 16, 1024);
  const uint64_t db = smem_desc_sw128(smem_u32(sm.b[0]), 16, 1024);
  constexpr uint64_t kStepA = kSimABytes >> 4, kStepB = kSimBBytes >> 4;
  const TileRange tr = my_tiles(p);
  uint32_t it = 0, i = 0;
  bool ok = true, issued = false;
  for (long long t = tr.t0; ok && t < tr.t1; ++t, ++i) {
    const uint32_t buf = i & 1;
    if (i >= 2 && !__all_sync(0xffffffffu, mbar_wait(&sm.acc_empty[buf], ((i >> 1) + 1) & 1, abort, p.err,
                                                     p.wait_budget, SAF3R_ERR_TIMEOUT)))
      break;
    tc_fence_after();
    for (int kc = 0; kc < p.n_kc; ++kc, ++it) {
      const uint32_t st = it % kSimStages, ph = (it / kSimStages) & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.full[st], ph, abort, p.err, p.wait_budget, SAF3R_ERR_TIMEOUT))) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(tmem + buf * 256, da + st * kStepA + 2 * kk, db + st * kStepB + 2 * kk, idesc,
                 (kc > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&sm.empty[st]);
      }
      __syncwarp();
      issued = true;
    }
    if (!ok) break;
    if (elect_one()) mma_commit(&sm.acc_full[buf]);
    __syncwarp();
  }
  // every product issued (also of a tile left unfinished after an abort) must finish before
  // TMEM is released: one more commit covers them all
  if (issued) {
    if (elect_one()) mma_commit(&sm.drained);
    __syncwarp();
    mbar_wait_drain(&sm.drained, 0, kDrainBudget);
  }
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ void sim_epilogue(const TokenSimParams& p, SimSmem& sm, uint32_t tmem, int warp, int lane) {
  volatile int* abort = &sm.abort;
  const int quarter = warp & 3;  // TMEM lanes [32 * quarter, +32) are this warp's
  const TileRange tr = my_tiles(p);
  uint32_t i = 0;
  for (long long t = tr.t0; t < tr.t1; ++t, ++i) {
    const uint32_t buf = i & 1;
    if (!__all_sync(0xffffffffu, mbar_wait(&sm.acc_full[buf], (i >> 1) & 1, abort, p.err, p.wait_budget,
                                           SAF3R_ERR_TIMEOUT)))
      break;
    tc_fence_after();
    const int rb = static_cast<int>(t / p.n_ct), ct = static_cast<int>(t - static_cast<long long>(rb) * p.n_ct);
    const int row = rb * 128 + quarter * 32 + lane;  // row of the chunk
    const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + buf * 256;
    __half* dst = reinterpret_cast<__half*>(p.scores) + static_cast<size_t>(row) * p.ld;
#pragma unroll 1
    for (int c = 0; c < 256; c += 64) {
      uint32_t r0[32], r1[32];
      tmem_ld32(taddr + c, r0);
      tmem_ld32(taddr + c + 32, r1);
      tmem_wait_ld();
      const long long col0 = static_cast<long long>(ct) * 256 + c;
      if (row < p.rows) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (col0 + 8 * j + 8 <= p.ld)
            *reinterpret_cast<uint4*>(dst + col0 + 8 * j) =
                make_uint4(pack_half2(__uint_as_float(r0[8 * j]), __uint_as_float(r0[8 * j + 1])),
                           pack_half2(__uint_as_float(r0[8 * j + 2]), __uint_as_float(r0[8 * j + 3])),
                           pack_half2(__uint_as_float(r0[8 * j + 4]), __uint_as_float(r0[8 * j + 5])),
                           pack_half2(__uint_as_float(r0[8 * j + 6]), __uint_as_float(r0[8 * j + 7])));
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (col0 + 32 + 8 * j + 8 <= p.ld)
            *reinterpret_cast<uint4*>(dst + col0 + 32 + 8 * j) =
                make_uint4(pack_half2(__uint_as_float(r1[8 * j]), __uint_as_float(r1[8 * j + 1])),
                           pack_half2(__uint_as_float(r1[8 * j + 2]), __uint_as_float(r1[8 * j + 3])),
                           pack_half2(__uint_as_float(r1[8 * j + 4]), __uint_as_float(r1[8 * j + 5])),
                           pack_half2(__uint_as_float(r1[8 * j + 6]), __uint_as_float(r1[8 * j + 7])));
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.acc_empty[buf]);
  }
}

}  // namespace

__global__ void __launch_bounds__(kSimThreads, 1)
    token_sim_kernel(const __grid_constant__ TokenSimParams p, const __grid_constant__ CUtensorMap tm) {
  extern __shared__ uint8_t smem_raw[];
  SimSmem& sm = *reinterpret_cast<SimSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kSimStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.acc_full[b], 1);
      mbar_init(&sm.acc_empty[b], 4);
    }
    mbar_init(&sm.drained, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  if (warp == 0) {
    if (lane == 0) sim_producer(p, sm, tm);
    __syncwarp();
  } else if (warp == 1) {
    sim_mma(p, sm, tmem);
  } else {
    sim_epilogue(p, sm, tmem, warp, lane);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

size_t token_sim_smem_bytes() { return sizeof(SimSmem) + 1024; }

cudaError_t launch_token_sim(const TokenSimParams& p, const CUtensorMap& tm, int num_sms, cudaStream_t stream) {
  const long long tiles = static_cast<long long>(p.n_rb) * p.n_ct;
  if (tiles <= 0) return cudaSuccess;
  const size_t smem = token_sim_smem_bytes();
  cudaError_t e =
      cudaFuncSetAttribute(token_sim_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int grid = tiles < num_sms ? static_cast<int>(tiles) : num_sms;
  token_sim_kernel<<<grid, kSimThreads, smem, stream>>>(p, tm);
  return cudaGetLastError();
}

}  // namespace saf3r
