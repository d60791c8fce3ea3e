// Online index selection (SAF3R, section 4.3 "Online Pattern Adaptation").
//
//  * Query-probe Top-K: qbar = (1/N) sum_i q_i over all queries of the head
//    (fp64 sums, one rounding to fp32); score_j = qbar . k_j / sqrt(d) for
//    every key (fp64 dot, one rounding to fp32); the k patch keys of highest
//    score are kept, ties to the lower token index (radix select on
//    order-preserving 32-bit keys).
//  * Block-wise DINO Top-K: each flat 64-token tile gets the mean of the
//    L2-normalised DINO features of its patch tokens; tiles are compared by
//    cosine (fp64 dot of the normalised means); each query tile ranks all
//    tiles, itself included, best first, ties to the lower tile index.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"

namespace saf3r {

namespace {

constexpr int kProbePartials = 296;  // most row blocks (partial sums) per probe head
#ifndef SAF3R_PROBE_ROWS_IN_FLIGHT
#define SAF3R_PROBE_ROWS_IN_FLIGHT 4
#endif
constexpr int kProbeRowsInFlight = SAF3R_PROBE_ROWS_IN_FLIGHT;  // 16-byte loads per lane before use

__device__ __forceinline__ uint32_t order_key(float f) {
  // monotone map fp32 -> uint32 (larger float -> larger key)
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct ProbeArgs {
  int n_probe;
  int heads[kMaxHeads];      // head index of each probe head
  int k[kMaxHeads];          // kept patch keys
  int cache_off[kMaxHeads];  // int32 offset of the key list in the cache
};

// bf16 -> fp64 without a conversion instruction.  A bf16 is the top half of an fp32 (sign, 8-bit
// exponent, 7-bit mantissa).  Placed in the high word of a double with the exponent zero-extended
// to 11 bits, its bits read as x * 2^-896 exactly: for a normal x the exponent bias becomes 1023
// instead of 127, and a subnormal x stays subnormal with the same scale (finite x only).  Sums and
// products of such scaled values round exactly as those of the unscaled ones in the same order
// (a power-of-two scale commutes with rounding while the result is normal; below that, every sum
// of bf16 values is a multiple of 2^-133 and exact either way).
constexpr double kUnscale896 = 0x1p896;

// fp32 -> fp64 the same way: the sign, 8-bit exponent and 23-bit mantissa placed in a double's
// layout without rebiasing read as x * 2^-896 exactly (finite x, subnormals included).  Against an
// operand pre-multiplied by 2^896 the products are the unscaled ones, rounded alike.
__device__ __forceinline__ double f32_scaled(float f) {
  const uint32_t u = __float_as_uint(f);
  return __hiloint2double(static_cast<int>((u & 0x80000000u) | ((u & 0x7FFFFFFFu) >> 3)), static_cast<int>(u << 29));
}
__device__ __forceinline__ double bf16_lo_scaled(uint32_t w) {
  return __hiloint2double(static_cast<int>(((w & 0x8000u) << 16) | ((w & 0x7FFFu) << 13)), 0);
}
__device__ __forceinline__ double bf16_hi_scaled(uint32_t w) {
  return __hiloint2double(static_cast<int>((w & 0x80000000u) | ((w & 0x7FFF0000u) >> 3)), 0);
}

// The 8 bf16 features of a 16-byte chunk as fp64 scaled by 2^-896, in order.
__device__ __forceinline__ void bf16x8_to_f64(const uint4& w, double (&x)[8]) {
  x[0] = bf16_lo_scaled(w.x);
  x[1] = bf16_hi_scaled(w.x);
  x[2] = bf16_lo_scaled(w.y);
  x[3] = bf16_hi_scaled(w.y);
  x[4] = bf16_lo_scaled(w.z);
  x[5] = bf16_hi_scaled(w.z);
  x[6] = bf16_lo_scaled(w.w);
  x[7] = bf16_hi_scaled(w.w);
}

// acc[i] += feature i of a 16-byte chunk of 8 bf16 features (fp64 sums, scaled by 2^-896).
__device__ __forceinline__ void add_bf16x8(double (&acc)[8], const uint4& w) {
  double x[8];
  bf16x8_to_f64(w, x);
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] += x[i];
}

// qbar = (1/N) sum_i q_i for every probe head, in one launch.  Each block sums a contiguous
// range of rows: lane l of a warp reads the 16-byte chunk (l % 8) of row r + l / 8 (a warp reads
// 4 whole rows, 512 contiguous bytes, per load) and keeps the 8 column sums of its chunk; the
// next step's kProbeRowsInFlight rows are requested before this step's are added.  The lanes
// and warps that share a chunk are added in a fixed order into the block's partial sums; the
// last block of a head to finish (a counter, no waiting) adds the head's partials in a fixed
// order and rounds the mean once to fp32.  done[n_probe] starts at zero.
__global__ void __launch_bounds__(256) probe_mean_kernel(const uint16_t* __restrict__ q, int N, ProbeArgs a,
                                                         double* __restrict__ partial, unsigned* __restrict__ done,
                                                         float* __restrict__ qbar) {
  const int hp = blockIdx.y;
  const int h = a.heads[hp];
  const int rows_per = (N + gridDim.x - 1) / gridDim.x;
  const int r0 = blockIdx.x * rows_per;
  const int r1 = min(N, r0 + rows_per);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, sub = lane & 7;
  const uint4* qh = reinterpret_cast<const uint4*>(q + static_cast<size_t>(h) * N * kD);
  constexpr int kStep = 32 * kProbeRowsInFlight;
  double acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.0;
  const int rl = r0 + warp * 4 + (lane >> 3);  // this lane's first row
  uint4 w[kProbeRowsInFlight];
#pragma unroll
  for (int f = 0; f < kProbeRowsInFlight; ++f) {
    const int r = rl + 32 * f;
    w[f] = r < r1 ? qh[static_cast<size_t>(r) * 8 + sub] : make_uint4(0u, 0u, 0u, 0u);
  }
  for (int rb = rl; rb < r1; rb += kStep) {
    uint4 nx[kProbeRowsInFlight];
#pragma unroll
    for (int f = 0; f < kProbeRowsInFlight; ++f) {
      const int r = rb + kStep + 32 * f;
      nx[f] = r < r1 ? qh[static_cast<size_t>(r) * 8 + sub] : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int f = 0; f < kProbeRowsInFlight; ++f) add_bf16x8(acc, w[f]);  // rows past r1 add zeros
#pragma unroll
    for (int f = 0; f < kProbeRowsInFlight; ++f) w[f] = nx[f];
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 8);
    acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 16);
  }
  __shared__ double wsum[8][kD];
  __shared__ bool last;
  if (lane < 8) {
#pragma unroll
    for (int i = 0; i < 8; ++i) wsum[warp][8 * sub + i] = acc[i];
  }
  __syncthreads();
  double* hpart = partial + static_cast<size_t>(hp) * gridDim.x * kD;
  if (threadIdx.x < kD) {
    double t = 0.0;
    for (int w8 = 0; w8 < 8; ++w8) t += wsum[w8][threadIdx.x];
    hpart[static_cast<size_t>(blockIdx.x) * kD + threadIdx.x] = t * kUnscale896;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = atomicAdd(&done[hp], 1u) == gridDim.x - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  // four threads per column take every fourth partial, loads batched; fixed order throughout
  const int c = threadIdx.x & (kD - 1), g = threadIdx.x >> 6;
  double t = 0.0;
#pragma unroll 8
  for (int b2 = g; b2 < static_cast<int>(gridDim.x); b2 += 4) t += __ldcg(&hpart[static_cast<size_t>(b2) * kD + c]);
  wsum[g][c] = t;
  __syncthreads();
  if (g == 0)
    qbar[hp * kD + c] = static_cast<float>(((wsum[0][c] + wsum[1][c]) + (wsum[2][c] + wsum[3][c])) /
                                           static_cast<double>(N));
}

// score_j = qbar . k_j / 8 (fp64 dot, fp32 result); special keys get -inf so they are never ranked.
// Each block takes a contiguous range of key rows.  Eight lanes per key row, each with one 16-byte
// chunk (a warp reads 4 whole rows, 512 contiguous bytes, per load), kProbeRowsInFlight rows per
// lane group and step, the next step's requested before this step's are used; the 8 partial dots
// of a row meet in 3 shuffles.  All lanes
// of a warp take the same iterations (row validity is a per-group guard), so every shuffle has
// its whole warp.
__global__ void __launch_bounds__(256) probe_score_kernel(const uint16_t* __restrict__ k, int N, int V, int ns,
                                                          ProbeArgs a, const float* __restrict__ qbar,
                                                          float* __restrict__ scores) {
  const int hp = blockIdx.y;
  const int h = a.heads[hp];
  const int sub = threadIdx.x & 7, grp = threadIdx.x >> 3;  // 32 row groups per block
  double qv[8];  // this lane's 8 features of qbar, scaled by 2^896 against the 2^-896 of the keys
#pragma unroll
  for (int i = 0; i < 8; ++i) qv[i] = static_cast<double>(qbar[hp * kD + 8 * sub + i]) * kUnscale896;
  const uint4* kh = reinterpret_cast<const uint4*>(k + static_cast<size_t>(h) * N * kD);
  float* sc = scores + static_cast<size_t>(hp) * N;
  const int rows_per = (N + gridDim.x - 1) / gridDim.x;
  const int r0 = blockIdx.x * rows_per, r1 = min(N, r0 + rows_per);
  constexpr int kStep = 32 * kProbeRowsInFlight;
  uint4 w[kProbeRowsInFlight];
#pragma unroll
  for (int f = 0; f < kProbeRowsInFlight; ++f) {
    const int jf = r0 + 32 * f + grp;  // uniform over the 8 lanes of a row group
    w[f] = jf < r1 ? kh[static_cast<size_t>(jf) * 8 + sub] : make_uint4(0u, 0u, 0u, 0u);
  }
  for (int jb = r0; jb < r1; jb += kStep) {
    uint4 nx[kProbeRowsInFlight];  // the next step's rows, requested before this step's are used
#pragma unroll
    for (int f = 0; f < kProbeRowsInFlight; ++f) {
      const int jf = jb + kStep + 32 * f + grp;
      nx[f] = jf < r1 ? kh[static_cast<size_t>(jf) * 8 + sub] : make_uint4(0u, 0u, 0u, 0u);
    }
    double d[kProbeRowsInFlight];
#pragma unroll
    for (int f = 0; f < kProbeRowsInFlight; ++f) {
      double x[8];
      bf16x8_to_f64(w[f], x);
      d[f] = 0.0;
#pragma unroll
      for (int i = 0; i < 8; ++i) d[f] = fma(qv[i], x[i], d[f]);
    }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1)
#pragma unroll
      for (int f = 0; f < kProbeRowsInFlight; ++f) d[f] += __shfl_xor_sync(0xffffffffu, d[f], o);
    if (sub == 0) {
#pragma unroll
      for (int f = 0; f < kProbeRowsInFlight; ++f) {
        const int jf = jb + 32 * f + grp;
        if (jf < r1) sc[jf] = (jf % V) < ns ? -INFINITY : static_cast<float>(d[f] * 0.125);
      }
    }
#pragma unroll
    for (int f = 0; f < kProbeRowsInFlight; ++f) w[f] = nx[f];
  }
}

// ---- probe Top-K: a radix select spread over many blocks per head.
//
// The k-th largest order key is found one digit at a time (bits 31..21, 20..10, 9..0): every block
// histograms the digit of the keys that match the digits chosen so far, adds its histogram into
// the head's global one, and the last block to finish (a counter, no waiting) picks the digit
// holding the k-th key and how many keys of equal prefix are still to be taken.  Then every block
// counts, in its own contiguous chunk of keys, those above the final key and those equal to it,
// and writes its selected indices in ascending order at the offset the counts of the chunks
// before it give: all keys above the k-th, and the lowest-index keys equal to it.
constexpr int kRankBins = 2048;   // 11-bit digits
constexpr int kRankChunk = 4096;  // keys per block (256 threads x 16)
constexpr int kRankPasses = 3;

struct RankState {
  uint32_t prefix;  // digits chosen so far
  uint32_t mask;    // bits they cover
  int remaining;    // keys still to take among those matching prefix under mask
  int pad;
};

__host__ __device__ constexpr int rank_shift(int pass) { return pass == 0 ? 21 : (pass == 1 ? 10 : 0); }
__host__ __device__ constexpr uint32_t rank_digit_mask(int pass) { return pass == 2 ? 0x3FFu : 0x7FFu; }

// Exclusive scan of one int per thread over a block of kWarps warps; `total` gets the sum.
template <int kWarps>
__device__ __forceinline__ int block_exclusive_scan(int v, int* tmp /*[kWarps]*/, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kWarps ? tmp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kWarps) tmp[lane] = w;
  }
  __syncthreads();
  total = tmp[kWarps - 1];
  const int before = warp > 0 ? tmp[warp - 1] : 0;
  __syncthreads();
  return before + x - v;
}

// One digit pass over all keys of every probe head (grid: blocks per head x probe heads).
// hist [n_probe][kRankPasses][kRankBins] and done [n_probe][kRankPasses] start at zero.
__global__ void __launch_bounds__(256) probe_digit_kernel(const float* __restrict__ scores, int N, ProbeArgs a,
                                                          int pass, int* __restrict__ hist,
                                                          unsigned* __restrict__ done, RankState* __restrict__ st) {
  const int hp = blockIdx.y;
  const float* sc = scores + static_cast<size_t>(hp) * N;
  __shared__ int h[kRankBins];
  __shared__ int tmp[8];
  __shared__ bool last;
  for (int i = threadIdx.x; i < kRankBins; i += blockDim.x) h[i] = 0;
  uint32_t prefix = 0, mask = 0;
  int remaining = a.k[hp];
  if (pass > 0) {
    const RankState r = st[hp];  // written by the previous pass's launch
    prefix = r.prefix;
    mask = r.mask;
    remaining = r.remaining;
  }
  const int shift = rank_shift(pass);
  const uint32_t dmask = rank_digit_mask(pass);
  __syncthreads();
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < N; j += gridDim.x * blockDim.x) {
    const uint32_t key = order_key(sc[j]);
    if ((key & mask) == prefix) atomicAdd(&h[(key >> shift) & dmask], 1);
  }
  __syncthreads();
  int* gh = hist + (static_cast<size_t>(hp) * kRankPasses + pass) * kRankBins;
  for (int i = threadIdx.x; i < kRankBins; i += blockDim.x)
    if (h[i] != 0) atomicAdd(&gh[i], h[i]);
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = atomicAdd(&done[hp * kRankPasses + pass], 1u) == gridDim.x - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  // the last block: thread t holds bins 2047-8t .. 2040-8t (descending), so a scan in thread
  // order counts the keys above each bin
  constexpr int kPer = kRankBins / 256;
  int c[kPer], local = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    c[i] = __ldcg(&gh[kRankBins - 1 - kPer * threadIdx.x - i]);
    local += c[i];
  }
  int total;
  int above = block_exclusive_scan<8>(local, tmp, total);
  const bool lowest = threadIdx.x == blockDim.x - 1;
  if (above < remaining && (above + local >= remaining || lowest)) {
    int bin = kRankBins - 1 - kPer * threadIdx.x;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      bin = kRankBins - 1 - kPer * static_cast<int>(threadIdx.x) - i;
      if (above + c[i] >= remaining || bin == 0) break;
      above += c[i];
    }
    RankState r;
    r.prefix = prefix | (static_cast<uint32_t>(bin) << shift);
    r.mask = mask | (dmask << shift);
    r.remaining = remaining - above;
    r.pad = 0;
    st[hp] = r;
  }
}

// Keys above the k-th key and keys equal to it in each block's chunk: counts [n_probe][blocks][2].
__global__ void __launch_bounds__(256) probe_count_kernel(const float* __restrict__ scores, int N,
                                                          const RankState* __restrict__ st,
                                                          int* __restrict__ counts) {
  const int hp = blockIdx.y;
  const float* sc = scores + static_cast<size_t>(hp) * N;
  const uint32_t kth = st[hp].prefix;
  const int j0 = blockIdx.x * kRankChunk, j1 = min(N, j0 + kRankChunk);
  int gt = 0, eq = 0;
  for (int j = j0 + threadIdx.x; j < j1; j += blockDim.x) {
    const uint32_t key = order_key(sc[j]);
    gt += key > kth;
    eq += key == kth;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    gt += __shfl_xor_sync(0xffffffffu, gt, o);
    eq += __shfl_xor_sync(0xffffffffu, eq, o);
  }
  __shared__ int wg[8], we[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    wg[warp] = gt;
    we[warp] = eq;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int tg = 0, te = 0;
    for (int w = 0; w < 8; ++w) {
      tg += wg[w];
      te += we[w];
    }
    counts[(static_cast<size_t>(hp) * gridDim.x + blockIdx.x) * 2] = tg;
    counts[(static_cast<size_t>(hp) * gridDim.x + blockIdx.x) * 2 + 1] = te;
  }
}

// The selected indices of each block's chunk, ascending, at the offset of the chunks before it.
__global__ void __launch_bounds__(256) probe_write_kernel(const float* __restrict__ scores, int N, ProbeArgs a,
                                                          const RankState* __restrict__ st,
                                                          const int* __restrict__ counts,
                                                          int32_t* __restrict__ cache) {
  const int hp = blockIdx.y;
  const float* sc = scores + static_cast<size_t>(hp) * N;
  const uint32_t kth = st[hp].prefix;
  const int remaining = st[hp].remaining;
  __shared__ int tmp[8];
  // keys above / equal in the chunks before this one
  int gb = 0, eb = 0;
  for (int b = threadIdx.x; b < static_cast<int>(blockIdx.x); b += blockDim.x) {
    gb += counts[(static_cast<size_t>(hp) * gridDim.x + b) * 2];
    eb += counts[(static_cast<size_t>(hp) * gridDim.x + b) * 2 + 1];
  }
  int gt_before, eq_before;
  block_exclusive_scan<8>(gb, tmp, gt_before);
  block_exclusive_scan<8>(eb, tmp, eq_before);
  const int eq_chunk = max(0, remaining - eq_before);  // equal keys this chunk may still take
  int32_t* out = cache + a.cache_off[hp] + gt_before + min(eq_before, remaining);
  // each thread a contiguous run of the chunk, so the scans keep index order
  constexpr int kRun = kRankChunk / 256;
  const int j0 = blockIdx.x * kRankChunk + threadIdx.x * kRun, j1 = min(N, j0 + kRun);
  uint32_t keys[kRun];
  int n_gt = 0, n_eq = 0;
#pragma unroll
  for (int i = 0; i < kRun; ++i) {
    keys[i] = j0 + i < j1 ? order_key(sc[j0 + i]) : 0u;
    n_gt += j0 + i < j1 && keys[i] > kth;
    n_eq += j0 + i < j1 && keys[i] == kth;
  }
  int tot;
  const int eq_mine_before = block_exclusive_scan<8>(n_eq, tmp, tot);
  const int eq_take = max(0, min(n_eq, eq_chunk - eq_mine_before));
  int pos = block_exclusive_scan<8>(n_gt + eq_take, tmp, tot);
  int eq_seen = 0;
#pragma unroll
  for (int i = 0; i < kRun; ++i) {
    if (j0 + i >= j1) break;
    bool take = keys[i] > kth;
    if (keys[i] == kth) {
      take = eq_seen < eq_take;
      ++eq_seen;
    }
    if (take) out[pos++] = j0 + i;
  }
}

// Mean of L2-normalised DINO features over the patch tokens of each 64-token tile,
// then normalised to unit length (its cosine against other tiles is a plain dot).
// kChunks 16-byte chunks of a feature row per lane: dim <= 128 * kChunks.
template <int kChunks>
__global__ void __launch_bounds__(128) dino_pool_kernel(const float* __restrict__ dino, int N, int V, int ns,
                                                        int P, int dim, float* __restrict__ tilevec,
                                                        __half* __restrict__ tile16, int dim16) {
  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  extern __shared__ float pool_smem[];  // [4][dim] per-warp sums, then [dim] mean
  float* wsum = pool_smem;
  for (int i = threadIdx.x; i < 4 * dim; i += blockDim.x) wsum[i] = 0.f;
  __syncthreads();
  int count = 0;
  const int tok0 = t * kTile, tok1 = min(N, tok0 + kTile);
  const int nc = dim >> 2;  // 16-byte chunks per feature row (dim is a multiple of 4)
  // four token rows per warp in flight: each lane loads its chunks of all four, then the four
  // norms are reduced together and the normalised rows added to the warp's sums
  constexpr int kRows = 4;
  for (int tb = tok0 + warp * kRows; tb < tok1; tb += 4 * kRows) {
    float4 x[kRows][kChunks];
    float ss[kRows];
    bool patch[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int tok = tb + r;
      const int s = tok / V, loc = tok - s * V;
      patch[r] = tok < tok1 && loc >= ns;
      const float4* f = reinterpret_cast<const float4*>(dino + (static_cast<size_t>(s) * P + (loc - ns)) * dim);
      ss[r] = 0.f;
#pragma unroll
      for (int c = 0; c < kChunks; ++c) {
        const int i = 32 * c + lane;
        x[r][c] = (patch[r] && i < nc) ? f[i] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int r = 0; r < kRows; ++r)
#pragma unroll
      for (int c = 0; c < kChunks; ++c)
        ss[r] = fmaf(x[r][c].x, x[r][c].x,
                     fmaf(x[r][c].y, x[r][c].y, fmaf(x[r][c].z, x[r][c].z, fmaf(x[r][c].w, x[r][c].w, ss[r]))));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int r = 0; r < kRows; ++r) ss[r] += __shfl_xor_sync(0xffffffffu, ss[r], o);
    float4* w4 = reinterpret_cast<float4*>(wsum + warp * dim);
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
      const int i = 32 * c + lane;
      if (i < nc) {
        float4 acc = w4[i];
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          // a special token or a token past the tile contributes nothing
          const float inv = patch[r] ? 1.f / sqrtf(ss[r]) : 0.f;
          acc.x += x[r][c].x * inv;
          acc.y += x[r][c].y * inv;
          acc.z += x[r][c].z * inv;
          acc.w += x[r][c].w * inv;
        }
        w4[i] = acc;
      }
    }
  }
  for (int tok = tok0; tok < tok1; ++tok) count += ((tok % V) >= ns);
  __syncthreads();
  float* mean = pool_smem + 4 * dim;
  for (int c = threadIdx.x; c < dim; c += blockDim.x)
    mean[c] = (wsum[c] + wsum[dim + c] + wsum[2 * dim + c] + wsum[3 * dim + c]) / static_cast<float>(count);
  __syncthreads();
  __shared__ float red[4];
  float ss = 0.f;
  for (int c = threadIdx.x; c < dim; c += blockDim.x) ss = fmaf(mean[c], mean[c], ss);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) red[warp] = ss;
  __syncthreads();
  const float inv = 1.f / sqrtf(red[0] + red[1] + red[2] + red[3]);
  for (int c = threadIdx.x; c < dim; c += blockDim.x) tilevec[static_cast<size_t>(t) * dim + c] = mean[c] * inv;
  if (tile16 != nullptr) {
    // the same unit vector rounded to fp16, zero-padded to dim16 features (tensor-core operand)
    for (int c = threadIdx.x; c < dim16; c += blockDim.x)
      tile16[static_cast<size_t>(t) * dim16 + c] = __float2half_rn(c < dim ? mean[c] * inv : 0.f);
  }
}

// Inverse of order_key.
__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// From a 256-bin histogram wh of one digit: the bin holding the remaining-th largest key (bins
// counted from the top), with `remaining` reduced by the keys of the bins above it.  Lane l sums
// bins 255 - 8l .. 248 - 8l, a warp scan finds the lane whose bins cross, and that lane walks its
// eight.  Without a crossing (fewer keys than remaining) the answer is bin 0.
__device__ __forceinline__ int warp_pick_bin(const int* wh, int lane, int& remaining) {
  int c[8], local = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    c[i] = wh[255 - 8 * lane - i];
    local += c[i];
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const int above = incl - local;
  const uint32_t hit = __ballot_sync(0xffffffffu, above < remaining && incl >= remaining);
  int bin = 0, sub = 0;
  if (hit == 0) {
    sub = __shfl_sync(0xffffffffu, incl, 31) - wh[0];
  } else {
    const int src = __ffs(hit) - 1;
    if (lane == src) {
      int a = above;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        bin = 255 - 8 * lane - i;
        if (a + c[i] >= remaining) break;
        a += c[i];
      }
      sub = a;
    }
    bin = __shfl_sync(0xffffffffu, bin, src);
    sub = __shfl_sync(0xffffffffu, sub, src);
  }
  remaining -= sub;
  return bin;
}

// The warp's 8-bit-digit radix select over row[0..T): the key of the kmax-th largest value
// and how many keys equal to it are taken.  Histogram counts are aggregated per warp
// instruction (lanes that share a bin add once), so a narrow range of cosines, whose keys
// share their high digits, does not serialise 32 lanes on one shared-memory counter.
__device__ __forceinline__ void warp_radix_kth(const float* row, int T, int kmax, int* wh, int lane,
                                               uint32_t& prefix, int& remaining) {
  prefix = 0;
  uint32_t mask = 0;
  remaining = kmax;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = lane; i < 256; i += 32) wh[i] = 0;
    __syncwarp();
    for (int v0 = 0; v0 < T; v0 += 32) {
      const int v = v0 + lane;
      uint32_t key = 0;
      bool in = false;
      if (v < T) {
        key = order_key(row[v]);
        in = (key & mask) == prefix;
      }
      const uint32_t act = __ballot_sync(0xffffffffu, in);
      if (in) {
        const uint32_t bin = (key >> shift) & 0xFFu;
        const uint32_t peers = __match_any_sync(act, bin);
        if (lane == __ffs(peers) - 1) atomicAdd(&wh[bin], __popc(peers));
      }
    }
    __syncwarp();
    prefix |= static_cast<uint32_t>(warp_pick_bin(wh, lane, remaining)) << shift;
    mask |= 0xFFu << shift;
    __syncwarp();
  }
}

// Order-preserving 16-bit key of an fp16 value (larger value -> larger key) and its inverse.
__device__ __forceinline__ uint32_t order_key16(uint32_t h) { return (h & 0x8000u) ? (~h & 0xFFFFu) : (h | 0x8000u); }
__device__ __forceinline__ float key16_value(uint32_t key) {
  const uint32_t h = (key & 0x8000u) ? (key & 0x7FFFu) : (~key & 0xFFFFu);
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h)));
}

// The kmax largest values of row[0..T) (ties to the lower index) written to out[0..kmax) in
// rank order (value descending, then index ascending), as indices into row, or as map[index]
// when a map is given.  One warp.
__device__ __forceinline__ void warp_rank_row(const float* row, int T, int kmax, int* wh, int* widx, uint32_t* wkey,
                                              int lane, int32_t* __restrict__ out, const int* map = nullptr) {
  uint32_t prefix;
  int remaining;
  warp_radix_kth(row, T, kmax, wh, lane, prefix, remaining);
  // gather the selected tiles in index order (lane-strided chunks keep the order)
  int base = 0, eq_used = 0;
  for (int v0 = 0; v0 < T; v0 += 32) {
    const int v = v0 + lane;
    uint32_t key = 0;
    bool gt = false, eq = false;
    if (v < T) {
      key = order_key(row[v]);
      gt = key > prefix;
      eq = key == prefix;
    }
    const uint32_t eq_mask = __ballot_sync(0xffffffffu, eq);
    const int eq_rank = eq_used + __popc(eq_mask & ((1u << lane) - 1u));
    const bool take = gt || (eq && eq_rank < remaining);
    const uint32_t take_mask = __ballot_sync(0xffffffffu, take);
    if (take) {
      const int pos = base + __popc(take_mask & ((1u << lane) - 1u));
      widx[pos] = v;
      wkey[pos] = key;
    }
    base += __popc(take_mask);
    eq_used += __popc(eq_mask);
  }
  __syncwarp();
  // rank order: by key descending, then tile index ascending
  for (int i = lane; i < kmax; i += 32) {
    const uint32_t ki = wkey[i];
    const int vi = widx[i];
    int rank = 0;
    for (int j = 0; j < kmax; ++j) {
      const uint32_t kj = wkey[j];
      rank += (kj > ki) || (kj == ki && widx[j] < vi);
    }
    out[rank] = map != nullptr ? map[vi] : vi;
  }
  __syncwarp();
}

// Cosines of R query tiles against all T tiles (fp64 dots of unit vectors, rounded to
// fp32), then per query tile the kmax best tiles in rank order.  General form, any dim.
__global__ void __launch_bounds__(256) tile_topk_kernel(const float* __restrict__ tilevec, int T, int dim, int R,
                                                        int kmax, int32_t* __restrict__ ranked) {
  extern __shared__ uint8_t tk_smem[];
  float* qv = reinterpret_cast<float*>(tk_smem);     // [R][dim]
  float* cs = qv + R * dim;                           // [R][T]
  int* hist = reinterpret_cast<int*>(cs + static_cast<size_t>(R) * T);  // [8 warps][256]
  int* sel_idx = hist + 8 * 256;                      // [8 warps][kmax]
  uint32_t* sel_key = reinterpret_cast<uint32_t*>(sel_idx + 8 * kmax);  // [8 warps][kmax]
  const int u0 = blockIdx.x * R;
  const int nr = min(R, T - u0);
  for (int i = threadIdx.x; i < nr * dim; i += blockDim.x) qv[i] = tilevec[static_cast<size_t>(u0) * dim + i];
  __syncthreads();
  for (int v = threadIdx.x; v < T; v += blockDim.x) {
    const float* fv = tilevec + static_cast<size_t>(v) * dim;
    double acc[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) acc[r] = 0.0;
    for (int c = 0; c < dim; c += 4) {
      const float4 b = *reinterpret_cast<const float4*>(fv + c);
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        if (r < nr) {
          const float* a = qv + r * dim + c;
          acc[r] = fma(static_cast<double>(a[0]), static_cast<double>(b.x), acc[r]);
          acc[r] = fma(static_cast<double>(a[1]), static_cast<double>(b.y), acc[r]);
          acc[r] = fma(static_cast<double>(a[2]), static_cast<double>(b.z), acc[r]);
          acc[r] = fma(static_cast<double>(a[3]), static_cast<double>(b.w), acc[r]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < 16; ++r)
      if (r < nr) cs[static_cast<size_t>(r) * T + v] = static_cast<float>(acc[r]);
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int r = warp; r < nr; r += 8)
    warp_rank_row(cs + static_cast<size_t>(r) * T, T, kmax, hist + warp * 256, sel_idx + warp * kmax,
                  sel_key + warp * kmax, lane, ranked + static_cast<size_t>(u0 + r) * kmax);
}

// Lane slices of the exact fp64 dots: kTkChunks float4 chunks of 128 features (dim <= 384).
constexpr int kTkChunks = 3;

__device__ __forceinline__ float4 ld_f4(const float* p) { return *reinterpret_cast<const float4*>(p); }

// ---- token-wise DINO Top-K (section 4.1, "DINO Top-K Kernel": per query token, the Top-K most
// similar tokens of every frame; section 5.1: K per frame)
//
// Three steps: unit features (fp32, and an fp16 copy zero-padded to a multiple of 64 features);
// the fp16 cosines of a chunk of query rows against all patch tokens on the tensor cores
// (token_sim.cu, within kTokScoreErr of the exact cosine); and, per query row and frame, the
// ranking below, which recomputes exactly (fp64 dot, rounded to fp32) every candidate the
// bound cannot rule out.

// Unit DINO features, one warp per patch token: fp64 sum of squares, one scale in fp32.
__global__ void __launch_bounds__(256) unit_features_kernel(const float* __restrict__ dino, int rows, int dim,
                                                            float* __restrict__ unit, __half* __restrict__ unit16,
                                                            int dim16) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= rows) return;
  const float* f = dino + static_cast<size_t>(warp) * dim;
  double ss = 0.0;
  for (int c = lane; c < dim; c += 32) ss += static_cast<double>(f[c]) * f[c];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = ss > 0.0 ? static_cast<float>(1.0 / sqrt(ss)) : 0.f;
  for (int c = lane; c < dim16; c += 32) {
    const float u = c < dim ? f[c] * inv : 0.f;
    if (c < dim) unit[static_cast<size_t>(warp) * dim + c] = u;
    unit16[static_cast<size_t>(warp) * dim16 + c] = __float2half_rn(u);
  }
}

constexpr float kTokScoreErr = 2e-3f;  // |tensor-core fp16 score - exact cosine| (bound in token_sim.cu)
constexpr int kTokCap = 64;            // candidates of one (query, frame) the short ranking takes

// This lane's slice of unit vector `row` (features 128c + 4 lane .. +3, as q[4c] .. q[4c + 3]) in
// fp64, pre-multiplied by 2^896 for products with f32_scaled candidates; 0 past dim.
__device__ __forceinline__ void load_one_slice(const float* __restrict__ vec, int row, int dim, int lane,
                                               double (&q)[4 * kTkChunks]) {
#pragma unroll
  for (int c = 0; c < kTkChunks; ++c) {
    const int d = 128 * c + 4 * lane;
    const float4 f = d < dim ? ld_f4(vec + static_cast<size_t>(row) * dim + d) : make_float4(0.f, 0.f, 0.f, 0.f);
    q[4 * c] = static_cast<double>(f.x) * kUnscale896;
    q[4 * c + 1] = static_cast<double>(f.y) * kUnscale896;
    q[4 * c + 2] = static_cast<double>(f.z) * kUnscale896;
    q[4 * c + 3] = static_cast<double>(f.w) * kUnscale896;
  }
}

// fp64 dot of the lane slices q with candidate row fv, summed over the warp (every lane gets
// the same value: a butterfly adds the same two operands on both sides of each exchange).
__device__ __forceinline__ double exact_dot(const double (&q)[4 * kTkChunks], const float* __restrict__ fv, int dim,
                                           int lane) {
  double acc = 0.0;
#pragma unroll
  for (int c = 0; c < kTkChunks; ++c) {
    const int d = 128 * c + 4 * lane;
    if (d < dim) {
      const float4 b = ld_f4(fv + d);
      acc = fma(q[4 * c], f32_scaled(b.x), acc);
      acc = fma(q[4 * c + 1], f32_scaled(b.y), acc);
      acc = fma(q[4 * c + 2], f32_scaled(b.z), acc);
      acc = fma(q[4 * c + 3], f32_scaled(b.w), acc);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return acc;
}

struct TokWarpSmem {
  float* row;       // [P] approximate scores (general ranking)
  int* hist;        // [256]
  int* widx;        // [kmax]
  uint32_t* wkey;   // [kmax]
  int* cidx;        // [kTokCap] candidate patch indices (ascending)
  float* cval;      // [kTokCap] their approximate scores
  uint32_t* ckey;   // [kTokCap] order keys of their exact scores
};

// General ranking of one (query, frame): every candidate within 2 * kTokScoreErr of the
// approximate kmax-th score gets its exact value, then the whole frame is ranked.
__device__ void token_rank_general(const __half* __restrict__ seg, int P, int kmax, const double (&q)[4 * kTkChunks],
                                   const float* __restrict__ cand, int dim, const TokWarpSmem& w, int lane,
                                   int32_t* __restrict__ out) {
  for (int v = lane; v < P; v += 32) w.row[v] = __half2float(seg[v]);
  __syncwarp();
  uint32_t prefix;
  int remaining;
  warp_radix_kth(w.row, P, kmax, w.hist, lane, prefix, remaining);
  const float thr = key_value(prefix) - 2.f * kTokScoreErr;
  for (int v0 = 0; v0 < P; v0 += 32) {
    const int v = v0 + lane;
    uint32_t todo = __ballot_sync(0xffffffffu, v < P && w.row[v] >= thr);
    while (todo) {
      const int bit = __ffs(todo) - 1;
      todo &= todo - 1;
      const double e = exact_dot(q, cand + static_cast<size_t>(v0 + bit) * dim, dim, lane);
      if (lane == 0) w.row[v0 + bit] = static_cast<float>(e);
    }
  }
  __syncwarp();
  warp_rank_row(w.row, P, kmax, w.hist, w.widx, w.wkey, lane, out);
}

// Two fp64 dots at once (both rows' loads in flight together); see exact_dot.
__device__ __forceinline__ void exact_dot2(const double (&q)[4 * kTkChunks], const float* __restrict__ f1,
                                           const float* __restrict__ f2, int dim, int lane, double& e1, double& e2) {
  float4 b1[kTkChunks], b2[kTkChunks];
#pragma unroll
  for (int c = 0; c < kTkChunks; ++c) {
    const int d = 128 * c + 4 * lane;
    b1[c] = d < dim ? ld_f4(f1 + d) : make_float4(0.f, 0.f, 0.f, 0.f);
    b2[c] = d < dim ? ld_f4(f2 + d) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  double a1 = 0.0, a2 = 0.0;
#pragma unroll
  for (int c = 0; c < kTkChunks; ++c) {
    const double qx = q[4 * c], qy = q[4 * c + 1], qz = q[4 * c + 2], qw = q[4 * c + 3];
    a1 = fma(qx, f32_scaled(b1[c].x), a1);
    a2 = fma(qx, f32_scaled(b2[c].x), a2);
    a1 = fma(qy, f32_scaled(b1[c].y), a1);
    a2 = fma(qy, f32_scaled(b2[c].y), a2);
    a1 = fma(qz, f32_scaled(b1[c].z), a1);
    a2 = fma(qz, f32_scaled(b2[c].z), a2);
    a1 = fma(qw, f32_scaled(b1[c].w), a1);
    a2 = fma(qw, f32_scaled(b2[c].w), a2);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a1 += __shfl_xor_sync(0xffffffffu, a1, o);
    a2 += __shfl_xor_sync(0xffffffffu, a2, o);
  }
  e1 = a1;
  e2 = a2;
}

// The 8 scores of 16-byte chunk c of a score row (fp32) and which of them lie in the frame
// [e0, e0 + P) (bit j for score j; all 8 for a chunk inside the frame).
__device__ __forceinline__ uint32_t chunk_scores(const uint4 w, int c, int e0, int P, float (&v)[8]) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[i]));
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
  const int j0 = 8 * c - e0;  // frame index of v[0]
  uint32_t valid = 0xFFu;
  if (j0 < 0 || j0 + 8 > P) {
    valid = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const bool in = j0 + j >= 0 && j0 + j < P;
      valid |= static_cast<uint32_t>(in) << j;
      if (!in) v[j] = -INFINITY;
    }
  }
  return valid;
}

// Ranking of one (query, frame) from its approximate scores: frame s occupies elements
// [e0, e0 + P) of the score row srow (16-byte aligned).
//
// With a = approximate score, e = exact score, |a - e| <= b = kTokScoreErr, A_k = the kmax-th
// largest a and E_k the kmax-th largest e: A_k <= E_k + b (of the kmax largest a, one at least
// has e <= E_k), so every key of the exact Top-kmax has a >= E_k - b >= A_k - 2b, and every key
// with a < A_k - 2b has e < E_k.  The kmax-th largest of the 32 lane maxima t0 is <= A_k, so
// D = {a >= t0 - 2b} holds every such key; when D fits kTokCap the short path finds A_k inside D,
// recomputes C = {a >= A_k - 2b} exactly and ranks C (exact value descending, index ascending),
// which is the frame's exact ranking.  Otherwise (kmax > 32, or more than kTokCap keys in D)
// the general ranking runs.
__device__ void token_rank_frame(const __half* __restrict__ srow, int e0, int P, int kmax,
                                 const double (&q)[4 * kTkChunks], const float* __restrict__ cand, int dim,
                                 const TokWarpSmem& w, int lane, int32_t* __restrict__ out) {
  const float band = 2.f * kTokScoreErr;
  const uint4* row4 = reinterpret_cast<const uint4*>(srow);
  const int cb = e0 >> 3, ce = (e0 + P + 7) >> 3;
  bool general = kmax > 32;
  int n = 0;
  if (!general) {
    float m = -INFINITY;
    for (int c = cb + lane; c < ce; c += 32) {
      float v[8];
      chunk_scores(__ldg(row4 + c), c, e0, P, v);
      m = fmaxf(m, fmaxf(fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3])), fmaxf(fmaxf(v[4], v[5]), fmaxf(v[6], v[7]))));
    }
    // bitonic sort of the 32 lane maxima, descending: lane kmax-1 then holds the kmax-th largest
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1)
#pragma unroll
      for (int j = k >> 1; j > 0; j >>= 1) {
        const float y = __shfl_xor_sync(0xffffffffu, m, j);
        m = (((lane & j) == 0) == ((lane & k) == 0)) ? fmaxf(m, y) : fminf(m, y);
      }
    const float thr = __shfl_sync(0xffffffffu, m, kmax - 1) - band;  // -inf when fewer keys than lanes hold
    for (int c0 = cb; c0 < ce; c0 += 32) {
      const int c = c0 + lane;
      float v[8];
      uint32_t bits = 0;
      if (c < ce) {
        const uint32_t valid = chunk_scores(__ldg(row4 + c), c, e0, P, v);
#pragma unroll
        for (int j = 0; j < 8; ++j) bits |= static_cast<uint32_t>(v[j] >= thr) << j;
        bits &= valid;
      }
      const int cnt = __popc(bits);
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      int pos = n + incl - cnt;
      if (bits) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if ((bits >> j) & 1u) {
            if (pos < kTokCap) {
              w.cidx[pos] = 8 * c + j - e0;
              w.cval[pos] = v[j];
            }
            ++pos;
          }
      }
      n += __shfl_sync(0xffffffffu, incl, 31);
    }
    general = n > kTokCap || n < kmax;
  }
  if (general) {
    __syncwarp();
    token_rank_general(srow + e0, P, kmax, q, cand, dim, w, lane, out);
    return;
  }
  __syncwarp();
  // A_k: the kmax-th largest approximate score of D (ties by position)
  float ak = 0.f;
  {
    bool hit = false;
    float hv = 0.f;
    for (int i = lane; i < n; i += 32) {
      const float ai = w.cval[i];
      int r = 0;
      for (int j = 0; j < n; ++j) {
        const float aj = w.cval[j];
        r += (aj > ai) || (aj == ai && j < i);
      }
      if (r == kmax - 1) {
        hit = true;
        hv = ai;
      }
    }
    const int src = __ffs(__ballot_sync(0xffffffffu, hit)) - 1;
    ak = __shfl_sync(0xffffffffu, hv, src);
  }
  const float cthr = ak - band;
  // A key of C whose approximate score is more than `band` away from every other key of C has
  // the same order against each of them by exact value (|a - e| <= b on both sides), so only the
  // keys with a neighbour within `band` (ambiguous) need their exact value; ckey = 0 (no real
  // value has that order key) marks the others, which the ranking then orders by a.
  bool amb[2] = {false, false};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int i = lane + 32 * h;
    if (i < n) {
      const float ai = w.cval[i];
      if (ai >= cthr)
        for (int j = 0; j < n; ++j) {
          const float aj = w.cval[j];
          amb[h] |= j != i && aj >= cthr && fabsf(aj - ai) <= band;
        }
      w.ckey[i] = 0u;
    }
  }
  __syncwarp();
  // exact values of the ambiguous keys, two at a time
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int i0 = 32 * h;
    uint32_t todo = __ballot_sync(0xffffffffu, amb[h]);
    while (todo) {
      const int b1 = __ffs(todo) - 1;
      todo &= todo - 1;
      const int b2 = todo ? __ffs(todo) - 1 : b1;
      if (todo) todo &= todo - 1;
      double e1, e2;
      exact_dot2(q, cand + static_cast<size_t>(w.cidx[i0 + b1]) * dim, cand + static_cast<size_t>(w.cidx[i0 + b2]) * dim,
                 dim, lane, e1, e2);
      if (lane == 0) {
        w.ckey[i0 + b1] = order_key(static_cast<float>(e1));
        if (b2 != b1) w.ckey[i0 + b2] = order_key(static_cast<float>(e2));
      }
    }
  }
  __syncwarp();
  // rank C: exact value descending, then patch index ascending
  for (int i = lane; i < n; i += 32) {
    const float ai = w.cval[i];
    if (ai < cthr) continue;
    const uint32_t ki = w.ckey[i];
    const int vi = w.cidx[i];
    int r = 0;
    for (int j = 0; j < n; ++j) {
      const float aj = w.cval[j];
      if (aj < cthr || j == i) continue;
      const uint32_t kj = w.ckey[j];
      r += (ki != 0u && kj != 0u) ? ((kj > ki) || (kj == ki && w.cidx[j] < vi)) : (aj > ai);
    }
    if (r < kmax) out[r] = vi;
  }
  __syncwarp();
}

// One warp per query row of the chunk; frames in turn.  lists[(a * S + s) * kmax + rank] =
// patch index of rank `rank` in frame s for feature row a = r0 + row.
__global__ void __launch_bounds__(256, 3) token_rank_kernel(const __half* __restrict__ scores, long long ld, int r0,
                                                         int rows, const float* __restrict__ unit, int S, int P,
                                                         int dim, int kmax, int32_t* __restrict__ lists) {
  extern __shared__ uint8_t tr_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  TokWarpSmem w;
  {
    float* rows_f = reinterpret_cast<float*>(tr_smem);
    int* hist = reinterpret_cast<int*>(rows_f + static_cast<size_t>(8) * P);
    int* cidx = hist + 8 * 256;
    float* cval = reinterpret_cast<float*>(cidx + 8 * kTokCap);
    uint32_t* ckey = reinterpret_cast<uint32_t*>(cval + 8 * kTokCap);
    int* widx = reinterpret_cast<int*>(ckey + 8 * kTokCap);
    uint32_t* wkey = reinterpret_cast<uint32_t*>(widx + 8 * kmax);
    w.row = rows_f + static_cast<size_t>(warp) * P;
    w.hist = hist + warp * 256;
    w.cidx = cidx + warp * kTokCap;
    w.cval = cval + warp * kTokCap;
    w.ckey = ckey + warp * kTokCap;
    w.widx = widx + warp * kmax;
    w.wkey = wkey + warp * kmax;
  }
  const int row = blockIdx.x * 8 + warp;
  if (row >= rows) return;
  const int a = r0 + row;
  double q[4 * kTkChunks];
  load_one_slice(unit, a, dim, lane, q);
  const __half* srow = scores + static_cast<size_t>(row) * ld;
  for (int s = 0; s < S; ++s)
    token_rank_frame(srow, s * P, P, kmax, q, unit + static_cast<size_t>(s) * P * dim, dim, w, lane,
                     lists + (static_cast<size_t>(a) * S + s) * kmax);
}

// ---- query-tile grouping of the correspondence heads (a scheduling aid, cached with the indices)
//
// Four query tiles share one 256-row attention work item and the union of their key
// tiles.  Tiles whose ranked lists overlap are put together: sort by a canonical key
// (the smallest tile index among the first `r` ranks), then, inside windows of 64
// consecutive tiles, greedily grow groups of four by shared-tile counts.  The order
// changes only which rows share an item, never a result.
constexpr int kGroupWindow = 64;
constexpr int kMaxSortTiles = 16384;

// ---- block-wise DINO Top-K ranking (section 4.3, "DINO Top-K Kernel", block-wise variant)
//
// The cosines of a chunk of query tiles against all T tiles come from the tensor cores (the tile
// unit vectors rounded to fp16, token_sim.cu: within kTokScoreErr of the exact cosine).  One warp
// per query tile u ranks its row.  With A_k the kmax-th largest approximate cosine, every tile of
// the exact Top-kmax has an approximate cosine >= A_k - 2 kTokScoreErr, and every tile below that
// has an exact value below all of theirs (the argument above token_rank_frame).  Those candidates
// get their exact value (fp64 dot of the fp32 unit vectors, rounded to fp32) and are ranked by it,
// value descending, ties to the lower tile index: the row's exact ranking.  Up to kTrCap
// candidates are listed in index order and recomputed four at a time; a row with more (many
// near-equal cosines) is recomputed in place, one candidate at a time.
constexpr int kTrCap = 256;

__host__ __device__ inline size_t tile_rank_warp_bytes(int T, int kmax) {
  const size_t row = (sizeof(float) * static_cast<size_t>(T) + 15) & ~size_t(15);
  return row + (sizeof(int) + sizeof(float)) * kTrCap + sizeof(int) * 256 +
         ((3 * sizeof(int) * static_cast<size_t>(kmax) + 15) & ~size_t(15));
}

// fp64 dots of the lane slices q with candidate rows idx[0..kN) (idx[j] for j >= n repeats
// idx[0]), all kN rows' loads in flight together, each summed over the warp.
template <int kN>
__device__ __forceinline__ void exact_dots(const double (&q)[4 * kTkChunks], const float* __restrict__ cand,
                                           const int* idx, int n, int dim, int lane, double (&e)[kN]) {
  float4 b[kN][kTkChunks];
#pragma unroll
  for (int j = 0; j < kN; ++j) {
    const float* f = cand + static_cast<size_t>(idx[j < n ? j : 0]) * dim;
#pragma unroll
    for (int c = 0; c < kTkChunks; ++c) {
      const int d = 128 * c + 4 * lane;
      b[j][c] = d < dim ? ld_f4(f + d) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
#pragma unroll
  for (int j = 0; j < kN; ++j) e[j] = 0.0;
#pragma unroll
  for (int c = 0; c < kTkChunks; ++c) {
    const double qx = q[4 * c], qy = q[4 * c + 1], qz = q[4 * c + 2], qw = q[4 * c + 3];
#pragma unroll
    for (int j = 0; j < kN; ++j) {
      e[j] = fma(qx, f32_scaled(b[j][c].x), e[j]);
      e[j] = fma(qy, f32_scaled(b[j][c].y), e[j]);
      e[j] = fma(qz, f32_scaled(b[j][c].z), e[j]);
      e[j] = fma(qw, f32_scaled(b[j][c].w), e[j]);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
#pragma unroll
    for (int j = 0; j < kN; ++j) e[j] += __shfl_xor_sync(0xffffffffu, e[j], o);
}

// Rows r0 .. r0 + rows of the ranked tile lists from the chunk's approximate cosines
// scores[rows][ld] (fp16); blockDim.x / 32 warps, one query tile each.
__global__ void __launch_bounds__(256) tile_rank_kernel(const __half* __restrict__ scores, long long ld, int r0,
                                                        int rows, const float* __restrict__ tilevec, int T, int dim,
                                                        int kmax, int32_t* __restrict__ ranked) {
  extern __shared__ __align__(16) uint8_t tr_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int lr = blockIdx.x * (blockDim.x >> 5) + warp;
  if (lr >= rows) return;  // no block-wide barrier below
  uint8_t* w = tr_smem + static_cast<size_t>(warp) * tile_rank_warp_bytes(T, kmax);
  float* row = reinterpret_cast<float*>(w);  // [T] approximate cosines
  int* cl = reinterpret_cast<int*>(w + ((sizeof(float) * static_cast<size_t>(T) + 15) & ~size_t(15)));  // [kTrCap]
  float* ev = reinterpret_cast<float*>(cl + kTrCap);   // [kTrCap] exact values of the listed candidates
  int* hist = reinterpret_cast<int*>(ev + kTrCap);     // [256]
  int* widx = hist + 256;                              // [kmax]
  uint32_t* wkey = reinterpret_cast<uint32_t*>(widx + kmax);  // [kmax]
  const int u = r0 + lr;
  double q[4 * kTkChunks];
  load_one_slice(tilevec, u, dim, lane, q);
  // the row's approximate cosines as 16-bit order keys (the row buffer's first half), read in
  // 16-byte chunks (the row starts 16-byte aligned: ld is a multiple of 8)
  const __half* srow = scores + static_cast<size_t>(lr) * ld;
  uint16_t* keys = reinterpret_cast<uint16_t*>(row);
  for (int c = lane; 8 * c < T; c += 32) {
    const uint4 w = *reinterpret_cast<const uint4*>(srow + 8 * c);
    const uint32_t h[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (8 * c + i < T) keys[8 * c + i] = static_cast<uint16_t>(order_key16((h[i >> 1] >> (16 * (i & 1))) & 0xFFFFu));
  }
  __syncwarp();
  // the kmax-th largest key by bisection: the largest x with at least kmax keys >= x
  uint32_t lo = 0u, hi = 0xFFFFu;
  while (lo < hi) {
    const uint32_t mid = (lo + hi + 1u) >> 1;
    int c = 0;
    for (int v = lane; v < T; v += 32) c += keys[v] >= mid;
    if (static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(c))) >= kmax) lo = mid;
    else hi = mid - 1u;
  }
  const float thr = key16_value(lo) - 2.f * kTokScoreErr;
  // candidates: approximate cosine >= thr, i.e. key >= the key of the least fp16 value >= thr
  const uint32_t thr_key = order_key16(__half_as_ushort(__float2half_ru(thr)));
  int m = 0;
  for (int v0 = 0; v0 < T; v0 += 32) {
    const int v = v0 + lane;
    const bool take = v < T && keys[v] >= thr_key;
    const uint32_t mask = __ballot_sync(0xffffffffu, take);
    const int pos = m + __popc(mask & ((1u << lane) - 1u));
    if (take && pos < kTrCap) cl[pos] = v;
    m += __popc(mask);
  }
  __syncwarp();
  int32_t* out = ranked + static_cast<size_t>(u) * kmax;
  if (m <= kTrCap) {
    for (int i = 0; i < m; i += 4) {
      double e[4];
      exact_dots<4>(q, tilevec, cl + i, m - i, dim, lane, e);
      if (lane == 0) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (i + j < m) ev[i + j] = static_cast<float>(e[j]);
      }
    }
    __syncwarp();
    // rank of each candidate: how many beat it (exact value descending, then tile index
    // ascending: the list is in index order, so a lower position wins a tie)
    for (int j = lane; j < m; j += 32) {
      const uint32_t kj = order_key(ev[j]);
      int rank = 0;
      for (int i = 0; i < m; ++i) {
        const uint32_t ki = order_key(ev[i]);
        rank += (ki > kj) || (ki == kj && i < j);
      }
      if (rank < kmax) out[rank] = cl[j];
    }
  } else {
    // the whole row as fp32 (over the keys, no longer needed); every other tile keeps its
    // approximate value, below all exact Top-kmax values
    for (int v = lane; v < T; v += 32) row[v] = __half2float(srow[v]);
    __syncwarp();
    for (int v0 = 0; v0 < T; v0 += 32) {
      const int v = v0 + lane;
      uint32_t todo = __ballot_sync(0xffffffffu, v < T && row[v] >= thr);
      while (todo) {
        const int bit = __ffs(todo) - 1;
        todo &= todo - 1;
        const double e = exact_dot(q, tilevec + static_cast<size_t>(v0 + bit) * dim, dim, lane);
        if (lane == 0) row[v0 + bit] = static_cast<float>(e);
      }
    }
    __syncwarp();
    warp_rank_row(row, T, kmax, hist, widx, wkey, lane, out);
  }
}

// Canonical order of the query tiles for the grouping: by the lowest tile index among the r best
// of each tile's ranked list, then by tile index.  corr_key_kernel forms each tile's 64-bit key
// (that minimum over the tile index); corr_rank_kernel gives each tile its position, the number of
// keys below its own (keys are distinct), with every key of the block held in shared memory.
__global__ void __launch_bounds__(256) corr_key_kernel(const int32_t* __restrict__ ranked, int T, int kmax, int r,
                                                       unsigned long long* __restrict__ keys) {
  const int u = blockIdx.x * blockDim.x + threadIdx.x;
  if (u >= T) return;
  const int32_t* rr = ranked + static_cast<size_t>(u) * kmax;
  int mn = 0x7fffffff;
#pragma unroll 8
  for (int i = 0; i < r; ++i) mn = min(mn, __ldg(rr + i));
  keys[u] = (static_cast<unsigned long long>(static_cast<uint32_t>(mn)) << 32) | static_cast<uint32_t>(u);
}

__global__ void __launch_bounds__(256) corr_rank_kernel(const unsigned long long* __restrict__ keys, int T,
                                                        int32_t* __restrict__ sorted) {
  extern __shared__ unsigned long long skeys[];  // [T]
  for (int v = threadIdx.x; v < T; v += blockDim.x) skeys[v] = keys[v];
  __syncthreads();
  // four threads per tile, each counting over every fourth key; a shuffle pair adds the four
  const int u = blockIdx.x * (blockDim.x >> 2) + (threadIdx.x >> 2), part = threadIdx.x & 3;
  const unsigned long long ku = u < T ? skeys[u] : 0ull;
  int rank = 0;
#pragma unroll 4
  for (int v = part; v < T; v += 4) rank += skeys[v] < ku;
  rank += __shfl_xor_sync(0xffffffffu, rank, 1);
  rank += __shfl_xor_sync(0xffffffffu, rank, 2);
  if (u < T && part == 0) sorted[rank] = u;
}

__global__ void corr_bitset_kernel(const int32_t* __restrict__ ranked, int T, int kmax, int words,
                                   uint32_t* __restrict__ bits) {
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < static_cast<long long>(T) * kmax;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int u = static_cast<int>(e / kmax);
    const int v = ranked[e];
    if (v >= 0 && v < T) atomicOr(&bits[static_cast<size_t>(u) * words + (v >> 5)], 1u << (v & 31));
  }
}

// One window of kGroupWindow sorted query tiles: the window's bitsets staged in shared memory
// (rows of words | 1 words, an odd stride, so the lanes of a warp hit distinct banks), the
// pairwise intersection counts, then one warp forms greedy groups of four.
__global__ void __launch_bounds__(256) corr_group_kernel(const uint32_t* __restrict__ bits, int T, int words,
                                                         const int32_t* __restrict__ sorted,
                                                         int32_t* __restrict__ order) {
  extern __shared__ uint32_t gbits[];  // [kGroupWindow][words | 1]
  __shared__ uint16_t inter[kGroupWindow][kGroupWindow];
  __shared__ int tiles[kGroupWindow];
  const int ws = words | 1;
  const int w0 = blockIdx.x * kGroupWindow;
  const int n = min(kGroupWindow, T - w0);
  for (int i = threadIdx.x; i < n; i += blockDim.x) tiles[i] = sorted[w0 + i];
  __syncthreads();
  for (int e = threadIdx.x; e < n * words; e += blockDim.x) {
    const int a = e / words, w = e - a * words;
    gbits[a * ws + w] = bits[static_cast<size_t>(tiles[a]) * words + w];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < n * n; e += blockDim.x) {
    const int a = e / n, b = e - a * n;
    if (b < a) continue;
    const uint32_t* ba = gbits + a * ws;
    const uint32_t* bb = gbits + b * ws;
    int c = 0;
    for (int w = 0; w < words; ++w) c += __popc(ba[w] & bb[w]);
    inter[a][b] = inter[b][a] = static_cast<uint16_t>(min(c, 65535));
  }
  __syncthreads();
  if (threadIdx.x >= 32) return;
  // one warp: greedy groups of four inside the window; lane l owns candidates l and l + 32.  A
  // candidate's key packs its score over the position from the end, so the warp maximum is the
  // highest score, ties to the earlier position; 0 marks a candidate already taken.
  const int lane = threadIdx.x;
  bool left0 = lane < n, left1 = lane + 32 < n;
  int out = w0;
  for (int u = 0; u < n; ++u) {
    const bool u_left = __shfl_sync(0xffffffffu, u < 32 ? left0 : left1, u & 31);
    if (!u_left) continue;
    if (lane == (u & 31)) {
      if (u < 32) left0 = false; else left1 = false;
    }
    if (lane == 0) order[out] = tiles[u];
    ++out;
    int sc0 = left0 ? inter[u][lane] : -1;
    int sc1 = left1 ? inter[u][lane + 32] : -1;
    for (int k = 0; k < 3; ++k) {
      const uint32_t k0 = sc0 >= 0 ? (static_cast<uint32_t>(sc0) << 7) | static_cast<uint32_t>(127 - lane) : 0u;
      const uint32_t k1 = sc1 >= 0 ? (static_cast<uint32_t>(sc1) << 7) | static_cast<uint32_t>(95 - lane) : 0u;
      const uint32_t best = __reduce_max_sync(0xffffffffu, max(k0, k1));
      if (best == 0u) break;
      const int pos = 127 - static_cast<int>(best & 127u);
      if (lane == 0) order[out] = tiles[pos];
      ++out;
      if (pos == lane) left0 = false;
      if (pos == lane + 32) left1 = false;
      sc0 = left0 ? sc0 + inter[pos][lane] : -1;
      sc1 = left1 ? sc1 + inter[pos][lane + 32] : -1;
    }
  }
}

__global__ void identity_order_kernel(int T, int32_t* order) {
  const int u = blockIdx.x * blockDim.x + threadIdx.x;
  if (u < T) order[u] = u;
}

__global__ void cache_header_kernel(CacheHeader h, CacheHeader* dst) {
  if (threadIdx.x == 0) *dst = h;
}

}  // namespace

// Workspace of the token-wise selection, after everything else: fp32 unit features [R][dim],
// fp16 unit features [R][dim16] (dim16 = dim rounded up to 64, zero-padded), and fp16 scores of
// one chunk of query rows [rows][ld] (ld = R rounded up to 8; chunks of at most ~1 GiB).
struct TokWs {
  int dim16;
  long long ld;
  int chunk_rows;
  size_t unit, unit16, scores, end;  // byte offsets from the token part's start
};

constexpr size_t kTokScoreBudget = size_t(1) << 30;

TokWs token_ws(long long R, int dim) {
  TokWs t;
  t.dim16 = (dim + 63) / 64 * 64;
  t.ld = (R + 7) / 8 * 8;
  long long rows = static_cast<long long>(kTokScoreBudget / (static_cast<size_t>(t.ld) * 2)) / 128 * 128;
  if (rows < 128) rows = 128;
  t.chunk_rows = static_cast<int>(rows < R ? rows : R);
  t.unit = 0;
  t.unit16 = (static_cast<size_t>(R) * dim * sizeof(float) + 255) & ~size_t(255);
  t.scores = (t.unit16 + static_cast<size_t>(R) * t.dim16 * 2 + 255) & ~size_t(255);
  t.end = t.scores + static_cast<size_t>(t.chunk_rows) * t.ld * 2;
  return t;
}

// Correspondence part of the select workspace, offsets from its (256-byte aligned) start: fp32 tile
// unit vectors [T][dim], grouping bitsets [T][words], sorted tiles [T], their sort keys [T]; with the tensor-core
// cosines (dim <= 384) also fp16 tile unit vectors [T][dim16] (zero-padded to a multiple of 64
// features) and the fp16 cosines of one chunk of query tiles [chunk_rows][ld] (ld = T rounded up
// to 8; chunks of at most kTileScoreBudget bytes).
constexpr size_t kTileScoreBudget = size_t(16) << 20;

struct CorrWs {
  bool tc;
  int dim16, chunk_rows;
  long long ld;
  size_t tilevec, bits, sorted, keys, tile16, scores, end;
};

CorrWs corr_ws(int T, int dim) {
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  CorrWs c;
  c.tc = dim <= 128 * kTkChunks;
  c.dim16 = (dim + 63) / 64 * 64;
  c.ld = (static_cast<long long>(T) + 7) / 8 * 8;
  long long rows = static_cast<long long>(kTileScoreBudget / (static_cast<size_t>(c.ld) * 2)) / 128 * 128;
  if (rows < 128) rows = 128;
  c.chunk_rows = static_cast<int>(rows < T ? rows : T);
  c.tilevec = 0;
  c.bits = al(static_cast<size_t>(T) * dim * sizeof(float));
  c.sorted = al(c.bits + static_cast<size_t>(T) * ((T + 31) / 32) * sizeof(uint32_t));
  c.keys = al(c.sorted + static_cast<size_t>(T) * sizeof(int32_t));
  c.end = al(c.keys + static_cast<size_t>(T) * sizeof(unsigned long long));
  c.tile16 = c.scores = c.end;
  if (c.tc) {
    c.scores = al(c.tile16 + static_cast<size_t>(T) * c.dim16 * 2);
    c.end = al(c.scores + static_cast<size_t>(c.chunk_rows) * c.ld * 2);
  }
  return c;
}

// Probe scratch: digit histograms and pass counters (zeroed per build, with one more counter per
// head for the mean's partial sums), per-chunk counts.
size_t rank_zero_bytes(int n_probe) {
  return static_cast<size_t>(n_probe) * (kRankPasses * (kRankBins * sizeof(int) + sizeof(unsigned)) + sizeof(unsigned));
}
size_t rank_counts_bytes(int n_probe, int N) {
  return static_cast<size_t>(n_probe) * ((N + kRankChunk - 1) / kRankChunk) * 2 * sizeof(int);
}

size_t select_workspace_bytes(int n_probe, int N, int T, int dim, bool corr, long long tok_rows, int tiles_P) {
  size_t b = 0;
  b += static_cast<size_t>(n_probe) * kProbePartials * kD * sizeof(double);
  b += static_cast<size_t>(n_probe) * kD * sizeof(float);
  b = (b + 255) & ~size_t(255);
  b += static_cast<size_t>(n_probe) * N * sizeof(float);
  b = (b + 255) & ~size_t(255);
  b += rank_zero_bytes(n_probe);
  b = (b + 255) & ~size_t(255);
  b += static_cast<size_t>(n_probe) * sizeof(RankState);
  b = (b + 255) & ~size_t(255);
  b += rank_counts_bytes(n_probe, N);
  b = (b + 255) & ~size_t(255);
  if (corr) b += corr_ws(T, dim).end;
  b = ((b + 255) & ~size_t(255)) + 256;
  if (tok_rows > 0) b += token_ws(tok_rows, dim).end;
  if (tok_rows > 0 && tiles_P > 0)
    b = ((b + 255) & ~size_t(255)) + tok_tiles_workspace_bytes(static_cast<int>(tok_rows / tiles_P), tiles_P);
  return b;
}

size_t token_rank_smem_bytes(int P, int kmax) {
  return 8 * (sizeof(float) * static_cast<size_t>(P) + sizeof(int) * 256 + 3 * sizeof(int) * kTokCap +
              2 * sizeof(int) * static_cast<size_t>(kmax));
}


int tile_rows_per_block(int T, int dim, int kmax) {
  // smem: R*dim + R*T floats + 8*256 ints + 16*kmax ints  <= 200 KB
  for (int R = 16; R >= 1; --R) {
    const size_t bytes = sizeof(float) * (static_cast<size_t>(R) * dim + static_cast<size_t>(R) * T) +
                         sizeof(int) * (8 * 256 + 16 * static_cast<size_t>(kmax));
    if (bytes <= 200 * 1024) return R;
  }
  return 0;
}

cudaError_t launch_select(const SelectPlan& sp, const uint16_t* q, const uint16_t* k, const float* dino,
                          int32_t* cache, uint8_t* ws, cudaStream_t stream, int* n_launch) {
  cache_header_kernel<<<1, 32, 0, stream>>>(sp.header, reinterpret_cast<CacheHeader*>(cache));
  ++*n_launch;
  size_t off = 0;
  double* partial = reinterpret_cast<double*>(ws + off);
  off += static_cast<size_t>(sp.n_probe) * kProbePartials * kD * sizeof(double);
  float* qbar = reinterpret_cast<float*>(ws + off);
  off += static_cast<size_t>(sp.n_probe) * kD * sizeof(float);
  off = (off + 255) & ~size_t(255);
  float* scores = reinterpret_cast<float*>(ws + off);
  off += static_cast<size_t>(sp.n_probe) * sp.N * sizeof(float);
  off = (off + 255) & ~size_t(255);
  int* rank_hist = reinterpret_cast<int*>(ws + off);  // zeroed with rank_done in one memset
  unsigned* rank_done = reinterpret_cast<unsigned*>(rank_hist + static_cast<size_t>(sp.n_probe) * kRankPasses * kRankBins);
  unsigned* mean_done = rank_done + static_cast<size_t>(sp.n_probe) * kRankPasses;
  off += rank_zero_bytes(sp.n_probe);
  off = (off + 255) & ~size_t(255);
  RankState* rank_state = reinterpret_cast<RankState*>(ws + off);
  off += static_cast<size_t>(sp.n_probe) * sizeof(RankState);
  off = (off + 255) & ~size_t(255);
  int* rank_counts = reinterpret_cast<int*>(ws + off);
  off += rank_counts_bytes(sp.n_probe, sp.N);
  off = (off + 255) & ~size_t(255);
  float* tilevec = reinterpret_cast<float*>(ws + off);

  if (sp.n_probe > 0) {
    ProbeArgs a;
    a.n_probe = sp.n_probe;
    for (int i = 0; i < sp.n_probe; ++i) {
      a.heads[i] = sp.probe_heads[i];
      a.k[i] = sp.probe_k[i];
      a.cache_off[i] = sp.probe_off[i];
    }
    cudaError_t e = cudaMemsetAsync(rank_hist, 0, rank_zero_bytes(sp.n_probe), stream);
    if (e != cudaSuccess) return e;
    // one wave: as many blocks per head as the SMs hold at once, split over the probe heads
    int occ_mean = 1, occ_score = 1;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_mean, probe_mean_kernel, 256, 0);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_score, probe_score_kernel, 256, 0);
    const int mean_blocks =
        std::max(1, std::min(kProbePartials, std::max(1, occ_mean) * sp.num_sms / sp.n_probe));
    probe_mean_kernel<<<dim3(mean_blocks, sp.n_probe), 256, 0, stream>>>(q, sp.N, a, partial, mean_done, qbar);
    // contiguous ranges of key rows, 32 x kProbeRowsInFlight rows per block and step
    const int score_blocks =
        std::max(1, std::min((sp.N + 127) / 128, std::max(1, occ_score) * sp.num_sms / sp.n_probe));
    probe_score_kernel<<<dim3(score_blocks, sp.n_probe), 256, 0, stream>>>(k, sp.N, sp.V, sp.ns, a, qbar, scores);
    const int rank_blocks = (sp.N + kRankChunk - 1) / kRankChunk;
    for (int pass = 0; pass < kRankPasses; ++pass)
      probe_digit_kernel<<<dim3(rank_blocks, sp.n_probe), 256, 0, stream>>>(scores, sp.N, a, pass, rank_hist,
                                                                           rank_done, rank_state);
    probe_count_kernel<<<dim3(rank_blocks, sp.n_probe), 256, 0, stream>>>(scores, sp.N, rank_state, rank_counts);
    probe_write_kernel<<<dim3(rank_blocks, sp.n_probe), 256, 0, stream>>>(scores, sp.N, a, rank_state, rank_counts,
                                                                         cache);
    *n_launch += 2 + kRankPasses + 2;
  }
  if (sp.corr_kmax > 0) {
    const CorrWs cw = corr_ws(sp.T, sp.dim);
    uint8_t* cbase = reinterpret_cast<uint8_t*>(tilevec);
    const size_t pool_smem = sizeof(float) * 5 * sp.dim;
    const size_t rank_warp = tile_rank_warp_bytes(sp.T, sp.corr_kmax);
    const int rank_warps = static_cast<int>(std::min<size_t>(8, (112 * 1024) / rank_warp));
    cudaError_t e = cudaSuccess;
    if (cw.tc && rank_warps >= 1) {
      // cosines on the tensor cores (fp16 operands), exact ranking of the candidates they leave
      __half* tile16 = reinterpret_cast<__half*>(cbase + cw.tile16);
      __half* tscores = reinterpret_cast<__half*>(cbase + cw.scores);
      dino_pool_kernel<3><<<sp.T, 128, pool_smem, stream>>>(dino, sp.N, sp.V, sp.ns, sp.P, sp.dim, tilevec, tile16,
                                                            cw.dim16);
      ++*n_launch;
      CUtensorMap tm;
      if (!make_map_f16_rows(&tm, tile16, sp.T, cw.dim16)) return cudaErrorInvalidValue;
      const size_t rsmem = rank_warps * rank_warp;
      e = cudaFuncSetAttribute(tile_rank_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(rsmem));
      if (e != cudaSuccess) return e;
      for (int r0 = 0; r0 < sp.T; r0 += cw.chunk_rows) {
        const int rows = std::min(cw.chunk_rows, sp.T - r0);
        TokenSimParams tp;
        tp.r0 = r0;
        tp.rows = rows;
        tp.n_rb = (rows + 127) / 128;
        tp.n_ct = (sp.T + 255) / 256;
        tp.n_kc = cw.dim16 / 64;
        tp.ld = cw.ld;
        tp.scores = reinterpret_cast<uint16_t*>(tscores);
        tp.err = sp.err;
        tp.wait_budget = sp.wait_budget;
        e = launch_token_sim(tp, tm, sp.num_sms, stream);
        if (e != cudaSuccess) return e;
        tile_rank_kernel<<<(rows + rank_warps - 1) / rank_warps, 32 * rank_warps, rsmem, stream>>>(
            tscores, cw.ld, r0, rows, tilevec, sp.T, sp.dim, sp.corr_kmax, cache + sp.corr_off);
        *n_launch += 2;
      }
    } else {
      if (sp.dim <= 128 * 3)
        dino_pool_kernel<3><<<sp.T, 128, pool_smem, stream>>>(dino, sp.N, sp.V, sp.ns, sp.P, sp.dim, tilevec,
                                                              nullptr, 0);
      else
        dino_pool_kernel<8><<<sp.T, 128, pool_smem, stream>>>(dino, sp.N, sp.V, sp.ns, sp.P, sp.dim, tilevec,
                                                              nullptr, 0);
      const int R = tile_rows_per_block(sp.T, sp.dim, sp.corr_kmax);
      if (R <= 0) return cudaErrorInvalidValue;
      const size_t smem = sizeof(float) * (static_cast<size_t>(R) * sp.dim + static_cast<size_t>(R) * sp.T) +
                          sizeof(int) * (8 * 256 + 16 * static_cast<size_t>(sp.corr_kmax));
      e = cudaFuncSetAttribute(tile_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      if (e != cudaSuccess) return e;
      tile_topk_kernel<<<(sp.T + R - 1) / R, 256, smem, stream>>>(tilevec, sp.T, sp.dim, R, sp.corr_kmax,
                                                                  cache + sp.corr_off);
      *n_launch += 2;
    }
    // query-tile grouping for the attention work items
    const int words = (sp.T + 31) / 32;
    uint32_t* bits = reinterpret_cast<uint32_t*>(cbase + cw.bits);
    int32_t* sorted = reinterpret_cast<int32_t*>(cbase + cw.sorted);
    int32_t* order = cache + sp.order_off;
    if (sp.T <= kMaxSortTiles) {
      unsigned long long* gkeys = reinterpret_cast<unsigned long long*>(cbase + cw.keys);
      corr_key_kernel<<<(sp.T + 255) / 256, 256, 0, stream>>>(cache + sp.corr_off, sp.T, sp.corr_kmax,
                                                               sp.corr_kmax > 1 ? sp.corr_kmax / 2 : 1, gkeys);
      const size_t ksmem = sizeof(unsigned long long) * static_cast<size_t>(sp.T);
      e = cudaFuncSetAttribute(corr_rank_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(ksmem));
      if (e != cudaSuccess) return e;
      corr_rank_kernel<<<(sp.T + 63) / 64, 256, ksmem, stream>>>(gkeys, sp.T, sorted);
      e = cudaMemsetAsync(bits, 0, static_cast<size_t>(sp.T) * words * sizeof(uint32_t), stream);
      if (e != cudaSuccess) return e;
      corr_bitset_kernel<<<148, 256, 0, stream>>>(cache + sp.corr_off, sp.T, sp.corr_kmax, words, bits);
      const size_t gsmem = sizeof(uint32_t) * kGroupWindow * static_cast<size_t>(words | 1);
      e = cudaFuncSetAttribute(corr_group_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(gsmem));
      if (e != cudaSuccess) return e;
      corr_group_kernel<<<(sp.T + kGroupWindow - 1) / kGroupWindow, 256, gsmem, stream>>>(bits, sp.T, words, sorted,
                                                                                          order);
      *n_launch += 4;
    } else {
      identity_order_kernel<<<(sp.T + 255) / 256, 256, 0, stream>>>(sp.T, order);
      *n_launch += 1;
    }
  }
  if (sp.tok_kmax > 0) {
    // the token part of the workspace, after everything else
    uint8_t* base = ws + select_workspace_bytes(sp.n_probe, sp.N, sp.T, sp.dim, sp.corr_kmax > 0, 0, 0);
    const long long R = static_cast<long long>(sp.S) * sp.P;
    const TokWs tw = token_ws(R, sp.dim);
    float* unit = reinterpret_cast<float*>(base + tw.unit);
    __half* unit16 = reinterpret_cast<__half*>(base + tw.unit16);
    __half* scores = reinterpret_cast<__half*>(base + tw.scores);
    unit_features_kernel<<<static_cast<unsigned>((R + 7) / 8), 256, 0, stream>>>(dino, static_cast<int>(R), sp.dim,
                                                                                 unit, unit16, tw.dim16);
    ++*n_launch;
    CUtensorMap tm;
    if (!make_map_f16_rows(&tm, unit16, R, tw.dim16)) return cudaErrorInvalidValue;
    const size_t rsmem = token_rank_smem_bytes(sp.P, sp.tok_kmax);
    cudaError_t e = cudaFuncSetAttribute(token_rank_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(rsmem));
    if (e != cudaSuccess) return e;
    for (long long r0 = 0; r0 < R; r0 += tw.chunk_rows) {
      const int rows = static_cast<int>(R - r0 < tw.chunk_rows ? R - r0 : tw.chunk_rows);
      TokenSimParams tp;
      tp.r0 = static_cast<int>(r0);
      tp.rows = rows;
      tp.n_rb = (rows + 127) / 128;
      tp.n_ct = static_cast<int>((R + 255) / 256);
      tp.n_kc = tw.dim16 / 64;
      tp.ld = tw.ld;
      tp.scores = reinterpret_cast<uint16_t*>(scores);
      tp.err = sp.err;
      tp.wait_budget = sp.wait_budget;
      e = launch_token_sim(tp, tm, sp.num_sms, stream);
      if (e != cudaSuccess) return e;
      token_rank_kernel<<<(rows + 7) / 8, 256, rsmem, stream>>>(scores, tw.ld, static_cast<int>(r0), rows, unit, sp.S,
                                                                sp.P, sp.dim, sp.tok_kmax, cache + sp.tok_off);
      *n_launch += 2;
    }
    if (sp.tperm_off >= 0) {
      // the patch query order and every group's unions and masks, after the lists
      e = launch_tok_tiles(cache + sp.tok_off, sp.S, sp.P, sp.V, sp.ns, sp.tok_kmax, sp.tperm_off, sp.tg, sp.n_tg,
                           cache, base + ((tw.end + 255) & ~size_t(255)), sp.err, stream, n_launch);
      if (e != cudaSuccess) return e;
    }
  }
  return cudaGetLastError();
}

}  // namespace saf3r
