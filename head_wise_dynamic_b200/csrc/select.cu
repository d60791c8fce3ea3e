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

constexpr int kProbePartials = 296;  // row blocks per probe head (2 x 148 SMs)

__device__ __forceinline__ uint32_t order_key(float f) {
  // monotone map fp32 -> uint32 (larger float -> larger key)
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

struct ProbeArgs {
  int n_probe;
  int heads[kMaxHeads];      // head index of each probe head
  int k[kMaxHeads];          // kept patch keys
  int cache_off[kMaxHeads];  // int32 offset of the key list in the cache
};

// The 8 bf16 features of a 16-byte chunk as fp64, in order.
__device__ __forceinline__ void bf16x8_to_f64(const uint4& w, double (&x)[8]) {
  x[0] = static_cast<double>(bf16_lo(w.x));
  x[1] = static_cast<double>(bf16_hi(w.x));
  x[2] = static_cast<double>(bf16_lo(w.y));
  x[3] = static_cast<double>(bf16_hi(w.y));
  x[4] = static_cast<double>(bf16_lo(w.z));
  x[5] = static_cast<double>(bf16_hi(w.z));
  x[6] = static_cast<double>(bf16_lo(w.w));
  x[7] = static_cast<double>(bf16_hi(w.w));
}

// acc[i] += feature i of a 16-byte chunk of 8 bf16 features (fp64 sums).
__device__ __forceinline__ void add_bf16x8(double (&acc)[8], const uint4& w) {
  acc[0] += static_cast<double>(bf16_lo(w.x));
  acc[1] += static_cast<double>(bf16_hi(w.x));
  acc[2] += static_cast<double>(bf16_lo(w.y));
  acc[3] += static_cast<double>(bf16_hi(w.y));
  acc[4] += static_cast<double>(bf16_lo(w.z));
  acc[5] += static_cast<double>(bf16_hi(w.z));
  acc[6] += static_cast<double>(bf16_lo(w.w));
  acc[7] += static_cast<double>(bf16_hi(w.w));
}

// Partial fp64 column sums of Q_h over a range of rows.  Lane l of a warp reads the 16-byte
// chunk (l % 8) of row r + l / 8 (a warp reads 4 whole rows, 512 contiguous bytes, per load) and
// keeps the 8 column sums of its chunk; two rows per lane are in flight per step.  The lanes and
// warps that share a chunk are added in a fixed order at the end.
__global__ void __launch_bounds__(256) probe_partial_kernel(const uint16_t* __restrict__ q, int N,
                                                            ProbeArgs a, double* __restrict__ partial) {
  const int hp = blockIdx.y;
  const int h = a.heads[hp];
  const int rows_per = (N + gridDim.x - 1) / gridDim.x;
  const int r0 = blockIdx.x * rows_per;
  const int r1 = min(N, r0 + rows_per);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, sub = lane & 7;
  const uint4* qh = reinterpret_cast<const uint4*>(q + static_cast<size_t>(h) * N * kD);
  double acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.0;
  int r = r0 + warp * 4 + (lane >> 3);
  for (; r + 32 < r1; r += 64) {
    const uint4 w0 = qh[static_cast<size_t>(r) * 8 + sub];
    const uint4 w1 = qh[static_cast<size_t>(r + 32) * 8 + sub];
    add_bf16x8(acc, w0);
    add_bf16x8(acc, w1);
  }
  if (r < r1) add_bf16x8(acc, qh[static_cast<size_t>(r) * 8 + sub]);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 8);
    acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 16);
  }
  __shared__ double wsum[8][kD];
  if (lane < 8) {
#pragma unroll
    for (int i = 0; i < 8; ++i) wsum[warp][8 * sub + i] = acc[i];
  }
  __syncthreads();
  if (threadIdx.x < kD) {
    double t = 0.0;
    for (int w = 0; w < 8; ++w) t += wsum[w][threadIdx.x];
    partial[(static_cast<size_t>(hp) * gridDim.x + blockIdx.x) * kD + threadIdx.x] = t;
  }
}

// qbar = (sum of partials) / N, rounded once to fp32.  Four threads per column take every
// fourth partial; their sums are added in a fixed order.
__global__ void __launch_bounds__(256) probe_mean_kernel(const double* __restrict__ partial, int nparts, int N,
                                                         float* __restrict__ qbar) {
  const int hp = blockIdx.x, c = threadIdx.x & (kD - 1), g = threadIdx.x >> 6;
  const double* base = partial + static_cast<size_t>(hp) * nparts * kD + c;
  double t0 = 0.0, t1 = 0.0;
  int b = g;
  for (; b + 4 < nparts; b += 8) {
    t0 += base[static_cast<size_t>(b) * kD];
    t1 += base[static_cast<size_t>(b + 4) * kD];
  }
  if (b < nparts) t0 += base[static_cast<size_t>(b) * kD];
  __shared__ double gs[4][kD];
  gs[g][c] = t0 + t1;
  __syncthreads();
  if (g == 0) qbar[hp * kD + c] = static_cast<float>(((gs[0][c] + gs[1][c]) + (gs[2][c] + gs[3][c])) /
                                                    static_cast<double>(N));
}

// score_j = qbar . k_j / 8 (fp64 dot, fp32 result); special keys get -inf so they are never ranked.
// Eight lanes per key row, each with one 16-byte chunk (a warp reads 4 whole rows, 512 contiguous
// bytes, per load), two rows per lane group in flight; the 8 partial dots meet in 3 shuffles.
__global__ void __launch_bounds__(256) probe_score_kernel(const uint16_t* __restrict__ k, int N, int V, int ns,
                                                          ProbeArgs a, const float* __restrict__ qbar,
                                                          float* __restrict__ scores) {
  const int hp = blockIdx.y;
  const int h = a.heads[hp];
  const int sub = threadIdx.x & 7;
  double qv[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) qv[i] = static_cast<double>(qbar[hp * kD + 8 * sub + i]);
  const uint4* kh = reinterpret_cast<const uint4*>(k + static_cast<size_t>(h) * N * kD);
  const int groups = (gridDim.x * blockDim.x) >> 3;
  for (int j = (blockIdx.x * blockDim.x + threadIdx.x) >> 3; j < N; j += 2 * groups) {
    const int j1 = j + groups;
    const bool two = j1 < N;  // uniform over the 8 lanes of a row group
    const uint4 w0 = kh[static_cast<size_t>(j) * 8 + sub];
    const uint4 w1 = two ? kh[static_cast<size_t>(j1) * 8 + sub] : make_uint4(0u, 0u, 0u, 0u);
    double x[8], d0 = 0.0, d1 = 0.0;
    bf16x8_to_f64(w0, x);
#pragma unroll
    for (int i = 0; i < 8; ++i) d0 = fma(qv[i], x[i], d0);
    bf16x8_to_f64(w1, x);
#pragma unroll
    for (int i = 0; i < 8; ++i) d1 = fma(qv[i], x[i], d1);
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
      d0 += __shfl_xor_sync(0xffffffffu, d0, o);
      d1 += __shfl_xor_sync(0xffffffffu, d1, o);
    }
    if (sub == 0) {
      scores[static_cast<size_t>(hp) * N + j] = (j % V) < ns ? -INFINITY : static_cast<float>(d0 * 0.125);
      if (two) scores[static_cast<size_t>(hp) * N + j1] = (j1 % V) < ns ? -INFINITY : static_cast<float>(d1 * 0.125);
    }
  }
}

// Block-wide exclusive scan of one int per thread (blockDim.x == 1024).
__device__ __forceinline__ int block_exclusive_scan(int v, int* tmp /*[32]*/, int& total) {
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
    int w = tmp[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    tmp[lane] = w;
  }
  __syncthreads();
  total = tmp[31];
  const int before = warp > 0 ? tmp[warp - 1] : 0;
  __syncthreads();
  return before + x - v;
}

// Top-k of one probe head's scores: radix select of the k-th largest key, then an
// ordered compaction that keeps every key above it and the lowest-index keys equal to it.
__global__ void __launch_bounds__(1024) probe_topk_kernel(const float* __restrict__ scores, int N, ProbeArgs a,
                                                          int32_t* __restrict__ cache) {
  const int hp = blockIdx.x;
  const int K = a.k[hp];
  const float* sc = scores + static_cast<size_t>(hp) * N;
  int32_t* out = cache + a.cache_off[hp];
  __shared__ int hist[256];
  __shared__ int tmp[32];
  __shared__ uint32_t s_prefix;
  __shared__ int s_remaining;

  uint32_t prefix = 0, mask = 0;
  int remaining = K;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int j = threadIdx.x; j < N; j += blockDim.x) {
      const uint32_t key = order_key(sc[j]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 0xFF], 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int above = 0, b = 255;
      for (; b > 0; --b) {
        if (above + hist[b] >= remaining) break;
        above += hist[b];
      }
      s_prefix = prefix | (static_cast<uint32_t>(b) << shift);
      s_remaining = remaining - above;
    }
    __syncthreads();
    prefix = s_prefix;
    remaining = s_remaining;
    mask |= 0xFFu << shift;
    __syncthreads();
  }
  // prefix is the k-th largest key; `remaining` keys equal to it are kept (lowest indices first).
  const int per = (N + blockDim.x - 1) / blockDim.x;
  const int j0 = threadIdx.x * per, j1 = min(N, j0 + per);
  int n_gt = 0, n_eq = 0;
  for (int j = j0; j < j1; ++j) {
    const uint32_t key = order_key(sc[j]);
    n_gt += key > prefix;
    n_eq += key == prefix;
  }
  int tot_eq = 0, tot_gt = 0;
  const int eq_before = block_exclusive_scan(n_eq, tmp, tot_eq);
  const int eq_take = max(0, min(n_eq, remaining - eq_before));
  const int mine = n_gt + eq_take;
  const int pos0 = block_exclusive_scan(mine, tmp, tot_gt);
  int pos = pos0, eq_seen = 0;
  for (int j = j0; j < j1; ++j) {
    const uint32_t key = order_key(sc[j]);
    bool take = key > prefix;
    if (key == prefix) {
      take = eq_seen < eq_take;
      ++eq_seen;
    }
    if (take) out[pos++] = j;
  }
}

// Mean of L2-normalised DINO features over the patch tokens of each 64-token tile,
// then normalised to unit length (its cosine against other tiles is a plain dot).
__global__ void __launch_bounds__(128) dino_pool_kernel(const float* __restrict__ dino, int N, int V, int ns,
                                                        int P, int dim, float* __restrict__ tilevec) {
  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  extern __shared__ float pool_smem[];  // [4][dim] per-warp sums, then [dim] mean
  float* wsum = pool_smem;
  for (int i = threadIdx.x; i < 4 * dim; i += blockDim.x) wsum[i] = 0.f;
  __syncthreads();
  int count = 0;
  const int tok0 = t * kTile, tok1 = min(N, tok0 + kTile);
  const int nc = dim >> 2;  // 16-byte chunks per feature row (dim is a multiple of 4, at most 1024)
  for (int tok = tok0 + warp; tok < tok1; tok += 4) {
    const int s = tok / V, loc = tok - s * V;
    if (loc < ns) continue;
    // the row once, in 16-byte loads, kept in registers for both passes
    const float4* f = reinterpret_cast<const float4*>(dino + (static_cast<size_t>(s) * P + (loc - ns)) * dim);
    float4 x[8];
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int i = 32 * c + lane;
      x[c] = i < nc ? f[i] : make_float4(0.f, 0.f, 0.f, 0.f);
      ss = fmaf(x[c].x, x[c].x, fmaf(x[c].y, x[c].y, fmaf(x[c].z, x[c].z, fmaf(x[c].w, x[c].w, ss))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = 1.f / sqrtf(ss);
    float4* w4 = reinterpret_cast<float4*>(wsum + warp * dim);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int i = 32 * c + lane;
      if (i < nc) {
        float4 a = w4[i];
        a.x += x[c].x * inv;
        a.y += x[c].y * inv;
        a.z += x[c].z * inv;
        a.w += x[c].w * inv;
        w4[i] = a;
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
}

// Inverse of order_key.
__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
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
    int b = 255, above = 0;
    for (; b > 0; --b) {
      if (above + wh[b] >= remaining) break;
      above += wh[b];
    }
    prefix |= static_cast<uint32_t>(b) << shift;
    remaining -= above;
    mask |= 0xFFu << shift;
    __syncwarp();
  }
}

// The kmax largest values of row[0..T) (ties to the lower index) written to out[0..kmax) in
// rank order (value descending, then index ascending).  One warp.
__device__ __forceinline__ void warp_rank_row(const float* row, int T, int kmax, int* wh, int* widx, uint32_t* wkey,
                                              int lane, int32_t* __restrict__ out) {
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
    out[rank] = vi;
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

// Fast form for dim <= 384 (kTkChunks float4 chunks of 128 features per lane).
//
// Eight query tiles per block, one per warp for the ranking.  Every lane keeps its slice of
// the eight query vectors in registers; a warp takes one candidate tile v at a time with
// coalesced loads, forms eight fp32 partial dots and folds them over the warp with a
// transposing butterfly (after it, lane group (lane>>2)&7 holds row r's full dot).
//
// fp32 accumulation misses the fp64 dot by at most (12 + 5) * 2^-24 * sum|a_i b_i| <= 1.02e-6
// (unit vectors: sum|a_i b_i| <= 1; 12 products per lane, 5 butterfly levels).  So every tile
// of the exact top-kmax has an fp32 cosine >= (the fp32 kmax-th value) - 2.04e-6, and every
// tile below (the fp32 kmax-th value) - kTkBand cannot reach it.  The ranking therefore
// recomputes exactly (fp64 dot, rounded to fp32 as the general form does) every tile within
// kTkBand of the fp32 kmax-th value, and ranks the row: the result is the general form's.
constexpr int kTkRows = 8;
constexpr int kTkChunks = 3;
constexpr float kTkBand = 4e-6f;

__device__ __forceinline__ float4 ld_f4(const float* p) { return *reinterpret_cast<const float4*>(p); }

// This lane's slice of kTkRows unit vectors (rows u0.. of `vec`; absent rows and features are 0).
__device__ __forceinline__ void load_row_slices(const float* __restrict__ vec, int u0, int nr, int dim, int lane,
                                                float4 (&q)[kTkRows][kTkChunks]) {
#pragma unroll
  for (int r = 0; r < kTkRows; ++r)
#pragma unroll
    for (int c = 0; c < kTkChunks; ++c) {
      const int d = 128 * c + 4 * lane;
      q[r][c] = (r < nr && d < dim) ? ld_f4(vec + static_cast<size_t>(u0 + r) * dim + d)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

// fp32 dots of the kTkRows query vectors with candidates cand[0..n) (unit vectors, row-major,
// `dim` wide) into cs[r * ld + v]: each warp takes one candidate at a time with coalesced loads
// and folds its eight partial dots over the warp with a transposing butterfly (after it, lane
// group (lane>>2)&7 holds row r's full dot).  All warps of the block take part.
__device__ __forceinline__ void dots_fp32(const float4 (&q)[kTkRows][kTkChunks], const float* __restrict__ cand,
                                          int n, int dim, int nr, float* cs, int ld, int warp, int lane) {
  const int b2 = (lane >> 2) & 1, b3 = (lane >> 3) & 1, b4 = (lane >> 4) & 1;
  const int my_row = (lane >> 2) & 7;
  for (int v = warp; v < n; v += 8) {
    const float* fv = cand + static_cast<size_t>(v) * dim;
    float a[kTkRows];
#pragma unroll
    for (int r = 0; r < kTkRows; ++r) a[r] = 0.f;
#pragma unroll
    for (int c = 0; c < kTkChunks; ++c) {
      const int d = 128 * c + 4 * lane;
      if (d < dim) {
        const float4 b = ld_f4(fv + d);
#pragma unroll
        for (int r = 0; r < kTkRows; ++r) {
          a[r] = fmaf(q[r][c].x, b.x, a[r]);
          a[r] = fmaf(q[r][c].y, b.y, a[r]);
          a[r] = fmaf(q[r][c].z, b.z, a[r]);
          a[r] = fmaf(q[r][c].w, b.w, a[r]);
        }
      }
    }
    float h4[4], h2[2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float send = b4 ? a[i] : a[i + 4], keep = b4 ? a[i + 4] : a[i];
      h4[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float send = b3 ? h4[i] : h4[i + 2], keep = b3 ? h4[i + 2] : h4[i];
      h2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    float h1;
    {
      const float send = b2 ? h2[0] : h2[1], keep = b2 ? h2[1] : h2[0];
      h1 = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    h1 += __shfl_xor_sync(0xffffffffu, h1, 2);
    h1 += __shfl_xor_sync(0xffffffffu, h1, 1);
    if ((lane & 3) == 0 && my_row < nr) cs[static_cast<size_t>(my_row) * ld + v] = h1;
  }
}

// One warp: rank row[0..n) (fp32 dots of query row `rq` with candidates cand[0..n)) exactly.
// Every candidate within kTkBand of the fp32 kmax-th value gets its exact value (fp64 dot,
// rounded to fp32), then the row is ranked; out[0..kmax) receives candidate indices.
__device__ __forceinline__ void rank_row_exact(float* row, int n, int kmax, const float4 (&q)[kTkRows][kTkChunks],
                                               int rq, const float* __restrict__ cand, int dim, int* wh, int* widx,
                                               uint32_t* wkey, int lane, int32_t* __restrict__ out) {
  uint32_t prefix;
  int remaining;
  warp_radix_kth(row, n, kmax, wh, lane, prefix, remaining);
  const float thr = key_value(prefix) - kTkBand;
  for (int v0 = 0; v0 < n; v0 += 32) {
    const int v = v0 + lane;
    uint32_t todo = __ballot_sync(0xffffffffu, v < n && row[v] >= thr);
    while (todo) {
      const int bit = __ffs(todo) - 1;
      todo &= todo - 1;
      const int w = v0 + bit;
      const float* fv = cand + static_cast<size_t>(w) * dim;
      double acc = 0.0;
#pragma unroll
      for (int c = 0; c < kTkChunks; ++c) {
        const int d = 128 * c + 4 * lane;
        if (d < dim) {
          const float4 b = ld_f4(fv + d);
          float4 qa = q[0][c];
#pragma unroll
          for (int r = 1; r < kTkRows; ++r)
            if (r == rq) qa = q[r][c];
          acc = fma(static_cast<double>(qa.x), static_cast<double>(b.x), acc);
          acc = fma(static_cast<double>(qa.y), static_cast<double>(b.y), acc);
          acc = fma(static_cast<double>(qa.z), static_cast<double>(b.z), acc);
          acc = fma(static_cast<double>(qa.w), static_cast<double>(b.w), acc);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) row[w] = static_cast<float>(acc);
    }
  }
  __syncwarp();
  warp_rank_row(row, n, kmax, wh, widx, wkey, lane, out);
}

__global__ void __launch_bounds__(256) tile_topk_fast_kernel(const float* __restrict__ tilevec, int T, int dim,
                                                             int kmax, int32_t* __restrict__ ranked) {
  extern __shared__ uint8_t tk_smem[];
  float* cs = reinterpret_cast<float*>(tk_smem);                               // [8][T]
  int* hist = reinterpret_cast<int*>(cs + static_cast<size_t>(kTkRows) * T);  // [8 warps][256]
  int* sel_idx = hist + 8 * 256;                                               // [8 warps][kmax]
  uint32_t* sel_key = reinterpret_cast<uint32_t*>(sel_idx + 8 * kmax);         // [8 warps][kmax]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u0 = blockIdx.x * kTkRows;
  const int nr = min(kTkRows, T - u0);
  float4 q[kTkRows][kTkChunks];
  load_row_slices(tilevec, u0, nr, dim, lane, q);
  dots_fp32(q, tilevec, T, dim, nr, cs, T, warp, lane);
  __syncthreads();
  if (warp >= nr) return;
  rank_row_exact(cs + static_cast<size_t>(warp) * T, T, kmax, q, warp, tilevec, dim, hist + warp * 256,
                 sel_idx + warp * kmax, sel_key + warp * kmax, lane, ranked + static_cast<size_t>(u0 + warp) * kmax);
}

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

// This lane's slice of unit vector `row` (features 128c + 4 lane .. +3).
__device__ __forceinline__ void load_one_slice(const float* __restrict__ vec, int row, int dim, int lane,
                                               float4 (&q)[kTkChunks]) {
#pragma unroll
  for (int c = 0; c < kTkChunks; ++c) {
    const int d = 128 * c + 4 * lane;
    q[c] = d < dim ? ld_f4(vec + static_cast<size_t>(row) * dim + d) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// fp64 dot of the lane slices q with candidate row fv, summed over the warp (every lane gets
// the same value: a butterfly adds the same two operands on both sides of each exchange).
__device__ __forceinline__ double exact_dot(const float4 (&q)[kTkChunks], const float* __restrict__ fv, int dim,
                                           int lane) {
  double acc = 0.0;
#pragma unroll
  for (int c = 0; c < kTkChunks; ++c) {
    const int d = 128 * c + 4 * lane;
    if (d < dim) {
      const float4 b = ld_f4(fv + d);
      acc = fma(static_cast<double>(q[c].x), static_cast<double>(b.x), acc);
      acc = fma(static_cast<double>(q[c].y), static_cast<double>(b.y), acc);
      acc = fma(static_cast<double>(q[c].z), static_cast<double>(b.z), acc);
      acc = fma(static_cast<double>(q[c].w), static_cast<double>(b.w), acc);
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
__device__ void token_rank_general(const __half* __restrict__ seg, int P, int kmax, const float4 (&q)[kTkChunks],
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
__device__ __forceinline__ void exact_dot2(const float4 (&q)[kTkChunks], const float* __restrict__ f1,
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
    const double qx = q[c].x, qy = q[c].y, qz = q[c].z, qw = q[c].w;
    a1 = fma(qx, static_cast<double>(b1[c].x), a1);
    a2 = fma(qx, static_cast<double>(b2[c].x), a2);
    a1 = fma(qy, static_cast<double>(b1[c].y), a1);
    a2 = fma(qy, static_cast<double>(b2[c].y), a2);
    a1 = fma(qz, static_cast<double>(b1[c].z), a1);
    a2 = fma(qz, static_cast<double>(b2[c].z), a2);
    a1 = fma(qw, static_cast<double>(b1[c].w), a1);
    a2 = fma(qw, static_cast<double>(b2[c].w), a2);
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
                                 const float4 (&q)[kTkChunks], const float* __restrict__ cand, int dim,
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
  float4 q[kTkChunks];
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

__global__ void __launch_bounds__(1024) corr_sort_kernel(const int32_t* __restrict__ ranked, int T, int kmax,
                                                         int r, int32_t* __restrict__ order) {
  extern __shared__ unsigned long long keys[];  // [pow2 >= T]
  int n2 = 1;
  while (n2 < T) n2 <<= 1;
  for (int u = threadIdx.x; u < n2; u += blockDim.x) {
    unsigned long long k = ~0ull;
    if (u < T) {
      int mn = 0x7fffffff;
      for (int i = 0; i < r; ++i) mn = min(mn, ranked[static_cast<size_t>(u) * kmax + i]);
      k = (static_cast<unsigned long long>(static_cast<uint32_t>(mn)) << 32) | static_cast<uint32_t>(u);
    }
    keys[u] = k;
  }
  __syncthreads();
  for (int size = 2; size <= n2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < n2; i += blockDim.x) {
        const int j = i ^ stride;
        if (j > i) {
          const bool up = (i & size) == 0;
          const unsigned long long a = keys[i], b = keys[j];
          if ((a > b) == up) {
            keys[i] = b;
            keys[j] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int u = threadIdx.x; u < T; u += blockDim.x) order[u] = static_cast<int32_t>(keys[u] & 0xffffffffu);
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

__global__ void __launch_bounds__(256) corr_group_kernel(const uint32_t* __restrict__ bits, int T, int words,
                                                         const int32_t* __restrict__ sorted,
                                                         int32_t* __restrict__ order) {
  __shared__ uint16_t inter[kGroupWindow][kGroupWindow];
  __shared__ int tiles[kGroupWindow];
  const int w0 = blockIdx.x * kGroupWindow;
  const int n = min(kGroupWindow, T - w0);
  for (int i = threadIdx.x; i < n; i += blockDim.x) tiles[i] = sorted[w0 + i];
  __syncthreads();
  for (int e = threadIdx.x; e < n * n; e += blockDim.x) {
    const int a = e / n, b = e - a * n;
    if (b < a) continue;
    const uint32_t* ba = bits + static_cast<size_t>(tiles[a]) * words;
    const uint32_t* bb = bits + static_cast<size_t>(tiles[b]) * words;
    int c = 0;
    for (int w = 0; w < words; ++w) c += __popc(ba[w] & bb[w]);
    inter[a][b] = inter[b][a] = static_cast<uint16_t>(min(c, 65535));
  }
  __syncthreads();
  if (threadIdx.x >= 32) return;
  // one warp: greedy groups of four inside the window; lane l owns candidates l and l + 32
  const int lane = threadIdx.x;
  bool left0 = lane < n, left1 = lane + 32 < n;
  int out = w0;
  for (int u = 0; u < n; ++u) {
    const bool u_left = __shfl_sync(0xffffffffu, (u & 31) < 32 ? ((u < 32) ? left0 : left1) : false, u & 31);
    if (!u_left) continue;
    if (lane == (u & 31)) {
      if (u < 32) left0 = false; else left1 = false;
    }
    if (lane == 0) order[out] = tiles[u];
    ++out;
    int sc0 = left0 ? inter[u][lane] : -1;
    int sc1 = left1 ? inter[u][lane + 32] : -1;
    for (int k = 0; k < 3; ++k) {
      // argmax over the window (ties to the earlier position)
      int best = sc0 >= sc1 ? sc0 : sc1;
      int pos = sc0 >= sc1 ? lane : lane + 32;
      if (best < 0) pos = 1 << 20;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const int ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int op = __shfl_xor_sync(0xffffffffu, pos, o);
        if (ob > best || (ob == best && op < pos)) {
          best = ob;
          pos = op;
        }
      }
      if (best < 0) break;
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

size_t select_workspace_bytes(int n_probe, int N, int T, int dim, bool corr, long long tok_rows) {
  size_t b = 0;
  b += static_cast<size_t>(n_probe) * kProbePartials * kD * sizeof(double);
  b += static_cast<size_t>(n_probe) * kD * sizeof(float);
  b = (b + 255) & ~size_t(255);
  b += static_cast<size_t>(n_probe) * N * sizeof(float);
  b = (b + 255) & ~size_t(255);
  if (corr) {
    b += static_cast<size_t>(T) * dim * sizeof(float);
    b = (b + 255) & ~size_t(255);
    b += static_cast<size_t>(T) * ((T + 31) / 32) * sizeof(uint32_t);  // grouping bitsets
    b = (b + 255) & ~size_t(255);
    b += static_cast<size_t>(T) * sizeof(int32_t);                      // sorted tiles
  }
  b = ((b + 255) & ~size_t(255)) + 256;
  if (tok_rows > 0) b += token_ws(tok_rows, dim).end;
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
  float* tilevec = reinterpret_cast<float*>(ws + off);

  if (sp.n_probe > 0) {
    ProbeArgs a;
    a.n_probe = sp.n_probe;
    for (int i = 0; i < sp.n_probe; ++i) {
      a.heads[i] = sp.probe_heads[i];
      a.k[i] = sp.probe_k[i];
      a.cache_off[i] = sp.probe_off[i];
    }
    probe_partial_kernel<<<dim3(kProbePartials, sp.n_probe), 256, 0, stream>>>(q, sp.N, a, partial);
    probe_mean_kernel<<<sp.n_probe, 4 * kD, 0, stream>>>(partial, kProbePartials, sp.N, qbar);
    // 32 key rows per 256-thread block and step; at most 8 blocks per SM and head
    const int score_blocks = std::max(1, std::min((sp.N + 63) / 64, 8 * sp.num_sms));
    probe_score_kernel<<<dim3(score_blocks, sp.n_probe), 256, 0, stream>>>(k, sp.N, sp.V, sp.ns, a, qbar, scores);
    probe_topk_kernel<<<sp.n_probe, 1024, 0, stream>>>(scores, sp.N, a, cache);
    *n_launch += 4;
  }
  if (sp.corr_kmax > 0) {
    const size_t pool_smem = sizeof(float) * 5 * sp.dim;
    dino_pool_kernel<<<sp.T, 128, pool_smem, stream>>>(dino, sp.N, sp.V, sp.ns, sp.P, sp.dim, tilevec);
    cudaError_t e = cudaSuccess;
    const size_t fast_smem = sizeof(float) * static_cast<size_t>(kTkRows) * sp.T +
                             sizeof(int) * (8 * 256 + 16 * static_cast<size_t>(sp.corr_kmax));
    if (sp.dim <= 128 * kTkChunks && fast_smem <= 200 * 1024) {
      e = cudaFuncSetAttribute(tile_topk_fast_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(fast_smem));
      if (e != cudaSuccess) return e;
      tile_topk_fast_kernel<<<(sp.T + kTkRows - 1) / kTkRows, 256, fast_smem, stream>>>(
          tilevec, sp.T, sp.dim, sp.corr_kmax, cache + sp.corr_off);
    } else {
      const int R = tile_rows_per_block(sp.T, sp.dim, sp.corr_kmax);
      if (R <= 0) return cudaErrorInvalidValue;
      const size_t smem = sizeof(float) * (static_cast<size_t>(R) * sp.dim + static_cast<size_t>(R) * sp.T) +
                          sizeof(int) * (8 * 256 + 16 * static_cast<size_t>(sp.corr_kmax));
      e = cudaFuncSetAttribute(tile_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      if (e != cudaSuccess) return e;
      tile_topk_kernel<<<(sp.T + R - 1) / R, 256, smem, stream>>>(tilevec, sp.T, sp.dim, R, sp.corr_kmax,
                                                                  cache + sp.corr_off);
    }
    *n_launch += 2;
    // query-tile grouping for the attention work items
    size_t goff = static_cast<size_t>(reinterpret_cast<uint8_t*>(tilevec) - ws) +
                  static_cast<size_t>(sp.T) * sp.dim * sizeof(float);
    goff = (goff + 255) & ~size_t(255);
    const int words = (sp.T + 31) / 32;
    uint32_t* bits = reinterpret_cast<uint32_t*>(ws + goff);
    goff += static_cast<size_t>(sp.T) * words * sizeof(uint32_t);
    goff = (goff + 255) & ~size_t(255);
    int32_t* sorted = reinterpret_cast<int32_t*>(ws + goff);
    int32_t* order = cache + sp.order_off;
    if (sp.T <= kMaxSortTiles) {
      int n2 = 1;
      while (n2 < sp.T) n2 <<= 1;
      const size_t ssmem = sizeof(unsigned long long) * n2;
      e = cudaFuncSetAttribute(corr_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(ssmem));
      if (e != cudaSuccess) return e;
      corr_sort_kernel<<<1, 1024, ssmem, stream>>>(cache + sp.corr_off, sp.T, sp.corr_kmax,
                                                   sp.corr_kmax > 1 ? sp.corr_kmax / 2 : 1, sorted);
      e = cudaMemsetAsync(bits, 0, static_cast<size_t>(sp.T) * words * sizeof(uint32_t), stream);
      if (e != cudaSuccess) return e;
      corr_bitset_kernel<<<148, 256, 0, stream>>>(cache + sp.corr_off, sp.T, sp.corr_kmax, words, bits);
      corr_group_kernel<<<(sp.T + kGroupWindow - 1) / kGroupWindow, 256, 0, stream>>>(bits, sp.T, words, sorted,
                                                                                      order);
      *n_launch += 3;
    } else {
      identity_order_kernel<<<(sp.T + 255) / 256, 256, 0, stream>>>(sp.T, order);
      *n_launch += 1;
    }
  }
  if (sp.tok_kmax > 0) {
    // the token part of the workspace, after everything else
    uint8_t* base = ws + select_workspace_bytes(sp.n_probe, sp.N, sp.T, sp.dim, sp.corr_kmax > 0, 0);
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
  }
  return cudaGetLastError();
}

}  // namespace saf3r
