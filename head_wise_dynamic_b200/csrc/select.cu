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

// Partial fp64 column sums of Q_h over a range of rows.
__global__ void __launch_bounds__(256) probe_partial_kernel(const uint16_t* __restrict__ q, int N,
                                                            ProbeArgs a, double* __restrict__ partial) {
  const int hp = blockIdx.y;
  const int h = a.heads[hp];
  const int rows_per = (N + gridDim.x - 1) / gridDim.x;
  const int r0 = blockIdx.x * rows_per;
  const int r1 = min(N, r0 + rows_per);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t* qh = reinterpret_cast<const uint32_t*>(q + static_cast<size_t>(h) * N * kD);
  double s0 = 0.0, s1 = 0.0;
  for (int r = r0 + warp; r < r1; r += 8) {
    const uint32_t w = qh[static_cast<size_t>(r) * (kD / 2) + lane];
    s0 += static_cast<double>(bf16_lo(w));
    s1 += static_cast<double>(bf16_hi(w));
  }
  __shared__ double acc[8][kD];
  acc[warp][2 * lane] = s0;
  acc[warp][2 * lane + 1] = s1;
  __syncthreads();
  if (threadIdx.x < kD) {
    double t = 0.0;
    for (int w = 0; w < 8; ++w) t += acc[w][threadIdx.x];
    partial[(static_cast<size_t>(hp) * gridDim.x + blockIdx.x) * kD + threadIdx.x] = t;
  }
}

// qbar = (sum of partials, in block order) / N, rounded once to fp32.
__global__ void probe_mean_kernel(const double* __restrict__ partial, int nparts, int N,
                                  float* __restrict__ qbar) {
  const int hp = blockIdx.x, c = threadIdx.x;
  double t = 0.0;
  for (int b = 0; b < nparts; ++b) t += partial[(static_cast<size_t>(hp) * nparts + b) * kD + c];
  qbar[hp * kD + c] = static_cast<float>(t / static_cast<double>(N));
}

// score_j = qbar . k_j / 8 (fp64 dot, fp32 result); special keys get -inf so they are never ranked.
__global__ void __launch_bounds__(256) probe_score_kernel(const uint16_t* __restrict__ k, int N, int V, int ns,
                                                          ProbeArgs a, const float* __restrict__ qbar,
                                                          float* __restrict__ scores) {
  const int hp = blockIdx.y;
  const int h = a.heads[hp];
  const int lane = threadIdx.x & 31;
  const double q0 = static_cast<double>(qbar[hp * kD + 2 * lane]);
  const double q1 = static_cast<double>(qbar[hp * kD + 2 * lane + 1]);
  const uint32_t* kh = reinterpret_cast<const uint32_t*>(k + static_cast<size_t>(h) * N * kD);
  const int warps_total = gridDim.x * 8;
  for (int j = blockIdx.x * 8 + (threadIdx.x >> 5); j < N; j += warps_total) {
    const uint32_t w = kh[static_cast<size_t>(j) * (kD / 2) + lane];
    double d = q0 * static_cast<double>(bf16_lo(w)) + q1 * static_cast<double>(bf16_hi(w));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
    if (lane == 0) {
      const bool special = (j % V) < ns;
      scores[static_cast<size_t>(hp) * N + j] = special ? -INFINITY : static_cast<float>(d * 0.125);
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
  for (int tok = tok0 + warp; tok < tok1; tok += 4) {
    const int s = tok / V, loc = tok - s * V;
    if (loc < ns) continue;
    const float* f = dino + (static_cast<size_t>(s) * P + (loc - ns)) * dim;
    float ss = 0.f;
    for (int c = lane; c < dim; c += 32) ss = fmaf(f[c], f[c], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = 1.f / sqrtf(ss);
    for (int c = lane; c < dim; c += 32) wsum[warp * dim + c] += f[c] * inv;
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

// Cosines of R query tiles against all T tiles (fp64 dots of unit vectors,
// rounded to fp32), then per query tile the kmax best tiles in rank order.
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
  int* wh = hist + warp * 256;
  int* widx = sel_idx + warp * kmax;
  uint32_t* wkey = sel_key + warp * kmax;
  for (int r = warp; r < nr; r += 8) {
    const float* row = cs + static_cast<size_t>(r) * T;
    uint32_t prefix = 0, mask = 0;
    int remaining = kmax;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = lane; i < 256; i += 32) wh[i] = 0;
      __syncwarp();
      for (int v = lane; v < T; v += 32) {
        const uint32_t key = order_key(row[v]);
        if ((key & mask) == prefix) atomicAdd(&wh[(key >> shift) & 0xFF], 1);
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
      ranked[static_cast<size_t>(u0 + r) * kmax + rank] = vi;
    }
    __syncwarp();
  }
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

size_t select_workspace_bytes(int n_probe, int N, int T, int dim, bool corr) {
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
  return b + 256;
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
    probe_mean_kernel<<<sp.n_probe, kD, 0, stream>>>(partial, kProbePartials, sp.N, qbar);
    probe_score_kernel<<<dim3(296, sp.n_probe), 256, 0, stream>>>(k, sp.N, sp.V, sp.ns, a, qbar, scores);
    probe_topk_kernel<<<sp.n_probe, 1024, 0, stream>>>(scores, sp.N, a, cache);
    *n_launch += 4;
  }
  if (sp.corr_kmax > 0) {
    const size_t pool_smem = sizeof(float) * 5 * sp.dim;
    dino_pool_kernel<<<sp.T, 128, pool_smem, stream>>>(dino, sp.N, sp.V, sp.ns, sp.P, sp.dim, tilevec);
    const int R = tile_rows_per_block(sp.T, sp.dim, sp.corr_kmax);
    if (R <= 0) return cudaErrorInvalidValue;
    const size_t smem = sizeof(float) * (static_cast<size_t>(R) * sp.dim + static_cast<size_t>(R) * sp.T) +
                        sizeof(int) * (8 * 256 + 16 * static_cast<size_t>(sp.corr_kmax));
    cudaError_t e =
        cudaFuncSetAttribute(tile_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    tile_topk_kernel<<<(sp.T + R - 1) / R, 256, smem, stream>>>(tilevec, sp.T, sp.dim, R, sp.corr_kmax,
                                                                cache + sp.corr_off);
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
  return cudaGetLastError();
}

}  // namespace saf3r
