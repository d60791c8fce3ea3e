// Token-wise heads on the tensor cores: the index-build side.
//
// SAF3R ("SAF3R: Dynamic Sparse Attention for Feed-Forward 3D Reconstruction Transformers"),
// section 4.1 "DINO Top-K Kernel" and section 4.3: a token-wise head keeps, for every patch
// query, the Top-K most similar patch tokens of every frame (plus the special tokens).  Such
// per-row key sets share little inside a fixed tile of neighbouring queries, but queries that
// show the same scene point in different views have nearly the same lists.  This file
//   * orders the patch queries by their best match in frame 0, then in frame 1, then by row, so
//     that queries of one scene point become neighbours (a counting sort on the frame-0 match,
//     then a rank by count inside each bucket: deterministic);
//   * builds, for every 256-row work item of that order, the union of its rows' kept tokens,
//     ascending, and one bitmask per row over that union (bit set = the row keeps that token);
//   * writes, at every attention call, each item's key runs: the head's derived special rows,
//     then the item's union.
// The attention kernel then streams each item's union once for all 256 rows through the tensor
// cores and masks per row, so every row still gets the exact softmax over its own keys.
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"

namespace saf3r {

namespace {

constexpr int kScanThreads = 1024;
constexpr size_t kUnionSmemLimit = 200 * 1024;

struct TokGroups {
  int n;
  TokTileGroup g[kMaxHeads];
};

// Union builder shared memory: the frame's bitmap over P patches and its word prefix, then a
// window of mask words (slot j = union half-block hb0 + j, one 64-bit word per item row).
__host__ __device__ inline int union_words(int P) { return (P + 31) / 32; }
__host__ __device__ inline int union_slots(int P) { return (P + 63) / 64 + 1; }
size_t union_smem_bytes(int P) {
  return sizeof(uint64_t) * static_cast<size_t>(union_slots(P)) * kItemRows +
         sizeof(uint32_t) * 2 * static_cast<size_t>(union_words(P)) + 16;
}

// The best match of patch query u in frame f (entry 0 of its ranked list), clamped into [0, P):
// the order only groups rows, an out-of-range entry is reported where the lists are consumed.
__device__ __forceinline__ int best_match(const int32_t* lists, long long u, int S, int kmax, int f, int P) {
  const int p = lists[(u * S + f) * kmax];
  return (p >= 0 && p < P) ? p : 0;
}

__global__ void tok_order_count_kernel(const int32_t* __restrict__ lists, long long R, int S, int kmax, int P,
                                       int* __restrict__ hist) {
  for (long long u = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; u < R;
       u += static_cast<long long>(gridDim.x) * blockDim.x)
    atomicAdd(&hist[best_match(lists, u, S, kmax, 0, P)], 1);
}

// start[b] = rows in buckets before b (start[P] = R); one block.
__global__ void __launch_bounds__(kScanThreads) tok_order_scan_kernel(const int* __restrict__ hist, int P,
                                                                      int* __restrict__ start) {
  __shared__ int warp_tot[kScanThreads / 32];
  __shared__ int carry_s;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry_s = 0;
  __syncthreads();
  for (int base = 0; base < P; base += kScanThreads) {
    const int i = base + threadIdx.x;
    const int v = i < P ? hist[i] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int before = carry_s;
    for (int w = 0; w < warp; ++w) before += warp_tot[w];
    if (i < P) start[i] = before + incl - v;
    __syncthreads();
    if (threadIdx.x == kScanThreads - 1) carry_s = before + incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) start[P] = carry_s;
}

// Every row into its bucket (any order inside it), with its sort key (frame-1 match, row).
__global__ void tok_order_scatter_kernel(const int32_t* __restrict__ lists, long long R, int S, int kmax, int P,
                                         const int* __restrict__ start, int* __restrict__ cursor,
                                         uint64_t* __restrict__ keys) {
  for (long long u = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; u < R;
       u += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int b = best_match(lists, u, S, kmax, 0, P);
    const int k2 = S > 1 ? best_match(lists, u, S, kmax, 1, P) : 0;
    const int pos = atomicAdd(&cursor[b], 1);
    keys[start[b] + pos] = (static_cast<uint64_t>(k2) << 32) | static_cast<uint64_t>(u);
  }
}

// perm[start[b] + rank] = row, the rank counted among the bucket's keys.
__global__ void tok_order_rank_kernel(const int32_t* __restrict__ lists, long long R, int S, int kmax, int P,
                                      const int* __restrict__ start, const uint64_t* __restrict__ keys,
                                      int32_t* __restrict__ perm) {
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < R;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint64_t key = keys[i];
    const long long u = static_cast<long long>(key & 0xffffffffull);
    const int b = best_match(lists, u, S, kmax, 0, P);
    const int lo = start[b], hi = start[b + 1];
    int rank = 0;
    for (int j = lo; j < hi; ++j) rank += keys[j] < key;
    perm[lo + rank] = static_cast<int32_t>(u);
  }
}

// One block per (item, group), one thread per item row.  Frame by frame: the bitmap of the
// patches any row keeps, its prefix counts (a kept patch's rank in the frame's union), the
// union's tokens, then each row's bits, accumulated in the row's column of the mask window and
// written out once a 64-entry half-block is complete.
__global__ void __launch_bounds__(kItemRows) tok_union_kernel(const int32_t* __restrict__ lists,
                                                              const int32_t* __restrict__ perm, int S, int P, int V,
                                                              int ns, int kmax, const TokGroups groups,
                                                              int32_t* __restrict__ cache, int* err) {
  extern __shared__ uint64_t win[];  // [slots][kItemRows]
  const int W = union_words(P);
  uint32_t* bm = reinterpret_cast<uint32_t*>(win + static_cast<size_t>(union_slots(P)) * kItemRows);
  uint32_t* pre = bm + W;
  __shared__ int uf_s;
  const TokTileGroup g = groups.g[blockIdx.y];
  const int item = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long R = static_cast<long long>(S) * P;
  const long long row = static_cast<long long>(item) * kItemRows + tid;
  long long u = -1;
  if (row < R) {
    u = perm[row];
    if (u < 0 || u >= R) {
      atomicCAS(err, 0, SAF3R_ERR_INDEX);
      u = -1;
    }
  }
  int32_t* tu = cache + g.tu_off + static_cast<long long>(item) * g.ucap;
  uint64_t* tm = reinterpret_cast<uint64_t*>(cache + g.tm_off) + static_cast<long long>(item) * (g.ucap / 64) * kItemRows;
  const int slots = union_slots(P);
  for (int j = 0; j < slots; ++j) win[j * kItemRows + tid] = 0ull;
  int base = 0, hb0 = 0;
  for (int f = 0; f < S; ++f) {
    for (int w = tid; w < W; w += kItemRows) bm[w] = 0u;
    __syncthreads();
    const int32_t* lf = u >= 0 ? lists + (u * S + f) * kmax : lists;
    if (u >= 0) {
      for (int e = 0; e < g.k; ++e) {
        const int p = lf[e];
        if (p >= 0 && p < P)
          atomicOr(&bm[p >> 5], 1u << (p & 31));
        else
          atomicCAS(err, 0, SAF3R_ERR_INDEX);
      }
    }
    __syncthreads();
    if (warp == 0) {
      int run = 0;
      for (int w0 = 0; w0 < W; w0 += 32) {
        const int w = w0 + lane;
        const int c = w < W ? __popc(bm[w]) : 0;
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        if (w < W) pre[w] = run + incl - c;
        run += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) uf_s = run;
    }
    __syncthreads();
    const int uf = uf_s;
    for (int w = tid; w < W; w += kItemRows) {
      uint32_t bits = bm[w];
      int pos = base + pre[w];
      while (bits) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1u;
        tu[pos++] = f * V + ns + 32 * w + b;
      }
    }
    if (u >= 0) {
      for (int e = 0; e < g.k; ++e) {
        const int p = lf[e];
        if (p < 0 || p >= P) continue;
        const uint32_t word = bm[p >> 5];
        const int pos = base + pre[p >> 5] + __popc(word & ((1u << (p & 31)) - 1u));
        win[((pos >> 6) - hb0) * kItemRows + tid] |= 1ull << (pos & 63);
      }
    }
    // half-blocks before the one holding the next frame's first entry are complete
    const int nb = base + uf;
    const int last = (nb >> 6) - hb0;
    for (int j = 0; j < last; ++j) tm[static_cast<long long>(hb0 + j) * kItemRows + tid] = win[j * kItemRows + tid];
    if (last > 0) {
      win[tid] = win[last * kItemRows + tid];
      for (int j = 1; j <= last; ++j) win[j * kItemRows + tid] = 0ull;
    }
    base = nb;
    hb0 += last;
    __syncthreads();  // bm and pre are rewritten by the next frame
  }
  if (base & 63) tm[static_cast<long long>(hb0) * kItemRows + tid] = win[tid];
  if (tid == 0) cache[g.tn_off + item] = base;
}

// Per call: item m's runs are the nsp derived special rows, then its union (gathered keys).
__global__ void plan_token_kernel(const int32_t* __restrict__ tn, int ucap, int n_items, int nsp,
                                  Seg* __restrict__ segs, int* __restrict__ counts, int* err) {
  const int m = blockIdx.x * blockDim.x + threadIdx.x;
  if (m >= n_items) return;
  int U = tn[m];
  if (U < 0 || U > ucap) {
    atomicCAS(err, 0, SAF3R_ERR_INDEX);
    U = 0;
  }
  segs[2 * m] = Seg{1, 0, nsp, kSegAllQuarters};
  segs[2 * m + 1] = Seg{2, m * ucap, U, kSegAllQuarters};
  const int nhb = (nsp + 63) / 64 + (U + 63) / 64;
  counts[2 * m] = 2;
  counts[2 * m + 1] = max(1, (nhb + 1) / 2);
}

}  // namespace

bool tok_tiles_fit(int P) { return P >= 1 && union_smem_bytes(P) <= kUnionSmemLimit; }

size_t tok_tiles_workspace_bytes(int S, int P) {
  const size_t ints = (3 * static_cast<size_t>(P) + 1 + 63) & ~size_t(63);
  return ints * sizeof(int) + static_cast<size_t>(S) * P * sizeof(uint64_t);
}

cudaError_t launch_tok_tiles(const int32_t* lists, int S, int P, int V, int ns, int tok_kmax, long long tperm_off,
                             const TokTileGroup* tg, int n_tg, int32_t* cache, uint8_t* ws, int* err,
                             cudaStream_t stream, int* n_launch) {
  const long long R = static_cast<long long>(S) * P;
  int* hist = reinterpret_cast<int*>(ws);
  int* start = hist + P;
  int* cursor = start + P + 1;
  const size_t ints = (3 * static_cast<size_t>(P) + 1 + 63) & ~size_t(63);
  uint64_t* keys = reinterpret_cast<uint64_t*>(ws + ints * sizeof(int));
  int32_t* perm = cache + tperm_off;
  cudaError_t e = cudaMemsetAsync(hist, 0, (3 * static_cast<size_t>(P) + 1) * sizeof(int), stream);
  if (e != cudaSuccess) return e;
  const int grid = static_cast<int>((R + 255) / 256);
  tok_order_count_kernel<<<grid, 256, 0, stream>>>(lists, R, S, tok_kmax, P, hist);
  tok_order_scan_kernel<<<1, kScanThreads, 0, stream>>>(hist, P, start);
  tok_order_scatter_kernel<<<grid, 256, 0, stream>>>(lists, R, S, tok_kmax, P, start, cursor, keys);
  tok_order_rank_kernel<<<grid, 256, 0, stream>>>(lists, R, S, tok_kmax, P, start, keys, perm);
  *n_launch += 4;
  TokGroups groups;
  groups.n = n_tg;
  for (int i = 0; i < n_tg; ++i) groups.g[i] = tg[i];
  const size_t smem = union_smem_bytes(P);
  e = cudaFuncSetAttribute(tok_union_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int items = static_cast<int>((R + kItemRows - 1) / kItemRows);
  if (n_tg > 0) {
    tok_union_kernel<<<dim3(items, n_tg), kItemRows, smem, stream>>>(lists, perm, S, P, V, ns, tok_kmax, groups,
                                                                      cache, err);
    ++*n_launch;
  }
  return cudaGetLastError();
}

cudaError_t launch_plan_token(const int32_t* tn, int ucap, int n_items, int nsp, Seg* segs, int* counts, int* err,
                              cudaStream_t stream) {
  plan_token_kernel<<<(n_items + 127) / 128, 128, 0, stream>>>(tn, ucap, n_items, nsp, segs, counts, err);
  return cudaGetLastError();
}

}  // namespace saf3r
