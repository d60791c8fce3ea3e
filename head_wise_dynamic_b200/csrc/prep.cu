// Per-call preparation for the attention kernel, and the NMSE reduction.
//
//  * cache check: the index cache header must match the layout/config hash;
//  * derived rows: each head's shared key rows are copied into one contiguous
//    region (special tokens; the anchor view's patches; the probe's kept keys;
//    the stride lattice), and position heads get cell-major copies of Q (and
//    of K/V for views 1..S-1) so that the 3x3 neighbourhood of a grid cell
//    in every view becomes a few contiguous runs of rows;
//  * plans: per 256-row work item, the list of key runs covering the union of
//    its rows' kept sets (position and correspondence heads);
//  * NMSE (SAF3R eq. 1): sum (O_full - O_sparse)^2 and sum O_full^2 per head in
//    fp64, reduced in a fixed order.
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"

namespace saf3r {

namespace {

__device__ __forceinline__ int special_token(int r, int V, int ns) {
  const int s = r / ns;
  return s * V + (r - s * ns);
}

__device__ __forceinline__ int derived_token(const DerivedArgs& a, const DerivedHead& d, int r,
                                             const int32_t* cache, const int* offlists, int* err) {
  const int nsp = a.ns * a.S;
  switch (d.kind) {
    case SAF3R_POSITION: {
      if (r < nsp) return special_token(r, a.V, a.ns);
      r -= nsp;
      if (r < a.P) return a.ns + r;  // anchor view 0 patches
      r -= a.P;
      const int cell = r / (a.S - 1), s = 1 + (r - cell * (a.S - 1));
      return s * a.V + a.ns + cell;
    }
    case SAF3R_PROBE: {
      if (r < nsp) return special_token(r, a.V, a.ns);
      const int t = cache[d.probe_off + (r - nsp)];
      if (t < 0 || t >= a.N || (t % a.V) < a.ns) {
        atomicCAS(err, 0, SAF3R_ERR_INDEX);
        return 0;
      }
      return t;
    }
    case SAF3R_SCAN:
    case SAF3R_HYBRID:  // the lattice, then the specials off it
      if (r < d.n_lat) return d.phase + r * d.stride;
      return offlists[d.off_list + (r - d.n_lat)];
    default:  // SAF3R_CORR, SAF3R_TOKEN: the special tokens
      return special_token(r, a.V, a.ns);
  }
}

__device__ __forceinline__ int cm_query_token(int i, int S, int V, int ns, int P) {
  if (i < P * S) {
    const int cell = i / S, s = i - cell * S;
    return s * V + ns + cell;
  }
  const int sp = i - P * S;
  const int s = sp / ns;
  return s * V + (sp - s * ns);
}

}  // namespace

// Header check: writes 1 to *ok when the cache was built for this (layout, cfg).
__global__ void cache_check_kernel(const CacheHeader* h, uint64_t hash, int N, int T, int* ok, int* err) {
  if (threadIdx.x != 0) return;
  const bool good = h->magic == kCacheMagic && h->version == kCacheVersion && h->hash == hash && h->N == N &&
                    h->T == T;
  *ok = good ? 1 : 0;
  if (!good) atomicCAS(err, 0, SAF3R_ERR_INVALID);
}

// Off-lattice special tokens of each scan head, ascending (one warp per head).
__global__ void scan_specials_kernel(DerivedArgs a, int* offlists) {
  const DerivedHead& d = a.h[blockIdx.x];
  if (!lattice_kind(d.kind)) return;
  const int lane = threadIdx.x;
  const int nsp = a.ns * a.S;
  int base = 0;
  for (int r0 = 0; r0 < nsp; r0 += 32) {
    const int r = r0 + lane;
    int t = 0;
    bool off = false;
    if (r < nsp) {
      t = special_token(r, a.V, a.ns);
      off = (t % d.stride) != d.phase;
    }
    const uint32_t m = __ballot_sync(0xffffffffu, off);
    if (off) offlists[d.off_list + base + __popc(m & ((1u << lane) - 1u))] = t;
    base += __popc(m);
  }
}

// Copy derived K/V rows (and cell-major Q rows): 8 threads per 128-byte row.
__global__ void __launch_bounds__(256) gather_rows_kernel(DerivedArgs a, const uint16_t* __restrict__ q,
                                                          const uint16_t* __restrict__ k,
                                                          const uint16_t* __restrict__ v,
                                                          const int32_t* __restrict__ cache,
                                                          const int* __restrict__ offlists, uint16_t* __restrict__ kc,
                                                          uint16_t* __restrict__ vc, uint16_t* __restrict__ qc,
                                                          int* err) {
  const long long total = a.kc_total + a.qc_total;
  const int sub = threadIdx.x & 7;
  for (long long task = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 3; task < total;
       task += (static_cast<long long>(gridDim.x) * blockDim.x) >> 3) {
    if (task < a.kc_total) {
      const int row = static_cast<int>(task);
      int hi = 0;
      while (hi + 1 < a.n && row >= a.h[hi + 1].kc_begin) ++hi;
      const DerivedHead& d = a.h[hi];
      const int tok = derived_token(a, d, row - d.kc_begin, cache, offlists, err);
      const size_t src = (static_cast<size_t>(d.head) * a.N + tok) * kD;
      const uint4* ks = reinterpret_cast<const uint4*>(k + src);
      const uint4* vs = reinterpret_cast<const uint4*>(v + src);
      reinterpret_cast<uint4*>(kc + static_cast<size_t>(row) * kD)[sub] = ks[sub];
      reinterpret_cast<uint4*>(vc + static_cast<size_t>(row) * kD)[sub] = vs[sub];
    } else {
      const int row = static_cast<int>(task - a.kc_total);
      int hi = -1;
      for (int i = 0; i < a.n; ++i)
        if (a.h[i].qc_begin >= 0 && row >= a.h[i].qc_begin && row < a.h[i].qc_begin + a.h[i].n_q) hi = i;
      if (hi < 0) continue;
      const DerivedHead& d = a.h[hi];
      // position heads: every query in cell-major order; token-wise heads: the special tokens,
      // then (tensor-core plan) the patch queries in the cached order
      const int r = row - d.qc_begin;
      int tok;
      if (d.kind != SAF3R_TOKEN) {
        tok = cm_query_token(r, a.S, a.V, a.ns, a.P);
      } else if (r < a.ns * a.S) {
        tok = special_token(r, a.V, a.ns);
      } else {
        const int u = cache[a.tperm_off + (r - a.ns * a.S)];
        if (u < 0 || u >= a.S * a.P) {
          if (sub == 0) atomicCAS(err, 0, SAF3R_ERR_INDEX);
          tok = a.ns;  // a patch token: the row is computed and never written
        } else {
          tok = (u / a.P) * a.V + a.ns + (u % a.P);
        }
      }
      const size_t src = (static_cast<size_t>(d.head) * a.N + tok) * kD;
      reinterpret_cast<uint4*>(qc + static_cast<size_t>(row) * kD)[sub] =
          reinterpret_cast<const uint4*>(q + src)[sub];
    }
  }
}

// Key runs of every 256-row item of a position head (one thread per item).
__global__ void plan_position_kernel(int n_items, int S, int gh, int gw, int ns, int N, int R, int cap,
                                     Seg* __restrict__ segs, int* __restrict__ counts) {
  const int m = blockIdx.x * blockDim.x + threadIdx.x;
  if (m >= n_items) return;
  const int P = gh * gw;
  Seg* out = segs + static_cast<size_t>(m) * cap;
  int n = 0;
  out[n++] = Seg{1, 0, ns * S + P, kSegAllQuarters};
  const int i0 = m * kItemRows;
  const int i1 = min(N, i0 + kItemRows);
  const int nb_base = ns * S + P;
  if (S > 1 && i0 < P * S && R >= 0) {  // R < 0: the anchor frame only, no neighbourhood runs
    const int c_lo = i0 / S, c_hi = (min(i1, P * S) - 1) / S;
    const int r_lo = c_lo / gw, r_hi = c_hi / gw;
    int prev_end = -1;
    for (int rr = max(r_lo - R, 0); rr <= min(r_hi + R, gh - 1); ++rr) {
      int ia[2 * kMaxRadius + 1], ib[2 * kMaxRadius + 1], ni = 0;
      for (int r = max(rr - R, r_lo); r <= min(rr + R, r_hi); ++r) {
        const int qa = (r == r_lo) ? c_lo % gw : 0;
        const int qb = (r == r_hi) ? c_hi % gw : gw - 1;
        int a = max(qa - R, 0), b = min(qb + R, gw - 1);
        // insert sorted by start
        int pos = ni++;
        while (pos > 0 && ia[pos - 1] > a) {
          ia[pos] = ia[pos - 1];
          ib[pos] = ib[pos - 1];
          --pos;
        }
        ia[pos] = a;
        ib[pos] = b;
      }
      for (int x = 0; x < ni;) {
        int a = ia[x], b = ib[x];
        int y = x + 1;
        while (y < ni && ia[y] <= b + 1) {
          b = max(b, ib[y]);
          ++y;
        }
        x = y;
        const int start = nb_base + (rr * gw + a) * (S - 1);
        const int end = nb_base + (rr * gw + b + 1) * (S - 1);
        if (start == prev_end && n > 1) {
          out[n - 1].len += end - start;
        } else if (n < cap) {
          out[n++] = Seg{1, start, end - start, kSegAllQuarters | kSegCellMask};
        }
        prev_end = end;
      }
    }
  }
  int nhb = 0;  // 64-key half-blocks of the item's runs
  for (int x = 0; x < n; ++x) nhb += (out[x].len + 63) >> 6;
  counts[2 * m] = n;
  counts[2 * m + 1] = (nhb + 1) >> 1;
}

// Key runs of every 256-row item of a correspondence head: the union of its four
// query tiles' selected key tiles (ascending, with the quarters that keep each),
// then the special tokens.  Quarter q of item m is query tile order[4m + q].
__global__ void __launch_bounds__(256) plan_corr_kernel(const int32_t* __restrict__ ranked,
                                                        const int32_t* __restrict__ order, int kmax, int kt, int T,
                                                        int N, int V, int ns, int tail_len, Seg* __restrict__ segs,
                                                        int cap, int* __restrict__ counts, int* err) {
  extern __shared__ uint32_t memb[];  // [T]
  __shared__ int tmp[32];
  const int m = blockIdx.x;
  for (int v = threadIdx.x; v < T; v += blockDim.x) memb[v] = 0;
  __syncthreads();
  for (int e = threadIdx.x; e < 4 * kt; e += blockDim.x) {
    const int q = e / kt, r = e - q * kt;
    if (4 * m + q >= T) continue;
    const int u = order[4 * m + q];
    if (u < 0 || u >= T) {
      atomicCAS(err, 0, SAF3R_ERR_INDEX);
      continue;
    }
    const int v = ranked[static_cast<size_t>(u) * kmax + r];
    if (v < 0 || v >= T) {
      atomicCAS(err, 0, SAF3R_ERR_INDEX);
      continue;
    }
    atomicOr(&memb[v], 1u << q);
  }
  __syncthreads();
  Seg* out = segs + static_cast<size_t>(m) * cap;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int base = 0;
  for (int v0 = 0; v0 < T; v0 += blockDim.x) {
    const int v = v0 + threadIdx.x;
    const uint32_t mb = v < T ? memb[v] : 0u;
    const bool take = mb != 0u;
    const uint32_t bal = __ballot_sync(0xffffffffu, take);
    if (lane == 0) tmp[warp] = __popc(bal);
    __syncthreads();
    int before = 0, tot = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
      if (w < warp) before += tmp[w];
      tot += tmp[w];
    }
    if (take) {
      const int pos = base + before + __popc(bal & ((1u << lane) - 1u));
      const int t0 = v * kTile, t1 = min(N, t0 + kTile);
      const int s = t0 / V, loc = t0 - s * V;
      int lo = 0, hi = 0;
      if (loc < ns) {
        hi = min(ns - loc, t1 - t0);
      } else {
        const int nv = (s + 1) * V;
        if (nv < t1) {
          lo = nv - t0;
          hi = min(nv + ns, t1) - t0;
        }
      }
      if (pos < cap - 1)
        out[pos] = Seg{0, t0, t1 - t0, mb | (static_cast<uint32_t>(lo) << 8) | (static_cast<uint32_t>(hi) << 16)};
    }
    base += tot;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const int nu = min(base, cap - 1);
    out[nu] = Seg{1, 0, tail_len, kSegAllQuarters};  // the head's derived rows: specials (and its lattice)
    counts[2 * m] = nu + 1;
    counts[2 * m + 1] = (nu + ((tail_len + 63) >> 6) + 1) >> 1;  // each key tile is one half-block
  }
}

// NMSE partial sums: per (head, block) sum (a-b)^2 and sum a^2 in fp64.
__global__ void __launch_bounds__(256) nmse_partial_kernel(const float* __restrict__ full,
                                                           const float* __restrict__ sparse, long long per_head,
                                                           double* __restrict__ part) {
  const int h = blockIdx.y;
  const float* a = full + static_cast<size_t>(h) * per_head;
  const float* b = sparse + static_cast<size_t>(h) * per_head;
  double se = 0.0, sf = 0.0;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < per_head;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const double x = a[i], y = b[i];
    se += (x - y) * (x - y);
    sf += x * x;
  }
  __shared__ double r0[256], r1[256];
  r0[threadIdx.x] = se;
  r1[threadIdx.x] = sf;
  __syncthreads();
  for (int s = 128; s > 0; s >>= 1) {
    if (threadIdx.x < s) {
      r0[threadIdx.x] += r0[threadIdx.x + s];
      r1[threadIdx.x] += r1[threadIdx.x + s];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    part[(static_cast<size_t>(h) * gridDim.x + blockIdx.x) * 2] = r0[0];
    part[(static_cast<size_t>(h) * gridDim.x + blockIdx.x) * 2 + 1] = r1[0];
  }
}

__global__ void nmse_final_kernel(const double* __restrict__ part, int nblk, int H, double* __restrict__ out) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h >= H) return;
  double se = 0.0, sf = 0.0;
  for (int b = 0; b < nblk; ++b) {
    se += part[(static_cast<size_t>(h) * nblk + b) * 2];
    sf += part[(static_cast<size_t>(h) * nblk + b) * 2 + 1];
  }
  out[2 * h] = se;
  out[2 * h + 1] = sf;
}

// ---------------------------------------------------------------- launchers

cudaError_t launch_cache_check(const void* cache, uint64_t hash, int N, int T, int* ok, int* err,
                               cudaStream_t stream) {
  cache_check_kernel<<<1, 32, 0, stream>>>(static_cast<const CacheHeader*>(cache), hash, N, T, ok, err);
  return cudaGetLastError();
}

cudaError_t launch_derived(const DerivedArgs& a, bool any_scan, const uint16_t* q, const uint16_t* k,
                           const uint16_t* v, const int32_t* cache, int* offlists, uint16_t* kc, uint16_t* vc,
                           uint16_t* qc, int* err, int num_sms, cudaStream_t stream, int* n_launch) {
  if (any_scan) {
    scan_specials_kernel<<<a.n, 32, 0, stream>>>(a, offlists);
    ++*n_launch;
  }
  const long long total = a.kc_total + a.qc_total;
  if (total > 0) {
    long long blocks = (total * 8 + 255) / 256;
    const long long cap = static_cast<long long>(num_sms) * 8;
    if (blocks > cap) blocks = cap;
    gather_rows_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(a, q, k, v, cache, offlists, kc, vc, qc, err);
    ++*n_launch;
  }
  return cudaGetLastError();
}

cudaError_t launch_plan_position(int n_items, int S, int gh, int gw, int ns, int N, int R, int cap, Seg* segs,
                                 int* counts, cudaStream_t stream) {
  plan_position_kernel<<<(n_items + 127) / 128, 128, 0, stream>>>(n_items, S, gh, gw, ns, N, R, cap, segs, counts);
  return cudaGetLastError();
}

cudaError_t launch_plan_corr(const int32_t* ranked, const int32_t* order, int kmax, int kt, int T, int N, int V,
                             int ns, int tail_len, Seg* segs, int cap, int* counts, int* err, cudaStream_t stream) {
  const int n_items = (T + 3) / 4;
  const size_t smem = sizeof(uint32_t) * T;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(plan_corr_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  plan_corr_kernel<<<n_items, 256, smem, stream>>>(ranked, order, kmax, kt, T, N, V, ns, tail_len, segs, cap,
                                                   counts, err);
  return cudaGetLastError();
}

constexpr int kNmseBlocks = 148;

size_t nmse_workspace_bytes(int H) { return static_cast<size_t>(H) * kNmseBlocks * 2 * sizeof(double); }

cudaError_t launch_nmse(const float* full, const float* sparse, int H, long long per_head, double* part,
                        double* out, cudaStream_t stream) {
  nmse_partial_kernel<<<dim3(kNmseBlocks, H), 256, 0, stream>>>(full, sparse, per_head, part);
  nmse_final_kernel<<<(H + 63) / 64, 64, 0, stream>>>(part, kNmseBlocks, H, out);
  return cudaGetLastError();
}

}  // namespace saf3r
