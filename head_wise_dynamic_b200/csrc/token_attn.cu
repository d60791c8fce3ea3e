// Attention of the patch queries of token-wise correspondence heads: every such query row keeps
// its own keys.
//
// SAF3R ("SAF3R: Dynamic Sparse Attention for Feed-Forward 3D Reconstruction Transformers"),
// section 4.1, "DINO Top-K Kernel": a patch query keeps, in every frame, the Top-K patch tokens
// most similar to it in DINO features (section 5.1: K per frame), here plus every special
// token.  Exact softmax over the kept keys (logit -inf elsewhere), scale 1/sqrt(64).  (A
// special-token query has no DINO feature and keeps every key: those rows are dense and run in
// the tensor-core attention kernel.)
//
// This kernel takes the patch queries of the token-wise heads that do not run in the tensor-core
// kernel (a layout the union builder does not fit, or more plans than the plan array holds).
// Each row walks its own keys: one warp per query row, split into 8 groups of 4 lanes; a group takes kept keys n, n + 8 together
// (every 16th pair), each lane of it 16 of the 64 features (a 128-byte K row and V row gathered
// from L2 by one group in one coalesced access each; both keys' K and V rows are requested
// before any of them is used).  A group keeps its own running max, sum and accumulator in fp32;
// the 8 group states are merged at the end and the warp stores the row with one coalesced access.
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "ptx.cuh"

namespace saf3r {

namespace {

constexpr float kLog2eOver8 = 0.18033688011112042f;  // log2(e) / sqrt(64)
constexpr float kThresh = 8.0f;                        // keep a stale max until it is 2^8 off

// 16 consecutive bf16 features (32 bytes) as fp32.
__device__ __forceinline__ void load16(const uint16_t* p, float (&x)[16]) {
  const uint4* r = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const uint4 w = r[c];
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[8 * c + 2 * i] = __uint_as_float(u[i] << 16);
      x[8 * c + 2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
    }
  }
}

// n / d and n % d for a divisor fixed per row: one multiply-high by m = ceil(2^32 / d) (exact for
// n < 2^32 / d, which holds for every key rank here; one correction step covers the rest), the
// divisor 1 on its own path.
struct Divider {
  uint32_t d, m;
  __device__ explicit Divider(uint32_t dd) : d(dd), m(dd > 1u ? 0xFFFFFFFFu / dd + 1u : 0u) {}
  __device__ __forceinline__ uint32_t div(uint32_t n, uint32_t& r) const {
    if (d == 1u) {
      r = 0u;
      return n;
    }
    uint32_t q = __umulhi(n, m);
    int rr = static_cast<int>(n - q * d);
    if (rr < 0) {
      --q;
      rr += static_cast<int>(d);
    } else if (rr >= static_cast<int>(d)) {
      ++q;
      rr -= static_cast<int>(d);
    }
    r = static_cast<uint32_t>(rr);
    return q;
  }
};

// Token of kept key n of a patch query: ranks n < nl come from the per-frame lists (frame n / kf),
// the rest are the special tokens (view by view).  An out-of-range list entry is recorded in the
// error word and read as patch 0 (the group stays converged).
__device__ __forceinline__ int key_token(const TokenAttnParams& p, const int32_t* lists, int n, int nl,
                                         const Divider& by_kf, const Divider& by_ns) {
  uint32_t r;
  if (n >= nl) {
    const uint32_t s = by_ns.div(static_cast<uint32_t>(n - nl), r);
    return static_cast<int>(s) * p.V + static_cast<int>(r);
  }
  const uint32_t s = by_kf.div(static_cast<uint32_t>(n), r);
  int pp = lists[static_cast<int>(s) * p.tok_kmax + static_cast<int>(r)];
  if (pp < 0 || pp >= p.P) {
    atomicCAS(p.err, 0, SAF3R_ERR_INDEX);
    pp = 0;
  }
  return static_cast<int>(s) * p.V + p.ns + pp;
}

}  // namespace

// Four blocks per SM (64 registers; a few spill): more warps to hide the gathers' L2 latency
// measured faster than three blocks at 80 registers without spills (S=32 token layer 4.39-4.52 vs
// 4.58-4.68 ms).
__global__ void __launch_bounds__(256, 4) token_attn_kernel(const TokenAttnParams p) {
  if (p.ok_flag != nullptr && *p.ok_flag == 0) return;  // cache check failed: leave `out` untouched
  const int lane = threadIdx.x & 31;
  const int grp = lane >> 2, sub = lane & 3;            // key group, feature quarter [16*sub, 16*sub+16)
  const unsigned gmask = 0xFu << (grp * 4);
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  const int R = p.S * p.P;  // patch query rows of a head (its special rows run in the tensor-core kernel)
  const long long total = static_cast<long long>(p.n_heads) * R;
  const int nsp = p.ns * p.S;
  for (long long task = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; task < total;
       task += warps) {
    const int hi = static_cast<int>(task / R);
    const int a = static_cast<int>(task - static_cast<long long>(hi) * R);  // patch row a = s*P + patch
    const int i = (a / p.P) * p.V + p.ns + (a % p.P);
    const int h = p.heads[hi], kf = p.k[hi];  // kf: per-frame budget of this head
    const Divider by_kf(static_cast<uint32_t>(kf)), by_ns(static_cast<uint32_t>(p.ns > 0 ? p.ns : 1));
    const size_t hb = static_cast<size_t>(h) * p.N * kD;
    const int nl = p.S * kf;  // ranked keys; the special tokens follow
    const int nk = nl + nsp;
    const int32_t* lists = p.cache + p.tok_off + static_cast<size_t>(a) * p.S * p.tok_kmax;
    float qv[16];
    load16(p.q + hb + static_cast<size_t>(i) * kD + 16 * sub, qv);
    float m = -INFINITY, l = 0.f;
    float o[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) o[c] = 0.f;
    for (int n = grp; n < nk; n += 16) {
      const bool two = n + 8 < nk;
      const int tok0 = key_token(p, lists, n, nl, by_kf, by_ns);
      const int tok1 = two ? key_token(p, lists, n + 8, nl, by_kf, by_ns) : tok0;
      float k0[16], k1[16], v0[16], v1[16];
      load16(p.k_ + hb + static_cast<size_t>(tok0) * kD + 16 * sub, k0);
      load16(p.k_ + hb + static_cast<size_t>(tok1) * kD + 16 * sub, k1);
      load16(p.v + hb + static_cast<size_t>(tok0) * kD + 16 * sub, v0);
      load16(p.v + hb + static_cast<size_t>(tok1) * kD + 16 * sub, v1);
      float d0 = 0.f, d1 = 0.f, e0 = 0.f, e1 = 0.f;
#pragma unroll
      for (int c = 0; c < 16; c += 2) {
        d0 = fmaf(qv[c], k0[c], d0);
        d1 = fmaf(qv[c + 1], k0[c + 1], d1);
        e0 = fmaf(qv[c], k1[c], e0);
        e1 = fmaf(qv[c + 1], k1[c + 1], e1);
      }
      float x0 = d0 + d1, x1 = e0 + e1;
      x0 += __shfl_xor_sync(gmask, x0, 1);
      x1 += __shfl_xor_sync(gmask, x1, 1);
      x0 += __shfl_xor_sync(gmask, x0, 2);
      x1 += __shfl_xor_sync(gmask, x1, 2);
      x0 *= kLog2eOver8;
      x1 = two ? x1 * kLog2eOver8 : -INFINITY;
      const float xm = fmaxf(x0, x1);
      if (xm > m + kThresh || m == -INFINITY) {
        const float alpha = m == -INFINITY ? 0.f : fast_exp2(m - xm);
        l *= alpha;
#pragma unroll
        for (int c = 0; c < 16; ++c) o[c] *= alpha;
        m = xm;
      }
      const float w0 = fast_exp2(x0 - m), w1 = fast_exp2(x1 - m);
      l += w0 + w1;
#pragma unroll
      for (int c = 0; c < 16; ++c) o[c] = fmaf(w1, v1[c], fmaf(w0, v0[c], o[c]));
    }
    // merge the 8 group states (lanes of one feature quarter: xor over lane bits 2..4)
    float mm = m;
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) mm = fmaxf(mm, __shfl_xor_sync(0xffffffffu, mm, off));
    const float f = (m == -INFINITY) ? 0.f : fast_exp2(m - mm);
    l *= f;
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      o[c] *= f;
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) o[c] += __shfl_xor_sync(0xffffffffu, o[c], off);
    }
    // every group now holds the row; group g stores features 16*sub + 2g, +1
    float y0 = o[0], y1 = o[1];
#pragma unroll
    for (int g = 1; g < 8; ++g)
      if (grp == g) {
        y0 = o[2 * g];
        y1 = o[2 * g + 1];
      }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    y0 *= inv;
    y1 *= inv;
    const size_t orow = hb + static_cast<size_t>(i) * kD + 16 * sub + 2 * grp;
    if (p.out_fp32) {
      reinterpret_cast<float2*>(static_cast<float*>(p.out) + orow)[0] = make_float2(y0, y1);
    } else {
      reinterpret_cast<uint32_t*>(static_cast<uint16_t*>(p.out) + orow)[0] = pack_bf16x2(y0, y1);
    }
  }
}

cudaError_t launch_token_attention(const TokenAttnParams& p, int num_sms, cudaStream_t stream) {
  if (p.n_heads <= 0) return cudaSuccess;
  token_attn_kernel<<<num_sms * 8, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace saf3r
