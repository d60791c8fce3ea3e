// Attention of token-wise correspondence heads: every query row keeps its own keys.
//
// SAF3R ("SAF3R: Dynamic Sparse Attention for Feed-Forward 3D Reconstruction Transformers"),
// section 4.1, "DINO Top-K Kernel": a patch query keeps, in every frame, the Top-K patch tokens
// most similar to it in DINO features (section 5.1: K per frame), here plus every special
// token; a special-token query has no DINO feature and keeps every key.  Exact softmax over the
// kept keys (logit -inf elsewhere), scale 1/sqrt(64).
//
// No two query rows share a key set, so there is no dense block for the tensor cores: one warp
// per query row, split into 8 groups of 4 lanes; a group takes every 8th kept key, each lane
// of it 16 of the 64 features (a 128-byte K row and V row gathered from L2 by one group in one
// coalesced access each).  A group keeps its own running max, sum and accumulator in fp32; the
// 8 group states are merged at the end and the warp stores the row with one coalesced access.
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

__device__ __forceinline__ int special_tok(int r, int V, int ns) {
  const int s = r / ns;
  return s * V + (r - s * ns);
}

}  // namespace

__global__ void __launch_bounds__(256) token_attn_kernel(const TokenAttnParams p) {
  if (p.ok_flag != nullptr && *p.ok_flag == 0) return;  // cache check failed: leave `out` untouched
  const int lane = threadIdx.x & 31;
  const int grp = lane >> 2, sub = lane & 3;            // key group, feature quarter [16*sub, 16*sub+16)
  const unsigned gmask = 0xFu << (grp * 4);
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  const long long total = static_cast<long long>(p.n_heads) * p.N;
  const int nsp = p.ns * p.S;
  for (long long task = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; task < total;
       task += warps) {
    const int hi = static_cast<int>(task / p.N);
    const int i = static_cast<int>(task - static_cast<long long>(hi) * p.N);
    const int h = p.heads[hi], kf = p.k[hi];  // kf: per-frame budget of this head
    const size_t hb = static_cast<size_t>(h) * p.N * kD;
    const int s_i = i / p.V, loc = i - s_i * p.V;
    const bool special = loc < p.ns;
    const int nk = special ? p.N : p.S * kf + nsp;
    const int32_t* lists =
        special ? nullptr
                : p.cache + p.tok_off + (static_cast<size_t>(s_i) * p.P + (loc - p.ns)) * p.S * p.tok_kmax;
    float qv[16];
    load16(p.q + hb + static_cast<size_t>(i) * kD + 16 * sub, qv);
    float m = -INFINITY, l = 0.f;
    float o[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) o[c] = 0.f;
    for (int n = grp; n < nk; n += 8) {
      int tok;
      if (special) {
        tok = n;
      } else if (n < p.S * kf) {
        const int s = n / kf, r = n - s * kf;
        int pp = lists[s * p.tok_kmax + r];
        if (pp < 0 || pp >= p.P) {
          atomicCAS(p.err, 0, SAF3R_ERR_INDEX);
          pp = 0;  // keep the group converged; the error word reports the bad index
        }
        tok = s * p.V + p.ns + pp;
      } else {
        tok = special_tok(n - p.S * kf, p.V, p.ns);
      }
      float kv[16];
      load16(p.k_ + hb + static_cast<size_t>(tok) * kD + 16 * sub, kv);
      float d0 = 0.f, d1 = 0.f;
#pragma unroll
      for (int c = 0; c < 16; c += 2) {
        d0 = fmaf(qv[c], kv[c], d0);
        d1 = fmaf(qv[c + 1], kv[c + 1], d1);
      }
      float d = d0 + d1;
      d += __shfl_xor_sync(gmask, d, 1);
      d += __shfl_xor_sync(gmask, d, 2);
      const float x = d * kLog2eOver8;
      if (x > m + kThresh || m == -INFINITY) {
        const float alpha = m == -INFINITY ? 0.f : fast_exp2(m - x);
        l *= alpha;
#pragma unroll
        for (int c = 0; c < 16; ++c) o[c] *= alpha;
        m = x;
      }
      const float pw = fast_exp2(x - m);
      l += pw;
      load16(p.v + hb + static_cast<size_t>(tok) * kD + 16 * sub, kv);
#pragma unroll
      for (int c = 0; c < 16; ++c) o[c] = fmaf(pw, kv[c], o[c]);
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
    const float inv = l > 0.f ? 1.f / l : 0.f;
    float y0 = o[0], y1 = o[1];
#pragma unroll
    for (int g = 1; g < 8; ++g)
      if (grp == g) {
        y0 = o[2 * g];
        y1 = o[2 * g + 1];
      }
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
