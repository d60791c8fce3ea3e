// Sparse / dense global attention over kept key runs, tcgen05 + TMA (sm_100a).
//
// Exact softmax attention restricted to each query's kept keys: SAF3R
// ("SAF3R: Dynamic Sparse Attention for Feed-Forward 3D Reconstruction
// Transformers"), section 4.1 - every query is kept, keys outside the head's
// set take no part in the softmax.
//
// One CTA per SM, persistent over work items.  A work item is 256 query rows
// of one head (two 128-row MMA tiles) plus the list of key runs ("segments")
// that cover the union of those rows' kept sets; keys that a given row does
// not keep are masked to -inf in its softmax.  Keys stream 128 per block as
// two 64-row halves, each a 2-D/3-D TMA tile load from the caller's K/V or
// from rows the prep kernels compacted into the workspace.
//
// Warp roles (12 warps, three warpgroups):
//   warp 0      TMA producer: Q tiles, then K and V blocks into a 4-stage ring
//   warp 1      MMA issuer (one thread): S_t = Q_t K^T and O_t += P_t V
//   warps 2-3   idle (their registers go to the softmax warpgroups)
//   warps 4-7   softmax of tile 0 (one thread per row; warp w reads TMEM lanes 32*(w%4)..+31)
//   warps 8-11  softmax of tile 1
// TMEM (512 columns): per tile t, S_t (128 fp32 cols), P_t (64 cols of packed
// bf16 pairs), O_t (64 fp32 cols).  The two softmax groups alternate with the
// tensor core: while group 0 turns S_0 into P_0, the tensor core runs group
// 1's products, and the other way round.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>

#include "internal.h"
#include "ptx.cuh"

namespace saf3r {

namespace {

constexpr int kThreads = 384;
constexpr int kStages = 4;
constexpr int kTileBytes = 128 * 64 * 2;  // 128 rows x 64 bf16
constexpr int kHalfBytes = 64 * 64 * 2;   // 64 rows x 64 bf16
constexpr float kScaleLog2 = 0.18033688011112042f;  // log2(e) / sqrt(64)
constexpr float kRescaleThreshold = 8.0f;           // log2 units: keep a stale max until it is 256x off

struct AttnSmem {
  uint8_t q[2][kTileBytes];
  uint8_t k[kStages][kTileBytes];
  uint8_t v[kStages][kTileBytes];
  uint64_t q_full, q_empty;
  uint64_t k_full[kStages], k_empty[kStages], v_full[kStages], v_empty[kStages];
  uint64_t s_full[2], s_free[2], p_full[2], o_done[2];
  uint32_t tmem_base;
  int abort;
};

// Iterates the 64-row half-blocks of one item's key runs.
struct Walker {
  const Seg* list;
  Seg implicit;
  int nseg;
  int idx;
  int off;

  __device__ __forceinline__ Seg seg_at(int i) const { return list ? list[i] : implicit; }

  // Next half-block: its run, offset of its first row inside the run, row count.
  __device__ __forceinline__ bool next(Seg& s, int& o, int& cnt) {
    while (idx < nseg) {
      Seg c = seg_at(idx);
      if (off < c.len) {
        s = c;
        o = off;
        cnt = min(64, c.len - off);
        off += 64;
        return true;
      }
      ++idx;
      off = 0;
    }
    return false;
  }
};

struct ItemInfo {
  int hi;      // index into p.heads
  int local;   // item index within the head
  int q0;      // first query row (head's Q row space)
  int nblk;    // 128-key blocks
  Walker w;
};

__device__ __forceinline__ ItemInfo item_info(const AttnParams& p, int item) {
  ItemInfo it;
  int hi = 0;
  while (hi + 1 < p.n_heads && item >= p.heads[hi].item_begin + p.heads[hi].n_items) ++hi;
  it.hi = hi;
  const HeadPlan& hp = p.heads[hi];
  it.local = item - hp.item_begin;
  it.q0 = it.local * kItemRows;
  it.w.idx = 0;
  it.w.off = 0;
  if (hp.seg_list < 0) {
    it.w.list = nullptr;
    it.w.implicit = hp.seg;
    it.w.nseg = 1;
  } else {
    it.w.list = p.segs + hp.seg_list + static_cast<long long>(it.local) * hp.seg_cap;
    it.w.implicit = hp.seg;
    it.w.nseg = p.seg_counts[hp.cnt_list + it.local];
  }
  int nhb = 0;
  for (int i = 0; i < it.w.nseg; ++i) nhb += (it.w.seg_at(i).len + 63) >> 6;
  it.nblk = (nhb + 1) >> 1;
  return it;
}

__device__ __forceinline__ uint64_t range_bits(int a, int b) {
  // bits [a, b) of a 64-bit word, 0 <= a <= b <= 64
  if (a >= b) return 0ull;
  const uint64_t hi = (b >= 64) ? ~0ull : ((1ull << b) - 1ull);
  const uint64_t lo = (a <= 0) ? 0ull : ((1ull << a) - 1ull);
  return hi & ~lo;
}

__device__ __forceinline__ void load_half(const AttnParams& p, const HeadPlan& hp, bool have, const Seg& s, int off,
                                          void* dst, const CUtensorMap* m3, const CUtensorMap* m2, uint64_t* bar) {
  if (!have) {
    // fully out-of-range box: TMA fills zeros (so a missing half contributes P = 0 times V = 0)
    tma_load_3d(dst, m3, 0, -64, hp.head, bar);
  } else if (s.src == 0) {
    tma_load_3d(dst, m3, 0, s.row0 + off, hp.head, bar);
  } else {
    tma_load_2d(dst, m2, 0, hp.kc_base + s.row0 + off, bar);
  }
}

__device__ __forceinline__ int position_token(const AttnParams& p, int i) {
  // cell-major query order: rows [0, P*S) are (cell, view), then the special tokens (view, slot)
  if (i < p.P * p.S) {
    const int cell = i / p.S, s = i - cell * p.S;
    return s * p.V + p.ns + cell;
  }
  const int sp = i - p.P * p.S;
  const int s = sp / p.ns;
  return s * p.V + (sp - s * p.ns);
}

}  // namespace

__device__ __forceinline__ void producer_role(const AttnParams& p, AttnSmem& sm, uint32_t tmem, int warp, int lane, const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmQC, const CUtensorMap& tmKC, const CUtensorMap& tmVC) {
  volatile int* abort = &sm.abort;
  const long long budget = p.wait_budget;
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      uint32_t k_issued = 0, v_issued = 0, q_issued = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < p.total_items; item += gridDim.x) {
        ItemInfo it = item_info(p, item);
        const HeadPlan& hp = p.heads[it.hi];
        if (q_issued > 0 && !mbar_wait(&sm.q_empty, (q_issued - 1) & 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT))
          break;
        mbar_arrive_expect_tx(&sm.q_full, 2 * kTileBytes);
        for (int t = 0; t < 2; ++t) {
          for (int half = 0; half < 2; ++half) {
            const int row = it.q0 + t * 128 + half * 64;
            void* dst = sm.q[t] + half * kHalfBytes;
            if (hp.q_src == 0)
              tma_load_3d(dst, &tmQ, 0, row, hp.head, &sm.q_full);
            else
              tma_load_2d(dst, &tmQC, 0, hp.q_base + row, &sm.q_full);
          }
        }
        ++q_issued;
        for (int b = 0; b < it.nblk; ++b) {
          Seg s0, s1;
          int o0 = 0, o1 = 0, c0 = 0, c1 = 0;
          const bool h0 = it.w.next(s0, o0, c0);
          const bool h1 = it.w.next(s1, o1, c1);
          const uint32_t stage = k_issued % kStages, ph = (k_issued / kStages) & 1;
          if (k_issued >= kStages &&
              !mbar_wait(&sm.k_empty[stage], ph ^ 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.k_full[stage], kTileBytes);
          load_half(p, hp, h0, s0, o0, sm.k[stage], &tmK, &tmKC, &sm.k_full[stage]);
          load_half(p, hp, h1, s1, o1, sm.k[stage] + kHalfBytes, &tmK, &tmKC, &sm.k_full[stage]);
          ++k_issued;
          if (v_issued >= kStages &&
              !mbar_wait(&sm.v_empty[stage], ph ^ 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.v_full[stage], kTileBytes);
          load_half(p, hp, h0, s0, o0, sm.v[stage], &tmV, &tmVC, &sm.v_full[stage]);
          load_half(p, hp, h1, s1, o1, sm.v[stage] + kHalfBytes, &tmV, &tmVC, &sm.v_full[stage]);
          ++v_issued;
        }
      }
      // Teardown: every copy this thread issued must have landed before the CTA exits
      // (these waits ignore the abort flag but stay bounded).
      const long long drain = budget / 4;
      if (q_issued > 0) mbar_wait_drain(&sm.q_full, (q_issued - 1) & 1, drain);
      for (uint32_t c = (k_issued > kStages ? k_issued - kStages : 0); c < k_issued; ++c)
        mbar_wait_drain(&sm.k_full[c % kStages], (c / kStages) & 1, drain);
      for (uint32_t c = (v_issued > kStages ? v_issued - kStages : 0); c < v_issued; ++c)
        mbar_wait_drain(&sm.v_full[c % kStages], (c / kStages) & 1, drain);
    }
}

__device__ __forceinline__ void mma_role(const AttnParams& p, AttnSmem& sm, uint32_t tmem, int warp, int lane, const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmQC, const CUtensorMap& tmKC, const CUtensorMap& tmVC) {
  volatile int* abort = &sm.abort;
  const long long budget = p.wait_budget;
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 64, 0, 1);
      uint32_t kv_c = 0, items = 0;
      uint32_t sfree_c[2] = {0, 0}, pfull_c[2] = {0, 0}, qk_done[2] = {0, 0};
      const uint32_t qaddr[2] = {smem_u32(sm.q[0]), smem_u32(sm.q[1])};
      bool ok = true;

      auto issue_qk = [&](int t, uint32_t stage) -> bool {
        if (qk_done[t] > 0) {
          if (!mbar_wait(&sm.s_free[t], sfree_c[t] & 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT)) return false;
          ++sfree_c[t];
          tc_fence_after();
        }
        const uint32_t kaddr = smem_u32(sm.k[stage]);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t da = smem_desc_sw128(qaddr[t] + kk * 32, 16, 1024);
          const uint64_t db = smem_desc_sw128(kaddr + kk * 32, 16, 1024);
          mma_ss(tmem + t * 256, da, db, idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(&sm.s_full[t]);
        ++qk_done[t];
        return true;
      };

      for (int item = blockIdx.x; ok && item < p.total_items; item += gridDim.x) {
        ItemInfo it = item_info(p, item);
        if (!mbar_wait(&sm.q_full, items & 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT)) break;
        tc_fence_after();
        {
          const uint32_t stage = kv_c % kStages, ph = (kv_c / kStages) & 1;
          if (!mbar_wait(&sm.k_full[stage], ph, abort, p.err, budget, SAF3R_ERR_TIMEOUT)) break;
          tc_fence_after();
          if (!issue_qk(0, stage) || !issue_qk(1, stage)) break;
          mma_commit(&sm.k_empty[stage]);
          if (it.nblk == 1) mma_commit(&sm.q_empty);
        }
        for (int j = 0; ok && j < it.nblk; ++j) {
          const uint32_t c = kv_c + j;
          const uint32_t cs = c % kStages, cph = (c / kStages) & 1;
          const bool has_next = j + 1 < it.nblk;
          const uint32_t ns = (c + 1) % kStages, nph = ((c + 1) / kStages) & 1;
          if (has_next && !mbar_wait(&sm.k_full[ns], nph, abort, p.err, budget, SAF3R_ERR_TIMEOUT)) {
            ok = false;
            break;
          }
          if (!mbar_wait(&sm.v_full[cs], cph, abort, p.err, budget, SAF3R_ERR_TIMEOUT)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t vaddr = smem_u32(sm.v[cs]);
          for (int t = 0; t < 2; ++t) {
            if (!mbar_wait(&sm.p_full[t], pfull_c[t] & 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT)) {
              ok = false;
              break;
            }
            ++pfull_c[t];
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t db = smem_desc_sw128(vaddr + kk * 2048, 8192, 1024);
              mma_ts(tmem + t * 256 + 192, tmem + t * 256 + 128 + kk * 8, db, idesc_pv,
                     (j > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&sm.o_done[t]);
            if (has_next && !issue_qk(t, ns)) {
              ok = false;
              break;
            }
          }
          if (!ok) break;
          mma_commit(&sm.v_empty[cs]);
          if (has_next) {
            mma_commit(&sm.k_empty[ns]);
            if (j + 2 == it.nblk) mma_commit(&sm.q_empty);
          }
        }
        kv_c += it.nblk;
        ++items;
      }
    }
}

__device__ __forceinline__ void softmax_role(const AttnParams& p, AttnSmem& sm, uint32_t tmem, int warp, int lane, const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmQC, const CUtensorMap& tmKC, const CUtensorMap& tmVC) {
  volatile int* abort = &sm.abort;
  const long long budget = p.wait_budget;
    const int t = (warp - 4) >> 2;
    const int wq = warp & 3;
    const int r = wq * 32 + lane;               // row inside the 128-row tile
    const int quarter = (t * 128 + r) >> 6;     // 64-row quarter of the 256-row item
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + t * 256;
    const uint32_t tP = tS + 128;
    const uint32_t tO = tS + 192;
    uint32_t sfull_c = 0, odone_c = 0;
    bool ok = true;

    for (int item = blockIdx.x; ok && item < p.total_items; item += gridDim.x) {
      ItemInfo it = item_info(p, item);
      const HeadPlan& hp = p.heads[it.hi];
      const int qrow = it.q0 + t * 128 + r;

      // per-row neighbourhood intervals (position heads): kept derived rows [lo, hi)
      int nb_lo[2 * kMaxRadius + 1], nb_hi[2 * kMaxRadius + 1];
      {
        const bool patch_row = hp.kind == SAF3R_POSITION && qrow < p.P * p.S && p.S > 1;
        const int cell = patch_row ? qrow / p.S : 0;
        const int qr = cell / p.gw, qc = cell - qr * p.gw;
        const int R = hp.radius;
#pragma unroll
        for (int x = 0; x < 2 * kMaxRadius + 1; ++x) {
          const int dr = x - kMaxRadius;
          const int rr = qr + dr;
          const bool use = patch_row && dr >= -R && dr <= R && rr >= 0 && rr < p.gh;
          const int ca = rr * p.gw + max(qc - R, 0);
          const int cb = rr * p.gw + min(qc + R, p.gw - 1);
          nb_lo[x] = use ? hp.nb_base + ca * (p.S - 1) : 0;
          nb_hi[x] = use ? hp.nb_base + (cb + 1) * (p.S - 1) : 0;
        }
      }

      float m = -INFINITY;  // running max, log2 units
      float l = 0.f;        // running row sum
      for (int j = 0; j < it.nblk; ++j) {
        // kept-key masks of the two halves of this block
        uint64_t valid[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          Seg s;
          int o = 0, cnt = 0;
          valid[h] = 0ull;
          if (it.w.next(s, o, cnt) && ((s.flags >> quarter) & 1u)) {
            uint64_t v = range_bits(0, cnt);
            const int lo = (s.flags >> 8) & 0xFF, hi = (s.flags >> 16) & 0xFF;
            if (hi > lo) v &= ~range_bits(max(lo - o, 0), min(hi - o, 64));
            if (s.flags & kSegCellMask) {
              const int base = s.row0 + o;
              uint64_t nb = 0ull;
#pragma unroll
              for (int x = 0; x < 2 * kMaxRadius + 1; ++x)
                nb |= range_bits(max(nb_lo[x] - base, 0), min(nb_hi[x] - base, cnt));
              v &= nb;
            }
            valid[h] = v;
          }
        }

        if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[t], sfull_c & 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT))) {
          ok = false;
          break;
        }
        ++sfull_c;
        tc_fence_after();
        float s[128];
        {
          uint32_t raw[32];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            tmem_ld32(tS + c * 32, raw);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(raw[i]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.s_free[t]);

#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (valid[h] != ~0ull) {
#pragma unroll
            for (int i = 0; i < 64; ++i)
              if (!((valid[h] >> i) & 1ull)) s[h * 64 + i] = -INFINITY;
          }
        }
        float mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < 128; ++i) mx = fmaxf(mx, s[i]);
        mx *= kScaleLog2;
        float alpha = 1.f;
        bool rescale = false;
        if (j == 0) {
          m = mx;
        } else if (mx > m + kRescaleThreshold) {
          alpha = fast_exp2(m - mx);  // m may be -inf: alpha = 0
          m = mx;
          rescale = true;
        }
        const float m_use = (m == -INFINITY) ? 0.f : m;
        uint32_t pk[64];
        float rs = 0.f;
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const float e0 = fast_exp2(fmaf(s[2 * i], kScaleLog2, -m_use));
          const float e1 = fast_exp2(fmaf(s[2 * i + 1], kScaleLog2, -m_use));
          rs += e0 + e1;
          pk[i] = pack_bf16x2(e0, e1);
        }
        l = l * alpha + rs;

        if (j > 0) {
          if (!__all_sync(0xffffffffu, mbar_wait(&sm.o_done[t], odone_c & 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT))) {
            ok = false;
            break;
          }
          ++odone_c;
          tc_fence_after();
          if (__any_sync(0xffffffffu, rescale)) {
            uint32_t o[32];
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              tmem_ld32(tO + c * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st32(tO + c * 32, o);
            }
          }
        }
        {
          uint32_t half[32];
#pragma unroll
          for (int c = 0; c < 2; ++c) {
#pragma unroll
            for (int i = 0; i < 32; ++i) half[i] = pk[c * 32 + i];
            tmem_st32(tP + c * 32, half);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full[t]);
      }
      if (!ok) break;

      // epilogue: O / l of this row
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.o_done[t], odone_c & 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT))) {
        ok = false;
        break;
      }
      ++odone_c;
      tc_fence_after();
      float o[64];
      {
        uint32_t raw[32];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          tmem_ld32(tO + c * 32, raw);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[c * 32 + i] = __uint_as_float(raw[i]);
        }
      }
      tc_fence_before();
      if (qrow < p.N) {
        const int token = (hp.q_src == 1) ? position_token(p, qrow) : qrow;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const long long rowoff = (static_cast<long long>(hp.head) * p.N + token) * kD;
        if (p.out_fp32) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + rowoff);
#pragma unroll
          for (int i = 0; i < 16; ++i)
            dst[i] = make_float4(o[4 * i] * inv, o[4 * i + 1] * inv, o[4 * i + 2] * inv, o[4 * i + 3] * inv);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + rowoff);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_uint4(pack_bf16x2(o[8 * i] * inv, o[8 * i + 1] * inv),
                                pack_bf16x2(o[8 * i + 2] * inv, o[8 * i + 3] * inv),
                                pack_bf16x2(o[8 * i + 4] * inv, o[8 * i + 5] * inv),
                                pack_bf16x2(o[8 * i + 6] * inv, o[8 * i + 7] * inv));
        }
      }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_sm100_kernel(const __grid_constant__ AttnParams p, const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmQC, const __grid_constant__ CUtensorMap tmKC,
                      const __grid_constant__ CUtensorMap tmVC) {
  extern __shared__ uint8_t smem_raw[];
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (p.ok_flag != nullptr && *p.ok_flag == 0) return;  // cache check failed: leave `out` untouched

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&sm.s_full[t], 1);
      mbar_init(&sm.s_free[t], 4);
      mbar_init(&sm.p_full[t], 4);
      mbar_init(&sm.o_done[t], 1);
    }
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

  if (warp < 4) reg_dealloc_dec<104>();  // 104*128 + 200*256 = 168*384 registers
  if (warp == 0) {
    producer_role(p, sm, tmem, warp, lane, tmQ, tmK, tmV, tmQC, tmKC, tmVC);
    __syncwarp();
  } else if (warp == 1) {
    mma_role(p, sm, tmem, warp, lane, tmQ, tmK, tmV, tmQC, tmKC, tmVC);
    __syncwarp();
  } else if (warp >= 4) {
    reg_alloc_inc<200>();
    softmax_role(p, sm, tmem, warp, lane, tmQ, tmK, tmV, tmQC, tmKC, tmVC);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

size_t attn_smem_bytes() { return sizeof(AttnSmem) + 1024; }

cudaError_t launch_attention(const AttnParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                             const CUtensorMap& tmV, const CUtensorMap& tmQC, const CUtensorMap& tmKC,
                             const CUtensorMap& tmVC, int num_sms, cudaStream_t stream) {
  const size_t smem = attn_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(attn_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int grid = p.total_items < num_sms ? p.total_items : num_sms;
  if (grid <= 0) return cudaSuccess;
  attn_sm100_kernel<<<grid, kThreads, smem, stream>>>(p, tmQ, tmK, tmV, tmQC, tmKC, tmVC);
  return cudaGetLastError();
}

}  // namespace saf3r
