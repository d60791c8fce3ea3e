// Sparse / dense global attention over kept key runs, tcgen05 + TMA (sm_100a).
//
// Exact softmax attention restricted to each query's kept keys: SAF3R
// ("SAF3R: Dynamic Sparse Attention for Feed-Forward 3D Reconstruction
// Transformers"), section 4.1 - every query is kept, keys outside the head's
// set take no part in the softmax (logit -inf).
//
// One CTA per SM, persistent over work items.  A work item is 256 query rows
// of one head (two 128-row MMA tiles, four 64-row quarters) plus the list of
// key runs ("segments") that cover the union of those rows' kept sets.  Keys
// stream 128 per block as two 64-row halves, each one TMA tile load from the
// caller's K/V or from rows the prep kernels compacted into the workspace.
// Keys a row does not keep (another quarter's tile, a special token already
// counted, a cell outside its neighbourhood, the ragged end of a run) are
// masked to -inf in its softmax.
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

// One 64-row half-block of keys.
struct Half {
  bool have;
  Seg s;
  int off;  // first row inside the run
  int cnt;  // rows (<= 64)
};

// Iterates the 64-row half-blocks of one item's key runs.
struct Walker {
  const Seg* list;
  Seg implicit;
  int nseg;
  int idx;
  int off;

  __device__ __forceinline__ Seg seg_at(int i) const { return list ? list[i] : implicit; }

  __device__ __forceinline__ Half next() {
    Half h;
    h.have = false;
    while (idx < nseg) {
      const Seg c = seg_at(idx);
      if (off < c.len) {
        h.have = true;
        h.s = c;
        h.off = off;
        h.cnt = min(64, c.len - off);
        off += 64;
        return h;
      }
      ++idx;
      off = 0;
    }
    return h;
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
  it.w.implicit = hp.seg;
  if (hp.seg_list < 0) {
    it.w.list = nullptr;
    it.w.nseg = 1;
  } else {
    it.w.list = p.segs + hp.seg_list + static_cast<long long>(it.local) * hp.seg_cap;
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

__device__ __forceinline__ void load_half(const HeadPlan& hp, const Half& h, void* dst, const CUtensorMap* m3,
                                          const CUtensorMap* m2, uint64_t* bar) {
  if (h.s.src == 0)
    tma_load_3d(dst, m3, 0, h.s.row0 + h.off, hp.head, bar);
  else
    tma_load_2d(dst, m2, 0, hp.kc_base + h.s.row0 + h.off, bar);
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

// Query tile of quarter `quarter` of a tile-mapped item, or -1 past the last tile.
__device__ __forceinline__ int mapped_tile(const AttnParams& p, const HeadPlan& hp, int local, int quarter) {
  const int i = 4 * local + quarter;
  return i < p.T ? p.qmap[hp.q_base + i] : -1;
}

// ------------------------------------------------------------------ TMA producer (one thread)
__device__ __forceinline__ void producer_role(const AttnParams& p, AttnSmem& sm, const CUtensorMap& tmQ,
                                              const CUtensorMap& tmK, const CUtensorMap& tmV,
                                              const CUtensorMap& tmQC, const CUtensorMap& tmKC,
                                              const CUtensorMap& tmVC) {
  volatile int* abort = &sm.abort;
  const long long budget = p.wait_budget;
  tma_prefetch_desc(&tmQ);
  tma_prefetch_desc(&tmK);
  tma_prefetch_desc(&tmV);
  uint32_t k_issued = 0, v_issued = 0, q_issued = 0;
  bool ok = true;
  for (int item = blockIdx.x; ok && item < p.total_items; item += gridDim.x) {
    ItemInfo it = item_info(p, item);
    const HeadPlan& hp = p.heads[it.hi];
    if (q_issued > 0 && !mbar_wait(&sm.q_empty, (q_issued - 1) & 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT)) break;
    mbar_arrive_expect_tx(&sm.q_full, 2 * kTileBytes);
    for (int quarter = 0; quarter < 4; ++quarter) {
      void* dst = sm.q[quarter >> 1] + (quarter & 1) * kHalfBytes;
      if (hp.q_src == 1) {
        tma_load_2d(dst, &tmQC, 0, hp.q_base + it.q0 + quarter * 64, &sm.q_full);
      } else {
        int row = it.q0 + quarter * 64;
        if (hp.q_src == 2) {
          const int u = mapped_tile(p, hp, it.local, quarter);
          row = u >= 0 ? u * 64 : -64;  // past the last tile: an all-zero box
        }
        tma_load_3d(dst, &tmQ, 0, row, hp.head, &sm.q_full);
      }
    }
    ++q_issued;
    for (int b = 0; b < it.nblk; ++b) {
      const Half h0 = it.w.next();
      const Half h1 = it.w.next();
      const uint32_t stage = k_issued % kStages, ph = (k_issued / kStages) & 1;
      if (k_issued >= kStages && !mbar_wait(&sm.k_empty[stage], ph ^ 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT)) {
        ok = false;
        break;
      }
      mbar_arrive_expect_tx(&sm.k_full[stage], kTileBytes);
      if (h0.have) load_half(hp, h0, sm.k[stage], &tmK, &tmKC, &sm.k_full[stage]); else tma_load_3d(sm.k[stage], &tmK, 0, -64, hp.head, &sm.k_full[stage]);
      if (h1.have) load_half(hp, h1, sm.k[stage] + kHalfBytes, &tmK, &tmKC, &sm.k_full[stage]); else tma_load_3d(sm.k[stage] + kHalfBytes, &tmK, 0, -64, hp.head, &sm.k_full[stage]);
      ++k_issued;
      if (v_issued >= kStages && !mbar_wait(&sm.v_empty[stage], ph ^ 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT)) {
        ok = false;
        break;
      }
      mbar_arrive_expect_tx(&sm.v_full[stage], kTileBytes);
      if (h0.have) load_half(hp, h0, sm.v[stage], &tmV, &tmVC, &sm.v_full[stage]); else tma_load_3d(sm.v[stage], &tmV, 0, -64, hp.head, &sm.v_full[stage]);
      if (h1.have) load_half(hp, h1, sm.v[stage] + kHalfBytes, &tmV, &tmVC, &sm.v_full[stage]); else tma_load_3d(sm.v[stage] + kHalfBytes, &tmV, 0, -64, hp.head, &sm.v_full[stage]);
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

// ------------------------------------------------------------------ MMA issuer (one thread)
//
// For each key block and each tile in turn: O_t += P_t V once softmax t has written P_t,
// then S_t = Q_t K^T of the next block.  The two softmax groups so alternate with the
// tensor core: while group t computes, the tensor core runs the other tile's products.
// This thread sits on that critical path, so it does nothing but wait, add descriptor
// offsets and issue: every product covers the whole 128-key block (keys a row does not
// keep are masked in its softmax and get P = 0).
struct MmaState {
  uint32_t sfree_c[2] = {0, 0};
  uint32_t pfull_c[2] = {0, 0};
  uint32_t qk_done[2] = {0, 0};
};

// Shared-memory descriptors of the operand tiles, computed once: a K-step of 16 keys or 16
// features is then one 64-bit add (the start address sits in the low bits, in 16-byte units).
struct Descs {
  uint64_t q[2];  // Q tiles (K-major, 128-byte swizzle)
  uint64_t k0;    // K stage 0 (K-major); stage s adds s * kTileBytes / 16
  uint64_t v0;    // V stage 0 (MN-major); stage s adds s * kTileBytes / 16
};
constexpr uint64_t kStageDesc = kTileBytes >> 4;

// S_t = Q_t K^T for one 128-key block; commits s_full[t].
__device__ __forceinline__ bool issue_qk(const AttnParams& p, AttnSmem& sm, MmaState& st, const Descs& d,
                                         uint32_t tmem, int t, uint32_t stage) {
  if (st.qk_done[t] > 0) {
    if (!mbar_wait(&sm.s_free[t], st.sfree_c[t] & 1, &sm.abort, p.err, p.wait_budget, SAF3R_ERR_TIMEOUT))
      return false;
    ++st.sfree_c[t];
    tc_fence_after();
  }
  constexpr uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
  const uint64_t dq = d.q[t];
  const uint64_t dk = d.k0 + stage * kStageDesc;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) mma_ss(tmem + t * 256, dq + 2 * kk, dk + 2 * kk, idesc, kk > 0 ? 1u : 0u);
  mma_commit(&sm.s_full[t]);
  ++st.qk_done[t];
  return true;
}

__device__ __forceinline__ void mma_role(const AttnParams& p, AttnSmem& sm, uint32_t tmem) {
  volatile int* abort = &sm.abort;
  const long long budget = p.wait_budget;
  constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 64, 0, 1);
  Descs d;
  d.q[0] = smem_desc_sw128(smem_u32(sm.q[0]), 16, 1024);
  d.q[1] = smem_desc_sw128(smem_u32(sm.q[1]), 16, 1024);
  d.k0 = smem_desc_sw128(smem_u32(sm.k[0]), 16, 1024);
  d.v0 = smem_desc_sw128(smem_u32(sm.v[0]), 8192, 1024);
  MmaState st;
  uint32_t kv_c = 0, items = 0;
  bool ok = true;
  for (int item = blockIdx.x; ok && item < p.total_items; item += gridDim.x) {
    const int nblk = item_info(p, item).nblk;
    if (!mbar_wait(&sm.q_full, items & 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT)) break;
    tc_fence_after();
    {
      const uint32_t stage = kv_c % kStages, ph = (kv_c / kStages) & 1;
      if (!mbar_wait(&sm.k_full[stage], ph, abort, p.err, budget, SAF3R_ERR_TIMEOUT)) break;
      tc_fence_after();
      if (!issue_qk(p, sm, st, d, tmem, 0, stage) || !issue_qk(p, sm, st, d, tmem, 1, stage)) break;
      mma_commit(&sm.k_empty[stage]);
      if (nblk == 1) mma_commit(&sm.q_empty);
    }
    for (int j = 0; ok && j < nblk; ++j) {
      const uint32_t c = kv_c + j;
      const uint32_t cs = c % kStages, cph = (c / kStages) & 1;
      const bool has_next = j + 1 < nblk;
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
      const uint64_t dv = d.v0 + cs * kStageDesc;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (!mbar_wait(&sm.p_full[t], st.pfull_c[t] & 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT)) {
          ok = false;
          break;
        }
        ++st.pfull_c[t];
        tc_fence_after();
        const uint32_t o_col = tmem + t * 256 + 192, p_col = tmem + t * 256 + 128;
        mma_ts(o_col, p_col, dv, idesc_pv, j > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 1; kk < 8; ++kk) mma_ts(o_col, p_col + kk * 8, dv + 128 * kk, idesc_pv, 1u);
        mma_commit(&sm.o_done[t]);
        if (has_next && !issue_qk(p, sm, st, d, tmem, t, ns)) {
          ok = false;
          break;
        }
      }
      if (!ok) break;
      mma_commit(&sm.v_empty[cs]);
      if (has_next) {
        mma_commit(&sm.k_empty[ns]);
        if (j + 2 == nblk) mma_commit(&sm.q_empty);
      }
    }
    kv_c += nblk;
    ++items;
  }
}

// ------------------------------------------------------------------ softmax (one thread per row)
//
// Key masks, by head kind (the loop is instantiated once per kind, so a head pays only
// for the masks it can have):
//   kMaskPlain     - only the ragged end of a run (probe, stride and dense heads)
//   kMaskTiles     - + tiles this row's quarter does not keep, special tokens already
//                    counted inside a tile (correspondence heads)
//   kMaskCells     - + neighbour cells of this row's grid cell (position heads)
constexpr int kMaskPlain = 0, kMaskTiles = 1, kMaskCells = 2;

struct RowCtx {
  int t, lane, quarter;
  uint32_t tS, tP, tO;
  int nb_lo[2 * kMaxRadius + 1], nb_hi[2 * kMaxRadius + 1];  // kMaskCells: kept derived rows [lo, hi)
};

template <int kMask>
__device__ __forceinline__ uint64_t key_mask(const Half& hb, const RowCtx& rc) {
  if (!hb.have) return 0ull;
  if (kMask == kMaskTiles && !((hb.s.flags >> rc.quarter) & 1u)) return 0ull;
  uint64_t v = hb.cnt >= 64 ? ~0ull : ((1ull << hb.cnt) - 1ull);
  if (kMask == kMaskTiles) {
    const int lo = (hb.s.flags >> 8) & 0xFF, hi = (hb.s.flags >> 16) & 0xFF;
    if (hi > lo) v &= ~range_bits(max(lo - hb.off, 0), min(hi - hb.off, 64));
  }
  if (kMask == kMaskCells && (hb.s.flags & kSegCellMask)) {
    const int base = hb.s.row0 + hb.off;
    uint64_t nb = 0ull;
#pragma unroll
    for (int x = 0; x < 2 * kMaxRadius + 1; ++x)
      nb |= range_bits(max(rc.nb_lo[x] - base, 0), min(rc.nb_hi[x] - base, hb.cnt));
    v &= nb;
  }
  return v;
}

// All key blocks of one item for one row; returns false if a wait gave up.
template <int kMask>
__device__ __forceinline__ bool softmax_blocks(const AttnParams& p, AttnSmem& sm, ItemInfo& it, const RowCtx& rc,
                                               uint32_t& sfull_c, uint32_t& odone_c, float& l_out) {
  volatile int* abort = &sm.abort;
  const long long budget = p.wait_budget;
  const int t = rc.t, lane = rc.lane;
  const uint32_t tS = rc.tS, tP = rc.tP, tO = rc.tO;
  bool ok = true;
  float m = -INFINITY;  // running max, log2 units
  float l = 0.f;        // running row sum
  for (int j = 0; j < it.nblk; ++j) {
    uint64_t valid[2];
    valid[0] = key_mask<kMask>(it.w.next(), rc);
    valid[1] = key_mask<kMask>(it.w.next(), rc);
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[t], sfull_c & 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT))) {
        ok = false;
        break;
      }
      ++sfull_c;
      tc_fence_after();
      float s[128];
      {
        uint32_t raw[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, raw[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(raw[c][i]);
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
      float mp[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mp[i] = s[i];
#pragma unroll
      for (int i = 8; i < 128; ++i) mp[i & 7] = fmaxf(mp[i & 7], s[i]);
      float mx = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])), fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
      mx *= kScaleLog2;
      float alpha = 1.f;
      bool rescale = false;
      if (j == 0) {
        m = mx;
      } else if (mx > m + kRescaleThreshold) {
        alpha = fast_exp2(m - mx);
        m = mx;
        rescale = true;
      }
      const float m_use = (m == -INFINITY) ? 0.f : m;
      // 8 independent partial row sums: a single running sum would be a chain of 128 dependent adds
      uint32_t pk[64];
      float rp[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) rp[i] = 0.f;
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const float e0 = fast_exp2(fmaf(s[2 * i], kScaleLog2, -m_use));
        const float e1 = fast_exp2(fmaf(s[2 * i + 1], kScaleLog2, -m_use));
        rp[i & 7] += e0 + e1;
        pk[i] = pack_bf16x2(e0, e1);
      }
      const float rs = ((rp[0] + rp[1]) + (rp[2] + rp[3])) + ((rp[4] + rp[5]) + (rp[6] + rp[7]));
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
  l_out = l;
  return ok;
}

__device__ __forceinline__ void softmax_role(const AttnParams& p, AttnSmem& sm, uint32_t tmem, int warp, int lane) {
  volatile int* abort = &sm.abort;
  const long long budget = p.wait_budget;
  RowCtx rc;
  rc.t = (warp - 4) >> 2;
  rc.lane = lane;
  const int t = rc.t;
  const int wq = warp & 3;
  const int r = wq * 32 + lane;   // row inside the 128-row tile
  rc.quarter = (t * 128 + r) >> 6;  // 64-row quarter of the 256-row item
  const int quarter = rc.quarter;
  const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
  rc.tS = tmem + lane_off + t * 256;
  rc.tP = rc.tS + 128;
  rc.tO = rc.tS + 192;
  const uint32_t tO = rc.tO;
  uint32_t sfull_c = 0, odone_c = 0;
  bool ok = true;

  for (int item = blockIdx.x; ok && item < p.total_items; item += gridDim.x) {
    ItemInfo it = item_info(p, item);
    const HeadPlan& hp = p.heads[it.hi];
    const int qrow = it.q0 + t * 128 + r;
    float l = 0.f;
    if (hp.kind == SAF3R_POSITION) {
      // neighbour cells of this row's grid cell, as kept derived rows [lo, hi)
      const bool patch_row = qrow < p.P * p.S && p.S > 1;
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
        rc.nb_lo[x] = use ? hp.nb_base + ca * (p.S - 1) : 0;
        rc.nb_hi[x] = use ? hp.nb_base + (cb + 1) * (p.S - 1) : 0;
      }
      ok = softmax_blocks<kMaskCells>(p, sm, it, rc, sfull_c, odone_c, l);
    } else if (hp.kind == SAF3R_CORR) {
      ok = softmax_blocks<kMaskTiles>(p, sm, it, rc, sfull_c, odone_c, l);
    } else {
      ok = softmax_blocks<kMaskPlain>(p, sm, it, rc, sfull_c, odone_c, l);
    }
    if (!ok) break;

    // epilogue: O / l of this row
    if (!__all_sync(0xffffffffu, mbar_wait(&sm.o_done[t], odone_c & 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT))) {
      ok = false;
      break;
    }
    ++odone_c;
    tc_fence_after();
    uint32_t o[2][32];
    tmem_ld32(tO, o[0]);
    tmem_ld32(tO + 32, o[1]);
    tmem_wait_ld();
    tc_fence_before();
    int token = -1;
    if (hp.q_src == 1) {
      if (qrow < p.N) token = position_token(p, qrow);
    } else if (hp.q_src == 2) {
      const int u = mapped_tile(p, hp, it.local, quarter);
      if (u >= 0 && u * 64 + (r & 63) < p.N) token = u * 64 + (r & 63);
    } else if (qrow < p.N) {
      token = qrow;
    }
    if (token >= 0) {
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const long long rowoff = (static_cast<long long>(hp.head) * p.N + token) * kD;
      if (p.out_fp32) {
        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + rowoff);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint32_t* w = &o[i >> 3][(4 * i) & 31];
          dst[i] = make_float4(__uint_as_float(w[0]) * inv, __uint_as_float(w[1]) * inv,
                               __uint_as_float(w[2]) * inv, __uint_as_float(w[3]) * inv);
        }
      } else {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + rowoff);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t* w = &o[i >> 2][(8 * i) & 31];
          dst[i] = make_uint4(pack_bf16x2(__uint_as_float(w[0]) * inv, __uint_as_float(w[1]) * inv),
                              pack_bf16x2(__uint_as_float(w[2]) * inv, __uint_as_float(w[3]) * inv),
                              pack_bf16x2(__uint_as_float(w[4]) * inv, __uint_as_float(w[5]) * inv),
                              pack_bf16x2(__uint_as_float(w[6]) * inv, __uint_as_float(w[7]) * inv));
        }
      }
    }
  }
}

}  // namespace

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
    if (lane == 0) producer_role(p, sm, tmQ, tmK, tmV, tmQC, tmKC, tmVC);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) mma_role(p, sm, tmem);
    __syncwarp();
  } else if (warp >= 4) {
    reg_alloc_inc<200>();
    softmax_role(p, sm, tmem, warp, lane);
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
