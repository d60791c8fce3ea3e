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
// Token-wise heads' patch queries (q_src 4) come in a cached order that makes queries with the
// same best matches neighbours; each item streams the head's special keys (derived rows) and then
// the union of its rows' per-frame keys, whose scattered K and V rows the two otherwise idle warps
// copy (cp.async, 16 bytes per lane, many rows in flight); every row keeps its own keys of that
// union through a cached bitmask.
//
// Warp roles (12 warps, three warpgroups):
//   warp 0      TMA producer: Q tiles, then K and V blocks into a 4-stage ring
//   warp 1      MMA issuer: O_t += P_t V, then S_t = Q_t K^T of the next block (the whole warp
//               waits and computes descriptors, one elected lane issues)
//   warps 2-3   token-wise items only: copy the union's K and V rows (cp.async), one key half each
//               (most of their registers go to the softmax warpgroups)
//   warps 4-11  softmax: warp w owns rows 32*(w%4)..+31 of a tile (the TMEM lanes it may
//               read) and key half (w-4)/4 of every 128-key block; all eight warps work
//               on tile 0, then on tile 1, so each tile's products run on the tensor
//               core while the other tile's exponentials run on the SFUs.
// TMEM (512 columns): per tile t, S_t (128 fp32 cols; each warp writes its bf16 P over the
// first 32 columns of its own key half once it has read them) and two accumulators
// O_t,a / O_t,b (64 fp32 cols each), one per key half, merged with the halves' running
// maxima and sums when the item ends.
// The softmax warps never walk the key-run lists: a head with one implicit run (probe,
// stride, dense) gets block j's half-blocks in closed form, and for list heads the producer,
// which walks the list anyway, leaves each block's halves in shared memory next to its V
// stage.  Warps whose 32 rows keep no key of a half-block (correspondence tiles of another
// quarter, cells outside the neighbourhood) write P = 0 without computing anything.
//
// Exponentials: one pair in eight (kPolyPairs) is computed on the FMA pipe instead of the SFU,
// which the softmax otherwise keeps busiest: 2^x = 2^floor(x) * p(x - floor(x)), the floor from
// one round-down addition of 1.5 * 2^23, p a cubic fitted to 2^f on [0, 1) for least maximum
// relative error (a linear-programming minimax fit with p(0) = 1: relative error below 8.6e-5,
// far below the 2^-9 of the bf16 P it feeds), and 2^floor(x) added to p's exponent field.  x is
// clamped at -127 first, where the construction gives exactly +0 (masked keys).
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
constexpr int kSegBuf = 1024;             // key runs of one item staged in shared memory (longer lists are read in place)
constexpr float kScaleLog2 = 0.18033688011112042f;  // log2(e) / sqrt(64)
constexpr float kRescaleThreshold = 8.0f;           // log2 units: keep a stale max until it is 256x off
// Pairs (of the 32 per 64-key half-block) whose exponentials run on the FMA pipe: bit i = pair i.
#ifndef SAF3R_POLY_PAIRS
#define SAF3R_POLY_PAIRS 0x80808080u
#endif
constexpr uint32_t kPolyPairs = SAF3R_POLY_PAIRS;
// the cubic of the FMA-pipe exponential: p(f) = 1 + f (c1 + f (c2 + f c3))
constexpr float kExpC1 = 0.6951168179512024f, kExpC2 = 0.22764486074447632f, kExpC3 = 0.07706713676452637f;

// One 64-row half-block of keys.
struct Half {
  bool have;
  Seg s;
  int off;  // first row inside the run
  int cnt;  // rows (<= 64)
};

struct AttnSmem {
  uint8_t q[2][kTileBytes];
  uint8_t k[kStages][kTileBytes];
  uint8_t v[kStages][kTileBytes];
  uint64_t q_full, q_empty;
  uint64_t k_full[kStages], k_empty[kStages], v_full[kStages], v_empty[kStages];
  uint64_t s_full[2], p_full[2], o_done[2];
  uint64_t vg_go[kStages];    // token-wise items: the producer found the stage free for the gather warps
  uint64_t vg_done[kStages];  // token-wise items: both gather warps' K/V rows of the stage have landed
  Half info[kStages][2];      // the key halves of the block in each K/V stage (written by the producer)
  Seg segbuf[kSegBuf];        // the current item's key runs (copied by the producer warp, read by its lane 0)
  uint64_t pair[4];           // the two warps sharing rows 32*w..+31 (w = warp % 4) meet here at an item's end
  float stats[2][2][128][2];  // [key half][tile][row] = (running max, running sum) for the final merge
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
    it.nblk = (((hp.seg.len + 63) >> 6) + 1) >> 1;
  } else {
    // the plan stored the item's segment and block counts side by side
    it.w.list = p.segs + hp.seg_list + static_cast<long long>(it.local) * hp.seg_cap;
    const int2 c = *reinterpret_cast<const int2*>(p.seg_counts + hp.cnt_list + 2 * it.local);
    it.w.nseg = c.x;
    it.nblk = c.y;
  }
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

// One item's loads (lane 0 of the producer warp): the Q tiles, then every 128-key block's K and V
// halves into the ring.  Returns false when a wait gave up.
__device__ __forceinline__ bool producer_item(const AttnParams& p, AttnSmem& sm, const CUtensorMap& tmQ,
                                              const CUtensorMap& tmK, const CUtensorMap& tmV,
                                              const CUtensorMap& tmQC, const CUtensorMap& tmKC,
                                              const CUtensorMap& tmVC, ItemInfo& it, const HeadPlan& hp,
                                              uint32_t& k_issued, uint32_t& v_issued, uint32_t& q_issued) {
  volatile int* abort = &sm.abort;
  const long long budget = p.wait_budget;
  if (q_issued > 0 && !mbar_wait(&sm.q_empty, (q_issued - 1) & 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT))
    return false;
  mbar_arrive_expect_tx(&sm.q_full, 2 * kTileBytes);
  for (int quarter = 0; quarter < 4; ++quarter) {
    void* dst = sm.q[quarter >> 1] + (quarter & 1) * kHalfBytes;
    if (hp.q_src == 1 || hp.q_src == 3) {
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
    if (k_issued >= kStages && !mbar_wait(&sm.k_empty[stage], ph ^ 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT))
      return false;
    mbar_arrive_expect_tx(&sm.k_full[stage], kTileBytes);
    if (h0.have) load_half(hp, h0, sm.k[stage], &tmK, &tmKC, &sm.k_full[stage]); else tma_load_3d(sm.k[stage], &tmK, 0, -64, hp.head, &sm.k_full[stage]);
    if (h1.have) load_half(hp, h1, sm.k[stage] + kHalfBytes, &tmK, &tmKC, &sm.k_full[stage]); else tma_load_3d(sm.k[stage] + kHalfBytes, &tmK, 0, -64, hp.head, &sm.k_full[stage]);
    ++k_issued;
    if (v_issued >= kStages && !mbar_wait(&sm.v_empty[stage], ph ^ 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT))
      return false;
    // the block's halves for the softmax warps; the arrival below releases them with the stage
    sm.info[stage][0] = h0;
    sm.info[stage][1] = h1;
    mbar_arrive_expect_tx(&sm.v_full[stage], kTileBytes);
    if (h0.have) load_half(hp, h0, sm.v[stage], &tmV, &tmVC, &sm.v_full[stage]); else tma_load_3d(sm.v[stage], &tmV, 0, -64, hp.head, &sm.v_full[stage]);
    if (h1.have) load_half(hp, h1, sm.v[stage] + kHalfBytes, &tmV, &tmVC, &sm.v_full[stage]); else tma_load_3d(sm.v[stage] + kHalfBytes, &tmV, 0, -64, hp.head, &sm.v_full[stage]);
    ++v_issued;
  }
  return true;
}

// One item of a token-wise head's patch queries, run by the whole producer warp: derived Q rows
// and the derived special K/V rows as TMA boxes; the union's K and V rows come from the gather
// warps (gather_role).  A stage's full barriers expect the bytes of its TMA halves and get this
// warp's arrival once both gather warps report its rows landed (checked one block later).
__device__ __forceinline__ bool producer_item_gather(const AttnParams& p, AttnSmem& sm, const CUtensorMap& tmQC,
                                                     const CUtensorMap& tmKC, const CUtensorMap& tmVC, ItemInfo& it,
                                                     const HeadPlan& hp, uint32_t& k_issued, uint32_t& v_issued,
                                                     uint32_t& q_issued, uint32_t& vg_par, int lane) {
  volatile int* abort = &sm.abort;
  const long long budget = p.wait_budget;
  int pend = -1;  // the stage waiting for the gather warps
  auto release_v = [&]() -> bool {
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&sm.vg_done[pend], (vg_par >> pend) & 1u, abort, p.err,
                                                      budget, SAF3R_ERR_TIMEOUT));
    vg_par ^= 1u << pend;
    if (lane == 0) {
      mbar_arrive(&sm.k_full[pend]);
      mbar_arrive(&sm.v_full[pend]);
    }
    pend = -1;
    return ok;
  };
  if (q_issued > 0 &&
      !__all_sync(0xffffffffu, mbar_wait(&sm.q_empty, (q_issued - 1) & 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT)))
    return false;
  if (lane == 0) {
    mbar_arrive_expect_tx(&sm.q_full, 2 * kTileBytes);
    for (int quarter = 0; quarter < 4; ++quarter)
      tma_load_2d(sm.q[quarter >> 1] + (quarter & 1) * kHalfBytes, &tmQC, 0, hp.q_base + it.q0 + quarter * 64,
                  &sm.q_full);
  }
  ++q_issued;
  for (int b = 0; b < it.nblk; ++b) {
    const Half h0 = it.w.next();
    const Half h1 = it.w.next();
    const uint32_t stage = k_issued % kStages, ph = (k_issued / kStages) & 1;
    if (k_issued >= kStages &&
        !__all_sync(0xffffffffu, mbar_wait(&sm.k_empty[stage], ph ^ 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT)))
      return false;
    if (lane == 0) {
      const bool s0 = h0.have && h0.s.src == 1, s1 = h1.have && h1.s.src == 1;
      if (s0 || s1) {
        mbar_expect_tx(&sm.k_full[stage], (s0 ? kHalfBytes : 0) + (s1 ? kHalfBytes : 0));
        if (s0) tma_load_2d(sm.k[stage], &tmKC, 0, hp.kc_base + h0.s.row0 + h0.off, &sm.k_full[stage]);
        if (s1) tma_load_2d(sm.k[stage] + kHalfBytes, &tmKC, 0, hp.kc_base + h1.s.row0 + h1.off, &sm.k_full[stage]);
      }
    }
    ++k_issued;
    if (v_issued >= kStages &&
        !__all_sync(0xffffffffu, mbar_wait(&sm.v_empty[stage], ph ^ 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT))) {
      if (pend >= 0) release_v();
      return false;
    }
    const bool t0 = h0.have && h0.s.src == 1, t1 = h1.have && h1.s.src == 1;
    if (lane == 0) {
      mbar_arrive(&sm.vg_go[stage]);  // the gather warps may fill this stage now
      // the block's halves for the softmax warps; the arrival releases them with the stage
      sm.info[stage][0] = h0;
      sm.info[stage][1] = h1;
      if (t0 || t1) {
        mbar_expect_tx(&sm.v_full[stage], (t0 ? kHalfBytes : 0) + (t1 ? kHalfBytes : 0));
        if (t0) tma_load_2d(sm.v[stage], &tmVC, 0, hp.kc_base + h0.s.row0 + h0.off, &sm.v_full[stage]);
        if (t1) tma_load_2d(sm.v[stage] + kHalfBytes, &tmVC, 0, hp.kc_base + h1.s.row0 + h1.off, &sm.v_full[stage]);
      }
    }
    ++v_issued;
    if (pend >= 0 && !release_v()) {
      pend = static_cast<int>(stage);
      release_v();
      return false;
    }
    pend = static_cast<int>(stage);
  }
  return pend < 0 || release_v();
}

// Warps 2-3 on the items of token-wise heads' patch queries: warp 2 copies the union's K and V rows
// of each block's first key half, warp 3 those of the second (cp.async, 16 bytes per lane, laid out
// as a TMA box with 128-byte swizzle would be: chunk c of row r at chunk c ^ (r & 7); an absent
// half, rows past its count and out-of-range tokens (reported) are zero), and each arrives on the
// stage's vg_done once its rows have landed (checked one block later, so two blocks' copies are
// in flight).  They start a block when the producer, which takes every block in order, reports
// its stage free (vg_go): walking the other items' blocks themselves, they could otherwise run
// phases ahead of the ring.  Other items are skipped; only the stage count advances.
__device__ __forceinline__ void gather_role(const AttnParams& p, AttnSmem& sm, int kh, int lane) {
  volatile int* abort = &sm.abort;
  const long long budget = p.wait_budget;
  const int col = lane & 7;
  uint32_t kv = 0;      // key blocks of every item so far (the producer's count)
  uint32_t go_par = 0;  // phase parity of each stage's vg_go
  bool ok = true;
  for (int item = blockIdx.x; ok && item < p.total_items; item += gridDim.x) {
    ItemInfo it = item_info(p, item);
    const HeadPlan& hp = p.heads[it.hi];
    if (hp.q_src != 4) {
      kv += it.nblk;
      continue;
    }
    const uint16_t* vrows = p.v_rows + static_cast<size_t>(hp.head) * p.N * kD + col * 8;
    const uint16_t* krows = p.k_rows + static_cast<size_t>(hp.head) * p.N * kD + col * 8;
    int pend = -1;
    for (int b = 0; b < it.nblk; ++b) {
      const Half h0 = it.w.next();
      const Half h1 = it.w.next();
      const Half h = kh ? h1 : h0;
      const bool copy = !(h.have && h.s.src == 1);
      // listed tokens of this half: lane l holds rows l and l + 32 (-1: none)
      int ta = -1, tb = -1;
      if (copy && h.have) {
        if (lane < h.cnt) ta = hp.glist[h.s.row0 + h.off + lane];
        if (lane + 32 < h.cnt) tb = hp.glist[h.s.row0 + h.off + lane + 32];
      }
      const uint32_t stage = kv % kStages;
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&sm.vg_go[stage], (go_par >> stage) & 1u, abort, p.err, budget, SAF3R_ERR_TIMEOUT))) {
        ok = false;
        break;
      }
      go_par ^= 1u << stage;
      if (copy) {
        const uint32_t base = smem_u32(sm.v[stage] + kh * kHalfBytes);
        const uint32_t kbase = smem_u32(sm.k[stage] + kh * kHalfBytes);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int r = (lane >> 3) + 4 * i;
          int t = __shfl_sync(0xffffffffu, i < 8 ? ta : tb, r & 31);
          if (t >= p.N || t < -1) {
            atomicCAS(p.err, 0, SAF3R_ERR_INDEX);
            t = -1;
          }
          cp_async16(kbase + r * 128 + ((col ^ (r & 7)) << 4),
                     t >= 0 ? static_cast<const void*>(krows + static_cast<size_t>(t) * kD)
                            : static_cast<const void*>(p.v_rows),
                     t >= 0 ? 16u : 0u);
          cp_async16(base + r * 128 + ((col ^ (r & 7)) << 4),
                     t >= 0 ? static_cast<const void*>(vrows + static_cast<size_t>(t) * kD)
                            : static_cast<const void*>(p.v_rows),
                     t >= 0 ? 16u : 0u);
        }
      }
      cp_async_commit();
      if (pend >= 0) {
        cp_async_wait<1>();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.vg_done[pend]);
      }
      pend = static_cast<int>(stage);
      ++kv;
    }
    cp_async_wait<0>();
    if (pend >= 0) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.vg_done[pend]);
    }
  }
  cp_async_wait<0>();
}

// ------------------------------------------------------------------ TMA producer (one warp, lane 0 issues)
//
// At each item the whole warp copies the item's key runs into shared memory (a list head's runs
// would otherwise be read one by one from global memory as lane 0 walks them); lane 0 then walks
// them and issues every load.
__device__ __forceinline__ void producer_role(const AttnParams& p, AttnSmem& sm, const CUtensorMap& tmQ,
                                              const CUtensorMap& tmK, const CUtensorMap& tmV,
                                              const CUtensorMap& tmQC, const CUtensorMap& tmKC,
                                              const CUtensorMap& tmVC, int lane) {
  if (lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  uint32_t k_issued = 0, v_issued = 0, q_issued = 0;
  uint32_t vg_par = 0;  // phase parity of each stage's vg_done
  bool ok = true;
  for (int item = blockIdx.x; ok && item < p.total_items; item += gridDim.x) {
    ItemInfo it = item_info(p, item);
    const HeadPlan& hp = p.heads[it.hi];
    if (it.w.list != nullptr && it.w.nseg <= kSegBuf) {
      for (int i = lane; i < it.w.nseg; i += 32) sm.segbuf[i] = it.w.list[i];
      it.w.list = sm.segbuf;
    }
    __syncwarp();
    if (hp.q_src == 4) {
      ok = producer_item_gather(p, sm, tmQC, tmKC, tmVC, it, hp, k_issued, v_issued, q_issued, vg_par, lane);
      __syncwarp();
    } else {
      if (lane == 0) ok = producer_item(p, sm, tmQ, tmK, tmV, tmQC, tmKC, tmVC, it, hp, k_issued, v_issued, q_issued);
      ok = __shfl_sync(0xffffffffu, ok, 0);  // the runs are not overwritten before lane 0 has walked them
      k_issued = __shfl_sync(0xffffffffu, k_issued, 0);
      v_issued = __shfl_sync(0xffffffffu, v_issued, 0);
      q_issued = __shfl_sync(0xffffffffu, q_issued, 0);
    }
  }
  if (lane != 0) return;
  // Teardown: every copy lane 0 issued must have landed before the CTA exits
  // (these waits ignore the abort flag but stay bounded).
  const long long drain = kDrainBudget;
  if (q_issued > 0) mbar_wait_drain(&sm.q_full, (q_issued - 1) & 1, drain);
  for (uint32_t c = (k_issued > kStages ? k_issued - kStages : 0); c < k_issued; ++c)
    mbar_wait_drain(&sm.k_full[c % kStages], (c / kStages) & 1, drain);
  for (uint32_t c = (v_issued > kStages ? v_issued - kStages : 0); c < v_issued; ++c)
    mbar_wait_drain(&sm.v_full[c % kStages], (c / kStages) & 1, drain);
}

// ------------------------------------------------------------------ MMA issuer (one warp)
//
// For each key block and each tile in turn: O_t,a += P_t,a V[0:64] and O_t,b += P_t,b V[64:128]
// once all eight softmax warps have written P_t, then S_t = Q_t K^T of the next block (it
// overwrites P_t, which the products just issued have read: one lane issues every product,
// and a lane's products execute in issue order).  The warp sits on the critical path, so it
// does nothing but wait, add descriptor offsets and issue.  Running it converged (rather than
// as a lone lane) keeps the descriptors warp-uniform, which measurably shortens the issue of
// each 12-product tile step.  Every product covers the whole block (keys a row does not keep
// get P = 0).
struct MmaState {
  uint32_t pfull_c[2] = {0, 0};
};

// Shared-memory descriptors of the operand tiles, computed once: a K-step of 16 keys or 16
// features is then one 64-bit add (the start address sits in the low bits, in 16-byte units).
struct Descs {
  uint64_t q[2];  // Q tiles (K-major, 128-byte swizzle)
  uint64_t k0;    // K stage 0 (K-major); stage s adds s * kTileBytes / 16
  uint64_t v0;    // V stage 0 (MN-major); stage s adds s * kTileBytes / 16
};
constexpr uint64_t kStageDesc = kTileBytes >> 4;

// S_t = Q_t K^T for one 128-key block.
__device__ __forceinline__ void issue_qk(const Descs& d, uint32_t tmem, int t, uint32_t stage) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
  const uint64_t dq = d.q[t];
  const uint64_t dk = d.k0 + stage * kStageDesc;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) mma_ss(tmem + t * 256, dq + 2 * kk, dk + 2 * kk, idesc, kk > 0 ? 1u : 0u);
}

// Run by the whole warp: every lane waits and computes the (warp-uniform) descriptors, one
// elected lane issues the products and their commits.
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
    if (!__all_sync(0xffffffffu, mbar_wait(&sm.q_full, items & 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT))) break;
    tc_fence_after();
    {
      const uint32_t stage = kv_c % kStages, ph = (kv_c / kStages) & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.k_full[stage], ph, abort, p.err, budget, SAF3R_ERR_TIMEOUT))) break;
      tc_fence_after();
      if (elect_one()) {
        issue_qk(d, tmem, 0, stage);
        mma_commit(&sm.s_full[0]);
        issue_qk(d, tmem, 1, stage);
        mma_commit(&sm.s_full[1]);
        mma_commit(&sm.k_empty[stage]);
        if (nblk == 1) mma_commit(&sm.q_empty);
      }
      __syncwarp();
    }
    for (int j = 0; ok && j < nblk; ++j) {
      const uint32_t c = kv_c + j;
      const uint32_t cs = c % kStages, cph = (c / kStages) & 1;
      const bool has_next = j + 1 < nblk;
      const uint32_t ns = (c + 1) % kStages, nph = ((c + 1) / kStages) & 1;
      if (has_next &&
          !__all_sync(0xffffffffu, mbar_wait(&sm.k_full[ns], nph, abort, p.err, budget, SAF3R_ERR_TIMEOUT))) {
        ok = false;
        break;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.v_full[cs], cph, abort, p.err, budget, SAF3R_ERR_TIMEOUT))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t dv = d.v0 + cs * kStageDesc;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (!__all_sync(0xffffffffu,
                        mbar_wait(&sm.p_full[t], st.pfull_c[t] & 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT))) {
          ok = false;
          break;
        }
        ++st.pfull_c[t];
        tc_fence_after();
        const uint32_t s_col = tmem + t * 256, o_col = s_col + 128;
        if (elect_one()) {
          // key half a: P in S columns 0..31, keys 0..63 of V; key half b: S columns 64..95, keys 64..127
          mma_ts(o_col, s_col, dv, idesc_pv, j > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 1; kk < 4; ++kk) mma_ts(o_col, s_col + kk * 8, dv + 128 * kk, idesc_pv, 1u);
          mma_ts(o_col + 64, s_col + 64, dv + 128 * 4, idesc_pv, j > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 1; kk < 4; ++kk)
            mma_ts(o_col + 64, s_col + 64 + kk * 8, dv + 128 * (4 + kk), idesc_pv, 1u);
          if (has_next) {
            issue_qk(d, tmem, t, ns);
            mma_commit(&sm.s_full[t]);
          } else {
            mma_commit(&sm.o_done[t]);
          }
        }
        __syncwarp();
      }
      if (!ok) break;
      if (elect_one()) {
        mma_commit(&sm.v_empty[cs]);
        if (has_next) {
          mma_commit(&sm.k_empty[ns]);
          if (j + 2 == nblk) mma_commit(&sm.q_empty);
        }
      }
      __syncwarp();
    }
    kv_c += nblk;
    ++items;
  }
}

// ------------------------------------------------------------------ softmax (one thread per row and key half)
//
// Key masks, by head kind (the loop is instantiated once per kind, so a head pays only
// for the masks it can have):
//   kMaskPlain     - only the ragged end of a run (probe, stride and dense heads)
//   kMaskTiles     - + tiles this row's quarter does not keep, special tokens already
//                    counted inside a tile (correspondence heads)
//   kMaskCells     - + neighbour cells of this row's grid cell (position heads)
//   kMaskBits      - the row's cached bitmask over the item's union (token-wise patch queries;
//                    computed by softmax_blocks_bits, which passes it in)
constexpr int kMaskPlain = 0, kMaskTiles = 1, kMaskCells = 2, kMaskBits = 3;
constexpr int kNbIntervals = 2 * kMaxRadius + 1;

struct RowCtx {
  int kh;            // key half of every block this warp owns (0: keys 0..63, 1: keys 64..127)
  int r;             // row inside each 128-row tile
  int lane;
  uint32_t lane_off; // TMEM lane field of this warp
  int nb_lo[2][kNbIntervals], nb_hi[2][kNbIntervals];  // position heads: kept derived rows [lo, hi) per tile
  int lat_stride, lat_phase;  // hybrid heads: the lattice (counted in the derived run), 0 = none
  const uint64_t* gmask;      // token-wise patch queries: [half-block of the union][item row] bitmasks
  bool withhold;     // test hook: skip the next P-ready arrival (the MMA warp's wait then runs out)
};

// Bits b of a 64-key half-block starting at token j0 whose token j0 + b lies on the lattice
// j = phase (mod stride).
__device__ __forceinline__ uint64_t lattice_bits(int j0, int stride, int phase) {
  int b = (phase - j0) % stride;
  if (b < 0) b += stride;
  uint64_t m = 0ull;
  for (; b < 64; b += stride) m |= 1ull << b;
  return m;
}

template <int kMask>
__device__ __forceinline__ uint64_t key_mask(const Half& hb, const RowCtx& rc, int t) {
  if (!hb.have) return 0ull;
  const int quarter = (t * 128 + rc.r) >> 6;
  if (kMask == kMaskTiles && !((hb.s.flags >> quarter) & 1u)) return 0ull;
  uint64_t v = hb.cnt >= 64 ? ~0ull : ((1ull << hb.cnt) - 1ull);
  if (kMask == kMaskTiles) {
    const int lo = (hb.s.flags >> 8) & 0xFF, hi = (hb.s.flags >> 16) & 0xFF;
    if (hi > lo) v &= ~range_bits(max(lo - hb.off, 0), min(hi - hb.off, 64));
    // a hybrid head's lattice keys inside a tile are already counted in its derived run
    if (rc.lat_stride > 0 && hb.s.src == 0) v &= ~lattice_bits(hb.s.row0 + hb.off, rc.lat_stride, rc.lat_phase);
  }
  if (kMask == kMaskCells && (hb.s.flags & kSegCellMask)) {
    const int base = hb.s.row0 + hb.off;
    uint64_t nb = 0ull;
#pragma unroll
    for (int x = 0; x < kNbIntervals; ++x)
      nb |= range_bits(max(rc.nb_lo[t][x] - base, 0), min(rc.nb_hi[t][x] - base, hb.cnt));
    v &= nb;
  }
  return v;
}

// This warp's share of "P_t is in TMEM" (p_full counts one arrival per softmax warp).
__device__ __forceinline__ void arrive_p_full(AttnSmem& sm, RowCtx& rc, int t) {
  if (rc.withhold) {  // test hook only: this one arrival never comes
    rc.withhold = false;
    return;
  }
  if (rc.lane == 0) mbar_arrive(&sm.p_full[t]);
}

struct SoftmaxState {
  uint32_t kv_c = 0;  // key blocks seen (all items): the K/V stage and its phase
  uint32_t sfull_c[2] = {0, 0};
  uint32_t odone_c = 0;
  uint32_t pair_c = 0;
};


// O_t of this warp's key half (64 columns from tO) times alpha: the running max grew by more
// than the threshold.  O_t already holds the previous blocks' products (s_full of this block
// was committed after them).
__device__ __forceinline__ void rescale_o(uint32_t tO, float alpha) {
#pragma unroll 1
  for (int q = 0; q < 4; ++q) {
    uint32_t o[16];
    tmem_ld16(tO + q * 16, o);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
    tmem_st16(tO + q * 16, o);
  }
}

// 2^x0, 2^x1 on the FMA pipe (see the head of this file).
__device__ __forceinline__ void exp2_poly2(float x0, float x1, float& e0, float& e1) {
  constexpr float kMagic = 12582912.f;  // 1.5 * 2^23: x + kMagic rounded down holds floor(x) in its low bits
  x0 = fmaxf(x0, -127.f);
  x1 = fmaxf(x1, -127.f);
  uint64_t t, xi, f, pp;
  asm("add.rm.f32x2 %0, %1, %2;" : "=l"(t) : "l"(f32x2(x0, x1)), "l"(f32x2(kMagic, kMagic)));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(xi) : "l"(t), "l"(f32x2(kMagic, kMagic)));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(f) : "l"(f32x2(x0, x1)), "l"(xi));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(pp) : "l"(f), "l"(f32x2(kExpC3, kExpC3)), "l"(f32x2(kExpC2, kExpC2)));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(pp) : "l"(pp), "l"(f), "l"(f32x2(kExpC1, kExpC1)));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(pp) : "l"(pp), "l"(f), "l"(f32x2(1.f, 1.f)));
  // exponent field += floor(x): (bits of t) << 23 is floor(x) << 23 modulo 2^32
  e0 = __uint_as_float(static_cast<uint32_t>(pp) + (static_cast<uint32_t>(t) << 23));
  e1 = __uint_as_float(static_cast<uint32_t>(pp >> 32) + (static_cast<uint32_t>(t >> 32) << 23));
}

// 2^x0, 2^x1 of pair i of a half-block: on the FMA pipe for the pairs of kPolyPairs, else the SFU.
__device__ __forceinline__ void exp2_pair(int i, float x0, float x1, float& e0, float& e1) {
  if ((kPolyPairs >> i) & 1u) {
    exp2_poly2(x0, x1, e0, e1);
  } else {
    e0 = fast_exp2(x0);
    e1 = fast_exp2(x1);
  }
}

// P = 2^(s * scale - m) for the row's 64 logits as 32 bf16 pairs, and 8 partial row sums (a
// single running sum would be a chain of dependent adds).
__device__ __forceinline__ void exponentials(const float (&s)[64], float m, uint32_t (&pk)[32], float (&rp)[8]) {
  const float m_use = (m == -INFINITY) ? 0.f : m;
#pragma unroll
  for (int i = 0; i < 8; ++i) rp[i] = 0.f;
  float x[64];
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    x[2 * i] = s[2 * i];
    x[2 * i + 1] = s[2 * i + 1];
    ffma2(x[2 * i], x[2 * i + 1], kScaleLog2, -m_use);
  }
#pragma unroll
  for (int i = 0; i < 32; ++i) exp2_pair(i, x[2 * i], x[2 * i + 1], x[2 * i], x[2 * i + 1]);
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    fadd2(rp[2 * (i & 3)], rp[2 * (i & 3) + 1], x[2 * i], x[2 * i + 1]);
    pk[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
  }
}

// One 64-key half-block of one tile for this thread's row: masks, running max, exponentials,
// P (bf16) written over the half's first 32 S columns, arrival on p_full[t].
template <int kMask>
__device__ __forceinline__ bool softmax_half(const AttnParams& p, AttnSmem& sm, SoftmaxState& ss, uint32_t tmem,
                                             RowCtx& rc, int t, int j, uint64_t valid, float& m, float& l) {
  if (!__all_sync(0xffffffffu,
                  mbar_wait(&sm.s_full[t], ss.sfull_c[t] & 1, &sm.abort, p.err, p.wait_budget, SAF3R_ERR_TIMEOUT)))
    return false;
  ++ss.sfull_c[t];
  tc_fence_after();
  const uint32_t tS = tmem + rc.lane_off + t * 256 + rc.kh * 64;
  if (kMask != kMaskPlain && __all_sync(0xffffffffu, valid == 0ull)) {
    // no row of this warp keeps a key of this half-block: P = 0, the running max and sum stay
    if (j == 0) m = -INFINITY;
    uint32_t zero[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) zero[i] = 0u;
    tmem_st32(tS, zero);
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    arrive_p_full(sm, rc, t);
    return true;
  }
  float s[64];
  {
    uint32_t raw[64];
    tmem_ld64(tS, raw);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 64; ++i) s[i] = __uint_as_float(raw[i]);
  }
  if (valid != ~0ull) {
#pragma unroll
    for (int i = 0; i < 64; ++i)
      if (!((valid >> i) & 1ull)) s[i] = -INFINITY;
  }
  uint32_t pk[32];
  float rp[8];
  float alpha = 1.f;
  if (kMask == kMaskPlain) {
    // Probe, stride and dense heads: exponentials against the running max of the earlier
    // blocks, with this block's max taken in the same pass; only on the first block, or when
    // the max grew past the threshold, are they redone against the new max.
    const float m_spec = (m == -INFINITY) ? 0.f : m;
    float mp[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      rp[i] = 0.f;
      mp[i] = s[i];
    }
    float x[64];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      x[2 * i] = s[2 * i];
      x[2 * i + 1] = s[2 * i + 1];
      if (i >= 4) mp[i & 7] = max3f(mp[i & 7], x[2 * i], x[2 * i + 1]);
      ffma2(x[2 * i], x[2 * i + 1], kScaleLog2, -m_spec);
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) exp2_pair(i, x[2 * i], x[2 * i + 1], x[2 * i], x[2 * i + 1]);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      fadd2(rp[2 * (i & 3)], rp[2 * (i & 3) + 1], x[2 * i], x[2 * i + 1]);
      pk[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
    }
    const float mx =
        max3f(max3f(mp[0], mp[1], mp[2]), max3f(mp[3], mp[4], mp[5]), fmaxf(mp[6], mp[7])) * kScaleLog2;
    const bool grow = (j == 0) || (mx > m + kRescaleThreshold);
    if (__any_sync(0xffffffffu, grow)) {
      const float m_new = grow ? mx : m;
      if (j > 0) {
        // rows whose max moved rescale O_t of this half (the others multiply by 1)
        alpha = grow ? fast_exp2(m - m_new) : 1.f;  // m may be -inf: alpha = 0
        rescale_o(tmem + rc.lane_off + t * 256 + 128 + rc.kh * 64, alpha);
      }
      m = m_new;
      exponentials(s, m, pk, rp);
    }
  } else {
    // Position and correspondence heads (whose masks move the max more often): the block's
    // max first, then the exponentials.
    float mp[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) mp[i] = s[i];
#pragma unroll
    for (int i = 4; i < 32; ++i) mp[i & 7] = max3f(mp[i & 7], s[2 * i], s[2 * i + 1]);
    const float mx =
        max3f(max3f(mp[0], mp[1], mp[2]), max3f(mp[3], mp[4], mp[5]), fmaxf(mp[6], mp[7])) * kScaleLog2;
    bool rescale = false;
    if (j == 0) {
      m = mx;
    } else if (mx > m + kRescaleThreshold) {
      alpha = fast_exp2(m - mx);  // m may be -inf: alpha = 0
      m = mx;
      rescale = true;
    }
    if (__any_sync(0xffffffffu, rescale)) rescale_o(tmem + rc.lane_off + t * 256 + 128 + rc.kh * 64, alpha);
    exponentials(s, m, pk, rp);
  }
  l = l * alpha + (((rp[0] + rp[1]) + (rp[2] + rp[3])) + ((rp[4] + rp[5]) + (rp[6] + rp[7])));
  tmem_st32(tS, pk);
  tmem_wait_st();
  tc_fence_before();
  __syncwarp();
  arrive_p_full(sm, rc, t);
  return true;
}

// All key blocks of one item: tile 0 then tile 1 for every block.
template <int kMask>
__device__ __forceinline__ bool softmax_blocks(const AttnParams& p, AttnSmem& sm, SoftmaxState& ss, uint32_t tmem,
                                               ItemInfo& it, RowCtx& rc, float (&m)[2], float (&l)[2]) {
  for (int j = 0; j < it.nblk; ++j) {
    Half hb;
    if (kMask == kMaskPlain) {
      // one implicit run: this warp's half-block of block j is a closed form
      hb.s = it.w.implicit;
      hb.off = (2 * j + rc.kh) * 64;
      hb.have = hb.off < hb.s.len;
      hb.cnt = min(64, hb.s.len - hb.off);
    } else {
      // the producer wrote this block's halves next to its V stage; that stage is not refilled
      // before the products of this block, which wait for these warps
      const uint32_t c = ss.kv_c + j, st = c % kStages;
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.v_full[st], (c / kStages) & 1, &sm.abort, p.err, p.wait_budget,
                                             SAF3R_ERR_TIMEOUT)))
        return false;
      hb = sm.info[st][rc.kh];
    }
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const uint64_t valid = key_mask<kMask>(hb, rc, t);
      if (!softmax_half<kMask>(p, sm, ss, tmem, rc, t, j, valid, m[t], l[t])) return false;
    }
  }
  ss.kv_c += it.nblk;
  return true;
}

// All key blocks of one item of a token-wise head's patch queries.  Its runs are the derived
// special rows, then its union: half-block i of the item is a special one for i < nsh (every row
// keeps those keys), else union half-block i - nsh, whose mask words (one per item row) sit at a
// known place, so this thread loads its words for the next block while the current one runs.
__device__ __forceinline__ bool softmax_blocks_bits(const AttnParams& p, AttnSmem& sm, SoftmaxState& ss,
                                                    uint32_t tmem, ItemInfo& it, RowCtx& rc, float (&m)[2],
                                                    float (&l)[2]) {
  const Seg sp = it.w.list[0], un = it.w.list[1];
  const int nsh = (sp.len + 63) >> 6, nuh = (un.len + 63) >> 6;
  const uint64_t* gm = rc.gmask + static_cast<long long>(un.row0 >> 6) * kItemRows + rc.r;
  auto words = [&](int j, uint64_t& w0, uint64_t& w1) {
    const int u = 2 * j + rc.kh - nsh;
    if (u >= 0 && u < nuh) {
      w0 = gm[static_cast<long long>(u) * kItemRows];
      w1 = gm[static_cast<long long>(u) * kItemRows + 128];
    } else {
      w0 = w1 = ~0ull;
    }
  };
  uint64_t c0, c1;
  words(0, c0, c1);
  for (int j = 0; j < it.nblk; ++j) {
    uint64_t n0 = ~0ull, n1 = ~0ull;
    if (j + 1 < it.nblk) words(j + 1, n0, n1);
    const uint32_t c = ss.kv_c + j, st = c % kStages;
    if (!__all_sync(0xffffffffu, mbar_wait(&sm.v_full[st], (c / kStages) & 1, &sm.abort, p.err, p.wait_budget,
                                           SAF3R_ERR_TIMEOUT)))
      return false;
    const Half hb = sm.info[st][rc.kh];
    const uint64_t cnt = !hb.have ? 0ull : (hb.cnt >= 64 ? ~0ull : ((1ull << hb.cnt) - 1ull));
    if (!softmax_half<kMaskBits>(p, sm, ss, tmem, rc, 0, j, cnt & c0, m[0], l[0])) return false;
    if (!softmax_half<kMaskBits>(p, sm, ss, tmem, rc, 1, j, cnt & c1, m[1], l[1])) return false;
    c0 = n0;
    c1 = n1;
  }
  ss.kv_c += it.nblk;
  return true;
}

__device__ __forceinline__ void softmax_role(const AttnParams& p, AttnSmem& sm, uint32_t tmem, int warp, int lane) {
  volatile int* abort = &sm.abort;
  const long long budget = p.wait_budget;
  RowCtx rc;
  const int wq = warp & 3;
  rc.kh = (warp - 4) >> 2;
  rc.r = wq * 32 + lane;
  rc.lane = lane;
  rc.lane_off = static_cast<uint32_t>(wq * 32) << 16;
  rc.withhold = p.withhold_arrive != 0 && blockIdx.x == 0 && warp == 4;
  const int r = rc.r;
  SoftmaxState ss;
  bool ok = true;

  for (int item = blockIdx.x; ok && item < p.total_items; item += gridDim.x) {
    ItemInfo it = item_info(p, item);
    const HeadPlan& hp = p.heads[it.hi];
    float m[2] = {-INFINITY, -INFINITY};  // running max of this key half, log2 units, per tile
    float l[2] = {0.f, 0.f};              // running sum of this key half, per tile
    if (hp.q_src == 4) {
      rc.gmask = hp.gmask;
      ok = softmax_blocks_bits(p, sm, ss, tmem, it, rc, m, l);
    } else if (hp.kind == SAF3R_POSITION) {
      // neighbour cells of each tile row's grid cell, as kept derived rows [lo, hi)
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int qrow = it.q0 + t * 128 + r;
        const bool patch_row = qrow < p.P * p.S && p.S > 1;
        const int cell = patch_row ? qrow / p.S : 0;
        const int qr = cell / p.gw, qc = cell - qr * p.gw;
        const int R = hp.radius;
#pragma unroll
        for (int x = 0; x < kNbIntervals; ++x) {
          const int dr = x - kMaxRadius;
          const int rr = qr + dr;
          const bool use = patch_row && dr >= -R && dr <= R && rr >= 0 && rr < p.gh;
          const int ca = rr * p.gw + max(qc - R, 0);
          const int cb = rr * p.gw + min(qc + R, p.gw - 1);
          rc.nb_lo[t][x] = use ? hp.nb_base + ca * (p.S - 1) : 0;
          rc.nb_hi[t][x] = use ? hp.nb_base + (cb + 1) * (p.S - 1) : 0;
        }
      }
      ok = softmax_blocks<kMaskCells>(p, sm, ss, tmem, it, rc, m, l);
    } else if (hp.kind == SAF3R_CORR || hp.kind == SAF3R_HYBRID) {
      rc.lat_stride = hp.lat_stride;
      rc.lat_phase = hp.lat_phase;
      ok = softmax_blocks<kMaskTiles>(p, sm, ss, tmem, it, rc, m, l);
    } else {
      ok = softmax_blocks<kMaskPlain>(p, sm, ss, tmem, it, rc, m, l);
    }
    if (!ok) break;

    // epilogue: merge the two key halves of each row; the warp of key half kh writes tile kh
    const int t = rc.kh;
    if (!__all_sync(0xffffffffu, mbar_wait(&sm.o_done[t], ss.odone_c & 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT))) {
      ok = false;
      break;
    }
    ++ss.odone_c;
    tc_fence_after();
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
      sm.stats[rc.kh][tt][r][0] = m[tt];
      sm.stats[rc.kh][tt][r][1] = l[tt];
    }
    // meet the other warp of these rows (bounded waits: a partner that gave up cannot hang this one)
    mbar_arrive(&sm.pair[wq]);
    if (!__all_sync(0xffffffffu, mbar_wait(&sm.pair[wq], ss.pair_c & 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT))) {
      ok = false;
      break;
    }
    ++ss.pair_c;
    const float ma = sm.stats[0][t][r][0], la = sm.stats[0][t][r][1];
    const float mb = sm.stats[1][t][r][0], lb = sm.stats[1][t][r][1];
    mbar_arrive(&sm.pair[wq]);  // stats may be overwritten by the next item once both warps are past this
    if (!__all_sync(0xffffffffu, mbar_wait(&sm.pair[wq], ss.pair_c & 1, abort, p.err, budget, SAF3R_ERR_TIMEOUT))) {
      ok = false;
      break;
    }
    ++ss.pair_c;
    const float mmax = fmaxf(ma, mb);
    const float fa = ma == -INFINITY ? 0.f : fast_exp2(ma - mmax);
    const float fb = mb == -INFINITY ? 0.f : fast_exp2(mb - mmax);
    const float den = la * fa + lb * fb;
    const float ia = den > 0.f ? fa / den : 0.f, ib = den > 0.f ? fb / den : 0.f;
    uint32_t oa[2][32], ob[2][32];
    const uint32_t tO = tmem + rc.lane_off + t * 256 + 128;
    tmem_ld32(tO, oa[0]);
    tmem_ld32(tO + 32, oa[1]);
    tmem_ld32(tO + 64, ob[0]);
    tmem_ld32(tO + 96, ob[1]);
    tmem_wait_ld();
    tc_fence_before();
    float o[64];
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int i = 0; i < 32; ++i) o[c * 32 + i] = __uint_as_float(oa[c][i]) * ia + __uint_as_float(ob[c][i]) * ib;
    const int qrow = it.q0 + t * 128 + r;
    const int quarter = (t * 128 + r) >> 6;
    int token = -1;
    if (hp.q_src == 1) {
      if (qrow < p.N) token = position_token(p, qrow);
    } else if (hp.q_src == 3) {
      if (qrow < p.ns * p.S) token = position_token(p, p.P * p.S + qrow);  // the special tokens, view by view
    } else if (hp.q_src == 2) {
      const int u = mapped_tile(p, hp, it.local, quarter);
      if (u >= 0 && u * 64 + (r & 63) < p.N) token = u * 64 + (r & 63);
    } else if (hp.q_src == 4) {
      // a token-wise head's patch query, in the cached order
      if (qrow < p.P * p.S) {
        const int u = p.tok_perm[qrow];
        if (u >= 0 && u < p.P * p.S)
          token = (u / p.P) * p.V + p.ns + (u % p.P);
        else
          atomicCAS(p.err, 0, SAF3R_ERR_INDEX);
      }
    } else if (qrow < p.N) {
      token = qrow;
    }
    if (token >= 0) {
      const long long rowoff = (static_cast<long long>(hp.head) * p.N + token) * kD;
      if (p.out_fp32) {
        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + rowoff);
#pragma unroll
        for (int i = 0; i < 16; ++i) dst[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
      } else {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + rowoff);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          dst[i] = make_uint4(pack_bf16x2(o[8 * i], o[8 * i + 1]), pack_bf16x2(o[8 * i + 2], o[8 * i + 3]),
                              pack_bf16x2(o[8 * i + 4], o[8 * i + 5]), pack_bf16x2(o[8 * i + 6], o[8 * i + 7]));
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
      mbar_init(&sm.p_full[t], 8);
      mbar_init(&sm.o_done[t], 1);
    }
    for (int w = 0; w < 4; ++w) mbar_init(&sm.pair[w], 64);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.vg_go[s], 1);
      mbar_init(&sm.vg_done[s], 2);
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
    producer_role(p, sm, tmQ, tmK, tmV, tmQC, tmKC, tmVC, lane);
    __syncwarp();
  } else if (warp == 1) {
    mma_role(p, sm, tmem);
    __syncwarp();
  } else if (warp == 2 || warp == 3) {
    gather_role(p, sm, warp - 2, lane);
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
