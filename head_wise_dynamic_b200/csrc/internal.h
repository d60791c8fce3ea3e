// Host/device plan structures of the saf3r library (not part of the C ABI).
#pragma once
#include <cstdint>

#include "../../include/saf3r.h"

namespace saf3r {

constexpr int kD = 64;            // head dimension
constexpr int kTile = 64;         // DINO token tile
constexpr int kMaxHeads = 64;
constexpr int kItemRows = 256;    // query rows of one attention work item (two 128-row MMA tiles)
constexpr int kMaxRadius = 3;
constexpr int kTokenMaxDim = 384;  // DINO width the token-wise selection keeps in registers

constexpr uint32_t kCacheMagic = 0x52334653u;  // "SF3R"
// Teardown waits (copies already issued must land before a CTA exits) have their own fixed
// budget, independent of the per-call wait budget, so a short test budget cannot cut them off.
constexpr long long kDrainBudget = 1000000000LL;  // clock cycles (~0.5 s)
constexpr uint32_t kCacheVersion = 3;

// Heads whose keys include ranked DINO tiles (they share the cached tile lists), and heads
// whose keys include the stride lattice (they get the lattice as derived rows).
__host__ __device__ inline bool tile_kind(int type) { return type == SAF3R_CORR || type == SAF3R_HYBRID; }
__host__ __device__ inline bool lattice_kind(int type) { return type == SAF3R_SCAN || type == SAF3R_HYBRID; }

// Derived layout numbers.
struct Dims {
  int S, gh, gw, ns, H, dino_dim;
  int P, V, N, T;
};

inline Dims make_dims(const saf3r_layout& L) {
  Dims d;
  d.S = L.S; d.gh = L.grid_h; d.gw = L.grid_w; d.ns = L.n_special; d.H = L.H; d.dino_dim = L.dino_dim;
  d.P = L.grid_h * L.grid_w;
  d.V = d.P + L.n_special;
  d.N = L.S * d.V;
  d.T = (d.N + kTile - 1) / kTile;
  return d;
}

// Cache header (first 256 bytes of the index cache).
struct CacheHeader {
  uint32_t magic;
  uint32_t version;
  uint64_t hash;            // hash of (layout, cfg)
  int32_t N, T;
  int32_t corr_kmax;        // width of the ranked tile list (0 = none)
  int32_t corr_off;         // int32 offset of the ranked tile list
  int32_t order_off;        // int32 offset of the query-tile grouping order [T] (correspondence heads)
  int32_t tok_kmax;         // width of the token-wise per-frame lists (0 = none)
  int64_t tok_off;          // int32 offset of the token-wise lists [S*P][S][tok_kmax]
  int32_t probe_off[kMaxHeads];  // int32 offset of each probe head's key list (-1 = not a probe head)
};
static_assert(sizeof(CacheHeader) <= 512, "cache header too large");
constexpr int kCacheHeaderBytes = 512;

// A run of key rows of one head, fed to the attention kernel 64 rows at a time.
// src 0: the caller's K/V ([H][N][64], row = token); src 1: the head's derived
// rows in the workspace (row relative to the head's derived base); src 2: the tokens
// listed at the head's gathered-key list (entry row0 + i), rows copied from the caller's K/V.
struct Seg {
  int32_t src;
  int32_t row0;
  int32_t len;
  uint32_t flags;   // bits 0-3: member quarters of the 256-row item; bit 4: per-row cell mask;
                    // bits 8-15 / 16-23: [lo, hi) rows of the run excluded (special tokens inside a tile)
};
constexpr uint32_t kSegAllQuarters = 0xFu;
constexpr uint32_t kSegCellMask = 0x10u;

// Token-wise heads on the tensor cores.  The patch queries are ordered so that queries with
// the same best matches are neighbours (perm[i] = patch query row s*P + p of row i); each
// 256-row item then streams the union of its rows' per-frame keys, ascending by token, and
// every row keeps its own keys of that union through a bitmask.  One group per distinct
// per-frame budget k; int32 offsets into the cache:
//   tn_off: [items] union length U of each item
//   tu_off: [items][ucap] the union's tokens (entries [U, ucap) unused)
//   tm_off: [items][ucap / 64][256] uint64 masks: bit b of word (item, h, r) = row r keeps
//           union entry 64 h + b
struct TokTileGroup {
  int k;
  int ucap;  // a multiple of 64, at least every item's union
  long long tn_off, tu_off, tm_off;
};
__host__ __device__ inline int tok_tile_ucap(int S, int P, int k) {
  const long long per_frame = static_cast<long long>(k) * kItemRows < P ? static_cast<long long>(k) * kItemRows : P;
  return static_cast<int>((static_cast<long long>(S) * per_frame + 63) / 64 * 64);
}

// Per-head plan of one attention launch (kernel parameter).
struct HeadPlan {
  int32_t head;       // head index h in [0, H)
  int32_t kind;       // saf3r_head_type
  int32_t q_src;      // 0: caller Q rows are tokens; 1: derived cell-major Q rows (position heads);
                      // 2: caller Q, each 64-row quarter of an item is the query tile qmap[4*item + quarter];
                      // 3: derived Q rows of the special tokens only, view by view (token-wise heads);
                      // 4: derived Q rows of the patch queries in the order perm (token-wise heads)
  int32_t q_base;     // derived Q row base (q_src == 1); qmap offset (q_src == 2)
  int32_t kc_base;    // derived K/V row base
  int32_t n_items;    // work items (256 query rows each)
  int32_t item_begin; // first global item index
  int32_t seg_list;   // -1: one implicit segment (below); else Seg offset of item 0's list
  int32_t seg_cap;    // Seg entries per item
  int32_t cnt_list;   // offset of the per-item counts: [2*item] segments, [2*item + 1] 128-key blocks
  Seg seg;            // implicit segment
  int32_t radius;     // position heads
  int32_t nb_base;    // position heads: derived row where the cell-major neighbour rows start
  int32_t lat_stride; // hybrid heads: lattice keys inside a kept tile are counted in the derived run
  int32_t lat_phase;  //   (so the tile runs mask them); 0 = no lattice mask
  // q_src 4 (token-wise patch queries): the group's union tokens and row masks (see TokTileGroup)
  const int32_t* glist;
  const uint64_t* gmask;
};

struct AttnParams {
  int32_t n_heads;    // entries of heads[] (heads in launch order)
  int32_t total_items;
  int32_t S, gh, gw, ns, V, N, P;
  int32_t out_fp32;
  void* out;
  const Seg* segs;
  const int32_t* seg_counts;
  const int32_t* qmap;    // query-tile order of the correspondence heads (in the cache)
  int32_t T;              // 64-token tiles
  int* err;
  const int* ok_flag;  // nonzero: cache check passed (NULL: no check)
  long long wait_budget;
  int32_t withhold_arrive;  // test hook: CTA 0's first softmax warp withholds its first P-ready arrival
  const uint16_t* k_rows;   // the caller's K and V ([H][N][64] bf16): rows of gathered key runs
  const uint16_t* v_rows;
  const int32_t* tok_perm;  // patch query order of the token-wise heads (in the cache)
  HeadPlan heads[kMaxHeads];
};


// Token-wise correspondence heads (token_attn.cu): every patch query row has its own kept keys
// (the special-token rows, which keep every key, run in the tensor-core kernel as dense rows).
struct TokenAttnParams {
  int32_t n_heads;
  int32_t heads[kMaxHeads];   // head index h
  int32_t k[kMaxHeads];       // kept patch tokens per frame
  int32_t N, S, V, ns, P, tok_kmax;
  long long tok_off;          // int32 offset of the per-frame lists in the cache
  const uint16_t* q;
  const uint16_t* k_;
  const uint16_t* v;
  void* out;
  int32_t out_fp32;
  const int32_t* cache;
  const int* ok_flag;
  int* err;
};

// Tensor-core cosines of the token-wise selection (token_sim.cu): scores[r][c] (fp16, row
// stride ld halves) = unit16[r0 + r] . unit16[c] for r < rows, c < ld, over n_kc 64-feature slices.
struct TokenSimParams {
  int r0, rows;          // first query row of this chunk, rows in the chunk
  int n_rb, n_ct, n_kc;  // 128-row blocks, 256-column tiles, 64-feature slices
  long long ld;          // score row stride in halves (a multiple of 8, >= the candidate rows)
  uint16_t* scores;
  int* err;
  long long wait_budget;
};

// Selection plan (select.cu).
struct SelectPlan {
  int N, V, ns, P, T, dim;
  int n_probe;
  int probe_heads[kMaxHeads];
  int probe_k[kMaxHeads];
  int probe_off[kMaxHeads];
  int corr_kmax;
  int corr_off;
  int order_off;
  int S;
  int tok_kmax;             // token-wise heads: widest per-frame budget (0 = none)
  long long tok_off;
  long long tperm_off;      // token-wise query order [S*P] (-1: no tensor-core token plans)
  int n_tg;                 // token-wise union groups (one per distinct k)
  TokTileGroup tg[kMaxHeads];
  int num_sms;
  int* err;                 // device error word (bounded waits of the tensor-core kernels)
  long long wait_budget;
  CacheHeader header;
};

// One head's derived-row mapping (prep.cu).
struct DerivedHead {
  int head;
  int kind;
  int kc_begin;     // first global derived K/V row
  int n_rows;       // derived K/V rows of this head
  int qc_begin;     // first global derived Q row (position and token-wise heads), -1 if none
  int n_q;          // derived Q rows of this head
  int stride, phase, n_lat;  // scan heads
  int probe_off;    // cache int32 offset of the probe key list
  int off_list;     // scan heads: int offset of the off-lattice special list in the workspace
};

struct DerivedArgs {
  int n;                    // heads with derived rows
  int S, V, ns, P, N;
  long long tperm_off;      // token-wise heads: cache int32 offset of the patch query order
  long long kc_total;       // derived K/V rows
  long long qc_total;       // derived Q rows
  DerivedHead h[kMaxHeads];
};

}  // namespace saf3r

#include <cuda.h>
#include <cuda_runtime.h>

namespace saf3r {

// check_layout + check_cfg of the C ABI (api.cu): SAF3R_OK, SAF3R_ERR_INVALID or SAF3R_ERR_UNSUPPORTED
saf3r_status validate_layout_cfg(const saf3r_layout* L, const saf3r_head_cfg* cfg);

// launchers (each returns the launch error, if any)
size_t attn_smem_bytes();
cudaError_t launch_attention(const AttnParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                             const CUtensorMap& tmV, const CUtensorMap& tmQC, const CUtensorMap& tmKC,
                             const CUtensorMap& tmVC, int num_sms, cudaStream_t stream);
size_t select_workspace_bytes(int n_probe, int N, int T, int dim, bool corr, long long tok_rows, int tiles_P);
size_t token_rank_smem_bytes(int P, int kmax);
size_t token_sim_smem_bytes();
cudaError_t launch_token_sim(const TokenSimParams& p, const CUtensorMap& tm, int num_sms, cudaStream_t stream);
// [rows][cols] fp16, 64 x 128 boxes, 128-byte swizzle, zero fill out of range (api.cu)
bool make_map_f16_rows(CUtensorMap* m, const void* base, long long rows, int cols);
cudaError_t launch_select(const SelectPlan& sp, const uint16_t* q, const uint16_t* k, const float* dino,
                          int32_t* cache, uint8_t* ws, cudaStream_t stream, int* n_launch);
cudaError_t launch_cache_check(const void* cache, uint64_t hash, int N, int T, int* ok, int* err,
                               cudaStream_t stream);
cudaError_t launch_derived(const DerivedArgs& a, bool any_scan, const uint16_t* q, const uint16_t* k,
                           const uint16_t* v, const int32_t* cache, int* offlists, uint16_t* kc, uint16_t* vc,
                           uint16_t* qc, int* err, int num_sms, cudaStream_t stream, int* n_launch);
cudaError_t launch_plan_position(int n_items, int S, int gh, int gw, int ns, int N, int R, int cap, Seg* segs,
                                 int* counts, cudaStream_t stream);
cudaError_t launch_plan_corr(const int32_t* ranked, const int32_t* order, int kmax, int kt, int T, int N, int V,
                             int ns, int tail_len, Seg* segs, int cap, int* counts, int* err, cudaStream_t stream);
cudaError_t launch_token_attention(const TokenAttnParams& p, int num_sms, cudaStream_t stream);
// token-wise heads on the tensor cores (token_tiles.cu): does the union builder fit this layout;
// its workspace; the index-build launches (query order, then every group's unions and masks);
// the per-call key runs of every item: the nsp derived special rows, then the item's union
bool tok_tiles_fit(int P);
size_t tok_tiles_workspace_bytes(int S, int P);
cudaError_t launch_tok_tiles(const int32_t* lists, int S, int P, int V, int ns, int tok_kmax, long long tperm_off,
                             const TokTileGroup* tg, int n_tg, int32_t* cache, uint8_t* ws, int* err,
                             cudaStream_t stream, int* n_launch);
cudaError_t launch_plan_token(const int32_t* tn, int ucap, int n_items, int nsp, Seg* segs, int* counts, int* err,
                              cudaStream_t stream);
size_t nmse_workspace_bytes(int H);
cudaError_t launch_nmse(const float* full, const float* sparse, int H, long long per_head, double* part,
                        double* out, cudaStream_t stream);

}  // namespace saf3r
