// C ABI of the saf3r library: argument checks, cache and workspace layouts,
// TMA descriptors, launch orchestration and the offline profiling rule.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <vector>

#include "internal.h"


using namespace saf3r;

namespace {

__device__ int g_device_error;  // the one piece of library state: first device-side error since the last check

thread_local int t_launches = 0;
thread_local cudaEvent_t t_ev_start = nullptr, t_ev_stop = nullptr;

constexpr long long kWaitBudget = 4000000000LL;  // default: clock cycles (~2 s) before a device wait gives up
thread_local long long t_wait_budget = kWaitBudget;
thread_local bool t_withhold_arrive = false;       // test hook, consumed by the next attention launch

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// ------------------------------------------------------------------ devices
struct DeviceInfo {
  bool ok = false;
  int sms = 0;
  int major = 0;
  int* err = nullptr;
};

std::mutex g_mu;
std::map<int, DeviceInfo> g_devices;

bool device_info(DeviceInfo& out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_devices.find(dev);
  if (it != g_devices.end()) {
    out = it->second;
    return out.ok;
  }
  DeviceInfo d;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) == cudaSuccess) {
    d.sms = prop.multiProcessorCount;
    d.major = prop.major;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) == cudaSuccess) {
      d.err = static_cast<int*>(p);
      d.ok = true;
    }
  }
  g_devices[dev] = d;
  out = d;
  return d.ok;
}

// ------------------------------------------------------------------ TMA descriptors
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [H][rows][64] bf16 with 64x64 boxes, 128-byte swizzle, zero fill out of range.
bool make_map_3d(CUtensorMap* m, const void* base, long long rows, int H) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(H)};
  cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(rows) * 128};
  cuuint32_t box[3] = {64, 64, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_2d(CUtensorMap* m, const void* base, long long rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {64, static_cast<cuuint64_t>(rows < 1 ? 1 : rows)};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ validation
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

saf3r_status check_layout(const saf3r_layout* L) {
  if (!L) return SAF3R_ERR_INVALID;
  if (L->S < 1 || L->grid_h < 1 || L->grid_w < 1 || L->n_special < 0 || L->n_special > 63) return SAF3R_ERR_INVALID;
  if (L->H < 1 || L->H > kMaxHeads) return SAF3R_ERR_INVALID;
  if (L->tile != kTile || L->dino_dim < 4 || L->dino_dim > 1024 || (L->dino_dim & 3)) return SAF3R_ERR_INVALID;
  if (L->d != kD) return SAF3R_ERR_UNSUPPORTED;
  const long long P = static_cast<long long>(L->grid_h) * L->grid_w;
  const long long N = static_cast<long long>(L->S) * (P + L->n_special);
  if (P > (1 << 20) || N > (1 << 24)) return SAF3R_ERR_INVALID;
  return SAF3R_OK;
}

saf3r_status check_cfg(const Dims& d, const saf3r_head_cfg* cfg, int H) {
  if (!cfg) return SAF3R_ERR_INVALID;
  for (int h = 0; h < H; ++h) {
    const saf3r_head_cfg& c = cfg[h];
    switch (c.type) {
      case SAF3R_POSITION:
        if (c.radius < -1 || c.radius > kMaxRadius) return SAF3R_ERR_INVALID;
        break;
      case SAF3R_PROBE:
        if (c.k < 1 || c.k > d.S * d.P) return SAF3R_ERR_INVALID;
        break;
      case SAF3R_CORR:
        if (c.k < 1 || c.k > d.T || d.V < kTile + d.ns) return SAF3R_ERR_INVALID;
        break;
      case SAF3R_SCAN:
        if (c.stride < 1 || c.phase < 0 || c.phase >= c.stride || c.phase >= d.N) return SAF3R_ERR_INVALID;
        break;
      case SAF3R_HYBRID:
        if (c.k < 1 || c.k > d.T || d.V < kTile + d.ns) return SAF3R_ERR_INVALID;
        if (c.stride < 1 || c.phase < 0 || c.phase >= c.stride || c.phase >= d.N) return SAF3R_ERR_INVALID;
        break;
      case SAF3R_DENSE:
        break;
      case SAF3R_TOKEN:
        if (c.k < 1 || c.k > d.P) return SAF3R_ERR_INVALID;
        if (d.dino_dim > kTokenMaxDim || token_rank_smem_bytes(d.P, c.k) > 200 * 1024) return SAF3R_ERR_UNSUPPORTED;
        break;
      default:
        return SAF3R_ERR_INVALID;
    }
  }
  return SAF3R_OK;
}

uint64_t fnv1a(uint64_t h, const void* p, size_t n) {
  const uint8_t* b = static_cast<const uint8_t*>(p);
  for (size_t i = 0; i < n; ++i) {
    h ^= b[i];
    h *= 1099511628211ull;
  }
  return h;
}

// Hash of what the cache depends on: the layout and, per head, the kind and its selection parameter.
uint64_t cache_hash(const saf3r_layout* L, const saf3r_head_cfg* cfg) {
  uint64_t h = 1469598103934665603ull;
  h = fnv1a(h, L, sizeof(saf3r_layout));
  for (int i = 0; i < L->H; ++i) {
    const int32_t v[2] = {cfg[i].type,
                          (cfg[i].type == SAF3R_PROBE || tile_kind(cfg[i].type) || cfg[i].type == SAF3R_TOKEN) ? cfg[i].k
                                                                                                       : 0};
    h = fnv1a(h, v, sizeof(v));
  }
  return h;
}

// ------------------------------------------------------------------ cache layout
struct CacheLayout {
  int probe_off[kMaxHeads];
  int corr_off = 0;
  int corr_kmax = 0;
  int order_off = 0;
  int tok_kmax = 0;        // token-wise heads: widest per-frame budget
  long long tok_off = 0;   // int32 offset of the per-frame lists [S*P][S][tok_kmax]
  long long tperm_off = -1;  // token-wise heads on the tensor cores: patch query order [S*P] (-1: none)
  int n_tg = 0;              // their union groups, one per distinct per-frame budget
  TokTileGroup tg[kMaxHeads];
  int tg_of[kMaxHeads];      // per head: its group, or -1
  size_t bytes = 0;
};

// Token-wise heads run on the tensor cores when the union builder fits the layout and the
// unions' worst-case storage stays bounded (else the gather kernel takes their patch queries).
constexpr long long kTokTileMaxEntries = 1ll << 28;  // union entries over all items of a group

bool tok_tiles_on(const Dims& d, const saf3r_head_cfg* cfg) {
  if (!tok_tiles_fit(d.P)) return false;
  const long long items = (static_cast<long long>(d.S) * d.P + kItemRows - 1) / kItemRows;
  bool any = false;
  for (int h = 0; h < d.H; ++h) {
    if (cfg[h].type != SAF3R_TOKEN) continue;
    any = true;
    if (items * tok_tile_ucap(d.S, d.P, cfg[h].k) > kTokTileMaxEntries) return false;
  }
  return any;
}

CacheLayout cache_layout(const Dims& d, const saf3r_head_cfg* cfg) {
  CacheLayout c;
  size_t ints = kCacheHeaderBytes / 4;
  for (int h = 0; h < d.H; ++h) {
    c.probe_off[h] = -1;
    if (cfg[h].type == SAF3R_PROBE) {
      c.probe_off[h] = static_cast<int>(ints);
      ints += (cfg[h].k + 63) & ~63;
    }
    if (tile_kind(cfg[h].type)) c.corr_kmax = std::max(c.corr_kmax, cfg[h].k);
    if (cfg[h].type == SAF3R_TOKEN) c.tok_kmax = std::max(c.tok_kmax, cfg[h].k);
  }
  c.corr_off = static_cast<int>(ints);
  ints += static_cast<size_t>(d.T) * c.corr_kmax;
  c.order_off = static_cast<int>(ints);
  if (c.corr_kmax > 0) ints += static_cast<size_t>(d.T);
  ints = (ints + 63) & ~size_t(63);
  c.tok_off = static_cast<long long>(ints);
  ints += static_cast<size_t>(d.S) * d.P * d.S * c.tok_kmax;
  for (int h = 0; h < d.H; ++h) c.tg_of[h] = -1;
  if (tok_tiles_on(d, cfg)) {
    const size_t items = (static_cast<size_t>(d.S) * d.P + kItemRows - 1) / kItemRows;
    ints = (ints + 63) & ~size_t(63);
    c.tperm_off = static_cast<long long>(ints);
    ints += static_cast<size_t>(d.S) * d.P;
    for (int h = 0; h < d.H; ++h) {
      if (cfg[h].type != SAF3R_TOKEN) continue;
      int g = 0;
      while (g < c.n_tg && c.tg[g].k != cfg[h].k) ++g;
      if (g == c.n_tg) {
        TokTileGroup& t = c.tg[c.n_tg++];
        t.k = cfg[h].k;
        t.ucap = tok_tile_ucap(d.S, d.P, t.k);
        ints = (ints + 63) & ~size_t(63);
        t.tn_off = static_cast<long long>(ints);
        ints += items;
        ints = (ints + 63) & ~size_t(63);
        t.tu_off = static_cast<long long>(ints);
        ints += items * t.ucap;
        ints = (ints + 63) & ~size_t(63);
        t.tm_off = static_cast<long long>(ints);
        ints += items * (t.ucap / 64) * kItemRows * 2;
      }
      c.tg_of[h] = g;
    }
  }
  c.bytes = align256(ints * 4);
  return c;
}

// ------------------------------------------------------------------ sparse workspace layout
struct SparseLayout {
  size_t ok_off = 0, kc_off = 0, vc_off = 0, qc_off = 0, offl_off = 0, seg_off = 0, cnt_off = 0, total = 0;
  long long kc_rows = 0, qc_rows = 0, seg_total = 0, cnt_total = 0;
  int off_total = 0;
  std::vector<int> kc_begin, n_rows, qc_begin, n_q, n_lat, n_off, off_list;
  // token-wise heads whose patch queries run in the tensor-core kernel (one extra plan each, while
  // the plans fit; the gather kernel takes the others)
  std::vector<int> use_tile;
  // shared plan lists
  struct List {
    int kind, param, tail, cap, n_items;  // tail: rows of the derived run that ends every item (tile lists)
    int grp;                              // token-wise lists: the union group
    long long seg_begin, cnt_begin;
  };
  std::vector<List> lists;
  std::vector<int> list_of;  // per head: index into lists, or -1
};

int items_of(int N) { return (N + kItemRows - 1) / kItemRows; }

int position_cap(const Dims& d, int R) {
  const int cells = (kItemRows + d.S - 1) / d.S + 1;
  const int rows = (cells + d.gw - 1) / d.gw + 1;
  return 1 + 2 * (rows + 2 * R) + 1;
}

SparseLayout sparse_layout(const Dims& d, const saf3r_head_cfg* cfg) {
  SparseLayout s;
  const int H = d.H;
  s.kc_begin.assign(H, 0);
  s.n_rows.assign(H, 0);
  s.qc_begin.assign(H, -1);
  s.n_q.assign(H, 0);
  s.n_lat.assign(H, 0);
  s.n_off.assign(H, 0);
  s.off_list.assign(H, 0);
  s.list_of.assign(H, -1);
  s.use_tile.assign(H, 0);
  const int nsp = d.ns * d.S;
  const CacheLayout cl = cache_layout(d, cfg);
  if (cl.tperm_off >= 0) {
    int plans = 0;  // plans of the tensor-core kernel without the extra ones
    for (int h = 0; h < H; ++h) plans += cfg[h].type != SAF3R_TOKEN || nsp > 0;
    for (int h = 0; h < H; ++h)
      if (cfg[h].type == SAF3R_TOKEN && plans < kMaxHeads) {
        s.use_tile[h] = 1;
        ++plans;
      }
  }
  for (int h = 0; h < H; ++h) {
    const saf3r_head_cfg& c = cfg[h];
    int rows = 0;
    switch (c.type) {
      case SAF3R_POSITION:
        rows = nsp + d.P + d.P * (d.S - 1);
        s.qc_begin[h] = static_cast<int>(s.qc_rows);
        s.n_q[h] = d.N;
        s.qc_rows += d.N;
        break;
      case SAF3R_PROBE:
        rows = nsp + c.k;
        break;
      case SAF3R_TOKEN:  // the special-token queries, gathered for the tensor-core kernel; with a
                         // tensor-core plan for the patch queries, also those (in the cached order)
                         // and the special keys
        s.n_q[h] = nsp + (s.use_tile[h] ? d.S * d.P : 0);
        if (s.n_q[h] > 0) {
          s.qc_begin[h] = static_cast<int>(s.qc_rows);
          s.qc_rows += s.n_q[h];
        }
        if (s.use_tile[h]) rows = nsp;
        break;
      case SAF3R_SCAN:
      case SAF3R_HYBRID: {  // the lattice, then the specials off it
        s.n_lat[h] = (d.N - c.phase + c.stride - 1) / c.stride;
        int off = 0;
        for (int sv = 0; sv < d.S; ++sv)
          for (int i = 0; i < d.ns; ++i)
            if (((sv * d.V + i) % c.stride) != c.phase) ++off;
        s.n_off[h] = off;
        s.off_list[h] = s.off_total;
        s.off_total += off;
        rows = s.n_lat[h] + off;
        break;
      }
      case SAF3R_CORR:
        rows = nsp;
        break;
      default:
        rows = 0;
    }
    s.kc_begin[h] = static_cast<int>(s.kc_rows);
    s.n_rows[h] = rows;
    s.kc_rows += rows;
    if (s.use_tile[h]) {
      const int g = cl.tg_of[h];
      int found = -1;
      for (size_t i = 0; i < s.lists.size(); ++i)
        if (s.lists[i].kind == SAF3R_TOKEN && s.lists[i].grp == g) found = static_cast<int>(i);
      if (found < 0) {
        SparseLayout::List l;
        l.kind = SAF3R_TOKEN;
        l.param = c.k;
        l.tail = nsp;
        l.grp = g;
        l.n_items = items_of(d.S * d.P);
        l.cap = 2;
        l.seg_begin = s.seg_total;
        l.cnt_begin = s.cnt_total;
        s.seg_total += static_cast<long long>(l.cap) * l.n_items;
        s.cnt_total += 2 * l.n_items;
        s.lists.push_back(l);
        found = static_cast<int>(s.lists.size()) - 1;
      }
      s.list_of[h] = found;
    }
    if (c.type == SAF3R_POSITION || tile_kind(c.type)) {
      // tile heads share a list when their budget and derived-run length agree (the lattice
      // masks of a hybrid head are applied in the kernel, not stored in the list)
      const int kind = c.type == SAF3R_POSITION ? SAF3R_POSITION : SAF3R_CORR;
      const int param = c.type == SAF3R_POSITION ? c.radius : c.k;
      const int tail = c.type == SAF3R_POSITION ? 0 : rows;
      int found = -1;
      for (size_t i = 0; i < s.lists.size(); ++i)
        if (s.lists[i].kind == kind && s.lists[i].param == param && s.lists[i].tail == tail)
          found = static_cast<int>(i);
      if (found < 0) {
        SparseLayout::List l;
        l.kind = kind;
        l.param = param;
        l.tail = tail;
        l.grp = -1;
        l.n_items = c.type == SAF3R_POSITION ? items_of(d.N) : (d.T + 3) / 4;
        l.cap = c.type == SAF3R_POSITION ? position_cap(d, c.radius) : 4 * c.k + 1;
        l.seg_begin = s.seg_total;
        l.cnt_begin = s.cnt_total;
        s.seg_total += static_cast<long long>(l.cap) * l.n_items;
        s.cnt_total += 2 * l.n_items;  // per item: segments, then 128-key blocks
        s.lists.push_back(l);
        found = static_cast<int>(s.lists.size()) - 1;
      }
      s.list_of[h] = found;
    }
  }
  size_t off = 256;  // ok flag
  s.ok_off = 0;
  s.kc_off = off;
  off = align256(off + static_cast<size_t>(s.kc_rows) * 128);
  s.vc_off = off;
  off = align256(off + static_cast<size_t>(s.kc_rows) * 128);
  s.qc_off = off;
  off = align256(off + static_cast<size_t>(s.qc_rows) * 128);
  s.offl_off = off;
  off = align256(off + static_cast<size_t>(s.off_total) * 4);
  s.seg_off = off;
  off = align256(off + static_cast<size_t>(s.seg_total) * sizeof(Seg));
  s.cnt_off = off;
  off = align256(off + static_cast<size_t>(s.cnt_total) * 4);
  s.total = off;
  return s;
}

// estimated kept keys per query row (launch order: most expensive heads first)
double est_keys(const Dims& d, const saf3r_head_cfg& c, const SparseLayout& s, int h) {
  switch (c.type) {
    case SAF3R_POSITION:
      return d.ns * d.S + d.P + 12.0 * (d.S - 1);
    case SAF3R_PROBE:
    case SAF3R_SCAN:
      return s.n_rows[h];
    case SAF3R_CORR:
      return 1.5 * kTile * c.k + d.ns * d.S;
    case SAF3R_HYBRID:
      return 1.5 * kTile * c.k + s.n_rows[h];
    case SAF3R_TOKEN:  // the patch queries' plan: the specials, then about twelve times the
                       // per-frame budget per frame in an item's union
      return d.ns * d.S + 12.0 * d.S * c.k;
    default:
      return d.N;
  }
}

saf3r_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SAF3R_OK : SAF3R_ERR_CUDA; }

saf3r_status prepare_device(DeviceInfo& dev) {
  if (!device_info(dev)) return SAF3R_ERR_CUDA;
  if (dev.major != 10) return SAF3R_ERR_UNSUPPORTED;
  return SAF3R_OK;
}

// Attention over the heads of `cfg` (which may all be DENSE), writing `out`.
saf3r_status run_attention(const saf3r_layout* L, const saf3r_head_cfg* cfg, const void* cache, const void* q,
                           const void* k, const void* v, void* out, int out_is_fp32, void* workspace,
                           cudaStream_t stream) {
  DeviceInfo dev;
  saf3r_status st = prepare_device(dev);
  if (st != SAF3R_OK) return st;
  const Dims d = make_dims(*L);
  const SparseLayout s = sparse_layout(d, cfg);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* ok_flag = cache ? reinterpret_cast<int*>(ws + s.ok_off) : nullptr;
  uint16_t* kc = reinterpret_cast<uint16_t*>(ws + s.kc_off);
  uint16_t* vc = reinterpret_cast<uint16_t*>(ws + s.vc_off);
  uint16_t* qc = reinterpret_cast<uint16_t*>(ws + s.qc_off);
  int* offl = reinterpret_cast<int*>(ws + s.offl_off);
  Seg* segs = reinterpret_cast<Seg*>(ws + s.seg_off);
  int* cnts = reinterpret_cast<int*>(ws + s.cnt_off);
  const CacheLayout cl = cache_layout(d, cfg);
  const int32_t* cache_i = static_cast<const int32_t*>(cache);
  int launches = 0;

  if (cache) {
    st = cuda_status(launch_cache_check(cache, cache_hash(L, cfg), d.N, d.T, ok_flag, dev.err, stream));
    ++launches;
    if (st != SAF3R_OK) return st;
  }

  // derived rows
  DerivedArgs da;
  std::memset(&da, 0, sizeof(da));
  da.S = d.S; da.V = d.V; da.ns = d.ns; da.P = d.P; da.N = d.N;
  da.tperm_off = cl.tperm_off;
  bool any_scan = false;
  for (int h = 0; h < d.H; ++h) {
    if (s.n_rows[h] == 0 && s.qc_begin[h] < 0) continue;
    DerivedHead& x = da.h[da.n++];
    x.head = h;
    x.kind = cfg[h].type;
    x.kc_begin = s.kc_begin[h];
    x.n_rows = s.n_rows[h];
    x.qc_begin = s.qc_begin[h];
    x.n_q = s.n_q[h];
    x.stride = cfg[h].stride;
    x.phase = cfg[h].phase;
    x.n_lat = s.n_lat[h];
    x.probe_off = cl.probe_off[h];
    x.off_list = s.off_list[h];
    any_scan |= lattice_kind(cfg[h].type);
  }
  da.kc_total = s.kc_rows;
  da.qc_total = s.qc_rows;
  if (da.n > 0) {
    st = cuda_status(launch_derived(da, any_scan, static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k),
                                    static_cast<const uint16_t*>(v), cache_i, offl, kc, vc, qc, dev.err, dev.sms,
                                    stream, &launches));
    if (st != SAF3R_OK) return st;
  }
  // plans
  for (const auto& l : s.lists) {
    if (l.kind == SAF3R_POSITION) {
      st = cuda_status(launch_plan_position(l.n_items, d.S, d.gh, d.gw, d.ns, d.N, l.param, l.cap,
                                            segs + l.seg_begin, cnts + l.cnt_begin, stream));
    } else if (l.kind == SAF3R_TOKEN) {
      const TokTileGroup& g = cl.tg[l.grp];
      st = cuda_status(launch_plan_token(cache_i + g.tn_off, g.ucap, l.n_items, l.tail, segs + l.seg_begin,
                                         cnts + l.cnt_begin, dev.err, stream));
    } else {
      st = cuda_status(launch_plan_corr(cache_i + cl.corr_off, cache_i + cl.order_off, cl.corr_kmax, l.param, d.T,
                                        d.N, d.V, d.ns, l.tail, segs + l.seg_begin, l.cap, cnts + l.cnt_begin,
                                        dev.err, stream));
    }
    ++launches;
    if (st != SAF3R_OK) return st;
  }

  // attention
  AttnParams p;
  std::memset(&p, 0, sizeof(p));
  // every head runs here; a token-wise head has two plans: its special-token queries (every key:
  // dense rows) and its patch queries (the cached order, each item over the special keys and
  // its rows' union of per-frame keys).  A token-wise head whose second plan does not fit the
  // plan array has its patch queries run in the gather kernel instead
  struct PlanRef {
    int h;
    bool part;  // a token-wise head's patch queries
  };
  std::vector<PlanRef> order;
  TokenAttnParams tp;
  std::memset(&tp, 0, sizeof(tp));
  const int nsp = d.ns * d.S;
  for (int h = 0; h < d.H; ++h) {
    if (cfg[h].type == SAF3R_TOKEN) {
      if (s.use_tile[h]) {
        order.push_back({h, true});
      } else {
        tp.heads[tp.n_heads] = h;
        tp.k[tp.n_heads] = cfg[h].k;
        ++tp.n_heads;
      }
      if (nsp > 0) order.push_back({h, false});
    } else {
      order.push_back({h, false});
    }
  }
  auto plan_keys = [&](const PlanRef& r) {
    return (cfg[r.h].type == SAF3R_TOKEN && !r.part) ? static_cast<double>(d.N) : est_keys(d, cfg[r.h], s, r.h);
  };
  std::stable_sort(order.begin(), order.end(),
                   [&](const PlanRef& a, const PlanRef& b) { return plan_keys(a) > plan_keys(b); });
  const int n_main = static_cast<int>(order.size());
  int item = 0;
  for (int i = 0; i < n_main; ++i) {
    const int h = order[i].h;
    const bool part = order[i].part;
    const saf3r_head_cfg& c = cfg[h];
    HeadPlan& hp = p.heads[i];
    hp.head = h;
    hp.kind = c.type;
    hp.q_src = part ? 4 : (c.type == SAF3R_POSITION ? 1 : (tile_kind(c.type) ? 2 : (c.type == SAF3R_TOKEN ? 3 : 0)));
    hp.q_base = part ? s.qc_begin[h] + nsp
                     : (tile_kind(c.type) ? cl.order_off : (s.qc_begin[h] < 0 ? 0 : s.qc_begin[h]));
    hp.lat_stride = c.type == SAF3R_HYBRID ? c.stride : 0;
    hp.lat_phase = c.type == SAF3R_HYBRID ? c.phase : 0;
    hp.kc_base = s.kc_begin[h];
    hp.n_items = c.type == SAF3R_TOKEN ? items_of(part ? d.S * d.P : nsp) : items_of(d.N);
    hp.item_begin = item;
    item += hp.n_items;
    hp.seg_list = -1;
    hp.seg_cap = 0;
    hp.cnt_list = 0;
    hp.radius = c.radius;
    hp.nb_base = d.ns * d.S + d.P;
    hp.glist = nullptr;
    hp.gmask = nullptr;
    if (part) {
      // per item: the head's derived special rows, then the union of its rows' per-frame keys
      const TokTileGroup& g = cl.tg[cl.tg_of[h]];
      const auto& l = s.lists[s.list_of[h]];
      hp.seg_list = static_cast<int>(l.seg_begin);
      hp.seg_cap = l.cap;
      hp.cnt_list = static_cast<int>(l.cnt_begin);
      hp.seg = Seg{0, 0, 0, 0};
      hp.glist = cache_i + g.tu_off;
      hp.gmask = reinterpret_cast<const uint64_t*>(cache_i + g.tm_off);
      continue;
    }
    switch (c.type) {
      case SAF3R_PROBE:
      case SAF3R_SCAN:
        hp.seg = Seg{1, 0, s.n_rows[h], kSegAllQuarters};
        break;
      case SAF3R_DENSE:
      case SAF3R_TOKEN:  // special-token queries of a token-wise head keep every key
        hp.seg = Seg{0, 0, d.N, kSegAllQuarters};
        break;
      default: {
        const auto& l = s.lists[s.list_of[h]];
        hp.seg_list = static_cast<int>(l.seg_begin);
        hp.seg_cap = l.cap;
        hp.cnt_list = static_cast<int>(l.cnt_begin);
        hp.seg = Seg{0, 0, 0, 0};
      }
    }
  }
  p.n_heads = n_main;
  p.total_items = item;
  p.S = d.S; p.gh = d.gh; p.gw = d.gw; p.ns = d.ns; p.V = d.V; p.N = d.N; p.P = d.P;
  p.out_fp32 = out_is_fp32 ? 1 : 0;
  p.out = out;
  p.segs = segs;
  p.seg_counts = cnts;
  p.qmap = cache_i;
  p.T = d.T;
  p.err = dev.err;
  p.ok_flag = ok_flag;
  p.wait_budget = t_wait_budget;
  p.withhold_arrive = t_withhold_arrive ? 1 : 0;
  t_withhold_arrive = false;
  p.k_rows = static_cast<const uint16_t*>(k);
  p.v_rows = static_cast<const uint16_t*>(v);
  p.tok_perm = cl.tperm_off >= 0 && cache_i ? cache_i + cl.tperm_off : nullptr;

  if (t_ev_start && t_ev_stop && cudaEventRecord(t_ev_start, stream) != cudaSuccess) return SAF3R_ERR_CUDA;
  if (n_main > 0) {
    CUtensorMap tq, tk, tv, tqc, tkc, tvc;
    if (!make_map_3d(&tq, q, d.N, d.H) || !make_map_3d(&tk, k, d.N, d.H) || !make_map_3d(&tv, v, d.N, d.H))
      return SAF3R_ERR_CUDA;
    const void* kc_base = s.kc_rows > 0 ? static_cast<const void*>(kc) : k;
    const void* vc_base = s.kc_rows > 0 ? static_cast<const void*>(vc) : v;
    const void* qc_base = s.qc_rows > 0 ? static_cast<const void*>(qc) : q;
    if (!make_map_2d(&tkc, kc_base, s.kc_rows > 0 ? s.kc_rows : 1) ||
        !make_map_2d(&tvc, vc_base, s.kc_rows > 0 ? s.kc_rows : 1) ||
        !make_map_2d(&tqc, qc_base, s.qc_rows > 0 ? s.qc_rows : 1))
      return SAF3R_ERR_CUDA;
    st = cuda_status(launch_attention(p, tq, tk, tv, tqc, tkc, tvc, dev.sms, stream));
    ++launches;
    if (st != SAF3R_OK) return st;
  }
  if (tp.n_heads > 0) {
    tp.N = d.N; tp.S = d.S; tp.V = d.V; tp.ns = d.ns; tp.P = d.P;
    tp.tok_kmax = cl.tok_kmax;
    tp.tok_off = cl.tok_off;
    tp.q = static_cast<const uint16_t*>(q);
    tp.k_ = static_cast<const uint16_t*>(k);
    tp.v = static_cast<const uint16_t*>(v);
    tp.out = out;
    tp.out_fp32 = out_is_fp32 ? 1 : 0;
    tp.cache = cache_i;
    tp.ok_flag = ok_flag;
    tp.err = dev.err;
    st = cuda_status(launch_token_attention(tp, dev.sms, stream));
    ++launches;
    if (st != SAF3R_OK) return st;
  }
  if (t_ev_start && t_ev_stop && cudaEventRecord(t_ev_stop, stream) != cudaSuccess) return SAF3R_ERR_CUDA;
  t_launches += launches;
  return st;
}

}  // namespace

saf3r_status saf3r::validate_layout_cfg(const saf3r_layout* L, const saf3r_head_cfg* cfg) {
  const saf3r_status st = check_layout(L);
  if (st != SAF3R_OK) return st;
  return check_cfg(make_dims(*L), cfg, L->H);
}

bool saf3r::make_map_f16_rows(CUtensorMap* m, const void* base, long long rows, int cols) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows < 1 ? 1 : rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ======================================================================== C ABI
extern "C" {

const char* saf3r_status_string(saf3r_status s) {
  switch (s) {
    case SAF3R_OK: return "ok";
    case SAF3R_ERR_INVALID: return "invalid argument or cache/layout mismatch";
    case SAF3R_ERR_CUDA: return "CUDA error";
    case SAF3R_ERR_TIMEOUT: return "device wait timed out";
    case SAF3R_ERR_INDEX: return "cached index out of range";
    case SAF3R_ERR_UNSUPPORTED: return "unsupported shape or device";
  }
  return "unknown status";
}

int saf3r_last_launch_count(void) { return t_launches; }

void saf3r_set_kernel_events(void* start, void* stop) {
  t_ev_start = static_cast<cudaEvent_t>(start);
  t_ev_stop = static_cast<cudaEvent_t>(stop);
}

void saf3r_set_wait_budget(long long cycles) { t_wait_budget = cycles > 0 ? cycles : kWaitBudget; }

void saf3r_test_withhold_arrive(void) { t_withhold_arrive = true; }

int32_t saf3r_baseline_stride(double sigma) {
  if (!(sigma >= 0.0 && sigma < 1.0)) return -1;
  // the smallest s with sparsity 1 - 1/s >= sigma (the 1e-12 absorbs the rounding of 1 - 1/s)
  int32_t s = 1;
  while (1.0 - 1.0 / s < sigma - 1e-12) ++s;
  return s;
}

size_t saf3r_cache_bytes(const saf3r_layout* L, const saf3r_head_cfg* cfg) {
  if (check_layout(L) != SAF3R_OK) return 0;
  const Dims d = make_dims(*L);
  if (check_cfg(d, cfg, L->H) != SAF3R_OK) return 0;
  return cache_layout(d, cfg).bytes;
}

size_t saf3r_workspace_bytes(const saf3r_layout* L, const saf3r_head_cfg* cfg, int op) {
  if (check_layout(L) != SAF3R_OK) return 0;
  const Dims d = make_dims(*L);
  if (op == SAF3R_OP_DENSE) return 256;
  if (check_cfg(d, cfg, L->H) != SAF3R_OK) return 0;
  if (op == SAF3R_OP_SELECT) {
    int n_probe = 0;
    bool corr = false, tok = false;
    for (int h = 0; h < d.H; ++h) {
      n_probe += cfg[h].type == SAF3R_PROBE;
      corr |= tile_kind(cfg[h].type);
      tok |= cfg[h].type == SAF3R_TOKEN;
    }
    return select_workspace_bytes(n_probe, d.N, d.T, d.dino_dim, corr, tok ? static_cast<long long>(d.S) * d.P : 0,
                                  cache_layout(d, cfg).tperm_off >= 0 ? d.P : 0);
  }
  if (op == SAF3R_OP_SPARSE) return sparse_layout(d, cfg).total;
  return 0;
}

saf3r_status saf3r_select_kv(const saf3r_layout* L, const saf3r_head_cfg* cfg, const void* q, const void* k,
                             const float* dino, void* cache, void* workspace, void* stream) {
  t_launches = 0;
  saf3r_status st = check_layout(L);
  if (st != SAF3R_OK) return st;
  const Dims d = make_dims(*L);
  if ((st = check_cfg(d, cfg, L->H)) != SAF3R_OK) return st;
  bool corr = false;
  for (int h = 0; h < d.H; ++h) corr |= tile_kind(cfg[h].type) || cfg[h].type == SAF3R_TOKEN;
  if (!q || !k || !cache || !workspace || !aligned16(q) || !aligned16(k) || !aligned16(cache) ||
      !aligned16(workspace) || (corr && (!dino || !aligned16(dino))))
    return SAF3R_ERR_INVALID;
  DeviceInfo dev;
  if ((st = prepare_device(dev)) != SAF3R_OK) return st;
  const CacheLayout cl = cache_layout(d, cfg);
  SelectPlan sp;
  std::memset(&sp, 0, sizeof(sp));
  sp.N = d.N; sp.V = d.V; sp.ns = d.ns; sp.P = d.P; sp.T = d.T; sp.dim = d.dino_dim;
  for (int h = 0; h < d.H; ++h) {
    if (cfg[h].type == SAF3R_PROBE) {
      sp.probe_heads[sp.n_probe] = h;
      sp.probe_k[sp.n_probe] = cfg[h].k;
      sp.probe_off[sp.n_probe] = cl.probe_off[h];
      ++sp.n_probe;
    }
  }
  sp.corr_kmax = cl.corr_kmax;
  sp.corr_off = cl.corr_off;
  sp.order_off = cl.order_off;
  sp.S = d.S;
  sp.tok_kmax = cl.tok_kmax;
  sp.tok_off = cl.tok_off;
  sp.tperm_off = cl.tperm_off;
  sp.n_tg = cl.n_tg;
  for (int g = 0; g < cl.n_tg; ++g) sp.tg[g] = cl.tg[g];
  sp.num_sms = dev.sms;
  sp.err = dev.err;
  sp.wait_budget = t_wait_budget;
  CacheHeader& hd = sp.header;
  std::memset(&hd, 0, sizeof(hd));
  hd.magic = kCacheMagic;
  hd.version = kCacheVersion;
  hd.hash = cache_hash(L, cfg);
  hd.N = d.N;
  hd.T = d.T;
  hd.corr_kmax = cl.corr_kmax;
  hd.corr_off = cl.corr_off;
  hd.order_off = cl.order_off;
  hd.tok_kmax = cl.tok_kmax;
  hd.tok_off = cl.tok_off;
  for (int h = 0; h < kMaxHeads; ++h) hd.probe_off[h] = h < d.H ? cl.probe_off[h] : -1;
  int launches = 0;
  cudaError_t e = launch_select(sp, static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k), dino,
                                static_cast<int32_t*>(cache), static_cast<uint8_t*>(workspace),
                                static_cast<cudaStream_t>(stream), &launches);
  t_launches = launches;
  return cuda_status(e);
}

saf3r_status saf3r_sparse_attn(const saf3r_layout* L, const saf3r_head_cfg* cfg, const void* cache, const void* q,
                               const void* k, const void* v, void* out, int out_is_fp32, void* workspace,
                               void* stream) {
  t_launches = 0;
  saf3r_status st = check_layout(L);
  if (st != SAF3R_OK) return st;
  const Dims d = make_dims(*L);
  if ((st = check_cfg(d, cfg, L->H)) != SAF3R_OK) return st;
  if (!cache || !q || !k || !v || !out || !workspace || !aligned16(cache) || !aligned16(q) || !aligned16(k) ||
      !aligned16(v) || !aligned16(out) || !aligned16(workspace))
    return SAF3R_ERR_INVALID;
  return run_attention(L, cfg, cache, q, k, v, out, out_is_fp32, workspace, static_cast<cudaStream_t>(stream));
}

saf3r_status saf3r_dense_attn(const saf3r_layout* L, const void* q, const void* k, const void* v, void* out,
                              int out_is_fp32, void* workspace, void* stream) {
  t_launches = 0;
  saf3r_status st = check_layout(L);
  if (st != SAF3R_OK) return st;
  if (!q || !k || !v || !out || !workspace || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      !aligned16(workspace))
    return SAF3R_ERR_INVALID;
  std::vector<saf3r_head_cfg> cfg(L->H, saf3r_head_cfg{SAF3R_DENSE, 0, 0, 0, 0});
  return run_attention(L, cfg.data(), nullptr, q, k, v, out, out_is_fp32, workspace,
                       static_cast<cudaStream_t>(stream));
}

saf3r_status saf3r_check(void* stream) {
  DeviceInfo dev;
  if (!device_info(dev)) return SAF3R_ERR_CUDA;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SAF3R_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return SAF3R_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return SAF3R_ERR_CUDA;
  }
  return static_cast<saf3r_status>(v);
}

saf3r_status saf3r_cache_export(const saf3r_layout* L, const saf3r_head_cfg* cfg, const void* cache, int head,
                                int32_t* host_idx, size_t cap, size_t* n, void* stream) {
  saf3r_status st = check_layout(L);
  if (st != SAF3R_OK) return st;
  const Dims d = make_dims(*L);
  if ((st = check_cfg(d, cfg, L->H)) != SAF3R_OK) return st;
  if (!cache || !n || head < 0 || head >= d.H) return SAF3R_ERR_INVALID;
  const CacheLayout cl = cache_layout(d, cfg);
  const saf3r_head_cfg& c = cfg[head];
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SAF3R_ERR_CUDA;
  const int32_t* base = static_cast<const int32_t*>(cache);
  if (c.type == SAF3R_PROBE) {
    *n = static_cast<size_t>(c.k);
    const size_t m = std::min(cap, *n);
    if (m && cudaMemcpy(host_idx, base + cl.probe_off[head], m * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
      return SAF3R_ERR_CUDA;
    return SAF3R_OK;
  }
  if (c.type == SAF3R_TOKEN) {
    const size_t rows = static_cast<size_t>(d.S) * d.P * d.S;  // (query patch, frame) pairs
    *n = rows * c.k;
    if (!host_idx) return SAF3R_OK;
    std::vector<int32_t> all(rows * cl.tok_kmax);
    if (cudaMemcpy(all.data(), base + cl.tok_off, all.size() * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
      return SAF3R_ERR_CUDA;
    size_t w = 0;
    for (size_t u = 0; u < rows && w < cap; ++u)
      for (int r = 0; r < c.k && w < cap; ++r) host_idx[w++] = all[u * cl.tok_kmax + r];
    return SAF3R_OK;
  }
  if (tile_kind(c.type)) {
    *n = static_cast<size_t>(d.T) * c.k;
    if (!host_idx) return SAF3R_OK;
    std::vector<int32_t> all(static_cast<size_t>(d.T) * cl.corr_kmax);
    if (cudaMemcpy(all.data(), base + cl.corr_off, all.size() * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
      return SAF3R_ERR_CUDA;
    size_t w = 0;
    for (int u = 0; u < d.T && w < cap; ++u)
      for (int r = 0; r < c.k && w < cap; ++r) host_idx[w++] = all[static_cast<size_t>(u) * cl.corr_kmax + r];
    return SAF3R_OK;
  }
  return SAF3R_ERR_INVALID;
}

// ---------------------------------------------------------------- profiling (section 4.2)

static saf3r_head_cfg apply_candidate(const saf3r_head_cfg& c, int h) {
  saf3r_head_cfg r = c;
  if (lattice_kind(c.type)) r.phase = h % c.stride;
  return r;
}

size_t saf3r_profile_workspace_bytes(const saf3r_layout* L, const saf3r_head_cfg* cand, int n_cand) {
  if (check_layout(L) != SAF3R_OK || !cand || n_cand < 1) return 0;
  const Dims d = make_dims(*L);
  size_t cache_max = 0, sel_max = 0, sp_max = 0;
  std::vector<saf3r_head_cfg> cfg(d.H);
  for (int c = 0; c < n_cand; ++c) {
    for (int h = 0; h < d.H; ++h) cfg[h] = apply_candidate(cand[c], h);
    if (check_cfg(d, cfg.data(), d.H) != SAF3R_OK) return 0;
    cache_max = std::max(cache_max, cache_layout(d, cfg.data()).bytes);
    sel_max = std::max(sel_max, saf3r_workspace_bytes(L, cfg.data(), SAF3R_OP_SELECT));
    sp_max = std::max(sp_max, saf3r_workspace_bytes(L, cfg.data(), SAF3R_OP_SPARSE));
  }
  const size_t out_bytes = align256(static_cast<size_t>(d.H) * d.N * kD * sizeof(float));
  return 2 * out_bytes + align256(cache_max) + align256(std::max(sel_max, sp_max)) +
         align256(nmse_workspace_bytes(d.H)) + align256(static_cast<size_t>(n_cand) * d.H * 2 * sizeof(double));
}

static long long pairs_of(const Dims& d, const saf3r_head_cfg& c, const std::vector<int32_t>& ranked, int kmax) {
  const long long N = d.N;
  const long long nsp = static_cast<long long>(d.ns) * d.S;
  switch (c.type) {
    case SAF3R_DENSE:
      return N * N;
    case SAF3R_TOKEN:  // patch queries: k per frame + the specials; special queries: every key
      return static_cast<long long>(d.S) * d.P * (static_cast<long long>(d.S) * c.k + nsp) + nsp * N;
    case SAF3R_PROBE:
      return N * (c.k + nsp);
    case SAF3R_SCAN: {
      const long long lat = (N - c.phase + c.stride - 1) / c.stride;
      long long off = 0;
      for (int sv = 0; sv < d.S; ++sv)
        for (int i = 0; i < d.ns; ++i)
          if (((static_cast<long long>(sv) * d.V + i) % c.stride) != c.phase) ++off;
      return N * (lat + off);
    }
    case SAF3R_POSITION: {
      const long long base = nsp + d.P;
      long long tot = nsp * base;  // special-token queries
      for (int r = 0; r < d.gh; ++r)
        for (int col = 0; col < d.gw; ++col) {
          const long long nb =
              c.radius < 0 ? 0
                           : static_cast<long long>(std::min(r + c.radius, d.gh - 1) - std::max(r - c.radius, 0) + 1) *
                                 (std::min(col + c.radius, d.gw - 1) - std::max(col - c.radius, 0) + 1);
          tot += d.S * (base + (d.S - 1) * nb);
        }
      return tot;
    }
    case SAF3R_CORR:
    case SAF3R_HYBRID: {
      // specials (and the lattice), then the patch tokens of the kept tiles not already counted
      const bool lat = c.type == SAF3R_HYBRID;
      long long base = nsp;
      if (lat) {
        base = (N - c.phase + c.stride - 1) / c.stride;
        for (int sv = 0; sv < d.S; ++sv)
          for (int i = 0; i < d.ns; ++i)
            if (((static_cast<long long>(sv) * d.V + i) % c.stride) != c.phase) ++base;
      }
      long long tot = 0;
      for (int u = 0; u < d.T; ++u) {
        const long long rows = std::min<long long>(kTile, N - static_cast<long long>(u) * kTile);
        long long keys = base;
        for (int r = 0; r < c.k; ++r) {
          const long long v = ranked[static_cast<size_t>(u) * kmax + r];
          const long long t0 = v * kTile, t1 = std::min(N, t0 + kTile);
          for (long long t = t0; t < t1; ++t)
            keys += (t % d.V) >= d.ns && !(lat && t % c.stride == c.phase);
        }
        tot += rows * keys;
      }
      return tot;
    }
  }
  return 0;
}

saf3r_status saf3r_kept_pairs(const saf3r_layout* L, const saf3r_head_cfg* cfg, const void* cache, int64_t* pairs,
                              void* stream) {
  saf3r_status st = check_layout(L);
  if (st != SAF3R_OK) return st;
  const Dims d = make_dims(*L);
  if ((st = check_cfg(d, cfg, L->H)) != SAF3R_OK) return st;
  if (!pairs) return SAF3R_ERR_INVALID;
  const CacheLayout cl = cache_layout(d, cfg);
  std::vector<int32_t> ranked;
  if (cl.corr_kmax > 0) {
    if (!cache) return SAF3R_ERR_INVALID;
    ranked.resize(static_cast<size_t>(d.T) * cl.corr_kmax);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(ranked.data(), static_cast<const int32_t*>(cache) + cl.corr_off, ranked.size() * 4,
                        cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return SAF3R_ERR_CUDA;
  }
  for (int h = 0; h < d.H; ++h) pairs[h] = pairs_of(d, cfg[h], ranked, cl.corr_kmax);
  return SAF3R_OK;
}

saf3r_status saf3r_profile_heads(const saf3r_layout* L, const saf3r_head_cfg* cand, int n_cand, const void* q,
                                 const void* k, const void* v, const float* dino, double nmse_max,
                                 saf3r_head_cfg* chosen, double* nmse, int64_t* pairs, void* workspace, void* stream) {
  saf3r_status st = check_layout(L);
  if (st != SAF3R_OK) return st;
  if (!cand || n_cand < 1 || !chosen || !nmse || !pairs || !q || !k || !v || !workspace) return SAF3R_ERR_INVALID;
  const Dims d = make_dims(*L);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::vector<saf3r_head_cfg> cfg(d.H);
  bool any_corr = false;
  for (int c = 0; c < n_cand; ++c) {
    for (int h = 0; h < d.H; ++h) cfg[h] = apply_candidate(cand[c], h);
    if ((st = check_cfg(d, cfg.data(), d.H)) != SAF3R_OK) return st;
    any_corr |= tile_kind(cand[c].type) || cand[c].type == SAF3R_TOKEN;
  }
  if (any_corr && !dino) return SAF3R_ERR_INVALID;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t out_bytes = align256(static_cast<size_t>(d.H) * d.N * kD * sizeof(float));
  size_t cache_max = 0, sel_max = 0, sp_max = 0;
  for (int c = 0; c < n_cand; ++c) {
    for (int h = 0; h < d.H; ++h) cfg[h] = apply_candidate(cand[c], h);
    cache_max = std::max(cache_max, cache_layout(d, cfg.data()).bytes);
    sel_max = std::max(sel_max, saf3r_workspace_bytes(L, cfg.data(), SAF3R_OP_SELECT));
    sp_max = std::max(sp_max, saf3r_workspace_bytes(L, cfg.data(), SAF3R_OP_SPARSE));
  }
  float* o_full = reinterpret_cast<float*>(ws);
  float* o_sparse = reinterpret_cast<float*>(ws + out_bytes);
  uint8_t* cache = ws + 2 * out_bytes;
  uint8_t* inner = cache + align256(cache_max);
  double* part = reinterpret_cast<double*>(inner + align256(std::max(sel_max, sp_max)));
  double* sums = reinterpret_cast<double*>(reinterpret_cast<uint8_t*>(part) + align256(nmse_workspace_bytes(d.H)));

  int launches = 0;
  if ((st = saf3r_dense_attn(L, q, k, v, o_full, 1, inner, stream)) != SAF3R_OK) return st;
  launches += t_launches;
  std::vector<std::vector<int32_t>> ranked(n_cand);
  std::vector<int> kmax(n_cand, 0);
  for (int c = 0; c < n_cand; ++c) {
    for (int h = 0; h < d.H; ++h) cfg[h] = apply_candidate(cand[c], h);
    if ((st = saf3r_select_kv(L, cfg.data(), q, k, dino, cache, inner, stream)) != SAF3R_OK) return st;
    launches += t_launches;
    if (tile_kind(cand[c].type)) {
      const CacheLayout cl = cache_layout(d, cfg.data());
      kmax[c] = cl.corr_kmax;
      ranked[c].resize(static_cast<size_t>(d.T) * cl.corr_kmax);
      if (cudaMemcpyAsync(ranked[c].data(), reinterpret_cast<int32_t*>(cache) + cl.corr_off, ranked[c].size() * 4,
                          cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return SAF3R_ERR_CUDA;
    }
    if ((st = saf3r_sparse_attn(L, cfg.data(), cache, q, k, v, o_sparse, 1, inner, stream)) != SAF3R_OK) return st;
    launches += t_launches;
    if (cuda_status(launch_nmse(o_full, o_sparse, d.H, static_cast<long long>(d.N) * kD, part,
                                sums + static_cast<size_t>(c) * d.H * 2, s)) != SAF3R_OK)
      return SAF3R_ERR_CUDA;
    launches += 2;
    if (tile_kind(cand[c].type) && cudaStreamSynchronize(s) != cudaSuccess) return SAF3R_ERR_CUDA;
  }
  std::vector<double> hs(static_cast<size_t>(n_cand) * d.H * 2);
  if (cudaMemcpyAsync(hs.data(), sums, hs.size() * sizeof(double), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return SAF3R_ERR_CUDA;
  int v_err = 0;
  if (cudaMemcpyFromSymbol(&v_err, g_device_error, sizeof(int)) != cudaSuccess) return SAF3R_ERR_CUDA;
  if (v_err != 0) return static_cast<saf3r_status>(v_err);
  for (int h = 0; h < d.H; ++h) {
    int best = -1;
    for (int c = 0; c < n_cand; ++c) {
      const saf3r_head_cfg hc = apply_candidate(cand[c], h);
      const double se = hs[(static_cast<size_t>(c) * d.H + h) * 2], sf = hs[(static_cast<size_t>(c) * d.H + h) * 2 + 1];
      nmse[static_cast<size_t>(h) * n_cand + c] = sf > 0 ? se / sf : (se > 0 ? INFINITY : 0.0);
      pairs[static_cast<size_t>(h) * n_cand + c] = pairs_of(d, hc, ranked[c], kmax[c]);
    }
    // cheapest qualifying candidate (ties to the lower index), else least NMSE (ties to the lower index)
    for (int c = 0; c < n_cand; ++c) {
      if (nmse[static_cast<size_t>(h) * n_cand + c] <= nmse_max &&
          (best < 0 || pairs[static_cast<size_t>(h) * n_cand + c] < pairs[static_cast<size_t>(h) * n_cand + best]))
        best = c;
    }
    if (best < 0) {
      best = 0;
      for (int c = 1; c < n_cand; ++c)
        if (nmse[static_cast<size_t>(h) * n_cand + c] < nmse[static_cast<size_t>(h) * n_cand + best]) best = c;
    }
    chosen[h] = apply_candidate(cand[best], h);
  }
  t_launches = launches;
  return SAF3R_OK;
}

saf3r_status saf3r_choose_eq2(int n_inputs, int H, int n_cand, const double* nmse, const int64_t* pairs,
                              int base, int32_t* choice, double* nmse_mean) {
  if (!nmse || !pairs || !choice || n_inputs < 1 || H < 1 || n_cand < 1 || base < 0 || base >= n_cand)
    return SAF3R_ERR_INVALID;
  const size_t per = static_cast<size_t>(H) * n_cand;
  std::vector<double> e(per, 0.0), w(per, 0.0);
  for (int i = 0; i < n_inputs; ++i)
    for (size_t x = 0; x < per; ++x) {
      e[x] += nmse[i * per + x];
      w[x] += static_cast<double>(pairs[i * per + x]);
    }
  for (size_t x = 0; x < per; ++x) {
    e[x] /= n_inputs;
    w[x] /= n_inputs;
  }
  for (int h = 0; h < H; ++h) {
    const double* eh = e.data() + static_cast<size_t>(h) * n_cand;
    const double* wh = w.data() + static_cast<size_t>(h) * n_cand;
    int cur = base;
    for (int c = 0; c < n_cand; ++c) {
      if (c == base) continue;
      if (wh[c] <= wh[base] && eh[c] < eh[cur]) cur = c;
    }
    choice[h] = cur;
  }
  if (nmse_mean)
    for (size_t x = 0; x < per; ++x) nmse_mean[x] = e[x];
  return SAF3R_OK;
}

}  // extern "C"
