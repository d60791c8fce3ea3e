// saf3r_select_kv_static: the per-input index build without a caller workspace.
//
// saf3r_select_kv needs a device workspace for its partial sums, probe scores,
// tile descriptors, tile cosines and grouping bitsets, and expects the caller to
// allocate it.  Some callers cannot: engines whose latency-critical loop must
// never enter an allocator, and plug-in hosts that hand a library only its input
// and output buffers.  This entry point serves
// them from a fixed device array compiled into the library instead, so it calls
// no allocator at all; the array costs every GPU that loads the library
// kStaticScratchBytes of memory until the process exits.
#include <cuda_runtime.h>

#include <map>
#include <mutex>

#include "internal.h"

namespace {

// Largest select workspace this entry point can serve (saf3r_workspace_bytes with
// SAF3R_OP_SELECT): enough for the 274,800-token layer with 4 probe heads and
// 4 correspondence heads (32.3 MiB, most of it the fp16 tile cosines of one chunk).
constexpr size_t kStaticScratchBytes = size_t(40) << 20;

static __device__ __align__(256) unsigned char g_select_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
std::map<int, void*> g_scratch_addr;  // device id -> device address of g_select_scratch

// The device address of the scratch array on the current device.  The name of a
// __device__ array in host code is only a host-side stand-in, so its address is
// looked up once per device (with that device current) and remembered.
saf3r_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAF3R_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  auto it = g_scratch_addr.find(dev);
  if (it != g_scratch_addr.end()) {
    *out = it->second;
    return SAF3R_OK;
  }
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_select_scratch) != cudaSuccess || ptr == nullptr) return SAF3R_ERR_CUDA;
  g_scratch_addr[dev] = ptr;
  *out = ptr;
  return SAF3R_OK;
}

}  // namespace

extern "C" saf3r_status saf3r_select_kv_static(const saf3r_layout* layout, const saf3r_head_cfg* cfg,
                                               const void* q, const void* k, const float* dino, void* cache,
                                               void* stream) {
  const saf3r_status valid = saf3r::validate_layout_cfg(layout, cfg);  // the codes saf3r_select_kv returns
  if (valid != SAF3R_OK) return valid;
  const size_t need = saf3r_workspace_bytes(layout, cfg, SAF3R_OP_SELECT);
  if (need == 0) return SAF3R_ERR_INVALID;
  if (need > kStaticScratchBytes) return SAF3R_ERR_UNSUPPORTED;  // layer too large for the built-in scratch
  void* scratch = nullptr;
  const saf3r_status st = scratch_address(&scratch);
  if (st != SAF3R_OK) return st;
  // Everything the build reads from the scratch it first writes in the same call (the parts
  // that must start at zero - the probe ranking's counters, the grouping bitsets and the
  // token-wise ordering's buckets - are cleared by the call itself).
  return saf3r_select_kv(layout, cfg, q, k, dino, cache, scratch, stream);
}
