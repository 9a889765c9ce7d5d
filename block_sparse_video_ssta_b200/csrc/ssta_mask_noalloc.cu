// ssta_build_block_mask_noalloc: the block-mask builder for callers that cannot
// allocate device memory when they call it.
//
// Some callers are not allowed to call cudaMalloc (or any allocating routine)
// at call time: for example a plugin inside an inference engine that is only
// handed the tensors the engine planned ahead, or a service that reserved all
// device memory up front for its own pool and treats any further allocation as
// a failure.  Such callers cannot provide the workspace ssta_build_block_mask
// needs.  This variant runs the same kernels on a scratch area that is a
// file-scope device array of fixed size, so the call itself allocates nothing.
//
// Costs and rules of that choice:
//  * the array (SSTA_STATIC_SCRATCH_BYTES) exists on every GPU that loads this
//    library and stays resident until the process exits;
//  * every call on a device uses the same array, which keeps the contents of
//    the last call: every region is fully rewritten before it is read;
//  * the mask kernels report no device-side errors (their inputs are checked
//    on the host), and the array's address is not exported, so this call keeps
//    no device status word: its first bytes stay unused;
//  * calls whose kernels overlap on the GPU (different streams, or different
//    host threads, on the same device) race on the array: serialise them;
//  * in host code the array's name is only a host-side stand-in, so its device
//    address is looked up once per device with cudaGetSymbolAddress (with that
//    device current) on the first call made on that device; make that first
//    call before any stream capture.
#include <mutex>

#include "ssta_internal.h"

static __device__ __align__(256) unsigned char g_ssta_mask_scratch[SSTA_STATIC_SCRATCH_BYTES];

namespace ssta {
namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_ssta_mask_scratch on the current device (looked up once per device).
ssta_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SSTA_ERR_LAUNCH;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_ssta_mask_scratch) != cudaSuccess || p == nullptr) return SSTA_ERR_LAUNCH;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return SSTA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) % 16) == 0; }

}  // namespace
}  // namespace ssta

using namespace ssta;

extern "C" ssta_status ssta_build_block_mask_noalloc(const ssta_desc* desc, const void* q_packed,
                                                     const void* k_packed, int32_t* kv_idx, int32_t* kv_cnt,
                                                     float* tile_scores, void* stream) {
  Geom g;
  ssta_status st = make_geom(desc, &g);
  if (st != SSTA_OK) return st;
  // scratch layout: the workspace layout of ssta_build_block_mask, without the score
  // matrix when the caller supplies it
  const size_t bh = (size_t)g.B * g.H;
  const MaskWorkspace ws = mask_workspace_layout(g, tile_scores == nullptr);
  if (ws.total > (size_t)SSTA_STATIC_SCRATCH_BYTES) return SSTA_ERR_WORKSPACE;
  const bool empty = bh == 0;
  if (!empty && (q_packed == nullptr || k_packed == nullptr || kv_idx == nullptr || kv_cnt == nullptr))
    return SSTA_ERR_INVALID_ARG;
  if (!aligned16(q_packed) || !aligned16(k_packed) || !aligned16(kv_idx) || !aligned16(kv_cnt) ||
      !aligned16(tile_scores))
    return SSTA_ERR_ALIGNMENT;
  void* base_v = nullptr;
  st = scratch_address(&base_v);
  if (st != SSTA_OK) return st;
  uint8_t* base = static_cast<uint8_t*>(base_v);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (empty) return SSTA_OK;
  float* qbar = reinterpret_cast<float*>(base + ws.qbar);
  float* kbar = reinterpret_cast<float*>(base + ws.kbar);
  float* scores = tile_scores != nullptr ? tile_scores : reinterpret_cast<float*>(base + ws.scores);
  const bool imp = g.score_mode == SSTA_SCORE_IMPORTANCE;
  const ImportanceBufs ib = imp ? ImportanceBufs{reinterpret_cast<float*>(base + ws.inv_nq), reinterpret_cast<float*>(base + ws.inv_nk),
                                                 reinterpret_cast<float*>(base + ws.ksum)}
                                : ImportanceBufs{nullptr, nullptr, nullptr};
  // no status word (nullptr): nothing could read it back
  cudaError_t e = launch_tile_pool(g, q_packed, k_packed, qbar, kbar, nullptr, ib, s);
  if (e == cudaSuccess && imp) e = launch_tile_keysum(g, kbar, ib, s);
  if (e == cudaSuccess) e = launch_tile_scores(g, qbar, kbar, ib, scores, nullptr, s);
  if (e == cudaSuccess) e = launch_select_and_list(g, scores, kv_idx, kv_cnt, s);
  return from_cuda(e);
}
