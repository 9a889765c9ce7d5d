// C ABI of libssta.so: argument validation, size planning and kernel dispatch.
// Declared in include/ssta.h.  Nothing here allocates or synchronises, except
// ssta_read_device_status, whose job is to read a device word back.
#include <math.h>
#include <string.h>

#include <nvtx3/nvToolsExt.h>

#include "ssta_internal.h"

namespace ssta {
namespace {

constexpr int kMaxTileTokens = 4096;   // N; one shared-memory row map per tile
constexpr int kMaxTiles = 2048;        // NT; one warp holds a score row in registers

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// NVTX range over one library call (host side: validation and kernel enqueue), so a
// timeline tool shows each call by name; without a tool attached it costs a few ns.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

}  // namespace

// Host-side geometry (Step 1, "3D Block Partition").  Returns SSTA_OK or the
// reason the descriptor is rejected.
ssta_status make_geom(const ssta_desc* d, Geom* g) {
  if (d == nullptr || g == nullptr) return SSTA_ERR_INVALID_ARG;
  if (d->B < 0 || d->H < 0 || d->D <= 0) return SSTA_ERR_INVALID_ARG;
  if (d->T < 1 || d->Y < 1 || d->X < 1) return SSTA_ERR_INVALID_ARG;
  if (d->tT < 1 || d->tY < 1 || d->tX < 1) return SSTA_ERR_INVALID_ARG;
  if (d->wT < 1 || d->wY < 1 || d->wX < 1) return SSTA_ERR_INVALID_ARG;
  if (d->topk < 0 || d->L_text < 0) return SSTA_ERR_INVALID_ARG;
  if (d->dtype != SSTA_BF16 && d->dtype != SSTA_F32) return SSTA_ERR_INVALID_ARG;
  if (!(d->scale >= 0.0f) || isinf(d->scale)) return SSTA_ERR_INVALID_ARG;
  if (d->score_mode != SSTA_SCORE_SIMILARITY && d->score_mode != SSTA_SCORE_IMPORTANCE) return SSTA_ERR_INVALID_ARG;
  if (d->score_mode == SSTA_SCORE_IMPORTANCE && !(d->lambda >= 0.0f && d->lambda <= 1.0f)) return SSTA_ERR_INVALID_ARG;
  if (d->combine != SSTA_COMBINE_UNION && d->combine != SSTA_COMBINE_AND) return SSTA_ERR_INVALID_ARG;
  if (d->window_mode != SSTA_WINDOW_SHIFT && d->window_mode != SSTA_WINDOW_TRUNCATE) return SSTA_ERR_INVALID_ARG;
  if ((int64_t)d->B * d->H > 65535) return SSTA_ERR_UNSUPPORTED;
  if (d->D != 128) return SSTA_ERR_UNSUPPORTED;
  const int64_t N = (int64_t)d->tT * d->tY * d->tX;
  if (N > kMaxTileTokens) return SSTA_ERR_UNSUPPORTED;
  Geom x{};
  x.B = d->B; x.H = d->H; x.D = d->D;
  x.T = d->T; x.Y = d->Y; x.X = d->X;
  x.tT = d->tT; x.tY = d->tY; x.tX = d->tX;
  x.nT = ceil_div(d->T, d->tT);
  x.nY = ceil_div(d->Y, d->tY);
  x.nX = ceil_div(d->X, d->tX);
  x.N = (int)N;
  const int64_t NT = (int64_t)x.nT * x.nY * x.nX;
  if (NT > kMaxTiles) return SSTA_ERR_UNSUPPORTED;
  x.NT = (int)NT;
  x.L_text = d->L_text;
  x.n_text = d->L_text > 0 ? ceil_div(d->L_text, x.N) : 0;
  x.NQ = x.NT + x.n_text;
  x.Lq = (int64_t)x.NT * x.N + d->L_text;
  if (x.Lq >= (int64_t)1 << 31) return SSTA_ERR_UNSUPPORTED;
  x.k = d->topk < x.NT ? d->topk : x.NT;
  x.wT = d->wT; x.wY = d->wY; x.wX = d->wX;
  x.window_tiles = (d->wT < x.nT ? d->wT : x.nT) * (d->wY < x.nY ? d->wY : x.nY) * (d->wX < x.nX ? d->wX : x.nX);
  if (x.n_text > 0) {
    x.max_kept = x.NT + x.n_text;
  } else {
    const int64_t v = (int64_t)x.k + x.window_tiles;
    x.max_kept = (int)(v < x.NT ? v : x.NT);
  }
  x.words = ceil_div(x.NT, 32);
  x.dtype = d->dtype;
  x.esize = d->dtype == SSTA_BF16 ? 2 : 4;
  x.scale = d->scale > 0.0f ? d->scale : 1.0f / sqrtf((float)d->D);
  x.score_mode = d->score_mode;
  x.lambda = d->score_mode == SSTA_SCORE_IMPORTANCE ? d->lambda : 0.0f;
  x.combine = d->combine;
  x.window_mode = d->window_mode;
  x.norm_blocks = ceil_div(x.NT, 32);
  *g = x;
  return SSTA_OK;
}

}  // namespace ssta

using namespace ssta;

extern "C" {

ssta_status ssta_plan(const ssta_desc* desc, ssta_plan_info* info) {
  if (info == nullptr) return SSTA_ERR_INVALID_ARG;
  Geom g;
  ssta_status st = make_geom(desc, &g);
  if (st != SSTA_OK) return st;
  info->packed_len = g.Lq;
  info->num_tiles = g.NT;
  info->num_text_tiles = g.n_text;
  info->num_q_tiles = g.NQ;
  info->tile_tokens = g.N;
  info->topk = g.k;
  info->window_tiles = g.window_tiles;
  info->max_kept = g.max_kept;
  info->workspace_bytes = mask_workspace_layout(g).total;
  info->attn_workspace_bytes = 256;
  info->bwd_workspace_bytes = bwd_workspace_layout(g).total;
  return SSTA_OK;
}

ssta_status ssta_tile_reorder(const ssta_desc* desc, const void* x_raster, const void* x_text, void* x_packed,
                              void* stream) {
  NvtxRange nvtx("ssta_tile_reorder");
  Geom g;
  ssta_status st = make_geom(desc, &g);
  if (st != SSTA_OK) return st;
  const bool empty = (int64_t)g.B * g.H == 0;
  if (!empty && (x_raster == nullptr || x_packed == nullptr)) return SSTA_ERR_INVALID_ARG;
  if (!empty && g.L_text > 0 && x_text == nullptr) return SSTA_ERR_INVALID_ARG;
  if (!aligned(x_raster, 16) || !aligned(x_text, 16) || !aligned(x_packed, 16)) return SSTA_ERR_ALIGNMENT;
  return from_cuda(launch_tile_reorder(g, x_raster, x_text, x_packed, static_cast<cudaStream_t>(stream)));
}

ssta_status ssta_attention_bwd(const ssta_desc* desc, const void* q_packed, const void* k_packed,
                               const void* v_packed, const void* o_packed, const float* lse, const void* do_packed,
                               const int32_t* kv_idx, const int32_t* kv_cnt, void* dq_packed, void* dk_packed,
                               void* dv_packed, void* workspace, size_t workspace_bytes, void* stream) {
  NvtxRange nvtx("ssta_attention_bwd");
  Geom g;
  ssta_status st = make_geom(desc, &g);
  if (st != SSTA_OK) return st;
  if (g.dtype == SSTA_BF16 && g.N % 128 != 0) return SSTA_ERR_UNSUPPORTED;
  const BwdWorkspace ws = bwd_workspace_layout(g);
  if (workspace == nullptr || workspace_bytes < ws.total) return SSTA_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return SSTA_ERR_ALIGNMENT;
  const bool empty = (int64_t)g.B * g.H == 0;
  const void* in[] = {q_packed, k_packed, v_packed, o_packed, lse, do_packed, kv_idx, kv_cnt, dq_packed, dk_packed,
                      dv_packed};
  for (const void* p : in) {
    if (!empty && p == nullptr) return SSTA_ERR_INVALID_ARG;
    if (!aligned(p, 16)) return SSTA_ERR_ALIGNMENT;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, sizeof(int32_t), s) != cudaSuccess) return SSTA_ERR_LAUNCH;
  return from_cuda(launch_attention_bwd(g, q_packed, k_packed, v_packed, o_packed, lse, do_packed, kv_idx, kv_cnt,
                                        dq_packed, dk_packed, dv_packed, workspace, s));
}

ssta_status ssta_tile_unorder(const ssta_desc* desc, const void* x_packed, void* x_raster, void* x_text,
                              void* stream) {
  NvtxRange nvtx("ssta_tile_unorder");
  Geom g;
  ssta_status st = make_geom(desc, &g);
  if (st != SSTA_OK) return st;
  const bool empty = (int64_t)g.B * g.H == 0;
  if (!empty && (x_raster == nullptr || x_packed == nullptr)) return SSTA_ERR_INVALID_ARG;
  if (!aligned(x_raster, 16) || !aligned(x_text, 16) || !aligned(x_packed, 16)) return SSTA_ERR_ALIGNMENT;
  return from_cuda(launch_tile_unorder(g, x_packed, x_raster, g.L_text > 0 ? x_text : nullptr,
                                       static_cast<cudaStream_t>(stream)));
}

ssta_status ssta_build_block_mask(const ssta_desc* desc, const void* q_packed, const void* k_packed,
                                  int32_t* kv_idx, int32_t* kv_cnt, float* tile_scores, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  NvtxRange nvtx("ssta_build_block_mask");
  Geom g;
  ssta_status st = make_geom(desc, &g);
  if (st != SSTA_OK) return st;
  const MaskWorkspace ws = mask_workspace_layout(g);
  if (workspace == nullptr || workspace_bytes < ws.total) return SSTA_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return SSTA_ERR_ALIGNMENT;
  const bool empty = (int64_t)g.B * g.H == 0;
  if (!empty && (q_packed == nullptr || k_packed == nullptr || kv_idx == nullptr || kv_cnt == nullptr))
    return SSTA_ERR_INVALID_ARG;
  if (!aligned(q_packed, 16) || !aligned(k_packed, 16) || !aligned(kv_idx, 16) || !aligned(kv_cnt, 16) ||
      !aligned(tile_scores, 16))
    return SSTA_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  if (empty) return from_cuda(cudaMemsetAsync(w + ws.status, 0, sizeof(int32_t), s));
  float* qbar = reinterpret_cast<float*>(w + ws.qbar);
  float* kbar = reinterpret_cast<float*>(w + ws.kbar);
  float* scores = tile_scores != nullptr ? tile_scores : reinterpret_cast<float*>(w + ws.scores);
  const bool imp = g.score_mode == SSTA_SCORE_IMPORTANCE;
  const ImportanceBufs ib = imp ? ImportanceBufs{reinterpret_cast<float*>(w + ws.inv_nq), reinterpret_cast<float*>(w + ws.inv_nk),
                                                 reinterpret_cast<float*>(w + ws.ksum)}
                                : ImportanceBufs{nullptr, nullptr, nullptr};
  // the pool kernel also clears the status word
  cudaError_t e = launch_tile_pool(g, q_packed, k_packed, qbar, kbar, reinterpret_cast<int32_t*>(w + ws.status), ib, s);
  if (e == cudaSuccess && imp) e = launch_tile_keysum(g, kbar, ib, s);
  if (e == cudaSuccess) e = launch_tile_scores(g, qbar, kbar, ib, scores, reinterpret_cast<int32_t*>(w + ws.status), s);
  if (e == cudaSuccess) e = launch_select_and_list(g, scores, kv_idx, kv_cnt, s);
  return from_cuda(e);
}

ssta_status ssta_attention_fwd(const ssta_desc* desc, const void* q_packed, const void* k_packed,
                               const void* v_packed, const int32_t* kv_idx, const int32_t* kv_cnt, void* o_packed,
                               float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  NvtxRange nvtx("ssta_attention_fwd");
  Geom g;
  ssta_status st = make_geom(desc, &g);
  if (st != SSTA_OK) return st;
  if (g.dtype == SSTA_BF16 && g.N % 128 != 0) return SSTA_ERR_UNSUPPORTED;
  if (workspace == nullptr || workspace_bytes < 256) return SSTA_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return SSTA_ERR_ALIGNMENT;
  const bool empty = (int64_t)g.B * g.H == 0;
  if (!empty && (q_packed == nullptr || k_packed == nullptr || v_packed == nullptr || kv_idx == nullptr ||
                 kv_cnt == nullptr || o_packed == nullptr || lse == nullptr))
    return SSTA_ERR_INVALID_ARG;
  if (!aligned(q_packed, 16) || !aligned(k_packed, 16) || !aligned(v_packed, 16) || !aligned(kv_idx, 16) ||
      !aligned(kv_cnt, 16) || !aligned(o_packed, 16) || !aligned(lse, 16))
    return SSTA_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* status = static_cast<int32_t*>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(int32_t), s) != cudaSuccess) return SSTA_ERR_LAUNCH;
  if (empty) return SSTA_OK;
  cudaError_t e;
  if (g.dtype == SSTA_BF16)
    e = launch_attention_bf16_tc(g, q_packed, k_packed, v_packed, kv_idx, kv_cnt, o_packed, lse, status, s);
  else
    e = launch_attention_f32(g, static_cast<const float*>(q_packed), static_cast<const float*>(k_packed),
                             static_cast<const float*>(v_packed), kv_idx, kv_cnt, static_cast<float*>(o_packed), lse,
                             status, s);
  return from_cuda(e);
}

ssta_status ssta_read_device_status(const void* workspace, void* stream, int32_t* code) {
  if (workspace == nullptr || code == nullptr) return SSTA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(code, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return SSTA_ERR_LAUNCH;
  if (cudaStreamSynchronize(s) != cudaSuccess) return SSTA_ERR_LAUNCH;
  return SSTA_OK;
}

const char* ssta_status_string(ssta_status status) {
  switch (status) {
    case SSTA_OK: return "SSTA_OK";
    case SSTA_ERR_INVALID_ARG: return "SSTA_ERR_INVALID_ARG";
    case SSTA_ERR_UNSUPPORTED: return "SSTA_ERR_UNSUPPORTED";
    case SSTA_ERR_ALIGNMENT: return "SSTA_ERR_ALIGNMENT";
    case SSTA_ERR_WORKSPACE: return "SSTA_ERR_WORKSPACE";
    case SSTA_ERR_LAUNCH: return "SSTA_ERR_LAUNCH";
    case SSTA_ERR_DEVICE_TIMEOUT: return "SSTA_ERR_DEVICE_TIMEOUT";
    case SSTA_ERR_DEVICE_BOUNDS: return "SSTA_ERR_DEVICE_BOUNDS";
  }
  return "SSTA_ERR_UNKNOWN";
}

}  // extern "C"
