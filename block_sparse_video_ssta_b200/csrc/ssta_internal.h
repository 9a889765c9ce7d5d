// Internal declarations shared by the SSTA CUDA translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ssta.h"

namespace ssta {

// Every size the kernels need, derived once on the host from an ssta_desc.
struct Geom {
  int B, H, D;
  int T, Y, X;          // valid grid
  int tT, tY, tX;       // tile extents
  int nT, nY, nX;       // tiles per axis
  int N;                // tokens per tile
  int NT;               // video tiles
  int L_text;
  int n_text;           // text tiles
  int NQ;               // query tiles
  int64_t Lq;           // packed length
  int k;                // top-k, clamped
  int wT, wY, wX;       // window (tiles)
  int window_tiles;
  int max_kept;
  int words;            // 32-bit words per selection-bitset row = ceil(NT/32)
  int esize;            // bytes per element (2 or 4)
  int dtype;
  float scale;          // softmax scale
  int score_mode;       // ssta_score_mode
  float lambda;         // importance score weight
  int combine;          // ssta_combine
  int window_mode;      // ssta_window
  int norm_blocks;      // 32-tile blocks of the importance key sums = ceil(NT/32)
};

// Workspace layout of ssta_build_block_mask (byte offsets, 256-aligned).
struct MaskWorkspace {
  size_t status;   // int32 device status word
  size_t qbar;     // fp32 [BH, D, NT] (channel-major)
  size_t kbar;     // fp32 [BH, D, NT] (channel-major)
  size_t inv_nq;   // importance score only: fp32 [BH, NT], 1 / |Qbar_i| (0 for a zero mean)
  size_t inv_nk;   //   fp32 [BH, NT], 1 / |Kbar_j|
  size_t ksum;     //   fp32 [BH, norm_blocks, D], per 32-tile block sum of unit Kbar_j
  size_t scores;   // fp32 [BH, NT, NT]; absent when `with_scores` is false
  size_t total;
};

// Offsets from 0; `with_scores` = false when the caller supplies the score matrix.
MaskWorkspace mask_workspace_layout(const Geom& g, bool with_scores = true);

// The importance buffers of a mask workspace at `base` (all NULL for the similarity score).
struct ImportanceBufs {
  float* inv_nq;
  float* inv_nk;
  float* ksum;
};

// Workspace layout of ssta_attention_bwd (byte offsets, 256-aligned).
struct BwdWorkspace {
  size_t status;   // int32 device status word
  size_t rowdot;   // fp32 [BH, Lq], D = rowsum(dO * O)
  size_t nl2;      // fp32 [BH, NQ * N], -LSE * log2(e) per packed row (-inf: pad row or no kept key)
  size_t nd;       // fp32 [BH, NQ * N], -D per packed row (0 where nl2 is -inf)
  size_t tcnt;     // int32 [BH, NQ], query tiles keeping each key tile
  size_t tidx;     // int32 [BH, NQ, NQ], those query tiles, ascending
  size_t total;
};
BwdWorkspace bwd_workspace_layout(const Geom& g);

// Validate a descriptor and derive every size (host only, no CUDA call).
ssta_status make_geom(const ssta_desc* d, Geom* g);

// Launchers (return cudaGetLastError() of their launches).
cudaError_t launch_tile_reorder(const Geom& g, const void* raster, const void* text, void* packed,
                                cudaStream_t s);
cudaError_t launch_tile_unorder(const Geom& g, const void* packed, void* raster, void* text,
                                cudaStream_t s);
// Also writes 0 to *status (when non-NULL) after the previous kernel of the stream has
// finished, so a mask build needs no separate reset of its status word, and, for the
// importance score (ib.inv_nq != NULL), the inverse norms of the tile means.
cudaError_t launch_tile_pool(const Geom& g, const void* qp, const void* kp, float* qbar, float* kbar,
                             int32_t* status, const ImportanceBufs& ib, cudaStream_t s);
// Importance score only: per 32-tile block sums of the unit key means.
cudaError_t launch_tile_keysum(const Geom& g, const float* kbar, const ImportanceBufs& ib, cudaStream_t s);
// Block scores: raw dot products (on the tensor cores, ssta_mask_tc.cu), or the
// importance score when ib.ksum != NULL (SIMT).  `status` may be NULL.
cudaError_t launch_tile_scores(const Geom& g, const float* qbar, const float* kbar, const ImportanceBufs& ib,
                               float* scores, int32_t* status, cudaStream_t s);
cudaError_t launch_tile_scores_tc(const Geom& g, const float* qbar, const float* kbar, float* scores,
                                  int32_t* status, cudaStream_t s);
cudaError_t launch_select_and_list(const Geom& g, const float* scores, int32_t* kv_idx, int32_t* kv_cnt,
                                   cudaStream_t s);
cudaError_t launch_attention_f32(const Geom& g, const float* qp, const float* kp, const float* vp,
                                 const int32_t* kv_idx, const int32_t* kv_cnt, float* o, float* lse,
                                 int32_t* status, cudaStream_t s);
cudaError_t launch_attention_bwd(const Geom& g, const void* q, const void* k, const void* v, const void* o,
                                 const float* lse, const void* dO, const int32_t* kv_idx, const int32_t* kv_cnt,
                                 void* dq, void* dk, void* dv, void* workspace, cudaStream_t s);
// bf16, N % 128 == 0: dQ on the tensor cores (Dv = rowsum(dO * O) already computed).
cudaError_t launch_attention_bwd_dq_tc(const Geom& g, const void* q, const void* k, const void* v, const void* dO,
                                       const float* lse, const float* Dv, const int32_t* kv_idx,
                                       const int32_t* kv_cnt, void* dq, int32_t* status, cudaStream_t s);
// bf16, N % 128 == 0: dK and dV on the tensor cores (tidx/tcnt: the transposed lists).
cudaError_t launch_attention_bwd_rowstat_tc(const Geom& g, const void* o, const void* dO, const float* lse, float* Dv,
                                            float* nl2, float* nd, cudaStream_t s);
cudaError_t launch_attention_bwd_dkdv_tc(const Geom& g, const void* q, const void* k, const void* v, const void* dO,
                                         const float* nl2, const float* nd, const int32_t* tidx,
                                         const int32_t* tcnt, void* dk, void* dv, int32_t* status, cudaStream_t s);
cudaError_t launch_attention_bf16_tc(const Geom& g, const void* qp, const void* kp, const void* vp,
                                     const int32_t* kv_idx, const int32_t* kv_cnt, void* o, float* lse,
                                     int32_t* status, cudaStream_t s);

// Device-side helpers shared by kernels.
__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Status of a host-side CUDA runtime call (a launch, a memset): SSTA_ERR_LAUNCH on any error.
inline ssta_status from_cuda(cudaError_t e) { return e == cudaSuccess ? SSTA_OK : SSTA_ERR_LAUNCH; }

// Number of valid tokens along one axis of tile coordinate c (tile extent t, valid extent n).
__host__ __device__ inline int axis_valid(int c, int t, int n) {
  int v = n - c * t;
  return v < t ? v : t;
}

}  // namespace ssta
