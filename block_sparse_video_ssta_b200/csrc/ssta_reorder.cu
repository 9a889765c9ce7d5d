// Step 1 of SSTA ("HunyuanVideo 1.5 Technical Report", section "SSTA: Selective
// and Sliding Tile Attention", Step 1 "3D Block Partition"): tokens of the
// F x H x W latent grid are grouped into contiguous tiles of N = tT*tY*tX tokens.
//
// tile_reorder:  raster [B,H,T,Y,X,D] (+ text [B,H,L,D]) -> packed [B,H,Lq,D]
// tile_unorder:  packed -> raster (pad rows dropped) (+ text)
//
// Both are HBM-bound copies.  One CTA owns one (batch*head, tile) pair: it first
// resolves the N packed-row -> raster-row mapping into shared memory (so the
// integer divisions happen once per row, not once per 16-byte vector), then
// streams the tile with 16-byte vector loads/stores that are coalesced on the
// packed side and contiguous over runs of tX tokens on the raster side.
#include "ssta_internal.h"

namespace ssta {
namespace {

constexpr int kCopyThreads = 256;

// Fill map[o] for the N rows of tile `c` of one head: raster row (within the
// head) of packed row c*N+o, -1 for a pad row, -2 for a row beyond Lq.
__device__ void build_row_map(const Geom& g, int c, int* map) {
  if (c < g.NT) {
    int cX = c % g.nX;
    int rest = c / g.nX;
    int cY = rest % g.nY;
    int cT = rest / g.nY;
    for (int o = threadIdx.x; o < g.N; o += blockDim.x) {
      int dx = o % g.tX;
      int r2 = o / g.tX;
      int dy = r2 % g.tY;
      int dt = r2 / g.tY;
      int t = cT * g.tT + dt, y = cY * g.tY + dy, x = cX * g.tX + dx;
      map[o] = (t < g.T && y < g.Y && x < g.X) ? (t * g.Y + y) * g.X + x : -1;
    }
  } else {
    for (int o = threadIdx.x; o < g.N; o += blockDim.x) {
      int j = (c - g.NT) * g.N + o;
      map[o] = j < g.L_text ? j : -2;
    }
  }
}

__global__ void __launch_bounds__(kCopyThreads)
tile_reorder_kernel(Geom g, const int4* __restrict__ raster, const int4* __restrict__ text,
                    int4* __restrict__ packed, int vpr_log2) {
  extern __shared__ int map[];
  const int c = blockIdx.x;
  const int64_t bh = blockIdx.y;
  build_row_map(g, c, map);
  __syncthreads();
  const int vpr = 1 << vpr_log2;
  const int64_t raster_rows = (int64_t)g.T * g.Y * g.X;
  const int64_t dst_base = (bh * g.Lq + (int64_t)c * g.N) << vpr_log2;
  const int nvec = g.N << vpr_log2;
#pragma unroll 4
  for (int e = threadIdx.x; e < nvec; e += kCopyThreads) {
    const int o = e >> vpr_log2;
    const int v = e & (vpr - 1);
    const int s = map[o];
    if (s == -2) continue;
    int4 val = make_int4(0, 0, 0, 0);
    if (s >= 0) {
      const int4* src = (c < g.NT) ? raster + ((bh * raster_rows + s) << vpr_log2)
                                    : text + ((bh * g.L_text + s) << vpr_log2);
      val = __ldg(src + v);
    }
    packed[dst_base + e] = val;
  }
}

__global__ void __launch_bounds__(kCopyThreads)
tile_unorder_kernel(Geom g, const int4* __restrict__ packed, int4* __restrict__ raster,
                    int4* __restrict__ text, int vpr_log2) {
  extern __shared__ int map[];
  const int c = blockIdx.x;
  const int64_t bh = blockIdx.y;
  if (c >= g.NT && text == nullptr) return;
  build_row_map(g, c, map);
  __syncthreads();
  const int vpr = 1 << vpr_log2;
  const int64_t raster_rows = (int64_t)g.T * g.Y * g.X;
  const int64_t src_base = (bh * g.Lq + (int64_t)c * g.N) << vpr_log2;
  const int nvec = g.N << vpr_log2;
#pragma unroll 4
  for (int e = threadIdx.x; e < nvec; e += kCopyThreads) {
    const int o = e >> vpr_log2;
    const int v = e & (vpr - 1);
    const int s = map[o];
    if (s < 0) continue;
    int4* dst = (c < g.NT) ? raster + ((bh * raster_rows + s) << vpr_log2)
                           : text + ((bh * g.L_text + s) << vpr_log2);
    dst[v] = __ldg(packed + src_base + e);
  }
}

int vectors_per_row_log2(const Geom& g) {
  int vpr = g.D * g.esize / 16;
  int l = 0;
  while ((1 << l) < vpr) ++l;
  return l;
}

}  // namespace

cudaError_t launch_tile_reorder(const Geom& g, const void* raster, const void* text, void* packed,
                                cudaStream_t s) {
  if ((int64_t)g.B * g.H == 0) return cudaSuccess;
  dim3 grid(g.NQ, g.B * g.H);
  tile_reorder_kernel<<<grid, kCopyThreads, g.N * sizeof(int), s>>>(
      g, static_cast<const int4*>(raster), static_cast<const int4*>(text), static_cast<int4*>(packed),
      vectors_per_row_log2(g));
  return cudaGetLastError();
}

cudaError_t launch_tile_unorder(const Geom& g, const void* packed, void* raster, void* text,
                                cudaStream_t s) {
  if ((int64_t)g.B * g.H == 0) return cudaSuccess;
  dim3 grid(g.NQ, g.B * g.H);
  tile_unorder_kernel<<<grid, kCopyThreads, g.N * sizeof(int), s>>>(
      g, static_cast<const int4*>(packed), static_cast<int4*>(raster), static_cast<int4*>(text),
      vectors_per_row_log2(g));
  return cudaGetLastError();
}

}  // namespace ssta
