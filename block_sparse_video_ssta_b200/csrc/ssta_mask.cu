// Steps 2-4 of SSTA up to the mask ("HunyuanVideo 1.5 Technical Report", section
// "SSTA: Selective and Sliding Tile Attention"):
//   Step 2  pooled tile representations Qbar, Kbar; Score_s = Qbar Kbar^T per
//           head; Topk + Indexes2mask per head and query tile;
//   Step 3  STA window mask over the tile grid, WS = (w_t, w_h, w_w) tiles;
//   Step 4  combined mask (union of selection and window, plus an always-dense
//           text segment), emitted as compact ascending kept-tile lists.
//
// Kernels, in launch order:
//   tile_pool_kernel      HBM-bound: one CTA per (head, tile) streams the tile's
//                         valid q and k rows with 16-byte coalesced loads and
//                         reduces per-channel fp32 sums across row groups.
//   tile_scores_kernel    fp32 SIMT, 64x64 score blocks per CTA, channels
//                         summed in order 0..D-1 with FMA.
//   select_topk_kernel    one warp per (head, query tile): scores held in
//                         registers as order-preserving 32-bit keys, k-th key
//                         found by a bitwise binary search with warp-wide
//                         counts, ties resolved to the lower tile index by
//                         ballots in index order; writes a selection bitset.
//   build_kv_lists_kernel one warp per (head, query tile): window membership
//                         computed per candidate, OR-ed with the bitset and the
//                         text tiles, compacted in ascending order by ballot
//                         prefix counts.
#include "ssta_internal.h"

#include <cuda_bf16.h>

namespace ssta {
namespace {

constexpr int kPoolThreads = 256;

__device__ __forceinline__ void add_vec(float* acc, const int4& raw, const __nv_bfloat16*) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    acc[2 * i] += f.x;
    acc[2 * i + 1] += f.y;
  }
}

__device__ __forceinline__ void add_vec(float* acc, const int4& raw, const float*) {
  const float* f = reinterpret_cast<const float*>(&raw);
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i] += f[i];
}

// Step 2, pooled (average) representation of each video tile over its valid tokens.
template <typename T>
__global__ void __launch_bounds__(kPoolThreads)
tile_pool_kernel(Geom g, const int4* __restrict__ qp, const int4* __restrict__ kp,
                 float* __restrict__ qbar, float* __restrict__ kbar) {
  constexpr int EPV = 16 / sizeof(T);        // elements per 16-byte vector
  const int vpr = g.D / EPV;                 // vectors per row
  const int rpp = kPoolThreads / vpr;        // rows per pass
  const int c = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int vec = threadIdx.x % vpr;
  const int rsub = threadIdx.x / vpr;

  const int cX = c % g.nX, cY = (c / g.nX) % g.nY, cT = c / (g.nX * g.nY);
  const int vt = axis_valid(cT, g.tT, g.T), vy = axis_valid(cY, g.tY, g.Y),
            vx = axis_valid(cX, g.tX, g.X);
  const bool full = (vt == g.tT) && (vy == g.tY) && (vx == g.tX);

  const int64_t base = (bh * g.Lq + (int64_t)c * g.N) * vpr + vec;
  float aq[EPV], ak[EPV];
#pragma unroll
  for (int i = 0; i < EPV; ++i) aq[i] = ak[i] = 0.f;

  if (full) {
    int o = rsub;
    for (; o + 3 * rpp < g.N; o += 4 * rpp) {
      int4 rq[4], rk[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        rq[u] = __ldg(qp + base + (int64_t)(o + u * rpp) * vpr);
        rk[u] = __ldg(kp + base + (int64_t)(o + u * rpp) * vpr);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        add_vec(aq, rq[u], (const T*)nullptr);
        add_vec(ak, rk[u], (const T*)nullptr);
      }
    }
    for (; o < g.N; o += rpp) {
      add_vec(aq, __ldg(qp + base + (int64_t)o * vpr), (const T*)nullptr);
      add_vec(ak, __ldg(kp + base + (int64_t)o * vpr), (const T*)nullptr);
    }
  } else {
    for (int o = rsub; o < g.N; o += rpp) {
      const int dx = o % g.tX, dy = (o / g.tX) % g.tY, dt = o / (g.tX * g.tY);
      if (dt < vt && dy < vy && dx < vx) {
        add_vec(aq, __ldg(qp + base + (int64_t)o * vpr), (const T*)nullptr);
        add_vec(ak, __ldg(kp + base + (int64_t)o * vpr), (const T*)nullptr);
      }
    }
  }

  // Reduce the rpp row groups: red[tensor][rsub][channel].
  extern __shared__ float red[];
  const int D = g.D;
#pragma unroll
  for (int i = 0; i < EPV; ++i) {
    red[(0 * rpp + rsub) * D + vec * EPV + i] = aq[i];
    red[(1 * rpp + rsub) * D + vec * EPV + i] = ak[i];
  }
  __syncthreads();
  const float inv = 1.0f / (float)(vt * vy * vx);
  for (int t = threadIdx.x; t < 2 * D; t += kPoolThreads) {
    const int which = t / D, ch = t % D;
    float s = 0.f;
    for (int r = 0; r < rpp; ++r) s += red[(which * rpp + r) * D + ch];
    float* out = which ? kbar : qbar;
    out[(bh * g.NT + c) * D + ch] = s * inv;
  }
}

// Step 2, Score_s = Qbar Kbar^T: 64x64 output block per CTA, 16x16 threads,
// each thread 4x4 outputs at stride 16; channels in chunks of 32 via smem.
constexpr int kScoreTile = 64;
constexpr int kScoreChunk = 32;

__global__ void __launch_bounds__(256)
tile_scores_kernel(Geom g, const float* __restrict__ qbar, const float* __restrict__ kbar,
                   float* __restrict__ scores) {
  __shared__ float qs[kScoreTile][kScoreChunk + 1];
  __shared__ float ks[kScoreTile][kScoreChunk + 1];
  const int64_t bh = blockIdx.z;
  const int i0 = blockIdx.y * kScoreTile, j0 = blockIdx.x * kScoreTile;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const float* qh = qbar + bh * g.NT * g.D;
  const float* kh = kbar + bh * g.NT * g.D;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;

  for (int d0 = 0; d0 < g.D; d0 += kScoreChunk) {
    for (int e = threadIdx.x; e < kScoreTile * kScoreChunk; e += 256) {
      const int r = e / kScoreChunk, cc = e % kScoreChunk;
      qs[r][cc] = (i0 + r < g.NT) ? qh[(int64_t)(i0 + r) * g.D + d0 + cc] : 0.f;
      ks[r][cc] = (j0 + r < g.NT) ? kh[(int64_t)(j0 + r) * g.D + d0 + cc] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int cc = 0; cc < kScoreChunk; ++cc) {
      float qv[4], kv[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) qv[a] = qs[ty + 16 * a][cc];
#pragma unroll
      for (int b = 0; b < 4; ++b) kv[b] = ks[tx + 16 * b][cc];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(qv[a], kv[b], acc[a][b]);
    }
    __syncthreads();
  }
  float* sh = scores + bh * g.NT * (int64_t)g.NT;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int i = i0 + ty + 16 * a;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int j = j0 + tx + 16 * b;
      if (i < g.NT && j < g.NT) sh[(int64_t)i * g.NT + j] = acc[a][b];
    }
  }
}

// Order-preserving map of a float to uint32 (larger float -> larger key);
// -0.0 is folded onto +0.0 first so equal values get equal keys.
__device__ __forceinline__ uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Step 2, Topk + Indexes2mask.  One warp per (head, query tile); candidate j
// sits in lane j % 32, slot j / 32.
template <int SLOTS>
__global__ void __launch_bounds__(256)
select_topk_kernel(Geom g, const float* __restrict__ scores, uint32_t* __restrict__ selbits) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);   // bh * NT + i
  if (row >= (int64_t)g.B * g.H * g.NT) return;
  const float* s = scores + row * g.NT;
  uint32_t* out = selbits + row * g.words;
  const int k = g.k;
  uint32_t key[SLOTS];
#pragma unroll
  for (int w = 0; w < SLOTS; ++w) {
    const int j = w * 32 + lane;
    key[w] = (w < g.words && j < g.NT) ? float_key(s[j]) : 0u;   // 0 is below every real key
  }
  if (k == 0) {
    for (int w = lane; w < g.words; w += 32) out[w] = 0u;
    return;
  }
  // Largest threshold thr with #(key >= thr) >= k: the k-th largest key.
  uint32_t thr = 0;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = thr | (1u << bit);
    int cnt = 0;
#pragma unroll
    for (int w = 0; w < SLOTS; ++w) cnt += (key[w] >= cand) ? 1 : 0;
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (cnt >= k) thr = cand;
  }
  int gt = 0;
#pragma unroll
  for (int w = 0; w < SLOTS; ++w) gt += (key[w] > thr) ? 1 : 0;
  gt = __reduce_add_sync(0xffffffffu, gt);
  const int need = k - gt;          // equal keys to take, lowest tile index first
  int eq_before = 0;
  const uint32_t lt_mask = (1u << lane) - 1u;
#pragma unroll
  for (int w = 0; w < SLOTS; ++w) {
    if (w < g.words) {
      const bool eq = key[w] == thr;
      const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
      const bool take = key[w] > thr || (eq && eq_before + __popc(eqm & lt_mask) < need);
      const uint32_t word = __ballot_sync(0xffffffffu, take);
      if (lane == 0) out[w] = word;
      eq_before += __popc(eqm);
    }
  }
}

// Per-axis window start: the window of span min(w, n) slides inward at the edges.
__device__ __forceinline__ int window_start(int c, int w, int n) {
  const int span = w < n ? w : n;
  int s = c - w / 2;
  s = s < 0 ? 0 : s;
  return s > n - span ? n - span : s;
}

// Steps 3-4: union of selection, window and text tiles -> ascending lists.
__global__ void __launch_bounds__(256)
build_kv_lists_kernel(Geom g, const uint32_t* __restrict__ selbits, int32_t* __restrict__ kv_idx,
                      int32_t* __restrict__ kv_cnt) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);   // bh * NQ + i
  if (row >= (int64_t)g.B * g.H * g.NQ) return;
  const int64_t bh = row / g.NQ;
  const int i = (int)(row - bh * g.NQ);
  int32_t* out = kv_idx + row * g.max_kept;
  const uint32_t lt_mask = (1u << lane) - 1u;
  int base = 0;
  if (i < g.NT) {
    const int cX = i % g.nX, cY = (i / g.nX) % g.nY, cT = i / (g.nX * g.nY);
    const int sT = window_start(cT, g.wT, g.nT), sY = window_start(cY, g.wY, g.nY),
              sX = window_start(cX, g.wX, g.nX);
    const int eT = sT + min(g.wT, g.nT), eY = sY + min(g.wY, g.nY), eX = sX + min(g.wX, g.nX);
    const uint32_t* bits = selbits + (bh * g.NT + i) * g.words;
    for (int w = 0; w < g.words; ++w) {
      const int j = w * 32 + lane;
      bool keep = false;
      if (j < g.NT) {
        const int jX = j % g.nX, jY = (j / g.nX) % g.nY, jT = j / (g.nX * g.nY);
        const bool in_win = jT >= sT && jT < eT && jY >= sY && jY < eY && jX >= sX && jX < eX;
        keep = in_win || ((bits[w] >> lane) & 1u);
      }
      const uint32_t m = __ballot_sync(0xffffffffu, keep);
      if (keep) out[base + __popc(m & lt_mask)] = j;
      base += __popc(m);
    }
    for (int t = lane; t < g.n_text; t += 32) out[base + t] = g.NT + t;
    base += g.n_text;
  } else {
    // text query tile: every video and text tile
    const int total = g.NT + g.n_text;
    for (int t = lane; t < total; t += 32) out[t] = t;
    base = total;
  }
  for (int t = base + lane; t < g.max_kept; t += 32) out[t] = -1;
  if (lane == 0) kv_cnt[row] = base;
}

}  // namespace

MaskWorkspace mask_workspace_layout(const Geom& g) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t bh = (size_t)g.B * g.H;
  MaskWorkspace w;
  w.status = 0;
  w.qbar = 256;
  w.kbar = w.qbar + up(bh * g.NT * g.D * sizeof(float));
  w.scores = w.kbar + up(bh * g.NT * g.D * sizeof(float));
  w.selbits = w.scores + up(bh * g.NT * (size_t)g.NT * sizeof(float));
  w.total = w.selbits + up(bh * g.NT * (size_t)g.words * sizeof(uint32_t));
  return w;
}

cudaError_t launch_tile_pool(const Geom& g, const void* qp, const void* kp, float* qbar, float* kbar,
                             cudaStream_t s) {
  if ((int64_t)g.B * g.H == 0) return cudaSuccess;
  dim3 grid(g.NT, g.B * g.H);
  const int epv = 16 / g.esize;
  const int rpp = kPoolThreads / (g.D / epv);
  const size_t smem = 2 * rpp * g.D * sizeof(float);
  if (g.dtype == SSTA_BF16)
    tile_pool_kernel<__nv_bfloat16><<<grid, kPoolThreads, smem, s>>>(
        g, static_cast<const int4*>(qp), static_cast<const int4*>(kp), qbar, kbar);
  else
    tile_pool_kernel<float><<<grid, kPoolThreads, smem, s>>>(
        g, static_cast<const int4*>(qp), static_cast<const int4*>(kp), qbar, kbar);
  return cudaGetLastError();
}

cudaError_t launch_tile_scores(const Geom& g, const float* qbar, const float* kbar, float* scores,
                               cudaStream_t s) {
  if ((int64_t)g.B * g.H == 0) return cudaSuccess;
  dim3 grid(ceil_div(g.NT, kScoreTile), ceil_div(g.NT, kScoreTile), g.B * g.H);
  tile_scores_kernel<<<grid, 256, 0, s>>>(g, qbar, kbar, scores);
  return cudaGetLastError();
}

cudaError_t launch_select_topk(const Geom& g, const float* scores, uint32_t* selbits, cudaStream_t s) {
  const int64_t rows = (int64_t)g.B * g.H * g.NT;
  if (rows == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((rows + 7) / 8);
  if (g.words <= 8)
    select_topk_kernel<8><<<blocks, 256, 0, s>>>(g, scores, selbits);
  else if (g.words <= 16)
    select_topk_kernel<16><<<blocks, 256, 0, s>>>(g, scores, selbits);
  else if (g.words <= 32)
    select_topk_kernel<32><<<blocks, 256, 0, s>>>(g, scores, selbits);
  else
    select_topk_kernel<64><<<blocks, 256, 0, s>>>(g, scores, selbits);
  return cudaGetLastError();
}

cudaError_t launch_build_kv_lists(const Geom& g, const uint32_t* selbits, int32_t* kv_idx,
                                  int32_t* kv_cnt, cudaStream_t s) {
  const int64_t rows = (int64_t)g.B * g.H * g.NQ;
  if (rows == 0) return cudaSuccess;
  build_kv_lists_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(g, selbits, kv_idx, kv_cnt);
  return cudaGetLastError();
}

}  // namespace ssta
