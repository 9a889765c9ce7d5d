// Backward of Step 4 ("HunyuanVideo 1.5 Technical Report", section "SSTA:
// Selective and Sliding Tile Attention", Step 4 "Combine Masks and Block-Sparse
// Attention": softmax(Q K^T / sqrt(d_k)) V over the kept tiles), for the
// distillation training the pages apply SSTA in.  With P recomputed from the
// forward's LSE, D = rowsum(dO * O) and dS = P * (dO V^T - D):
//   dQ = scale * dS K,  dK = scale * dS^T Q,  dV = P^T dO,
// over the valid keys of the kept tiles of each query tile; pad query rows take
// no part (dQ = 0) and pad keys get dK = dV = 0.
//
// Kernels, in launch order:
//   bwd_rowdot_kernel     D per packed row (fp32; bf16 runs bwd_rowstat_tc_kernel,
//                         which also writes -LSE * log2(e) and -D per row of whole
//                         tiles, as the tensor-core dK/dV kernel reads them).
//   bwd_transpose_kernel  for each key tile, the ascending list of query tiles
//                         that keep it (one warp per key tile: a binary search
//                         in every query tile's sorted list, ballots, prefix).
//   bwd_dq_kernel         one warp per query row, walking its tile's kept list
//                         (fp32; bf16 runs bwd_dq_tc_kernel on the tensor cores).
//   bwd_dkdv_kernel       one warp per key row, walking the transposed list
//                         (fp32; bf16 runs bwd_dkdv_tc_kernel on the tensor cores).
// The SIMT kernels (fp32 storage) use fp32 arithmetic, one lane per four
// channels; for bf16 every product runs on the tensor cores
// (ssta_attn_bwd_tc.cu).
#include "ssta_internal.h"

#include <cuda_bf16.h>

#include <algorithm>

namespace ssta {
namespace {

constexpr int kBwdWarps = 8;

// Four channels of a row as fp32 (lane `lane` of a 128-channel row).
__device__ __forceinline__ float4 load4(const float* base, int64_t row, int lane) {
  return reinterpret_cast<const float4*>(base + row * 128)[lane];
}
__device__ __forceinline__ float4 load4(const __nv_bfloat16* base, int64_t row, int lane) {
  const uint2 raw = reinterpret_cast<const uint2*>(base + row * 128)[lane];
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ void store4(float* base, int64_t row, int lane, float4 v) {
  reinterpret_cast<float4*>(base + row * 128)[lane] = v;
}
__device__ __forceinline__ void store4(__nv_bfloat16* base, int64_t row, int lane, float4 v) {
  const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
  uint2 raw;
  raw.x = *reinterpret_cast<const uint32_t*>(&a);
  raw.y = *reinterpret_cast<const uint32_t*>(&b);
  reinterpret_cast<uint2*>(base + row * 128)[lane] = raw;
}
__device__ __forceinline__ float dot4(float4 a, float4 b) { return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w; }
__device__ __forceinline__ void axpy4(float a, float4 x, float4& y) {
  y.x = fmaf(a, x.x, y.x); y.y = fmaf(a, x.y, y.y); y.z = fmaf(a, x.z, y.z); y.w = fmaf(a, x.w, y.w);
}
// Two warp-wide sums at once (butterfly: every lane ends with both totals).
__device__ __forceinline__ void warp_sum2(float& a, float& b) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, off);
    b += __shfl_xor_sync(0xffffffffu, b, off);
  }
}

// Valid extents of tile t: video tiles may be partial at the grid's far edges;
// text tiles hold the text rows that remain.
struct TileValid {
  int vt, vy, vx, text;
};
__device__ __forceinline__ TileValid tile_valid(const Geom& g, int t) {
  TileValid v{g.tT, g.tY, g.tX, g.N};
  if (t < g.NT) {
    const int cX = t % g.nX, cY = (t / g.nX) % g.nY, cT = t / (g.nX * g.nY);
    v.vt = axis_valid(cT, g.tT, g.T);
    v.vy = axis_valid(cY, g.tY, g.Y);
    v.vx = axis_valid(cX, g.tX, g.X);
  } else {
    v.text = g.L_text - (t - g.NT) * g.N;
  }
  return v;
}
__device__ __forceinline__ bool row_valid(const Geom& g, int t, const TileValid& v, int o) {
  if (t < g.NT) {
    const int dx = o % g.tX, dy = (o / g.tX) % g.tY, dt = o / (g.tX * g.tY);
    return dt < v.vt && dy < v.vy && dx < v.vx;
  }
  return o < v.text;
}

// D = rowsum(dO * O) per packed row for the fp32 kernels (bf16 uses
// bwd_rowstat_tc_kernel): each lane reads 16 bytes (4 channels), 32 lanes per row,
// four rows per warp with every load issued before the first sum; grid.y is the head.
constexpr int kRowdotRows = 4;
template <typename T>
__global__ void __launch_bounds__(kBwdWarps * 32)
bwd_rowdot_kernel(Geom g, int64_t bh0, const T* __restrict__ o, const T* __restrict__ dO, float* __restrict__ Dv) {
  const int lane = threadIdx.x & 31;
  const int64_t bh = bh0 + blockIdx.y;
  const int64_t r0 = ((int64_t)blockIdx.x * kBwdWarps + (threadIdx.x >> 5)) * kRowdotRows;
  float4 va[kRowdotRows], vb[kRowdotRows];
  bool valid[kRowdotRows];
#pragma unroll
  for (int it = 0; it < kRowdotRows; ++it) {
    const int64_t row = r0 + it;
    const int t = (int)(row / g.N);
    valid[it] = row < g.Lq && row_valid(g, t, tile_valid(g, t), (int)(row - (int64_t)t * g.N));
    va[it] = valid[it] ? load4(o, bh * g.Lq + row, lane) : make_float4(0.f, 0.f, 0.f, 0.f);
    vb[it] = valid[it] ? load4(dO, bh * g.Lq + row, lane) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int it = 0; it < kRowdotRows; it += 2) {
    float d0 = dot4(va[it], vb[it]), d1 = dot4(va[it + 1], vb[it + 1]);
    warp_sum2(d0, d1);
    if (lane == 0) {
      if (r0 + it < g.Lq) Dv[bh * g.Lq + r0 + it] = d0;
      if (r0 + it + 1 < g.Lq) Dv[bh * g.Lq + r0 + it + 1] = d1;
    }
  }
}

// For key tile j of head bh: tidx[bh][j][0..tcnt) = query tiles i (ascending) whose
// kept list holds j.  Lists are ascending (as ssta_build_block_mask writes them).
__global__ void __launch_bounds__(kBwdWarps * 32)
bwd_transpose_kernel(Geom g, const int32_t* __restrict__ kv_idx, const int32_t* __restrict__ kv_cnt,
                     int32_t* __restrict__ tidx, int32_t* __restrict__ tcnt, int32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const int64_t w = (int64_t)blockIdx.x * kBwdWarps + (threadIdx.x >> 5);   // bh * NQ + j
  if (w >= (int64_t)g.B * g.H * g.NQ) return;
  const int64_t bh = w / g.NQ;
  const int j = (int)(w - bh * g.NQ);
  int32_t* out = tidx + w * g.NQ;
  int n = 0;
  for (int i0 = 0; i0 < g.NQ; i0 += 32) {
    const int i = i0 + lane;
    bool keeps = false;
    if (i < g.NQ) {
      const int64_t lr = bh * g.NQ + i;
      int c = kv_cnt[lr];
      if (c < 0 || c > g.max_kept) {
        atomicExch(status, (int)SSTA_ERR_DEVICE_BOUNDS);
        c = c < 0 ? 0 : g.max_kept;
      }
      const int32_t* l = kv_idx + lr * g.max_kept;
      int lo = 0, hi = c;                      // first entry >= j
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (l[mid] < j) lo = mid + 1; else hi = mid;
      }
      keeps = lo < c && l[lo] == j;
    }
    const uint32_t m = __ballot_sync(0xffffffffu, keeps);
    if (keeps) out[n + __popc(m & ((1u << lane) - 1u))] = i;
    n += __popc(m);
  }
  if (lane == 0) tcnt[w] = n;
}

template <typename T>
__global__ void __launch_bounds__(kBwdWarps * 32)
bwd_dq_kernel(Geom g, const T* __restrict__ qp, const T* __restrict__ kp, const T* __restrict__ vp,
              const T* __restrict__ dOp, const float* __restrict__ lse, const float* __restrict__ Dv,
              const int32_t* __restrict__ kv_idx, const int32_t* __restrict__ kv_cnt, T* __restrict__ dq,
              int32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const int64_t w = (int64_t)blockIdx.x * kBwdWarps + (threadIdx.x >> 5);   // bh * Lq + row
  if (w >= (int64_t)g.B * g.H * g.Lq) return;
  const int64_t bh = w / g.Lq, row = w % g.Lq, head = bh * g.Lq;
  const int i = (int)(row / g.N);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  const float L = lse[w];
  if (row_valid(g, i, tile_valid(g, i), (int)(row - (int64_t)i * g.N)) && L > -INFINITY) {
    const float4 q = load4(qp, w, lane), d_o = load4(dOp, w, lane);
    const float Dr = Dv[w];
    const int64_t lr = bh * g.NQ + i;
    int cnt = kv_cnt[lr];
    if (cnt < 0 || cnt > g.max_kept) {
      if (lane == 0) atomicExch(status, (int)SSTA_ERR_DEVICE_BOUNDS);
      cnt = cnt < 0 ? 0 : g.max_kept;
    }
    const int32_t* list = kv_idx + lr * g.max_kept;
    for (int e = 0; e < cnt; ++e) {
      const int t = list[e];
      if (t < 0 || t >= g.NQ) {
        if (lane == 0) atomicExch(status, (int)SSTA_ERR_DEVICE_BOUNDS);
        continue;
      }
      const TileValid tv = tile_valid(g, t);
      for (int kk = 0; kk < g.N; ++kk) {
        if (!row_valid(g, t, tv, kk)) continue;
        const int64_t krow = head + (int64_t)t * g.N + kk;
        const float4 k = load4(kp, krow, lane), v = load4(vp, krow, lane);
        float s = dot4(q, k), dp = dot4(d_o, v);
        warp_sum2(s, dp);
        const float p = expf(s * g.scale - L);
        axpy4(p * (dp - Dr), k, acc);
      }
    }
  }
  acc.x *= g.scale; acc.y *= g.scale; acc.z *= g.scale; acc.w *= g.scale;
  store4(dq, w, lane, acc);
}

template <typename T>
__global__ void __launch_bounds__(kBwdWarps * 32)
bwd_dkdv_kernel(Geom g, const T* __restrict__ qp, const T* __restrict__ kp, const T* __restrict__ vp,
                const T* __restrict__ dOp, const float* __restrict__ lse, const float* __restrict__ Dv,
                const int32_t* __restrict__ tidx, const int32_t* __restrict__ tcnt, T* __restrict__ dk,
                T* __restrict__ dv) {
  const int lane = threadIdx.x & 31;
  const int64_t w = (int64_t)blockIdx.x * kBwdWarps + (threadIdx.x >> 5);   // bh * Lq + key row
  if (w >= (int64_t)g.B * g.H * g.Lq) return;
  const int64_t bh = w / g.Lq, row = w % g.Lq, head = bh * g.Lq;
  const int j = (int)(row / g.N);
  float4 ak = make_float4(0.f, 0.f, 0.f, 0.f), av = make_float4(0.f, 0.f, 0.f, 0.f);
  if (row_valid(g, j, tile_valid(g, j), (int)(row - (int64_t)j * g.N))) {
    const float4 k = load4(kp, w, lane), v = load4(vp, w, lane);
    const int64_t tr = bh * g.NQ + j;
    const int n = tcnt[tr];
    const int32_t* list = tidx + tr * g.NQ;
    for (int e = 0; e < n; ++e) {
      const int i = list[e];
      const TileValid tv = tile_valid(g, i);
      for (int r = 0; r < g.N; ++r) {
        const int64_t qrow = (int64_t)i * g.N + r;
        if (qrow >= g.Lq || !row_valid(g, i, tv, r)) continue;
        const float L = lse[head + qrow];
        if (!(L > -INFINITY)) continue;
        const float4 q = load4(qp, head + qrow, lane), d_o = load4(dOp, head + qrow, lane);
        float s = dot4(q, k), dp = dot4(d_o, v);
        warp_sum2(s, dp);
        const float p = expf(s * g.scale - L);
        axpy4(p, d_o, av);
        axpy4(p * (dp - Dv[head + qrow]), q, ak);
      }
    }
  }
  ak.x *= g.scale; ak.y *= g.scale; ak.z *= g.scale; ak.w *= g.scale;
  store4(dk, w, lane, ak);
  store4(dv, w, lane, av);
}

template <typename T>
constexpr bool kTensorCores = false;   // bf16: dQ, dK and dV run on the tensor cores (ssta_attn_bwd_tc.cu)
template <>
constexpr bool kTensorCores<__nv_bfloat16> = true;

template <typename T>
cudaError_t launch_bwd_typed(const Geom& g, const void* q, const void* k, const void* v, const void* o,
                             const float* lse, const void* dO, const int32_t* kv_idx, const int32_t* kv_cnt,
                             void* dq, void* dk, void* dv, const BwdWorkspace& ws, uint8_t* base, cudaStream_t s) {
  const int64_t rows = (int64_t)g.B * g.H * g.Lq, tiles = (int64_t)g.B * g.H * g.NQ;
  float* Dv = reinterpret_cast<float*>(base + ws.rowdot);
  int32_t* tidx = reinterpret_cast<int32_t*>(base + ws.tidx);
  int32_t* tcnt = reinterpret_cast<int32_t*>(base + ws.tcnt);
  int32_t* status = reinterpret_cast<int32_t*>(base + ws.status);
  const unsigned rb = (unsigned)((rows + kBwdWarps - 1) / kBwdWarps), tb = (unsigned)((tiles + kBwdWarps - 1) / kBwdWarps);
  const T* tq = static_cast<const T*>(q);
  const T* tk = static_cast<const T*>(k);
  const T* tv = static_cast<const T*>(v);
  const T* tO = static_cast<const T*>(dO);
  float* nl2 = reinterpret_cast<float*>(base + ws.nl2);
  float* nd = reinterpret_cast<float*>(base + ws.nd);
  if constexpr (kTensorCores<T>) {
    cudaError_t e = launch_attention_bwd_rowstat_tc(g, o, dO, lse, Dv, nl2, nd, s);
    if (e != cudaSuccess) return e;
  } else {
    const int64_t rows_per_block = (int64_t)kBwdWarps * kRowdotRows, BH = (int64_t)g.B * g.H;
    for (int64_t bh0 = 0; bh0 < BH; bh0 += 65535) {   // grid.y holds at most 65535 heads
      const dim3 grid((unsigned)((g.Lq + rows_per_block - 1) / rows_per_block), (unsigned)std::min<int64_t>(BH - bh0, 65535));
      bwd_rowdot_kernel<T><<<grid, kBwdWarps * 32, 0, s>>>(g, bh0, static_cast<const T*>(o), tO, Dv);
    }
  }
  bwd_transpose_kernel<<<tb, kBwdWarps * 32, 0, s>>>(g, kv_idx, kv_cnt, tidx, tcnt, status);
  if constexpr (kTensorCores<T>) {   // bf16: the API guarantees N % 128 == 0
    cudaError_t e = launch_attention_bwd_dq_tc(g, q, k, v, dO, lse, Dv, kv_idx, kv_cnt, dq, status, s);
    if (e != cudaSuccess) return e;
    e = launch_attention_bwd_dkdv_tc(g, q, k, v, dO, nl2, nd, tidx, tcnt, dk, dv, status, s);
    if (e != cudaSuccess) return e;
  } else {
    bwd_dq_kernel<T><<<rb, kBwdWarps * 32, 0, s>>>(g, tq, tk, tv, tO, lse, Dv, kv_idx, kv_cnt, static_cast<T*>(dq),
                                                   status);
    bwd_dkdv_kernel<T><<<rb, kBwdWarps * 32, 0, s>>>(g, tq, tk, tv, tO, lse, Dv, tidx, tcnt, static_cast<T*>(dk),
                                                     static_cast<T*>(dv));
  }
  return cudaGetLastError();
}

}  // namespace

BwdWorkspace bwd_workspace_layout(const Geom& g) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t bh = (size_t)g.B * g.H;
  BwdWorkspace w{};
  w.status = 0;
  w.rowdot = 256;
  w.nl2 = w.rowdot + up(bh * (size_t)g.Lq * sizeof(float));
  w.nd = w.nl2 + up(bh * (size_t)g.NQ * g.N * sizeof(float));
  w.tcnt = w.nd + up(bh * (size_t)g.NQ * g.N * sizeof(float));
  w.tidx = w.tcnt + up(bh * (size_t)g.NQ * sizeof(int32_t));
  w.total = w.tidx + up(bh * (size_t)g.NQ * g.NQ * sizeof(int32_t));
  return w;
}

cudaError_t launch_attention_bwd(const Geom& g, const void* q, const void* k, const void* v, const void* o,
                                 const float* lse, const void* dO, const int32_t* kv_idx, const int32_t* kv_cnt,
                                 void* dq, void* dk, void* dv, void* workspace, cudaStream_t s) {
  if ((int64_t)g.B * g.H == 0) return cudaSuccess;
  const BwdWorkspace ws = bwd_workspace_layout(g);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  if (g.dtype == SSTA_BF16)
    return launch_bwd_typed<__nv_bfloat16>(g, q, k, v, o, lse, dO, kv_idx, kv_cnt, dq, dk, dv, ws, base, s);
  return launch_bwd_typed<float>(g, q, k, v, o, lse, dO, kv_idx, kv_cnt, dq, dk, dv, ws, base, s);
}

}  // namespace ssta
