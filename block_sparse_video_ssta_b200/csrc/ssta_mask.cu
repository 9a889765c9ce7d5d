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
//                         reduces per-channel fp32 sums across row groups; the
//                         means are stored channel-major for the score kernel.
//   tile_keysum_kernel    importance score only: per 32-tile block sums of the
//                         unit key means (the pool kernel writes the norms);
//                         the score kernel turns them into each key tile's
//                         redundancy (mean key-key similarity to the other key
//                         tiles) in O(NT*D) per head, without an NT x NT product.
//   tile_scores_tc_kernel similarity score on the tensor cores, fp32 means split
//                         into three bf16 parts (ssta_mask_tc.cu).
//   tile_scores_kernel    importance score: fp32 SIMT, 128x128 score blocks per CTA,
//                         8x8 per thread, 16-channel stages double-buffered in
//                         shared memory by cp.async, channels summed in order
//                         0..D-1 with FMA (packed f32x2, two columns per
//                         instruction); the importance score is formed in the
//                         epilogue.
//   select_and_list_kernel one warp per (head, query tile): top-k over scores
//                         held in registers as order-preserving 32-bit keys
//                         (bitwise binary search for the k-th key with warp-wide
//                         counts, ties to the lower tile index by ballots in
//                         index order), OR-ed (or AND-ed) word by word with the window
//                         (contiguous index ranges) and compacted into the
//                         ascending kept list by a warp prefix sum.
#include "ssta_internal.h"

#include <cuda_bf16.h>

#include "ssta_f32x2.cuh"

namespace ssta {
namespace {

using namespace f32x2;

// Programmatic dependent launch: a kernel launched with launch_dependent() may start
// while the previous kernel of the stream is still running; grid_dependency_wait()
// blocks until that kernel has completed and its writes are visible, and
// allow_dependents() lets the next kernel start launching.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
// A pointer to data the previous kernel writes, passed through an empty asm after the wait: the
// compiler then cannot issue loads through it (which it may treat as reads of invariant memory,
// being const __restrict__) ahead of griddepcontrol.wait.
template <typename T>
__device__ __forceinline__ T* after_wait(T* p) {
  asm volatile("" : "+l"(p)::"memory");
  return p;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

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

// Valid rows of a video tile, one bit per token, for each of the 8 tile classes (bit 2 of
// the class: last tile along T with padding, bit 1: along Y, bit 0: along X); built on the
// host, so a partial tile's rows are tested with a shift instead of three divisions.
constexpr int kMaxRowWords = 4096 / 32;   // N <= 4096
struct PoolRowMask {
  uint32_t w[8][kMaxRowWords];
};
PoolRowMask make_pool_row_mask(const Geom& g) {
  PoolRowMask m{};
  for (int cls = 0; cls < 8; ++cls) {
    const int vt = (cls & 4) ? g.T - (g.nT - 1) * g.tT : g.tT;
    const int vy = (cls & 2) ? g.Y - (g.nY - 1) * g.tY : g.tY;
    const int vx = (cls & 1) ? g.X - (g.nX - 1) * g.tX : g.tX;
    for (int o = 0; o < g.N && o < 32 * kMaxRowWords; ++o) {
      const int dx = o % g.tX, dy = (o / g.tX) % g.tY, dt = o / (g.tX * g.tY);
      if (dt < vt && dy < vy && dx < vx) m.w[cls][o >> 5] |= 1u << (o & 31);
    }
  }
  return m;
}

// Step 2, pooled (average) representation of each video tile over its valid tokens.
template <typename T>
__global__ void __launch_bounds__(kPoolThreads, 4)   // 64 registers: four CTAs per SM
tile_pool_kernel(Geom g, const __grid_constant__ PoolRowMask rm, const int4* __restrict__ qp,
                 const int4* __restrict__ kp, float* __restrict__ qbar, float* __restrict__ kbar,
                 int32_t* __restrict__ status, ImportanceBufs ib) {
  allow_dependents();
  grid_dependency_wait();   // q and k are packed by the previous kernels
  qp = after_wait(qp);
  kp = after_wait(kp);
  if (status != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *status = 0;
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
  __shared__ uint32_t mask[kMaxRowWords];   // this tile's valid rows (partial tiles)
  if (!full) {
    const int cls = (vt < g.tT ? 4 : 0) | (vy < g.tY ? 2 : 0) | (vx < g.tX ? 1 : 0);
    for (int i = threadIdx.x; i < (g.N + 31) / 32; i += kPoolThreads) mask[i] = rm.w[cls][i];
    __syncthreads();
  }

  const int64_t base = (bh * g.Lq + (int64_t)c * g.N) * vpr + vec;
  float aq[EPV], ak[EPV];
#pragma unroll
  for (int i = 0; i < EPV; ++i) aq[i] = ak[i] = 0.f;

  if (full) {
    int o = rsub;
    for (; o + 7 * rpp < g.N; o += 8 * rpp) {
      int4 rq[8], rk[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        rq[u] = __ldg(qp + base + (int64_t)(o + u * rpp) * vpr);
        rk[u] = __ldg(kp + base + (int64_t)(o + u * rpp) * vpr);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        add_vec(aq, rq[u], (const T*)nullptr);
        add_vec(ak, rk[u], (const T*)nullptr);
      }
    }
    for (; o < g.N; o += rpp) {
      add_vec(aq, __ldg(qp + base + (int64_t)o * vpr), (const T*)nullptr);
      add_vec(ak, __ldg(kp + base + (int64_t)o * vpr), (const T*)nullptr);
    }
  } else {
    // the same batched loads; pad rows load nothing and add zeros, which leaves every sum
    // (taken in the same row order) unchanged
    const int4 zero = make_int4(0, 0, 0, 0);
    int o = rsub;
    for (; o + 7 * rpp < g.N; o += 8 * rpp) {
      int4 rq[8], rk[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int r = o + u * rpp;
        const bool ok = (mask[r >> 5] >> (r & 31)) & 1u;
        rq[u] = ok ? __ldg(qp + base + (int64_t)r * vpr) : zero;
        rk[u] = ok ? __ldg(kp + base + (int64_t)r * vpr) : zero;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        add_vec(aq, rq[u], (const T*)nullptr);
        add_vec(ak, rk[u], (const T*)nullptr);
      }
    }
    for (; o < g.N; o += rpp) {
      if ((mask[o >> 5] >> (o & 31)) & 1u) {
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
  float sq[2] = {0.f, 0.f};   // squares of this thread's means, for q and for k
  for (int t = threadIdx.x; t < 2 * D; t += kPoolThreads) {
    const int which = t / D, ch = t % D;
    float s = 0.f;
    for (int r = 0; r < rpp; ++r) s += red[(which * rpp + r) * D + ch];
    float* out = which ? kbar : qbar;
    const float mean = s * inv;
    out[(bh * D + ch) * g.NT + c] = mean;     // channel-major: [head][channel][tile]
    sq[which] = fmaf(mean, mean, sq[which]);
  }
  if (ib.inv_nq != nullptr) {
    // importance score: 1 / |mean| of q and of k (0 for an all-zero mean), fixed-order reduction
    __shared__ float nsq[2][kPoolThreads / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      float v = sq[which];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_down_sync(0xffffffffu, v, off);
      if (lane == 0) nsq[which][warp] = v;
    }
    __syncthreads();
    if (threadIdx.x < 2) {
      float a = 0.f;
      for (int w = 0; w < kPoolThreads / 32; ++w) a += nsq[threadIdx.x][w];
      (threadIdx.x ? ib.inv_nk : ib.inv_nq)[bh * g.NT + c] = a > 0.f ? 1.0f / sqrtf(a) : 0.f;
    }
  }
}

// Step 2, importance score, pre-pass (one CTA per 32 key tiles of one head, one
// thread per channel): this block's sum of the unit-length key means,
// sum_j Kbar_j[d] / |Kbar_j| in tile order, for the redundancy term.
constexpr int kKeySumTiles = 32;

__global__ void __launch_bounds__(128)
tile_keysum_kernel(Geom g, const float* __restrict__ kbar_t, ImportanceBufs ib) {
  allow_dependents();
  grid_dependency_wait();   // the means and norms are written by the previous kernel
  kbar_t = after_wait(kbar_t);
  ib.inv_nk = after_wait(ib.inv_nk);
  const int64_t bh = blockIdx.y;
  const int NT = g.NT;
  const int c0 = blockIdx.x * kKeySumTiles, c1 = min(c0 + kKeySumTiles, NT);
  __shared__ float ik[kKeySumTiles];
  if (threadIdx.x < kKeySumTiles) ik[threadIdx.x] = c0 + (int)threadIdx.x < NT ? ib.inv_nk[bh * NT + c0 + threadIdx.x] : 0.f;
  __syncthreads();
  for (int d = threadIdx.x; d < g.D; d += 128) {
    const float* row = kbar_t + (bh * g.D + d) * (int64_t)NT;
    float a = 0.f;
    for (int c = c0; c < c1; ++c) a = fmaf(row[c], ik[c - c0], a);
    ib.ksum[(bh * g.norm_blocks + blockIdx.x) * g.D + d] = a;
  }
}

// Step 2, Score_s = Qbar Kbar^T.  One CTA computes a 128 x 128 block of scores
// of one head with 256 threads; thread (ty, tx) of a 16 x 16 grid owns rows
// {4ty..4ty+3, 64+4ty..64+4ty+3} and the same pattern of columns, i.e. 8 x 8
// scores, so one channel costs it four 16-byte shared loads for 64 FMAs.  The
// pooled means arrive channel-major ([head][channel][tile]); 16 channels of the
// CTA's 128 query tiles and 128 key tiles form one stage, copied global ->
// shared by cp.async (16-byte copies when NT % 4 == 0, else 4-byte ones; tiles
// past NT are zero-filled) into two buffers, so the next stage is in flight
// while the current one is consumed.  Every score is accumulated over channels
// 0..D-1 in order with FMA, two adjacent columns per fma.rn.f32x2 instruction.

constexpr int kScoreBlock = 128;
constexpr int kScoreStage = 16;   // channels per stage

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem), "r"(valid ? 16 : 0) : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem, const void* gmem, bool valid) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(s), "l"(gmem), "r"(valid ? 4 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// One stage: channels d0..d0+15 of the CTA's query tiles (Qbar) and key tiles (Kbar).
// Out-of-range tiles copy zero bytes from the head's base address (always valid).
template <bool kVec>
__device__ __forceinline__ void score_stage_copy(float (*qs)[kScoreBlock], float (*ks)[kScoreBlock], const float* qh,
                                                 const float* kh, int NT, int i0, int j0, int d0) {
  if constexpr (kVec) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int e = threadIdx.x + 256 * u, ch = e >> 5, r = (e & 31) * 4;
      const bool qi = i0 + r < NT, kj = j0 + r < NT;
      cp_async16(&qs[ch][r], qi ? qh + (int64_t)(d0 + ch) * NT + i0 + r : qh, qi);
      cp_async16(&ks[ch][r], kj ? kh + (int64_t)(d0 + ch) * NT + j0 + r : kh, kj);
    }
  } else {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = threadIdx.x + 256 * u, ch = e >> 7, r = e & 127;
      const bool qi = i0 + r < NT, kj = j0 + r < NT;
      cp_async4(&qs[ch][r], qi ? qh + (int64_t)(d0 + ch) * NT + i0 + r : qh, qi);
      cp_async4(&ks[ch][r], kj ? kh + (int64_t)(d0 + ch) * NT + j0 + r : kh, kj);
    }
  }
}

template <bool kVec>
__global__ void __launch_bounds__(256, 2)
tile_scores_kernel(Geom g, const float* __restrict__ qbar_t, const float* __restrict__ kbar_t,
                   ImportanceBufs ib, float* __restrict__ scores) {
  __shared__ __align__(16) float qs[2][kScoreStage][kScoreBlock];
  __shared__ __align__(16) float ks[2][kScoreStage][kScoreBlock];
  const int64_t bh = blockIdx.z;
  const int NT = g.NT;
  const int i0 = blockIdx.y * kScoreBlock, j0 = blockIdx.x * kScoreBlock;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const float* qh = qbar_t + bh * g.D * (int64_t)NT;
  const float* kh = kbar_t + bh * g.D * (int64_t)NT;
  uint64_t acc[8][4];   // pairs of adjacent columns (f32x2)
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0ull;

  const int nst = g.D / kScoreStage;
  allow_dependents();
  grid_dependency_wait();   // the pooled means are written by the previous kernel
  qbar_t = after_wait(qbar_t);
  kbar_t = after_wait(kbar_t);
  ib.inv_nq = after_wait(ib.inv_nq);
  ib.inv_nk = after_wait(ib.inv_nk);
  ib.ksum = after_wait(ib.ksum);
  // importance score: u = sum of the unit key means of the head (partial sums added in
  // block order), and Kbar_j . u for this CTA's 128 key tiles, accumulated from the
  // staged key means by two threads per tile (channels 0-7 and 8-15 of each stage)
  const bool imp = ib.ksum != nullptr;
  __shared__ float u_s[128], kd_s[2][kScoreBlock], red_s[kScoreBlock];
  float kd = 0.f;
  if (imp) {
    for (int d = threadIdx.x; d < g.D; d += 256) {
      float a = 0.f;
      for (int b = 0; b < g.norm_blocks; ++b) a += ib.ksum[(bh * g.norm_blocks + b) * g.D + d];
      u_s[d] = a;
    }
  }
  score_stage_copy<kVec>(qs[0], ks[0], qh, kh, NT, i0, j0, 0);
  cp_async_commit();
  for (int st = 0; st < nst; ++st) {
    const int buf = st & 1;
    if (st + 1 < nst) {
      // buffer buf^1 was last read in stage st-1, which every thread has left
      score_stage_copy<kVec>(qs[buf ^ 1], ks[buf ^ 1], qh, kh, NT, i0, j0, (st + 1) * kScoreStage);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();   // stage st visible to every thread
#pragma unroll
    for (int c = 0; c < kScoreStage; ++c) {
      const float4 qa = *reinterpret_cast<const float4*>(&qs[buf][c][4 * ty]);
      const float4 qb = *reinterpret_cast<const float4*>(&qs[buf][c][64 + 4 * ty]);
      const float4 ka = *reinterpret_cast<const float4*>(&ks[buf][c][4 * tx]);
      const float4 kb = *reinterpret_cast<const float4*>(&ks[buf][c][64 + 4 * tx]);
      const float qv[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
      const uint64_t k2[4] = {f2_pack(ka.x, ka.y), f2_pack(ka.z, ka.w), f2_pack(kb.x, kb.y), f2_pack(kb.z, kb.w)};
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        const uint64_t q2 = f2_pack(qv[a], qv[a]);
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = f2_fma(q2, k2[b], acc[a][b]);
      }
    }
    if (imp) {
      const int cc = threadIdx.x & 127, c8 = (threadIdx.x >> 7) * 8;
#pragma unroll
      for (int c = 0; c < 8; ++c) kd = fmaf(ks[buf][c8 + c][cc], u_s[st * kScoreStage + c8 + c], kd);
    }
    __syncthreads();   // every thread is done with buffer buf before it is refilled
  }
  float* sh = scores + bh * NT * (int64_t)NT;
  // importance score: lambda (cos + 1) / 2 - (1 - lambda) red_j with cos = dot / (|Qbar_i| |Kbar_j|)
  // and red_j = the mean over j' != j of (u_j' . u_j + 1) / 2 (u = unit key means),
  // through sum_{j' != j} u_j' . u_j = (sum_j' u_j') . u_j - |u_j|^2 (0 when NT = 1)
  float ck[8], rk[8];
  if (imp) {
    kd_s[threadIdx.x >> 7][threadIdx.x & 127] = kd;
    __syncthreads();
    if (threadIdx.x < kScoreBlock) {
      const int j = j0 + (int)threadIdx.x;
      const float ik = j < NT ? ib.inv_nk[bh * NT + j] : 0.f;
      const float self = ik > 0.f ? 1.0f : 0.f;
      const float dot = (kd_s[0][threadIdx.x] + kd_s[1][threadIdx.x]) * ik;
      red_s[threadIdx.x] = NT > 1 ? 0.5f + (dot - self) / (2.0f * (float)(NT - 1)) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      const int jj = b < 4 ? 4 * tx + b : 64 + 4 * tx + b - 4, j = j0 + jj;
      ck[b] = j < NT ? ib.inv_nk[bh * NT + j] : 0.f;
      rk[b] = (1.0f - g.lambda) * red_s[jj];
    }
  }
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int i = i0 + (a < 4 ? 4 * ty + a : 64 + 4 * ty + a - 4);
    if (i >= NT) continue;
    float* srow = sh + (int64_t)i * NT;
    const float cq = imp ? ib.inv_nq[bh * NT + i] : 0.f;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int j = j0 + 64 * half + 4 * tx;
      float v[4];
      f2_unpack(acc[a][2 * half], v[0], v[1]);
      f2_unpack(acc[a][2 * half + 1], v[2], v[3]);
      if (imp) {
#pragma unroll
        for (int b = 0; b < 4; ++b)
          v[b] = g.lambda * 0.5f * (v[b] * cq * ck[4 * half + b] + 1.0f) - rk[4 * half + b];
      }
      if constexpr (kVec) {
        if (j < NT) *reinterpret_cast<float4*>(srow + j) = make_float4(v[0], v[1], v[2], v[3]);
      } else {
#pragma unroll
        for (int b = 0; b < 4; ++b)
          if (j + b < NT) srow[j + b] = v[b];
      }
    }
  }
}

// Order-preserving map of a float to uint32 (larger float -> larger key);
// -0.0 is folded onto +0.0 first so equal values get equal keys.
__device__ __forceinline__ uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Per-axis window start: the window of span min(w, n) slides inward at the edges.
__device__ __forceinline__ int window_start(int c, int w, int n) {
  const int span = w < n ? w : n;
  int s = c - w / 2;
  s = s < 0 ? 0 : s;
  return s > n - span ? n - span : s;
}

// Bits of tile indices [32*word, 32*word+32) that fall in [lo, hi).
__device__ __forceinline__ uint32_t range_bits(int word, int lo, int hi) {
  const int a = max(lo - 32 * word, 0), b = min(hi - 32 * word, 32);
  if (a >= b) return 0u;
  const uint32_t upto_b = b == 32 ? 0xffffffffu : ((1u << b) - 1u);
  return upto_b & ~((1u << a) - 1u);
}

// Steps 2-4 for one (head, query tile) per warp:
//  * Topk + Indexes2mask (video query tiles): the scores of the row are held in
//    registers as order-preserving 32-bit keys (candidate j in lane j % 32, slot
//    j / 32); the k-th largest key is found by a bitwise binary search with
//    warp-wide counts (upper 16 bits over all keys, lower 16 bits over the keys
//    sharing that upper half); keys above it are taken, and keys equal to it are
//    taken in ascending tile order until k are chosen (ties to the lower index);
//  * the window (Step 3, shifted or truncated at the grid edges) as unions of
//    contiguous index ranges, one per (t, y) tile row of the window, OR-ed (union)
//    or AND-ed (Algorithm 1's intersection) word by word with the selection;
//  * the union (Step 4) written as an ascending list by a warp prefix sum over the
//    32-tile words, followed by the text tiles and -1 padding.
// Text query tiles keep every tile.
constexpr int kBucketCap = 64;
constexpr int kHiBits = 12;       // prefix bits searched over every key
constexpr int kHiBitsWide = 16;   // ... when the 12-bit bucket holds more than kBucketCap keys

template <int SLOTS>
__global__ void __launch_bounds__(256, 4)   // 4 CTAs per SM: 62 registers, no spills at SLOTS <= 32
select_and_list_kernel(Geom g, const float* __restrict__ scores, int32_t* __restrict__ kv_idx,
                       int32_t* __restrict__ kv_cnt) {
  __shared__ uint32_t bucket_smem[8 * kBucketCap];
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);   // bh * NQ + i
  if (row >= (int64_t)g.B * g.H * g.NQ) return;
  grid_dependency_wait();   // the scores are written by the previous kernel
  scores = after_wait(scores);
  const int64_t bh = row / g.NQ;
  const int i = (int)(row - bh * g.NQ);
  int32_t* out = kv_idx + row * g.max_kept;
  const uint32_t lt_mask = (1u << lane) - 1u;
  int base = 0;
  if (i < g.NT) {
    // ---- selection
    const float* srow = scores + (bh * g.NT + i) * (int64_t)g.NT;
    uint32_t key[SLOTS];
#pragma unroll
    for (int w = 0; w < SLOTS; ++w) {
      const int j = w * 32 + lane;
      key[w] = (w < g.words && j < g.NT) ? float_key(srow[j]) : 0u;   // 0 is below every real key
    }
    uint32_t myword[(SLOTS + 31) / 32];   // lane holds selection words lane and lane + 32
#pragma unroll
    for (int q = 0; q < (SLOTS + 31) / 32; ++q) myword[q] = 0u;
    const int k = g.k;
    if (k > 0) {
      // k-th largest key in two levels: a bitwise search over the upper 12 bits of every
      // key (16 when more than 64 keys share the found 12-bit prefix, as for scores
      // packed into a narrow range), then over the remaining low bits of the keys that
      // share the found prefix (the boundary bucket, compacted into shared memory when
      // it holds at most 64; otherwise the low bits are searched over all keys).
      // `above` = keys whose prefix is larger (the count of the last candidate that
      // failed); `at_or_above` = keys whose prefix is at least the found one (the count
      // of the last candidate that passed).
      uint32_t hi = 0;
      int above = 0, at_or_above = g.NT;
      int hi_bits = kHiBits;
      for (int bit = 31; bit >= 32 - hi_bits; --bit) {
        const uint32_t cand = (hi | (1u << bit));
        int c0 = 0, c1 = 0;
#pragma unroll
        for (int w = 0; w < SLOTS; w += 2) {
          c0 += (key[w] >= cand) ? 1 : 0;
          if (w + 1 < SLOTS) c1 += (key[w + 1] >= cand) ? 1 : 0;
        }
        const int cnt = __reduce_add_sync(0xffffffffu, c0 + c1);
        if (cnt >= k) {
          hi = cand;
          at_or_above = cnt;
        } else {
          above = cnt;
        }
        if (bit == 32 - kHiBits && hi_bits == kHiBits && at_or_above - above > kBucketCap) hi_bits = kHiBitsWide;
      }
      const int lo_bits = 32 - hi_bits;
      hi >>= lo_bits;
      int bsize = 0;
      uint32_t* bucket = bucket_smem + (threadIdx.x >> 5) * kBucketCap;
#pragma unroll
      for (int w = 0; w < SLOTS; ++w) {
        const bool in = key[w] != 0u && (key[w] >> lo_bits) == hi;
        const uint32_t m = __ballot_sync(0xffffffffu, in);
        if (m) {   // warp-uniform; most slots hold no key of the bucket
          const int pos = bsize + __popc(m & lt_mask);
          if (in && pos < kBucketCap) bucket[pos] = key[w];
          bsize += __popc(m);
        }
      }
      __syncwarp();
      const int need_lo = k - above;     // keys to take from the bucket (>= 1)
      uint32_t thr = hi << lo_bits;
      if (bsize <= kBucketCap) {
        const uint32_t b0 = lane < bsize ? bucket[lane] : 0u;
        const uint32_t b1 = lane + 32 < bsize ? bucket[lane + 32] : 0u;
        for (int bit = lo_bits - 1; bit >= 0; --bit) {
          const uint32_t cand = thr | (1u << bit);
          const int cnt = __reduce_add_sync(0xffffffffu, (b0 >= cand ? 1 : 0) + (b1 >= cand ? 1 : 0));
          if (cnt >= need_lo) thr = cand;
        }
      } else {
        for (int bit = lo_bits - 1; bit >= 0; --bit) {
          const uint32_t cand = thr | (1u << bit);
          int cnt = 0;
#pragma unroll
          for (int w = 0; w < SLOTS; ++w) cnt += (key[w] >= cand) ? 1 : 0;
          cnt = __reduce_add_sync(0xffffffffu, cnt);
          if (cnt >= k) thr = cand;
        }
      }
      __syncwarp();
      // keys above the k-th key, and keys equal to it (16-bit fields of one count)
      uint32_t gt_ge = 0;
#pragma unroll
      for (int w = 0; w < SLOTS; ++w) gt_ge += (key[w] > thr ? 1u : 0u) + (key[w] >= thr ? 0x10000u : 0u);
      gt_ge = __reduce_add_sync(0xffffffffu, gt_ge);
      const int gt = (int)(gt_ge & 0xffffu), ge = (int)(gt_ge >> 16);
      const int need = k - gt;
      if (ge == k) {
        // every key equal to the k-th is taken: no tie to break
#pragma unroll
        for (int w = 0; w < SLOTS; ++w) {
          if (w < g.words) {
            const uint32_t word = __ballot_sync(0xffffffffu, key[w] >= thr);
            if ((w & 31) == lane) myword[w >> 5] = word;
          }
        }
      } else {
        int eq_before = 0;
#pragma unroll
        for (int w = 0; w < SLOTS; ++w) {
          if (w < g.words) {
            const bool eq = key[w] == thr;
            const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
            const bool take = key[w] > thr || (eq && eq_before + __popc(eqm & lt_mask) < need);
            const uint32_t word = __ballot_sync(0xffffffffu, take);
            if ((w & 31) == lane) myword[w >> 5] = word;
            eq_before += __popc(eqm);
          }
        }
      }
    }
    // ---- window rows: for each (t, y) tile row of the window, a contiguous x range
    const int cX = i % g.nX, cY = (i / g.nX) % g.nY, cT = i / (g.nX * g.nY);
    int sT, sY, sX, eT, eY, nwX;
    if (g.window_mode == SSTA_WINDOW_TRUNCATE) {
      // [c - w/2, c - w/2 + w) cut at the grid
      const int lT = cT - g.wT / 2, lY = cY - g.wY / 2, lX = cX - g.wX / 2;
      sT = max(lT, 0); eT = min(lT + g.wT, g.nT);
      sY = max(lY, 0); eY = min(lY + g.wY, g.nY);
      sX = max(lX, 0); nwX = min(lX + g.wX, g.nX) - sX;
    } else {
      sT = window_start(cT, g.wT, g.nT); sY = window_start(cY, g.wY, g.nY); sX = window_start(cX, g.wX, g.nX);
      eT = sT + min(g.wT, g.nT); eY = sY + min(g.wY, g.nY); nwX = min(g.wX, g.nX);
    }
#pragma unroll
    for (int q = 0; q < (SLOTS + 31) / 32; ++q) {
      const int word = lane + 32 * q;
      if (word >= g.words) continue;
      uint32_t win = 0u;
      for (int wt = sT; wt < eT; ++wt)
        for (int wy = sY; wy < eY; ++wy) {
          const int lo = (wt * g.nY + wy) * g.nX + sX;
          win |= range_bits(word, lo, lo + nwX);
        }
      myword[q] = g.combine == SSTA_COMBINE_AND ? (myword[q] & win) : (myword[q] | win);
    }
    // ---- compaction: exclusive prefix of the kept counts over words in ascending order
#pragma unroll
    for (int q = 0; q < (SLOTS + 31) / 32; ++q) {
      const int word = lane + 32 * q;
      const uint32_t bits = word < g.words ? myword[q] : 0u;
      int c = __popc(bits);
      int incl = c;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      int pos = base + incl - c;
      uint32_t rest = bits;
      while (rest) {
        const int b = __ffs(rest) - 1;
        rest &= rest - 1u;
        out[pos++] = 32 * word + b;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
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

MaskWorkspace mask_workspace_layout(const Geom& g, bool with_scores) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t bh = (size_t)g.B * g.H;
  MaskWorkspace w{};
  w.status = 0;
  w.qbar = 256;
  w.kbar = w.qbar + up(bh * g.NT * g.D * sizeof(float));
  size_t end = w.kbar + up(bh * g.NT * g.D * sizeof(float));
  if (g.score_mode == SSTA_SCORE_IMPORTANCE) {
    w.inv_nq = end;
    w.inv_nk = w.inv_nq + up(bh * g.NT * sizeof(float));
    w.ksum = w.inv_nk + up(bh * g.NT * sizeof(float));
    end = w.ksum + up(bh * g.norm_blocks * g.D * sizeof(float));
  }
  w.scores = end;
  w.total = end + (with_scores ? up(bh * g.NT * (size_t)g.NT * sizeof(float)) : 0);
  return w;
}

cudaError_t launch_tile_pool(const Geom& g, const void* qp, const void* kp, float* qbar, float* kbar,
                             int32_t* status, const ImportanceBufs& ib, cudaStream_t s) {
  if ((int64_t)g.B * g.H == 0) return cudaSuccess;
  dim3 grid(g.NT, g.B * g.H);
  const int epv = 16 / g.esize;
  const int rpp = kPoolThreads / (g.D / epv);
  const size_t smem = 2 * rpp * g.D * sizeof(float);
  const int4* q4 = static_cast<const int4*>(qp);
  const int4* k4 = static_cast<const int4*>(kp);
  const PoolRowMask rm = make_pool_row_mask(g);
  if (g.dtype == SSTA_BF16)
    return launch_dependent(tile_pool_kernel<__nv_bfloat16>, grid, dim3(kPoolThreads), smem, s, g, rm, q4, k4, qbar,
                            kbar, status, ib);
  return launch_dependent(tile_pool_kernel<float>, grid, dim3(kPoolThreads), smem, s, g, rm, q4, k4, qbar, kbar,
                          status, ib);
}

cudaError_t launch_tile_keysum(const Geom& g, const float* kbar, const ImportanceBufs& ib, cudaStream_t s) {
  if ((int64_t)g.B * g.H == 0) return cudaSuccess;
  return launch_dependent(tile_keysum_kernel, dim3(g.norm_blocks, g.B * g.H), dim3(128), 0, s, g, kbar, ib);
}

cudaError_t launch_tile_scores(const Geom& g, const float* qbar, const float* kbar, const ImportanceBufs& ib,
                               float* scores, int32_t* status, cudaStream_t s) {
  if ((int64_t)g.B * g.H == 0) return cudaSuccess;
  if (ib.ksum == nullptr) return launch_tile_scores_tc(g, qbar, kbar, scores, status, s);
  dim3 grid(ceil_div(g.NT, kScoreBlock), ceil_div(g.NT, kScoreBlock), g.B * g.H);
  if (g.NT % 4 == 0)
    return launch_dependent(tile_scores_kernel<true>, grid, dim3(256), 0, s, g, qbar, kbar, ib, scores);
  return launch_dependent(tile_scores_kernel<false>, grid, dim3(256), 0, s, g, qbar, kbar, ib, scores);
}

cudaError_t launch_select_and_list(const Geom& g, const float* scores, int32_t* kv_idx, int32_t* kv_cnt,
                                   cudaStream_t s) {
  const int64_t rows = (int64_t)g.B * g.H * g.NQ;
  if (rows == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((rows + 7) / 8);
  if (g.words <= 8) return launch_dependent(select_and_list_kernel<8>, dim3(blocks), dim3(256), 0, s, g, scores, kv_idx, kv_cnt);
  if (g.words <= 16) return launch_dependent(select_and_list_kernel<16>, dim3(blocks), dim3(256), 0, s, g, scores, kv_idx, kv_cnt);
  if (g.words <= 32) return launch_dependent(select_and_list_kernel<32>, dim3(blocks), dim3(256), 0, s, g, scores, kv_idx, kv_cnt);
  return launch_dependent(select_and_list_kernel<64>, dim3(blocks), dim3(256), 0, s, g, scores, kv_idx, kv_cnt);
}

}  // namespace ssta
