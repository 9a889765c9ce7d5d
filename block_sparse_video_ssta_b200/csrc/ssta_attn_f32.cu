// Step 4 of SSTA, fp32 storage and arithmetic ("HunyuanVideo 1.5 Technical
// Report", section "SSTA: Selective and Sliding Tile Attention", Step 4 and the
// attention equation softmax(Q K^T / sqrt(d_k)) V restricted to kept tiles).
//
// SIMT kernel for the fp32 workloads: tensor cores have no exact-fp32 mode, so
// this path keeps fp32 end to end.  One warp owns one query row; each lane
// holds four channels of q, the dot product is a warp tree reduction, and the
// softmax is the online (running max / running sum) form with expf.
#include "ssta_internal.h"

namespace ssta {
namespace {

constexpr int kWarps = 4;

__global__ void __launch_bounds__(kWarps * 32)
attention_f32_kernel(Geom g, const float* __restrict__ qp, const float* __restrict__ kp,
                     const float* __restrict__ vp, const int32_t* __restrict__ kv_idx,
                     const int32_t* __restrict__ kv_cnt, float* __restrict__ o,
                     float* __restrict__ lse, int32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int i = blockIdx.x;            // query tile
  const int64_t bh = blockIdx.y;
  const int64_t list_row = bh * g.NQ + i;
  int cnt = kv_cnt[list_row];
  if (cnt < 0 || cnt > g.max_kept) {
    if (threadIdx.x == 0) atomicExch(status, (int)SSTA_ERR_DEVICE_BOUNDS);
    cnt = cnt < 0 ? 0 : g.max_kept;
  }
  const int32_t* list = kv_idx + list_row * g.max_kept;
  const int64_t head = bh * g.Lq;
  const int D = g.D;   // 128: four channels per lane

  for (int r = warp; r < g.N; r += kWarps) {
    const int64_t row = (int64_t)i * g.N + r;
    if (row >= g.Lq) break;
    const float4 q = reinterpret_cast<const float4*>(qp + (head + row) * D)[lane];
    float m = -INFINITY, l = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int e = 0; e < cnt; ++e) {
      const int t = list[e];
      if (t < 0 || t >= g.NQ) {
        if (lane == 0) atomicExch(status, (int)SSTA_ERR_DEVICE_BOUNDS);
        continue;
      }
      int vt = g.tT, vy = g.tY, vx = g.tX, text_valid = g.N;
      if (t < g.NT) {
        const int cX = t % g.nX, cY = (t / g.nX) % g.nY, cT = t / (g.nX * g.nY);
        vt = axis_valid(cT, g.tT, g.T);
        vy = axis_valid(cY, g.tY, g.Y);
        vx = axis_valid(cX, g.tX, g.X);
      } else {
        text_valid = g.L_text - (t - g.NT) * g.N;
      }
      for (int kk = 0; kk < g.N; ++kk) {
        bool valid;
        if (t < g.NT) {
          const int dx = kk % g.tX, dy = (kk / g.tX) % g.tY, dt = kk / (g.tX * g.tY);
          valid = dt < vt && dy < vy && dx < vx;
        } else {
          valid = kk < text_valid;
        }
        if (!valid) continue;
        const int64_t krow = head + (int64_t)t * g.N + kk;
        const float4 k = reinterpret_cast<const float4*>(kp + krow * D)[lane];
        float s = q.x * k.x + q.y * k.y + q.z * k.z + q.w * k.w;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        s *= g.scale;
        const float m_new = fmaxf(m, s);
        const float corr = expf(m - m_new);
        const float p = expf(s - m_new);
        l = l * corr + p;
        const float4 v = reinterpret_cast<const float4*>(vp + krow * D)[lane];
        acc.x = acc.x * corr + p * v.x;
        acc.y = acc.y * corr + p * v.y;
        acc.z = acc.z * corr + p * v.z;
        acc.w = acc.w * corr + p * v.w;
        m = m_new;
      }
    }
    const float inv = l > 0.f ? 1.0f / l : 0.f;
    reinterpret_cast<float4*>(o + (head + row) * D)[lane] =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    if (lane == 0) lse[head + row] = l > 0.f ? m + logf(l) : -INFINITY;
  }
}

}  // namespace

cudaError_t launch_attention_f32(const Geom& g, const float* qp, const float* kp, const float* vp,
                                 const int32_t* kv_idx, const int32_t* kv_cnt, float* o, float* lse,
                                 int32_t* status, cudaStream_t s) {
  if ((int64_t)g.B * g.H == 0) return cudaSuccess;
  dim3 grid(g.NQ, g.B * g.H);
  attention_f32_kernel<<<grid, kWarps * 32, 0, s>>>(g, qp, kp, vp, kv_idx, kv_cnt, o, lse, status);
  return cudaGetLastError();
}

}  // namespace ssta
