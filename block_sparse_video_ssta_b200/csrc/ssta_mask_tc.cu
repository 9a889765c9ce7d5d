// Step 2 of SSTA, Score_s = Qbar Kbar^T per head ("HunyuanVideo 1.5 Technical
// Report", section "SSTA: Selective and Sliding Tile Attention", Step 2), on the
// tensor cores, for the similarity score (the raw dot product of the pooled means).
//
// The pooled means are fp32 and the score is an fp32 quantity (it decides the
// top-k), so each mean x is split into three bf16 parts x = h + m + l (h = bf16(x),
// m = bf16(x - h), l = bf16(x - h - m); each subtraction is exact in fp32 and the
// three parts carry 24 significant bits), and the score is the sum of the six
// products whose parts reach 2^-16 of the leading one:
//   m.m + h.l + l.h + h.m + m.h + h.h
// (the dropped m.l, l.m and l.l are below 2^-24 relative), accumulated in fp32 by
// tcgen05.mma (kind::f16, bf16 inputs, M = N = 128, K = 16 per instruction).
//
// One CTA (256 threads, two per SM) computes the 128 x 128 block of scores of query
// tiles i0..i0+127 and key tiles j0..j0+127 of one head, over the channels in two
// passes of 64:
//   1. every thread reads the fp32 means (channel-major, [head][channel][tile]) of its
//      share of (channel, 8 tiles) groups of both operands for the pass, splits them
//      and stores the three parts into shared memory in the MN-major 128-byte-swizzled
//      operand layout (two 64-tile boxes of 64 channel rows per part);
//   2. one thread issues the pass's 6 x 4 MMAs into one TMEM accumulator (128 columns)
//      and commits to an mbarrier, which every thread waits on before the next pass
//      overwrites the operands;
//   3. each thread loads 64 of its query tile's 128 scores from TMEM and stores them.
// Tiles past NT are zero in shared memory; their scores are not stored.
#include "ssta_tc_common.cuh"

namespace ssta {
namespace {

using namespace wait;
using namespace tc;

constexpr int kScThreads = 256;
constexpr int kScChannels = 64;                        // channels per pass
constexpr uint32_t kScBox = kScChannels * 128;         // one 64-tile box: 64 rows of 128 B
constexpr uint32_t kScPart = 2 * kScBox;               // one bf16 part of one operand (128 tiles)
constexpr uint32_t kScOffB = 3 * kScPart;              // A parts (h, m, l), then B parts
constexpr uint32_t kScOffBar = 6 * kScPart;
constexpr uint32_t kScSmemUsed = kScOffBar + 64;
constexpr uint32_t kScSmemAlloc = kScSmemUsed + 1024;  // slack to align the base to 1024 B
static_assert(2 * kScSmemAlloc <= 228 * 1024, "two CTAs per SM");
constexpr uint64_t kScTimeoutNs = 1500000000ull;
// both operands MN-major (the tile index is contiguous in the channel-major means)
constexpr uint32_t kIdescMNMN = kIdescKMN | (1u << 15);

// MN-major 128-byte-swizzled operand whose two 64-element boxes are kScBox apart (LBO);
// 8-row groups 1024 B apart (SBO).
__device__ __forceinline__ uint64_t desc_mn_sc(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(kScBox >> 4) << 16) | ((uint64_t)(1024 >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ void split3(float x, __nv_bfloat16& h, __nv_bfloat16& m, __nv_bfloat16& l) {
  h = __float2bfloat16_rn(x);
  const float r1 = x - __bfloat162float(h);
  m = __float2bfloat16_rn(r1);
  l = __float2bfloat16_rn(r1 - __bfloat162float(m));
}

__global__ void __launch_bounds__(kScThreads, 2)
tile_scores_tc_kernel(const Geom g, const float* __restrict__ qbar_t, const float* __restrict__ kbar_t,
                      float* __restrict__ scores, int32_t* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t bar = base + kScOffBar;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + kScOffBar + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + kScOffBar + 16);
  __shared__ int32_t local_status;   // stands in when the caller has no status word
  const Ctl ctl{abort_flag, status != nullptr ? status : &local_status, kScTimeoutNs};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NT = g.NT;
  const int i0 = blockIdx.y * 128, j0 = blockIdx.x * 128;
  const int64_t bh = blockIdx.z;
  const bool vec = (NT % 4) == 0;

  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    *abort_flag = 0;
    local_status = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(128u)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }

  // every load of a pass is issued before the first is used: vector loads (predicated, no
  // branch) for groups of 8 tiles inside NT, then scalar loads for a ragged or unaligned
  // group.  Item = (operand, channel, group of 8 tiles): 2 x 64 x 16 items per pass, 8 per
  // thread; consecutive threads take consecutive groups of one channel, so each warp reads
  // two 512-byte channel rows.
  float4 va[8], vb[8];
  auto load_pass = [&](int pass) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int item = (int)threadIdx.x + kScThreads * r;
      const int g8 = item & 15, ch = (item >> 4) & 63, op = item >> 10;
      const int t0 = (op ? j0 : i0) + 8 * g8;
      const float4* src = reinterpret_cast<const float4*>((op ? kbar_t : qbar_t) +
                                                          (bh * g.D + kScChannels * pass + ch) * (int64_t)NT + t0);
      const bool full = vec && t0 + 8 <= NT;
      va[r] = full ? __ldg(src) : make_float4(0.f, 0.f, 0.f, 0.f);
      vb[r] = full ? __ldg(src + 1) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int item = (int)threadIdx.x + kScThreads * r;
      const int g8 = item & 15, ch = (item >> 4) & 63, op = item >> 10;
      const int t0 = (op ? j0 : i0) + 8 * g8;
      if (!(vec && t0 + 8 <= NT) && t0 < NT) {
        const float* src = (op ? kbar_t : qbar_t) + (bh * g.D + kScChannels * pass + ch) * (int64_t)NT + t0;
        float w[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) w[e] = t0 + e < NT ? __ldg(src + e) : 0.f;
        va[r] = make_float4(w[0], w[1], w[2], w[3]);
        vb[r] = make_float4(w[4], w[5], w[6], w[7]);
      }
    }
  };

  bool ok = true;
  int issued = 0;   // passes whose MMAs thread 0 committed
  load_pass(0);
  for (int pass = 0; pass < 2 && ok; ++pass) {
    // ---- 1. split the loaded means of channels 64 pass .. +63 into the operand layout
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int item = (int)threadIdx.x + kScThreads * r;
      const int g8 = item & 15, ch = (item >> 4) & 63, op = item >> 10;
      const float v[8] = {va[r].x, va[r].y, va[r].z, va[r].w, vb[r].x, vb[r].y, vb[r].z, vb[r].w};
      __align__(16) __nv_bfloat16 hp[8], mp[8], lp[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) split3(v[e], hp[e], mp[e], lp[e]);
      // box (tiles 64b..64b+63) of 64 rows x 128 B; row = channel; 16-byte chunk c of the
      // row at position c ^ (row mod 8)
      const uint32_t off = (uint32_t)(g8 >> 3) * kScBox + (uint32_t)ch * 128u + ((uint32_t)((g8 & 7) ^ (ch & 7)) << 4);
      uint8_t* dst = base_ptr + (op ? kScOffB : 0u) + off;
      *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(hp);
      *reinterpret_cast<uint4*>(dst + kScPart) = *reinterpret_cast<const uint4*>(mp);
      *reinterpret_cast<uint4*>(dst + 2 * kScPart) = *reinterpret_cast<const uint4*>(lp);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // visible to the tensor cores
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // ---- 2. the six products, smallest first, into one accumulator
    if (threadIdx.x == 0) {
      const int pa[6] = {1, 0, 2, 0, 1, 0}, pb[6] = {1, 2, 0, 1, 0, 0};   // parts: 0 = h, 1 = m, 2 = l
#pragma unroll
      for (int p = 0; p < 6; ++p) {
        const uint32_t a = base + (uint32_t)pa[p] * kScPart, b = base + kScOffB + (uint32_t)pb[p] * kScPart;
#pragma unroll
        for (int kk = 0; kk < kScChannels / 16; ++kk)
          mma_ss(tmem, desc_mn_sc(a + 2048u * kk), desc_mn_sc(b + 2048u * kk), kIdescMNMN,
                 (pass > 0 || p > 0 || kk > 0) ? 1u : 0u);
      }
      tc_commit(bar);
      ++issued;
    }
    __syncwarp();
    if (pass == 0) load_pass(1);                  // in flight while the tensor cores work
    ok = wait_warp(bar, (uint32_t)pass, ctl);     // the operands are read before they are overwritten
    ok = __syncthreads_and(ok);
    tc_fence_after();
  }
  const uint32_t tmem = *tmem_slot;

  // ---- 3. scores out: warp w holds query tile i0 + 32 (w mod 4) + lane, key tiles
  // j0 + 64 (w / 4) .. +63
  const int i = i0 + (warp & 3) * 32 + lane;
  float* srow = scores + (bh * NT + i) * (int64_t)NT;
  if (ok) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      float v[32];
      const int col = 64 * (warp >> 2) + 32 * q;
      tmem_ld32(tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)col, v);
      if (i < NT) {
        const int jb = j0 + col;
        if (vec && jb + 32 <= NT) {
#pragma unroll
          for (int e = 0; e < 8; ++e)
            reinterpret_cast<float4*>(srow + jb)[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (jb + e < NT) srow[jb + e] = v[e];
        }
      }
    }
  } else if (threadIdx.x == 0 && issued > 0) {
    drain_wait(bar, (uint32_t)(issued - 1), kScTimeoutNs);   // the MMAs retire before TMEM is released
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(*tmem_slot), "r"(128u) : "memory");
  }
}

}  // namespace

cudaError_t launch_tile_scores_tc(const Geom& g, const float* qbar, const float* kbar, float* scores,
                                  int32_t* status, cudaStream_t s) {
  const int64_t BH = (int64_t)g.B * g.H;
  if (BH == 0) return cudaSuccess;
  static std::atomic<bool> attr_set[64];
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(tile_scores_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kScSmemAlloc);
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_release);
  }
  const unsigned nb = (unsigned)((g.NT + 127) / 128);
  tile_scores_tc_kernel<<<dim3(nb, nb, (unsigned)BH), kScThreads, kScSmemAlloc, s>>>(g, qbar, kbar, scores, status);
  return cudaGetLastError();
}

}  // namespace ssta
