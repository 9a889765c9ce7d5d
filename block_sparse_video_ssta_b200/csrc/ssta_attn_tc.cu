// Step 4 of SSTA on the 5th-generation tensor cores of sm_100a: block-sparse
// flash-attention forward ("HunyuanVideo 1.5 Technical Report", section "SSTA:
// Selective and Sliding Tile Attention", Step 4 "Combine Masks and Block-Sparse
// Attention": only the kept key/value tiles of a query tile are loaded, full
// attention inside each kept tile, softmax over the attended keys only).
//
// One CTA owns a band of 256 query rows (two 128-row halves) of one query tile
// of one (batch, head).  It walks that tile's kept-tile list in 128-key chunks.
// Warp roles:
//   warps 0-3  softmax + epilogue for query half 0 (one thread per query row)
//   warps 4-7  softmax + epilogue for query half 1
//   warp  8    TMA producer: Q once, then K and V chunks into 2-stage rings
//   warp  9    TMEM allocator and tcgen05.mma issuer
// Tensor memory (512 columns x 128 lanes x 32 bit):
//   S_h = Q_h K^T  fp32, columns [128h, 128h+128)        (h = query half)
//   P_h = bf16 probabilities packed two per column, written over the first
//         64 columns of S_h and fed to the PV MMA straight from TMEM
//   O_h = sum P V  fp32, columns [256+128h, 256+128h+128)
// MMA schedule per chunk j (the next chunk's S overlaps the softmax of the
// other half):  PV_0(j-1), S_0(j), PV_1(j-1), S_1(j).
// Softmax: one 128-column TMEM load per chunk, base-2 exponentials with the
// scale folded in, running max and sum in fp32 (scale-and-shift and the row sum
// two lanes per instruction with f32x2); the reference max moves only when the
// row max exceeds it by more than 8 (probabilities stay below 2^8), so O is
// rescaled in TMEM rarely.
//
// Every mbarrier wait is bounded in time.  A wait that runs out records
// SSTA_ERR_DEVICE_TIMEOUT in the status word, raises a CTA-wide abort flag that
// all other waits also watch, the producer and MMA warps wait (bounded) for
// their own copies and MMAs in flight, TMEM is freed and the CTA returns.
#include "ssta_internal.h"

#include <atomic>

#include "ssta_tc_common.cuh"
#include "ssta_wait.cuh"

namespace ssta {
namespace {

using namespace wait;
using namespace tc;

constexpr int kThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kStages = 2;
constexpr uint32_t kOffQ = 0;                       // [half][2 boxes]
constexpr uint32_t kOffK = kOffQ + 2 * kTileBytes;  // [stage][2 boxes]
constexpr uint32_t kOffV = kOffK + kStages * kTileBytes;
constexpr uint32_t kOffBar = kOffV + kStages * kTileBytes;
constexpr int kNumBars = 16;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmemUsed = kOffMisc + 64;
constexpr uint32_t kSmemAlloc = kSmemUsed + 1024;  // slack to align the base to 1024 B
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kTimeoutNs = 1500000000ull;      // 1.5 s per wait
constexpr int kMaxDevices = 64;

enum : int {
  BAR_Q = 0, BAR_KFULL = 1, BAR_KEMPTY = 3, BAR_VFULL = 5, BAR_VEMPTY = 7,
  BAR_SFULL = 9, BAR_PREADY = 11, BAR_ODONE = 13, BAR_DRAIN = 15
};

// Instruction descriptors (ssta_tc_common.cuh): S = Q K^T with both operands
// K-major, P V with V (the B operand) MN-major; M = N = 128, bf16 in, fp32 out.
constexpr uint32_t kIdescS = kIdescKK;
constexpr uint32_t kIdescPV = kIdescKMN;

// ------------------------------------------------------------------- kernel
__global__ void __launch_bounds__(kThreads, 1)
ssta_attention_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const Geom g, const __grid_constant__ ChunkTables tb,
                         const int32_t* __restrict__ kv_idx, const int32_t* __restrict__ kv_cnt,
                         __nv_bfloat16* __restrict__ out, float* __restrict__ lse, int32_t* __restrict__ status,
                         float scale_log2) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t sQ = base + kOffQ, sK = base + kOffK, sV = base + kOffV;
  auto bar = [&](int i) { return base + kOffBar + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + kOffMisc + 8);
  const Ctl ctl{abort_flag, status, kTimeoutNs};

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work unit: text query tiles first (longest lists), then video tiles head-major
  const int bands = (g.N + 255) / 256;
  const int64_t BH = (int64_t)g.B * g.H;
  const int64_t text_units = BH * g.n_text * bands;
  int64_t u = blockIdx.x;
  int64_t bh;
  int qt, band;
  if (u < text_units) {
    bh = u / ((int64_t)g.n_text * bands);
    const int rem = (int)(u - bh * g.n_text * bands);
    qt = g.NT + rem / bands;
    band = rem % bands;
  } else {
    u -= text_units;
    bh = u / ((int64_t)g.NT * bands);
    const int rem = (int)(u - bh * g.NT * bands);
    qt = rem / bands;
    band = rem % bands;
  }
  const int halves_left = g.N / 128 - 2 * band;
  const int nh = halves_left < 2 ? halves_left : 2;
  const int qrow0 = qt * g.N + band * 256;              // first packed row of this band
  const int64_t tile_end = (int64_t)qt * g.N + g.N < g.Lq ? (int64_t)qt * g.N + g.N : g.Lq;
  const int64_t list_row = bh * g.NQ + qt;
  int cnt = __ldg(kv_cnt + list_row);
  if (cnt < 0 || cnt > g.max_kept) {
    if (threadIdx.x == 0) atomicExch(status, (int)SSTA_ERR_DEVICE_BOUNDS);
    cnt = cnt < 0 ? 0 : g.max_kept;
  }
  const int32_t* list = kv_idx + list_row * g.max_kept;

  // ---- setup: barriers, abort flag, TMEM
  if (threadIdx.x == 0) {
    mbar_init(bar(BAR_Q), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(BAR_KFULL + s), 1);
      mbar_init(bar(BAR_KEMPTY + s), 1);
      mbar_init(bar(BAR_VFULL + s), 1);
      mbar_init(bar(BAR_VEMPTY + s), 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(bar(BAR_SFULL + h), 1);
      mbar_init(bar(BAR_PREADY + h), 128);
      mbar_init(bar(BAR_ODONE + h), 1);
    }
    mbar_init(bar(BAR_DRAIN), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (int e = 0; e < cnt; ++e) {
      const int t = __ldg(list + e);
      if (t < 0 || t >= g.NQ) { atomicExch(status, (int)SSTA_ERR_DEVICE_BOUNDS); break; }
    }
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS[2] = {tmem, tmem + 128};
  const uint32_t tO[2] = {tmem + 256, tmem + 384};

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmQ)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmK)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmV)) : "memory");
      const int z = (int)bh;
      mbar_expect_tx(bar(BAR_Q), nh * kTileBytes);
      for (int h = 0; h < nh; ++h)
        for (int b = 0; b < 2; ++b)
          tma_load_3d(sQ + h * kTileBytes + b * kBox, &tmQ, b * 64, qrow0 + h * 128, z, bar(BAR_Q));
      int nK[kStages] = {0, 0}, nV[kStages] = {0, 0};   // copies issued per stage
      const int n = for_each_chunk(g, tb, list, cnt, [&](int j, int t, int ch, bool) -> bool {
        const int s = j & 1;
        const uint32_t ph = (uint32_t)((j >> 1) & 1);
        const int krow = t * g.N + ch * kChunk;
        if (!wait_bounded(bar(BAR_KEMPTY + s), ph ^ 1u, ctl)) return false;
        mbar_expect_tx(bar(BAR_KFULL + s), kTileBytes);
        tma_load_3d(sK + s * kTileBytes, &tmK, 0, krow, z, bar(BAR_KFULL + s));
        tma_load_3d(sK + s * kTileBytes + kBox, &tmK, 64, krow, z, bar(BAR_KFULL + s));
        ++nK[s];
        if (!wait_bounded(bar(BAR_VEMPTY + s), ph ^ 1u, ctl)) return false;
        mbar_expect_tx(bar(BAR_VFULL + s), kTileBytes);
        tma_load_3d(sV + s * kTileBytes, &tmV, 0, krow, z, bar(BAR_VFULL + s));
        tma_load_3d(sV + s * kTileBytes + kBox, &tmV, 64, krow, z, bar(BAR_VFULL + s));
        ++nV[s];
        return true;
      });
      if (n < 0) {
        // abort: let every copy this thread started land before shared memory is released
        drain_wait(bar(BAR_Q), 0, kTimeoutNs);
        for (int s = 0; s < kStages; ++s) {
          if (nK[s] > 0) drain_wait(bar(BAR_KFULL + s), (uint32_t)((nK[s] - 1) & 1), kTimeoutNs);
          if (nV[s] > 0) drain_wait(bar(BAR_VFULL + s), (uint32_t)((nV[s] - 1) & 1), kTimeoutNs);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = wait_bounded(bar(BAR_Q), 0, ctl);
      int prev = 0;
      auto issue_S = [&](int h, int s) {
        const uint32_t qa = sQ + h * kTileBytes, kb = sK + s * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (uint32_t)(kk >> 2) * kBox + (uint32_t)(kk & 3) * 32u;
          mma_ss(tS[h], desc_kmajor(qa + off), desc_kmajor(kb + off), kIdescS, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_PV = [&](int h, int s, bool first) {
        const uint32_t vb = sV + s * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tO[h], tS[h] + 8u * kk, desc_mnmajor(vb + 2048u * kk), kIdescPV, (!first || kk > 0) ? 1u : 0u);
      };
      int n = -1;
      if (ok) {
        n = for_each_chunk(g, tb, list, cnt, [&](int j, int, int, bool) -> bool {
          const int s = j & 1;
          const uint32_t ph = (uint32_t)((j >> 1) & 1);
          if (j == 0) {
            if (!wait_bounded(bar(BAR_KFULL + s), ph, ctl)) return false;
            tc_fence_after();
            for (int h = 0; h < nh; ++h) {
              issue_S(h, s);
              tc_commit(bar(BAR_SFULL + h));
            }
          } else {
            if (!wait_bounded(bar(BAR_VFULL + prev), (uint32_t)(((j - 1) >> 1) & 1), ctl)) return false;
            for (int h = 0; h < nh; ++h) {
              if (!wait_bounded(bar(BAR_PREADY + h), (uint32_t)((j - 1) & 1), ctl)) return false;
              tc_fence_after();
              issue_PV(h, prev, j == 1);
              tc_commit(bar(BAR_ODONE + h));
              if (h == 0) {
                if (!wait_bounded(bar(BAR_KFULL + s), ph, ctl)) return false;
                tc_fence_after();
              }
              issue_S(h, s);
              tc_commit(bar(BAR_SFULL + h));
            }
            tc_commit(bar(BAR_VEMPTY + prev));
          }
          tc_commit(bar(BAR_KEMPTY + s));
          prev = s;
          return true;
        });
      }
      if (n > 0) {
        const int j = n;   // PV of the last chunk
        if (wait_bounded(bar(BAR_VFULL + prev), (uint32_t)(((j - 1) >> 1) & 1), ctl)) {
          for (int h = 0; h < nh; ++h) {
            if (!wait_bounded(bar(BAR_PREADY + h), (uint32_t)((j - 1) & 1), ctl)) break;
            tc_fence_after();
            issue_PV(h, prev, j == 1);
            tc_commit(bar(BAR_ODONE + h));
          }
          tc_commit(bar(BAR_VEMPTY + prev));
        }
      }
      // every MMA (and its commit arrivals) retires before TMEM and smem are released
      tc_commit(bar(BAR_DRAIN));
      drain_wait(bar(BAR_DRAIN), 0, kTimeoutNs);
    }
  } else if (warp < 4 * nh) {
    // ------------------------------------------------------ softmax + epilogue
    const int h = warp >> 2;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tSh = tS[h] + lane_off, tOh = tO[h] + lane_off;
    float m = -INFINITY;   // running max of the scaled scores, base-2 units
    float l = 0.f;         // running sum of exponentials
    const int n = for_each_chunk(g, tb, list, cnt, [&](int j, int t, int ch, bool full) -> bool {
      if (!wait_warp(bar(BAR_SFULL + h), (uint32_t)(j & 1), ctl)) return false;
      tc_fence_after();
      float sv[128];
      tmem_ld128(tSh, sv);
      if (!full) {
        // pad keys of this chunk (same columns for every row) never enter the softmax
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t vm = chunk_vmask(g, tb, t, ch, q);
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (!((vm >> i) & 1u)) sv[q * 32 + i] = -INFINITY;
        }
      }
      float mx[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx[i] = fmaxf(sv[i], sv[i + 8]);
#pragma unroll
      for (int i = 16; i < 128; i += 16)
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = max3(mx[k], sv[i + k], sv[i + 8 + k]);
      const float rmax = max3(max3(mx[0], mx[1], mx[2]), max3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) *
                         scale_log2;
      // Lazy rescaling: the reference max only moves when the row max exceeds it by more
      // than 8 (base 2), so probabilities stay below 2^8 and O is rescaled rarely.
      const bool moved = rmax > m + 8.0f;
      const float m_new = moved ? rmax : m;
      const float alpha = moved ? ex2(m - m_new) : 1.0f;
      m = m_new;
      const float neg_m = -m_new;
      // scale-and-shift and the row sum run two lanes per instruction (f32x2)
      const uint64_t c2 = f2_pack(scale_log2, scale_log2), nm2 = f2_pack(neg_m, neg_m);
      uint64_t sum2[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) sum2[i] = f2_pack(0.f, 0.f);
      uint32_t pk[64];
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        float x0, x1;
        f2_unpack(f2_fma(f2_pack(sv[2 * i], sv[2 * i + 1]), c2, nm2), x0, x1);
        const float p0 = ex2(x0), p1 = ex2(x1);
        sum2[i & 3] = f2_add(sum2[i & 3], f2_pack(p0, p1));
        pk[i] = pack_bf16x2(p0, p1);
      }
      float sum[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) f2_unpack(sum2[i], sum[2 * i], sum[2 * i + 1]);
      tmem_st64(tSh, pk);
      tmem_wait_st();
      l = l * alpha + (((sum[0] + sum[1]) + (sum[2] + sum[3])) + ((sum[4] + sum[5]) + (sum[6] + sum[7])));
      if (j > 0 && __any_sync(0xffffffffu, moved)) {
        if (!wait_warp(bar(BAR_ODONE + h), (uint32_t)((j - 1) & 1), ctl)) return false;
        tc_fence_after();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float v[32];
          tmem_ld32(tOh + 32u * q, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= alpha;
          tmem_st32(tOh + 32u * q, v);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(bar(BAR_PREADY + h));
      return true;
    });
    // epilogue: O / l in bf16, LSE in natural log
    bool have = n > 0;
    if (have) {
      have = wait_warp(bar(BAR_ODONE + h), (uint32_t)((n - 1) & 1), ctl);
      tc_fence_after();
    }
    const int64_t row = (int64_t)qrow0 + h * 128 + (warp & 3) * 32 + lane;
    const bool write = row < tile_end && !*abort_flag;
    const float inv = l > 0.f ? 1.0f / l : 0.f;
    __nv_bfloat16* orow = out + (bh * g.Lq + row) * 128;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float v[32];
      if (have) {
        tmem_ld32(tOh + 32u * q, v);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
      }
      if (write) {
        uint4* dst = reinterpret_cast<uint4*>(orow + 32 * q);
#pragma unroll
        for (int w4 = 0; w4 < 4; ++w4) {
          uint4 pk;
          pk.x = pack_bf16x2(v[8 * w4 + 0] * inv, v[8 * w4 + 1] * inv);
          pk.y = pack_bf16x2(v[8 * w4 + 2] * inv, v[8 * w4 + 3] * inv);
          pk.z = pack_bf16x2(v[8 * w4 + 4] * inv, v[8 * w4 + 5] * inv);
          pk.w = pack_bf16x2(v[8 * w4 + 6] * inv, v[8 * w4 + 7] * inv);
          dst[w4] = pk;
        }
      }
    }
    if (write) lse[bh * g.Lq + row] = l > 0.f ? m * 0.69314718055994531f + logf(l) : -INFINITY;
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

}  // namespace

cudaError_t launch_attention_bf16_tc(const Geom& g, const void* qp, const void* kp, const void* vp,
                                     const int32_t* kv_idx, const int32_t* kv_cnt, void* o, float* lse,
                                     int32_t* status, cudaStream_t s) {
  const int64_t BH = (int64_t)g.B * g.H;
  if (BH == 0) return cudaSuccess;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, qp, g) || !make_map(&mk, kp, g) || !make_map(&mv, vp, g)) return cudaErrorInvalidValue;
  // the shared-memory opt-in is a per-device attribute of the kernel: set it once per device
  static std::atomic<bool> attr_set[kMaxDevices];
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(ssta_attention_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemAlloc);
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_release);
  }
  const int bands = (g.N + 255) / 256;
  const int64_t units = BH * (int64_t)g.NQ * bands;
  const float scale_log2 = g.scale * 1.4426950408889634f;
  ssta_attention_tc_kernel<<<(unsigned)units, kThreads, kSmemAlloc, s>>>(
      mq, mk, mv, g, make_chunk_tables(g), kv_idx, kv_cnt, static_cast<__nv_bfloat16*>(o), lse, status,
      scale_log2);
  return cudaGetLastError();
}

}  // namespace ssta
