// Backward of Step 4 on the tensor cores, dQ part ("HunyuanVideo 1.5 Technical
// Report", section "SSTA: Selective and Sliding Tile Attention", Step 4; the
// attention equation softmax(Q K^T / sqrt(d_k)) V over the kept tiles):
//   dQ = scale * dS K,  dS = P * (dO V^T - D),  P = exp(Q K^T * scale - LSE),
// with LSE from the forward and D = rowsum(dO * O).
//
// One CTA owns 128 query rows of one query tile and walks the tile's kept list
// in 128-key chunks.  Warp roles:
//   warps 0-7  elementwise: warp w serves query rows 32 (w mod 4) .. +31 and key
//              columns 64 (w / 4) .. +63 of each chunk: P and dS from S and dP in
//              tensor memory, dS (bf16) back into tensor memory; epilogue dQ * scale
//   warp  8    TMA producer: Q and dO once, then K (3-stage ring: K(j) is read by
//              S(j) and, a chunk later, by dQ) and V (2-stage ring) chunks
//   warp  9    TMEM allocator and tcgen05.mma issuer
// Tensor memory: S (fp32, 128 columns), dP (128), dQ accumulator (128), dS (bf16
// pairs: key columns 64h .. 64h+63 packed in columns 64h .. 64h+31 of the last 128).
// Shared memory: Q, dO and the K and V rings (128-byte swizzle).
// Per chunk j the MMA warp issues S(j) = Q K(j)^T and dP(j) = dO V(j)^T as soon
// as the elementwise warps have loaded S(j-1) and dP(j-1) into registers, then
// dQ += dS(j-1) K(j-1) (A = dS from tensor memory, B = K read MN-major) once
// dS(j-1) is written: the next chunk's S and dP run during this chunk's
// exponentials.  dS is overwritten only after the previous dQ product finished.
// Every wait is bounded (ssta_wait.cuh), as in the forward kernel.
#include "ssta_tc_common.cuh"

#include <algorithm>

namespace ssta {
namespace {

using namespace wait;
using namespace tc;

constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kTimeoutNs = 1500000000ull;

// dQ kernel: 8 elementwise warps (two per TMEM lane group, 64 key columns each),
// the producer and the MMA issuer.
constexpr int kDqThreads = 320;
constexpr int kDqProducerWarp = 8;
constexpr int kDqMmaWarp = 9;
constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffDO = kOffQ + kTileBytes;
constexpr uint32_t kOffK = kOffDO + kTileBytes;
constexpr uint32_t kOffV = kOffK + kKStages * kTileBytes;
constexpr uint32_t kOffBar = kOffV + kVStages * kTileBytes;
constexpr int kNumBars = 16;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmemAlloc = kOffMisc + 64 + 1024;
static_assert(kSmemAlloc <= 227 * 1024, "shared memory");

enum : int {
  BAR_Q = 0, BAR_KFULL = 1, BAR_KEMPTY = 4, BAR_VFULL = 7, BAR_VEMPTY = 9,
  BAR_SFULL = 11, BAR_SFREE = 12, BAR_DSREADY = 13, BAR_DQDONE = 14, BAR_DRAIN = 15
};

// dS and P^T are written back in bf16 pairs over (or, for dS in the dQ kernel, beside)
// fp32 columns each warp read: key (or query) columns 64h .. 64h+63 are packed in
// tensor-memory columns 64h .. 64h+31 of the region, so the two warps of a lane group
// never write columns the other one reads.  Column of the bf16 A operand for the 16
// columns 16 kk .. 16 kk + 15:
__device__ __forceinline__ uint32_t pcol(int kk) { return 8u * (uint32_t)kk + ((uint32_t)(kk >> 2) << 5); }

__global__ void __launch_bounds__(kDqThreads, 1)
bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO, const Geom g,
                 const __grid_constant__ ChunkTables tb, const int32_t* __restrict__ kv_idx, const int32_t* __restrict__ kv_cnt,
                 const float* __restrict__ lse, const float* __restrict__ Dv, __nv_bfloat16* __restrict__ dq,
                 int32_t* __restrict__ status, float scale_log2) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t sQ = base + kOffQ, sDO = base + kOffDO, sK = base + kOffK, sV = base + kOffV;
  auto bar = [&](int i) { return base + kOffBar + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + kOffMisc + 8);
  const Ctl ctl{abort_flag, status, kTimeoutNs};
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work unit: one 128-row block of a query tile; text query tiles first
  const int blocks = g.N / 128;
  const int64_t BH = (int64_t)g.B * g.H;
  const int64_t text_units = BH * g.n_text * blocks;
  int64_t u = blockIdx.x;
  int64_t bh;
  int qt, blk;
  if (u < text_units) {
    bh = u / ((int64_t)g.n_text * blocks);
    const int rem = (int)(u - bh * g.n_text * blocks);
    qt = g.NT + rem / blocks;
    blk = rem % blocks;
  } else {
    u -= text_units;
    bh = u / ((int64_t)g.NT * blocks);
    const int rem = (int)(u - bh * g.NT * blocks);
    qt = rem / blocks;
    blk = rem % blocks;
  }
  const int qrow0 = qt * g.N + blk * 128;
  const int64_t list_row = bh * g.NQ + qt;
  int cnt = __ldg(kv_cnt + list_row);
  if (cnt < 0 || cnt > g.max_kept) {
    if (threadIdx.x == 0) atomicExch(status, (int)SSTA_ERR_DEVICE_BOUNDS);
    cnt = cnt < 0 ? 0 : g.max_kept;
  }
  const int32_t* list = kv_idx + list_row * g.max_kept;

  if (threadIdx.x == 0) {
    mbar_init(bar(BAR_Q), 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(bar(BAR_KFULL + s), 1);
      mbar_init(bar(BAR_KEMPTY + s), 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(bar(BAR_VFULL + s), 1);
      mbar_init(bar(BAR_VEMPTY + s), 1);
    }
    mbar_init(bar(BAR_SFULL), 1);
    mbar_init(bar(BAR_SFREE), 256);
    mbar_init(bar(BAR_DSREADY), 256);
    mbar_init(bar(BAR_DQDONE), 1);
    mbar_init(bar(BAR_DRAIN), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (int e = 0; e < cnt; ++e) {
      const int t = __ldg(list + e);
      if (t < 0 || t >= g.NQ) { atomicExch(status, (int)SSTA_ERR_DEVICE_BOUNDS); break; }
    }
  }
  if (warp == kDqMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tP = tmem + 128, tDQ = tmem + 256, tDS = tmem + 384;

  if (warp == kDqProducerWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const int z = (int)bh;
      mbar_expect_tx(bar(BAR_Q), 2 * kTileBytes);
      for (int b = 0; b < 2; ++b) {
        tma_load_3d(sQ + b * kBox, &tmQ, b * 64, qrow0, z, bar(BAR_Q));
        tma_load_3d(sDO + b * kBox, &tmDO, b * 64, qrow0, z, bar(BAR_Q));
      }
      int nK[kKStages] = {0, 0, 0}, nV[kVStages] = {0, 0};
      const int n = for_each_chunk(g, tb, list, cnt, [&](int j, int t, int ch, bool) -> bool {
        const int ks = j % kKStages, vs = j & 1;
        const int krow = t * g.N + ch * kChunk;
        if (!wait_bounded(bar(BAR_KEMPTY + ks), (uint32_t)(((j / kKStages) & 1) ^ 1), ctl)) return false;
        mbar_expect_tx(bar(BAR_KFULL + ks), kTileBytes);
        tma_load_3d(sK + ks * kTileBytes, &tmK, 0, krow, z, bar(BAR_KFULL + ks));
        tma_load_3d(sK + ks * kTileBytes + kBox, &tmK, 64, krow, z, bar(BAR_KFULL + ks));
        ++nK[ks];
        if (!wait_bounded(bar(BAR_VEMPTY + vs), (uint32_t)(((j >> 1) & 1) ^ 1), ctl)) return false;
        mbar_expect_tx(bar(BAR_VFULL + vs), kTileBytes);
        tma_load_3d(sV + vs * kTileBytes, &tmV, 0, krow, z, bar(BAR_VFULL + vs));
        tma_load_3d(sV + vs * kTileBytes + kBox, &tmV, 64, krow, z, bar(BAR_VFULL + vs));
        ++nV[vs];
        return true;
      });
      if (n < 0) {
        drain_wait(bar(BAR_Q), 0, kTimeoutNs);
        for (int s = 0; s < kKStages; ++s)
          if (nK[s] > 0) drain_wait(bar(BAR_KFULL + s), (uint32_t)((nK[s] - 1) & 1), kTimeoutNs);
        for (int s = 0; s < kVStages; ++s)
          if (nV[s] > 0) drain_wait(bar(BAR_VFULL + s), (uint32_t)((nV[s] - 1) & 1), kTimeoutNs);
      }
    }
  } else if (warp == kDqMmaWarp) {
    // ------------------------------------------------------------- MMA issuer
    // Per chunk j: S(j) = Q K(j)^T and dP(j) = dO V(j)^T as soon as the elementwise
    // warps have loaded S(j-1) and dP(j-1), then dQ += dS(j-1) K(j-1) once dS(j-1) is
    // in shared memory, so S and dP of the next chunk run during this chunk's exponentials.
    if (lane == 0) {
      const bool ok = wait_bounded(bar(BAR_Q), 0, ctl);
      // dQ += dS(jp) K(jp): A = dS in tensor memory, B = K stage read MN-major
      auto dq_step = [&](int jp) -> bool {
        if (!wait_bounded(bar(BAR_DSREADY), (uint32_t)(jp & 1), ctl)) return false;
        tc_fence_after();
        const uint32_t kb = sK + (jp % kKStages) * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tDQ, tDS + pcol(kk), desc_mnmajor(kb + 2048u * kk), kIdescKMN, (jp > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bar(BAR_DQDONE));
        tc_commit(bar(BAR_KEMPTY + jp % kKStages));
        return true;
      };
      int n = -1;
      if (ok) {
        n = for_each_chunk(g, tb, list, cnt, [&](int j, int, int, bool) -> bool {
          const int ks = j % kKStages, vs = j & 1;
          if (j > 0) {
            if (!wait_bounded(bar(BAR_SFREE), (uint32_t)((j - 1) & 1), ctl)) return false;
            tc_fence_after();
          }
          if (!wait_bounded(bar(BAR_KFULL + ks), (uint32_t)((j / kKStages) & 1), ctl)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (uint32_t)(kk >> 2) * kBox + (uint32_t)(kk & 3) * 32u;
            mma_ss(tS, desc_kmajor(sQ + off), desc_kmajor(sK + ks * kTileBytes + off), kIdescKK, kk > 0 ? 1u : 0u);
          }
          if (!wait_bounded(bar(BAR_VFULL + vs), (uint32_t)((j >> 1) & 1), ctl)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (uint32_t)(kk >> 2) * kBox + (uint32_t)(kk & 3) * 32u;
            mma_ss(tP, desc_kmajor(sDO + off), desc_kmajor(sV + vs * kTileBytes + off), kIdescKK, kk > 0 ? 1u : 0u);
          }
          tc_commit(bar(BAR_SFULL));
          tc_commit(bar(BAR_VEMPTY + vs));
          return j == 0 ? true : dq_step(j - 1);
        });
      }
      if (n > 0) dq_step(n - 1);
      tc_commit(bar(BAR_DRAIN));
      drain_wait(bar(BAR_DRAIN), 0, kTimeoutNs);
    }
  } else {
    // ------------------------------------------------ P, dS and the epilogue
    // warp w: TMEM lanes 32 (w mod 4) .. +31 (its query rows), key columns 64 (w / 4) .. +63
    const int grp = warp & 3, half = warp >> 2;
    const uint32_t lane_off = (uint32_t)(grp * 32) << 16;
    const int r = grp * 32 + lane;   // row within the block
    const int64_t row = (int64_t)qrow0 + r;
    const int qoff = (int)(row - (int64_t)qt * g.N);
    const bool row_ok = row < g.Lq && key_valid(g, tb, qt, qoff);
    const float L2 = row_ok ? __ldg(lse + bh * g.Lq + row) * 1.4426950408889634f : 0.f;
    const bool live = row_ok && L2 > -INFINITY;
    const float Dr = live ? __ldg(Dv + bh * g.Lq + row) : 0.f;
    // per-row constants as f32x2 pairs: the scale, -LSE (log2 units; -inf for a row that takes
    // no part, whose P is then exactly 0) and -D
    const uint64_t c2 = f2_pack(scale_log2, scale_log2);
    const float nl = live ? -L2 : -INFINITY;
    const uint64_t nl2 = f2_pack(nl, nl), nd2 = f2_pack(-Dr, -Dr);
    const int n = for_each_chunk(g, tb, list, cnt, [&](int j, int t, int ch, bool full) -> bool {
      if (!wait_warp(bar(BAR_SFULL), (uint32_t)(j & 1), ctl)) return false;
      tc_fence_after();
      float sv[64], dpv[64];
      tmem_ld64(tS + lane_off + 64u * half, sv);
      tmem_ld64(tP + lane_off + 64u * half, dpv);
      tc_fence_before();
      mbar_arrive(bar(BAR_SFREE));   // S and dP of this chunk are in registers
      if (!full) {
        // pad keys of this chunk (same columns for every row): S = -inf, so P = 0
#pragma unroll
        for (int w2 = 0; w2 < 2; ++w2) {
          const uint32_t vm = chunk_vmask(g, tb, t, ch, 2 * half + w2);
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (!((vm >> i) & 1u)) sv[32 * w2 + i] = -INFINITY;
        }
      }
      // P = 2^(s * scale - LSE), dS = P (dP - D), two key columns per f32x2 instruction
      uint32_t pk[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        float x0, x1, ds0, ds1;
        f2_unpack(f2_fma(f2_pack(sv[2 * i], sv[2 * i + 1]), c2, nl2), x0, x1);
        const float p0 = ex2(x0), p1 = ex2(x1);
        f2_unpack(f2_mul(f2_pack(p0, p1), f2_add(f2_pack(dpv[2 * i], dpv[2 * i + 1]), nd2)), ds0, ds1);
        pk[i] = pack_bf16x2(ds0, ds1);
      }
      // dQ(j-1) reads dS from tensor memory: it must have finished before dS is overwritten
      if (j > 0 && !wait_warp(bar(BAR_DQDONE), (uint32_t)((j - 1) & 1), ctl)) return false;
      tc_fence_after();
      tmem_st32u(tDS + lane_off + 64u * half, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(BAR_DSREADY));
      return true;
    });
    // epilogue: dQ * scale in bf16 (pad rows and rows without keys write zeros); warp w
    // writes channels 64 (w / 4) .. +63 of its rows
    bool have = n > 0;
    if (have) have = wait_warp(bar(BAR_DQDONE), (uint32_t)((n - 1) & 1), ctl);
    tc_fence_after();
    const bool write = row < g.Lq && !*abort_flag;
    const float sc = scale_log2 * 0.69314718055994531f;   // the softmax scale
    __nv_bfloat16* orow = dq + (bh * g.Lq + row) * 128 + 64 * half;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      float v[32];
      if (have) {
        tmem_ld32(tDQ + lane_off + 64u * half + 32u * q, v);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
      }
      if (write) {
        uint4* dst = reinterpret_cast<uint4*>(orow + 32 * q);
#pragma unroll
        for (int w4 = 0; w4 < 4; ++w4) {
          const float m = row_ok ? sc : 0.f;
          uint4 pkv;
          pkv.x = pack_bf16x2(v[8 * w4 + 0] * m, v[8 * w4 + 1] * m);
          pkv.y = pack_bf16x2(v[8 * w4 + 2] * m, v[8 * w4 + 3] * m);
          pkv.z = pack_bf16x2(v[8 * w4 + 4] * m, v[8 * w4 + 5] * m);
          pkv.w = pack_bf16x2(v[8 * w4 + 6] * m, v[8 * w4 + 7] * m);
          dst[w4] = pkv;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kDqMmaWarp) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

}  // namespace

namespace {

// Row statistics for the tensor-core kernels, per packed row of whole tiles:
// D = rowsum(dO * O) (rows < Lq), and the values the dK/dV kernel adds,
// -LSE * log2(e) and -D (-inf and 0 for pad rows and rows without a kept key).
// 16 lanes per row (16-byte loads of 8 bf16 channels), 8 rows per warp with every
// load issued before the first sum; row validity from the tile tables, so no lane
// divides by the grid extents; grid.y is the head.
constexpr int kRsWarps = 8;
constexpr int kRsRows = 8;   // rows per warp

__global__ void __launch_bounds__(kRsWarps * 32)
bwd_rowstat_tc_kernel(const Geom g, const __grid_constant__ ChunkTables tb, int64_t bh0,
                      const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dO,
                      const float* __restrict__ lse, float* __restrict__ Dv, float* __restrict__ nl2,
                      float* __restrict__ nd) {
  const int lane = threadIdx.x & 31, sub = lane >> 4, part = lane & 15;
  const int64_t bh = bh0 + blockIdx.y;
  const int64_t Lp = (int64_t)g.NQ * g.N;
  const int64_t r0 = ((int64_t)blockIdx.x * kRsWarps + (threadIdx.x >> 5)) * kRsRows;
  int4 va[kRsRows / 2], vb[kRsRows / 2];
  bool valid[kRsRows / 2];
#pragma unroll
  for (int it = 0; it < kRsRows / 2; ++it) {
    const int64_t row = r0 + 2 * it + sub;
    bool ok = row < g.Lq;   // rows past Lq exist only in the last text tile
    if (ok) {
      const int t = (int)(row / g.N);
      ok = key_valid(g, tb, t, (int)(row - (int64_t)t * g.N));
    }
    valid[it] = ok;
    const int64_t wq = bh * g.Lq + row;
    va[it] = ok ? reinterpret_cast<const int4*>(o + wq * 128)[part] : make_int4(0, 0, 0, 0);
    vb[it] = ok ? reinterpret_cast<const int4*>(dO + wq * 128)[part] : make_int4(0, 0, 0, 0);
  }
#pragma unroll
  for (int it = 0; it < kRsRows / 2; ++it) {
    const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(&va[it]);
    const __nv_bfloat162* y = reinterpret_cast<const __nv_bfloat162*>(&vb[it]);
    float d = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 u = __bfloat1622float2(x[i]), v = __bfloat1622float2(y[i]);
      d = fmaf(u.x, v.x, d);
      d = fmaf(u.y, v.y, d);
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
    const int64_t row = r0 + 2 * it + sub;
    if (part == 0 && row < Lp) {
      const int64_t wq = bh * g.Lq + row;
      if (row < g.Lq) Dv[wq] = d;
      const float L = valid[it] ? lse[wq] : -INFINITY;
      nl2[bh * Lp + row] = L > -INFINITY ? -(L * 1.4426950408889634f) : -INFINITY;
      nd[bh * Lp + row] = L > -INFINITY ? -d : 0.f;
    }
  }
}

}  // namespace

cudaError_t launch_attention_bwd_rowstat_tc(const Geom& g, const void* o, const void* dO, const float* lse, float* Dv,
                                            float* nl2, float* nd, cudaStream_t s) {
  const int64_t BH = (int64_t)g.B * g.H;
  const int64_t Lp = (int64_t)g.NQ * g.N, rows_per_block = (int64_t)kRsWarps * kRsRows;
  const ChunkTables tb = make_chunk_tables(g);
  for (int64_t bh0 = 0; bh0 < BH; bh0 += 65535) {   // grid.y holds at most 65535 heads
    const dim3 grid((unsigned)((Lp + rows_per_block - 1) / rows_per_block), (unsigned)std::min<int64_t>(BH - bh0, 65535));
    bwd_rowstat_tc_kernel<<<grid, kRsWarps * 32, 0, s>>>(g, tb, bh0, static_cast<const __nv_bfloat16*>(o),
                                                         static_cast<const __nv_bfloat16*>(dO), lse, Dv, nl2, nd);
  }
  return cudaGetLastError();
}

cudaError_t launch_attention_bwd_dq_tc(const Geom& g, const void* q, const void* k, const void* v, const void* dO,
                                       const float* lse, const float* Dv, const int32_t* kv_idx,
                                       const int32_t* kv_cnt, void* dq, int32_t* status, cudaStream_t s) {
  const int64_t BH = (int64_t)g.B * g.H;
  if (BH == 0) return cudaSuccess;
  CUtensorMap mq, mk, mv, mdo;
  if (!make_map(&mq, q, g) || !make_map(&mk, k, g) || !make_map(&mv, v, g) || !make_map(&mdo, dO, g))
    return cudaErrorInvalidValue;
  static std::atomic<bool> attr_set[64];
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemAlloc);
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_release);
  }
  const int64_t units = BH * (int64_t)g.NQ * (g.N / 128);
  bwd_dq_tc_kernel<<<(unsigned)units, kDqThreads, kSmemAlloc, s>>>(mq, mk, mv, mdo, g, make_chunk_tables(g), kv_idx,
                                                                   kv_cnt, lse, Dv, static_cast<__nv_bfloat16*>(dq),
                                                                   status, g.scale * 1.4426950408889634f);
  return cudaGetLastError();
}

// ============================================================================
// dK and dV on the tensor cores:  dV = P^T dO,  dK = scale * dS^T Q, for one
// 128-key block, summed over the 128-row query chunks of every query tile that
// keeps the block's tile (the transposed kept lists).  Warp roles:
//   warps 0-7  elementwise: warp w serves key rows 32 (w mod 4) .. +31 and query
//              columns 64 (w / 4) .. +63 of each step, in two phases: P^T from
//              S^T (bf16, written over the S^T columns the warp read), then dS^T
//              from dP^T and P (bf16, likewise over dP^T); the per-query -LSE
//              (log2 units) and -D are the rows the row-dot kernel wrote, staged
//              in shared memory with dO; epilogue (the warps of query half 0
//              write dV, those of half 1 dK)
//   warp  8    producer: K and V of the block once; per step Q (3-stage ring)
//              by TMA, and dO (2-stage ring) by TMA with the step's -LSE and -D
//              rows by bulk copy onto the same barrier (the dO stage is released
//              after dK(s), when the elementwise step has read them)
//   warp  9    TMEM allocator and MMA issuer, in the order
//                dV(s) += P^T(s) dO(s),  S^T(s+1) = K Q(s+1)^T,
//                dK(s) += dS^T(s) Q(s),  dP^T(s+1) = V dO(s+1)^T,
//              so the tensor cores run dV(s) and S^T(s+1) while the elementwise
//              warps form dS^T(s), and dK(s) and dP^T(s+1) while they take the
//              exponentials of step s+1.  A product that writes tensor-memory
//              columns is issued after the one that reads them (one CTA's
//              products run in issue order): S^T(s+1) after dV(s) reads P^T(s),
//              dP^T(s+1) after dK(s) reads dS^T(s).
// Tensor memory: S^T / P^T | dP^T / dS^T | dV | dK, 128 columns each.
// ============================================================================
namespace {

using namespace wait;
using namespace tc;

constexpr int kKvThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kQStages = 3;   // Q is read by S^T(s) and, a step later, by dK(s)
constexpr int kOStages = 2;
constexpr uint32_t kKvOffK = 0;
constexpr uint32_t kKvOffV = kTileBytes;
constexpr uint32_t kKvOffQ = 2 * kTileBytes;
constexpr uint32_t kKvOffO = kKvOffQ + kQStages * kTileBytes;
constexpr uint32_t kKvOffLD = kKvOffO + kOStages * kTileBytes;   // per dO stage: -LSE[128] | -D[128]
constexpr uint32_t kKvLDBytes = 2 * 128 * sizeof(float);
constexpr uint32_t kKvOffBar = kKvOffLD + kOStages * kKvLDBytes;
constexpr int kKvNumBars = 17;
constexpr uint32_t kKvOffMisc = kKvOffBar + kKvNumBars * 8;
constexpr uint32_t kKvSmemUsed = kKvOffMisc + 64;
constexpr uint32_t kSmemMax = 227 * 1024;
// The layout leaves less than 1 KB for aligning the dynamic shared memory base to
// 1024 bytes (which the 128-byte swizzle needs); the kernel checks the base it got
// (the runtime places it 1024-aligned when the kernel declares no static shared
// memory) and reports SSTA_ERR_ALIGNMENT rather than overrun.
constexpr uint32_t kKvSmemAlloc = kKvSmemUsed + 1024 <= kSmemMax ? kKvSmemUsed + 1024 : kSmemMax;
static_assert(kKvSmemUsed <= kSmemMax, "shared memory");

enum : int {
  KB_KV = 0, KB_QFULL = 1, KB_QEMPTY = 4, KB_OFULL = 7, KB_OEMPTY = 9, KB_SFULL = 11, KB_PREADY = 12,
  KB_DPFULL = 13, KB_DSREADY = 14, KB_DONE = 15, KB_DRAIN = 16
};

// Calls f(step, t, ch) for every 128-row chunk with a valid row of every query tile
// in the transposed list, in list order; stops early when f returns false.
template <typename F>
__device__ __forceinline__ int for_each_qchunk(const Geom& g, const ChunkTables& tb, const int32_t* tlist, int tcount,
                                               F&& f) {
  const int nch = g.N / kChunk;
  int step = 0;
  for (int e = 0; e < tcount; ++e) {
    const int t = __ldg(tlist + e);
    uint32_t any, full;
    chunk_bits(g, tb, t, any, full);
    for (int ch = 0; ch < nch; ++ch) {
      if (!((any >> ch) & 1u)) continue;
      if (!f(step, t, ch)) return -1;
      ++step;
    }
  }
  return step;
}

__global__ void __launch_bounds__(kKvThreads, 1)
bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO, const Geom g,
                   const __grid_constant__ ChunkTables tb, const int32_t* __restrict__ tidx, const int32_t* __restrict__ tcnt,
                   const float* __restrict__ nl2, const float* __restrict__ nd, __nv_bfloat16* __restrict__ dk,
                   __nv_bfloat16* __restrict__ dv, int32_t* __restrict__ status, float scale_log2) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t sK = base + kKvOffK, sV = base + kKvOffV;
  auto sQ = [&](int i) { return base + kKvOffQ + (uint32_t)i * kTileBytes; };
  auto sO = [&](int i) { return base + kKvOffO + (uint32_t)i * kTileBytes; };
  auto sLD = [&](int i) { return base + kKvOffLD + (uint32_t)i * kKvLDBytes; };
  auto bar = [&](int i) { return base + kKvOffBar + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + kKvOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + kKvOffMisc + 8);
  volatile int* bad_list = reinterpret_cast<volatile int*>(base_ptr + kKvOffMisc + 16);
  const Ctl ctl{abort_flag, status, kTimeoutNs};
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (base - raw + kKvSmemUsed > kKvSmemAlloc) {   // uniform over the CTA: nothing started yet
    if (threadIdx.x == 0) atomicExch(status, (int)SSTA_ERR_ALIGNMENT);
    return;
  }

  // ---- work unit: one 128-key block of a key tile; text key tiles first (longest lists)
  const int blocks = g.N / 128;
  const int64_t BH = (int64_t)g.B * g.H;
  const int64_t text_units = BH * g.n_text * blocks;
  int64_t u = blockIdx.x;
  int64_t bh;
  int kt, blk;
  if (u < text_units) {
    bh = u / ((int64_t)g.n_text * blocks);
    const int rem = (int)(u - bh * g.n_text * blocks);
    kt = g.NT + rem / blocks;
    blk = rem % blocks;
  } else {
    u -= text_units;
    bh = u / ((int64_t)g.NT * blocks);
    const int rem = (int)(u - bh * g.NT * blocks);
    kt = rem / blocks;
    blk = rem % blocks;
  }
  const int krow0 = kt * g.N + blk * 128;
  const int64_t trow = bh * g.NQ + kt;
  int tcount = __ldg(tcnt + trow);
  if (tcount < 0 || tcount > g.NQ) {
    if (threadIdx.x == 0) atomicExch(status, (int)SSTA_ERR_DEVICE_BOUNDS);
    tcount = tcount < 0 ? 0 : g.NQ;
  }
  const int32_t* tlist = tidx + trow * g.NQ;
  // per-query rows of -LSE and -D: whole tiles per head
  const int64_t Lp = (int64_t)g.NQ * g.N;

  if (threadIdx.x == 0) {
    mbar_init(bar(KB_KV), 1);
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(bar(KB_QFULL + s), 1);
      mbar_init(bar(KB_QEMPTY + s), 1);
    }
    for (int s = 0; s < kOStages; ++s) {
      mbar_init(bar(KB_OFULL + s), 1);
      mbar_init(bar(KB_OEMPTY + s), 1);
    }
    mbar_init(bar(KB_SFULL), 1);
    mbar_init(bar(KB_PREADY), 256);
    mbar_init(bar(KB_DPFULL), 1);
    mbar_init(bar(KB_DSREADY), 256);
    mbar_init(bar(KB_DONE), 1);
    mbar_init(bar(KB_DRAIN), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    *bad_list = 0;
    for (int e = 0; e < tcount; ++e) {
      const int t = __ldg(tlist + e);
      if (t < 0 || t >= g.NQ) { atomicExch(status, (int)SSTA_ERR_DEVICE_BOUNDS); *bad_list = 1; break; }
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
  // a bad list entry (recorded above) walks no query chunk at all
  if (*bad_list) tcount = 0;
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tP = tmem + 128, tDV = tmem + 256, tDK = tmem + 384;

  if (warp == kProducerWarp) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      const int z = (int)bh;
      mbar_expect_tx(bar(KB_KV), 2 * kTileBytes);
      for (int b = 0; b < 2; ++b) {
        tma_load_3d(sK + b * kBox, &tmK, b * 64, krow0, z, bar(KB_KV));
        tma_load_3d(sV + b * kBox, &tmV, b * 64, krow0, z, bar(KB_KV));
      }
      int nq[kQStages] = {0, 0, 0}, no[kOStages] = {0, 0};
      const int n = for_each_qchunk(g, tb, tlist, tcount, [&](int step, int t, int ch) -> bool {
        const int qs = step % kQStages, os = step & 1;
        const int qrow = t * g.N + ch * kChunk;
        if (!wait_bounded(bar(KB_QEMPTY + qs), (uint32_t)(((step / kQStages) & 1) ^ 1), ctl)) return false;
        mbar_expect_tx(bar(KB_QFULL + qs), kTileBytes);
        for (int b = 0; b < 2; ++b) tma_load_3d(sQ(qs) + b * kBox, &tmQ, b * 64, qrow, z, bar(KB_QFULL + qs));
        ++nq[qs];
        if (!wait_bounded(bar(KB_OEMPTY + os), (uint32_t)(((step >> 1) & 1) ^ 1), ctl)) return false;
        // dO and the step's 128 values of -LSE and of -D, on one barrier
        mbar_expect_tx(bar(KB_OFULL + os), kTileBytes + kKvLDBytes);
        for (int b = 0; b < 2; ++b) tma_load_3d(sO(os) + b * kBox, &tmDO, b * 64, qrow, z, bar(KB_OFULL + os));
        bulk_load(sLD(os), nl2 + bh * Lp + qrow, kKvLDBytes / 2, bar(KB_OFULL + os));
        bulk_load(sLD(os) + kKvLDBytes / 2, nd + bh * Lp + qrow, kKvLDBytes / 2, bar(KB_OFULL + os));
        ++no[os];
        return true;
      });
      if (n < 0) {
        drain_wait(bar(KB_KV), 0, kTimeoutNs);
        for (int s = 0; s < kQStages; ++s)
          if (nq[s] > 0) drain_wait(bar(KB_QFULL + s), (uint32_t)((nq[s] - 1) & 1), kTimeoutNs);
        for (int s = 0; s < kOStages; ++s)
          if (no[s] > 0) drain_wait(bar(KB_OFULL + s), (uint32_t)((no[s] - 1) & 1), kTimeoutNs);
      }
      if (n >= 0 && tcount == 0) drain_wait(bar(KB_KV), 0, kTimeoutNs);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const bool ok = wait_bounded(bar(KB_KV), 0, ctl);
      auto s_step = [&](int s) -> bool {   // S^T(s) = K Q(s)^T
        if (!wait_bounded(bar(KB_QFULL + s % kQStages), (uint32_t)((s / kQStages) & 1), ctl)) return false;
        tc_fence_after();
        const uint32_t qb = sQ(s % kQStages);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (uint32_t)(kk >> 2) * kBox + (uint32_t)(kk & 3) * 32u;
          mma_ss(tS, desc_kmajor(sK + off), desc_kmajor(qb + off), kIdescKK, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(KB_SFULL));
        return true;
      };
      auto dp_step = [&](int s) -> bool {   // dP^T(s) = V dO(s)^T
        if (!wait_bounded(bar(KB_OFULL + (s & 1)), (uint32_t)((s >> 1) & 1), ctl)) return false;
        tc_fence_after();
        const uint32_t ob = sO(s & 1);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (uint32_t)(kk >> 2) * kBox + (uint32_t)(kk & 3) * 32u;
          mma_ss(tP, desc_kmajor(sV + off), desc_kmajor(ob + off), kIdescKK, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(KB_DPFULL));
        return true;
      };
      auto dv_step = [&](int s) -> bool {   // dV += P^T(s) dO(s): A = P^T in tensor memory, B = dO MN-major
        if (!wait_bounded(bar(KB_PREADY), (uint32_t)(s & 1), ctl)) return false;
        tc_fence_after();
        const uint32_t ob = sO(s & 1);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tDV, tS + pcol(kk), desc_mnmajor(ob + 2048u * kk), kIdescKMN, (s > 0 || kk > 0) ? 1u : 0u);
        return true;
      };
      auto dk_step = [&](int s) -> bool {   // dK += dS^T(s) Q(s): A = dS^T in tensor memory, B = Q MN-major
        if (!wait_bounded(bar(KB_DSREADY), (uint32_t)(s & 1), ctl)) return false;
        tc_fence_after();
        const uint32_t qb = sQ(s % kQStages);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tDK, tP + pcol(kk), desc_mnmajor(qb + 2048u * kk), kIdescKMN, (s > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bar(KB_QEMPTY + s % kQStages));
        // the dO stage also holds the -LSE and -D the elementwise step read up to DSREADY(s)
        tc_commit(bar(KB_OEMPTY + (s & 1)));
        return true;
      };
      int n = -1;
      if (ok) {
        n = for_each_qchunk(g, tb, tlist, tcount, [&](int step, int, int) -> bool {
          if (step == 0) return s_step(0) && dp_step(0);
          return dv_step(step - 1) && s_step(step) && dk_step(step - 1) && dp_step(step);
        });
      }
      if (n > 0 && dv_step(n - 1) && dk_step(n - 1)) tc_commit(bar(KB_DONE));
      tc_commit(bar(KB_DRAIN));
      drain_wait(bar(KB_DRAIN), 0, kTimeoutNs);
    }
  } else {
    // --------------------------------------------- P^T, dS^T and the epilogue
    // warp w: TMEM lanes 32 (w mod 4) .. +31 (its key rows), query columns 64 (w / 4) .. +63
    const int grp = warp & 3, half = warp >> 2;
    const uint32_t lane_off = (uint32_t)(grp * 32) << 16;
    const int64_t row = (int64_t)krow0 + grp * 32 + lane;
    const bool key_ok = row < g.Lq && key_valid(g, tb, kt, (int)(row - (int64_t)kt * g.N));
    const uint64_t c2 = f2_pack(scale_log2, scale_log2);
    const int n = for_each_qchunk(g, tb, tlist, tcount, [&](int step, int, int) -> bool {
      const float* ld = reinterpret_cast<const float*>(base_ptr + kKvOffLD + (size_t)(step & 1) * kKvLDBytes);
      const float4* nlv = reinterpret_cast<const float4*>(ld + 64 * half);
      const float4* ndv = reinterpret_cast<const float4*>(ld + 128 + 64 * half);
      // P^T = 2^(S^T * scale - LSE), two query columns per f32x2 instruction (-LSE is -inf
      // for a query row without meaning: P = 0); kept in fp32 for dS, written over S^T in bf16.
      // The stage's -LSE and -D arrive with dO: acquire them from its barrier.
      if (!wait_warp(bar(KB_OFULL + (step & 1)), (uint32_t)((step >> 1) & 1), ctl)) return false;
      if (!wait_warp(bar(KB_SFULL), (uint32_t)(step & 1), ctl)) return false;
      tc_fence_after();
      float pv[64];
      tmem_ld64(tS + lane_off + 64u * half, pv);
      uint32_t pk[32];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float4 nl = nlv[i];
        float x[4];
        f2_unpack(f2_fma(f2_pack(pv[4 * i], pv[4 * i + 1]), c2, f2_pack(nl.x, nl.y)), x[0], x[1]);
        f2_unpack(f2_fma(f2_pack(pv[4 * i + 2], pv[4 * i + 3]), c2, f2_pack(nl.z, nl.w)), x[2], x[3]);
#pragma unroll
        for (int e = 0; e < 4; ++e) pv[4 * i + e] = ex2(x[e]);
        pk[2 * i] = pack_bf16x2(pv[4 * i], pv[4 * i + 1]);
        pk[2 * i + 1] = pack_bf16x2(pv[4 * i + 2], pv[4 * i + 3]);
      }
      tmem_st32u(tS + lane_off + 64u * half, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(KB_PREADY));
      // dS^T = P^T (dP^T - D), written over dP^T in bf16
      if (!wait_warp(bar(KB_DPFULL), (uint32_t)(step & 1), ctl)) return false;
      tc_fence_after();
      float dpv[64];
      tmem_ld64(tP + lane_off + 64u * half, dpv);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float4 d4 = ndv[i];
        float ds[4];
        f2_unpack(f2_mul(f2_pack(pv[4 * i], pv[4 * i + 1]), f2_add(f2_pack(dpv[4 * i], dpv[4 * i + 1]), f2_pack(d4.x, d4.y))),
                  ds[0], ds[1]);
        f2_unpack(f2_mul(f2_pack(pv[4 * i + 2], pv[4 * i + 3]),
                         f2_add(f2_pack(dpv[4 * i + 2], dpv[4 * i + 3]), f2_pack(d4.z, d4.w))),
                  ds[2], ds[3]);
        pk[2 * i] = pack_bf16x2(ds[0], ds[1]);
        pk[2 * i + 1] = pack_bf16x2(ds[2], ds[3]);
      }
      tmem_st32u(tP + lane_off + 64u * half, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(KB_DSREADY));
      return true;
    });
    // epilogue: the warps of column half 0 write dV, those of half 1 write dK
    bool have = n > 0;
    if (have) have = wait_warp(bar(KB_DONE), 0u, ctl);
    tc_fence_after();
    const bool write = row < g.Lq && !*abort_flag;
    const float sc = scale_log2 * 0.69314718055994531f;
    const int which = half;
    __nv_bfloat16* orow = (which ? dk : dv) + (bh * g.Lq + row) * 128;
    const float m = key_ok ? (which ? sc : 1.0f) : 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float v[32];
      if (have) {
        tmem_ld32((which ? tDK : tDV) + lane_off + 32u * q, v);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
      }
      if (write) {
        uint4* dst = reinterpret_cast<uint4*>(orow + 32 * q);
#pragma unroll
        for (int w4 = 0; w4 < 4; ++w4) {
          uint4 pkv;
          pkv.x = pack_bf16x2(v[8 * w4 + 0] * m, v[8 * w4 + 1] * m);
          pkv.y = pack_bf16x2(v[8 * w4 + 2] * m, v[8 * w4 + 3] * m);
          pkv.z = pack_bf16x2(v[8 * w4 + 4] * m, v[8 * w4 + 5] * m);
          pkv.w = pack_bf16x2(v[8 * w4 + 6] * m, v[8 * w4 + 7] * m);
          dst[w4] = pkv;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

}  // namespace

cudaError_t launch_attention_bwd_dkdv_tc(const Geom& g, const void* q, const void* k, const void* v, const void* dO,
                                         const float* nl2, const float* nd, const int32_t* tidx,
                                         const int32_t* tcnt, void* dk, void* dv, int32_t* status, cudaStream_t s) {
  const int64_t BH = (int64_t)g.B * g.H;
  if (BH == 0) return cudaSuccess;
  CUtensorMap mq, mk, mv, mdo;
  if (!make_map(&mq, q, g) || !make_map(&mk, k, g) || !make_map(&mv, v, g) || !make_map(&mdo, dO, g))
    return cudaErrorInvalidValue;
  static std::atomic<bool> attr_set[64];
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(bwd_dkdv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kKvSmemAlloc);
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_release);
  }
  const int64_t units = BH * (int64_t)g.NQ * (g.N / 128);
  bwd_dkdv_tc_kernel<<<(unsigned)units, kKvThreads, kKvSmemAlloc, s>>>(
      mq, mk, mv, mdo, g, make_chunk_tables(g), tidx, tcnt, nl2, nd, static_cast<__nv_bfloat16*>(dk),
      static_cast<__nv_bfloat16*>(dv), status, g.scale * 1.4426950408889634f);
  return cudaGetLastError();
}

}  // namespace ssta
