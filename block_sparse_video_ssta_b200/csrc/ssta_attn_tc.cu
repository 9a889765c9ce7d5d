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

#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <atomic>

#include "ssta_wait.cuh"

namespace ssta {
namespace {

using namespace wait;

constexpr int kThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kChunk = 128;                         // keys per pipeline step
constexpr int kStages = 2;
constexpr uint32_t kBox = 128 * 128;                // bytes of one TMA box: 128 rows x 64 bf16
constexpr uint32_t kTileBytes = 2 * kBox;           // 128 rows x 128 channels
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

// Instruction descriptors (kind::f16): D fp32, A and B bf16, M = 128, N = 128.
//   bits [4,6) D format (1 = f32); [7,10) A format (1 = bf16); [10,13) B format;
//   bit 15 A major (0 = K); bit 16 B major (1 = MN); [17,23) N >> 3; [24,29) M >> 4.
constexpr uint32_t kIdescS = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescPV = kIdescS | (1u << 16);

// Which 128-key chunks of a tile hold at least one valid key / only valid keys,
// for the 8 classes of video tiles (bit 2: last along T with padding, bit 1:
// last along Y, bit 0: last along X).  Bit c of a word = chunk c.
struct ChunkTables {
  uint32_t any[8];
  uint32_t full[8];
};

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 consecutive TMEM columns of this thread's lane, waited in the same asm block
// so no use of the registers can be scheduled before the data has arrived.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
      ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
        "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
        "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])),
        "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
        "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
        "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])),
        "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}
// 128 consecutive TMEM columns of this thread's lane in one load, waited in the same asm block.
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, float (&v)[128]) {
  uint32_t r[128];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x128.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63, %64, %65, %66, %67, %68, %69, %70, %71, %72, %73, %74, %75, %76, %77, %78, %79, %80, %81, %82, %83, %84, %85, %86, %87, %88, %89, %90, %91, %92, %93, %94, %95, %96, %97, %98, %99, %100, %101, %102, %103, %104, %105, %106, %107, %108, %109, %110, %111, %112, %113, %114, %115, %116, %117, %118, %119, %120, %121, %122, %123, %124, %125, %126, %127}, [%128];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]), "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]), "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]), "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]), "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]), "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]), "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]), "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]), "=r"(r[119]), "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 128; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st64(uint32_t taddr, const uint32_t (&p)[64]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x64.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63, %64};"
      ::"r"(taddr), "r"(p[0]), "r"(p[1]), "r"(p[2]), "r"(p[3]), "r"(p[4]), "r"(p[5]), "r"(p[6]), "r"(p[7]), "r"(p[8]), "r"(p[9]), "r"(p[10]), "r"(p[11]), "r"(p[12]), "r"(p[13]), "r"(p[14]), "r"(p[15]), "r"(p[16]), "r"(p[17]), "r"(p[18]), "r"(p[19]), "r"(p[20]), "r"(p[21]), "r"(p[22]), "r"(p[23]), "r"(p[24]), "r"(p[25]), "r"(p[26]), "r"(p[27]), "r"(p[28]), "r"(p[29]), "r"(p[30]), "r"(p[31]), "r"(p[32]), "r"(p[33]), "r"(p[34]), "r"(p[35]), "r"(p[36]), "r"(p[37]), "r"(p[38]), "r"(p[39]), "r"(p[40]), "r"(p[41]), "r"(p[42]), "r"(p[43]), "r"(p[44]), "r"(p[45]), "r"(p[46]), "r"(p[47]), "r"(p[48]), "r"(p[49]), "r"(p[50]), "r"(p[51]), "r"(p[52]), "r"(p[53]), "r"(p[54]), "r"(p[55]), "r"(p[56]), "r"(p[57]), "r"(p[58]), "r"(p[59]), "r"(p[60]), "r"(p[61]), "r"(p[62]), "r"(p[63])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// Two-lane fp32 arithmetic (sm_100): one instruction for a pair of values.
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Shared-memory matrix descriptors (tcgen05 format, version 1), 128-byte swizzle.
// K-major (Q, K): rows of 128 B, 8-row groups 1024 B apart (SBO); LBO unused (1).
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) |
         (2ull << 61);
}
// MN-major (V as the B operand of P V): 64-channel blocks kBox apart (LBO),
// 8-key groups 1024 B apart (SBO).
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(kBox >> 4) << 16) | ((uint64_t)(1024 >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}

// ------------------------------------------------------------- chunk sequence
__device__ __forceinline__ void chunk_bits(const Geom& g, const ChunkTables& tb, int t, uint32_t& any,
                                           uint32_t& full) {
  const int nch = g.N / kChunk;
  if (t < g.NT) {
    const int cX = t % g.nX, cY = (t / g.nX) % g.nY, cT = t / (g.nX * g.nY);
    const int cls = ((cT == g.nT - 1 && g.T % g.tT) ? 4 : 0) | ((cY == g.nY - 1 && g.Y % g.tY) ? 2 : 0) |
                    ((cX == g.nX - 1 && g.X % g.tX) ? 1 : 0);
    any = tb.any[cls];
    full = tb.full[cls];
  } else {
    const int rem = g.L_text - (t - g.NT) * g.N;   // valid keys in this text tile
    any = 0;
    full = 0;
    for (int c = 0; c < nch; ++c) {
      if (c * kChunk < rem) any |= 1u << c;
      if ((c + 1) * kChunk <= rem) full |= 1u << c;
    }
  }
}

// Calls f(j, t, ch, full) for every chunk with a valid key, in list order; stops
// early when f returns false.  Returns the number of chunks visited.
template <typename F>
__device__ __forceinline__ int for_each_chunk(const Geom& g, const ChunkTables& tb, const int32_t* list, int cnt,
                                              F&& f) {
  const int nch = g.N / kChunk;
  int j = 0;
  for (int e = 0; e < cnt; ++e) {
    const int t = __ldg(list + e);
    if (t < 0 || t >= g.NQ) continue;
    uint32_t any, full;
    chunk_bits(g, tb, t, any, full);
    for (int ch = 0; ch < nch; ++ch) {
      if (!((any >> ch) & 1u)) continue;
      if (!f(j, t, ch, ((full >> ch) & 1u) != 0)) return -1;
      ++j;
    }
  }
  return j;
}

__device__ __forceinline__ bool key_valid(const Geom& g, int t, int o) {
  if (t < g.NT) {
    const int cX = t % g.nX, cY = (t / g.nX) % g.nY, cT = t / (g.nX * g.nY);
    const int dx = o % g.tX, dy = (o / g.tX) % g.tY, dt = o / (g.tX * g.tY);
    return dt < axis_valid(cT, g.tT, g.T) && dy < axis_valid(cY, g.tY, g.Y) && dx < axis_valid(cX, g.tX, g.X);
  }
  return (t - g.NT) * g.N + o < g.L_text;
}

// ------------------------------------------------------------------- kernel
__global__ void __launch_bounds__(kThreads, 1)
ssta_attention_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const Geom g, const ChunkTables tb,
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
          const uint32_t vm = __ballot_sync(0xffffffffu, key_valid(g, t, ch * kChunk + q * 32 + lane));
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

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

bool make_map(CUtensorMap* map, const void* ptr, const Geom& g) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)g.D, (cuuint64_t)g.Lq, (cuuint64_t)g.B * g.H};
  cuuint64_t strides[2] = {(cuuint64_t)g.D * 2, (cuuint64_t)g.Lq * g.D * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

ChunkTables make_chunk_tables(const Geom& g) {
  ChunkTables tb{};
  const int nch = g.N / kChunk;
  for (int cls = 0; cls < 8; ++cls) {
    const int vt = (cls & 4) ? g.T - (g.nT - 1) * g.tT : g.tT;
    const int vy = (cls & 2) ? g.Y - (g.nY - 1) * g.tY : g.tY;
    const int vx = (cls & 1) ? g.X - (g.nX - 1) * g.tX : g.tX;
    for (int c = 0; c < nch; ++c) {
      int valid = 0;
      for (int o = c * kChunk; o < (c + 1) * kChunk; ++o) {
        const int dx = o % g.tX, dy = (o / g.tX) % g.tY, dt = o / (g.tX * g.tY);
        valid += (dt < vt && dy < vy && dx < vx) ? 1 : 0;
      }
      if (valid > 0) tb.any[cls] |= 1u << c;
      if (valid == kChunk) tb.full[cls] |= 1u << c;
    }
  }
  return tb;
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
