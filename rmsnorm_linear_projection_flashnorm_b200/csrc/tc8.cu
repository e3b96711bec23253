// Fused RMSNorm + projection, tile path (M > 64) for fp8 e4m3 weights with an
// fp32 scale per 128 x 128 block, and for MXFP8 weights (e4m3 with a ue8m0
// scale per 32 k values and column), sm_100a.
//
// The arithmetic is FlashNorm's (FlashNorm talk summary, Proposal 2: matmul on
// raw x, the sum of squares alongside, 1/rms applied after; the folded weight
// may be quantised, Proposal 1):
//
//   y[m, n] = r[m] * sum_b s[b, n] * sum_{k in block b} q[k, n] x[m, k]
//
// The e4m3 weight codes go to the tensor cores as they are stored: TMA copies
// them into shared memory with the 128-byte swizzle and they are the B operand
// (N-major) of tcgen05.mma kind::f8f6f4.  The activations are converted
// instead, exactly, once per call: a small kernel splits each row and
// 128-deep k block of x into hi = e4m3(a) and lo = e4m3(a - hi) with
// a = x * 2^e (the power of two that puts the block's largest magnitude in
// [128, 256)), writes the two code planes, 2^-e per (block, row), and the
// partial sums of squares per (block, row).  In the tile kernel every 128-deep k block is one
// pipeline stage: eight MMAs (four 32-deep steps for x_hi, four for x_lo) sum
// the exact products into a TMEM buffer of its own, and scaler warps read the
// buffer back and add it, times s[b, n] * 2^-e[b, m], to fp32 running sums in
// registers, in ascending k order.  This is the block-scale promotion of the
// Marlin explainer's section 4 (dequantisation hidden under the MMA stream),
// applied to the sums instead of the weights: no weight tile is converted and
// no bf16 copy of the weight is written.
//
// MXFP8 weights (the MX instance): the split runs per 32-deep block and its
// powers of two become the activations' ue8m0 scale bytes, so block-scaled
// MMAs (kind::mxf8f6f4.block_scale) apply both operands' scales in hardware
// and one TMEM accumulator holds a work item's whole k range; the scalers only
// read it once per item.
//
// Compared with converting the staged weight tiles to bf16 on chip, the weight
// bytes per flop in shared memory are the same (B is read once per half of the
// split), and the conversion work moves off the MMA's critical path; compared
// with dequantising the whole weight into the workspace first, it saves a
// write and a read of a bf16 weight copy per call.
//
// Layout (persistent, one CTA per SM, 128 x 256 output tiles):
//   warp 0      TMA producer (x_hi, x_lo, two e4m3 weight boxes per stage)
//   warp 1      TMEM owner and MMA issuer
//   warps 2-9   scalers and epilogue: warp w reads TMEM lane quarter w % 4;
//               the two warps of a quarter take the two halves of the tile's
//               columns (SwiGLU: matching 64-column halves of gate and up)
#include <cstddef>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace fn {
namespace tc8 {

constexpr int BM = 128, BN = 256, BKQ = 128;
constexpr int XQ_BYTES = BM * BKQ;                    // one e4m3 code plane tile: 128 rows x 128 k (16 KB)
constexpr int WQ_BOX = 128 * BKQ;                     // 128 weight columns x 128 k rows (16 KB)
constexpr int OPERAND_BYTES = 2 * XQ_BYTES + 2 * WQ_BOX;   // x_hi, x_lo, weight: 64 KB
constexpr int SF_CHUNK = 512;                         // MXFP8: 128 rows or columns x 4 scale bytes
// MXFP8 stages also hold the x scale chunk and the two weight scale chunks
template <bool MX> __host__ __device__ constexpr int stage_bytes() { return OPERAND_BYTES + (MX ? 2048 : 0); }
constexpr int STAGES = 3;
constexpr int NUM_THREADS = 320;
constexpr int TMEM_COLS = 2 * BN;   // fp8: two per-k-block accumulators; MXFP8: one accumulator + scales
constexpr int SF_TMEM = BN;         // MXFP8: per stage 12 scale words (x, then two weight chunks) from here
constexpr int GROUP_M = 16;                           // tile raster: bands of 16 row blocks

enum : unsigned { kSiteProdEmpty = 1, kSiteMmaAccEmpty, kSiteMmaFull, kSiteScaleAccFull };

struct Params {
  int M, d, ncols, nout;
  int num_m, num_n, num_tiles, kblocks, nblk;
  float eps, inv_d;
  __nv_bfloat16* y;
  unsigned int* status;
  unsigned long long budget_ns;
  int withhold;
  const float* scales;   // weight block scales [kblocks][nblk]
  const float* fac;      // 2^-e of each (k block, row) of the split [kblocks][M]; NaN: non-finite block
  const float* ssq_part; // sum of squares of each (k block, row) [kblocks][M]
  const uint8_t* wsf;    // MXFP8: weight scale chunks [kblocks][nblk][512] (none for fp8)
  const uint8_t* xsf;    // MXFP8: x scale chunks [kblocks][num_m][512]
  int split_tail;        // 1: launched as 2-CTA clusters; the tiles after the full waves are split in k
  int full_waves;        //   between the two CTAs of a cluster (tile full_waves * grid + cluster index)
  int tail;              //   number of such tiles (<= clusters)
};

// The i-th work item of this CTA: a tile and its k-block range.  Without the
// split tail, tiles are dealt round-robin over the CTAs.  With it, every CTA
// first takes full_waves whole tiles the same way, and then the two CTAs of
// cluster c share tile full_waves * grid + c (c < tail): rank 0 takes the
// lower half of the k blocks, rank 1 the upper half.  A last wave that would
// leave more than half of the SMs idle thus takes half as long.
struct Work {
  int t, kb0, kb1;
  bool split;
};
__device__ __forceinline__ bool work_item(const Params& p, int i, Work& w) {
  const int G = static_cast<int>(gridDim.x);
  w.split = false;
  w.kb0 = 0;
  w.kb1 = p.kblocks;
  if (!p.split_tail || i < p.full_waves) {
    w.t = static_cast<int>(blockIdx.x) + i * G;
    return w.t < p.num_tiles && (!p.split_tail || i < p.full_waves);
  }
  const int c = static_cast<int>(blockIdx.x) >> 1, r = static_cast<int>(blockIdx.x) & 1;
  if (i != p.full_waves || c >= p.tail) return false;
  w.t = p.full_waves * G + c;
  w.kb0 = r * p.kblocks / 2;
  w.kb1 = (r + 1) * p.kblocks / 2;
  w.split = true;
  return true;
}

struct alignas(8) Bars {
  uint64_t full[STAGES], empty[STAGES];
  uint64_t accf[2], acce[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <bool MX> constexpr size_t smem_bytes() { return 1024 + STAGES * stage_bytes<MX>() + sizeof(Bars); }
static_assert(smem_bytes<false>() <= 232448 && smem_bytes<true>() <= 232448, "shared memory budget");
static_assert(SF_TMEM + STAGES * 12 <= TMEM_COLS, "MXFP8 scale words fit TMEM beside the accumulator");

__device__ __forceinline__ void tile_coords(int t, const Params& p, int& mb, int& nb) {
  const int per_group = GROUP_M * p.num_n;
  const int group = t / per_group;
  const int first_m = group * GROUP_M;
  const int gm = min(p.num_m - first_m, GROUP_M);
  const int r = t - group * per_group;
  mb = first_m + r % gm;
  nb = r / gm;
}

// Store 8 bytes into another CTA's shared memory (a shared::cluster address).
__device__ __forceinline__ void st_cluster_u64(uint32_t cluster_addr, uint64_t v) {
  asm volatile("st.shared::cluster.u64 [%0], %1;" ::"r"(cluster_addr), "l"(v) : "memory");
}

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, unsigned long long budget) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > budget) return;
  }
}

// ---------------------------------------------------------------------------
// Split x once per call.  One warp per (row, 128-deep k block); lane l takes
// k values 4l .. 4l+3, so the eight warps of a block read 2 KB of one row in
// one coalesced sweep.  Each warp writes its 128 hi and lo codes, 2^-e and the
// block's partial sum of squares (lane sums reduced in a fixed tree); the tile
// kernel adds a row's partial sums in k order, so repeated calls agree bit for
// bit.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) xsplit_rows_kernel(const __nv_bfloat16* __restrict__ x, int M, int d,
                                                          uint8_t* __restrict__ xhi, uint8_t* __restrict__ xlo,
                                                          float* __restrict__ fac, float* __restrict__ ssq_part) {
  grid_launch_dependents();     // the tile kernel may set up meanwhile
  grid_dependency_wait();       // x may have been written by the preceding kernel
  const int kblocks = d / BKQ;
  const long long wg = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int row = static_cast<int>(wg / kblocks), kb = static_cast<int>(wg - static_cast<long long>(row) * kblocks);
  if (row >= M) return;
  const int64_t off = static_cast<int64_t>(row) * d + kb * BKQ + lane * 4;
  const uint2 v = __ldg(reinterpret_cast<const uint2*>(x + off));
  uint32_t amax = max(max(v.x & 0x7FFFu, (v.x >> 16) & 0x7FFFu), max(v.y & 0x7FFFu, (v.y >> 16) & 0x7FFFu));
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  // amax is a bf16 bit pattern (|x| orders like its bits): exponent field in
  // bits 7..14, 255 for inf / NaN
  const int E = static_cast<int>(amax >> 7);
  int e = amax == 0 ? 0 : 134 - E;          // amax * 2^e in [128, 256)
  e = e > 126 ? 126 : (e < -126 ? -126 : e);
  const float sc = __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
  const uint64_t sc2 = f2_pack(sc, sc);
  const uint64_t a = f2_pack_u(v.x << 16, v.x & 0xFFFF0000u), b = f2_pack_u(v.y << 16, v.y & 0xFFFF0000u);
  const uint64_t ss2 = f2_fma(b, b, f2_mul(a, a));
  uint16_t h0, l0, h1, l1;
  split_e4m3x2(f2_mul(a, sc2), h0, l0);
  split_e4m3x2(f2_mul(b, sc2), h1, l1);
  *reinterpret_cast<uint32_t*>(xhi + off) = static_cast<uint32_t>(h0) | (static_cast<uint32_t>(h1) << 16);
  *reinterpret_cast<uint32_t*>(xlo + off) = static_cast<uint32_t>(l0) | (static_cast<uint32_t>(l1) << 16);
  float ss = f2_lo(ss2) + f2_hi(ss2);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) {
    fac[static_cast<int64_t>(kb) * M + row] =
        E == 255 ? __int_as_float(0x7fc00000) : __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
    ssq_part[static_cast<int64_t>(kb) * M + row] = ss;
  }
}

// MXFP8 weights: the same split per 32-deep block instead of per 128-deep
// block, the power of two stored as a ue8m0 byte (127 - e) in the chunk layout
// the block-scaled MMA reads (per 128-row block and 128-deep k group, a
// 512-byte chunk; row r's byte for 32-deep block b at 16 (r mod 32) +
// 4 (r div 32 mod 4) + b).  Rows from M up to the last 128-row block get
// byte 127 (their operand rows are TMA zero fill).  The partial sums of
// squares per (128-deep group, row) are those of the fp8 split.
__global__ void __launch_bounds__(256) xsplit_mx_rows_kernel(const __nv_bfloat16* __restrict__ x, int M, int Mpad,
                                                             int d, uint8_t* __restrict__ xhi,
                                                             uint8_t* __restrict__ xlo, uint8_t* __restrict__ xsf,
                                                             float* __restrict__ ssq_part) {
  grid_launch_dependents();
  grid_dependency_wait();
  const int kblocks = d / BKQ;
  const long long wg = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int row = static_cast<int>(wg / kblocks), kb = static_cast<int>(wg - static_cast<long long>(row) * kblocks);
  if (row >= Mpad) return;
  const bool live = row < M;
  const int64_t off = static_cast<int64_t>(row) * d + kb * BKQ + lane * 4;
  uint2 v = make_uint2(0u, 0u);
  if (live) v = __ldg(reinterpret_cast<const uint2*>(x + off));
  uint32_t amax = max(max(v.x & 0x7FFFu, (v.x >> 16) & 0x7FFFu), max(v.y & 0x7FFFu, (v.y >> 16) & 0x7FFFu));
#pragma unroll
  for (int o = 4; o >= 1; o >>= 1) amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, o));   // 8 lanes: 32 k
  const int E = static_cast<int>(amax >> 7);
  int e = amax == 0 ? 0 : 134 - E;
  e = e > 126 ? 126 : (e < -126 ? -126 : e);
  const float sc = __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
  const uint64_t sc2 = f2_pack(sc, sc);
  const uint64_t a = f2_pack_u(v.x << 16, v.x & 0xFFFF0000u), b = f2_pack_u(v.y << 16, v.y & 0xFFFF0000u);
  const uint64_t ss2 = f2_fma(b, b, f2_mul(a, a));
  if (live) {
    uint16_t h0, l0, h1, l1;
    split_e4m3x2(f2_mul(a, sc2), h0, l0);
    split_e4m3x2(f2_mul(b, sc2), h1, l1);
    *reinterpret_cast<uint32_t*>(xhi + off) = static_cast<uint32_t>(h0) | (static_cast<uint32_t>(h1) << 16);
    *reinterpret_cast<uint32_t*>(xlo + off) = static_cast<uint32_t>(l0) | (static_cast<uint32_t>(l1) << 16);
  }
  if ((lane & 7) == 0) {
    const int r = row & 127;
    xsf[(static_cast<int64_t>(kb) * (Mpad / BM) + row / BM) * SF_CHUNK + 16 * (r & 31) + 4 * (r >> 5) + (lane >> 3)] =
        static_cast<uint8_t>(live ? 127 - e : 127);
  }
  float ss = f2_lo(ss2) + f2_hi(ss2);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0 && live) ssq_part[static_cast<int64_t>(kb) * M + row] = ss;
}

// Epilogue of one thread's share of a tile: row `row`, column half `half`.
// 1/rms of the raw row (FlashNorm's deferred normalisation), then SwiGLU (the
// two chunks hold matching gate and up columns) or the plain projection (the
// two chunks are 128 consecutive columns), one RN to bf16, 16-byte stores.
template <bool SWIGLU>
__device__ __forceinline__ void store_tile_half(const Params& p, const uint64_t (&acc)[64], int row, int nb, int half,
                                                float ssq) {
  // a row holding inf or NaN has a non-finite sum of squares: all its
  // outputs are NaN, as in a bf16 matmul (the fp8 factors already carry it)
  const float r = isfinite(ssq) ? inv_rms(ssq, p.inv_d, p.eps) : __int_as_float(0x7fc00000);
  if constexpr (SWIGLU) {
    __nv_bfloat16* yrow = p.y + static_cast<int64_t>(row) * p.nout + nb * (BN / 2) + half * 64;
#pragma unroll
    for (int g16 = 0; g16 < 8; ++g16) {
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint64_t gv = acc[g16 * 4 + j], uv = acc[32 + g16 * 4 + j];
        const float g0 = f2_lo(gv) * r, g1 = f2_hi(gv) * r, u0 = f2_lo(uv) * r, u1 = f2_hi(uv) * r;
        o[j] = pack_bf16x2(silu_f32(g0) * u0, silu_f32(g1) * u1);
      }
      reinterpret_cast<uint4*>(yrow)[g16] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  } else {
    const int col0 = nb * BN + half * 128;
    if (col0 >= p.nout) return;   // the half of a last tile that lies past the weight
    __nv_bfloat16* yrow = p.y + static_cast<int64_t>(row) * p.nout + col0;
#pragma unroll
    for (int g16 = 0; g16 < 16; ++g16) {
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint64_t v = acc[g16 * 4 + j];
        o[j] = pack_bf16x2(f2_lo(v) * r, f2_hi(v) * r);
      }
      reinterpret_cast<uint4*>(yrow)[g16] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

// ---------------------------------------------------------------------------
// The tile kernel.
// ---------------------------------------------------------------------------
// MX: MXFP8 weights (e4m3 with a ue8m0 scale per 32 k values and column):
// the same stages plus the scale chunks, block-scaled MMAs
// (kind::mxf8f6f4.block_scale, x_hi and x_lo under the same x scales) that
// accumulate a work item's whole k range in one TMEM accumulator, and scaler
// warps that only read the accumulator once per item for the epilogue.
template <bool SWIGLU, bool MX>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    tc8_kernel(const __grid_constant__ CUtensorMap tmap_xh, const __grid_constant__ CUtensorMap tmap_xl,
               const __grid_constant__ CUtensorMap tmap_w, const Params p) {
  constexpr int STAGE_BYTES = stage_bytes<MX>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars& bars = *reinterpret_cast<Bars*>(smem + STAGES * STAGE_BYTES);
  // stage: [x_hi 128 x 128][x_lo 128 x 128][weight: two 128-column boxes]
  //        (MXFP8: [x scale chunk][weight scale chunks]), 1024-byte multiples
  auto stage_xh = [&](int s) { return smem + s * STAGE_BYTES; };
  auto stage_xl = [&](int s) { return smem + s * STAGE_BYTES + XQ_BYTES; };
  auto stage_w = [&](int s) { return smem + s * STAGE_BYTES + 2 * XQ_BYTES; };
  auto stage_sf = [&](int s) { return smem + s * STAGE_BYTES + OPERAND_BYTES; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.empty[s], 1);       // MMA commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars.accf[b], 1);        // MMA commit
      mbar_init(&bars.acce[b], 8);        // one arrival per scaler warp
    }
    mbar_init(&bars.drain, 1);
    bars.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmap_xh);
    tma_prefetch_desc(&tmap_xl);
    tma_prefetch_desc(&tmap_w);
  }
  if (warp == 1) {
    tmem_alloc(&bars.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Everything above overlaps the preceding kernel (the x split); nothing
  // below touches global memory before it has completed.
  grid_dependency_wait();
  grid_launch_dependents();
  const uint32_t tmem_base = bars.tmem_base;
  const WaitCtl ctl{&bars.abort_flag, p.status, p.budget_ns};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0, issued = 0, last_ph = 0;
      bool ok = true;
      Work w;
      for (int i = 0; ok && work_item(p, i, w); ++i) {
        int mb, nb;
        tile_coords(w.t, p, mb, nb);
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!mbar_wait(&bars.empty[s], ph ^ 1, ctl, kSiteProdEmpty)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars.full[s], OPERAND_BYTES + (MX ? 3 * SF_CHUNK : 0));
          if constexpr (MX) {
            // x scale chunk of (k group, row block); weight chunks of the tile's two
            // 128-column blocks (a block past the weight reuses the last chunk:
            // its weight box is zero fill)
            bulk_load(stage_sf(s), p.xsf + (static_cast<int64_t>(kb) * p.num_m + mb) * SF_CHUNK, SF_CHUNK,
                      &bars.full[s]);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int cb = min(2 * nb + h, p.nblk - 1);
              bulk_load(stage_sf(s) + (1 + h) * SF_CHUNK, p.wsf + (static_cast<int64_t>(kb) * p.nblk + cb) * SF_CHUNK,
                        SF_CHUNK, &bars.full[s]);
            }
          }
          tma_load_2d(stage_xh(s), &tmap_xh, &bars.full[s], kb * BKQ, mb * BM);
          tma_load_2d(stage_xl(s), &tmap_xl, &bars.full[s], kb * BKQ, mb * BM);
          // a plain projection with an odd number of 128-column blocks has a
          // last tile whose second box lies past the weight: TMA fills zeros
          tma_load_2d(stage_w(s), &tmap_w, &bars.full[s], nb * BN, kb * BKQ);
          tma_load_2d(stage_w(s) + WQ_BOX, &tmap_w, &bars.full[s], nb * BN + 128, kb * BKQ);
          issued |= 1u << s;
          last_ph = (last_ph & ~(1u << s)) | (ph << s);
          if (++s == STAGES) { s = 0; ph ^= 1; }
        }
      }
      // no copy may still be landing in shared memory when the CTA exits
      for (int i = 0; i < STAGES; ++i)
        if (issued & (1u << i)) drain_wait(&bars.full[i], (last_ph >> i) & 1u, p.budget_ns);
    }
    __syncwarp();
    if (p.split_tail) {   // the exchange of the scalers below: every thread takes part
      cluster_sync_all();
      cluster_sync_all();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (MX && lane == 0) {
      // One accumulator per work item over its whole k range.  Per stage the
      // three scale chunks go to this stage's TMEM scale words (tcgen05.cp,
      // ordered with the MMAs after it), then per 32-deep k step one
      // block-scaled MMA for x_hi and one for x_lo, both under the x scales.
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      Work w;
      for (int i = 0; ok && work_item(p, i, w); ++i) {
        if (!mbar_wait(&bars.acce[0], (static_cast<uint32_t>(i) & 1u) ^ 1u, ctl, kSiteMmaAccEmpty)) break;
        tc_fence_after();
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!mbar_wait(&bars.full[s], ph, ctl, kSiteMmaFull)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sf_t = tmem_base + SF_TMEM + s * 12;
          const uint32_t sf_s = smem_u32(stage_sf(s));
#pragma unroll
          for (int c = 0; c < 3; ++c) tmem_cp_32x128b_x4(sf_t + 4 * c, sdesc_plain(sf_s + c * SF_CHUNK, 128, 128));
          const uint32_t xh = smem_u32(stage_xh(s)), xl = smem_u32(stage_xl(s)), w0 = smem_u32(stage_w(s));
#pragma unroll
          for (int kk = 0; kk < BKQ / 32; ++kk) {
            // the scale byte of this 32-deep block is byte kk of each scale word
            const uint32_t idesc = idesc_mx_e4m3(BM, BN, /*a MN-major*/ false, /*b MN-major*/ true, kk);
            const uint64_t bdesc = sdesc_sw128(w0 + kk * 4096, WQ_BOX, 1024);
#pragma unroll
            for (int part = 0; part < 2; ++part) {
              const uint64_t adesc = sdesc_sw128((part == 0 ? xh : xl) + kk * 32, 16, 1024);
              umma_mx_e4m3(tmem_base, adesc, bdesc, idesc, sf_t, sf_t + 4,
                           (kb != w.kb0 || kk != 0 || part != 0) ? 1u : 0u);
            }
          }
          umma_commit(&bars.empty[s]);
          if (++s == STAGES) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        umma_commit(&bars.accf[0]);
      }
      umma_commit(&bars.drain);
      drain_wait(&bars.drain, 0, p.budget_ns);
    } else if (!MX && lane == 0) {
      // A = x_hi / x_lo rows, K-major; B = e4m3 weight, N-major
      constexpr uint32_t IDESC = idesc_e4m3_f32(BM, BN, /*a MN-major*/ false, /*b MN-major*/ true);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      uint32_t it = 0;   // k blocks processed by this CTA: selects the TMEM buffer
      Work w;
      for (int i = 0; ok && work_item(p, i, w); ++i) {
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
          const uint32_t b = it & 1, aph = (it >> 1) & 1;
          if (!mbar_wait(&bars.acce[b], aph ^ 1, ctl, kSiteMmaAccEmpty)) { ok = false; break; }
          if (!mbar_wait(&bars.full[s], ph, ctl, kSiteMmaFull)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + b * BN;
          const uint32_t xh = smem_u32(stage_xh(s)), xl = smem_u32(stage_xl(s)), w0 = smem_u32(stage_w(s));
#pragma unroll
          for (int part = 0; part < 2; ++part) {
#pragma unroll
            for (int kk = 0; kk < BKQ / 32; ++kk) {
              // A: 128-byte rows of e4m3 codes, 8-row groups 1024 B apart; a
              //    32-deep step is 32 bytes further along the (swizzled) row.
              const uint64_t adesc = sdesc_sw128((part == 0 ? xh : xl) + kk * 32, 16, 1024);
              // B: k rows of 128 columns (128 bytes), the two column boxes
              //    16 KB apart (LBO), 8-row k groups 1024 B apart (SBO); a
              //    32-deep step is 32 rows = 4096 B.
              const uint64_t bdesc = sdesc_sw128(w0 + kk * 4096, WQ_BOX, 1024);
              umma_e4m3(d_tmem, adesc, bdesc, IDESC, (part | kk) != 0 ? 1u : 0u);
            }
          }
          umma_commit(&bars.empty[s]);
          umma_commit(&bars.accf[b]);
          if (++s == STAGES) { s = 0; ph ^= 1; }
        }
      }
      umma_commit(&bars.drain);
      drain_wait(&bars.drain, 0, p.budget_ns);
    }
    __syncwarp();
    if (p.split_tail) {
      cluster_sync_all();
      cluster_sync_all();
    }
  } else {
    // ------------------------------------------------------------ scalers and epilogue
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;       // 0: warps 2-5, 1: warps 6-9
    // the two 64-column chunks of the 256-column accumulator this thread adds up
    const int c0 = SWIGLU ? half * 64 : half * 128;
    const int c1 = SWIGLU ? BN / 2 + half * 64 : half * 128 + 64;
    uint32_t it = 0;
    bool ok = true;
    uint64_t acc[64];   // packed fp32 pairs: chunk 0 columns in acc[0..31], chunk 1 in acc[32..63]
    bool split_pending = false;             // a k-split tile's partial sums wait for the exchange
    int s_row = 0, s_nb = 0;
    float s_ssq = 0.f;
    Work w;
    for (int i = 0; ok && work_item(p, i, w); ++i) {
      int mb, nb;
      tile_coords(w.t, p, mb, nb);
      const int row = mb * BM + q * 32 + lane;
      const bool live = row < p.M;
      // 128-column weight blocks of the two chunks (the scale columns)
      const int blk0 = SWIGLU ? 2 * nb : 2 * nb + half;
      const int blk1 = SWIGLU ? 2 * nb + 1 : 2 * nb + half;
      const bool have0 = blk0 < p.nblk, have1 = blk1 < p.nblk;
      // the row's sum of squares: its k blocks' partial sums, in k order
      float ssq = 0.f;
      if (live) {
#pragma unroll 8
        for (int kb = 0; kb < p.kblocks; ++kb) ssq += __ldg(p.ssq_part + static_cast<int64_t>(kb) * p.M + row);
      }
      if constexpr (MX) {
        // the accumulator holds the item's whole sums: read it once
        if (!__all_sync(0xffffffffu, mbar_wait(&bars.accf[0], static_cast<uint32_t>(i) & 1u, ctl,
                                               kSiteScaleAccFull))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll
        for (int rd = 0; rd < 4; ++rd) {
          uint32_t v0[16], v1[16];
          const uint32_t col = (rd < 2 ? c0 : c1) + (rd & 1) * 32;
          tmem_ld16(taddr + col, v0);
          tmem_ld16(taddr + col + 16, v1);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            acc[rd * 16 + j] = f2_pack_u(v0[2 * j], v0[2 * j + 1]);
            acc[rd * 16 + 8 + j] = f2_pack_u(v1[2 * j], v1[2 * j + 1]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0 && !(p.withhold && i == 0)) mbar_arrive(&bars.acce[0]);
      } else {
#pragma unroll
      for (int j = 0; j < 64; ++j) acc[j] = 0;
      // 2^-e and the block scales, loaded one k block ahead
      auto load_fac = [&](int kb) { return live ? __ldg(p.fac + static_cast<int64_t>(kb) * p.M + row) : 0.f; };
      auto load_s = [&](int kb, int blk, bool have) {
        return have ? __ldg(p.scales + static_cast<int64_t>(kb) * p.nblk + blk) : 0.f;
      };
      float f_n = load_fac(w.kb0), s0_n = load_s(w.kb0, blk0, have0), s1_n = load_s(w.kb0, blk1, have1);
      for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
        const float f = f_n, s0 = s0_n, s1 = s1_n;
        if (kb + 1 < w.kb1) {
          f_n = load_fac(kb + 1);
          s0_n = load_s(kb + 1, blk0, have0);
          s1_n = load_s(kb + 1, blk1, have1);
        }
        const uint32_t b = it & 1, aph = (it >> 1) & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&bars.accf[b], aph, ctl, kSiteScaleAccFull))) { ok = false; break; }
        tc_fence_after();
        // s * 2^-e: the product is exact unless it leaves the normal range
        const float k0 = f * s0, k1 = f * s1;
        const uint64_t kk0 = f2_pack(k0, k0), kk1 = f2_pack(k1, k1);
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + b * BN;
        // four rounds of 32 columns (two 16-column loads each), so that the
        // loaded values and the 128 running sums fit the register budget of
        // 10 warps per SM (at most 3 warps on a scheduler: 168 registers)
#pragma unroll
        for (int rd = 0; rd < 4; ++rd) {
          uint32_t v0[16], v1[16];
          const uint32_t col = (rd < 2 ? c0 : c1) + (rd & 1) * 32;
          tmem_ld16(taddr + col, v0);
          tmem_ld16(taddr + col + 16, v1);
          tmem_ld_wait();
          if (rd == 3) {
            // every TMEM read of this buffer has completed: hand it back
            tc_fence_before();
            __syncwarp();
            if (lane == 0 && !(p.withhold && it == 0)) mbar_arrive(&bars.acce[b]);
          }
          const uint64_t kc = rd < 2 ? kk0 : kk1;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            acc[rd * 16 + j] = f2_fma(kc, f2_pack_u(v0[2 * j], v0[2 * j + 1]), acc[rd * 16 + j]);
            acc[rd * 16 + 8 + j] = f2_fma(kc, f2_pack_u(v1[2 * j], v1[2 * j + 1]), acc[rd * 16 + 8 + j]);
          }
        }
      }
      }
      if (!ok) break;
      if (w.split) {   // the CTA's last item: its partner holds the other half of the k range
        split_pending = true;
        s_row = row;
        s_nb = nb;
        s_ssq = ssq;
        break;
      }
      if (live) store_tile_half<SWIGLU>(p, acc, row, nb, half, ssq);
    }
    if (p.split_tail) {
      // Both CTAs of the cluster are past their main loops (their loads have
      // landed and their MMAs completed), so the pipeline memory of each is
      // free.  Each CTA finishes one column half of a split tile: rank r the
      // half r.  The other half's partial sums go to the partner's shared
      // memory, [pair j][tile row] in 8-byte words, and come back added in a
      // fixed order (fp32 a + b is the same either way round).
      const uint32_t rank = blockIdx.x & 1u;
      cluster_sync_all();
      if (split_pending && static_cast<uint32_t>(half) != rank) {
        const uint32_t dst = dsmem_addr(smem, rank ^ 1u) + 8u * static_cast<uint32_t>(q * 32 + lane);
#pragma unroll
        for (int j = 0; j < 64; ++j) st_cluster_u64(dst + 1024u * j, acc[j]);
      }
      cluster_sync_all();
      if (split_pending && static_cast<uint32_t>(half) == rank && ok && s_row < p.M) {
        const uint64_t* src = reinterpret_cast<const uint64_t*>(smem) + (q * 32 + lane);
#pragma unroll
        for (int j = 0; j < 64; ++j) acc[j] = f2_add(acc[j], src[128 * j]);
        store_tile_half<SWIGLU>(p, acc, s_row, s_nb, half, s_ssq);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

template <bool SWIGLU, bool MX>
cudaError_t launch_kernel(int grid, cudaStream_t stream, const CUtensorMap& th, const CUtensorMap& tl,
                          const CUtensorMap& tw, const Params& p) {
  constexpr size_t SMEM = smem_bytes<MX>();
  const cudaError_t e = ensure_smem_limit<tc8_kernel<SWIGLU, MX>>(static_cast<int>(SMEM));
  if (e != cudaSuccess) return e;
  if (p.split_tail)
    return launch_pdl_cluster(tc8_kernel<SWIGLU, MX>, static_cast<unsigned>(grid), 2, NUM_THREADS, SMEM, stream, th,
                              tl, tw, p);
  return launch_pdl(tc8_kernel<SWIGLU, MX>, grid, NUM_THREADS, SMEM, stream, th, tl, tw, p);
}

}  // namespace tc8

size_t tc8_workspace_bytes(int64_t M, int64_t d, bool mx) {
  const size_t planes = (static_cast<size_t>(M) * d + 255) / 256 * 256;
  // per (k block, row): 2^-e of the split, or (MXFP8) the x scale chunks over
  // whole 128-row blocks; then the partial sums of squares
  const int64_t rows = mx ? (M + tc8::BM - 1) / tc8::BM * tc8::BM : M;
  const size_t facb = (static_cast<size_t>(d / tc8::BKQ) * rows * 4 + 255) / 256 * 256;
  const size_t ssqb = (static_cast<size_t>(d / tc8::BKQ) * M * 4 + 255) / 256 * 256;
  return kWsHeaderBytes + 2 * planes + facb + ssqb;
}

cudaError_t launch_tc8(const CallArgs& a) {
  using namespace tc8;
  const bool mx = a.wtype == 2;   // MXFP8
  if (a.ws_bytes < tc8_workspace_bytes(a.M, a.d, mx)) return cudaErrorInvalidValue;
  uint8_t* ws = static_cast<uint8_t*>(a.ws);
  const int M = static_cast<int>(a.M), d = static_cast<int>(a.d);
  const int Mpad = (M + BM - 1) / BM * BM;
  const size_t planes = (static_cast<size_t>(a.M) * a.d + 255) / 256 * 256;
  const size_t facb = (static_cast<size_t>(a.d / BKQ) * (mx ? Mpad : M) * 4 + 255) / 256 * 256;
  uint8_t* xhi = ws + kWsHeaderBytes;
  uint8_t* xlo = xhi + planes;
  float* fac = reinterpret_cast<float*>(xlo + planes);
  float* ssq_part = reinterpret_cast<float*>(xlo + planes + facb);

  cudaError_t e;
  if (mx) {
    const long long warps = static_cast<long long>(Mpad) * (d / BKQ);
    e = launch_pdl(xsplit_mx_rows_kernel, static_cast<unsigned>((warps + 7) / 8), 256, 0, a.stream,
                   static_cast<const __nv_bfloat16*>(a.x), M, Mpad, d, xhi, xlo, reinterpret_cast<uint8_t*>(fac),
                   ssq_part);
  } else {
    const long long warps = static_cast<long long>(M) * (d / BKQ);
    e = launch_pdl(xsplit_rows_kernel, static_cast<unsigned>((warps + 7) / 8), 256, 0, a.stream,
                   static_cast<const __nv_bfloat16*>(a.x), M, d, xhi, xlo, fac, ssq_part);
  }
  if (e != cudaSuccess) return e;

  CUtensorMap th, tl, tw;
  if (!make_tmap_2d(&th, xhi, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.M, a.d, BM, BKQ)) return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tl, xlo, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.M, a.d, BM, BKQ)) return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tw, a.Wp, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.d, a.ncols, BKQ, 128)) return cudaErrorInvalidValue;
  Params p;
  p.M = M;
  p.d = d;
  p.ncols = static_cast<int>(a.ncols);
  p.nout = static_cast<int>(a.N);
  p.num_m = (M + BM - 1) / BM;
  p.num_n = static_cast<int>((a.ncols + BN - 1) / BN);
  p.num_tiles = p.num_m * p.num_n;
  p.kblocks = d / BKQ;
  p.nblk = static_cast<int>(a.ncols / 128);
  p.eps = a.eps;
  p.inv_d = 1.0f / static_cast<float>(a.d);
  p.y = static_cast<__nv_bfloat16*>(a.y);
  p.status = reinterpret_cast<unsigned int*>(ws);
  p.budget_ns = a.budget_ns;
  p.withhold = a.withhold;
  p.scales = mx ? nullptr : a.scales;
  p.fac = mx ? nullptr : fac;
  p.ssq_part = ssq_part;
  p.wsf = mx ? reinterpret_cast<const uint8_t*>(a.scales) : nullptr;
  p.xsf = mx ? reinterpret_cast<const uint8_t*>(fac) : nullptr;
  // Whole waves of tiles over all SMs; a last partial wave that would leave
  // more than half of the SMs idle is split in k between CTA pairs instead.
  const int G = a.num_sms & ~1;
  const int W = p.num_tiles / G, R = p.num_tiles % G;
  p.split_tail = (R > 0 && 2 * R <= G && p.kblocks >= 2) ? 1 : 0;
  p.full_waves = W;
  p.tail = R;
  int grid = p.num_tiles < a.num_sms ? p.num_tiles : a.num_sms;
  if (p.split_tail) grid = W > 0 ? G : 2 * R;
  if (mx) return a.swiglu ? launch_kernel<true, true>(grid, a.stream, th, tl, tw, p)
                          : launch_kernel<false, true>(grid, a.stream, th, tl, tw, p);
  return a.swiglu ? launch_kernel<true, false>(grid, a.stream, th, tl, tw, p)
                  : launch_kernel<false, false>(grid, a.stream, th, tl, tw, p);
}

}  // namespace fn
