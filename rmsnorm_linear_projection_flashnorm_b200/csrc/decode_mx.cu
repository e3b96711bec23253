// Fused RMSNorm + projection, small-M path (M <= 64), for MXFP8 weights:
// e4m3 codes with one power-of-two (ue8m0) scale per 32 consecutive k values
// of each weight column, sm_100a.
//
// The arithmetic is FlashNorm's (FlashNorm talk summary, Proposal 2: matmul
// on raw x, the sum of squares alongside, 1/rms after; Proposal 1: the gain is
// folded into the stored weight, here quantised):
//
//   y[m, n] = r[m] * sum_k (q[k, n] 2^Ew[k/32, n]) x[m, k]
//
// The tensor cores' block-scaled MMA (tcgen05.mma kind::mxf8f6f4.block_scale,
// the Blackwell block-scaled instruction family the FlashInfer PR #5521
// analysis uses for its low-precision FC1) multiplies e4m3 operands and
// applies one power-of-two scale per 32 k values of each A row and each B
// column, read from TMEM, before it accumulates in fp32.  So one TMEM
// accumulator spans the whole k range of a segment, with no per-block pass
// over the partial sums.  The bf16 activations enter the same way as on the
// fp8 path, exactly: per row and 32-deep k block, x * 2^e (largest magnitude
// in [128, 256)) is split into hi = e4m3(x 2^e) and lo = e4m3(x 2^e - hi);
// the two parts share the scale 2^-e.  x_hi and x_lo rows are stacked as the
// 2 x MPAD rows of one B operand (each with its row's scale byte), so one MMA
// per 32-deep k step gives both parts in adjacent accumulator columns, which
// the epilogue adds: an M = 128 MMA costs about the same for any N <= 64, so
// the stacked form halves the MMA time per weight byte.  A small kernel splits
// x once per call (codes, scale bytes, and each row's sum of squares per
// 128-deep k group).
//
// The weight stream, the stream-K split over all SMs and the fix-up kernel
// for tiles whose k range spans CTAs are those of the other decode kernels
// (decode_common.cuh).
//
// Layout: 8 warps.
//   warp 0      TMA producer (weight tile, split x rows, both scale chunks)
//   warp 1      TMEM owner and MMA issuer (copies the scale chunks into TMEM)
//   warp 2      sums of squares: adds each row's per-group sums over a segment
//   warps 4-7   epilogue / fix-up partials (one thread per weight column)
#include <cmath>
#include <cstddef>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "decode_common.cuh"

namespace fn {
namespace decmx {

using dec::Params;

constexpr int BKQ = 128;                  // k rows per stage: four 32-deep scale blocks
constexpr int WQ_BOX = 128 * BKQ;         // one e4m3 box: 128 columns x 128 k rows (16 KB)
constexpr int SF_CHUNK = 512;             // 128 rows x 4 scale bytes, in the MMA's chunk layout
constexpr int NUM_THREADS = 256;
constexpr int SMEM_BUDGET = 200 * 1024;   // pipeline stages; barriers and staging come on top

template <int MPAD, int HALVES>
struct Cfg {
  static constexpr int W_BYTES = HALVES * WQ_BOX;
  static constexpr int X_BYTES = 2 * MPAD * BKQ;                      // x_hi rows, then x_lo rows
  static constexpr int SF_BYTES = (HALVES + 1) * SF_CHUNK;            // weight chunks, then the x chunk
  static constexpr int STAGE_BYTES = (W_BYTES + X_BYTES + SF_BYTES + 1023) / 1024 * 1024;
  static constexpr int STAGES_RAW = SMEM_BUDGET / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static constexpr int ACC_COLS = HALVES * 2 * MPAD;                  // one buffer: [half][hi | lo rows]
  static constexpr int SF_COLS = (HALVES + 1) * 4;                    // TMEM scale words per stage
  // two accumulator buffers (the epilogue of one segment overlaps the next
  // segment's MMAs) when they fit TMEM beside the scale words, else one
  static constexpr int NBUF = 2 * ACC_COLS + STAGES * SF_COLS <= 512 ? 2 : 1;
  static constexpr int SF_BASE = NBUF * ACC_COLS;                     // after the accumulator buffers
  static constexpr int TMEM_NEED = SF_BASE + STAGES * SF_COLS;
  static constexpr int TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64 : TMEM_NEED <= 128 ? 128
                                   : TMEM_NEED <= 256 ? 256 : 512;
};

// Workspace of the once-per-call split of x: operand slabs [group][2 MPAD][128],
// scale chunks [group][512], per-group sums of squares [group][MPAD].
inline size_t presplit_bytes(int mpad, int64_t d) {
  const size_t groups = static_cast<size_t>(d / BKQ);
  return (groups * (2 * mpad * BKQ + SF_CHUNK + mpad * 4) + 255) / 256 * 256;
}

template <int MPAD, int STAGES>
struct alignas(16) Bars {
  uint64_t full[STAGES], empty[STAGES];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t ssq_full[2], ssq_empty[2];
  uint64_t drain;
  float ssq[2][MPAD];
  alignas(16) __nv_bfloat16 ybuf[MPAD * 128];
  uint32_t tmem_base;
  int abort_flag;
  int epi_ok[2];
};

// Split x once per call: one warp per (128-deep k group, padded row); lane l
// takes k values 4l .. 4l+3, so each group of 8 lanes holds one 32-deep scale
// block.  Writes the x_hi row r and x_lo row MPAD + r of the group's operand
// slab, the row's scale byte 127 - e for each block in the group's chunk at
// both operand rows r and MPAD + r (line row mod 32, word row div 32, byte =
// block), and the row's sum of squares over the group.  Padding rows are zero
// with scale byte 127.
template <int MPAD>
__global__ void __launch_bounds__(256) mxsplit_kernel(const Params p) {
  grid_launch_dependents();     // the decode kernel may set up meanwhile
  grid_dependency_wait();       // x may have been written by the preceding kernel
  const int wg = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int kg = wg / MPAD, row = wg % MPAD;
  if (kg >= p.kblocks) return;
  const bool live = row < p.M;
  uint2 v = make_uint2(0u, 0u);
  if (live) v = *reinterpret_cast<const uint2*>(p.x + static_cast<int64_t>(row) * p.d + kg * BKQ + lane * 4);
  uint32_t amax = max(max(v.x & 0x7FFFu, (v.x >> 16) & 0x7FFFu), max(v.y & 0x7FFFu, (v.y >> 16) & 0x7FFFu));
#pragma unroll
  for (int o = 4; o >= 1; o >>= 1) amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  // amax is a bf16 bit pattern of the block's largest magnitude: exponent
  // field in bits 7..14; amax * 2^e lands in [128, 256)
  const int E = static_cast<int>(amax >> 7);
  int e = amax == 0 ? 0 : 134 - E;
  e = e > 126 ? 126 : (e < -126 ? -126 : e);
  const float sc = __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
  const uint64_t sc2 = f2_pack(sc, sc);
  uint16_t h0 = 0, l0 = 0, h1 = 0, l1 = 0;
  uint64_t ss2 = 0;
  if (live) {
    const uint64_t a = f2_pack_u(v.x << 16, v.x & 0xFFFF0000u), b = f2_pack_u(v.y << 16, v.y & 0xFFFF0000u);
    ss2 = f2_fma(b, b, f2_fma(a, a, ss2));
    split_e4m3x2(f2_mul(a, sc2), h0, l0);
    split_e4m3x2(f2_mul(b, sc2), h1, l1);
  }
  float ss = f2_lo(ss2) + f2_hi(ss2);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  uint8_t* slab = p.xhilo + static_cast<int64_t>(kg) * 2 * MPAD * BKQ;
  *reinterpret_cast<uint32_t*>(slab + row * BKQ + lane * 4) = static_cast<uint32_t>(h0) | (static_cast<uint32_t>(h1) << 16);
  *reinterpret_cast<uint32_t*>(slab + (MPAD + row) * BKQ + lane * 4) =
      static_cast<uint32_t>(l0) | (static_cast<uint32_t>(l1) << 16);
  if ((lane & 7) == 0) {
    const uint8_t sb = static_cast<uint8_t>(live ? 127 - e : 127);
    uint8_t* chunk = p.xsf + static_cast<int64_t>(kg) * SF_CHUNK + (lane >> 3);
    const int rl = MPAD + row;   // the same row's x_lo operand row
    chunk[16 * (row & 31) + 4 * (row >> 5)] = sb;
    chunk[16 * (rl & 31) + 4 * (rl >> 5)] = sb;
  }
  if (lane == 0) p.xfac[static_cast<int64_t>(kg) * MPAD + row] = live ? ss : 0.f;
}

// OUT: bf16 y, NVFP4 codes and scales (SwiGLU only), or fp32 partials (OutKind).
template <int MPAD, int HALVES, int OUT = kOutBf16>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    decode_mx_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_q,
                     const Params p) {
  static_assert(OUT != kOutNvfp4 || HALVES == 2, "NVFP4 output is a SwiGLU epilogue");
  static_assert(OUT != kOutPartial || HALVES == 1, "partial output: plain projection of the stored columns");
  using C = Cfg<MPAD, HALVES>;
  constexpr int STAGES = C::STAGES;
  using B = Bars<MPAD, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  B& bars = *reinterpret_cast<B*>(smem + STAGES * C::STAGE_BYTES);
  // stage: [e4m3 weight boxes][x_hi | x_lo rows][weight scale chunks][x scale chunk]
  auto stage_w = [&](int s) { return smem + s * C::STAGE_BYTES; };
  auto stage_x = [&](int s) { return smem + s * C::STAGE_BYTES + C::W_BYTES; };
  auto stage_sf = [&](int s) { return smem + s * C::STAGE_BYTES + C::W_BYTES + C::X_BYTES; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const long long it0 = dec::it_begin(cta, p);
  const long long it1 = dec::it_begin(cta + 1, p);
  const int ncb = p.ncols >> 7;   // 128-column blocks of the weight (scale chunks per k group)

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.empty[s], 1);       // MMA commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars.acc_full[b], 1);
      mbar_init(&bars.acc_empty[b], 128);
      mbar_init(&bars.ssq_full[b], 32);
      mbar_init(&bars.ssq_empty[b], 128);
    }
    mbar_init(&bars.drain, 1);
    bars.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmap_w);
    tma_prefetch_desc(&tmap_q);
  }
  if (warp == 1) {
    tmem_alloc(&bars.tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Before the dependency wait: an L2 prefetch of the start of this CTA's
  // weight range (the weight does not depend on the previous kernel's output,
  // and an L2 prefetch cannot return stale data).  prefetch_iters counts
  // 64-row k blocks; this kernel's groups are 128 rows deep.
  if (p.prefetch_mode == 2 && warp >= 2) {
    const long long n_it = min(static_cast<long long>(p.prefetch_iters / 2), it1 - it0);
    const int total = static_cast<int>(n_it) * BKQ * HALVES;   // 128-byte lines
    for (int i = threadIdx.x - 64; i < total; i += NUM_THREADS - 64) {
      const int chunk = i % HALVES;
      const int r = (i / HALVES) % BKQ;
      const long long it = it0 + i / (HALVES * BKQ);
      const int tile = static_cast<int>(it / p.kblocks);
      const int kg = static_cast<int>(it - static_cast<long long>(tile) * p.kblocks);
      const uint8_t* a = p.wp + (static_cast<int64_t>(kg) * BKQ + r) * p.ncols +
                         static_cast<int64_t>(tile) * 128 * HALVES + chunk * 128;
      asm volatile("prefetch.global.L2 [%0];" ::"l"(a));
    }
  }
  grid_dependency_wait();
  grid_launch_dependents();
  const uint32_t tmem_base = bars.tmem_base;
  const WaitCtl ctl{&bars.abort_flag, p.status, p.budget_ns};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t w_policy = l2_policy_evict_first();   // the weight is streamed once
      int s = 0;
      uint32_t ph = 0, issued = 0, last_ph = 0;
      for (long long it = it0; it < it1; ++it) {
        const int tile = static_cast<int>(it / p.kblocks);
        const int kg = static_cast<int>(it - static_cast<long long>(tile) * p.kblocks);
        if (!mbar_wait(&bars.empty[s], ph ^ 1, ctl, dec::kSiteProdEmpty)) break;
        mbar_arrive_expect_tx(&bars.full[s], C::W_BYTES + C::X_BYTES + (HALVES + 1) * SF_CHUNK);
#pragma unroll
        for (int h = 0; h < HALVES; ++h) {
          tma_load_2d_hint(stage_w(s) + h * WQ_BOX, &tmap_w, &bars.full[s], (tile * HALVES + h) * 128, kg * BKQ,
                           w_policy);
          bulk_load(stage_sf(s) + h * SF_CHUNK,
                    p.wsf + (static_cast<int64_t>(kg) * ncb + tile * HALVES + h) * SF_CHUNK, SF_CHUNK, &bars.full[s]);
        }
        tma_load_2d(stage_x(s), &tmap_q, &bars.full[s], 0, kg * 2 * MPAD);
        bulk_load(stage_sf(s) + HALVES * SF_CHUNK, p.xsf + static_cast<int64_t>(kg) * SF_CHUNK, SF_CHUNK,
                  &bars.full[s]);
        issued |= 1u << s;
        last_ph = (last_ph & ~(1u << s)) | (ph << s);
        if (++s == STAGES) { s = 0; ph ^= 1; }
      }
      for (int i = 0; i < STAGES; ++i)
        if (issued & (1u << i)) dec::drain_wait(&bars.full[i], (last_ph >> i) & 1u, p.budget_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int seg = 0;
      for (long long it = it0; it < it1 && ok; ++seg) {
        const int tile = static_cast<int>(it / p.kblocks);
        const int kb0 = static_cast<int>(it - static_cast<long long>(tile) * p.kblocks);
        const int kb1 = static_cast<int>(min(static_cast<long long>(p.kblocks), kb0 + (it1 - it)));
        const int b = seg % C::NBUF;
        if (!mbar_wait(&bars.acc_empty[b], ((seg / C::NBUF) & 1) ^ 1u, ctl, dec::kSiteMmaAccEmpty)) break;
        tc_fence_after();
        for (int kg = kb0; kg < kb1; ++kg) {
          if (!mbar_wait(&bars.full[s], ph, ctl, dec::kSiteMmaFull)) { ok = false; break; }
          tc_fence_after();
          // this stage's scale chunks -> its TMEM scale words (weight halves, then x)
          const uint32_t sf_t = tmem_base + C::SF_BASE + s * C::SF_COLS;
          const uint32_t sf_s = smem_u32(stage_sf(s));
#pragma unroll
          for (int h = 0; h <= HALVES; ++h) tmem_cp_32x128b_x4(sf_t + 4 * h, sdesc_plain(sf_s + h * SF_CHUNK, 128, 128));
          const uint32_t w0 = smem_u32(stage_w(s));
          const uint32_t x0 = smem_u32(stage_x(s));
#pragma unroll
          for (int kk = 0; kk < BKQ / 32; ++kk) {
            // A = q^T: 128 weight columns (one 128-byte swizzle row), MN-major, 8-row
            //     k groups 1024 B apart, so K = 32 is 4096 B.  B = the x_hi rows
            //     followed by the x_lo rows, K-major; the scale byte of this 32-deep
            //     block is byte kk of each word.
            const uint32_t idesc = idesc_mx_e4m3(128, 2 * MPAD, /*a MN-major*/ true, /*b MN-major*/ false, kk);
#pragma unroll
            for (int h = 0; h < HALVES; ++h) {
              const uint32_t d_tmem = tmem_base + (b * HALVES + h) * 2 * MPAD;
              const uint64_t adesc = sdesc_sw128(w0 + h * WQ_BOX + kk * 4096, WQ_BOX, 1024);
              const uint32_t acc = (kg != kb0 || kk != 0) ? 1u : 0u;
              umma_mx_e4m3(d_tmem, adesc, sdesc_sw128(x0 + kk * 32, 16, 1024), idesc, sf_t + 4 * h,
                           sf_t + 4 * HALVES, acc);
            }
          }
          umma_commit(&bars.empty[s]);
          if (++s == STAGES) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        umma_commit(&bars.acc_full[b]);
        it += kb1 - kb0;
      }
      umma_commit(&bars.drain);
      dec::drain_wait(&bars.drain, 0, p.budget_ns);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------------ sums of squares
    // Each row's per-group sums over the segment's k range, in k order, from
    // the values the split kernel squared; runs alongside the MMA stream.
    constexpr int RPL = MPAD > 32 ? 2 : 1;     // rows per lane
    int seg = 0;
    for (long long it = it0; it < it1; ++seg) {
      const int tile = static_cast<int>(it / p.kblocks);
      const int kb0 = static_cast<int>(it - static_cast<long long>(tile) * p.kblocks);
      const int kb1 = static_cast<int>(min(static_cast<long long>(p.kblocks), kb0 + (it1 - it)));
      it += kb1 - kb0;
      float acc[RPL];
#pragma unroll
      for (int j = 0; j < RPL; ++j) {
        const int row = lane + 32 * j;
        acc[j] = 0.f;
        if (row < MPAD) {
          int kg = kb0;
          for (; kg + 4 <= kb1; kg += 4) {      // four independent loads in flight, added in order
            const float a0 = p.xfac[static_cast<int64_t>(kg) * MPAD + row];
            const float a1 = p.xfac[static_cast<int64_t>(kg + 1) * MPAD + row];
            const float a2 = p.xfac[static_cast<int64_t>(kg + 2) * MPAD + row];
            const float a3 = p.xfac[static_cast<int64_t>(kg + 3) * MPAD + row];
            acc[j] = (((acc[j] + a0) + a1) + a2) + a3;
          }
          for (; kg < kb1; ++kg) acc[j] += p.xfac[static_cast<int64_t>(kg) * MPAD + row];
        }
      }
      const int b = seg & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars.ssq_empty[b], ((seg >> 1) & 1) ^ 1u, ctl,
                                              dec::kSiteRedSsqEmpty)))
        break;
#pragma unroll
      for (int j = 0; j < RPL; ++j)
        if (lane + 32 * j < MPAD) bars.ssq[b][lane + 32 * j] = acc[j];
      if (!(p.withhold && seg == 0)) mbar_arrive(&bars.ssq_full[b]);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue / fix-up partials
    const int q = warp & 3;
    const int n = q * 32 + lane;                  // weight column within the 128-wide half
    const int et = threadIdx.x - 128;             // 0..127
    int seg = 0;
    for (long long it = it0; it < it1; ++seg) {
      const int tile = static_cast<int>(it / p.kblocks);
      const int kb0 = static_cast<int>(it - static_cast<long long>(tile) * p.kblocks);
      const int kb1 = static_cast<int>(min(static_cast<long long>(p.kblocks), kb0 + (it1 - it)));
      it += kb1 - kb0;
      const int ab = seg % C::NBUF;               // accumulator buffer
      const uint32_t aph = (seg / C::NBUF) & 1;
      const int b = seg & 1;                      // sums-of-squares buffer
      const uint32_t sph = (seg >> 1) & 1;
      // One thread waits and the whole epilogue group follows its decision, so
      // the group never splits at the named barriers or the .sync.aligned loads.
      if (et == 0) {
        bool ok = mbar_wait(&bars.acc_full[ab], aph, ctl, dec::kSiteEpiAccFull);
        ok = ok && mbar_wait(&bars.ssq_full[b], sph, ctl, dec::kSiteEpiSsqFull);
        bars.epi_ok[seg & 1] = ok ? 1 : 0;
      }
      named_bar_sync(1, 128);
      if (!bars.epi_ok[seg & 1]) break;
      tc_fence_after();
      // each half's x_hi columns plus its x_lo columns, 16 rows at a time
      float acc[HALVES][MPAD];
#pragma unroll
      for (int h = 0; h < HALVES; ++h) {
        const uint32_t ta = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + (ab * HALVES + h) * 2 * MPAD;
#pragma unroll
        for (int m0 = 0; m0 < MPAD; m0 += 16) {
          uint32_t hv[16], lv[16];
          tmem_ld16(ta + m0, hv);
          tmem_ld16(ta + MPAD + m0, lv);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) acc[h][m0 + j] = __uint_as_float(hv[j]) + __uint_as_float(lv[j]);
        }
      }
      tc_fence_before();
      mbar_arrive(&bars.acc_empty[ab]);
      // A row holding a non-finite activation in this k range has a non-finite
      // sum of squares; its (saturated) products become NaN, as they would in
      // a bf16 matmul.
#pragma unroll
      for (int m = 0; m < MPAD; ++m) {
        if (!isfinite(bars.ssq[b][m])) {
#pragma unroll
          for (int h = 0; h < HALVES; ++h) acc[h][m] = __int_as_float(0x7fc00000);
        }
      }
      const bool whole = (kb0 == 0 && kb1 == p.kblocks);
      if (whole && OUT == kOutPartial) {
        // the tile's fp32 accumulators and (tile 0) the sums of squares, not post-scaled
#pragma unroll
        for (int m = 0; m < MPAD; ++m) {
          if (m >= p.M) break;
          p.part_out[static_cast<int64_t>(m) * p.ncols + tile * 128 + n] = acc[0][m];
        }
        if (tile == 0 && et < p.M) p.part_out[static_cast<int64_t>(p.M) * p.ncols + et] = bars.ssq[b][et];
        mbar_arrive(&bars.ssq_empty[b]);
        continue;
      }
      if (whole) {
        uint8_t* qbuf = reinterpret_cast<uint8_t*>(bars.ybuf);   // NVFP4 staging
        const float gs = OUT == kOutNvfp4 ? __ldg(p.gscale) : 0.f;
#pragma unroll
        for (int m = 0; m < MPAD; ++m) {
          if (m >= p.M) break;
          const float r = inv_rms(bars.ssq[b][m], p.inv_d, p.eps);
          float v;
          if (HALVES == 2) v = silu_f32(acc[0][m] * r) * (acc[HALVES - 1][m] * r);
          else v = acc[0][m] * r;
          if constexpr (OUT == kOutNvfp4) dec::stage_fp4(qbuf, MPAD, m, n, v, gs);
          else bars.ybuf[m * 128 + n] = __float2bfloat16_rn(v);
        }
        mbar_arrive(&bars.ssq_empty[b]);
        named_bar_sync(1, 128);
        if constexpr (OUT == kOutNvfp4) dec::store_tile_fp4(qbuf, MPAD, p, tile, et, 128);
        else dec::store_tile_rows(bars.ybuf, p, tile, et, 128);
        continue;
      }
      // Split tile: this CTA's partial for the fix-up kernel, in the slot
      // layout float4 [half][row / 4][column] (rows < M only), then the MPAD
      // partial sums of squares.
      const int Q = (p.M + 3) >> 2;
      const int slot = cta * 2 + (seg == 0 ? 0 : 1);
      float* part = p.part + static_cast<int64_t>(slot) * dec::slot_floats<MPAD, HALVES>();
      float4* part4 = reinterpret_cast<float4*>(part);
#pragma unroll
      for (int h = 0; h < HALVES; ++h)
#pragma unroll
        for (int q4 = 0; q4 < MPAD / 4; ++q4)
          if (q4 < Q)
            __stcg(part4 + (h * (MPAD / 4) + q4) * 128 + n,
                   make_float4(acc[h][4 * q4], acc[h][4 * q4 + 1], acc[h][4 * q4 + 2], acc[h][4 * q4 + 3]));
      if (et < MPAD) __stcg(part + HALVES * MPAD * 128 + et, bars.ssq[b][et]);
      mbar_arrive(&bars.ssq_empty[b]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

template <int MPAD, int HALVES>
constexpr size_t smem_bytes() {
  using C = Cfg<MPAD, HALVES>;
  return 1024 + C::STAGES * C::STAGE_BYTES + sizeof(Bars<MPAD, C::STAGES>);
}

static_assert(smem_bytes<64, 2>() <= 227 * 1024 && smem_bytes<64, 1>() <= 227 * 1024 &&
                  smem_bytes<16, 2>() <= 227 * 1024 && smem_bytes<32, 2>() <= 227 * 1024,
              "shared memory per CTA");
static_assert(Cfg<64, 2>::STAGES >= 2, "pipeline needs two stages");
static_assert(Cfg<64, 2>::TMEM_NEED <= 512 && Cfg<16, 1>::TMEM_NEED <= 512, "TMEM columns");
using BarsLarge = Bars<64, Cfg<64, 2>::STAGES>;
static_assert(offsetof(BarsLarge, ybuf) % 16 == 0, "ybuf must be 16-byte aligned");

template <int MPAD, int HALVES, int OUT = kOutBf16>
cudaError_t launch_impl(const CallArgs& a) {
  using C = Cfg<MPAD, HALVES>;
  const size_t part_bytes = dec::workspace_bytes<MPAD, HALVES>(a.d, a.ncols, a.num_sms);
  if (a.ws_bytes < part_bytes + presplit_bytes(MPAD, a.d)) return cudaErrorInvalidValue;
  Params p;
  p.M = static_cast<int>(a.M);
  p.d = static_cast<int>(a.d);
  p.ncols = static_cast<int>(a.ncols);
  p.nout = static_cast<int>(a.N);
  p.kblocks = static_cast<int>(a.d / BKQ);
  p.tiles = static_cast<int>(a.ncols / (128 * HALVES));
  p.total = static_cast<long long>(p.tiles) * p.kblocks;
  p.grid = static_cast<int>(p.total < a.num_sms ? p.total : a.num_sms);
  p.eps = a.eps;
  p.inv_d = 1.0f / static_cast<float>(a.d);
  p.y = static_cast<__nv_bfloat16*>(a.y);
  uint8_t* ws = static_cast<uint8_t*>(a.ws);
  p.status = reinterpret_cast<unsigned int*>(ws);
  p.part = reinterpret_cast<float*>(ws + kWsHeaderBytes);
  p.budget_ns = a.budget_ns;
  p.withhold = a.withhold;
  p.wp = static_cast<const uint8_t*>(a.Wp);
  p.prefetch_iters = a.prefetch_iters;
  p.prefetch_mode = a.prefetch_mode;
  p.scales = nullptr;
  p.cluster = 1;
  p.narrow = dec::partition_is_narrow(p.total, p.grid) ? 1 : 0;
  p.x = static_cast<const __nv_bfloat16*>(a.x);
  // after the partial slots: operand slabs, scale chunks, per-group sums of squares
  p.xhilo = ws + part_bytes;
  p.xsf = p.xhilo + static_cast<size_t>(p.kblocks) * 2 * MPAD * BKQ;
  p.xfac = reinterpret_cast<float*>(p.xsf + static_cast<size_t>(p.kblocks) * SF_CHUNK);
  p.yq = static_cast<uint8_t*>(a.yq);
  p.ysf = static_cast<uint8_t*>(a.ysf);
  p.sf_chunked = a.sf_chunked;
  p.gscale = a.gscale;
  p.part_out = a.part_out;
  p.wsf = reinterpret_cast<const uint8_t*>(a.scales);
  CUtensorMap tw, tq;
  // e4m3 codes as bytes: 128 columns (one 128-byte swizzle row) x 128 k rows per box
  if (!make_tmap_2d(&tw, a.Wp, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.d, a.ncols, BKQ, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tq, p.xhilo, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(p.kblocks) * 2 * MPAD, BKQ,
                    2 * MPAD, BKQ))
    return cudaErrorInvalidValue;
  constexpr size_t SMEM = smem_bytes<MPAD, HALVES>();
  cudaError_t e = ensure_smem_limit<decode_mx_kernel<MPAD, HALVES, OUT>>(static_cast<int>(SMEM));
  if (e != cudaSuccess) return e;
  const int warps = p.kblocks * MPAD;
  e = launch_pdl(mxsplit_kernel<MPAD>, static_cast<unsigned>((warps + 7) / 8), 256, 0, a.stream, p);
  if (e != cudaSuccess) return e;
  e = launch_pdl(decode_mx_kernel<MPAD, HALVES, OUT>, p.grid, NUM_THREADS, SMEM, a.stream, tw, tq, p);
  if (e != cudaSuccess) return e;
  if (!dec::any_split_tile(p.grid, p.total, p.kblocks)) return cudaSuccess;
  return dec::launch_fixup<MPAD, HALVES, OUT>(p, a.stream);
}

}  // namespace decmx

size_t decode_mx_presplit_bytes(int64_t M, int64_t d) { return decmx::presplit_bytes(decode_mpad(M), d); }

cudaError_t launch_decode_mx(const CallArgs& a, int mpad) {
  if (a.part_out) {   // partial output: a plain projection of the stored columns
    if (mpad == 16) return decmx::launch_impl<16, 1, kOutPartial>(a);
    if (mpad == 32) return decmx::launch_impl<32, 1, kOutPartial>(a);
    return decmx::launch_impl<64, 1, kOutPartial>(a);
  }
  if (a.yq) {   // NVFP4 output (SwiGLU only)
    if (mpad == 16) return decmx::launch_impl<16, 2, kOutNvfp4>(a);
    if (mpad == 32) return decmx::launch_impl<32, 2, kOutNvfp4>(a);
    return decmx::launch_impl<64, 2, kOutNvfp4>(a);
  }
  if (mpad == 16) return a.swiglu ? decmx::launch_impl<16, 2>(a) : decmx::launch_impl<16, 1>(a);
  if (mpad == 32) return a.swiglu ? decmx::launch_impl<32, 2>(a) : decmx::launch_impl<32, 1>(a);
  return a.swiglu ? decmx::launch_impl<64, 2>(a) : decmx::launch_impl<64, 1>(a);
}

}  // namespace fn
