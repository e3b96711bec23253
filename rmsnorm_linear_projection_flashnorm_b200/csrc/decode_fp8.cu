// Fused RMSNorm + projection, small-M path (M <= 64), for fp8 e4m3 weights
// with an fp32 scale per 128 x 128 block, sm_100a.
//
// The arithmetic is FlashNorm's (FlashNorm talk summary, Proposal 2: the
// matmul runs on raw x, the sum of squares is reduced alongside, 1/rms is
// applied after; the folded weight may be quantised, Proposal 1):
//
//   y[m, n] = r[m] * sum_b s[b, n] * sum_{k in block b} q[k, n] x[m, k]
//
// At M <= 64 the weight stream is the whole cost, so the weight stays in its
// stored 8-bit form all the way into the tensor cores: TMA copies the e4m3
// codes q into shared memory with the 128-byte swizzle, and they are the A
// operand (MN-major) of tcgen05.mma kind::f8f6f4 as they are.  The bf16
// activations are the ones converted, and exactly: per activation row and
// 128-deep k block, x is scaled by a power of two 2^e that puts its largest
// magnitude in [128, 256), and each scaled value a is split into
// hi = e4m3(a) and lo = e4m3(a - hi), with a == hi + lo for every |a| >= 1/4
// (a bf16 value has 8 significant bits, hi keeps the top 4 and lo the rest).
// Elements below 1/4, under 2^-9 of the block's largest, are off by at most
// 2^-10 in the scaled units.  x_hi and x_lo are stacked as the 2 x MPAD
// columns of one B operand, so one MMA per k step gives both halves of the
// split; each k block has its own TMEM buffer, whose partial sums are exact
// products in fp32.  Scaler warps read each block's buffer back, add the hi
// and lo columns, multiply by s[b, n] * 2^-e and add the result to fp32
// running sums in registers.  (Small-N tcgen05.mma instructions cost nearly
// as much as large ones, so the stacking halves the tensor-core time per
// weight byte.)  This converts
// MPAD x 128 activations per k block instead of 128 x 128 (or 128 x 256)
// weight codes: 8 to 64 times fewer conversions (Marlin explainer, section
// 4: the conversion must hide under the memory stream).
//
// The work split is the stream-K partition of decode.cu, and tiles whose k
// range spans CTAs are finished by the shared fix-up kernel.
//
// With 17 to 64 activation rows every CTA would split the same x blocks again
// for each column tile it visits, and the conversion, a short dependent chain
// per element, becomes the bottleneck.  There a small kernel splits x once per
// call into the workspace (the same codes and scales, and each row's sum of
// squares per k block), and the main kernel stages those operand rows with TMA
// beside the weight; its converter warps then only add up each row's sums of
// squares over the k blocks of a segment, alongside the MMAs.
//
// Layout:
//   warp 0        TMA producer
//   warp 1        TMEM owner and MMA issuer
//   warps 2-5     activation converters (also reduce the sums of squares)
//   warps 6-9/13  scalers and epilogue (one thread per weight column and a
//                 half or all of the activation rows)
#include <cstddef>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "decode_common.cuh"

namespace fn {
namespace dec8 {

using dec::Params;

constexpr int BKQ = 128;                 // k rows per stage: one weight-scale block
constexpr int WQ_BOX = 128 * BKQ;        // one e4m3 box: 128 columns x 128 k rows (16 KB)
constexpr int CONV_THREADS = 128;        // warps 2-5
constexpr int FIRST_SCALER = 64 + CONV_THREADS;
constexpr int SMEM_BUDGET = 200 * 1024;  // pipeline stages; barriers and staging come on top
constexpr int XR = 4;                    // ring of per-row activation scales (converters -> scalers)

// Workspace for splitting x once per call: x_hi / x_lo slabs, then 2^-e and
// the sum of squares per (k block, row).
inline size_t presplit_bytes(int mpad, int64_t d) {
  return (static_cast<size_t>(2 * mpad) * d + static_cast<size_t>(2 * mpad) * (d / BKQ) * 4 + 255) / 256 * 256;
}

template <int MPAD, int HALVES, bool PRE = false>
struct Cfg {
  static constexpr int SCALE_WARPS = HALVES * MPAD >= 64 ? 8 : 4;
  static constexpr int SCALE_THREADS = 32 * SCALE_WARPS;
  static constexpr int THREADS = FIRST_SCALER + SCALE_THREADS;
  static constexpr int RPS = MPAD / (SCALE_WARPS / 4);    // activation rows per scaler thread
  static constexpr int W_BYTES = HALVES * WQ_BOX;          // e4m3 weight: 16 or 32 KB
  static constexpr int XB_BOX = MPAD * 128;                // bf16 x box: MPAD rows x 64 columns
  static constexpr int XB_BYTES = PRE ? 0 : 2 * XB_BOX;    // x split once per call: no bf16 x tile
  static constexpr int XQ_BYTES = MPAD * BKQ;              // e4m3 x_hi (or x_lo): MPAD rows x 128 B
  static constexpr int STAGE_BYTES = W_BYTES + XB_BYTES + 2 * XQ_BYTES;   // multiple of 1024
  static constexpr int STAGES_RAW = SMEM_BUDGET / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static constexpr int ACC_COLS = HALVES * 2 * MPAD;       // one k-block buffer: hi and lo columns
  static constexpr int TMEM_COLS = 2 * ACC_COLS;           // two k-block buffers: 64..512
  static constexpr int TPR = CONV_THREADS / MPAD;          // converter threads per row: 8, 4 or 2
  static constexpr int EPT = BKQ / TPR;                    // k elements per converter thread
};

template <int MPAD, int STAGES>
struct alignas(16) Bars {
  uint64_t full[STAGES], empty[STAGES], conv[STAGES];
  uint64_t accf[2], acce[2];           // per-k-block TMEM buffer: written by MMA / read by scalers
  uint64_t xsf[XR], xse[XR];           // activation scales: written / read
  uint64_t ssq_full[2], ssq_empty[2];  // per-segment sums of squares
  uint64_t drain;
  float xs[XR][MPAD];                  // 2^-e per activation row of one k block (NaN: non-finite block)
  float ssq[2][MPAD];
  alignas(16) __nv_bfloat16 ybuf[MPAD * 128];
  uint32_t tmem_base;
  int abort_flag;
  int seg_ok;
  int warp_ok[8];
};

// One activation row's share of a k block: this thread's EPT bf16 values,
// read from the two 64-column x boxes (128-byte swizzle).  First pass: the
// row's largest magnitude over its TPR threads, on the raw bit patterns
// (|x| orders like its bits; inf and NaN sort above every finite value).
// Second pass: the exact e4m3 split of x * 2^e into the x_hi / x_lo operand
// rows (K-major, 128-byte swizzle: 16-byte chunk j of row m at chunk
// j ^ (m & 7)) and the row's sum of squares.  Returns the sum of squares;
// *factor receives 2^-e (NaN when the block holds a non-finite value, so the
// row's outputs become NaN as the bf16 path's would).
template <int MPAD, int TPR, int EPT>
__device__ __forceinline__ float convert_row_block(const uint8_t* xb, uint8_t* xh, uint8_t* xl, int row, int sub,
                                                   bool live, float* factor) {
  constexpr int NCH = EPT / 8;          // 16-byte bf16 chunks of this thread
  // chunk i of this thread: k values 8 (sub * NCH + i) .. +7, in box g >> 3
  auto chunk = [&](int i) {
    const int g = sub * NCH + i;
    return *reinterpret_cast<const uint4*>(xb + (g >> 3) * (MPAD * 128) + row * 128 + (((g & 7) ^ (row & 7)) << 4));
  };
  uint32_t amax2 = 0;                   // |x| bit patterns, two bf16 lanes
  if (live) {
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const uint4 v = chunk(i);
      amax2 = __vmaxu2(amax2, v.x & 0x7FFF7FFFu);
      amax2 = __vmaxu2(amax2, v.y & 0x7FFF7FFFu);
      amax2 = __vmaxu2(amax2, v.z & 0x7FFF7FFFu);
      amax2 = __vmaxu2(amax2, v.w & 0x7FFF7FFFu);
    }
  }
  uint32_t amax = max(amax2 & 0xFFFFu, amax2 >> 16);
#pragma unroll
  for (int o = 1; o < TPR; o <<= 1) amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  // amax is a bf16 bit pattern: exponent field in bits 7..14 (255: inf / NaN)
  const int E = static_cast<int>(amax >> 7);
  int e = amax == 0 ? 0 : 134 - E;      // amax * 2^e in [128, 256)
  e = e > 126 ? 126 : (e < -126 ? -126 : e);
  const float sc = __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
  const uint64_t sc2 = f2_pack(sc, sc);
  *factor = E == 255 ? __int_as_float(0x7fc00000) : __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
  uint64_t ss2 = 0;                     // two partial sums of squares (+0.0f, +0.0f)
#pragma unroll
  for (int oc = 0; oc < EPT / 16; ++oc) {
    uint4 hv = make_uint4(0u, 0u, 0u, 0u), lv = hv;   // padding rows (TMA filled zeros) stay zero
    if (live) {
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const uint4 v = chunk(2 * oc + c);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          uint16_t h[2], l[2];
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const uint32_t x2 = w[2 * q + t];
            const uint64_t xf = f2_pack_u(x2 << 16, x2 & 0xFFFF0000u);   // two bf16 -> fp32 (exact)
            ss2 = f2_fma(xf, xf, ss2);
            split_e4m3x2(f2_mul(xf, sc2), h[t], l[t]);
          }
          hw[2 * c + q] = static_cast<uint32_t>(h[0]) | (static_cast<uint32_t>(h[1]) << 16);
          lw[2 * c + q] = static_cast<uint32_t>(l[0]) | (static_cast<uint32_t>(l[1]) << 16);
        }
      }
      hv = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      lv = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
    const int j = sub * (EPT / 16) + oc;   // 16-byte e4m3 chunk of the 128-byte operand row
    const int off = row * 128 + ((j ^ (row & 7)) << 4);
    *reinterpret_cast<uint4*>(xh + off) = hv;
    *reinterpret_cast<uint4*>(xl + off) = lv;
  }
  float ss = f2_lo(ss2) + f2_hi(ss2);
#pragma unroll
  for (int o = 1; o < TPR; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  return ss;
}

// Split x once per call (the 17..64-row case): one warp per (128-deep k block,
// padded row); lane l takes k values 4l .. 4l+3.  Codes and scale factors are
// those convert_row_block computes, written as the operand rows the decode
// kernel stages: x_hi at row r, x_lo at row MPAD + r of the k block's
// [2 MPAD][128-byte] slab; padding rows are zero.
template <int MPAD>
__global__ void __launch_bounds__(256) xsplit_kernel(const Params p) {
  grid_launch_dependents();     // the decode kernel may set up meanwhile
  grid_dependency_wait();       // x may have been written by the preceding kernel
  const int wg = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int kb = wg / MPAD, row = wg % MPAD;
  if (kb >= p.kblocks) return;
  const bool live = row < p.M;
  uint2 v = make_uint2(0u, 0u);
  if (live) v = *reinterpret_cast<const uint2*>(p.x + static_cast<int64_t>(row) * p.d + kb * BKQ + lane * 4);
  uint32_t amax = max(max(v.x & 0x7FFFu, (v.x >> 16) & 0x7FFFu), max(v.y & 0x7FFFu, (v.y >> 16) & 0x7FFFu));
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, o));
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
  uint8_t* slab = p.xhilo + static_cast<int64_t>(kb) * 2 * MPAD * 128;
  *reinterpret_cast<uint32_t*>(slab + row * 128 + lane * 4) = static_cast<uint32_t>(h0) | (static_cast<uint32_t>(h1) << 16);
  *reinterpret_cast<uint32_t*>(slab + (MPAD + row) * 128 + lane * 4) =
      static_cast<uint32_t>(l0) | (static_cast<uint32_t>(l1) << 16);
  if (lane == 0) {
    p.xfac[kb * MPAD + row] = !live ? 0.f
                              : (E == 255 ? __int_as_float(0x7fc00000)
                                          : __uint_as_float(static_cast<uint32_t>(127 - e) << 23));
    p.xfac[(p.kblocks + kb) * MPAD + row] = ss;   // the block's sum of squares
  }
}

// OUT: bf16 y, NVFP4 codes and scales (SwiGLU only), or fp32 partials (OutKind).
template <int MPAD, int HALVES, bool PRESPLIT, int OUT = kOutBf16>
__global__ void __launch_bounds__(Cfg<MPAD, HALVES, PRESPLIT>::THREADS, 1)
    decode_fp8_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                      const __grid_constant__ CUtensorMap tmap_q, const Params p) {
  static_assert(OUT != kOutNvfp4 || HALVES == 2, "NVFP4 output is a SwiGLU epilogue");
  static_assert(OUT != kOutPartial || HALVES == 1, "partial output: plain projection of the stored columns");
  using C = Cfg<MPAD, HALVES, PRESPLIT>;
  constexpr int STAGES = C::STAGES;
  using B = Bars<MPAD, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  B& bars = *reinterpret_cast<B*>(smem + STAGES * C::STAGE_BYTES);
  // stage: [e4m3 weight boxes][bf16 x boxes][x_hi][x_lo], each on a 1024-byte multiple
  auto stage_w = [&](int s) { return smem + s * C::STAGE_BYTES; };
  auto stage_xb = [&](int s) { return smem + s * C::STAGE_BYTES + C::W_BYTES; };
  auto stage_xh = [&](int s) { return smem + s * C::STAGE_BYTES + C::W_BYTES + C::XB_BYTES; };
  auto stage_xl = [&](int s) { return smem + s * C::STAGE_BYTES + C::W_BYTES + C::XB_BYTES + C::XQ_BYTES; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const long long it0 = dec::it_begin(cta, p);
  const long long it1 = dec::it_begin(cta + 1, p);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.empty[s], 1);             // MMA commit
      mbar_init(&bars.conv[s], CONV_THREADS);   // every converter thread
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars.accf[b], 1);
      mbar_init(&bars.acce[b], C::SCALE_THREADS);
      mbar_init(&bars.ssq_full[b], CONV_THREADS);
      mbar_init(&bars.ssq_empty[b], 1);
    }
    for (int r = 0; r < XR; ++r) {
      mbar_init(&bars.xsf[r], CONV_THREADS);
      mbar_init(&bars.xse[r], C::SCALE_THREADS);
    }
    mbar_init(&bars.drain, 1);
    bars.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmap_x);
    if (PRESPLIT) tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_w);
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
  // 64-row k blocks; this kernel's blocks are 128 rows deep.
  if (p.prefetch_mode == 2 && warp >= 2) {
    const long long n_it = min(static_cast<long long>(p.prefetch_iters / 2), it1 - it0);
    const int total = static_cast<int>(n_it) * BKQ * HALVES;   // 128-byte lines
    for (int i = threadIdx.x - 64; i < total; i += C::THREADS - 64) {
      const int chunk = i % HALVES;
      const int r = (i / HALVES) % BKQ;
      const long long it = it0 + i / (HALVES * BKQ);
      const int tile = static_cast<int>(it / p.kblocks);
      const int kb = static_cast<int>(it - static_cast<long long>(tile) * p.kblocks);
      const uint8_t* a = p.wp + (static_cast<int64_t>(kb) * BKQ + r) * p.ncols +
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
        const int kb = static_cast<int>(it - static_cast<long long>(tile) * p.kblocks);
        if (!mbar_wait(&bars.empty[s], ph ^ 1, ctl, dec::kSiteProdEmpty)) break;
        mbar_arrive_expect_tx(&bars.full[s], C::XB_BYTES + C::W_BYTES + (PRESPLIT ? 2 * C::XQ_BYTES : 0));
        if (!PRESPLIT) {
          tma_load_2d(stage_xb(s), &tmap_x, &bars.full[s], kb * BKQ, 0);
          tma_load_2d(stage_xb(s) + C::XB_BOX, &tmap_x, &bars.full[s], kb * BKQ + 64, 0);
        }
        // pre-split operand rows: x_hi and x_lo of this k block, one box
        if (PRESPLIT) tma_load_2d(stage_xh(s), &tmap_q, &bars.full[s], 0, kb * 2 * MPAD);
#pragma unroll
        for (int h = 0; h < HALVES; ++h)
          tma_load_2d_hint(stage_w(s) + h * WQ_BOX, &tmap_w, &bars.full[s], (tile * HALVES + h) * 128, kb * BKQ,
                           w_policy);
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
      // A = q^T: 128 weight columns (one 128-byte swizzle row), MN-major; 8-row
      //     k groups 1024 B apart, so K = 32 is 4096 B.
      // B = [x_hi; x_lo]: 2 x MPAD rows of 128 e4m3 k values, K-major (x_lo's
      //     rows follow x_hi's, so both are one operand of N = 2 x MPAD).
      constexpr uint32_t IDESC = idesc_e4m3_f32(128, 2 * MPAD, /*a MN-major*/ true, /*b MN-major*/ false);
      int s = 0;
      uint32_t ph = 0;
      long long gi = 0;
      for (long long it = it0; it < it1; ++it, ++gi) {
        const int ab = static_cast<int>(gi & 1);
        bool ok = mbar_wait(&bars.acce[ab], static_cast<uint32_t>((gi >> 1) & 1) ^ 1u, ctl, dec::kSiteMmaAccEmpty);
        ok = ok && mbar_wait(&bars.full[s], ph, ctl, dec::kSiteMmaFull);
        ok = ok && mbar_wait(&bars.conv[s], ph, ctl, dec::kSiteMmaConv);
        if (!ok) break;
        tc_fence_after();
        const uint32_t w0 = smem_u32(stage_w(s));
        const uint32_t xh = smem_u32(stage_xh(s));
#pragma unroll
        for (int h = 0; h < HALVES; ++h) {
          const uint32_t d_tmem = tmem_base + (ab * HALVES + h) * 2 * MPAD;
#pragma unroll
          for (int kk = 0; kk < BKQ / 32; ++kk) {
            const uint64_t adesc = sdesc_sw128(w0 + h * WQ_BOX + kk * 4096, WQ_BOX, 1024);
            umma_e4m3(d_tmem, adesc, sdesc_sw128(xh + kk * 32, 16, 1024), IDESC, kk != 0 ? 1u : 0u);
          }
        }
        umma_commit(&bars.empty[s]);
        umma_commit(&bars.accf[ab]);
        if (++s == STAGES) { s = 0; ph ^= 1; }
      }
      umma_commit(&bars.drain);
      dec::drain_wait(&bars.drain, 0, p.budget_ns);
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------------ activation converters
    const int ct = threadIdx.x - 64;
    const int row = ct / C::TPR, sub = ct % C::TPR;
    const bool live = row < p.M;
    // x split once per call: this row's scale factor and sum of squares for
    // iteration `it`, loaded three iterations ahead
    auto load_pre = [&](long long it, float& f, float& ss) {
      f = ss = 0.f;
      if (PRESPLIT && it < it1) {
        const int kb = static_cast<int>(it % p.kblocks);
        f = p.xfac[kb * MPAD + row];
        ss = p.xfac[(p.kblocks + kb) * MPAD + row];
      }
    };
    float pre_f[3] = {0.f, 0.f, 0.f}, pre_ss[3] = {0.f, 0.f, 0.f};
    if (PRESPLIT && sub == 0) {
      load_pre(it0, pre_f[0], pre_ss[0]);
      load_pre(it0 + 1, pre_f[1], pre_ss[1]);
      load_pre(it0 + 2, pre_f[2], pre_ss[2]);
    }
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    int seg = 0;
    long long gi = 0;
    for (long long it = it0; it < it1 && ok; ++seg) {
      const int tile = static_cast<int>(it / p.kblocks);
      const int kb0 = static_cast<int>(it - static_cast<long long>(tile) * p.kblocks);
      const int kb1 = static_cast<int>(min(static_cast<long long>(p.kblocks), kb0 + (it1 - it)));
      float rss = 0.f;
      for (int kb = kb0; kb < kb1; ++kb, ++gi) {
        const int xr = static_cast<int>(gi & (XR - 1));
        bool ready = mbar_wait(&bars.full[s], ph, ctl, dec::kSiteConvFull);
        ready = ready && mbar_wait(&bars.xse[xr], static_cast<uint32_t>((gi / XR) & 1) ^ 1u, ctl,
                                   dec::kSiteConvScaleEmpty);
        if (!__all_sync(0xffffffffu, ready)) { ok = false; break; }
        if (PRESPLIT) {
          if (sub == 0) {
            rss += pre_ss[0];
            bars.xs[xr][row] = pre_f[0];
            pre_f[0] = pre_f[1]; pre_ss[0] = pre_ss[1];
            pre_f[1] = pre_f[2]; pre_ss[1] = pre_ss[2];
            load_pre(it0 + gi + 3, pre_f[2], pre_ss[2]);
          }
        } else {
          float factor;
          rss += convert_row_block<MPAD, C::TPR, C::EPT>(stage_xb(s), stage_xh(s), stage_xl(s), row, sub, live,
                                                         &factor);
          if (sub == 0) bars.xs[xr][row] = factor;
          fence_proxy_async_smem();   // generic-proxy operand writes -> visible to tcgen05.mma
        }
        mbar_arrive(&bars.conv[s]);
        mbar_arrive(&bars.xsf[xr]);
        if (++s == STAGES) { s = 0; ph ^= 1; }
      }
      if (!ok) break;
      const int b = seg & 1;
      const uint32_t sph = (seg >> 1) & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars.ssq_empty[b], sph ^ 1, ctl, dec::kSiteRedSsqEmpty))) break;
      if (sub == 0) bars.ssq[b][row] = rss;
      if (!(p.withhold && seg == 0)) mbar_arrive(&bars.ssq_full[b]);
      it += kb1 - kb0;
    }
  } else {
    // ------------------------------------------------------------ scalers / epilogue
    constexpr int RPS = C::RPS;
    constexpr int CH = HALVES * RPS >= 64 ? 8 : 16;   // TMEM columns per load
    const int st = threadIdx.x - FIRST_SCALER;        // 0 .. SCALE_THREADS-1
    const int wq = warp & 3;                          // TMEM lane quarter this warp may read
    const int n = wq * 32 + lane;                     // weight column within a 128-column half
    const int m0 = (st >> 7) * RPS;                   // first activation row of this thread
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    const int scale_cols = p.ncols >> 7;
    // Block scales of iteration `it`, loaded three iterations ahead so that
    // the global-load latency never sits between two k blocks.
    auto load_scales = [&](long long it, float (&sv)[HALVES]) {
      const int t = static_cast<int>(it / p.kblocks);
      const int k = static_cast<int>(it - static_cast<long long>(t) * p.kblocks);
#pragma unroll
      for (int h = 0; h < HALVES; ++h)
        sv[h] = it < it1 ? __ldg(p.scales + static_cast<int64_t>(k) * scale_cols + t * HALVES + h) : 0.f;
    };
    float s0[HALVES], s1[HALVES], s2[HALVES];
    load_scales(it0, s0);
    load_scales(it0 + 1, s1);
    load_scales(it0 + 2, s2);
    bool ok = true;
    long long gi = 0;
    int seg = 0;
    for (long long it = it0; it < it1; ++seg) {
      const int tile = static_cast<int>(it / p.kblocks);
      const int kb0 = static_cast<int>(it - static_cast<long long>(tile) * p.kblocks);
      const int kb1 = static_cast<int>(min(static_cast<long long>(p.kblocks), kb0 + (it1 - it)));
      it += kb1 - kb0;
      uint64_t acc[HALVES][RPS / 2];   // fp32 running sums, rows in pairs
#pragma unroll
      for (int h = 0; h < HALVES; ++h)
#pragma unroll
        for (int j = 0; j < RPS / 2; ++j) acc[h][j] = 0;
      for (int kb = kb0; kb < kb1; ++kb, ++gi) {
        const int ab = static_cast<int>(gi & 1);
        const int xr = static_cast<int>(gi & (XR - 1));
        float sw[HALVES];
#pragma unroll
        for (int h = 0; h < HALVES; ++h) {
          sw[h] = s0[h];
          s0[h] = s1[h];
          s1[h] = s2[h];
        }
        load_scales(it0 + gi + 3, s2);
        if (ok) {
          bool ready = mbar_wait(&bars.accf[ab], static_cast<uint32_t>((gi >> 1) & 1), ctl, dec::kSiteEpiAccFull);
          ready = ready && mbar_wait(&bars.xsf[xr], static_cast<uint32_t>((gi / XR) & 1), ctl, dec::kSiteScaleFull);
          ok = __all_sync(0xffffffffu, ready);
        }
        if (!ok) continue;    // no further waits; the group decides at the segment end
        tc_fence_after();
        // 2^-e of this thread's rows, as fp32 pairs (shared-memory broadcast)
        const uint64_t* f2 = reinterpret_cast<const uint64_t*>(bars.xs[xr] + m0);
#pragma unroll
        for (int h = 0; h < HALVES; ++h) {
          const uint64_t s2 = f2_pack(sw[h], sw[h]);
          const uint32_t col = tmem_base + lane_base + (ab * HALVES + h) * 2 * MPAD + m0;
#pragma unroll
          for (int c = 0; c < RPS; c += CH) {   // CH columns at a time keeps register use low
            uint32_t ph[CH], pl[CH];            // x_hi and x_lo products of the same rows
            if constexpr (CH == 16) {
              tmem_ld16(col + c, ph);
              tmem_ld16(col + MPAD + c, pl);
            } else {
              tmem_ld8(col + c, ph);
              tmem_ld8(col + MPAD + c, pl);
            }
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < CH / 2; ++j) {
              const uint64_t sum = f2_add(f2_pack_u(ph[2 * j], ph[2 * j + 1]), f2_pack_u(pl[2 * j], pl[2 * j + 1]));
              acc[h][c / 2 + j] = f2_fma(sum, f2_mul(f2[c / 2 + j], s2), acc[h][c / 2 + j]);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&bars.acce[ab]);
        mbar_arrive(&bars.xse[xr]);
      }
      // Segment end.  One thread waits for the sums of squares; the whole
      // group then follows one decision, so it never splits at a barrier.
      const int b = seg & 1;
      if (lane == 0) bars.warp_ok[st >> 5] = ok ? 1 : 0;
      if (st == 0) {
        bars.seg_ok = (ok && mbar_wait(&bars.ssq_full[b], (seg >> 1) & 1, ctl, dec::kSiteEpiSsqFull)) ? 1 : 0;
      }
      named_bar_sync(1, C::SCALE_THREADS);
      bool all_ok = bars.seg_ok != 0;
#pragma unroll
      for (int w = 0; w < C::SCALE_WARPS; ++w) all_ok = all_ok && bars.warp_ok[w] != 0;
      if (!all_ok) break;
      const bool whole = (kb0 == 0 && kb1 == p.kblocks);
      uint8_t* qbuf = reinterpret_cast<uint8_t*>(bars.ybuf);   // NVFP4 staging
      if (whole && OUT == kOutPartial) {
        // the tile's fp32 accumulators and (tile 0) the sums of squares, not post-scaled
#pragma unroll
        for (int j = 0; j < RPS; ++j) {
          const int m = m0 + j;
          if (m >= p.M) break;
          p.part_out[static_cast<int64_t>(m) * p.ncols + tile * 128 + n] =
              (j & 1) ? f2_hi(acc[0][j / 2]) : f2_lo(acc[0][j / 2]);
        }
        if (tile == 0 && st < p.M) p.part_out[static_cast<int64_t>(p.M) * p.ncols + st] = bars.ssq[b][st];
      } else if (whole) {
        const float gs = OUT == kOutNvfp4 ? __ldg(p.gscale) : 0.f;
#pragma unroll
        for (int j = 0; j < RPS; ++j) {
          const int m = m0 + j;
          if (m >= p.M) break;   // uniform per warp (m0 is)
          const float r = inv_rms(bars.ssq[b][m], p.inv_d, p.eps);
          const float a0 = (j & 1) ? f2_hi(acc[0][j / 2]) : f2_lo(acc[0][j / 2]);
          float v = a0 * r;
          if (HALVES == 2) v = silu_f32(v) * (((j & 1) ? f2_hi(acc[1][j / 2]) : f2_lo(acc[1][j / 2])) * r);
          if constexpr (OUT == kOutNvfp4) dec::stage_fp4(qbuf, MPAD, m, n, v, gs);
          else bars.ybuf[m * 128 + n] = __float2bfloat16_rn(v);
        }
      } else {
        // Split tile: this CTA's partial for the fix-up kernel, in the slot
        // layout float4 [half][row / 4][column] (rows < M only), then the
        // MPAD partial sums of squares.
        const int Q = (p.M + 3) >> 2;
        const int slot = cta * 2 + (seg == 0 ? 0 : 1);
        float* part = p.part + static_cast<int64_t>(slot) * dec::slot_floats<MPAD, HALVES>();
        float4* part4 = reinterpret_cast<float4*>(part);
#pragma unroll
        for (int h = 0; h < HALVES; ++h)
#pragma unroll
          for (int q4 = 0; q4 < RPS / 4; ++q4)
            if (m0 / 4 + q4 < Q)
              __stcg(part4 + (h * (MPAD / 4) + m0 / 4 + q4) * 128 + n,
                     make_float4(f2_lo(acc[h][2 * q4]), f2_hi(acc[h][2 * q4]), f2_lo(acc[h][2 * q4 + 1]),
                                 f2_hi(acc[h][2 * q4 + 1])));
        if (st < MPAD) __stcg(part + HALVES * MPAD * 128 + st, bars.ssq[b][st]);
      }
      named_bar_sync(1, C::SCALE_THREADS);   // sums of squares read, staging complete
      if (st == 0) mbar_arrive(&bars.ssq_empty[b]);
      if (whole) {
        if constexpr (OUT == kOutNvfp4) dec::store_tile_fp4(qbuf, MPAD, p, tile, st, C::SCALE_THREADS);
        else if constexpr (OUT == kOutBf16) dec::store_tile_rows(bars.ybuf, p, tile, st, C::SCALE_THREADS);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

template <int MPAD, int HALVES, bool PRE = false>
constexpr size_t smem_bytes() {
  using C = Cfg<MPAD, HALVES, PRE>;
  return 1024 + C::STAGES * C::STAGE_BYTES + sizeof(Bars<MPAD, C::STAGES>);
}

static_assert(smem_bytes<64, 2>() <= 227 * 1024 && smem_bytes<64, 1>() <= 227 * 1024 &&
                  smem_bytes<16, 2>() <= 227 * 1024 && smem_bytes<32, 2>() <= 227 * 1024,
              "shared memory per CTA");
static_assert(Cfg<64, 2>::STAGES >= 2, "pipeline needs two stages");
static_assert(Cfg<16, 1>::TMEM_COLS == 64 && Cfg<64, 2>::TMEM_COLS == 512, "TMEM allocation: a power of two <= 512");

// Whether calls with this padded row count split x once per call.
template <int MPAD>
constexpr bool presplit() { return MPAD >= 32; }

template <int MPAD, int HALVES, int OUT = kOutBf16>
cudaError_t launch_impl(const CallArgs& a) {
  constexpr bool PRE = presplit<MPAD>();
  using C = Cfg<MPAD, HALVES, PRE>;
  const size_t part_bytes = dec::workspace_bytes<MPAD, HALVES>(a.d, a.ncols, a.num_sms);
  if (a.ws_bytes < part_bytes + (PRE ? presplit_bytes(MPAD, a.d) : 0)) return cudaErrorInvalidValue;
  CUtensorMap tx, tw, tq;
  if (!make_tmap_2d(&tx, a.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.M, a.d, MPAD, 64)) return cudaErrorInvalidValue;
  // e4m3 codes as bytes: 128 columns (one 128-byte swizzle row) x 128 k rows per box
  if (!make_tmap_2d(&tw, a.Wp, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.d, a.ncols, BKQ, 128)) return cudaErrorInvalidValue;
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
  p.scales = a.scales;
  p.cluster = 1;
  p.narrow = dec::partition_is_narrow(p.total, p.grid) ? 1 : 0;
  p.x = static_cast<const __nv_bfloat16*>(a.x);
  p.xhilo = nullptr;
  p.xfac = nullptr;
  p.yq = static_cast<uint8_t*>(a.yq);
  p.ysf = static_cast<uint8_t*>(a.ysf);
  p.sf_chunked = a.sf_chunked;
  p.gscale = a.gscale;
  p.part_out = a.part_out;
  p.wsf = nullptr;
  p.xsf = nullptr;
  tq = tw;   // unused unless x is split once per call
  if (PRE) {
    // after the partial slots: x_hi / x_lo slabs, then the scale factors
    p.xhilo = ws + part_bytes;
    p.xfac = reinterpret_cast<float*>(ws + part_bytes + static_cast<size_t>(2 * MPAD) * a.d);
    if (!make_tmap_2d(&tq, p.xhilo, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(p.kblocks) * 2 * MPAD,
                      BKQ, 2 * MPAD, BKQ))
      return cudaErrorInvalidValue;
  }
  constexpr size_t SMEM = smem_bytes<MPAD, HALVES, PRE>();
  cudaError_t e = ensure_smem_limit<decode_fp8_kernel<MPAD, HALVES, PRE, OUT>>(static_cast<int>(SMEM));
  if (e != cudaSuccess) return e;
  if (PRE) {
    const int warps = p.kblocks * MPAD;
    e = launch_pdl(xsplit_kernel<MPAD>, static_cast<unsigned>((warps + 7) / 8), 256, 0, a.stream, p);
    if (e != cudaSuccess) return e;
  }
  e = launch_pdl(decode_fp8_kernel<MPAD, HALVES, PRE, OUT>, p.grid, C::THREADS, SMEM, a.stream, tx, tw, tq, p);
  if (e != cudaSuccess) return e;
  if (!dec::any_split_tile(p.grid, p.total, p.kblocks)) return cudaSuccess;
  return dec::launch_fixup<MPAD, HALVES, OUT>(p, a.stream);
}

}  // namespace dec8

size_t decode_fp8_presplit_bytes(int64_t M, int64_t d) {
  const int mp = decode_mpad(M);
  if (mp == 32) return dec8::presplit<32>() ? dec8::presplit_bytes(32, d) : 0;
  if (mp == 64) return dec8::presplit<64>() ? dec8::presplit_bytes(64, d) : 0;
  return dec8::presplit<16>() ? dec8::presplit_bytes(16, d) : 0;
}

cudaError_t launch_decode_fp8(const CallArgs& a, int mpad) {
  if (a.part_out) {   // partial output: a plain projection of the stored columns
    if (mpad == 16) return dec8::launch_impl<16, 1, kOutPartial>(a);
    if (mpad == 32) return dec8::launch_impl<32, 1, kOutPartial>(a);
    return dec8::launch_impl<64, 1, kOutPartial>(a);
  }
  if (a.yq) {   // NVFP4 output (SwiGLU only)
    if (mpad == 16) return dec8::launch_impl<16, 2, kOutNvfp4>(a);
    if (mpad == 32) return dec8::launch_impl<32, 2, kOutNvfp4>(a);
    return dec8::launch_impl<64, 2, kOutNvfp4>(a);
  }
  if (mpad == 16) return a.swiglu ? dec8::launch_impl<16, 2>(a) : dec8::launch_impl<16, 1>(a);
  if (mpad == 32) return a.swiglu ? dec8::launch_impl<32, 2>(a) : dec8::launch_impl<32, 1>(a);
  return a.swiglu ? dec8::launch_impl<64, 2>(a) : dec8::launch_impl<64, 1>(a);
}

}  // namespace fn
