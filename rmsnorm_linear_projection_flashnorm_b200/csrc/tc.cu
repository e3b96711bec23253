// Fused RMSNorm + projection, tensor-core tile path (M > 64), sm_100a.
//
// What it computes is FlashNorm's deferred normalisation (FlashNorm talk
// summary, Proposal 2 "지연된 정규화"): with the gain already folded into W'
// (Proposal 1), y[m, n] = r[m] * sum_k x[m, k] W'[k, n], where
// r[m] = 1/sqrt(sum_k x[m,k]^2 / d + eps).  The matmul runs on the raw
// activations on the tensor cores while the per-row sum of squares is reduced
// on the CUDA cores from the same staged x tiles, and the scalar is applied
// afterwards.  The optional SwiGLU epilogue (FlashInfer PR #5521 analysis,
// design item "Register-level SwiGLU") turns a 256-column tile holding
// matching gate and up columns into silu(r * gate) * (r * up).
//
// The talk's bug ("실제 버그", "원인", "수정" bullets) was an implicit join:
// the post-scale read a matmul result that was not finished.  Here every join
// is an mbarrier: the epilogue waits on the MMA commit of *this* tile's
// accumulator buffer and on the reducers' barrier for *this* tile's sums of
// squares; a stage of x is refilled only after both the MMA and the reducers
// released it; an accumulator buffer is reused only after the epilogue
// drained it.
//
// Layout: one persistent CTA per SM, 10 warps (18 with fp8 weights: warps
// 10-17 convert each staged e4m3 weight tile to the bf16 operand tile).
//   warp 0      TMA producer: x tile 128x64 (K-major) and W' tile 64x256
//               (four 64-column boxes, N-major), 128-byte swizzle, 4 stages
//   warp 1      TMEM owner and MMA issuer (tcgen05.mma M=128 N=256 K=16)
//   warps 2-5   sum-of-squares reducers, one thread per tile row
//   warps 6-9   epilogue: TMEM -> registers, post-scale (+SwiGLU), bf16 store
// Accumulators are double-buffered in TMEM (2 x 256 columns) so the epilogue
// of one tile overlaps the main loop of the next.
//
// AdaLN variant (the "RMSNorm + AdaLN" front of the fused FC1 on the
// FlashInfer PR #5521 analysis: a per-token index selects a scale row and a
// shift row applied after the norm).  With h = RMSNorm(x; g) * s[c] + t[c]
// and W' = diag(g) W, the projection is r * ((x * s[c]) @ W') + (t[c] @ W):
// the scale multiplies the raw activations, so the reducer warps, which read
// every staged x row for the sum of squares anyway, also write x * s[c] (one
// rounding to bf16) into a second operand tile that the MMA reads, while the
// sum of squares still comes from the raw tile; the shift enters through the
// unfolded weight as a per-condition bias row added in the epilogue.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "nvfp4.cuh"
#include "ptx.cuh"

namespace fn {
namespace tc {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int A_BYTES = BM * BK * 2;            // 16 KB
constexpr int B_BOX_BYTES = 64 * BK * 2;        // 8 KB: 64 columns x 64 rows
constexpr int B_BYTES = BN * BK * 2;            // 32 KB
constexpr int E4_BYTES = BN * BK;               // fp8 weights: 16 KB e4m3 staging per stage
constexpr int TMEM_COLS = 2 * BN;

// bf16 weights: 4 stages of 48 KB, 10 warps.  fp8 weights: 3 stages of 64 KB
// (x, bf16 operand, e4m3 staging) and 8 more warps converting e4m3 to bf16.
// AdaLN (bf16 weights): 3 stages of 64 KB (raw x, modulated x, weight).
template <bool FP8, bool ADALN = false> struct Cfg {
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + (FP8 ? E4_BYTES : 0) + (ADALN ? A_BYTES : 0);
  static constexpr int STAGES = FP8 || ADALN ? 3 : 4;
  static constexpr int NUM_THREADS = FP8 ? 576 : 320;
};
constexpr int GROUP_M = 16;                     // tile raster: bands of 16 row blocks

// wait sites reported in the status word
enum : unsigned { kSiteProdEmpty = 1, kSiteMmaAccEmpty, kSiteMmaFull, kSiteRedFull, kSiteRedSsqEmpty,
                  kSiteEpiAccFull, kSiteEpiSsqFull, kSiteDrain, kSiteMmaConv, kSiteConvFull };

struct Params {
  int M, d, ncols, nout;
  int num_m, num_n, num_tiles, kblocks;
  float eps, inv_d;
  __nv_bfloat16* y;
  unsigned int* status;
  unsigned long long budget_ns;
  int withhold;
  const float* scales;   // fp8: block scales [d/128][ncols/128]
  uint8_t* yq;           // NVFP4 output (SwiGLU only; y is null then): codes [M][nout / 2]
  uint8_t* ysf;          //   and e4m3 scale codes [M][nout / 16]
  const float* gscale;   //   global scale (one fp32 value in device memory)
  float* part_out;       // partial output: fp32 [M][ncols] accumulators, then [M] sums of squares
  const float* ad_scale; // AdaLN: scale rows fp32 [n_cond][d]
  const float* ad_bias;  //   shift bias rows fp32 [n_cond][ncols] (the shift times the unfolded weight)
  const int* ad_index;   //   per-token condition index [M]
  int n_cond;
  int sf_chunked;        // NVFP4 output: scale bytes in the 128x4 chunked layout (else row-major)
};

template <int STAGES>
struct alignas(8) Bars {
  uint64_t full[STAGES], empty[STAGES];
  uint64_t conv[STAGES];   // fp8: the stage's weight tile has been converted to bf16; AdaLN: x modulated
  uint64_t acc_full[2], acc_empty[2];
  uint64_t ssq_full[2], ssq_empty[2];
  uint64_t drain;
  float ssq[2][BM];
  uint32_t tmem_base;
  int abort_flag;
};

template <bool FP8, bool ADALN = false>
constexpr size_t smem_bytes() {
  return 1024 + Cfg<FP8, ADALN>::STAGES * Cfg<FP8, ADALN>::STAGE_BYTES + sizeof(Bars<Cfg<FP8, ADALN>::STAGES>);
}
static_assert(smem_bytes<true>() <= 232448 && smem_bytes<false>() <= 232448 && smem_bytes<false, true>() <= 232448,
              "shared memory budget");

// AdaLN: condition of tile row `grow`, or -1 for an index outside [0, n_cond)
// (that row's outputs become NaN; padding rows past M take condition 0).
__device__ __forceinline__ int adaln_cond(const Params& p, int grow) {
  if (grow >= p.M) return 0;
  const int c = __ldg(p.ad_index + grow);
  return (c >= 0 && c < p.n_cond) ? c : -1;
}

// AdaLN: one staged x row (64 bf16, 128-byte swizzle) times the row's scale
// values s[k0 .. k0+63], each product rounded once to bf16, written to the same
// swizzled positions of the modulated operand tile.  srow is null for an
// invalid condition (the products become NaN).
__device__ __forceinline__ void modulate_row_sw128(const uint8_t* tile, uint8_t* mod, int row, const float* srow) {
  const uint8_t* src = tile + row * 128;
  uint8_t* dst = mod + row * 128;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const int off = (c ^ (row & 7)) << 4;
    const uint4 v = *reinterpret_cast<const uint4*>(src + off);
    float4 s0, s1;
    if (srow) {
      s0 = __ldg(reinterpret_cast<const float4*>(srow + 8 * c));
      s1 = __ldg(reinterpret_cast<const float4*>(srow + 8 * c + 4));
    } else {
      s0 = s1 = make_float4(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000), __int_as_float(0x7fc00000),
                            __int_as_float(0x7fc00000));
    }
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      o[j] = pack_bf16x2(bf16lo_to_f32(w[j]) * sv[2 * j], bf16hi_to_f32(w[j]) * sv[2 * j + 1]);
    *reinterpret_cast<uint4*>(dst + off) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

__device__ __forceinline__ void tile_coords(int t, const Params& p, int& mb, int& nb) {
  const int per_group = GROUP_M * p.num_n;
  const int group = t / per_group;
  const int first_m = group * GROUP_M;
  const int gm = min(p.num_m - first_m, GROUP_M);
  const int r = t - group * per_group;
  mb = first_m + r % gm;
  nb = r / gm;
}

// Bounded wait that ignores the abort flag: used only to drain this CTA's
// own asynchronous work before teardown.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, unsigned long long budget) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > budget) return;
  }
}

// OUT: bf16 y, NVFP4 codes and scales (SwiGLU only), or fp32 partials (OutKind).
template <bool SWIGLU, bool FP8, int OUT = kOutBf16, bool ADALN = false>
__global__ void __launch_bounds__(Cfg<FP8, ADALN>::NUM_THREADS, 1)
    tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
              const Params p) {
  static_assert(OUT != kOutNvfp4 || SWIGLU, "NVFP4 output is a SwiGLU epilogue");
  static_assert(!ADALN || (!FP8 && OUT == kOutBf16), "AdaLN: bf16 weights and bf16 output");
  constexpr int STAGES = Cfg<FP8, ADALN>::STAGES;
  constexpr int STAGE_BYTES = Cfg<FP8, ADALN>::STAGE_BYTES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars<STAGES>& bars = *reinterpret_cast<Bars<STAGES>*>(smem + STAGES * STAGE_BYTES);
  auto stage_a = [&](int s) { return smem + s * STAGE_BYTES; };
  auto stage_b = [&](int s) { return smem + s * STAGE_BYTES + A_BYTES; };
  auto stage_e4 = [&](int s) { return smem + s * STAGE_BYTES + A_BYTES + B_BYTES; };
  auto stage_am = [&](int s) { return smem + s * STAGE_BYTES + A_BYTES + B_BYTES; };   // AdaLN: modulated x

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.empty[s], 1 + 4);  // MMA commit + one arrival per reducer warp
      mbar_init(&bars.conv[s], ADALN ? 4 : 256);   // fp8: every converter thread; AdaLN: the reducer warps
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars.acc_full[b], 1);
      mbar_init(&bars.acc_empty[b], 128);
      mbar_init(&bars.ssq_full[b], 128);
      mbar_init(&bars.ssq_empty[b], 128);
    }
    mbar_init(&bars.drain, 1);
    bars.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmap_x);
    tma_prefetch_desc(&tmap_w);
  }
  if (warp == 1) {
    tmem_alloc(&bars.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Everything above overlaps the previous kernel in the stream; nothing
  // below may touch global memory before that kernel has completed.
  grid_dependency_wait();
  grid_launch_dependents();
  const uint32_t tmem_base = bars.tmem_base;
  const WaitCtl ctl{&bars.abort_flag, p.status, p.budget_ns};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      uint32_t issued = 0, last_ph = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        int mb, nb;
        tile_coords(t, p, mb, nb);
        for (int kb = 0; kb < p.kblocks; ++kb) {
          if (!mbar_wait(&bars.empty[s], ph ^ 1, ctl, kSiteProdEmpty)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars.full[s], FP8 ? A_BYTES + E4_BYTES : A_BYTES + B_BYTES);
          tma_load_2d(stage_a(s), &tmap_x, &bars.full[s], kb * BK, mb * BM);
          if (FP8) {
            // one unswizzled box of 256 e4m3 columns x 64 k rows
            tma_load_2d(stage_e4(s), &tmap_w, &bars.full[s], nb * BN, kb * BK);
          } else {
#pragma unroll
            for (int bx = 0; bx < BN / 64; ++bx)
              tma_load_2d(stage_b(s) + bx * B_BOX_BYTES, &tmap_w, &bars.full[s], nb * BN + bx * 64, kb * BK);
          }
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
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, /*a MN-major*/ false, /*b MN-major*/ true);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int i = 0;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x, ++i) {
        const int b = i & 1;
        const uint32_t aph = (i >> 1) & 1;
        if (!mbar_wait(&bars.acc_empty[b], aph ^ 1, ctl, kSiteMmaAccEmpty)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * BN;
        for (int kb = 0; kb < p.kblocks; ++kb) {
          if (!mbar_wait(&bars.full[s], ph, ctl, kSiteMmaFull)) { ok = false; break; }
          if ((FP8 || ADALN) && !mbar_wait(&bars.conv[s], ph, ctl, kSiteMmaConv)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(ADALN ? stage_am(s) : stage_a(s));
          const uint32_t b0 = smem_u32(stage_b(s));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // A: x rows, K-major, 128-byte rows, 8-row groups 1024 B apart; a K=16
            //    slice is 32 bytes further along the (swizzled) row.
            const uint64_t adesc = sdesc_sw128(a0 + kk * 32, 16, 1024);
            // B: W' rows k, N-major: 64-column groups 8 KB apart (LBO), 8-row
            //    k groups 1024 B apart (SBO); a K=16 slice is 16 rows = 2048 B.
            const uint64_t bdesc = sdesc_sw128(b0 + kk * 2048, B_BOX_BYTES, 1024);
            umma_bf16(d_tmem, adesc, bdesc, IDESC, (kb | kk) != 0);
          }
          umma_commit(&bars.empty[s]);
          if (++s == STAGES) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        umma_commit(&bars.acc_full[b]);
      }
      umma_commit(&bars.drain);
      drain_wait(&bars.drain, 0, p.budget_ns);
    }
    __syncwarp();
  } else if (warp >= 10) {
    // ------------------------------------------------------------ fp8 converters
    // e4m3 tile (64 k rows x 256 bytes, unswizzled) -> bf16 operand tile with
    // the 128x128 block scales folded in: bf16(fp32(q) * s), one rounding.
    if (FP8) {
      const int ct = threadIdx.x - 320;   // 0..255
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      const int sld = p.ncols >> 7;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        int mb, nb;
        tile_coords(t, p, mb, nb);
        for (int kb = 0; kb < p.kblocks; ++kb) {
          const float* srow = p.scales + static_cast<int64_t>((kb * BK) >> 7) * sld + nb * 2;
          // a plain projection with an odd number of 128-column blocks has a last
          // tile whose second half lies past the weight (TMA fills it with zeros)
          const float s0 = __ldg(srow), s1 = (nb * 2 + 1 < sld) ? __ldg(srow + 1) : 0.f;
          if (!__all_sync(0xffffffffu, mbar_wait(&bars.full[s], ph, ctl, kSiteConvFull))) { ok = false; break; }
          const uint8_t* e4 = stage_e4(s);
          uint8_t* wt = stage_b(s);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int u = ct + 256 * i;          // 64 rows x 16 chunks of 16 bytes
            const int k = u >> 4;
            const int n0 = (u & 15) * 16;
            e4m3x16_scale_to_bf16_sw128(e4 + k * BN + n0, n0 < 128 ? s0 : s1, wt, k, n0);
          }
          fence_proxy_async_smem();   // generic-proxy writes -> visible to tcgen05.mma
          mbar_arrive(&bars.conv[s]);
          if (++s == STAGES) { s = 0; ph ^= 1; }
        }
      }
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ sum-of-squares reducers
    const int row = (warp - 2) * 32 + lane;
    int s = 0;
    uint32_t ph = 0;
    int i = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x, ++i) {
      float acc = 0.f;
      const float* srow = nullptr;   // AdaLN: this row's scale row
      if constexpr (ADALN) {
        int mb, nb;
        tile_coords(t, p, mb, nb);
        const int c = adaln_cond(p, mb * BM + row);
        srow = c >= 0 ? p.ad_scale + static_cast<int64_t>(c) * p.d : nullptr;
      }
      for (int kb = 0; kb < p.kblocks; ++kb) {
        if (!__all_sync(0xffffffffu, mbar_wait(&bars.full[s], ph, ctl, kSiteRedFull))) { ok = false; break; }
        acc += row_sumsq_sw128(stage_a(s), row);
        if constexpr (ADALN) {
          modulate_row_sw128(stage_a(s), stage_am(s), row, srow ? srow + kb * BK : nullptr);
          fence_proxy_async_smem();   // generic-proxy operand writes -> visible to tcgen05.mma
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars.conv[s]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.empty[s]);
        if (++s == STAGES) { s = 0; ph ^= 1; }
      }
      if (!ok) break;
      const int b = i & 1;
      const uint32_t aph = (i >> 1) & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars.ssq_empty[b], aph ^ 1, ctl, kSiteRedSsqEmpty))) break;
      bars.ssq[b][row] = acc;
      if (!(p.withhold && i == 0)) mbar_arrive(&bars.ssq_full[b]);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;       // tile row == accumulator lane
    int i = 0;
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x, ++i) {
      int mb, nb;
      tile_coords(t, p, mb, nb);
      const int b = i & 1;
      const uint32_t aph = (i >> 1) & 1;
      // warp-uniform decision: tcgen05.ld below is .sync.aligned
      bool ok = mbar_wait(&bars.acc_full[b], aph, ctl, kSiteEpiAccFull);
      ok = ok && mbar_wait(&bars.ssq_full[b], aph, ctl, kSiteEpiSsqFull);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const float ssq_row = bars.ssq[b][row];
      const float r = inv_rms(ssq_row, p.inv_d, p.eps);
      mbar_arrive(&bars.ssq_empty[b]);
      const int grow = mb * BM + row;
      const bool row_ok = grow < p.M;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + b * BN;
      if constexpr (OUT == kOutPartial) {
        // One rank of a row-parallel split of d: the fp32 accumulators of the
        // stored columns and the row's sum of squares, before any post-scale.
        float* prow = p.part_out + static_cast<int64_t>(grow) * p.ncols + nb * BN;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t v[32];
          tmem_ld32(taddr + c, v);
          tmem_ld_wait();
          if (row_ok && nb * BN + c < p.ncols) {
            float4* dst = reinterpret_cast<float4*>(prow + c);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              dst[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                   __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
          }
        }
        if (row_ok && nb == 0) p.part_out[static_cast<int64_t>(p.M) * p.ncols + grow] = ssq_row;
      } else if constexpr (OUT == kOutNvfp4) {
        // NVFP4 output: this thread's row holds whole 16-column blocks
        const float gs = __ldg(p.gscale);
        uint8_t* qrow = p.yq + static_cast<int64_t>(grow) * (p.nout / 2) + nb * (BN / 4);
        uint64_t sfw = 0;   // the tile row's 8 scale bytes
#pragma unroll 1
        for (int c = 0; c < BN / 2; c += 32) {
          uint32_t gv[32], uv[32];
          tmem_ld32(taddr + c, gv);
          tmem_ld32(taddr + BN / 2 + c, uv);
          tmem_ld_wait();
          uint32_t w[4];
#pragma unroll
          for (int blk = 0; blk < 2; ++blk) {
            float o[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float g = __uint_as_float(gv[16 * blk + j]) * r, u = __uint_as_float(uv[16 * blk + j]) * r;
              o[j] = silu_f32(g) * u;
            }
            uint2 q;
            const uint32_t sf = fp4_quantize16(o, gs, q);
            w[2 * blk] = q.x;
            w[2 * blk + 1] = q.y;
            sfw |= static_cast<uint64_t>(sf) << (8 * (c / 16 + blk));
          }
          if (row_ok) *reinterpret_cast<uint4*>(qrow + c / 2) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        if (row_ok)
          fp4_store_sf8(p.ysf, grow, nb * (BN / 32), p.nout / kFp4Block, p.sf_chunked != 0,
                        make_uint2(static_cast<uint32_t>(sfw), static_cast<uint32_t>(sfw >> 32)));
      } else if constexpr (SWIGLU) {
        __nv_bfloat16* yrow = p.y + static_cast<int64_t>(grow) * p.nout + nb * (BN / 2);
        // AdaLN: the row's shift bias in stored column order (gate 128 | up 128)
        const float* brow = nullptr;
        if constexpr (ADALN) {
          const int cnd = adaln_cond(p, grow);
          brow = cnd >= 0 ? p.ad_bias + static_cast<int64_t>(cnd) * p.ncols + nb * BN : nullptr;
        }
#pragma unroll 1
        for (int c = 0; c < BN / 2; c += 32) {
          uint32_t gv[32], uv[32];
          tmem_ld32(taddr + c, gv);
          tmem_ld32(taddr + BN / 2 + c, uv);
          tmem_ld_wait();
          float bg[32], bu[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) bg[j] = bu[j] = 0.f;
          if constexpr (ADALN) {
            if (brow && row_ok) {
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const float4 a = __ldg(reinterpret_cast<const float4*>(brow + c) + j);
                const float4 b = __ldg(reinterpret_cast<const float4*>(brow + BN / 2 + c) + j);
                bg[4 * j] = a.x; bg[4 * j + 1] = a.y; bg[4 * j + 2] = a.z; bg[4 * j + 3] = a.w;
                bu[4 * j] = b.x; bu[4 * j + 1] = b.y; bu[4 * j + 2] = b.z; bu[4 * j + 3] = b.w;
              }
            }
          }
          uint32_t o[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            float g0 = __uint_as_float(gv[2 * j]) * r, g1 = __uint_as_float(gv[2 * j + 1]) * r;
            float u0 = __uint_as_float(uv[2 * j]) * r, u1 = __uint_as_float(uv[2 * j + 1]) * r;
            if constexpr (ADALN) {
              g0 += bg[2 * j]; g1 += bg[2 * j + 1];
              u0 += bu[2 * j]; u1 += bu[2 * j + 1];
            }
            o[j] = pack_bf16x2(silu_f32(g0) * u0, silu_f32(g1) * u1);
          }
          if (row_ok) {
            uint4* dst = reinterpret_cast<uint4*>(yrow + c);
#pragma unroll
            for (int j = 0; j < 4; ++j) dst[j] = make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
          }
        }
      } else {
        __nv_bfloat16* yrow = p.y + static_cast<int64_t>(grow) * p.nout;
        const float* brow = nullptr;   // AdaLN: the row's shift bias
        if constexpr (ADALN) {
          const int cnd = adaln_cond(p, grow);
          brow = cnd >= 0 ? p.ad_bias + static_cast<int64_t>(cnd) * p.ncols : nullptr;
        }
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t v[32];
          tmem_ld32(taddr + c, v);
          tmem_ld_wait();
          const int col = nb * BN + c;
          if (row_ok && col < p.nout) {
            float bv[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) bv[j] = 0.f;
            if constexpr (ADALN) {
              if (brow) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                  const float4 a = __ldg(reinterpret_cast<const float4*>(brow + col) + j);
                  bv[4 * j] = a.x; bv[4 * j + 1] = a.y; bv[4 * j + 2] = a.z; bv[4 * j + 3] = a.w;
                }
              }
            }
            uint32_t o[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
              o[j] = pack_bf16x2(__uint_as_float(v[2 * j]) * r + bv[2 * j], __uint_as_float(v[2 * j + 1]) * r + bv[2 * j + 1]);
            uint4* dst = reinterpret_cast<uint4*>(yrow + col);
#pragma unroll
            for (int j = 0; j < 4; ++j) dst[j] = make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bars.acc_empty[b]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

template <bool SWIGLU, bool FP8, int OUT = kOutBf16, bool ADALN = false>
cudaError_t launch_impl(const CallArgs& a) {
  CUtensorMap tx, tw;
  if (!make_tmap_2d(&tx, a.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.M, a.d, BM, BK)) return cudaErrorInvalidValue;
  if (FP8) {
    if (!make_tmap_2d(&tw, a.Wp, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.d, a.ncols, BK, BN, false))
      return cudaErrorInvalidValue;
  } else if (!make_tmap_2d(&tw, a.Wp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.d, a.ncols, BK, 64)) {
    return cudaErrorInvalidValue;
  }
  Params p;
  p.M = static_cast<int>(a.M);
  p.d = static_cast<int>(a.d);
  p.ncols = static_cast<int>(a.ncols);
  p.nout = static_cast<int>(a.N);
  p.num_m = static_cast<int>((a.M + BM - 1) / BM);
  p.num_n = static_cast<int>((a.ncols + BN - 1) / BN);
  p.num_tiles = p.num_m * p.num_n;
  p.kblocks = static_cast<int>(a.d / BK);
  p.eps = a.eps;
  p.inv_d = 1.0f / static_cast<float>(a.d);
  p.y = static_cast<__nv_bfloat16*>(a.y);
  p.status = static_cast<unsigned int*>(a.ws);
  p.budget_ns = a.budget_ns;
  p.withhold = a.withhold;
  p.scales = a.scales;
  p.yq = static_cast<uint8_t*>(a.yq);
  p.ysf = static_cast<uint8_t*>(a.ysf);
  p.gscale = a.gscale;
  p.part_out = a.part_out;
  p.ad_scale = a.ad_scale;
  p.ad_bias = a.ad_bias;
  p.ad_index = a.ad_index;
  p.n_cond = static_cast<int>(a.n_cond);
  p.sf_chunked = a.sf_chunked;
  constexpr size_t SMEM_BYTES = smem_bytes<FP8, ADALN>();
  cudaError_t e = ensure_smem_limit<tc_kernel<SWIGLU, FP8, OUT, ADALN>>(static_cast<int>(SMEM_BYTES));
  if (e != cudaSuccess) return e;
  const int grid = p.num_tiles < a.num_sms ? p.num_tiles : a.num_sms;
  return launch_pdl(tc_kernel<SWIGLU, FP8, OUT, ADALN>, grid, Cfg<FP8, ADALN>::NUM_THREADS, SMEM_BYTES, a.stream, tx,
                    tw, p);
}

}  // namespace tc

cudaError_t launch_tc(const CallArgs& a) {
  if (a.ad_index)   // AdaLN: bf16 weights (other types were converted to bf16 first), bf16 output
    return a.swiglu ? tc::launch_impl<true, false, kOutBf16, true>(a) : tc::launch_impl<false, false, kOutBf16, true>(a);
  if (a.yq) return a.wtype == 1 ? tc::launch_impl<true, true, kOutNvfp4>(a) : tc::launch_impl<true, false, kOutNvfp4>(a);
  // bf16 weights and output at large M: the kernel on pairs of SMs
  if (!a.yq && !a.part_out && a.wtype == 0 && a.M >= kPairTileMinM && !a.single_sm_tiles) return launch_tc_pair(a);
  // partial output: no activation, so every weight is a plain projection of its stored columns
  if (a.part_out)
    return a.wtype == 1 ? tc::launch_impl<false, true, kOutPartial>(a) : tc::launch_impl<false, false, kOutPartial>(a);
  if (a.wtype == 1) return a.swiglu ? tc::launch_impl<true, true>(a) : tc::launch_impl<false, true>(a);
  return a.swiglu ? tc::launch_impl<true, false>(a) : tc::launch_impl<false, false>(a);
}

}  // namespace fn
