// Fused RMSNorm + projection, small-M path (M <= 64), sm_100a.
//
// Same arithmetic as the tile path (FlashNorm talk summary, Proposal 2
// "지연된 정규화": matmul on raw x, sum of squares alongside, 1/rms applied
// after), shaped for decode, where the weight stream from HBM is the whole
// cost (FlashNorm talk: the norm is launched about 33 times per decode step;
// Marlin explainer, section 3: fused time is the larger of the memory time and
// the tensor-core time, not their sum).
//
// Swap-AB on the tensor cores: each MMA is D[n, m] += W'^T[n, k] x^T[k, m] with
// M = 128 weight columns on the lane side and the activation rows padded to
// 16/32/64 on the N side (tcgen05.mma M=128, N=MPAD, K=16).  The weight tile
// (N-major) and the x tile (K-major) are staged by TMA with 128-byte swizzle.
//
// The weight is split over every SM with a stream-K partition of the
// (column tile, 64-deep k block) iterations, so every SM streams the same
// number of weight bytes whatever the tile count.  A tile whose k range falls
// to one CTA is finished by that CTA.  A tile whose k range is split between
// CTAs is finished by a second, small kernel (decode_fixup_kernel): each
// contributing CTA writes its fp32 partial accumulators and partial sums of
// squares to the workspace, and the fix-up kernel, launched programmatically
// so it is resident before the first kernel ends, adds the partials in
// ascending k order (a fixed order, so repeated calls are bit-identical),
// applies the post-scale (and SwiGLU) and stores the result.  No atomics, no
// cross-CTA waits, no counters to reset.
//
// Layout: 8 warps.
//   warp 0      TMA producer
//   warp 1      TMEM owner and MMA issuer
//   warps 2-3   sum-of-squares reducers (one thread per activation row)
//   warps 4-7   epilogue / fix-up (one thread per weight column of the tile)
//
// This file holds the bf16-weight kernel; fp8 weights have their own kernel
// (decode_fp8.cu) that feeds the e4m3 tiles to the tensor cores unconverted.
#include <cstddef>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "decode_common.cuh"

namespace fn {
namespace dec {

constexpr int NUM_THREADS = 256;   // producer, MMA, 2 reducers, 4 epilogue warps
constexpr int W_BOX_BYTES = 64 * BK * 2;   // 64 columns x 64 k rows, bf16
constexpr int SMEM_BUDGET = 200 * 1024;   // pipeline stages; barriers and staging come on top

// One TMA ring whose stages hold the weight tile and the x tile.
template <int MPAD, int HALVES>
struct Cfg {
  static constexpr int W_BYTES = HALVES * 2 * W_BOX_BYTES;          // bf16 operand: 16 or 32 KB
  static constexpr int X_BYTES = MPAD * BK * 2;                     // 2, 4 or 8 KB
  static constexpr int STAGE_BYTES = W_BYTES + X_BYTES;             // multiple of 1024
  static constexpr int STAGES_RAW = SMEM_BUDGET / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static constexpr int ACC_COLS = HALVES * MPAD;                    // one accumulator buffer
  static constexpr int TMEM_COLS = 2 * ACC_COLS;                    // double buffered: 32..256
  static constexpr int SLOT_FLOATS = slot_floats<MPAD, HALVES>();
};

template <int MPAD, int HALVES, int STAGES>
struct alignas(16) Bars {
  uint64_t full[STAGES], empty[STAGES];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t ssq_full[2], ssq_empty[2];
  uint64_t drain;
  float ssq[2][MPAD];
  alignas(16) __nv_bfloat16 ybuf[MPAD * 128];   // one tile's output rows, staged for 16-byte stores
  uint32_t tmem_base;
  int abort_flag;
  int epi_ok[2];
  float rfix[MPAD];          // cluster mode: 1/rms of each row
};

// OUT: bf16 y, NVFP4 codes and scales (SwiGLU only), or fp32 partials (OutKind).
template <int MPAD, int HALVES, int OUT = kOutBf16>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                  const Params p) {
  static_assert(OUT != kOutNvfp4 || HALVES == 2, "NVFP4 output is a SwiGLU epilogue");
  static_assert(OUT != kOutPartial || HALVES == 1, "partial output: plain projection of the stored columns");
  using C = Cfg<MPAD, HALVES>;
  constexpr int STAGES = C::STAGES;
  using B = Bars<MPAD, HALVES, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  B& bars = *reinterpret_cast<B*>(smem + STAGES * C::STAGE_BYTES);
  // stage: [weight tile][x tile], each on a 1024-byte multiple
  auto stage_w = [&](int s) { return smem + s * C::STAGE_BYTES; };
  auto stage_x = [&](int s) { return smem + s * C::STAGE_BYTES + C::W_BYTES; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  // stream-K: an even share of all (tile, k block) iterations; cluster mode:
  // cluster c owns tile c and its CTAs split the tile's k blocks by rank
  long long it0, it1;
  if (p.cluster > 1) {
    const int tile = cta / p.cluster, rank = cta % p.cluster;
    it0 = static_cast<long long>(tile) * p.kblocks + static_cast<long long>(rank) * p.kblocks / p.cluster;
    it1 = static_cast<long long>(tile) * p.kblocks + static_cast<long long>(rank + 1) * p.kblocks / p.cluster;
  } else {
    it0 = it_begin(cta, p);
    it1 = it_begin(cta + 1, p);
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.empty[s], 1 + 2);   // MMA commit + two reducer warps
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars.acc_full[b], 1);
      mbar_init(&bars.acc_empty[b], 128);
      mbar_init(&bars.ssq_full[b], 64);
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
    tmem_alloc(&bars.tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Everything above overlaps the previous kernel in the stream.  So does an
  // L2 prefetch of the first part of this CTA's weight range (the weight does
  // not depend on the previous kernel's output, and an L2 prefetch cannot
  // return stale data).  Nothing below may read or write global memory
  // through shared memory or registers before the previous kernel completed.
  if (p.prefetch_mode == 1 && warp == 0 && lane == 0) {
    int n_pf = 0;
    for (long long it = it0; it < it1 && n_pf < p.prefetch_iters; ++it, ++n_pf) {
      const int tile = static_cast<int>(it / p.kblocks);
      const int kb = static_cast<int>(it - static_cast<long long>(tile) * p.kblocks);
      for (int bx = 0; bx < 2 * HALVES; ++bx) tma_prefetch_l2_2d(&tmap_w, tile * 128 * HALVES + bx * 64, kb * BK);
    }
  } else if (p.prefetch_mode == 2 && warp >= 2) {
    // one 128-byte line per thread and step: (k row, 128-byte column chunk)
    constexpr int WB = 2;                              // weight bytes per element
    const int lines_per_row = HALVES * WB;             // 128 * HALVES * WB bytes of a k row per tile
    const long long n_it = min(static_cast<long long>(p.prefetch_iters), it1 - it0);
    const int total = static_cast<int>(n_it) * BK * lines_per_row;
    for (int i = threadIdx.x - 64; i < total; i += NUM_THREADS - 64) {
      const int chunk = i % lines_per_row;
      const int r = (i / lines_per_row) % BK;
      const long long it = it0 + i / (lines_per_row * BK);
      const int tile = static_cast<int>(it / p.kblocks);
      const int kb = static_cast<int>(it - static_cast<long long>(tile) * p.kblocks);
      const uint8_t* a = p.wp + (static_cast<int64_t>(kb) * BK + r) * p.ncols * WB +
                         static_cast<int64_t>(tile) * 128 * HALVES * WB + chunk * 128;
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
      bool ok = true;
      for (long long it = it0; it < it1 && ok;) {
        const int tile = static_cast<int>(it / p.kblocks);
        const int kb0 = static_cast<int>(it - static_cast<long long>(tile) * p.kblocks);
        const int kb1 = static_cast<int>(min(static_cast<long long>(p.kblocks), kb0 + (it1 - it)));
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&bars.empty[s], ph ^ 1, ctl, kSiteProdEmpty)) { ok = false; break; }
          mbar_arrive_expect_tx(&bars.full[s], C::X_BYTES + C::W_BYTES);
          tma_load_2d(stage_x(s), &tmap_x, &bars.full[s], kb * BK, 0);
#pragma unroll
          for (int bx = 0; bx < 2 * HALVES; ++bx)
            tma_load_2d_hint(stage_w(s) + bx * W_BOX_BYTES, &tmap_w, &bars.full[s],
                             tile * 128 * HALVES + bx * 64, kb * BK, w_policy);
          issued |= 1u << s;
          last_ph = (last_ph & ~(1u << s)) | (ph << s);
          if (++s == STAGES) { s = 0; ph ^= 1; }
        }
        it += kb1 - kb0;
      }
      for (int i = 0; i < STAGES; ++i)
        if (issued & (1u << i)) drain_wait(&bars.full[i], (last_ph >> i) & 1u, p.budget_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(128, MPAD, /*a MN-major*/ true, /*b MN-major*/ false);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int seg = 0;
      for (long long it = it0; it < it1 && ok; ++seg) {
        const int tile = static_cast<int>(it / p.kblocks);
        const int kb0 = static_cast<int>(it - static_cast<long long>(tile) * p.kblocks);
        const int kb1 = static_cast<int>(min(static_cast<long long>(p.kblocks), kb0 + (it1 - it)));
        const int b = seg & 1;
        const uint32_t aph = (seg >> 1) & 1;
        if (!mbar_wait(&bars.acc_empty[b], aph ^ 1, ctl, kSiteMmaAccEmpty)) break;
        tc_fence_after();
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&bars.full[s], ph, ctl, kSiteMmaFull)) { ok = false; break; }
          tc_fence_after();
          const uint32_t w0 = smem_u32(stage_w(s));
          const uint32_t x0 = smem_u32(stage_x(s));
#pragma unroll
          for (int h = 0; h < HALVES; ++h) {
            const uint32_t d_tmem = tmem_base + (b * HALVES + h) * MPAD;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              // A = W'^T: 128 weight columns, N-major; 64-column groups one box
              //     (8 KB) apart, 8-row k groups 1024 B apart; K=16 is 2048 B.
              const uint64_t adesc = sdesc_sw128(w0 + h * 2 * W_BOX_BYTES + kk * 2048, W_BOX_BYTES, 1024);
              // B = x^T: MPAD activation rows, K-major, 128-byte rows.
              const uint64_t bdesc = sdesc_sw128(x0 + kk * 32, 16, 1024);
              umma_bf16(d_tmem, adesc, bdesc, IDESC, (kb != kb0 || kk != 0) ? 1u : 0u);
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
      drain_wait(&bars.drain, 0, p.budget_ns);
    }
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------------------------------------ sum-of-squares reducers
    const int row = (warp - 2) * 32 + lane;      // activation row
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    int seg = 0;
    for (long long it = it0; it < it1 && ok; ++seg) {
      const int tile = static_cast<int>(it / p.kblocks);
      const int kb0 = static_cast<int>(it - static_cast<long long>(tile) * p.kblocks);
      const int kb1 = static_cast<int>(min(static_cast<long long>(p.kblocks), kb0 + (it1 - it)));
      float acc = 0.f;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!__all_sync(0xffffffffu, mbar_wait(&bars.full[s], ph, ctl, kSiteRedFull))) { ok = false; break; }
        if (row < MPAD && row < p.M) acc += row_sumsq_sw128(stage_x(s), row);
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.empty[s]);
        if (++s == STAGES) { s = 0; ph ^= 1; }
      }
      if (!ok) break;
      const int b = seg & 1;
      const uint32_t aph = (seg >> 1) & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars.ssq_empty[b], aph ^ 1, ctl, kSiteRedSsqEmpty))) break;
      if (row < MPAD) bars.ssq[b][row] = acc;
      if (!(p.withhold && seg == 0)) mbar_arrive(&bars.ssq_full[b]);
      it += kb1 - kb0;
    }
  } else {
    // ------------------------------------------------------------ epilogue / fix-up
    const int q = warp & 3;
    const int n = q * 32 + lane;                  // weight column within the 128-wide half
    const int et = threadIdx.x - 128;             // 0..127
    int seg = 0;
    for (long long it = it0; it < it1; ++seg) {
      const int tile = static_cast<int>(it / p.kblocks);
      const int kb0 = static_cast<int>(it - static_cast<long long>(tile) * p.kblocks);
      const int kb1 = static_cast<int>(min(static_cast<long long>(p.kblocks), kb0 + (it1 - it)));
      it += kb1 - kb0;
      const int b = seg & 1;
      const uint32_t aph = (seg >> 1) & 1;
      // One thread waits and the whole epilogue group follows its decision, so
      // the group never splits at the named barriers or the .sync.aligned loads.
      if (et == 0) {
        bool ok = mbar_wait(&bars.acc_full[b], aph, ctl, kSiteEpiAccFull);
        ok = ok && mbar_wait(&bars.ssq_full[b], aph, ctl, kSiteEpiSsqFull);
        bars.epi_ok[seg & 1] = ok ? 1 : 0;
      }
      named_bar_sync(1, 128);
      if (!bars.epi_ok[seg & 1]) break;
      tc_fence_after();
      float acc[HALVES][MPAD];
#pragma unroll
      for (int h = 0; h < HALVES; ++h)
        tmem_ld_cols<MPAD>(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + (b * HALVES + h) * MPAD, acc[h]);
      tc_fence_before();
      mbar_arrive(&bars.acc_empty[b]);
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
          if (HALVES == 2) v = silu_f32(acc[0][m] * r) * (acc[1][m] * r);
          else v = acc[0][m] * r;
          if constexpr (OUT == kOutNvfp4) stage_fp4(qbuf, MPAD, m, n, v, gs);
          else bars.ybuf[m * 128 + n] = __float2bfloat16_rn(v);
        }
        mbar_arrive(&bars.ssq_empty[b]);
        named_bar_sync(1, 128);
        if constexpr (OUT == kOutNvfp4) store_tile_fp4(qbuf, MPAD, p, tile, et, 128);
        else store_tile_rows(bars.ybuf, p, tile, et, 128);
        continue;
      }
      if (p.cluster > 1) {
        // Cluster mode: this CTA's only segment.  Its pipeline stages are idle
        // now (every MMA and every reducer read has completed), so the partial
        // accumulators [half][row][column] and sums of squares go there for the
        // peers to read over distributed shared memory after the cluster barrier.
        float* red = reinterpret_cast<float*>(smem);
#pragma unroll
        for (int h = 0; h < HALVES; ++h)
#pragma unroll
          for (int m = 0; m < MPAD; ++m) red[(h * MPAD + m) * 128 + n] = acc[h][m];
        if (et < MPAD) red[HALVES * MPAD * 128 + et] = bars.ssq[b][et];
        mbar_arrive(&bars.ssq_empty[b]);
        continue;
      }
      // Split tile: publish this CTA's partial for the fix-up kernel.  A slot
      // holds float4 groups [half][row / 4][column] (a warp's 16-byte accesses
      // are contiguous), only for the rows < M, then the MPAD partial sums of
      // squares.
      const int Q = (p.M + 3) >> 2;
      const int slot = cta * 2 + (seg == 0 ? 0 : 1);
      float4* part4 = reinterpret_cast<float4*>(p.part + static_cast<int64_t>(slot) * C::SLOT_FLOATS);
#pragma unroll
      for (int h = 0; h < HALVES; ++h)
#pragma unroll
        for (int q4 = 0; q4 < MPAD / 4; ++q4)
          if (q4 < Q)
            __stcg(part4 + (h * (MPAD / 4) + q4) * 128 + n,
                   make_float4(acc[h][4 * q4], acc[h][4 * q4 + 1], acc[h][4 * q4 + 2], acc[h][4 * q4 + 3]));
      float* part = p.part + static_cast<int64_t>(slot) * C::SLOT_FLOATS;
      if (et < MPAD) __stcg(part + HALVES * MPAD * 128 + et, bars.ssq[b][et]);
      mbar_arrive(&bars.ssq_empty[b]);
    }
  }

  if (p.cluster > 1) {
    // every CTA of the cluster has its partial in shared memory
    cluster_sync_all();
    if (warp >= 4 && warp < 8) {
      const int et = threadIdx.x - 128;
      const uint32_t S = static_cast<uint32_t>(p.cluster);
      const uint32_t rank = cluster_ctarank();
      const int tile = cta / p.cluster;
      const float* red = reinterpret_cast<const float*>(smem);
      uint32_t base[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) base[q] = q < static_cast<int>(S) ? dsmem_addr(red, q) : 0u;
      if (et < p.M && et < MPAD) {
        float ss = 0.f;                      // partial sums of squares in rank (= k) order
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (q < static_cast<int>(S)) ss += dsmem_ld_f32(base[q] + 4u * (HALVES * MPAD * 128 + et));
        bars.rfix[et] = inv_rms(ss, p.inv_d, p.eps);
      }
      named_bar_sync(1, 128);
      // this rank finishes a contiguous share of the tile's (row, column) outputs
      const int E = p.M * 128;
      const int lo = static_cast<int>(static_cast<long long>(rank) * E / S);
      const int hi = static_cast<int>(static_cast<long long>(rank + 1) * E / S);
#pragma unroll 2
      for (int e = lo + et; e < hi; e += 128) {
        const int m = e >> 7, nn = e & 127;
        float g = 0.f, u = 0.f;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (q < static_cast<int>(S)) {
            g += dsmem_ld_f32(base[q] + 4u * (m * 128 + nn));
            if (HALVES == 2) u += dsmem_ld_f32(base[q] + 4u * ((MPAD + m) * 128 + nn));
          }
        }
        const float r = bars.rfix[m];
        float v = g * r;
        if (HALVES == 2) v = silu_f32(v) * (u * r);
        const int col = tile * 128 + nn;
        if (col < p.nout) p.y[static_cast<int64_t>(m) * p.nout + col] = __float2bfloat16_rn(v);
      }
    }
    // no CTA may leave while a peer still reads its shared memory
    cluster_sync_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// The staging buffer is read as 16-byte vectors; the barrier block itself is
// placed at a 1024-byte multiple.
using BarsSmall = Bars<16, 1, 8>;
using BarsLarge = Bars<64, 2, 5>;
static_assert(offsetof(BarsSmall, ybuf) % 16 == 0 && offsetof(BarsLarge, ybuf) % 16 == 0,
              "ybuf must be 16-byte aligned");
static_assert(Cfg<64, 2>::STAGES >= 2, "pipeline needs two stages");
// cluster mode reuses the ring for its partials: HALVES x MPAD x 128 floats + MPAD
static_assert(Cfg<64, 2>::STAGES * Cfg<64, 2>::STAGE_BYTES >= (2 * 64 * 128 + 64) * 4,
              "cluster partials must fit the ring");

template <int MPAD, int HALVES>
constexpr size_t smem_bytes() {
  using C = Cfg<MPAD, HALVES>;
  return 1024 + C::STAGES * C::STAGE_BYTES + sizeof(Bars<MPAD, HALVES, C::STAGES>);
}

// Cluster size for split-K with a distributed-shared-memory reduction: as
// many CTAs per column tile as the SMs allow (at most 8, at most one per k
// block); 1 when the tiles alone already occupy half the SMs or more.
inline int cluster_split(int tiles, int kblocks, int num_sms) {
  if (tiles * 2 > num_sms) return 1;
  int S = num_sms / tiles;
  if (S > 8) S = 8;
  if (S > kblocks) S = kblocks;
  return S;
}

template <int MPAD, int HALVES, int OUT = kOutBf16>
cudaError_t launch_impl(const CallArgs& a) {
  if (a.ws_bytes < workspace_bytes<MPAD, HALVES>(a.d, a.ncols, a.num_sms)) return cudaErrorInvalidValue;
  CUtensorMap tx, tw;
  if (!make_tmap_2d(&tx, a.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.M, a.d, MPAD, BK)) return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tw, a.Wp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.d, a.ncols, BK, 64)) return cudaErrorInvalidValue;
  Params p;
  p.M = static_cast<int>(a.M);
  p.d = static_cast<int>(a.d);
  p.ncols = static_cast<int>(a.ncols);
  p.nout = static_cast<int>(a.N);
  p.kblocks = static_cast<int>(a.d / BK);
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
  p.narrow = partition_is_narrow(p.total, p.grid) ? 1 : 0;
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
  constexpr size_t SMEM = smem_bytes<MPAD, HALVES>();
  cudaError_t e = ensure_smem_limit<decode_kernel<MPAD, HALVES, OUT>>(static_cast<int>(SMEM));
  if (e != cudaSuccess) return e;
  // Split K inside clusters when the tiles fill the GPU at least twice over
  // and every cluster can be resident at once; otherwise stream-K.
  // The largest cluster size whose clusters can all be resident (GPC sizes
  // decide that, not just the SM count), or the size forced by the caller.
  int S = a.cluster_mode >= 2 ? a.cluster_mode : cluster_split(p.tiles, p.kblocks, a.num_sms);
  if (OUT != kOutBf16) S = 1;   // the cluster finish writes bf16 only: other outputs take the stream-K path
  if (S > p.kblocks) S = p.kblocks;
  if (S > 8) S = 8;
  while (S >= 2 && !clusters_fit<decode_kernel<MPAD, HALVES, OUT>>(S, p.tiles, NUM_THREADS, SMEM)) --S;
  // Clusters only pay off when they occupy about as many SMs as stream-K
  // would: fewer SMs cannot pull the full HBM bandwidth.
  if (S >= 2 && a.cluster_mode != 0 && (a.cluster_mode >= 2 || 10LL * p.tiles * S >= 9LL * p.grid)) {
    p.cluster = S;
    p.grid = p.tiles * S;
    p.narrow = partition_is_narrow(p.total, p.grid) ? 1 : 0;
    return launch_pdl_cluster(decode_kernel<MPAD, HALVES, OUT>, static_cast<unsigned>(p.grid), S, NUM_THREADS, SMEM,
                              a.stream, tx, tw, p);
  }
  e = launch_pdl(decode_kernel<MPAD, HALVES, OUT>, p.grid, NUM_THREADS, SMEM, a.stream, tx, tw, p);
  if (e != cudaSuccess) return e;
  if (!any_split_tile(p.grid, p.total, p.kblocks)) return cudaSuccess;
  return launch_fixup<MPAD, HALVES, OUT>(p, a.stream);
}

}  // namespace dec

int decode_mpad(int64_t M) { return M <= 16 ? 16 : (M <= 32 ? 32 : 64); }

size_t decode_workspace_bytes(int64_t M, int64_t d, int64_t ncols, bool swiglu, int num_sms, int wtype) {
  const int mp = decode_mpad(M);
  const size_t extra = wtype == 1 ? decode_fp8_presplit_bytes(M, d) : wtype == 2 ? decode_mx_presplit_bytes(M, d) : 0;
  if (swiglu) {
    if (mp == 16) return dec::workspace_bytes<16, 2>(d, ncols, num_sms) + extra;
    if (mp == 32) return dec::workspace_bytes<32, 2>(d, ncols, num_sms) + extra;
    return dec::workspace_bytes<64, 2>(d, ncols, num_sms) + extra;
  }
  if (mp == 16) return dec::workspace_bytes<16, 1>(d, ncols, num_sms) + extra;
  if (mp == 32) return dec::workspace_bytes<32, 1>(d, ncols, num_sms) + extra;
  return dec::workspace_bytes<64, 1>(d, ncols, num_sms) + extra;
}

cudaError_t launch_decode(const CallArgs& a) {
  const int mp = decode_mpad(a.M);
  if (a.wtype == 1) return launch_decode_fp8(a, mp);
  if (a.wtype == 2) return launch_decode_mx(a, mp);
  int T = 0, S = 0;
  if (decode_cl_plan(a, T, S)) return launch_decode_cl(a, T, S);
  if (a.part_out) {   // partial output: a plain projection of the stored columns
    if (mp == 16) return dec::launch_impl<16, 1, kOutPartial>(a);
    if (mp == 32) return dec::launch_impl<32, 1, kOutPartial>(a);
    return dec::launch_impl<64, 1, kOutPartial>(a);
  }
  if (a.yq) {   // NVFP4 output (SwiGLU only)
    if (mp == 16) return dec::launch_impl<16, 2, kOutNvfp4>(a);
    if (mp == 32) return dec::launch_impl<32, 2, kOutNvfp4>(a);
    return dec::launch_impl<64, 2, kOutNvfp4>(a);
  }
  if (mp == 16) return a.swiglu ? dec::launch_impl<16, 2>(a) : dec::launch_impl<16, 1>(a);
  if (mp == 32) return a.swiglu ? dec::launch_impl<32, 2>(a) : dec::launch_impl<32, 1>(a);
  return a.swiglu ? dec::launch_impl<64, 2>(a) : dec::launch_impl<64, 1>(a);
}

}  // namespace fn
