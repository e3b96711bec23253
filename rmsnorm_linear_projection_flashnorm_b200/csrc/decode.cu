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
// number of weight bytes whatever the tile count.  A tile whose k range is
// split between CTAs is finished in the same kernel: each CTA writes its fp32
// partial accumulators and partial sums of squares to the workspace, and the
// CTA that arrives last on the tile's counter adds the partials in ascending
// k order (a fixed order, so repeated calls are bit-identical), applies the
// post-scale (and SwiGLU) and stores the result.  No floating-point atomics.
//
// Layout: 8 warps.
//   warp 0      TMA producer
//   warp 1      TMEM owner and MMA issuer
//   warps 2-3   sum-of-squares reducers (one thread per activation row)
//   warps 4-7   epilogue / fix-up (one thread per weight column of the tile)
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace fn {
namespace dec {

constexpr int BK = 64;
constexpr int NUM_THREADS = 256;
constexpr int W_BOX_BYTES = 64 * BK * 2;   // 64 columns x 64 k rows, bf16
constexpr int SMEM_BUDGET = 200 * 1024;

enum : unsigned { kSiteProdEmpty = 1, kSiteMmaAccEmpty, kSiteMmaFull, kSiteRedFull, kSiteRedSsqEmpty,
                  kSiteEpiAccFull, kSiteEpiSsqFull, kSiteDrain };

template <int MPAD, int HALVES>
struct Cfg {
  static constexpr int W_BYTES = HALVES * 2 * W_BOX_BYTES;          // 16 or 32 KB
  static constexpr int X_BYTES = MPAD * BK * 2;                     // 2, 4 or 8 KB
  static constexpr int STAGE_BYTES = W_BYTES + X_BYTES;             // multiple of 1024
  static constexpr int STAGES_RAW = SMEM_BUDGET / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static constexpr int ACC_COLS = HALVES * MPAD;                    // one accumulator buffer
  static constexpr int TMEM_COLS = 2 * ACC_COLS;                    // double buffered: 32..256
  static constexpr int SLOT_FLOATS = ((HALVES * MPAD * 128 + MPAD) + 31) / 32 * 32;
};

struct Params {
  int M, d, ncols, nout;
  int kblocks, tiles;
  long long total;   // tiles * kblocks
  int grid;
  float eps, inv_d;
  __nv_bfloat16* y;
  float* part;               // [grid][2][SLOT_FLOATS]
  unsigned int* counters;    // [tiles]
  unsigned int* status;
  unsigned long long budget_ns;
  int withhold;
};

template <int MPAD, int HALVES, int STAGES>
struct alignas(8) Bars {
  uint64_t full[STAGES], empty[STAGES];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t ssq_full[2], ssq_empty[2];
  uint64_t drain;
  float ssq[2][MPAD];
  uint32_t tmem_base;
  int abort_flag;
  int epi_ok[2];
  int last_flag[2];
};

__device__ __forceinline__ long long it_begin(int c, const Params& p) {
  return static_cast<long long>(c) * p.total / p.grid;
}
// CTA whose iteration range holds iteration `it`
__device__ __forceinline__ int owner_of(long long it, const Params& p) {
  return static_cast<int>(((it + 1) * p.grid - 1) / p.total);
}

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, unsigned long long budget) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > budget) return;
  }
}

template <int MPAD>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float (&v)[MPAD]) {
  if constexpr (MPAD == 16) {
    uint32_t r[16];
    tmem_ld16(taddr, r);
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
  } else {
#pragma unroll
    for (int c = 0; c < MPAD; c += 32) {
      uint32_t r[32];
      tmem_ld32(taddr + c, r);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 32; ++j) v[c + j] = __uint_as_float(r[j]);
    }
  }
}

template <int MPAD, int HALVES>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                  const Params p) {
  using C = Cfg<MPAD, HALVES>;
  constexpr int STAGES = C::STAGES;
  using B = Bars<MPAD, HALVES, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  B& bars = *reinterpret_cast<B*>(smem + STAGES * C::STAGE_BYTES);
  auto stage_w = [&](int s) { return smem + s * C::STAGE_BYTES; };
  auto stage_x = [&](int s) { return smem + s * C::STAGE_BYTES + C::W_BYTES; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const long long it0 = it_begin(cta, p);
  const long long it1 = it_begin(cta + 1, p);

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
          mbar_arrive_expect_tx(&bars.full[s], C::STAGE_BYTES);
          tma_load_2d(stage_x(s), &tmap_x, &bars.full[s], kb * BK, 0);
#pragma unroll
          for (int bx = 0; bx < 2 * HALVES; ++bx)
            tma_load_2d_hint(stage_w(s) + bx * W_BOX_BYTES, &tmap_w, &bars.full[s], tile * 128 * HALVES + bx * 64,
                             kb * BK, w_policy);
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
        if (row < MPAD) {
          const uint4* rp = reinterpret_cast<const uint4*>(stage_x(s) + row * 128);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 v = rp[c];
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float a = bf16lo_to_f32(w[j]), bb = bf16hi_to_f32(w[j]);
              acc = fmaf(a, a, acc);
              acc = fmaf(bb, bb, acc);
            }
          }
        }
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
      const int col = tile * 128 + n;            // output column
      const bool whole = (kb0 == 0 && kb1 == p.kblocks);
      if (whole) {
#pragma unroll
        for (int m = 0; m < MPAD; ++m) {
          if (m >= p.M) break;
          const float r = inv_rms(bars.ssq[b][m], p.inv_d, p.eps);
          float v;
          if (HALVES == 2) v = silu_f32(acc[0][m] * r) * (acc[1][m] * r);
          else v = acc[0][m] * r;
          if (col < p.nout) p.y[static_cast<int64_t>(m) * p.nout + col] = __float2bfloat16_rn(v);
        }
        mbar_arrive(&bars.ssq_empty[b]);
        continue;
      }
      // split tile: publish this CTA's partial, then the last arrival finishes it
      const int slot = cta * 2 + (seg == 0 ? 0 : 1);
      float* part = p.part + static_cast<int64_t>(slot) * C::SLOT_FLOATS;
#pragma unroll
      for (int h = 0; h < HALVES; ++h)
#pragma unroll
        for (int m = 0; m < MPAD; ++m)
          if (m < p.M) __stcg(part + (h * MPAD + m) * 128 + n, acc[h][m]);
      if (et < MPAD) __stcg(part + HALVES * MPAD * 128 + et, bars.ssq[b][et]);
      mbar_arrive(&bars.ssq_empty[b]);
      __threadfence();
      named_bar_sync(1, 128);
      const int c_first = owner_of(static_cast<long long>(tile) * p.kblocks, p);
      const int c_last = owner_of(static_cast<long long>(tile + 1) * p.kblocks - 1, p);
      if (et == 0) {
        const unsigned prev = atomicAdd(&p.counters[tile], 1u);
        bars.last_flag[seg & 1] = (prev == static_cast<unsigned>(c_last - c_first)) ? 1 : 0;
      }
      named_bar_sync(1, 128);
      if (!bars.last_flag[seg & 1]) continue;
      __threadfence();
#pragma unroll 1
      for (int m = 0; m < p.M && m < MPAD; ++m) {
        float tot[HALVES];
        float ssq = 0.f;
#pragma unroll
        for (int h = 0; h < HALVES; ++h) tot[h] = 0.f;
#pragma unroll 1
        for (int c = c_first; c <= c_last; ++c) {
          const long long cb = it_begin(c, p);
          const int cslot = c * 2 + (cb >= static_cast<long long>(tile) * p.kblocks ? 0 : 1);
          const float* cp = p.part + static_cast<int64_t>(cslot) * C::SLOT_FLOATS;
#pragma unroll
          for (int h = 0; h < HALVES; ++h) tot[h] += __ldcg(cp + (h * MPAD + m) * 128 + n);
          ssq += __ldcg(cp + HALVES * MPAD * 128 + m);
        }
        const float r = inv_rms(ssq, p.inv_d, p.eps);
        float v;
        if (HALVES == 2) v = silu_f32(tot[0] * r) * (tot[1] * r);
        else v = tot[0] * r;
        if (col < p.nout) p.y[static_cast<int64_t>(m) * p.nout + col] = __float2bfloat16_rn(v);
      }
      if (et == 0) p.counters[tile] = 0u;   // ready for the next call
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
  return 1024 + C::STAGES * C::STAGE_BYTES + sizeof(Bars<MPAD, HALVES, C::STAGES>);
}

struct Layout {
  int tiles, kblocks, grid;
  long long total;
  size_t counters_off, part_off, bytes;
};

template <int MPAD, int HALVES>
Layout layout_for(int64_t d, int64_t ncols, int num_sms) {
  Layout L;
  L.tiles = static_cast<int>(ncols / (128 * HALVES));
  L.kblocks = static_cast<int>(d / BK);
  L.total = static_cast<long long>(L.tiles) * L.kblocks;
  L.grid = static_cast<int>(L.total < num_sms ? L.total : num_sms);
  L.counters_off = kWsHeaderBytes;
  L.part_off = L.counters_off + (static_cast<size_t>(L.tiles) * 4 + 255) / 256 * 256;
  L.bytes = L.part_off + static_cast<size_t>(L.grid) * 2 * Cfg<MPAD, HALVES>::SLOT_FLOATS * 4;
  return L;
}

template <int MPAD, int HALVES>
cudaError_t launch_impl(const CallArgs& a) {
  const Layout L = layout_for<MPAD, HALVES>(a.d, a.ncols, a.num_sms);
  if (a.ws_bytes < L.bytes) return cudaErrorInvalidValue;
  CUtensorMap tx, tw;
  if (!make_tmap_2d(&tx, a.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.M, a.d, MPAD, BK)) return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tw, a.Wp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.d, a.ncols, BK, 64))
    return cudaErrorInvalidValue;
  Params p;
  p.M = static_cast<int>(a.M);
  p.d = static_cast<int>(a.d);
  p.ncols = static_cast<int>(a.ncols);
  p.nout = static_cast<int>(a.N);
  p.kblocks = L.kblocks;
  p.tiles = L.tiles;
  p.total = L.total;
  p.grid = L.grid;
  p.eps = a.eps;
  p.inv_d = 1.0f / static_cast<float>(a.d);
  p.y = static_cast<__nv_bfloat16*>(a.y);
  uint8_t* ws = static_cast<uint8_t*>(a.ws);
  p.status = reinterpret_cast<unsigned int*>(ws);
  p.counters = reinterpret_cast<unsigned int*>(ws + L.counters_off);
  p.part = reinterpret_cast<float*>(ws + L.part_off);
  p.budget_ns = a.budget_ns;
  p.withhold = a.withhold;
  constexpr size_t SMEM = smem_bytes<MPAD, HALVES>();
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<MPAD, HALVES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(SMEM));
  if (e != cudaSuccess) return e;
  decode_kernel<MPAD, HALVES><<<L.grid, NUM_THREADS, SMEM, a.stream>>>(tx, tw, p);
  return cudaGetLastError();
}

template <int MPAD>
cudaError_t launch_halves(const CallArgs& a) {
  return a.swiglu ? launch_impl<MPAD, 2>(a) : launch_impl<MPAD, 1>(a);
}

}  // namespace dec

int decode_mpad(int64_t M) { return M <= 16 ? 16 : (M <= 32 ? 32 : 64); }

size_t decode_workspace_bytes(int64_t M, int64_t d, int64_t ncols, bool swiglu, int num_sms) {
  const int mp = decode_mpad(M);
  if (swiglu) {
    if (mp == 16) return dec::layout_for<16, 2>(d, ncols, num_sms).bytes;
    if (mp == 32) return dec::layout_for<32, 2>(d, ncols, num_sms).bytes;
    return dec::layout_for<64, 2>(d, ncols, num_sms).bytes;
  }
  if (mp == 16) return dec::layout_for<16, 1>(d, ncols, num_sms).bytes;
  if (mp == 32) return dec::layout_for<32, 1>(d, ncols, num_sms).bytes;
  return dec::layout_for<64, 1>(d, ncols, num_sms).bytes;
}

cudaError_t launch_decode(const CallArgs& a) {
  const int mp = decode_mpad(a.M);
  if (mp == 16) return dec::launch_halves<16>(a);
  if (mp == 32) return dec::launch_halves<32>(a);
  return dec::launch_halves<64>(a);
}

}  // namespace fn
