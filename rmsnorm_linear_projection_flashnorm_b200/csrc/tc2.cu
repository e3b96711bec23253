// Fused RMSNorm + projection, tensor-core tile path on pairs of SMs, sm_100a.
//
// Same arithmetic and the same explicit joins as tc.cu (FlashNorm talk
// summary, Proposal 2: the matmul on raw x on the tensor cores, each row's
// sum of squares from the same staged x tiles on the CUDA cores, 1/rms after
// both are complete; optional SwiGLU epilogue of the FlashInfer PR #5521
// analysis), with the tile computed by the tensor cores of two SMs together
// (tcgen05.mma.cta_group::2, a 2-CTA cluster): a 256 x 256 output tile per
// pair, 128 rows per CTA.  Each CTA stages only its own 128 x 64 x tile and its
// own 64 x 128 half of the weight tile, so an SM moves 32 KB from L2 per
// 64-deep k step instead of 48 KB for the same flops; for SwiGLU the gate
// columns of a tile sit in CTA 0 and the up columns in CTA 1.  The wide form
// computes a 256 x 512 tile with two pair MMAs per K step (each CTA stages two
// 128-column halves, 48 KB per k step for twice the flops) into one
// 512-column accumulator.
//
// Joins (all bounded waits; a CTA that gives up raises its partner's abort
// flag too):
//   * both CTAs' TMA loads of a stage complete on CTA 0's `full` barrier
//     (which expects the pair's bytes); CTA 0's MMA thread waits there before
//     it issues the pair MMA, which reads both CTAs' tiles; CTA 0's reducers
//     wait there too;
//   * the MMA commit of a stage arrives on `mdone` in both CTAs: CTA 1's
//     reducers wait there for their x tile (it has landed, and it stays until
//     their own arrival frees the stage), so no thread has to signal the
//     other CTA per stage (a remote arrive with release semantics costs a
//     cluster-scope fence, which on the per-stage path halved the
//     throughput);
//   * the MMA commit arrives on `empty` in both CTAs (with the local
//     reducers' arrivals the stage may be refilled) and, per tile, on
//     `acc_full` in both CTAs;
//   * each CTA's epilogue waits on its own `acc_full` and `ssq_full` (the
//     join the FlashNorm talk's bug lacked), and releases its TMEM buffer to
//     CTA 0's `acc_empty` (CTA 1's epilogue arrives remotely once its 128
//     threads have read the buffer).
//
// Layout per CTA: 10 warps, as tc.cu.
//   warp 0      TMA producer (own x rows, own weight columns), 7 stages of 32 KB
//               (wide: 4 stages of 48 KB)
//   warp 1      TMEM owner; in CTA 0 the pair-MMA issuer (M=256 N=256 K=16; wide:
//               two per K step)
//   warps 2-5   sum-of-squares reducers, one thread per row of this CTA
//   warps 6-9   epilogue: TMEM -> registers, post-scale (+SwiGLU), bf16 store
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace fn {
namespace tc2 {

constexpr int BM = 128;                  // rows per CTA (256 per pair)
constexpr int BK = 64;
constexpr int A_BYTES = BM * BK * 2;     // 16 KB
constexpr int B_BOX_BYTES = 64 * BK * 2; // 8 KB: 64 columns x 64 k rows
constexpr int HALF_B = 2 * B_BOX_BYTES;  // 16 KB: 128 weight columns per CTA and MMA
constexpr int NUM_THREADS = 320;
constexpr int TMEM_COLS = 512;
constexpr int MMA_N = 256;               // columns of one pair MMA (128 from each CTA)

// Tile shapes.  Narrow: a 256 x 256 output tile per pair, one pair MMA per K
// step, two TMEM accumulators (the epilogue of one tile overlaps the next).
// Wide: 256 x 512, two pair MMAs per K step into one 512-column accumulator,
// so each staged byte feeds a third more flops (the kernel is bound by the
// operand delivery rate into the SMs) at the cost of an epilogue that the
// next tile's MMAs wait for.
template <bool WIDE>
struct Shape {
  static constexpr int H = WIDE ? 2 : 1;             // pair MMAs per K step
  static constexpr int BN = H * MMA_N;               // output tile columns (stored weight columns)
  static constexpr int B_BYTES = H * HALF_B;         // weight bytes staged per CTA and stage
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = WIDE ? 4 : 7;
  static constexpr int NBUF = WIDE ? 1 : 2;          // TMEM accumulators
};

enum : unsigned { kSiteProdEmpty = 1, kSiteMmaAccEmpty, kSiteMmaFull, kSiteRedFull, kSiteRedSsqEmpty,
                  kSiteEpiAccFull, kSiteEpiSsqFull, kSiteDrain, kSiteExit };

struct Params {
  int M, d, ncols, nout;
  int num_m, num_n, num_tiles, kblocks;   // num_m: 256-row pair blocks
  int group_m;                            // tile raster: bands of group_m pair blocks
  float eps, inv_d;
  __nv_bfloat16* y;
  unsigned int* status;
  unsigned long long budget_ns;
  int withhold;
};

template <int STAGES>
struct alignas(8) Bars {
  uint64_t full[STAGES], empty[STAGES];
  uint64_t mdone[STAGES];                // the pair MMA of the stage completed (both CTAs)
  uint64_t acc_full[2], acc_empty[2];
  uint64_t ssq_full[2], ssq_empty[2];
  uint64_t drain;                        // the last pair MMA completed (both CTAs)
  uint64_t exit_bar;                     // the partner is done with this CTA's memory
  float ssq[2][BM];
  uint32_t tmem_base;
  int abort_flag;
  int epi_ok[2];                         // the epilogue group's common wait outcome, per buffer
};

template <bool WIDE>
constexpr size_t smem_bytes() {
  using Sh = Shape<WIDE>;
  return 1024 + Sh::STAGES * Sh::STAGE_BYTES + sizeof(Bars<Sh::STAGES>);
}
static_assert(smem_bytes<false>() <= 232448 && smem_bytes<true>() <= 232448, "shared memory budget");

__device__ __forceinline__ void tile_coords(int t, const Params& p, int& mb, int& nb) {
  const int per_group = p.group_m * p.num_n;
  const int group = t / per_group;
  const int first_m = group * p.group_m;
  const int gm = min(p.num_m - first_m, p.group_m);
  const int r = t - group * per_group;
  mb = first_m + r % gm;
  nb = r / gm;
}

// Bounded wait polling without suspending, for the threads on the pair's
// critical path (the MMA issuer and the forwarder of CTA 1's stages).
__device__ __forceinline__ bool mbar_wait_spin(uint64_t* bar, uint32_t parity, const WaitCtl& c, unsigned site) {
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*c.abort_flag) return false;
    if (globaltimer_ns() - t0 > c.budget_ns) {
      raise_timeout(c, site);
      return false;
    }
  }
}

// Bounded wait that ignores the abort flag: only for draining this pair's own
// asynchronous work before teardown.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, unsigned long long budget) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait_cluster(bar, parity)) {
    if (globaltimer_ns() - t0 > budget) return;
  }
}

template <bool SWIGLU, bool WIDE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    tc2_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
               const Params p) {
  using Sh = Shape<WIDE>;
  constexpr int STAGES = Sh::STAGES, STAGE_BYTES = Sh::STAGE_BYTES, BN = Sh::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars<STAGES>& bars = *reinterpret_cast<Bars<STAGES>*>(smem + STAGES * STAGE_BYTES);
  auto stage_a = [&](int s) { return smem + s * STAGE_BYTES; };
  auto stage_b = [&](int s) { return smem + s * STAGE_BYTES + A_BYTES; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();          // 0: MMA issuer of the pair
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.empty[s], 1 + 4);   // pair-MMA commit + one arrival per reducer warp
      mbar_init(&bars.mdone[s], 1);       // pair-MMA commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars.acc_full[b], 1);
      mbar_init(&bars.acc_empty[b], 128 + 1);   // CTA 0's epilogue threads + CTA 1's epilogue
      mbar_init(&bars.ssq_full[b], 128);
      mbar_init(&bars.ssq_empty[b], 128);
    }
    mbar_init(&bars.drain, 1);
    mbar_init(&bars.exit_bar, 1);
    bars.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmap_x);
    tma_prefetch_desc(&tmap_w);
  }
  if (warp == 1) {
    tmem_alloc_pair(&bars.tmem_base, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  // both CTAs' barriers are initialised before any cross-CTA arrival
  cluster_sync_all();
  tc_fence_after();
  grid_dependency_wait();
  grid_launch_dependents();
  const uint32_t tmem_base = bars.tmem_base;
  WaitCtl ctl{&bars.abort_flag, p.status, p.budget_ns};
  ctl.peer_abort = dsmem_addr(&bars.abort_flag, rank ^ 1u);

  if (warp == 0) {
    // ------------------------------------------------------------ producer (own halves)
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0, issued = 0, last_ph = 0;
      bool ok = true;
      const uint32_t full0 = dsmem_addr(&bars.full[0], 0);   // CTA 0's barriers count both CTAs' bytes
      for (int t = pair; t < p.num_tiles && ok; t += npairs) {
        int mb, nb;
        tile_coords(t, p, mb, nb);
        const int row0 = mb * (2 * BM) + static_cast<int>(rank) * BM;
        // per pair MMA h, this CTA's 128 columns: [nb BN + h 256 + rank 128, +128)
        // (for SwiGLU the gate block in CTA 0, the matching up block in CTA 1)
        const int col0 = nb * BN + static_cast<int>(rank) * 128;
        for (int kb = 0; kb < p.kblocks; ++kb) {
          if (!mbar_wait_spin(&bars.empty[s], ph ^ 1, ctl, kSiteProdEmpty)) { ok = false; break; }
          if (rank == 0) mbar_arrive_expect_tx(&bars.full[s], 2 * STAGE_BYTES);
          const uint32_t fb = full0 + s * 8;
          tma_load_2d_pair(stage_a(s), &tmap_x, fb, kb * BK, row0);
#pragma unroll
          for (int h = 0; h < Sh::H; ++h) {
            tma_load_2d_pair(stage_b(s) + h * HALF_B, &tmap_w, fb, col0 + h * MMA_N, kb * BK);
            tma_load_2d_pair(stage_b(s) + h * HALF_B + B_BOX_BYTES, &tmap_w, fb, col0 + h * MMA_N + 64, kb * BK);
          }
          issued |= 1u << s;
          last_ph = (last_ph & ~(1u << s)) | (ph << s);
          if (++s == STAGES) { s = 0; ph ^= 1; }
        }
      }
      // no copy may still be landing in shared memory when the CTA exits: in
      // CTA 0 the stage barriers count both CTAs' copies; in CTA 1 the MMA that
      // consumed a stage completed after its copies landed
      for (int i = 0; i < STAGES; ++i)
        if (issued & (1u << i))
          drain_wait(rank == 0 ? &bars.full[i] : &bars.mdone[i], (last_ph >> i) & 1u, p.budget_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      if (rank == 0) {
        // -------------------------------------------------------- pair-MMA issuer
        constexpr uint32_t IDESC = idesc_bf16_f32(2 * BM, MMA_N, /*a MN-major*/ false, /*b MN-major*/ true);
        int s = 0;
        uint32_t ph = 0;
        bool ok = true;
        int i = 0;
        for (int t = pair; t < p.num_tiles && ok; t += npairs, ++i) {
          const int b = Sh::NBUF == 2 ? (i & 1) : 0;
          const uint32_t aph = Sh::NBUF == 2 ? (i >> 1) & 1 : i & 1;
          // CTA 1's epilogue arrives here after its TMEM loads completed (tcgen05.wait::ld),
          // so the buffer may be overwritten once the phase completes
          if (!mbar_wait_spin(&bars.acc_empty[b], aph ^ 1, ctl, kSiteMmaAccEmpty)) break;
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + b * BN;
          for (int kb = 0; kb < p.kblocks; ++kb) {
            if (!mbar_wait_spin(&bars.full[s], ph, ctl, kSiteMmaFull)) { ok = false; break; }
            tc_fence_after();
            const uint32_t a0 = smem_u32(stage_a(s));
            const uint32_t b0 = smem_u32(stage_b(s));
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              // A: this CTA's x rows, K-major (the partner's rows at the same offset)
              const uint64_t adesc = sdesc_sw128(a0 + kk * 32, 16, 1024);
#pragma unroll
              for (int h = 0; h < Sh::H; ++h) {
                // B: this CTA's 128 weight columns of MMA h, N-major, two 64-column boxes 8 KB apart
                const uint64_t bdesc = sdesc_sw128(b0 + h * HALF_B + kk * 2048, B_BOX_BYTES, 1024);
                umma_bf16_pair(d_tmem + h * MMA_N, adesc, bdesc, IDESC, (kb | kk) != 0);
              }
            }
            umma_commit_pair(&bars.empty[s], 0x3);
            umma_commit_pair(&bars.mdone[s], 0x3);
            if (++s == STAGES) { s = 0; ph ^= 1; }
          }
          if (!ok) break;
          umma_commit_pair(&bars.acc_full[b], 0x3);
        }
        umma_commit_pair(&bars.drain, 0x3);
        drain_wait(&bars.drain, 0, p.budget_ns);
      } else {
        drain_wait(&bars.drain, 0, p.budget_ns);   // the pair's last MMA no longer reads this CTA
      }
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------------ sum-of-squares reducers (own rows)
    const int row = (warp - 2) * 32 + lane;
    int s = 0;
    uint32_t ph = 0;
    int i = 0;
    bool ok = true;
    for (int t = pair; t < p.num_tiles && ok; t += npairs, ++i) {
      float acc = 0.f;
      for (int kb = 0; kb < p.kblocks; ++kb) {
        const bool landed = rank == 0 ? mbar_wait(&bars.full[s], ph, ctl, kSiteRedFull)
                                      : mbar_wait(&bars.mdone[s], ph, ctl, kSiteRedFull);
        if (!__all_sync(0xffffffffu, landed)) { ok = false; break; }
        acc += row_sumsq_sw128(stage_a(s), row);
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
    // ------------------------------------------------------------ epilogue (own rows)
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;       // tile row of this CTA == accumulator lane
    const int et = threadIdx.x - 192;    // 0..127
    const uint32_t acc_empty0 = dsmem_addr(&bars.acc_empty[0], 0);
    int i = 0;
    for (int t = pair; t < p.num_tiles; t += npairs, ++i) {
      int mb, nb;
      tile_coords(t, p, mb, nb);
      const int b = Sh::NBUF == 2 ? (i & 1) : 0;
      const uint32_t aph = Sh::NBUF == 2 ? (i >> 1) & 1 : i & 1;
      const int sb = i & 1;                 // sums-of-squares buffer
      const uint32_t sph = (i >> 1) & 1;
      // One thread waits and the whole epilogue group follows its decision, so
      // the group never splits at the named barrier or the .sync.aligned loads.
      if (et == 0) {
        bool ok = mbar_wait_spin(&bars.acc_full[b], aph, ctl, kSiteEpiAccFull);
        ok = ok && mbar_wait(&bars.ssq_full[sb], sph, ctl, kSiteEpiSsqFull);
        bars.epi_ok[sb] = ok ? 1 : 0;
      }
      named_bar_sync(1, 128);
      if (!bars.epi_ok[sb]) break;
      tc_fence_after();
      const float r = inv_rms(bars.ssq[sb][row], p.inv_d, p.eps);
      mbar_arrive(&bars.ssq_empty[sb]);
      const int grow = mb * (2 * BM) + static_cast<int>(rank) * BM + row;
      const bool row_ok = grow < p.M;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + b * BN;
      if constexpr (SWIGLU) {
        // accumulator columns of MMA h: [h 256, +128) gate, [h 256 + 128, +128) up,
        // output columns [nb BN/2 + h 128, +128).  Chunks of 32 columns; the next
        // chunk's TMEM loads are issued before this chunk's math, so their latency
        // hides under it (two register buffers).
        auto load_chunk = [&](int c, uint32_t(&gv)[32], uint32_t(&uv)[32]) {
          const int h = c / 128, cc = c % 128;
          tmem_ld32(taddr + h * MMA_N + cc, gv);
          tmem_ld32(taddr + h * MMA_N + 128 + cc, uv);
        };
        auto finish_chunk = [&](int c, const uint32_t(&gv)[32], const uint32_t(&uv)[32]) {
          const int ocol = nb * (BN / 2) + c;
          uint32_t o[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float g0 = __uint_as_float(gv[2 * j]) * r, g1 = __uint_as_float(gv[2 * j + 1]) * r;
            const float u0 = __uint_as_float(uv[2 * j]) * r, u1 = __uint_as_float(uv[2 * j + 1]) * r;
            o[j] = pack_bf16x2(silu_f32(g0) * u0, silu_f32(g1) * u1);
          }
          if (row_ok && ocol < p.nout) {
            uint4* dst = reinterpret_cast<uint4*>(p.y + static_cast<int64_t>(grow) * p.nout + ocol);
#pragma unroll
            for (int j = 0; j < 4; ++j) dst[j] = make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
          }
        };
        uint32_t ga[32], ua[32], gb[32], ub[32];
        load_chunk(0, ga, ua);
#pragma unroll 1
        for (int c = 0; c < BN / 2; c += 64) {
          tmem_ld_wait();                       // chunk c (buffer a) has landed
          load_chunk(c + 32, gb, ub);           // BN / 2 is a multiple of 64
          finish_chunk(c, ga, ua);
          tmem_ld_wait();                       // chunk c + 32 (buffer b)
          if (c + 64 < BN / 2) load_chunk(c + 64, ga, ua);
          finish_chunk(c + 32, gb, ub);
        }
      } else {
        __nv_bfloat16* yrow = p.y + static_cast<int64_t>(grow) * p.nout;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t v[32];
          tmem_ld32(taddr + c, v);
          tmem_ld_wait();
          const int col = nb * BN + c;
          if (row_ok && col < p.nout) {
            uint32_t o[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
              o[j] = pack_bf16x2(__uint_as_float(v[2 * j]) * r, __uint_as_float(v[2 * j + 1]) * r);
            uint4* dst = reinterpret_cast<uint4*>(yrow + col);
#pragma unroll
            for (int j = 0; j < 4; ++j) dst[j] = make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
          }
        }
      }
      // this CTA's 128 threads have read TMEM buffer b: release it to the MMA issuer
      tc_fence_before();
      if (rank == 0) {
        mbar_arrive(&bars.acc_empty[b]);
      } else {
        named_bar_sync(1, 128);
        if (et == 0) mbar_arrive_remote(acc_empty0 + b * 8);
      }
    }
  }

  // Teardown: every role of this CTA is done; wait (bounded) until the partner
  // is done with this CTA's memory too, then release TMEM in both CTAs.
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_remote(dsmem_addr(&bars.exit_bar, rank ^ 1u));
    drain_wait(&bars.exit_bar, 0, p.budget_ns);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

template <bool SWIGLU, bool WIDE>
cudaError_t launch_impl(const CallArgs& a) {
  constexpr int BN = Shape<WIDE>::BN;
  CUtensorMap tx, tw;
  if (!make_tmap_2d(&tx, a.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.M, a.d, BM, BK)) return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tw, a.Wp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.d, a.ncols, BK, 64))
    return cudaErrorInvalidValue;
  Params p;
  p.M = static_cast<int>(a.M);
  p.d = static_cast<int>(a.d);
  p.ncols = static_cast<int>(a.ncols);
  p.nout = static_cast<int>(a.N);
  p.num_m = static_cast<int>((a.M + 2 * BM - 1) / (2 * BM));
  p.num_n = static_cast<int>((a.ncols + BN - 1) / BN);
  p.num_tiles = p.num_m * p.num_n;
  p.kblocks = static_cast<int>(a.d / BK);
  // Raster band: as many 256-row blocks as keep the band's x rows within about
  // 40 MB of L2 (at most 16), so the weight columns are fetched from HBM once
  // per band while the band's x stays in L2.
  const int64_t band_rows = (40ll << 20) / (a.d * 2);
  p.group_m = static_cast<int>(band_rows / (2 * BM));
  if (p.group_m < 1) p.group_m = 1;
  if (p.group_m > 16) p.group_m = 16;
  p.eps = a.eps;
  p.inv_d = 1.0f / static_cast<float>(a.d);
  p.y = static_cast<__nv_bfloat16*>(a.y);
  p.status = static_cast<unsigned int*>(a.ws);
  p.budget_ns = a.budget_ns;
  p.withhold = a.withhold;
  constexpr size_t SMEM = smem_bytes<WIDE>();
  cudaError_t e = ensure_smem_limit<tc2_kernel<SWIGLU, WIDE>>(static_cast<int>(SMEM));
  if (e != cudaSuccess) return e;
  const int pairs = p.num_tiles < a.num_sms / 2 ? p.num_tiles : a.num_sms / 2;
  return launch_pdl(tc2_kernel<SWIGLU, WIDE>, static_cast<unsigned>(2 * pairs), NUM_THREADS, SMEM, a.stream, tx, tw,
                    p);
}

}  // namespace tc2

// 256 x 512 tiles where the k range is long enough to hide their
// non-overlapped epilogue: at d = 8192 (large prefill) they ran 17 % faster
// than 256 x 256 tiles; at d = 4096 (FFN, 4096 rows), with the epilogue's TMEM
// loads pipelined, about 1.5 % faster.
constexpr int64_t kWidePairTileMinD = 4096;

cudaError_t launch_tc_pair(const CallArgs& a) {
  const bool wide = a.pair_tile == 2 || (a.pair_tile == 0 && a.d >= kWidePairTileMinD);
  if (a.swiglu) return wide ? tc2::launch_impl<true, true>(a) : tc2::launch_impl<true, false>(a);
  return wide ? tc2::launch_impl<false, true>(a) : tc2::launch_impl<false, false>(a);
}

}  // namespace fn
