// Pieces shared by the two small-M (decode) kernels: the bf16-weight kernel
// (decode.cu) and the fp8-weight kernel (decode_fp8.cu).
//
// Both split the weight stream over every SM with the same stream-K partition
// of (column tile, k block) iterations and hand tiles whose k range is split
// between CTAs to one fix-up kernel, defined here: each contributing CTA
// writes its fp32 partial accumulators and partial sums of squares to a
// workspace slot, and the fix-up adds them in ascending k order (a fixed order,
// so repeated calls are bit-identical), applies the deferred 1/rms (FlashNorm
// talk summary, Proposal 2) and, for the gated projection, SwiGLU.
#pragma once
#include <atomic>
#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "nvfp4.cuh"
#include "ptx.cuh"

namespace fn {
namespace dec {

constexpr int BK = 64;   // k rows per pipeline stage of the bf16 kernel

// Wait sites reported in the status word (bits 8..15) on a timeout.
enum : unsigned { kSiteProdEmpty = 1, kSiteMmaAccEmpty, kSiteMmaFull, kSiteRedFull, kSiteRedSsqEmpty,
                  kSiteEpiAccFull, kSiteEpiSsqFull, kSiteDrain, kSiteMmaConv, kSiteConvFull,
                  kSiteConvScaleEmpty, kSiteScaleFull };

struct Params {
  int M, d, ncols, nout;
  int kblocks, tiles;
  long long total;   // tiles * kblocks
  int grid;
  float eps, inv_d;
  __nv_bfloat16* y;
  float* part;               // [grid][2][slot_floats]
  unsigned int* status;
  unsigned long long budget_ns;
  int withhold;
  const uint8_t* wp;         // folded weight base (L2 prefetch addresses)
  int prefetch_iters;        // k-blocks per CTA prefetched into L2 before the dependency wait
  int prefetch_mode;         // 0 none, 1 TMA prefetch, 2 per-thread prefetch from idle warps
  const float* scales;       // fp8: block scales [d/128][ncols/128]
  int cluster;               // > 1: split-K inside clusters of this many CTAs, one tile each
  int narrow;                // (total + 1) * grid fits 32 bits: partition arithmetic in 32 bits
  const __nv_bfloat16* x;    // the activations (read directly by the x-splitting kernel)
  uint8_t* xhilo;            // fp8, split once per call: e4m3 x_hi / x_lo rows [kblocks][2 MPAD][128]
  float* xfac;               // fp8, split once per call: 2^-e per [kblock][row]
  uint8_t* yq;               // NVFP4 output (SwiGLU only; y is null then): codes [M][nout / 2]
  uint8_t* ysf;              //   and e4m3 scale codes [M][nout / 16]
  const float* gscale;       //   global scale (one fp32 value in device memory)
  float* part_out;           // partial output: fp32 [M][ncols] accumulators, then [M] sums of squares
  const uint8_t* wsf;        // MXFP8 weights: ue8m0 scale chunks (k groups, then 128-column blocks)
  uint8_t* xsf;              // MXFP8 path, x split once per call: ue8m0 scale chunk per k group
  int sf_chunked;            // NVFP4 output: scale bytes in the 128x4 chunked layout (else row-major)
};

// One partial-result slot: float4 groups [half][row / 4][column] for the
// HALVES x MPAD x 128 accumulators, then MPAD partial sums of squares.
template <int MPAD, int HALVES>
__host__ __device__ constexpr int slot_floats() {
  return ((HALVES * MPAD * 128 + MPAD) + 31) / 32 * 32;
}

// First iteration of CTA c.  The 32-bit forms give the same values; they only
// avoid 64-bit division where the products fit.
__host__ __device__ __forceinline__ long long it_begin(int c, const Params& p) {
  if (p.narrow) return static_cast<unsigned>(c) * static_cast<unsigned>(p.total) / static_cast<unsigned>(p.grid);
  return static_cast<long long>(c) * p.total / p.grid;
}
// CTA whose iteration range holds iteration `it`
__device__ __forceinline__ int owner_of(long long it, const Params& p) {
  if (p.narrow)
    return static_cast<int>((static_cast<unsigned>(it + 1) * static_cast<unsigned>(p.grid) - 1u) /
                            static_cast<unsigned>(p.total));
  return static_cast<int>(((it + 1) * p.grid - 1) / p.total);
}
inline bool partition_is_narrow(long long total, int grid) {
  return (total + 1) * static_cast<long long>(grid) < (1ll << 32);
}

// Wait for a teardown barrier without reporting: the kernel is leaving anyway.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, unsigned long long budget) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > budget) return;
  }
}

// Copy the staged output rows of one 128-column tile to y with 16-byte
// stores: 16 consecutive threads write one 256-byte row segment.  `nthr`
// threads of the epilogue group take part, `et` is this thread's index.
__device__ __forceinline__ void store_tile_rows(const __nv_bfloat16* ybuf, const Params& p, int tile, int et,
                                                int nthr) {
  const int col0 = tile * 128;
  const int chunks = p.M * 16;
  for (int i = et; i < chunks; i += nthr) {
    const int m = i >> 4, c16 = i & 15;
    if (col0 + c16 * 8 < p.nout) {
      const uint4 v = *reinterpret_cast<const uint4*>(ybuf + m * 128 + c16 * 8);
      *reinterpret_cast<uint4*>(p.y + static_cast<int64_t>(m) * p.nout + col0 + c16 * 8) = v;
    }
  }
}

// NVFP4 form of store_tile_rows: the staged codes ([MPAD rows][64 bytes], the
// tile's 128 columns) and scale bytes ([MPAD rows][8 bytes] after them) go to
// yq and ysf with 16- and 8-byte stores.
__device__ __forceinline__ void store_tile_fp4(const uint8_t* qbuf, int mpad, const Params& p, int tile, int et,
                                               int nthr) {
  const int64_t qrow = p.nout / 2, srow = p.nout / kFp4Block;
  for (int i = et; i < p.M * 5; i += nthr) {
    const int m = i / 5, c = i - 5 * (i / 5);
    if (c < 4) {
      *reinterpret_cast<uint4*>(p.yq + m * qrow + tile * 64 + c * 16) =
          *reinterpret_cast<const uint4*>(qbuf + m * 64 + c * 16);
    } else {
      fp4_store_sf8(p.ysf, m, tile * 8, static_cast<int>(srow), p.sf_chunked != 0,
                    *reinterpret_cast<const uint2*>(qbuf + mpad * 64 + m * 8));
    }
  }
}

// Stage row m of a tile's NVFP4 output from the 128 epilogue threads that
// hold column n's value v (n = 0..127 across 4 warps; all lanes call).
__device__ __forceinline__ void stage_fp4(uint8_t* qbuf, int mpad, int m, int n, float v, float gs) {
  uint32_t pair;
  const uint32_t sf = fp4_quantize_lane16(v, gs, pair);
  if ((n & 1) == 0) qbuf[m * 64 + (n >> 1)] = static_cast<uint8_t>(pair);
  if ((n & 15) == 0) qbuf[mpad * 64 + m * 8 + (n >> 4)] = static_cast<uint8_t>(sf);
}

// COLS consecutive fp32 TMEM columns of this warp's 32 lanes (16 or a
// multiple of 32).
template <int COLS>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float (&v)[COLS]) {
  if constexpr (COLS == 16) {
    uint32_t r[16];
    tmem_ld16(taddr, r);
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
  } else {
    static_assert(COLS % 32 == 0, "16 or a multiple of 32 columns");
#pragma unroll
    for (int c = 0; c < COLS; c += 32) {
      uint32_t r[32];
      tmem_ld32(taddr + c, r);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 32; ++j) v[c + j] = __uint_as_float(r[j]);
    }
  }
}

// Fix-up of the tiles whose k range was split between CTAs.  One thread per
// (tile, row group of 4, column): it loads the float4 partials of every
// contributing CTA (up to four in flight at once), adds them in ascending k
// order together with the partial sums of squares of its four rows, applies
// 1/rms (and SwiGLU) and stores four bf16 outputs.
constexpr int FIX_THREADS = 128;

// OUT: bf16 y, NVFP4 codes and scales (SwiGLU only), or fp32 partials (OutKind).
template <int MPAD, int HALVES, int OUT = kOutBf16>
__global__ void __launch_bounds__(FIX_THREADS) decode_fixup_kernel(const Params p) {
  static_assert(OUT != kOutNvfp4 || HALVES == 2, "NVFP4 output is a SwiGLU epilogue");
  static_assert(OUT != kOutPartial || HALVES == 1, "partial output: plain projection of the stored columns");
  constexpr int SLOT = slot_floats<MPAD, HALVES>();
  // Let the next kernel in the stream launch now: its CTAs take SMs as the
  // stream-K CTAs leave and prefetch their weights into L2 meanwhile.  All
  // CTAs of the stream-K grid are resident by now (each triggered this
  // launch after its own start), so no generation can starve another.
  grid_launch_dependents();
  grid_dependency_wait();        // the partials of the stream-K kernel are complete and visible
  const int Q = (p.M + 3) >> 2;
  const long long gid = static_cast<long long>(blockIdx.x) * FIX_THREADS + threadIdx.x;
  const int n = static_cast<int>(gid & 127);
  const long long rest = gid >> 7;
  const int q = static_cast<int>(rest % Q);
  const int tile = static_cast<int>(rest / Q);
  if (tile >= p.tiles) return;
  const long long t_it0 = static_cast<long long>(tile) * p.kblocks;
  const int c_first = owner_of(t_it0, p);
  const int c_last = owner_of(t_it0 + p.kblocks - 1, p);
  if (c_first == c_last) return;   // finished by the stream-K kernel itself
  float4 acc[HALVES];
#pragma unroll
  for (int h = 0; h < HALVES; ++h) acc[h] = make_float4(0.f, 0.f, 0.f, 0.f);
  float4 ss = make_float4(0.f, 0.f, 0.f, 0.f);
  auto add = [](float4& t, const float4& v) { t.x += v.x; t.y += v.y; t.z += v.z; t.w += v.w; };
  constexpr int CB = 4;
  for (int c0 = c_first; c0 <= c_last; c0 += CB) {
    float4 v[CB][HALVES], s4[CB];
#pragma unroll
    for (int j = 0; j < CB; ++j) {
      const int c = c0 + j;
      if (c <= c_last) {
        const int slot = c * 2 + (it_begin(c, p) >= t_it0 ? 0 : 1);
        const float4* base = reinterpret_cast<const float4*>(p.part + static_cast<int64_t>(slot) * SLOT);
#pragma unroll
        for (int h = 0; h < HALVES; ++h) v[j][h] = __ldcg(base + (h * (MPAD / 4) + q) * 128 + n);
        s4[j] = __ldcg(base + HALVES * (MPAD / 4) * 128 + q);
      }
    }
#pragma unroll
    for (int j = 0; j < CB; ++j) {
      if (c0 + j <= c_last) {
#pragma unroll
        for (int h = 0; h < HALVES; ++h) add(acc[h], v[j][h]);
        add(ss, s4[j]);
      }
    }
  }
  const float a0[4] = {acc[0].x, acc[0].y, acc[0].z, acc[0].w};
  const float a1[4] = {acc[HALVES - 1].x, acc[HALVES - 1].y, acc[HALVES - 1].z, acc[HALVES - 1].w};
  const float sq[4] = {ss.x, ss.y, ss.z, ss.w};
  const int col = tile * 128 + n;
  if constexpr (OUT == kOutPartial) {
    // the summed fp32 accumulators and sums of squares, not post-scaled
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int m = 4 * q + i;
      if (m >= p.M) break;
      p.part_out[static_cast<int64_t>(m) * p.ncols + col] = a0[i];
      if (tile == 0 && n == 0) p.part_out[static_cast<int64_t>(p.M) * p.ncols + m] = sq[i];
    }
    return;
  }
  const float gs = OUT == kOutNvfp4 ? __ldg(p.gscale) : 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = 4 * q + i;
    if (m >= p.M) break;            // uniform: the block is one (tile, row group)
    const float r = inv_rms(sq[i], p.inv_d, p.eps);
    float v = a0[i] * r;
    if (HALVES == 2) v = silu_f32(v) * (a1[i] * r);
    if constexpr (OUT == kOutNvfp4) {
      // NVFP4 output (SwiGLU: every tile column is an output column)
      uint32_t pair;
      const uint32_t sf = fp4_quantize_lane16(v, gs, pair);
      if ((n & 1) == 0) p.yq[static_cast<int64_t>(m) * (p.nout / 2) + (col >> 1)] = static_cast<uint8_t>(pair);
      if ((n & 15) == 0)
        p.ysf[fp4_sf_offset(m, col >> 4, p.nout / kFp4Block, p.sf_chunked != 0)] = static_cast<uint8_t>(sf);
    } else if (col < p.nout) {
      p.y[static_cast<int64_t>(m) * p.nout + col] = __float2bfloat16_rn(v);
    }
  }
}

// Whether some tile's k range is split between CTAs of the stream-K grid
// (then the fix-up kernel must run).
inline bool any_split_tile(int grid, long long total, int kblocks) {
  if (grid > total / kblocks) return true;   // more CTAs than tiles
  for (int c = 0; c < grid; ++c) {
    const long long b0 = static_cast<long long>(c) * total / grid;
    const long long b1 = static_cast<long long>(c + 1) * total / grid;
    if ((b0 % kblocks) != 0 || (b1 % kblocks) != 0) return true;
  }
  return false;
}

// Launch the fix-up for the stream-K grid described by `p`.
template <int MPAD, int HALVES, int OUT = kOutBf16>
cudaError_t launch_fixup(const Params& p, cudaStream_t stream) {
  const long long threads = static_cast<long long>(p.tiles) * 128 * ((p.M + 3) / 4);
  const unsigned fgrid = static_cast<unsigned>((threads + FIX_THREADS - 1) / FIX_THREADS);
  return launch_pdl(decode_fixup_kernel<MPAD, HALVES, OUT>, fgrid, FIX_THREADS, 0, stream, p);
}

// Whether `tiles` clusters of S CTAs can all be resident at once (cached per
// device and cluster size).
template <auto Kernel>
bool clusters_fit(int S, int tiles, int threads, size_t smem) {
  static std::atomic<int> cache[64][9];   // 0 unknown, else max active clusters + 1
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64 || S > 8) return false;
  int v = cache[dev][S].load(std::memory_order_relaxed);
  if (v == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(tiles * S));
    cfg.blockDim = dim3(static_cast<unsigned>(threads));
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(S);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, Kernel, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
    v = n + 1;
    cache[dev][S].store(v, std::memory_order_relaxed);
  }
  return v - 1 >= tiles;
}

// Workspace needed by a decode call: the header and two partial slots per CTA
// (upper bound over both kernels: the fp8 kernel's 128-row k blocks give at
// most as many CTAs as the bf16 kernel's 64-row blocks).
template <int MPAD, int HALVES>
size_t workspace_bytes(int64_t d, int64_t ncols, int num_sms) {
  const long long tiles = ncols / (128 * HALVES);
  const long long total = tiles * (d / BK);
  const long long grid = total < num_sms ? total : num_sms;
  return kWsHeaderBytes + static_cast<size_t>(grid) * 2 * slot_floats<MPAD, HALVES>() * 4;
}

}  // namespace dec
}  // namespace fn
