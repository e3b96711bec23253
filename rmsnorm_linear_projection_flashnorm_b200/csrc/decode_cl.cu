// Fused RMSNorm + projection, small-M path (M <= 64) for weights small enough
// that a whole-GPU stream-K partition would split most column tiles: column
// groups per thread-block cluster, k split across the cluster's CTAs, the
// partial sums reduced through distributed shared memory.  No fix-up kernel.
//
// Arithmetic as everywhere in this library (FlashNorm talk summary, Proposal 2
// "지연된 정규화"): the matmul runs on the raw activations, each row's sum of
// squares is reduced from the same staged x tiles, and 1/rms is applied to the
// finished sums.
//
// Work split.  The folded weight W' [d, ncols] is cut into 64-column boxes.
// Cluster c (S CTAs) owns T adjacent boxes (T * 64 columns); CTA rank r of the
// cluster streams the k blocks [r kblocks / S, (r + 1) kblocks / S) of all T
// boxes, so every CTA reads T * 64 contiguous columns per k row (DRAM
// locality) and no column's k range leaves its cluster.  Per 64-deep k block
// the tensor cores compute D[n, m] += W'^T[n, k] x^T[k, m] (swap-AB,
// tcgen05.mma M = 128 weight columns, N = MPAD activation rows, K = 16): boxes
// go to the MMA in pairs; an odd last box shares its MMA with box 0, whose
// duplicate rows are ignored.
//
// Reduction.  After its k range, each CTA pushes its fp32 partial of every
// column to the CTA of the cluster that finishes that column (rank j finishes
// columns [j CS, (j + 1) CS), CS = T * 64 / S) with st.shared::cluster, and
// its partial sums of squares to every CTA; one cluster barrier
// (release/acquire) later each CTA adds the S partials of its columns in rank
// order (= k order, so repeated calls give the same bits), applies 1/rms and
// stores bf16.
//
// Layout: 8 warps, as the stream-K decode kernel, during the k range:
//   warp 0      TMA producer
//   warp 1      TMEM owner and MMA issuer
//   warps 2-3   sum-of-squares reducers (one thread per activation row)
//   warps 4-7   (idle until the exchange)
// and then all 8 for the exchange (warp w reads TMEM lane quarter w mod 4, half
// of the rows each, and pushes 16-byte pieces) and the finish of this CTA's
// column share (one thread per column and group of four rows).
#include <cstddef>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "decode_common.cuh"

namespace fn {
namespace dcl {

using dec::BK;
using dec::Params;
constexpr int NUM_THREADS = 256;
constexpr int BOX_BYTES = 64 * BK * 2;    // 64 columns x 64 k rows, bf16 (8 KB)
constexpr int MAX_S = 8;                  // cluster sizes 2..8 (portable limit)
constexpr int SMEM_LIMIT = 227 * 1024;

template <int MPAD, int T>
struct Cfg {
  static_assert(T >= 1 && T <= 3, "one to three boxes per cluster");
  // weight slots per stage: T = 1 keeps a second (unused) slot, because an
  // M = 128 MMA reads 128 rows; odd T >= 3 stores box T-1 first so that its
  // MMA's upper half falls on box 0
  static constexpr int SLOTS = T == 1 ? 2 : T;
  static constexpr int GROUPS = (T + 1) / 2;                // M = 128 MMAs per K step
  static constexpr int W_BYTES = SLOTS * BOX_BYTES;
  static constexpr int X_BYTES = MPAD * BK * 2;
  static constexpr int STAGE_BYTES = W_BYTES + X_BYTES;     // a multiple of 1024
  // partials of this CTA's columns, written by the peers: [S][CS][RS] fp32
  // (S * CS = T * 64); a column's rows are contiguous (16-byte pushes and
  // reads), padded by four so that consecutive columns fall on different banks
  static constexpr int RS = MPAD + 4;
  static constexpr int RED_BYTES = T * 64 * RS * 4;
  static constexpr int SSQ_BYTES = MAX_S * MPAD * 4;        // [S][MPAD] fp32
  static constexpr int ACC_COLS = GROUPS * MPAD;
  static constexpr int TMEM_COLS = ACC_COLS <= 32 ? 32 : (ACC_COLS <= 64 ? 64 : 128);
  static constexpr int STAGES_FIT = (SMEM_LIMIT - 1024 - RED_BYTES - SSQ_BYTES - 1024) / STAGE_BYTES;
  // four stages (about 100 KB in flight per SM) streamed the weight fastest in
  // measurements; more only queue
  static constexpr int STAGES = STAGES_FIT > 4 ? 4 : STAGES_FIT;
  static_assert(STAGES >= 2, "pipeline needs two stages");
};

template <int STAGES, int MPAD>
struct alignas(16) Bars {
  uint64_t full[STAGES], empty[STAGES];
  uint64_t acc_full, ssq_full, drain;
  float ssq[MPAD];       // this CTA's partial sums of squares
  float rinv[MPAD];      // 1/rms of each row (after the exchange)
  uint32_t tmem_base;
  int abort_flag;
  int epi_ok;
};

template <int MPAD, int T>
constexpr size_t smem_bytes() {
  using C = Cfg<MPAD, T>;
  return 1024 + static_cast<size_t>(C::STAGES) * C::STAGE_BYTES + C::RED_BYTES + C::SSQ_BYTES +
         sizeof(Bars<C::STAGES, MPAD>);
}

// Slot of box b inside a stage, and the slot where MMA group g starts.
template <int T>
__host__ __device__ constexpr int slot_of_box(int b) {
  return (T % 2 == 1 && T >= 3) ? (b == T - 1 ? 0 : b + 1) : b;
}
template <int T>
__host__ __device__ constexpr int group_slot(int g) {
  return (T % 2 == 1 && T >= 3) ? (g == (T + 1) / 2 - 1 ? 0 : 2 * g + 1) : 2 * g;
}
// Box held by row `lane128` (0..127) of MMA group g, or -1 (duplicate rows).
template <int T>
__host__ __device__ constexpr int box_of_row(int g, int lane128) {
  const int lower = lane128 < 64;
  if (T % 2 == 1 && T >= 3 && g == (T + 1) / 2 - 1) return lower ? T - 1 : -1;
  if (T == 1) return lower ? 0 : -1;
  return 2 * g + (lower ? 0 : 1);
}

__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}
__device__ __forceinline__ void st_cluster_f32(uint32_t cluster_addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(cluster_addr), "f"(v) : "memory");
}
__device__ __forceinline__ void st_cluster_v4(uint32_t cluster_addr, float a, float b, float c, float d) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(cluster_addr), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

template <int MPAD, int T>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    decode_cl_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                     const Params p) {
  using C = Cfg<MPAD, T>;
  constexpr int STAGES = C::STAGES;
  using B = Bars<STAGES, MPAD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // [stages: weight slots, x tile][partials of this CTA's columns][partial sums of squares][barriers]
  constexpr int RS = C::RS;
  float* red = reinterpret_cast<float*>(smem + STAGES * C::STAGE_BYTES);
  float* ssqbuf = reinterpret_cast<float*>(smem + STAGES * C::STAGE_BYTES + C::RED_BYTES);
  B& bars = *reinterpret_cast<B*>(smem + STAGES * C::STAGE_BYTES + C::RED_BYTES + C::SSQ_BYTES);
  auto stage_w = [&](int s) { return smem + s * C::STAGE_BYTES; };
  auto stage_x = [&](int s) { return smem + s * C::STAGE_BYTES + C::W_BYTES; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int S = p.cluster;
  const uint32_t rank = cluster_ctarank();
  const int group = static_cast<int>(blockIdx.x) / S;
  const int box0 = group * T;                       // first 64-column box of the cluster
  const int CS = T * 64 / S;                        // columns each rank finishes
  const int kb0 = static_cast<int>(rank) * p.kblocks / S;
  const int kb1 = (static_cast<int>(rank) + 1) * p.kblocks / S;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bars.full[s], 1);
      mbar_init(&bars.empty[s], 1 + 2);   // MMA commit + two reducer warps
    }
    mbar_init(&bars.acc_full, 1);
    mbar_init(&bars.ssq_full, 64);
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
  // This CTA has started: peers may write its partials buffer once they have
  // waited on this arrival.
  cluster_arrive_relaxed();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Overlaps the previous kernel: an L2 prefetch of the k blocks that the
  // first ring of stages will load (the weight does not depend on the
  // previous kernel's output, and an L2 prefetch cannot return stale data).
  // Deeper prefetches measured slower: they compete with the previous call's
  // own weight stream.
  const int n_pf = min(min(p.prefetch_iters, STAGES), kb1 - kb0);
  if (p.prefetch_mode == 1 && warp == 0 && lane == 0) {
    const int n = n_pf;
    for (int i = 0; i < n; ++i)
      for (int b = 0; b < T; ++b) tma_prefetch_l2_2d(&tmap_w, (box0 + b) * 64, (kb0 + i) * BK);
  } else if (p.prefetch_mode == 2 && warp >= 2) {
    // one 128-byte line per thread and step: (k row, box)
    const int n = n_pf;
    const int total = n * BK * T;
    for (int i = threadIdx.x - 64; i < total; i += NUM_THREADS - 64) {
      const int b = i % T;
      const int r = i / T;   // k row within the prefetched range
      if ((box0 + b) * 64 < p.ncols) {
        const uint8_t* a = p.wp + (static_cast<int64_t>(kb0) * BK + r) * p.ncols * 2 + static_cast<int64_t>(box0 + b) * 128;
        asm volatile("prefetch.global.L2 [%0];" ::"l"(a));
      }
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
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&bars.empty[s], ph ^ 1, ctl, dec::kSiteProdEmpty)) break;
        mbar_arrive_expect_tx(&bars.full[s], C::X_BYTES + T * BOX_BYTES);
        tma_load_2d(stage_x(s), &tmap_x, &bars.full[s], kb * BK, 0);
#pragma unroll
        for (int b = 0; b < T; ++b)   // boxes past the weight are zero fill
          tma_load_2d_hint(stage_w(s) + slot_of_box<T>(b) * BOX_BYTES, &tmap_w, &bars.full[s], (box0 + b) * 64,
                           kb * BK, w_policy);
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
      constexpr uint32_t IDESC = idesc_bf16_f32(128, MPAD, /*a MN-major*/ true, /*b MN-major*/ false);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&bars.full[s], ph, ctl, dec::kSiteMmaFull)) { ok = false; break; }
        tc_fence_after();
        const uint32_t w0 = smem_u32(stage_w(s));
        const uint32_t x0 = smem_u32(stage_x(s));
#pragma unroll
        for (int g = 0; g < C::GROUPS; ++g) {
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // A = W'^T: two boxes one slot (8 KB) apart, N-major; K = 16 rows are 2048 B
            const uint64_t adesc = sdesc_sw128(w0 + group_slot<T>(g) * BOX_BYTES + kk * 2048, BOX_BYTES, 1024);
            // B = x^T: MPAD activation rows, K-major, 128-byte rows
            const uint64_t bdesc = sdesc_sw128(x0 + kk * 32, 16, 1024);
            umma_bf16(tmem_base + g * MPAD, adesc, bdesc, IDESC, (kb != kb0 || kk != 0) ? 1u : 0u);
          }
        }
        umma_commit(&bars.empty[s]);
        if (++s == STAGES) { s = 0; ph ^= 1; }
      }
      if (ok && kb1 > kb0) umma_commit(&bars.acc_full);
      umma_commit(&bars.drain);
      dec::drain_wait(&bars.drain, 0, p.budget_ns);
    }
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------------------------------------ sum-of-squares reducers
    const int row = (warp - 2) * 32 + lane;      // activation row
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    float acc = 0.f;
    for (int kb = kb0; kb < kb1; ++kb) {
      if (!__all_sync(0xffffffffu, mbar_wait(&bars.full[s], ph, ctl, dec::kSiteRedFull))) { ok = false; break; }
      if (row < MPAD && row < p.M) acc += row_sumsq_sw128(stage_x(s), row);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.empty[s]);
      if (++s == STAGES) { s = 0; ph ^= 1; }
    }
    if (row < MPAD) bars.ssq[row] = acc;
    if (ok && !p.withhold) mbar_arrive(&bars.ssq_full);
  }
  __syncwarp();

  // ------------------------------------------------------------ exchange
  if (threadIdx.x == 128) {
    bool ok = kb1 > kb0 && mbar_wait(&bars.acc_full, 0, ctl, dec::kSiteEpiAccFull);
    ok = ok && mbar_wait(&bars.ssq_full, 0, ctl, dec::kSiteEpiSsqFull);
    bars.epi_ok = ok ? 1 : 0;
  }
  cluster_wait();   // every CTA of the cluster has started
  __syncthreads();
  if (bars.epi_ok) {
    // TMEM -> registers -> the finishing CTA's buffer: warp w reads lane quarter
    // w mod 4 (its columns) and rows [h MPAD/2, (h + 1) MPAD/2), h = w div 4
    tc_fence_after();
    constexpr int HM = MPAD / 2;
    const int q = warp & 3, h = warp >> 2;
    const int l128 = q * 32 + lane;
    const uint32_t red_local = smem_u32(red);
    if (h * HM < p.M) {
#pragma unroll
      for (int g = 0; g < C::GROUPS; ++g) {
        uint32_t v[HM];
        __syncwarp();
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + g * MPAD + h * HM;
        if constexpr (HM == 8) tmem_ld8(taddr, v);
        else if constexpr (HM == 16) tmem_ld16(taddr, v);
        else tmem_ld32(taddr, v);
        tmem_ld_wait();
        const int b = box_of_row<T>(g, l128);
        if (b < 0 || (box0 + b) * 64 >= p.ncols) continue;
        const int n_local = b * 64 + (l128 & 63);
        const int j = n_local / CS, cc = n_local - j * CS;
        uint32_t dst;
        asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(dst) : "r"(red_local), "r"(j));
        dst += 4u * static_cast<uint32_t>((static_cast<int>(rank) * CS + cc) * RS + h * HM);
#pragma unroll
        for (int m4 = 0; m4 < HM / 4; ++m4) {
          if (h * HM + 4 * m4 >= p.M) break;
          st_cluster_v4(dst + 16u * m4, __uint_as_float(v[4 * m4]), __uint_as_float(v[4 * m4 + 1]),
                        __uint_as_float(v[4 * m4 + 2]), __uint_as_float(v[4 * m4 + 3]));
        }
      }
    }
    if (threadIdx.x < p.M) {
      const uint32_t ss_local =
          smem_u32(ssqbuf) + 4u * static_cast<uint32_t>(static_cast<int>(rank) * MPAD + threadIdx.x);
      const float ss = bars.ssq[threadIdx.x];
      for (int j = 0; j < S; ++j) {
        uint32_t dst;
        asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(dst) : "r"(ss_local), "r"(j));
        st_cluster_f32(dst, ss);
      }
    }
  }
  // Every CTA's pushes are complete and visible after this barrier.
  cluster_sync_all();

  // ------------------------------------------------------------ finish this rank's columns
  if (threadIdx.x < p.M) {
    float ss = 0.f;                               // partial sums of squares in rank (= k) order
#pragma unroll
    for (int r = 0; r < MAX_S; ++r)
      if (r < S) ss += ssqbuf[r * MPAD + threadIdx.x];
    bars.rinv[threadIdx.x] = inv_rms(ss, p.inv_d, p.eps);
  }
  __syncthreads();
  {
    // one thread per (column, group of four rows): 16-byte reads of the S
    // partials, four bf16 stores that a warp makes contiguous per row
    const int col0 = box0 * 64 + static_cast<int>(rank) * CS;
    const int M4 = (p.M + 3) >> 2;
    const int E = M4 * CS;
    for (int e = threadIdx.x; e < E; e += NUM_THREADS) {
      const int m4 = e / CS, cc = e - m4 * CS;
      const int col = col0 + cc;
      if (col >= p.nout) continue;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int r = 0; r < MAX_S; ++r) {
        if (r < S) {
          const float4 t = *reinterpret_cast<const float4*>(red + (r * CS + cc) * RS + 4 * m4);
          v.x += t.x;
          v.y += t.y;
          v.z += t.z;
          v.w += t.w;
        }
      }
      const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int m = 4 * m4 + i;
        if (m < p.M) p.y[static_cast<int64_t>(m) * p.nout + col] = __float2bfloat16_rn(vv[i] * bars.rinv[m]);
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

template <int MPAD, int T>
cudaError_t launch_impl(const CallArgs& a, int S) {
  CUtensorMap tx, tw;
  if (!make_tmap_2d(&tx, a.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.M, a.d, MPAD, BK)) return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tw, a.Wp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.d, a.ncols, BK, 64)) return cudaErrorInvalidValue;
  Params p = {};
  p.M = static_cast<int>(a.M);
  p.d = static_cast<int>(a.d);
  p.ncols = static_cast<int>(a.ncols);
  p.nout = static_cast<int>(a.N);
  p.kblocks = static_cast<int>(a.d / BK);
  const int boxes = static_cast<int>(a.ncols / 64);
  p.tiles = (boxes + T - 1) / T;          // column groups = clusters
  p.cluster = S;
  p.grid = p.tiles * S;
  p.eps = a.eps;
  p.inv_d = 1.0f / static_cast<float>(a.d);
  p.y = static_cast<__nv_bfloat16*>(a.y);
  p.status = reinterpret_cast<unsigned int*>(a.ws);
  p.budget_ns = a.budget_ns;
  p.withhold = a.withhold;
  p.wp = static_cast<const uint8_t*>(a.Wp);
  p.prefetch_iters = a.prefetch_iters;
  p.prefetch_mode = a.prefetch_mode;
  p.x = static_cast<const __nv_bfloat16*>(a.x);
  constexpr size_t SMEM = smem_bytes<MPAD, T>();
  const cudaError_t e = ensure_smem_limit<decode_cl_kernel<MPAD, T>>(static_cast<int>(SMEM));
  if (e != cudaSuccess) return e;
  return launch_pdl_cluster(decode_cl_kernel<MPAD, T>, static_cast<unsigned>(p.grid), S, NUM_THREADS, SMEM, a.stream,
                            tx, tw, p);
}

template <int MPAD, int T>
bool fits(int S, int groups) {
  constexpr size_t SMEM = smem_bytes<MPAD, T>();
  // the occupancy query counts the kernel's shared-memory limit
  if (ensure_smem_limit<decode_cl_kernel<MPAD, T>>(static_cast<int>(SMEM)) != cudaSuccess) return false;
  return dec::clusters_fit<decode_cl_kernel<MPAD, T>>(S, groups, NUM_THREADS, SMEM);
}

template <int MPAD>
bool fits_t(int T, int S, int groups) {
  if (T == 1) return fits<MPAD, 1>(S, groups);
  if (T == 2) return fits<MPAD, 2>(S, groups);
  return fits<MPAD, 3>(S, groups);
}

}  // namespace dcl

// The cluster plan: among T in 1..3 boxes per cluster and S in 2..8 CTAs per
// cluster (T * 64 divisible by S, at most one CTA per 64-deep k block), the
// one whose busiest CTA streams the fewest weight bytes, with all clusters
// resident at once.  It is taken when the extra bytes its busiest CTA streams
// beyond a stream-K CTA's share cost less than the fix-up kernel and the
// kernel boundary it saves (about 2 us net of the cluster exchange, i.e. about
// 13 MB of weight at the HBM rate): best * W <= sk * (W + 13 MB), W the weight
// bytes; or, if stream-K would split no tile (no fix-up kernel), only when its
// busiest CTA streams no more.
bool decode_cl_plan(const CallArgs& a, int& T, int& S) {
  const int mode = a.group_mode & 0xF, want_t = (a.group_mode >> 4) & 0xF, want_s = (a.group_mode >> 8) & 0xF;
  if (mode == 1 || a.wtype != 0 || a.swiglu || a.yq || a.part_out || a.M > 64) return false;
  const long long kblocks = a.d / dec::BK;
  const long long boxes = a.ncols / 64;
  const int mpad = decode_mpad(a.M);
  long long best = -1;
  for (int t = 3; t >= 1; --t) {
    const long long groups = (boxes + t - 1) / t;
    for (int s = 2; s <= dcl::MAX_S; ++s) {
      if (mode == 2 && want_t && (t != want_t || s != want_s)) continue;   // a forced plan
      if ((t * 64) % s != 0 || s > kblocks || groups * s > a.num_sms) continue;
      const long long load = t * ((kblocks + s - 1) / s);
      if (best >= 0 && load >= best) continue;
      const bool ok = mpad == 16 ? dcl::fits_t<16>(t, s, static_cast<int>(groups))
                      : mpad == 32 ? dcl::fits_t<32>(t, s, static_cast<int>(groups))
                                   : dcl::fits_t<64>(t, s, static_cast<int>(groups));
      if (!ok) continue;
      best = load;
      T = t;
      S = s;
    }
  }
  if (best < 0) return false;
  if (mode == 2) return true;
  const long long tiles = a.ncols / 128;                 // the stream-K kernel's 128-column tiles
  const long long total = tiles * kblocks;
  const long long grid = total < a.num_sms ? total : a.num_sms;
  const long long sk_load = 2 * ((total + grid - 1) / grid);   // 64-column boxes x k blocks per CTA
  const bool split = dec::any_split_tile(static_cast<int>(grid), total, static_cast<int>(kblocks));
  if (!split) return best <= sk_load;
  const double wbytes = static_cast<double>(a.d) * static_cast<double>(a.ncols) * 2.0;
  return static_cast<double>(best) * wbytes <= static_cast<double>(sk_load) * (wbytes + 13.0e6);
}

cudaError_t launch_decode_cl(const CallArgs& a, int T, int S) {
  const int mp = decode_mpad(a.M);
  if (mp == 16) return T == 1 ? dcl::launch_impl<16, 1>(a, S) : T == 2 ? dcl::launch_impl<16, 2>(a, S)
                                                                        : dcl::launch_impl<16, 3>(a, S);
  if (mp == 32) return T == 1 ? dcl::launch_impl<32, 1>(a, S) : T == 2 ? dcl::launch_impl<32, 2>(a, S)
                                                                        : dcl::launch_impl<32, 3>(a, S);
  return T == 1 ? dcl::launch_impl<64, 1>(a, S) : T == 2 ? dcl::launch_impl<64, 2>(a, S) : dcl::launch_impl<64, 3>(a, S);
}

}  // namespace fn
