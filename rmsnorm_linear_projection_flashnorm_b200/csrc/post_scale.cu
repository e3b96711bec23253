// Post-scale of a row-parallel (d-split) norm + projection, sm_100a.
//
// The deferred normalisation (FlashNorm talk summary, Proposal 2) makes the
// RMS scalar a per-row factor applied after the matmul, and sum_k x[m,k]^2 is
// a sum over k like the matmul itself.  So when the k (= d) range is split
// across ranks, each rank's partial products and its partial sums of squares
// add up to the whole, and one all-reduce of the buffer
//   [M, ncols] fp32 accumulators (stored column order), then [M] sums of squares
// leaves every rank with what the single-GPU epilogue had.  This kernel then
// does that epilogue: r = 1/sqrt(ssq/d + eps) with d the full width, y = r * acc,
// or for a SwiGLU weight (128-column gate and up tiles interleaved)
// silu(r * gate) * (r * up), with one round to bf16.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace fn {
namespace {

constexpr int kPostThreads = 256;

// One thread per 8 consecutive output columns of one row.
__global__ void __launch_bounds__(kPostThreads)
    post_scale_kernel(const float* __restrict__ part, int64_t M, int64_t N, int64_t ncols, int swiglu, float inv_d,
                      float eps, __nv_bfloat16* __restrict__ y) {
  const int64_t groups = N / 8;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * kPostThreads + threadIdx.x;
  if (idx >= M * groups) return;
  const int64_t m = idx / groups;
  const int64_t n0 = (idx - m * groups) * 8;
  const float r = inv_rms(__ldg(part + M * ncols + m), inv_d, eps);
  const float* row = part + m * ncols;
  float v[8];
  if (swiglu) {
    // output column n is gate column 256 (n / 128) + n % 128 and the up column 128 after it
    const int64_t g0 = (n0 / 128) * 256 + (n0 % 128);
    const float4 ga = __ldg(reinterpret_cast<const float4*>(row + g0));
    const float4 gb = __ldg(reinterpret_cast<const float4*>(row + g0 + 4));
    const float4 ua = __ldg(reinterpret_cast<const float4*>(row + g0 + 128));
    const float4 ub = __ldg(reinterpret_cast<const float4*>(row + g0 + 132));
    const float g[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
    const float u[8] = {ua.x, ua.y, ua.z, ua.w, ub.x, ub.y, ub.z, ub.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = silu_f32(g[j] * r) * (u[j] * r);
  } else {
    const float4 a = __ldg(reinterpret_cast<const float4*>(row + n0));
    const float4 b = __ldg(reinterpret_cast<const float4*>(row + n0 + 4));
    const float acc[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = acc[j] * r;
  }
  *reinterpret_cast<uint4*>(y + m * N + n0) =
      make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                 pack_bf16x2(v[6], v[7]));
}

}  // namespace

cudaError_t launch_post_scale(const float* part, int64_t M, int64_t N, bool swiglu, int64_t d_total, float eps,
                              void* y, cudaStream_t s) {
  const int64_t threads = M * (N / 8);
  const unsigned grid = static_cast<unsigned>((threads + kPostThreads - 1) / kPostThreads);
  const int64_t ncols = swiglu ? 2 * N : N;
  post_scale_kernel<<<grid, kPostThreads, 0, s>>>(part, M, N, ncols, swiglu ? 1 : 0,
                                                  1.0f / static_cast<float>(d_total), eps,
                                                  static_cast<__nv_bfloat16*>(y));
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) count_launch();
  return e;
}

}  // namespace fn
