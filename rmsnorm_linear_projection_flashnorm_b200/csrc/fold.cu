// Offline weight fold and the unfused-chain helper kernels.
//
// The fold is Proposal 1 of the FlashNorm talk summary ("웨이트리스 정규화",
// weightless normalisation): the RMSNorm gain g is multiplied into the rows
// of the projection that consumes the norm, W'[k, n] = g[k] * W[k, n], once,
// offline.  At run time the norm then carries no weight.  For the SwiGLU FC1
// of the FlashInfer PR #5521 analysis ("pre-processed FC1 weight" argument
// of its fused API) the gate and up halves are stored with their 128-column
// tiles alternating so that one 256-column tile holds matching gate and up
// columns.  The fp8 variant stores e4m3 codes with one fp32 scale per 128x128
// block (scale = block amax / 448).
//
// Rounding: one fp32 product g*W (exact when g is bf16-representable), then a
// single round-to-nearest-even to bf16, or an IEEE fp32 division by the block
// scale and one satfinite round-to-nearest-even to e4m3.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace fn {
namespace {

constexpr int kFoldThreads = 256;

// Stored column c of the folded weight comes from half `src` (0 gate / plain,
// 1 up) at source column `n`.
__device__ __forceinline__ void stored_to_source(int64_t c, bool interleave, int& src, int64_t& n) {
  if (!interleave) {
    src = 0;
    n = c;
    return;
  }
  const int64_t j = c >> 8;
  const int64_t w = c & 255;
  src = w >= 128 ? 1 : 0;
  n = (j << 7) + (w & 127);
}

__global__ void __launch_bounds__(kFoldThreads) fold_bf16_kernel(const __nv_bfloat16* __restrict__ W0,
                                                                 const __nv_bfloat16* __restrict__ W1,
                                                                 const float* __restrict__ g, int64_t d,
                                                                 int64_t N, __nv_bfloat16* __restrict__ Wp) {
  const bool inter = W1 != nullptr;
  const int64_t ncols = inter ? 2 * N : N;
  const int64_t vec_per_row = ncols / 8;
  const int64_t total = d * vec_per_row;
  for (int64_t v = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; v < total;
       v += (int64_t)gridDim.x * blockDim.x) {
    const int64_t k = v / vec_per_row;
    const int64_t c = (v - k * vec_per_row) * 8;
    int src;
    int64_t n;
    stored_to_source(c, inter, src, n);
    const __nv_bfloat16* W = src ? W1 : W0;
    const uint4 w = *reinterpret_cast<const uint4*>(W + k * N + n);
    const float gk = g[k];
    const uint32_t in[4] = {w.x, w.y, w.z, w.w};
    uint32_t out[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float lo = __fmul_rn(gk, bf16lo_to_f32(in[i]));
      const float hi = __fmul_rn(gk, bf16hi_to_f32(in[i]));
      out[i] = pack_bf16x2(lo, hi);
    }
    *reinterpret_cast<uint4*>(Wp + k * ncols + c) = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

__device__ __forceinline__ uint16_t f32x2_to_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\tmov.b16 %0, t;\n\t}"
      : "=h"(r)
      : "f"(hi), "f"(lo));
  return r;
}

// One CTA per 128x128 block of the stored weight.
__global__ void __launch_bounds__(kFoldThreads) fold_fp8_kernel(const __nv_bfloat16* __restrict__ W0,
                                                                const __nv_bfloat16* __restrict__ W1,
                                                                const float* __restrict__ g, int64_t d,
                                                                int64_t N, uint8_t* __restrict__ Wq,
                                                                float* __restrict__ scales) {
  const bool inter = W1 != nullptr;
  const int64_t ncols = inter ? 2 * N : N;
  const int64_t kb = blockIdx.y, cb = blockIdx.x;
  // each thread: 8 consecutive columns of 8 rows (128 rows / 16 row groups)
  const int cg = threadIdx.x & 15;          // column group: 8 columns
  const int rg = threadIdx.x >> 4;          // row group: rows rg, rg+16, ...
  const int64_t c = cb * 128 + cg * 8;
  int src;
  int64_t n;
  stored_to_source(c, inter, src, n);
  const __nv_bfloat16* W = src ? W1 : W0;

  float p[8][8];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t k = kb * 128 + rg + 16 * i;
    const uint4 w = *reinterpret_cast<const uint4*>(W + k * N + n);
    const float gk = g[k];
    const uint32_t in[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      p[i][2 * j] = __fmul_rn(gk, bf16lo_to_f32(in[j]));
      p[i][2 * j + 1] = __fmul_rn(gk, bf16hi_to_f32(in[j]));
      amax = fmaxf(amax, fmaxf(fabsf(p[i][2 * j]), fabsf(p[i][2 * j + 1])));
    }
  }
  __shared__ float red[kFoldThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  float bmax = red[0];
#pragma unroll
  for (int i = 1; i < kFoldThreads / 32; ++i) bmax = fmaxf(bmax, red[i]);
  const float s = bmax > 0.f ? __fdiv_rn(bmax, 448.0f) : 1.0f;
  if (threadIdx.x == 0) scales[kb * (ncols / 128) + cb] = s;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t k = kb * 128 + rg + 16 * i;
    uint32_t q[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint16_t a = f32x2_to_e4m3x2(__fdiv_rn(p[i][4 * j], s), __fdiv_rn(p[i][4 * j + 1], s));
      const uint16_t b = f32x2_to_e4m3x2(__fdiv_rn(p[i][4 * j + 2], s), __fdiv_rn(p[i][4 * j + 3], s));
      q[j] = static_cast<uint32_t>(a) | (static_cast<uint32_t>(b) << 16);
    }
    *reinterpret_cast<uint2*>(Wq + k * ncols + c) = make_uint2(q[0], q[1]);
  }
}

// MXFP8 fold: e4m3 codes with one power-of-two scale per 32 consecutive k
// values of each stored column (the block-scaled format the tensor cores'
// kind::mxf8f6f4 MMAs read).  Per block the shared exponent is the smallest
// E with amax <= 448 * 2^E, i.e. E = ceil(log2(amax / 448)): with
// amax = m * 2^e0 (m in [1, 2)) and 448 = 1.75 * 2^8 that is e0 - 8, plus one
// when m > 1.75; clamped to [-127, 127]; an all-zero block stores E = -127.
// Codes are RN_e4m3(P * 2^-E), an exact scaling.  The scale byte E + 127 is
// stored in the chunked layout the block-scaled MMAs read (mx_sf_offset).
//
// Scale byte of stored column n, 32-deep k block kb32, for a weight of
// `ncb` 128-column blocks: 128-deep k groups one after another, in each group
// one 512-byte chunk per 128 columns, and in a chunk 32 lines of 16 bytes,
// line (n mod 32) holding columns n, n+32, n+64, n+96 of the chunk, each with
// its group's four k blocks.
__device__ __forceinline__ int64_t mx_sf_offset(int64_t n, int64_t kb32, int64_t ncb) {
  return 512 * ((kb32 >> 2) * ncb + (n >> 7)) + 16 * (n & 31) + 4 * ((n & 127) >> 5) + (kb32 & 3);
}

__device__ __forceinline__ float pow2f(int e) {   // 2^e for e in [-127, 127], exact
  return e >= -126 ? __uint_as_float(static_cast<uint32_t>(e + 127) << 23) : __uint_as_float(0x00400000u);
}

// One thread per (stored column, 32-deep k block); adjacent threads take
// adjacent columns, so the weight reads of a warp are contiguous.
__global__ void __launch_bounds__(kFoldThreads) fold_mxfp8_kernel(const __nv_bfloat16* __restrict__ W0,
                                                                  const __nv_bfloat16* __restrict__ W1,
                                                                  const float* __restrict__ g, int64_t d,
                                                                  int64_t N, uint8_t* __restrict__ Wq,
                                                                  uint8_t* __restrict__ sf) {
  const bool inter = W1 != nullptr;
  const int64_t ncols = inter ? 2 * N : N;
  const int64_t total = ncols * (d / 32);
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total; t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c = t % ncols, j = t / ncols;
    int src;
    int64_t n;
    stored_to_source(c, inter, src, n);
    const __nv_bfloat16* W = src ? W1 : W0;
    float p[32];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int64_t k = j * 32 + i;
      p[i] = __fmul_rn(g[k], __bfloat162float(W[k * N + n]));
      amax = fmaxf(amax, fabsf(p[i]));
    }
    int E = -127;
    if (amax > 0.f) {
      const uint32_t bits = __float_as_uint(amax);
      const int e0 = static_cast<int>(bits >> 23) - 127;       // subnormal amax: E clamps to -127 below
      E = e0 - 8 + ((bits & 0x7FFFFFu) > 0x600000u ? 1 : 0);
      E = E < -127 ? -127 : (E > 127 ? 127 : E);
    }
    const float inv = pow2f(-E);
    sf[mx_sf_offset(c, j, ncols / 128)] = static_cast<uint8_t>(E + 127);
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const uint16_t q2 = f32x2_to_e4m3x2(__fmul_rn(p[i], inv), __fmul_rn(p[i + 1], inv));
      Wq[(j * 32 + i) * ncols + c] = static_cast<uint8_t>(q2 & 0xFFu);
      Wq[(j * 32 + i + 1) * ncols + c] = static_cast<uint8_t>(q2 >> 8);
    }
  }
}

// MXFP8 -> bf16: W[k, c] = bf16(e4m3(q[k, c]) * 2^(s - 127)), exact for the
// scales a fold produces (a byte of 255, the format's NaN, gives NaN).
__global__ void __launch_bounds__(256) dequant_mxfp8_kernel(const uint8_t* __restrict__ q,
                                                            const uint8_t* __restrict__ sf, int64_t d,
                                                            int64_t ncols, __nv_bfloat16* __restrict__ W) {
  const int64_t vec_per_row = ncols / 8;
  const int64_t total = d * vec_per_row;
  for (int64_t v = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; v < total;
       v += (int64_t)gridDim.x * blockDim.x) {
    const int64_t k = v / vec_per_row;
    const int64_t c = (v - k * vec_per_row) * 8;
    const uint2 b = *reinterpret_cast<const uint2*>(q + k * ncols + c);
    const uint32_t in[2] = {b.x, b.y};
    uint32_t out[4];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t c0 = c + 4 * j + 2 * h;
        const uint32_t e0 = sf[mx_sf_offset(c0, k >> 5, ncols / 128)], e1 = sf[mx_sf_offset(c0 + 1, k >> 5, ncols / 128)];
        const float s0 = e0 == 255u ? __int_as_float(0x7fc00000) : pow2f(static_cast<int>(e0) - 127);
        const float s1 = e1 == 255u ? __int_as_float(0x7fc00000) : pow2f(static_cast<int>(e1) - 127);
        const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(
            static_cast<__nv_fp8x2_storage_t>((in[j] >> (16 * h)) & 0xFFFFu), __NV_E4M3);
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
        out[2 * j + h] = pack_bf16x2(__fmul_rn(f.x, s0), __fmul_rn(f.y, s1));
      }
    }
    *reinterpret_cast<uint4*>(W + k * ncols + c) = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

// AdaLN shift bias (fold time): the shift row of each condition through the
// unfolded weight, B[c, col] = sum_k shift[c, k] * W[k, n] for stored column
// col (gate/up interleaved like the folded weight), fp32 products summed in
// ascending k.  One thread per (condition, stored column); adjacent threads
// read adjacent weight columns.
__global__ void __launch_bounds__(256) adaln_shift_bias_kernel(const float* __restrict__ shift, int64_t n_cond,
                                                               const __nv_bfloat16* __restrict__ W0,
                                                               const __nv_bfloat16* __restrict__ W1, int64_t d,
                                                               int64_t N, float* __restrict__ B) {
  const bool inter = W1 != nullptr;
  const int64_t ncols = inter ? 2 * N : N;
  const int64_t total = n_cond * ncols;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < total; t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c = t / ncols, col = t - c * ncols;
    int src;
    int64_t n;
    stored_to_source(col, inter, src, n);
    const __nv_bfloat16* W = src ? W1 : W0;
    const float* sr = shift + c * d;
    float acc = 0.f;
    for (int64_t k = 0; k < d; ++k) acc = fmaf(sr[k], __bfloat162float(W[k * N + n]), acc);
    B[t] = acc;
  }
}

// Unfused chain, step 1: h = bf16((x * r) * g) per row, r = 1/sqrt(mean(x^2)+eps).
__global__ void __launch_bounds__(256) rmsnorm_kernel(const __nv_bfloat16* __restrict__ x, int64_t M, int64_t d,
                                                      const float* __restrict__ g, float eps,
                                                      __nv_bfloat16* __restrict__ h) {
  __shared__ float red[8];
  const float inv_d = 1.0f / static_cast<float>(d);
  for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
    const __nv_bfloat16* xr = x + m * d;
    float ss = 0.f;
    for (int64_t c = threadIdx.x * 8; c < d; c += 256 * 8) {
      const uint4 v = *reinterpret_cast<const uint4*>(xr + c);
      const uint32_t in[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float a = bf16lo_to_f32(in[j]), b = bf16hi_to_f32(in[j]);
        ss = fmaf(a, a, ss);
        ss = fmaf(b, b, ss);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) tot += red[i];
    __syncthreads();
    const float r = inv_rms(tot, inv_d, eps);
    for (int64_t c = threadIdx.x * 8; c < d; c += 256 * 8) {
      const uint4 v = *reinterpret_cast<const uint4*>(xr + c);
      const uint32_t in[4] = {v.x, v.y, v.z, v.w};
      uint32_t out[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        out[j] = pack_bf16x2((bf16lo_to_f32(in[j]) * r) * g[c + 2 * j],
                             (bf16hi_to_f32(in[j]) * r) * g[c + 2 * j + 1]);
      }
      *reinterpret_cast<uint4*>(h + m * d + c) = make_uint4(out[0], out[1], out[2], out[3]);
    }
  }
}

// Unfused fp8 chain: W[k, n] = bf16(e4m3(q[k, n]) * s[k/128, n/128]).
__global__ void __launch_bounds__(256) dequant_fp8_kernel(const uint8_t* __restrict__ q,
                                                          const float* __restrict__ scales, int64_t d,
                                                          int64_t ncols, __nv_bfloat16* __restrict__ W) {
  const int64_t vec_per_row = ncols / 8;
  const int64_t total = d * vec_per_row;
  for (int64_t v = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; v < total;
       v += (int64_t)gridDim.x * blockDim.x) {
    const int64_t k = v / vec_per_row;
    const int64_t c = (v - k * vec_per_row) * 8;
    const float s = scales[(k >> 7) * (ncols >> 7) + (c >> 7)];
    const uint2 b = *reinterpret_cast<const uint2*>(q + k * ncols + c);
    const uint32_t in[2] = {b.x, b.y};
    uint32_t out[4];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(
            static_cast<__nv_fp8x2_storage_t>((in[j] >> (16 * h)) & 0xFFFFu), __NV_E4M3);
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
        out[2 * j + h] = pack_bf16x2(__fmul_rn(f.x, s), __fmul_rn(f.y, s));
      }
    }
    *reinterpret_cast<uint4*>(W + k * ncols + c) = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

int grid_for(int64_t work, int threads) {
  int64_t b = (work + threads - 1) / threads;
  if (b > 148 * 32) b = 148 * 32;
  return static_cast<int>(b < 1 ? 1 : b);
}

}  // namespace

cudaError_t launch_fold_bf16(const void* W0, const void* W1, const float* g, int64_t d, int64_t N, void* Wp,
                             cudaStream_t s) {
  const int64_t ncols = W1 ? 2 * N : N;
  fold_bf16_kernel<<<grid_for(d * ncols / 8, kFoldThreads), kFoldThreads, 0, s>>>(
      static_cast<const __nv_bfloat16*>(W0), static_cast<const __nv_bfloat16*>(W1), g, d, N,
      static_cast<__nv_bfloat16*>(Wp));
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) count_launch();
  return e;
}

cudaError_t launch_fold_fp8(const void* W0, const void* W1, const float* g, int64_t d, int64_t N, void* Wq,
                            float* scales, cudaStream_t s) {
  const int64_t ncols = W1 ? 2 * N : N;
  dim3 grid(static_cast<unsigned>(ncols / 128), static_cast<unsigned>(d / 128));
  fold_fp8_kernel<<<grid, kFoldThreads, 0, s>>>(static_cast<const __nv_bfloat16*>(W0),
                                                static_cast<const __nv_bfloat16*>(W1), g, d, N,
                                                static_cast<uint8_t*>(Wq), scales);
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) count_launch();
  return e;
}

cudaError_t launch_fold_mxfp8(const void* W0, const void* W1, const float* g, int64_t d, int64_t N, void* Wq,
                              void* sf, cudaStream_t s) {
  const int64_t ncols = W1 ? 2 * N : N;
  fold_mxfp8_kernel<<<grid_for(ncols * (d / 32), kFoldThreads), kFoldThreads, 0, s>>>(
      static_cast<const __nv_bfloat16*>(W0), static_cast<const __nv_bfloat16*>(W1), g, d, N,
      static_cast<uint8_t*>(Wq), static_cast<uint8_t*>(sf));
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) count_launch();
  return e;
}

cudaError_t launch_dequant_mxfp8(const void* q, const void* sf, int64_t d, int64_t ncols, void* W, cudaStream_t s) {
  dequant_mxfp8_kernel<<<grid_for(d * ncols / 8, 256), 256, 0, s>>>(
      static_cast<const uint8_t*>(q), static_cast<const uint8_t*>(sf), d, ncols, static_cast<__nv_bfloat16*>(W));
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) count_launch();
  return e;
}

cudaError_t launch_adaln_shift_bias(const float* shift, int64_t n_cond, const void* W0, const void* W1, int64_t d,
                                    int64_t N, float* B, cudaStream_t s) {
  const int64_t ncols = W1 ? 2 * N : N;
  adaln_shift_bias_kernel<<<grid_for(n_cond * ncols, 256), 256, 0, s>>>(
      shift, n_cond, static_cast<const __nv_bfloat16*>(W0), static_cast<const __nv_bfloat16*>(W1), d, N, B);
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) count_launch();
  return e;
}

cudaError_t launch_rmsnorm(const void* x, int64_t M, int64_t d, const float* g, float eps, void* h,
                           cudaStream_t s) {
  const int grid = static_cast<int>(M < 148 * 16 ? M : 148 * 16);
  rmsnorm_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), M, d, g, eps,
                                      static_cast<__nv_bfloat16*>(h));
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) count_launch();
  return e;
}

cudaError_t launch_dequant_fp8(const void* q, const float* scales, int64_t d, int64_t ncols, void* W,
                               cudaStream_t s) {
  dequant_fp8_kernel<<<grid_for(d * ncols / 8, 256), 256, 0, s>>>(static_cast<const uint8_t*>(q), scales, d,
                                                                  ncols, static_cast<__nv_bfloat16*>(W));
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) count_launch();
  return e;
}

}  // namespace fn
