// Host-side launcher interface shared by the C-ABI layer (api.cu) and the
// kernel translation units.  Not part of the public ABI.
#pragma once
#include <atomic>
#include <cstddef>
#include <cstdint>
#include <utility>
#include <cuda.h>
#include <cuda_runtime.h>

namespace fn {

// Workspace header: the first 256 bytes hold the device status word.
constexpr size_t kWsHeaderBytes = 256;

// fp8 weights at M >= this: dequantise the weight once per call into the
// workspace (bf16) instead of converting every weight tile once per row tile.
constexpr int64_t kFp8DequantOnceM = 1024;

// What a fused call writes: bf16 y; NVFP4 codes and scale bytes (SwiGLU
// only); or, for one rank of a row-parallel split of d, the fp32 accumulators
// and sums of squares before the post-scale.
enum OutKind : int { kOutBf16 = 0, kOutNvfp4 = 1, kOutPartial = 2 };

// One fused norm+projection call, validated by the ABI layer.
struct CallArgs {
  const void* x;          // bf16 [M, d]
  int64_t M, d;
  const void* Wp;         // folded weight, bf16 or e4m3 [d, ncols]
  const float* scales;    // fp8 block scales [d/128, ncols/128], MXFP8 scale bytes (chunked), or null
  int wtype;              // 0 bf16, 1 e4m3 with 128x128 block scales, 2 MXFP8
  int64_t N;              // output columns
  int64_t ncols;          // stored weight columns: N or 2N (SwiGLU)
  bool swiglu;
  float eps;
  void* y;                // bf16 [M, N] (null with NVFP4 output)
  void* yq;               // NVFP4 output, SwiGLU only: e2m1 codes [M, N/2] bytes, or null
  void* ysf;              //   e4m3 scale codes [M, N/16], row-major or chunked (sf_chunked)
  int sf_chunked;         //   1: the 128x4 chunked scale layout
  const float* gscale;    //   global scale, one fp32 value in device memory
  float* part_out;        // kOutPartial: fp32 [M, ncols] accumulators, then [M] sums of squares
  void* ws;               // workspace (status word + decode scratch)
  size_t ws_bytes;
  cudaStream_t stream;
  int num_sms;
  uint64_t budget_ns;     // per-wait time limit
  int withhold;           // test knob: withhold one reducer arrival
  int prefetch_iters;     // decode: weight k-blocks per CTA prefetched into L2 early
  int prefetch_mode;      // decode: 0 none, 1 TMA prefetch, 2 per-thread prefetch
  int cluster_mode;       // decode: 1 allow split-K inside clusters, 0 stream-K only
  int group_mode;         // decode: column groups per cluster (decode_cl.cu): 0 auto, 1 never, 2 whenever they fit
  int single_sm_tiles;    // tile path: 1 keeps the one-SM kernel where the pair kernel would run
  int pair_tile;          // pair kernel tile: 0 automatic, 1 256 x 256, 2 256 x 512
  const float* ad_scale;  // AdaLN (tile path only): scale rows fp32 [n_cond, d], or null
  const float* ad_bias;   //   shift bias rows fp32 [n_cond, ncols]
  const int* ad_index;    //   condition index per row [M]; null: no AdaLN
  int64_t n_cond;
};

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn();

// 2D row-major tensor map with 128-byte swizzle: rows x cols elements of
// `elem_bytes`, box of box_rows x box_cols (box_cols * elem_bytes <= 128).
bool make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int elem_bytes, uint64_t rows,
                  uint64_t cols, uint32_t box_rows, uint32_t box_cols, bool swizzle128 = true);

// Decode (M <= 64) path: stream-K split over all SMs with a deterministic
// in-kernel fix-up through workspace partials.
int decode_mpad(int64_t M);
// wtype: 0 bf16, 1 e4m3 with 128x128 fp32 scales, 2 MXFP8 (e4m3 with ue8m0 per 32 k)
size_t decode_workspace_bytes(int64_t M, int64_t d, int64_t ncols, bool swiglu, int num_sms, int wtype);
// fp8 weights, 17..64 rows: workspace for x split once per call (decode_fp8.cu)
size_t decode_fp8_presplit_bytes(int64_t M, int64_t d);
// MXFP8 weights: workspace for x split once per call (decode_mx.cu)
size_t decode_mx_presplit_bytes(int64_t M, int64_t d);
cudaError_t launch_decode(const CallArgs& a);
// fp8 weights on the decode path (decode_fp8.cu); mpad is decode_mpad(M).
cudaError_t launch_decode_fp8(const CallArgs& a, int mpad);
// MXFP8 weights on the decode path: block-scaled MMAs (decode_mx.cu).
cudaError_t launch_decode_mx(const CallArgs& a, int mpad);

// Tensor-core tile path (M > 64): persistent 128x256 tiles, tcgen05 + TMEM.
cudaError_t launch_tc(const CallArgs& a);
// The same on pairs of SMs (2-CTA clusters, 256x256 tiles, cta_group::2 MMAs):
// bf16 weights, bf16 output, no AdaLN (tc2.cu).
cudaError_t launch_tc_pair(const CallArgs& a);
// Rows from which the tile path runs on pairs of SMs.
constexpr int64_t kPairTileMinM = 512;
// Small-M path for bf16 weights, plain projection, bf16 output, when the
// weight is too small to keep every SM busy without splitting most column
// tiles: T 64-column boxes per cluster of S CTAs, k split across the cluster,
// partials reduced through distributed shared memory (decode_cl.cu).  Returns
// false (and launches nothing) when no cluster plan is chosen for the shape.
bool decode_cl_plan(const CallArgs& a, int& T, int& S);
cudaError_t launch_decode_cl(const CallArgs& a, int T, int S);

// fp8 weights (128x128 block scales) at M > 64 with bf16 output: x split once
// into exact e4m3 hi/lo planes, the stored codes multiplied as they are, the
// block scales applied per 128-deep k block to fp32 sums (tc8.cu).  MXFP8
// weights: the split per 32-deep block, its powers of two as ue8m0 x scales,
// block-scaled MMAs over a tile's whole k range (mx = true).
size_t tc8_workspace_bytes(int64_t M, int64_t d, bool mx = false);
cudaError_t launch_tc8(const CallArgs& a);
// fp8 weights with bf16 output take the promotion kernel from this many rows:
// on the fp8 SwiGLU workload's shape (d=5120, N=13824) it ran 5-10 % faster
// than the split-K decode kernel at 33, 48 and 64 rows (where the decode
// kernel pads to 64 rows), 14 % slower at 32.
constexpr int64_t kFp8PromotionMinM = 33;

// Offline fold and the unfused-chain helper kernels.
cudaError_t launch_fold_bf16(const void* W0, const void* W1, const float* g, int64_t d, int64_t N, void* Wp,
                             cudaStream_t s);
cudaError_t launch_fold_fp8(const void* W0, const void* W1, const float* g, int64_t d, int64_t N, void* Wq,
                            float* scales, cudaStream_t s);
// MXFP8 weights: e4m3 codes and ue8m0 scale bytes in the chunked layout.
cudaError_t launch_fold_mxfp8(const void* W0, const void* W1, const float* g, int64_t d, int64_t N, void* Wq,
                              void* sf, cudaStream_t s);
cudaError_t launch_dequant_mxfp8(const void* q, const void* sf, int64_t d, int64_t ncols, void* W, cudaStream_t s);
cudaError_t launch_rmsnorm(const void* x, int64_t M, int64_t d, const float* g, float eps, void* h,
                           cudaStream_t s);
// Row-parallel split of d: the post-scale after the partials were summed (post_scale.cu).
cudaError_t launch_post_scale(const float* part, int64_t M, int64_t N, bool swiglu, int64_t d_total, float eps,
                              void* y, cudaStream_t s);
cudaError_t launch_dequant_fp8(const void* q, const float* scales, int64_t d, int64_t ncols, void* W,
                               cudaStream_t s);
// AdaLN shift bias B[c, n] = sum_k shift[c, k] W[k, n] in stored column order (fp32 accumulation).
cudaError_t launch_adaln_shift_bias(const float* shift, int64_t n_cond, const void* W0, const void* W1, int64_t d,
                                    int64_t N, float* B, cudaStream_t s);

// Raise a kernel's dynamic shared-memory limit once per device (a host-only
// call, done on the first launch so later launches can be graph-captured).
// One flag set per kernel: the kernel itself is the template argument.
template <auto Kernel>
cudaError_t ensure_smem_limit(int bytes) {
  static std::atomic<unsigned long long> done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// Process-wide count of kernels enqueued by the library.
void count_launch();

// Launch with programmatic stream serialization: the kernel may start (and
// run its prologue) while the preceding kernel in the stream finishes; it
// calls griddepcontrol.wait before touching global memory.
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), unsigned grid, unsigned block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e == cudaSuccess) count_launch();
  return e;
}

// Same, with thread-block clusters of `cluster` CTAs along x.
template <typename... Params, typename... Args>
cudaError_t launch_pdl_cluster(void (*kernel)(Params...), unsigned grid, int cluster, unsigned block, size_t smem,
                               cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = static_cast<unsigned>(cluster);
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e == cudaSuccess) count_launch();
  return e;
}

}  // namespace fn
