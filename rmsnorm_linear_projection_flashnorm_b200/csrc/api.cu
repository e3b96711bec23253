// C ABI layer: argument validation, dispatch, tensor-map encoding and the
// device status word.  Declarations and contracts are in include/flashnorm.h.
//
// Dispatch ladder: M <= 64 runs the split-K decode kernel, larger M the
// tensor-core tile kernel.  This mirrors the token-count ladder of the
// FlashInfer PR #5668 analysis (K23_LADDER: run M on the smallest compiled
// capacity that holds it, reject sizes out of range with an error, not an
// exception); inside the decode kernel M is padded to 16, 32 or 64.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "flashnorm.h"
#include "internal.h"

namespace fn {

namespace {
std::atomic<long long> g_budget_ns{2000000000LL};
std::atomic<int> g_withhold{0};
std::atomic<int> g_force_path{0};
std::atomic<int> g_prefetch_iters{8};
std::atomic<int> g_prefetch_mode{2};
std::atomic<int> g_cluster_mode{1};
std::atomic<int> g_pair_tile{0};
std::atomic<int> g_group_mode{0};

constexpr int kMaxDevices = 64;
std::atomic<int> g_sms[kMaxDevices];
std::atomic<int> g_cc_major[kMaxDevices];

bool device_info(int& dev, int& sms, int& cc_major) {
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return false;
  }
  sms = g_sms[dev].load(std::memory_order_relaxed);
  cc_major = g_cc_major[dev].load(std::memory_order_relaxed);
  if (sms <= 0) {
    int s = 0, c = 0;
    if (cudaDeviceGetAttribute(&s, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&c, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
      cudaGetLastError();
      return false;
    }
    g_sms[dev].store(s);
    g_cc_major[dev].store(c);
    sms = s;
    cc_major = c;
  }
  return true;
}

int current_sms_or_default() {
  int dev, sms, cc;
  if (device_info(dev, sms, cc) && sms > 0) return sms;
  return 148;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

bool eps_ok(float eps) { return std::isfinite(eps) && eps >= 0.0f; }

constexpr int64_t kMaxDim = (int64_t{1} << 31) - 1;
std::atomic<unsigned long long> g_launches{0};
}  // namespace

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

bool make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int elem_bytes, uint64_t rows,
                  uint64_t cols, uint32_t box_rows, uint32_t box_cols, bool swizzle128) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * static_cast<uint64_t>(elem_bytes)};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  std::memset(map, 0, sizeof(*map));
  const CUresult r = enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE,
                         swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

fn_status check_device(int& sms) {
  int dev, cc;
  if (!device_info(dev, sms, cc)) return FN_ERR_CUDA;
  if (cc != 10) return FN_ERR_UNSUPPORTED_DEVICE;
  return FN_OK;
}

// Fused call.  Output: bf16 y, or (SwiGLU only) NVFP4 codes yq, scale bytes
// ysf and the global scale gscale, with y null.
// AdaLN inputs of a fused call (all null: no AdaLN).
struct AdaLN {
  const float* scale = nullptr;   // fp32 [n_cond, d]
  const float* bias = nullptr;    // fp32 [n_cond, ncols]
  const int32_t* index = nullptr; // [M]
  int64_t n_cond = 0;
};

fn_status norm_proj_common(const void* x, int64_t M, int64_t d, const void* Wp, const float* scales, fn_wtype wt,
                           int64_t N, float eps, void* y, void* ws, size_t ws_bytes, fn_stream_t stream,
                           bool swiglu, void* yq = nullptr, void* ysf = nullptr, const float* gscale = nullptr,
                           float* part_out = nullptr, const AdaLN& ad = AdaLN(), bool sf_chunked = false) {
  const bool adaln = ad.index != nullptr || ad.scale != nullptr || ad.bias != nullptr;
  const bool fp4 = yq != nullptr || ysf != nullptr || gscale != nullptr;
  const bool partial = part_out != nullptr;
  if (M < 0 || d <= 0 || N <= 0) return FN_ERR_INVALID_ARG;
  if (wt != FN_W_BF16 && wt != FN_W_FP8_E4M3_B128 && wt != FN_W_MXFP8_E4M3) return FN_ERR_INVALID_ARG;
  if (!eps_ok(eps)) return FN_ERR_INVALID_ARG;
  if (d % 64 != 0 || N % 128 != 0) return FN_ERR_UNSUPPORTED_SHAPE;
  if (wt != FN_W_BF16 && d % 128 != 0) return FN_ERR_UNSUPPORTED_SHAPE;
  const int64_t ncols = swiglu ? 2 * N : N;
  if (M > kMaxDim || d > kMaxDim || ncols > kMaxDim) return FN_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return FN_OK;
  if (!x || !Wp) return FN_ERR_INVALID_ARG;
  if (partial ? (y || fp4 || swiglu) : fp4 ? (!yq || !ysf || !gscale || y || !swiglu) : !y)
    return FN_ERR_INVALID_ARG;
  if (!ws) return FN_ERR_WORKSPACE;
  if (adaln) {
    if (!ad.index || !ad.scale || !ad.bias || ad.n_cond <= 0 || partial || fp4) return FN_ERR_INVALID_ARG;
    if (ad.n_cond > kMaxDim) return FN_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(ad.scale) || !aligned16(ad.bias) || (reinterpret_cast<uintptr_t>(ad.index) & 3u))
      return FN_ERR_ALIGNMENT;
  }
  if (wt != FN_W_BF16 && !scales) return FN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(Wp) || !aligned16(ws)) return FN_ERR_ALIGNMENT;
  if (partial ? !aligned16(part_out)
              : fp4 ? (!aligned16(yq) || !aligned16(ysf) || (reinterpret_cast<uintptr_t>(gscale) & 3u))
                    : !aligned16(y))
    return FN_ERR_ALIGNMENT;
  if (scales && (reinterpret_cast<uintptr_t>(scales) & (wt == FN_W_MXFP8_E4M3 ? 15u : 3u))) return FN_ERR_ALIGNMENT;

  const size_t wbytes = static_cast<size_t>(d) * ncols * (wt == FN_W_BF16 ? 2 : 1);
  const size_t xbytes = static_cast<size_t>(M) * d * 2;
  const size_t ybytes = static_cast<size_t>(M) * N * 2;
  const size_t sbytes = !scales                  ? 0
                        : wt == FN_W_MXFP8_E4M3 ? static_cast<size_t>(d / 32) * ncols
                                                : static_cast<size_t>(d / 128) * (ncols / 128) * 4;
  if (overlaps(ws, ws_bytes, x, xbytes) || overlaps(ws, ws_bytes, Wp, wbytes) || overlaps(ws, ws_bytes, scales, sbytes))
    return FN_ERR_ALIAS;
  // every output region against every input region, the workspace and each other
  const size_t qbytes = static_cast<size_t>(M) * (N / 2);
  const size_t fbytes = static_cast<size_t>(sf_chunked ? (M + 127) / 128 * 128 : M) * (N / 16);
  const size_t pbytes = partial ? (static_cast<size_t>(M) * ncols + M) * 4 : 0;
  const struct { const void* p; size_t n; } outs[4] = {{y, ybytes}, {yq, qbytes}, {ysf, fbytes}, {part_out, pbytes}};
  const size_t adsb = adaln ? static_cast<size_t>(ad.n_cond) * d * 4 : 0;
  const size_t adbb = adaln ? static_cast<size_t>(ad.n_cond) * ncols * 4 : 0;
  const size_t adib = adaln ? static_cast<size_t>(M) * 4 : 0;
  if (adaln && (overlaps(ws, ws_bytes, ad.scale, adsb) || overlaps(ws, ws_bytes, ad.bias, adbb) ||
                overlaps(ws, ws_bytes, ad.index, adib)))
    return FN_ERR_ALIAS;
  for (int i = 0; i < 4; ++i) {
    if (!outs[i].p) continue;
    if (overlaps(outs[i].p, outs[i].n, x, xbytes) || overlaps(outs[i].p, outs[i].n, Wp, wbytes) ||
        overlaps(outs[i].p, outs[i].n, scales, sbytes) || overlaps(outs[i].p, outs[i].n, ws, ws_bytes) ||
        overlaps(outs[i].p, outs[i].n, gscale, gscale ? 4 : 0) || overlaps(outs[i].p, outs[i].n, ad.scale, adsb) ||
        overlaps(outs[i].p, outs[i].n, ad.bias, adbb) || overlaps(outs[i].p, outs[i].n, ad.index, adib))
      return FN_ERR_ALIAS;
    for (int j = i + 1; j < 4; ++j)
      if (outs[j].p && overlaps(outs[i].p, outs[i].n, outs[j].p, outs[j].n)) return FN_ERR_ALIAS;
  }

  int force = g_force_path.load();
  bool use_decode = M <= 64 && !adaln;   // AdaLN runs on the tile kernel at every M
  // fp8 weights with bf16 output: the promotion tile kernel from kFp8PromotionMinM rows
  if (wt == FN_W_FP8_E4M3_B128 && M >= kFp8PromotionMinM && !fp4 && !partial && force != 4) use_decode = false;
  if (force == 1) {
    if (M > 64 || adaln) return FN_ERR_INVALID_ARG;
    use_decode = true;
  } else if (force >= 2) {
    use_decode = false;
  }

  int sms = 0;
  fn_status st = check_device(sms);
  if (st != FN_OK) return st;
  // fp8 and MXFP8 weights with bf16 output on the tile path: the promotion
  // kernel (tc8.cu), which multiplies the stored e4m3 codes (fp8: block scales
  // applied per 128-deep k block in registers; MXFP8: block-scaled MMAs).  The
  // other tile forms with 8-bit weights (NVFP4 or partial output, AdaLN, or
  // forced) convert the staged fp8 weight tiles to bf16 (M < kFp8DequantOnceM)
  // or the whole weight once per call into the workspace (MXFP8 always).
  const bool fp8_tc8 = !use_decode && (wt == FN_W_FP8_E4M3_B128 || wt == FN_W_MXFP8_E4M3) && !adaln && !fp4 &&
                       !partial && force != 4;
  const bool dequant_once =
      !use_decode && !fp8_tc8 &&
      ((wt == FN_W_FP8_E4M3_B128 && (M >= kFp8DequantOnceM || adaln)) || wt == FN_W_MXFP8_E4M3);
  const size_t need = use_decode     ? decode_workspace_bytes(M, d, ncols, swiglu, sms, static_cast<int>(wt))
                      : fp8_tc8      ? tc8_workspace_bytes(M, d, wt == FN_W_MXFP8_E4M3)
                      : dequant_once ? kWsHeaderBytes + wbytes * 2
                                     : kWsHeaderBytes;
  if (ws_bytes < need) return FN_ERR_WORKSPACE;

  CallArgs a;
  a.x = x;
  a.M = M;
  a.d = d;
  a.Wp = Wp;
  a.scales = scales;
  a.wtype = static_cast<int>(wt);
  a.N = N;
  a.ncols = ncols;
  a.swiglu = swiglu;
  a.eps = eps;
  a.y = y;
  a.yq = yq;
  a.ysf = ysf;
  a.sf_chunked = sf_chunked ? 1 : 0;
  a.gscale = gscale;
  a.part_out = part_out;
  a.ws = ws;
  a.ws_bytes = ws_bytes;
  a.stream = reinterpret_cast<cudaStream_t>(stream);
  a.num_sms = sms;
  a.budget_ns = static_cast<uint64_t>(g_budget_ns.load());
  a.withhold = g_withhold.load();
  a.prefetch_iters = g_prefetch_iters.load();
  a.prefetch_mode = g_prefetch_mode.load();
  a.cluster_mode = g_cluster_mode.load();
  a.pair_tile = g_pair_tile.load();
  a.group_mode = g_group_mode.load();
  a.single_sm_tiles = force == 3 ? 1 : 0;
  a.ad_scale = ad.scale;
  a.ad_bias = ad.bias;
  a.ad_index = ad.index;
  a.n_cond = ad.n_cond;
  if (dequant_once) {
    // the bf16 weight bf16(fp32(q) * s), the rounding the on-chip conversion uses
    void* wbf = static_cast<uint8_t*>(ws) + kWsHeaderBytes;
    const cudaError_t de = wt == FN_W_MXFP8_E4M3 ? launch_dequant_mxfp8(Wp, scales, d, ncols, wbf, a.stream)
                                                 : launch_dequant_fp8(Wp, scales, d, ncols, wbf, a.stream);
    if (de != cudaSuccess) return FN_ERR_CUDA;
    a.Wp = wbf;
    a.wtype = FN_W_BF16;
    a.scales = nullptr;
  }
  const cudaError_t e = use_decode ? launch_decode(a) : fp8_tc8 ? launch_tc8(a) : launch_tc(a);
  return e == cudaSuccess ? FN_OK : FN_ERR_CUDA;
}

}  // namespace
}  // namespace fn

using namespace fn;

extern "C" {

fn_status fn_fold_weights(const void* W0, const void* W1, const float* g, int64_t d, int64_t N, fn_wtype out_type,
                          void* Wp, float* scales, fn_stream_t stream) {
  if (d <= 0 || N <= 0) return FN_ERR_INVALID_ARG;
  if (out_type != FN_W_BF16 && out_type != FN_W_FP8_E4M3_B128 && out_type != FN_W_MXFP8_E4M3)
    return FN_ERR_INVALID_ARG;
  if (!W0 || !g || !Wp) return FN_ERR_INVALID_ARG;
  if (out_type != FN_W_BF16 && !scales) return FN_ERR_INVALID_ARG;
  if (d % 64 != 0 || N % 128 != 0) return FN_ERR_UNSUPPORTED_SHAPE;
  if (out_type != FN_W_BF16 && d % 128 != 0) return FN_ERR_UNSUPPORTED_SHAPE;
  const int64_t ncols = W1 ? 2 * N : N;
  if (d > kMaxDim || ncols > kMaxDim) return FN_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(W0) || (W1 && !aligned16(W1)) || !aligned16(Wp) || (reinterpret_cast<uintptr_t>(g) & 3u) ||
      (scales && (reinterpret_cast<uintptr_t>(scales) & (out_type == FN_W_MXFP8_E4M3 ? 15u : 3u))))
    return FN_ERR_ALIGNMENT;
  const size_t in_bytes = static_cast<size_t>(d) * N * 2;
  const size_t out_bytes = static_cast<size_t>(d) * ncols * (out_type == FN_W_BF16 ? 2 : 1);
  const size_t s_bytes = !scales                        ? 0
                         : out_type == FN_W_MXFP8_E4M3 ? static_cast<size_t>(d / 32) * ncols
                                                       : static_cast<size_t>(d / 128) * (ncols / 128) * 4;
  if (overlaps(Wp, out_bytes, W0, in_bytes) || overlaps(Wp, out_bytes, W1, in_bytes) ||
      overlaps(Wp, out_bytes, g, static_cast<size_t>(d) * 4) || overlaps(scales, s_bytes, Wp, out_bytes) ||
      overlaps(scales, s_bytes, W0, in_bytes) || overlaps(scales, s_bytes, W1, in_bytes))
    return FN_ERR_ALIAS;
  int sms = 0;
  fn_status st = check_device(sms);
  if (st != FN_OK) return st;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const cudaError_t e = out_type == FN_W_BF16          ? launch_fold_bf16(W0, W1, g, d, N, Wp, s)
                        : out_type == FN_W_MXFP8_E4M3 ? launch_fold_mxfp8(W0, W1, g, d, N, Wp, scales, s)
                                                      : launch_fold_fp8(W0, W1, g, d, N, Wp, scales, s);
  return e == cudaSuccess ? FN_OK : FN_ERR_CUDA;
}

size_t fn_workspace_size(int64_t M, int64_t d, int64_t N, fn_wtype wt, int swiglu) {
  if (M <= 0 || d <= 0 || N <= 0 || d % 64 != 0 || N % 128 != 0) return kWsHeaderBytes;
  const int64_t ncols = swiglu ? 2 * N : N;
  if (M > 64) {
    const size_t copy = kWsHeaderBytes + static_cast<size_t>(d) * static_cast<size_t>(ncols) * 2;
    if (wt == FN_W_MXFP8_E4M3) {
      // the promotion kernel's split x and scale chunks, or (NVFP4, partial
      // or AdaLN output) the dequantised weight
      const size_t t8 = tc8_workspace_bytes(M, d, true);
      return copy > t8 ? copy : t8;
    }
    if (wt == FN_W_FP8_E4M3_B128) {
      // the promotion kernel's split x, or (NVFP4 / partial output at large M)
      // the dequantised weight
      const size_t t8 = tc8_workspace_bytes(M, d);
      return M >= kFp8DequantOnceM && copy > t8 ? copy : t8;
    }
    return kWsHeaderBytes;
  }
  const size_t dec = decode_workspace_bytes(M, d, ncols, swiglu != 0, current_sms_or_default(), static_cast<int>(wt));
  if (wt == FN_W_FP8_E4M3_B128 && M >= kFp8PromotionMinM) {
    // bf16 output runs the promotion kernel; NVFP4 and partial outputs the decode kernel
    const size_t t8 = tc8_workspace_bytes(M, d);
    return t8 > dec ? t8 : dec;
  }
  return dec;
}

fn_status fn_norm_proj(const void* x, int64_t M, int64_t d, const void* Wp, const float* scales, fn_wtype wt,
                       int64_t N, float eps, void* y, void* workspace, size_t ws_bytes, fn_stream_t stream) {
  return norm_proj_common(x, M, d, Wp, scales, wt, N, eps, y, workspace, ws_bytes, stream, false);
}

fn_status fn_norm_proj_swiglu(const void* x, int64_t M, int64_t d, const void* Wp, const float* scales,
                              fn_wtype wt, int64_t N, float eps, void* out, void* workspace, size_t ws_bytes,
                              fn_stream_t stream) {
  return norm_proj_common(x, M, d, Wp, scales, wt, N, eps, out, workspace, ws_bytes, stream, true);
}

fn_status fn_norm_proj_swiglu_nvfp4(const void* x, int64_t M, int64_t d, const void* Wp, const float* scales,
                                    fn_wtype wt, int64_t N, float eps, const float* global_scale, void* out_q,
                                    void* out_sf, void* workspace, size_t ws_bytes, fn_stream_t stream) {
  if (M > 0 && (!out_q || !out_sf || !global_scale)) return FN_ERR_INVALID_ARG;
  return norm_proj_common(x, M, d, Wp, scales, wt, N, eps, nullptr, workspace, ws_bytes, stream, true, out_q,
                          out_sf, global_scale);
}

fn_status fn_norm_proj_swiglu_nvfp4_swizzled(const void* x, int64_t M, int64_t d, const void* Wp, const float* scales,
                                             fn_wtype wt, int64_t N, float eps, const float* global_scale, void* out_q,
                                             void* out_sf, void* workspace, size_t ws_bytes, fn_stream_t stream) {
  if (M > 0 && (!out_q || !out_sf || !global_scale)) return FN_ERR_INVALID_ARG;
  return norm_proj_common(x, M, d, Wp, scales, wt, N, eps, nullptr, workspace, ws_bytes, stream, true, out_q,
                          out_sf, global_scale, nullptr, AdaLN(), true);
}

fn_status fn_norm_proj_partial(const void* x, int64_t M, int64_t d, const void* Wp, const float* scales,
                               fn_wtype wt, int64_t ncols, float* partial, void* workspace, size_t ws_bytes,
                               fn_stream_t stream) {
  if (M > 0 && !partial) return FN_ERR_INVALID_ARG;
  return norm_proj_common(x, M, d, Wp, scales, wt, ncols, 0.0f, nullptr, workspace, ws_bytes, stream, false,
                          nullptr, nullptr, nullptr, partial);
}

fn_status fn_norm_proj_adaln(const void* x, int64_t M, int64_t d, const void* Wp, const float* scales, fn_wtype wt,
                             int64_t N, int swiglu, float eps, const float* adaln_scale, const float* shift_bias,
                             const int32_t* adaln_index, int64_t n_cond, void* y, void* workspace, size_t ws_bytes,
                             fn_stream_t stream) {
  if (M > 0 && (!adaln_scale || !shift_bias || !adaln_index || n_cond <= 0)) return FN_ERR_INVALID_ARG;
  AdaLN ad;
  ad.scale = adaln_scale;
  ad.bias = shift_bias;
  ad.index = adaln_index;
  ad.n_cond = n_cond;
  return norm_proj_common(x, M, d, Wp, scales, wt, N, eps, y, workspace, ws_bytes, stream, swiglu != 0, nullptr,
                          nullptr, nullptr, nullptr, ad);
}

size_t fn_workspace_size_adaln(int64_t d, int64_t N, fn_wtype wt, int swiglu) {
  if (d <= 0 || N <= 0 || d % 64 != 0 || N % 128 != 0 || wt == FN_W_BF16) return kWsHeaderBytes;
  const int64_t ncols = swiglu ? 2 * N : N;
  return kWsHeaderBytes + static_cast<size_t>(d) * static_cast<size_t>(ncols) * 2;
}

fn_status fn_adaln_shift_bias(const float* shift, int64_t n_cond, const void* W0, const void* W1, int64_t d,
                              int64_t N, float* B, fn_stream_t stream) {
  if (n_cond <= 0 || d <= 0 || N <= 0 || !shift || !W0 || !B) return FN_ERR_INVALID_ARG;
  if (d % 64 != 0 || N % 128 != 0) return FN_ERR_UNSUPPORTED_SHAPE;
  const int64_t ncols = W1 ? 2 * N : N;
  if (d > kMaxDim || ncols > kMaxDim || n_cond > kMaxDim) return FN_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(W0) || (W1 && !aligned16(W1)) || (reinterpret_cast<uintptr_t>(shift) & 3u) ||
      (reinterpret_cast<uintptr_t>(B) & 3u))
    return FN_ERR_ALIGNMENT;
  const size_t bb = static_cast<size_t>(n_cond) * ncols * 4;
  if (overlaps(B, bb, shift, static_cast<size_t>(n_cond) * d * 4) || overlaps(B, bb, W0, static_cast<size_t>(d) * N * 2) ||
      overlaps(B, bb, W1, W1 ? static_cast<size_t>(d) * N * 2 : 0))
    return FN_ERR_ALIAS;
  int sms = 0;
  const fn_status st = check_device(sms);
  if (st != FN_OK) return st;
  return launch_adaln_shift_bias(shift, n_cond, W0, W1, d, N, B, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? FN_OK
             : FN_ERR_CUDA;
}

fn_status fn_post_scale(const float* partial, int64_t M, int64_t N, int swiglu, int64_t d_total, float eps, void* y,
                        fn_stream_t stream) {
  if (M < 0 || N <= 0 || d_total <= 0) return FN_ERR_INVALID_ARG;
  if (!eps_ok(eps)) return FN_ERR_INVALID_ARG;
  if (N % 128 != 0) return FN_ERR_UNSUPPORTED_SHAPE;
  const int64_t ncols = swiglu ? 2 * N : N;
  if (M > kMaxDim || ncols > kMaxDim || d_total > kMaxDim) return FN_ERR_UNSUPPORTED_SHAPE;
  if (M * (N / 8) / 256 > kMaxDim) return FN_ERR_UNSUPPORTED_SHAPE;   // one thread per 8 outputs, 256 per block
  if (M == 0) return FN_OK;
  if (!partial || !y) return FN_ERR_INVALID_ARG;
  if (!aligned16(partial) || !aligned16(y)) return FN_ERR_ALIGNMENT;
  if (overlaps(y, static_cast<size_t>(M) * N * 2, partial, (static_cast<size_t>(M) * ncols + M) * 4))
    return FN_ERR_ALIAS;
  int sms = 0;
  const fn_status st = check_device(sms);
  if (st != FN_OK) return st;
  const cudaError_t e =
      launch_post_scale(partial, M, N, swiglu != 0, d_total, eps, y, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FN_OK : FN_ERR_CUDA;
}

fn_status fn_query_device_status(void* workspace, unsigned int* detail, fn_stream_t stream) {
  if (!workspace) return FN_ERR_INVALID_ARG;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned int word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return FN_ERR_CUDA;
  }
  if (word != 0) {
    if (cudaMemsetAsync(workspace, 0, sizeof(word), s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess) {
      cudaGetLastError();
      return FN_ERR_CUDA;
    }
  }
  if (detail) *detail = word;
  if (word == 0) return FN_OK;
  return (word & 0xFFu) == FN_ERR_TIMEOUT ? FN_ERR_TIMEOUT : FN_ERR_CUDA;
}

fn_status fn_rmsnorm(const void* x, int64_t M, int64_t d, const float* g, float eps, void* h, fn_stream_t stream) {
  if (M < 0 || d <= 0 || !eps_ok(eps)) return FN_ERR_INVALID_ARG;
  if (d % 64 != 0 || M > kMaxDim || d > kMaxDim) return FN_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return FN_OK;
  if (!x || !g || !h) return FN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(h)) return FN_ERR_ALIGNMENT;
  const size_t bytes = static_cast<size_t>(M) * d * 2;
  if (overlaps(h, bytes, x, bytes) || overlaps(h, bytes, g, static_cast<size_t>(d) * 4)) return FN_ERR_ALIAS;
  int sms = 0;
  fn_status st = check_device(sms);
  if (st != FN_OK) return st;
  return launch_rmsnorm(x, M, d, g, eps, h, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? FN_OK
                                                                                                 : FN_ERR_CUDA;
}

fn_status fn_dequant_fp8(const void* q, const float* scales, int64_t d, int64_t ncols, void* W, fn_stream_t stream) {
  if (d <= 0 || ncols <= 0 || !q || !scales || !W) return FN_ERR_INVALID_ARG;
  if (d % 128 != 0 || ncols % 128 != 0 || d > kMaxDim || ncols > kMaxDim) return FN_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(q) || !aligned16(W) || (reinterpret_cast<uintptr_t>(scales) & 3u)) return FN_ERR_ALIGNMENT;
  const size_t out = static_cast<size_t>(d) * ncols * 2;
  if (overlaps(W, out, q, static_cast<size_t>(d) * ncols) ||
      overlaps(W, out, scales, static_cast<size_t>(d / 128) * (ncols / 128) * 4))
    return FN_ERR_ALIAS;
  int sms = 0;
  fn_status st = check_device(sms);
  if (st != FN_OK) return st;
  return launch_dequant_fp8(q, scales, d, ncols, W, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? FN_OK
             : FN_ERR_CUDA;
}

fn_status fn_dequant_mxfp8(const void* q, const void* scales, int64_t d, int64_t ncols, void* W,
                           fn_stream_t stream) {
  if (d <= 0 || ncols <= 0 || !q || !scales || !W) return FN_ERR_INVALID_ARG;
  if (d % 128 != 0 || ncols % 128 != 0 || d > kMaxDim || ncols > kMaxDim) return FN_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(q) || !aligned16(W) || !aligned16(scales)) return FN_ERR_ALIGNMENT;
  const size_t out = static_cast<size_t>(d) * ncols * 2;
  if (overlaps(W, out, q, static_cast<size_t>(d) * ncols) || overlaps(W, out, scales, static_cast<size_t>(d / 32) * ncols))
    return FN_ERR_ALIAS;
  int sms = 0;
  fn_status st = check_device(sms);
  if (st != FN_OK) return st;
  return launch_dequant_mxfp8(q, scales, d, ncols, W, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? FN_OK
             : FN_ERR_CUDA;
}

const char* fn_status_string(fn_status s) {
  switch (s) {
    case FN_OK: return "FN_OK";
    case FN_ERR_INVALID_ARG: return "FN_ERR_INVALID_ARG";
    case FN_ERR_UNSUPPORTED_SHAPE: return "FN_ERR_UNSUPPORTED_SHAPE";
    case FN_ERR_ALIGNMENT: return "FN_ERR_ALIGNMENT";
    case FN_ERR_ALIAS: return "FN_ERR_ALIAS";
    case FN_ERR_WORKSPACE: return "FN_ERR_WORKSPACE";
    case FN_ERR_CUDA: return "FN_ERR_CUDA";
    case FN_ERR_TIMEOUT: return "FN_ERR_TIMEOUT";
    case FN_ERR_UNSUPPORTED_DEVICE: return "FN_ERR_UNSUPPORTED_DEVICE";
  }
  return "FN_ERR_UNKNOWN";
}

int fn_version(void) { return 1; }

uint64_t fn_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

fn_status fn_set_debug(int key, int64_t value) {
  switch (key) {
    case FN_DEBUG_WAIT_BUDGET_NS:
      if (value <= 0) return FN_ERR_INVALID_ARG;
      g_budget_ns.store(value);
      return FN_OK;
    case FN_DEBUG_WITHHOLD_ARRIVE:
      g_withhold.store(value ? 1 : 0);
      return FN_OK;
    case FN_DEBUG_FORCE_PATH:
      if (value < 0 || value > 4) return FN_ERR_INVALID_ARG;
      g_force_path.store(static_cast<int>(value));
      return FN_OK;
    case FN_DEBUG_CLUSTER:
      if (value < 0 || value > 8) return FN_ERR_INVALID_ARG;
      g_cluster_mode.store(static_cast<int>(value));
      return FN_OK;
    case FN_DEBUG_DECODE_GROUPS:
      if (value < 0 || (value & 0xF) > 2 || ((value >> 4) & 0xF) > 3 || ((value >> 8) & 0xF) > 8 || (value >> 12))
        return FN_ERR_INVALID_ARG;
      g_group_mode.store(static_cast<int>(value));
      return FN_OK;
    case FN_DEBUG_PAIR_TILE:
      if (value < 0 || value > 2) return FN_ERR_INVALID_ARG;
      g_pair_tile.store(static_cast<int>(value));
      return FN_OK;
    case FN_DEBUG_PREFETCH:
      if (value < 0 || (value & 0xFF) > 2) return FN_ERR_INVALID_ARG;
      g_prefetch_mode.store(static_cast<int>(value & 0xFF));
      g_prefetch_iters.store(static_cast<int>(value >> 8));
      return FN_OK;
  }
  return FN_ERR_INVALID_ARG;
}

}  // extern "C"
