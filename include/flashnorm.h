/*
 * flashnorm.h — C ABI of the B200 (sm_100a) fused RMSNorm + linear projection
 * in the FlashNorm form.
 *
 * The method (FlashNorm talk summary, "RMS norm는 연산량 1할인데 왜 33번 호출로
 * 속도를 갉아먹나", news.juniverse.app):
 *   Proposal 1 ("웨이트리스 정규화", weightless normalisation): fold the norm
 *     gain into the projection offline, W' = diag(g) W.
 *   Proposal 2 ("지연된 정규화", deferred normalisation): run the matmul on the
 *     raw activations on the tensor cores, reduce each row's sum of squares on
 *     the vector units at the same time, then post-scale by 1/rms(x).
 *   Bug/cause/fix bullets: the post-scale must wait explicitly for both the
 *     matmul and the reduction.
 * SwiGLU epilogue: the fused FC1 + SwiGLU of the FlashInfer PR #5521 analysis
 * ("Register-level SwiGLU" design item): out = silu(gate) * up.
 * Further forms of the same call: the SwiGLU output quantised to NVFP4 in the
 * epilogue (FlashInfer PR #4040 analysis), and a row-parallel split of d for
 * tensor parallelism (per-rank partial products and sums of squares, one
 * all-reduce, a post-scale), which Proposal 2 makes a single exchange.
 *
 * Definitions (the pages print no formula; these are the plain readings):
 *   r[m]  = 1 / sqrt( (1/d) sum_k x[m,k]^2 + eps )
 *   y     = r[m] * sum_k x[m,k] W'[k,n]              (= RMSNorm(x; g) @ W)
 *   swiglu: out[m,n] = silu(r[m] * (x W'_gate)[m,n]) * (r[m] * (x W'_up)[m,n]),
 *           silu(z) = z / (1 + e^-z)
 * fp32 accumulation, one round-to-nearest-even to bf16 at the store.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers, owned and allocated by the
 *     caller; the library never allocates, frees or synchronises in the
 *     compute calls.  Tensors are dense row-major.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  Argument errors are returned synchronously, before any launch.
 *     A failed launch returns FN_ERR_CUDA.  A device-side wait that ran out of
 *     time is reported later by fn_query_device_status.
 *   - Base pointers must be 16-byte aligned (TMA); FN_ERR_ALIGNMENT otherwise.
 *   - No exception crosses the ABI; the functions are re-entrant.  Calls that
 *     may overlap on the GPU need distinct workspaces.
 */
#ifndef FLASHNORM_H_
#define FLASHNORM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* cudaStream_t without including the CUDA headers */
typedef struct CUstream_st* fn_stream_t;

typedef enum {
  FN_OK = 0,
  FN_ERR_INVALID_ARG = 1,        /* null pointer, negative size, bad eps or enum */
  FN_ERR_UNSUPPORTED_SHAPE = 2,  /* d % 64, N % 128, fp8 d % 128, sizes over int32 */
  FN_ERR_ALIGNMENT = 3,          /* a base pointer not 16-byte aligned */
  FN_ERR_ALIAS = 4,              /* the output overlaps an input or the workspace */
  FN_ERR_WORKSPACE = 5,          /* workspace missing or smaller than fn_workspace_size */
  FN_ERR_CUDA = 6,               /* a CUDA runtime/driver call failed */
  FN_ERR_TIMEOUT = 7,            /* a device-side wait exceeded its time budget */
  FN_ERR_UNSUPPORTED_DEVICE = 8  /* not a compute capability 10.0 (B200-class) GPU */
} fn_status;

typedef enum {
  FN_W_BF16 = 0,            /* W' stored as bf16 [d, ncols] */
  FN_W_FP8_E4M3_B128 = 1,   /* W' stored as e4m3 [d, ncols] + fp32 scales [d/128, ncols/128] */
  FN_W_MXFP8_E4M3 = 2       /* W' stored as e4m3 [d, ncols] + ue8m0 scale bytes, one per 32 k values
                               of each column, in the chunked layout below */
} fn_wtype;

/*
 * MXFP8 weights (FN_W_MXFP8_E4M3): the block-scaled format the tensor cores'
 * kind::mxf8f6f4 MMAs read (the FlashInfer PR #5521 analysis, design item 4,
 * runs its low-precision FC1 on the block-scaled MMA family).  Per stored
 * column n and block j of 32 consecutive k (rows 32j .. 32j+31) a shared
 * exponent E = ceil(log2(amax / 448)), the smallest E with amax <= 448 * 2^E
 * (clamped to [-127, 127]; -127 for an all-zero block), stored as the byte
 * E + 127; codes q = RN_e4m3(g*W / 2^E); value e4m3(q) * 2^E.  The d*ncols/32
 * scale bytes are grouped by 128-deep k groups (4 blocks); in each group one
 * 512-byte chunk per 128 columns; inside a chunk the byte of column n, block
 * j sits at 16*(n mod 32) + 4*((n mod 128) div 32) + (j mod 4).  So the byte
 * of (n, j) is at 512*((j div 4)*(ncols/128) + n div 128) + that offset, and
 * a row slice of the weight on 128-row boundaries owns a contiguous range.
 * Passed through the `scales` argument (its pointer type is nominal here);
 * 16-byte aligned; needs d % 128 == 0.
 */

/*
 * fn_fold_weights — offline fold (Proposal 1, weightless normalisation).
 *   W0      bf16 [d, N]: the projection weight (the gate half for SwiGLU)
 *   W1      bf16 [d, N]: the up half for SwiGLU, or NULL for a plain projection
 *   g       fp32 [d]: the norm gain, as the effective multiplier (a (1+w) style
 *           gain is the caller's conversion)
 *   out_type FN_W_BF16: Wp = bf16 [d, ncols], Wp[k,n] = RN_bf16(fp32 g[k] * W[k,n])
 *           FN_W_FP8_E4M3_B128: Wp = e4m3 bytes [d, ncols] and scales fp32
 *           [d/128, ncols/128]: per 128x128 block s = amax|g*W| / 448 (1 if the
 *           block is all zero), Wp = RN_e4m3_satfinite(fp32(g*W) / s); needs
 *           d % 128 == 0.
 *           FN_W_MXFP8_E4M3: Wp = e4m3 bytes [d, ncols] and `scales` receives
 *           the d*ncols/32 ue8m0 bytes described above (fp32 g*W, one exact
 *           power-of-two scaling, one RN to e4m3); needs d % 128 == 0.
 *   ncols = N, or 2N with W1: then 128-column tiles alternate gate, up, gate,
 *           up (stored columns [256j, 256j+128) = gate columns [128j, 128j+128),
 *           [256j+128, 256j+256) = the same up columns).
 *   Shapes: d >= 1, d % 64 == 0 (128 for fp8), N % 128 == 0.
 *   Wp must not overlap W0, W1 or g (FN_ERR_ALIAS).
 */
fn_status fn_fold_weights(const void* W0, const void* W1, const float* g, int64_t d, int64_t N,
                          fn_wtype out_type, void* Wp, float* scales, fn_stream_t stream);

/*
 * fn_workspace_size — bytes of workspace a call with these sizes needs.
 * The workspace holds a 256-byte header (the device status word) and, for
 * M <= 64, the per-CTA partial sums of the split-K decode path; with fp8
 * weights and 17 <= M <= 64 also the activations split once per call into
 * the two e4m3 operand parts (2 x 64 x d bytes at most) with their scale
 * factors and per-block sums of squares; with fp8 weights and M >= 33 the
 * activations split once per call for the block-scale promotion kernel
 * (2 M d bytes of e4m3 codes, 8 bytes per row and 128-deep k block), and at
 * M >= 1024 at least one bf16 copy of the weight (2 d ncols
 * bytes), which the NVFP4 and partial-output calls convert once per call with
 * the rounding of the on-chip conversion (bf16(fp32(q) * s)); with MXFP8
 * weights at M > 64 the larger of the same bf16 copy (NVFP4, partial and
 * AdaLN outputs) and the promotion kernel's split activations (2 M d bytes,
 * their scale chunks over whole 128-row blocks and per-block sums of squares),
 * and at M <= 64 the activations split once per call (2 x 64 x d bytes at
 * most, their scale chunks and per-group sums of squares).  Zero it once
 * before its first use (the status word must start at zero); the calls keep
 * the status word at zero unless a device-side wait times out.  Depends on
 * the SM count of the current device (148 is assumed when no device is
 * visible).
 */
size_t fn_workspace_size(int64_t M, int64_t d, int64_t N, fn_wtype wt, int swiglu);

/*
 * fn_norm_proj — y[M, N] = RMSNorm(x; g, eps) @ W, computed as
 *   r[m] * (x @ W')[m, :] with W' from fn_fold_weights (Proposal 2).
 *   x       bf16 [M, d] raw activations (never normalised in memory)
 *   Wp      folded weight [d, N] of type wt (scales: fp32 [d/128, N/128] for fp8,
 *           the chunked ue8m0 bytes for MXFP8)
 *   eps     >= 0 and finite, added to the mean inside the square root
 *   y       bf16 [M, N] output; must not overlap x, Wp, scales or workspace
 *   workspace, ws_bytes  >= fn_workspace_size(M, d, N, wt, 0), zeroed before first use
 *   M == 0 is a no-op.  M <= 64 runs the split-K decode kernel (plus a small
 *   fix-up kernel for the column tiles whose k range it split), larger M the
 *   tensor-core tile kernel; both are deterministic (repeated calls with the
 *   same inputs give the same bits).  fp8 weights from M = 33 (bf16
 *   output; NVFP4 and partial outputs from M = 65): the stored
 *   e4m3 codes go to the tensor cores as they are, against the activations
 *   split exactly into two e4m3 parts per row and 128-deep k block (one
 *   power-of-two scale each); each k block's exact sums are scaled by the
 *   block scale and added to fp32 sums in k order.  MXFP8 weights: at M <= 64 the e4m3
 *   codes and their scales go to block-scaled MMAs as stored (the bf16
 *   activations split exactly into two e4m3 parts sharing one power-of-two
 *   scale per 32 k values); at M > 64 the promotion tile kernel does the same
 *   per 128 x 256 tile (the split per 32-deep block, its powers of two as the
 *   activations' scale bytes, block-scaled MMAs over the whole k range).  The
 *   NVFP4 and partial outputs and AdaLN at M > 64 convert the weight to bf16
 *   once per call into the workspace (an exact conversion) for the tile kernel.
 *   bf16 weights at M <= 64 with a plain projection and bf16 output may run
 *   a decode kernel that splits k inside thread-block clusters over groups of
 *   columns and adds the partials over distributed shared memory (no fix-up
 *   kernel); its results are deterministic too.
 */
fn_status fn_norm_proj(const void* x, int64_t M, int64_t d, const void* Wp, const float* scales, fn_wtype wt,
                       int64_t N, float eps, void* y, void* workspace, size_t ws_bytes, fn_stream_t stream);

/*
 * fn_norm_proj_swiglu — out[M, N] = silu(h W_gate) * (h W_up), h = RMSNorm(x; g, eps),
 * computed as silu(r * (x W'_gate)) * (r * (x W'_up)): r is applied to both halves
 * before the nonlinearity.  Wp is the interleaved [d, 2N] fold of (W_gate, W_up);
 * scales fp32 [d/128, 2N/128] for fp8.  Other arguments as fn_norm_proj, with
 * workspace >= fn_workspace_size(M, d, N, wt, 1).
 */
fn_status fn_norm_proj_swiglu(const void* x, int64_t M, int64_t d, const void* Wp, const float* scales,
                              fn_wtype wt, int64_t N, float eps, void* out, void* workspace, size_t ws_bytes,
                              fn_stream_t stream);

/*
 * fn_norm_proj_swiglu_nvfp4 — the SwiGLU output of fn_norm_proj_swiglu written
 * in NVFP4 for the projection that follows, from the epilogue registers (no
 * bf16 intermediate in memory), as the FlashInfer PR #4040 analysis fuses
 * silu_and_mul with its NVFP4 quantisation (16 elements per scale factor, a
 * global scale).  For each row m and block b of 16 consecutive output columns,
 * with v the fp32 SwiGLU value and gs = *global_scale:
 *   sf[m, b] = RN_e4m3_satfinite(gs * max|v| / 6)         (6: largest e2m1 value)
 *   q[m, n]  = RN_e2m1_satfinite(v * (gs / sf[m, b]))      (0 where sf is 0)
 * A block holding a non-finite value gets sf = 0x7F (e4m3 NaN) and zero codes.
 * The consumer dequantises as e2m1(q) * e4m3(sf) / gs.
 *   global_scale  device pointer to one fp32 value, > 0 and finite (read on
 *                 the device, so a CUDA graph may keep it while it changes)
 *   out_q         [M, N/2] bytes: two e2m1 codes per byte, the even column in
 *                 the low nibble; 16-byte aligned
 *   out_sf        [M, N/16] e4m3 scale bytes, row-major (not the swizzled
 *                 tensor-core layout); 16-byte aligned
 * Other arguments and the workspace as fn_norm_proj_swiglu.  The outputs must
 * not overlap each other, the inputs, global_scale or the workspace
 * (FN_ERR_ALIAS).  M == 0 is a no-op.
 */
fn_status fn_norm_proj_swiglu_nvfp4(const void* x, int64_t M, int64_t d, const void* Wp, const float* scales,
                                    fn_wtype wt, int64_t N, float eps, const float* global_scale, void* out_q,
                                    void* out_sf, void* workspace, size_t ws_bytes, fn_stream_t stream);

/*
 * AdaLN-modulated form (the "RMSNorm + AdaLN" front of the fused FC1 on the
 * FlashInfer PR #5521 analysis: its API takes the norm weight, an AdaLN scale,
 * an AdaLN shift and an index for AdaLN; the page prints no formula).
 * Reading: each token m selects condition c = adaln_index[m], and the
 * normalised row is modulated before the projection,
 *   h[m, k] = RMSNorm(x; g, eps)[m, k] * scale[c, k] + shift[c, k],  y = h @ W
 *   (SwiGLU: out = silu(h @ W_gate) * (h @ W_up)),
 * scale being the effective multiplier (a DiT-style 1 + scale is the
 * caller's conversion).  With W' = diag(g) W this is
 *   y[m, :] = r[m] * ((x[m, :] * scale[c, :]) @ W') + B[c, :],
 *   B[c, :] = shift[c, :] @ W   (the unfolded weight),
 * so the scale multiplies the raw activations on chip (one rounding of
 * x * scale to bf16 for the MMA; the sum of squares is taken from the raw x),
 * the 1/rms scalar stays deferred, and the shift becomes a per-condition bias
 * row, computed once by fn_adaln_shift_bias.
 *
 * fn_adaln_shift_bias — B fp32 [n_cond, ncols] = shift fp32 [n_cond, d] times
 *   the unfolded weight (W0, and W1 for SwiGLU: columns in the interleaved
 *   stored order of fn_fold_weights), fp32 products summed in ascending k.
 *   Alignment: W0/W1 16 bytes, shift and B 4 bytes.  B must not overlap the
 *   inputs (FN_ERR_ALIAS).
 */
fn_status fn_adaln_shift_bias(const float* shift, int64_t n_cond, const void* W0, const void* W1, int64_t d,
                              int64_t N, float* B, fn_stream_t stream);

/*
 * fn_norm_proj_adaln — the AdaLN-modulated fn_norm_proj (swiglu = 0) or
 * fn_norm_proj_swiglu (swiglu != 0).
 *   adaln_scale  fp32 [n_cond, d], 16-byte aligned
 *   shift_bias   fp32 [n_cond, ncols] from fn_adaln_shift_bias, 16-byte aligned
 *   adaln_index  int32 [M]: the condition of each row; a row whose index lies
 *                outside [0, n_cond) gets NaN outputs (nothing is read out of
 *                range)
 *   workspace    >= fn_workspace_size_adaln(d, N, wt, swiglu), zeroed before
 *                first use
 * Runs the tensor-core tile kernel at every M; e4m3 and MXFP8 weights are
 * converted to bf16 once per call into the workspace first.  bf16 output only.
 * Other arguments, layout and errors as fn_norm_proj.
 */
fn_status fn_norm_proj_adaln(const void* x, int64_t M, int64_t d, const void* Wp, const float* scales, fn_wtype wt,
                             int64_t N, int swiglu, float eps, const float* adaln_scale, const float* shift_bias,
                             const int32_t* adaln_index, int64_t n_cond, void* y, void* workspace, size_t ws_bytes,
                             fn_stream_t stream);

/* fn_workspace_size_adaln — workspace bytes of fn_norm_proj_adaln: the 256-byte
 * header, plus a bf16 copy of the weight (2 d ncols bytes) for e4m3 and MXFP8
 * weights. */
size_t fn_workspace_size_adaln(int64_t d, int64_t N, fn_wtype wt, int swiglu);

/*
 * fn_norm_proj_swiglu_nvfp4_swizzled — fn_norm_proj_swiglu_nvfp4 with the
 * scale bytes in the layout block-scaled tensor-core GEMMs read directly (the
 * "swizzled" scale factors, is_swizzled, of the FlashInfer PR #4040 analysis),
 * so the down projection needs no re-layout pass.  Codes as
 * fn_norm_proj_swiglu_nvfp4.  out_sf holds ceil(M/128)*128 * N/16 bytes: rows
 * in blocks of 128 and scale columns (one per 16 output columns) in groups of
 * 4 form 512-byte chunks; chunk (m div 128, j div 4) sits at byte
 * 512 * ((m div 128) * (N/64) + j div 4), and inside it the scale of row m,
 * column j at 16*(m mod 32) + 4*((m mod 128) div 32) + (j mod 4).  Bytes of
 * the padding rows (M .. ceil(M/128)*128 - 1) are not written.
 */
fn_status fn_norm_proj_swiglu_nvfp4_swizzled(const void* x, int64_t M, int64_t d, const void* Wp, const float* scales,
                                             fn_wtype wt, int64_t N, float eps, const float* global_scale, void* out_q,
                                             void* out_sf, void* workspace, size_t ws_bytes, fn_stream_t stream);

/*
 * Row-parallel (d-split) projection, for tensor parallelism that shards the
 * input width d across ranks.  The deferred normalisation (FlashNorm talk
 * summary, Proposal 2) makes 1/rms a per-row factor applied after the matmul,
 * and sum_k x[m,k]^2 splits over k like the matmul, so each rank computes the
 * unscaled products and the sum of squares of its own k range, one all-reduce
 * (sum) of one buffer per rank combines them, and fn_post_scale finishes.
 *
 * fn_norm_proj_partial — this rank's share:
 *   x         bf16 [M, d] — this rank's contiguous columns of the activations
 *             (d = the rank's width: % 64, % 128 with fp8 weights)
 *   Wp        this rank's rows of the folded weight [d, ncols] (a row slice of
 *             fn_fold_weights' output; for fp8 the matching rows of scales, so
 *             the slice starts on a 128-row boundary)
 *   ncols     stored columns: N for a plain projection, 2N for a SwiGLU weight
 *             (computed as a plain projection of its stored columns here)
 *   partial   fp32, M * ncols + M values, 16-byte aligned: [M, ncols] sums
 *             x @ Wp in stored column order, then [M] sums of x^2 over this
 *             rank's columns; nothing is post-scaled
 *   workspace >= fn_workspace_size(M, d, ncols, wt, 0)
 *   M == 0 is a no-op.  The partial buffer must not overlap the inputs or the
 *   workspace (FN_ERR_ALIAS).
 */
fn_status fn_norm_proj_partial(const void* x, int64_t M, int64_t d, const void* Wp, const float* scales,
                               fn_wtype wt, int64_t ncols, float* partial, void* workspace, size_t ws_bytes,
                               fn_stream_t stream);

/*
 * fn_post_scale — finish a row-parallel projection from the summed partial
 * buffer (the all-reduce of every rank's fn_norm_proj_partial output):
 *   r[m] = 1/sqrt(ssq[m] / d_total + eps), d_total the full input width;
 *   y = r * acc (plain), or silu(r * gate) * (r * up) for swiglu != 0, with
 *   the gate and up columns read from the interleaved stored order;
 *   one round to bf16 into y [M, N], 16-byte aligned, not overlapping partial;
 *   M * N < 2^42 (one thread per 8 outputs), else FN_ERR_UNSUPPORTED_SHAPE.
 * With one rank (d_total = d) the result equals fn_norm_proj on the same
 * inputs up to the rounding order of the sums: bit for bit for M > 64 (every
 * column tile reduces a row's sum of squares in the same k order), while for
 * M <= 64 the fused call may cut different column tiles' k ranges at
 * different points, and the partial buffer carries one sum of squares per row.
 */
fn_status fn_post_scale(const float* partial, int64_t M, int64_t N, int swiglu, int64_t d_total, float eps, void* y,
                        fn_stream_t stream);

/*
 * fn_norm_proj_static — fn_norm_proj for callers that cannot allocate device
 * memory, so cannot pass a workspace: code recording work under a CUDA stream
 * capture (where cudaMalloc is not permitted), plug-ins whose host application
 * owns every device allocation, and loops that must never call cudaMalloc
 * because it can synchronise the device.  The pages have no counterpart of
 * this entry point; it only moves the scratch memory.
 *   Arguments, layout and results as fn_norm_proj, minus the workspace.  The
 *   call's scratch (status word, split-K partials, and for fp8 weights the
 *   activations split once per call) lives in a fixed 8 MiB array inside the
 *   library that every GPU loading the library holds until the process
 *   exits.  A shape is served exactly when fn_workspace_size(M, d, N, wt, 0)
 *   <= 8 MiB; larger ones are rejected with FN_ERR_WORKSPACE before any
 *   launch.  On a 148-SM B200 that admits bf16 weights at every M > 64 and at
 *   M <= 32, M in 33..64 while the split-K partials stay under 8 MiB; fp8
 *   weights at M <= 64 under the same rule, and at M > 64 while the split
 *   activations (2 M d bytes, plus 8 bytes per row and 128-deep k block) fit,
 *   and at M >= 1024 only while a bf16 copy of the weight (2 d N bytes) would
 *   fit too.
 *   The array is zero when the library loads, so no set-up copy is made; the
 *   first call on a device only fetches the array's device address (a host
 *   query): make that first call before any stream capture.  All calls on a
 *   device share the array and it keeps the last call's contents; calls that
 *   may overlap on the GPU race on it.  A device-side wait that ran out of
 *   time is recorded in the array's status word: fn_query_static_status
 *   reports and clears it.  The call allocates nothing.
 */
fn_status fn_norm_proj_static(const void* x, int64_t M, int64_t d, const void* Wp, const float* scales,
                              fn_wtype wt, int64_t N, float eps, void* y, fn_stream_t stream);

/*
 * fn_query_static_status — fn_query_device_status for the scratch array of
 * fn_norm_proj_static on the current device: synchronises `stream`, reads and
 * clears the status word.  Returns FN_OK or FN_ERR_TIMEOUT; *detail (if not
 * NULL) receives the raw word.  Allocates nothing.
 */
fn_status fn_query_static_status(unsigned int* detail, fn_stream_t stream);

/*
 * fn_query_device_status — synchronises `stream`, reads and clears the status
 * word in `workspace`.  Returns FN_OK or FN_ERR_TIMEOUT; *detail (if not NULL)
 * receives the raw word (bits 8-15 name the wait site that gave up).
 */
fn_status fn_query_device_status(void* workspace, unsigned int* detail, fn_stream_t stream);

/*
 * Unfused-chain helpers, for baselines (FlashInfer PR #5521 analysis,
 * "Segmented Chain" section: norm, then GEMM, then activation, each through HBM).
 * fn_rmsnorm: h[M, d] = bf16((x * r) * g).  fn_dequant_fp8: W[d, ncols] =
 * bf16(e4m3(q) * s).  Same conventions as above.
 */
fn_status fn_rmsnorm(const void* x, int64_t M, int64_t d, const float* g, float eps, void* h,
                     fn_stream_t stream);
fn_status fn_dequant_fp8(const void* q, const float* scales, int64_t d, int64_t ncols, void* W,
                         fn_stream_t stream);
/* fn_dequant_mxfp8: W[d, ncols] = bf16(e4m3(q) * 2^(s - 127)), s the chunked
 * MXFP8 scale bytes (exact for scales a fold produces). */
fn_status fn_dequant_mxfp8(const void* q, const void* scales, int64_t d, int64_t ncols, void* W,
                           fn_stream_t stream);

/* Human-readable name of a status code (static string). */
const char* fn_status_string(fn_status s);

/* ABI version of this library (increments on any signature change). */
int fn_version(void);

/* Number of kernels this library has enqueued in this process (all devices,
 * all streams); for accounting in benchmarks and tests. */
uint64_t fn_kernel_launches(void);

/*
 * fn_set_debug — process-wide knobs for tests and diagnostics (not thread-safe;
 * set them before issuing work):
 *   FN_DEBUG_WAIT_BUDGET_NS   per-wait time limit inside the kernels (default 2e9)
 *   FN_DEBUG_WITHHOLD_ARRIVE  1: the reducers withhold their first arrival, so the
 *                             epilogue's wait must run out (exercises FN_ERR_TIMEOUT)
 *   FN_DEBUG_FORCE_PATH       0 auto, 1 decode kernel (M <= 64 only), 2 tile kernel,
 *                             3 tile kernel on single SMs (never the pair kernel),
 *                             4 tile path, with fp8 weights through the on-chip
 *                             weight conversion (M < 1024) or the dequantised copy
 *                             instead of the block-scale promotion kernel
 *   FN_DEBUG_PREFETCH         decode path: weight prefetch into L2 before waiting on
 *                             the previous kernel; value = mode | (k_blocks << 8),
 *                             mode 0 off, 1 TMA prefetch, 2 per-thread prefetch
 *                             (default: mode 2, 8 k-blocks; the cluster decode kernel
 *                             prefetches at most its ring depth)
 *   FN_DEBUG_CLUSTER          decode path: 1 (default) split K inside thread-block
 *                             clusters when the column tiles fill at most half the SMs,
 *                             with the largest cluster size whose clusters all fit at
 *                             once; 2..8 start from that size; 0 always stream-K + fix-up
 *   FN_DEBUG_DECODE_GROUPS    decode path, bf16 weights, plain projection, bf16 output:
 *                             0 (default) column groups per thread-block cluster (k split
 *                             across the cluster, partials reduced in distributed shared
 *                             memory, no fix-up kernel) where that balances the SMs about
 *                             as well as stream-K; 1 never; 2 whenever such a plan fits;
 *                             2 | (T << 4) | (S << 8): T boxes of 64 columns per cluster
 *                             of S CTAs when that plan fits (T 1..3, S 2..8)
 *   FN_DEBUG_PAIR_TILE        tile path on pairs of SMs (bf16 weights, M >= 512): 0 automatic,
 *                             1 256 x 256 output tiles (two accumulators, overlapped epilogue),
 *                             2 256 x 512 output tiles (two pair MMAs per K step)
 */
enum { FN_DEBUG_WAIT_BUDGET_NS = 1, FN_DEBUG_WITHHOLD_ARRIVE = 2, FN_DEBUG_FORCE_PATH = 3, FN_DEBUG_PREFETCH = 4,
       FN_DEBUG_CLUSTER = 5, FN_DEBUG_DECODE_GROUPS = 6, FN_DEBUG_PAIR_TILE = 7 };
fn_status fn_set_debug(int key, int64_t value);

#ifdef __cplusplus
}
#endif

#endif /* FLASHNORM_H_ */
