/*
 * fourtune.h -- C ABI of the W4A4G4 triple-branch linear layer on NVIDIA B200 (sm_100a).
 *
 * The layer is the one of "FourTune: Towards Fully 4-Bit Efficient Post-Training for
 * Diffusion Models" (arXiv 2607.05711), section 3.  Layout (PyTorch's): X [M, K] tokens
 * by input features, W and its residual R [N, K], Y [M, N].  The paper writes
 * Y = X W with W in R^{m x n}; the algebra is the same, transposed.
 *
 *   Eq. (1)  W ~= R + L_stab,  L_stab = Ls_up * Ls_down     (frozen, high precision)
 *   Eq. (2)  Y  = GEMM4(Q(X), Q(R)) + X L_stab^T + s (X A^T) B^T
 *   Eq. (3)  dX = GEMM4(Q(G), Q(R)^T) + G L_stab + s (G B) A
 *   sec. 3.2 dB = s G^T (X A^T),  dA = s (G B)^T X           (only the adapter trains)
 *
 * with G = dL/dY, LoRA factors A [r, K] and B [N, r], s = alpha / r.
 *
 * Q(.) is the 16x16-block NVFP4 quantizer (sections 3.1-3.2, Table 5): E2M1 element
 * codes, one UE4M3 scale per 16x16 block, one fp32 factor g per tensor:
 *   g  = 2688 / max|x|                              (fp32; g = 1 and all-zero output
 *                                                    when max|x| == 0 or g overflows)
 *   sb = UE4M3_rn_sat( fl32(fl32(max_block|x| / 6) * g) )
 *   code(x) = sign(x) | E2M1_rn_sat( fl32(x * fl32(g / val(sb))) )   (0 when sb == 0)
 *   xhat = val(code) * val(sb) / g
 * Q is applied offline to R and on the fly to X and G.  Q(R)^T is the same codes and
 * scales transposed block by block; nothing is requantized (section 3.2).
 *
 * CONVENTIONS (all entry points)
 *  - Every pointer argument named *_dev or held in an ft_* struct is DEVICE memory owned
 *    by the caller and must be 16-byte aligned.  Host pointers appear only where noted.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls are
 *    asynchronous: they enqueue kernels and return.  The returned status reports
 *    argument validation and launch errors only.
 *  - Errors detected on the device (a bounded wait that expired) are recorded in a
 *    status word inside the workspace; read it with fourtune_device_status().
 *  - Matrices are row-major and dense (row stride == number of columns) unless an
 *    `ld` argument says otherwise.  bf16 is IEEE bfloat16 stored as 16-bit words.
 *  - The library allocates no device memory and keeps no state between calls other
 *    than per-process caches (driver entry points, device attributes).  All scratch
 *    comes from the caller's workspace `ws` of `ws_bytes` bytes (256-byte aligned);
 *    query the size first.  The one exception is fourtune_quantize_block16_noalloc:
 *    its scratch is a fixed array of FT_NOALLOC_SCRATCH_BYTES in the library's own
 *    device memory (held by every GPU that loads the library, until exit), whose
 *    device address the library caches per device and CUDA context.
 *  - Kernels never trap.  Shapes are checked on the host before any launch.
 */
#ifndef FOURTUNE_H_
#define FOURTUNE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FT_OK = 0,
    FT_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad flag */
    FT_ERR_SHAPE = 2,       /* a dimension is not a supported multiple (see each call) */
    FT_ERR_ALIGN = 3,       /* a device pointer is not 16-byte aligned */
    FT_ERR_WORKSPACE = 4,   /* workspace missing or smaller than the query returned */
    FT_ERR_CUDA = 5,        /* a CUDA runtime or driver call failed */
    FT_ERR_UNSUPPORTED = 6, /* the current device is not sm_100 */
    FT_ERR_TIMEOUT = 7      /* (device status) a bounded wait inside a kernel expired */
} ft_status;

/* Human-readable name of a status code (static string). */
const char* fourtune_status_string(int status);

/*
 * A 16x16-block quantized matrix [rows, cols] (section 3.1 NVFP4, 16x16 blocks).
 *   codes  : uint8 [rows, cols/2]; element (i, 2j) in the low nibble of byte (i, j),
 *            element (i, 2j+1) in the high nibble; nibble = sign<<3 | E2M1 magnitude.
 *   scales : uint8 [rows/16, cols/16], UE4M3 scale of each 16x16 block (row-major).
 *   sf_mma : the same scales expanded to one scale per (row, 16 columns) and laid out
 *            for the tensor core's block-scaled MMA: 512-byte atoms, one per 128 rows
 *            x 64 columns, atoms of a 128-row band stored consecutively along the
 *            columns; inside an atom the scale of (row m, column block b) sits at byte
 *            16*(m%32) + 4*((m%128)/32) + b%4.  Size rows*cols/16 bytes.  Needs
 *            rows % 128 == 0 and cols % 64 == 0.  May be NULL on output (not written).
 *   g      : float[1], the tensor factor g.
 */
typedef struct {
    uint8_t* codes;
    uint8_t* scales;
    uint8_t* sf_mma;
    float* g;
    int64_t rows;
    int64_t cols;
} ft_fp4;

/*
 * One frozen-backbone linear layer with its adapter (Eq. 1-2).
 *   qr      : Q(R), rows = N, cols = K, sf_mma required.
 *   qr_t    : Q(R)^T, rows = K, cols = N, sf_mma required (written by
 *             fourtune_quantize_block16 with an out_t argument).  codes (and
 *             scales) may be NULL: the backward's dX GEMM then transposes Q(R)'s
 *             codes tile by tile in shared memory (section 3.2, transposition on
 *             the fly), which saves the second copy of the codes (N*K/2 bytes);
 *             sf_mma and g stay required.
 *   ls_down : bf16 [r_s, K]   (L_stab = ls_up * ls_down)
 *   ls_up   : bf16 [N, r_s]
 *   lora_a  : bf16 [r, K]
 *   lora_b  : bf16 [N, r]
 *   lora_scale : s = alpha / r.
 * r_s + r must be >= 1 and <= 240 (either may be 0).
 */
typedef struct {
    int64_t N;
    int64_t K;
    int32_t r_s;
    int32_t r;
    float lora_scale;
    ft_fp4 qr;
    ft_fp4 qr_t;
    const void* ls_down;
    const void* ls_up;
    const void* lora_a;
    const void* lora_b;
} ft_linear;

/* Input element types for fourtune_quantize_block16. */
#define FT_DTYPE_BF16 0
#define FT_DTYPE_F32 1

/*
 * Workspace bytes needed by fourtune_quantize_block16 for a [rows, cols] input with a
 * fused down-projection of rank r_down (0 for none).
 */
size_t fourtune_quantize_workspace_bytes(int64_t rows, int64_t cols, int32_t r_down);

/*
 * Q(.) of sections 3.1-3.2: quantize x [rows, cols] (row stride ld elements) into
 * 16x16-block NVFP4 codes and scales, optionally fused with a down-projection
 * (section 3.3 "LoRA Fusion": the quantizer and the low-rank down-projections read
 * the same input once).
 *   x_dev          : bf16 or fp32 (x_dtype = FT_DTYPE_BF16 / FT_DTYPE_F32), device.
 *   rows, cols     : multiples of 16 (128 and 64 when out->sf_mma or out_t is used).
 *   amax_or_null   : device float[1] holding max|x| to use for g, or NULL to compute
 *                    it (one extra read of x).  A caller-supplied value smaller than
 *                    the true maximum saturates codes; larger values are valid.
 *   down_dev       : bf16 [r_down, cols] or NULL; down_out_dev: fp32 [rows, r_down]
 *                    receives x * down^T (exact fp32 accumulation order not specified).
 *                    bf16 input only.
 *   out            : codes/scales/g required, sf_mma optional.
 *   out_t          : optional Q(x)^T (rows = cols, cols = rows), the transpose of the
 *                    same codes and scales (no requantization); sf_mma required when set.
 * Errors: FT_ERR_INVALID_ARG, FT_ERR_SHAPE, FT_ERR_ALIGN, FT_ERR_WORKSPACE, FT_ERR_CUDA.
 */
ft_status fourtune_quantize_block16(const void* x_dev, int32_t x_dtype, int64_t rows,
                                    int64_t cols, int64_t ld, const float* amax_or_null,
                                    const void* down_dev, int32_t r_down, float* down_out_dev,
                                    const ft_fp4* out, const ft_fp4* out_t, void* ws,
                                    size_t ws_bytes, void* stream);

/*
 * fourtune_quantize_block16_noalloc -- fourtune_quantize_block16 for callers that cannot
 * allocate device memory.  The paper has no counterpart; this is a library convenience.
 *
 * Who needs it: code that is handed only its input and output buffers and has no way to
 * obtain scratch memory -- for example a plugin running inside a host framework whose
 * interface passes just the tensors, or a process whose device memory is budgeted up
 * front and owned by another runtime, so a cudaMalloc here would fail or is not allowed.
 *
 * Instead of a caller workspace, the quantizer's scratch (status word, tensor max, the
 * down factor padded to the MMA width, the per-slice partial sums of the down-projection)
 * lives in one fixed array of FT_NOALLOC_SCRATCH_BYTES in the library's own device
 * memory.  Every GPU that loads the library holds that array until the process exits.
 * Arguments, shapes, results and errors are those of fourtune_quantize_block16; inputs
 * and outputs are still the caller's.
 *  - A problem whose scratch (fourtune_quantize_workspace_bytes) exceeds
 *    FT_NOALLOC_SCRATCH_BYTES is refused with FT_ERR_WORKSPACE before anything runs.
 *  - The first call on a device (and again the first call in a new CUDA context of that
 *    device, e.g. after cudaDeviceReset) looks up the array's device address, with that
 *    device current, and keeps it; make that first call before any stream capture.
 *  - All calls share the one array and it keeps the previous call's contents (the call
 *    clears what must start at zero).  Calls whose kernels can overlap on the GPU --
 *    different streams with no ordering between them -- race and give wrong results.
 *  - Errors detected on the device (FT_ERR_TIMEOUT) go to the array's status word, which
 *    only the kernels set: read and clear it with fourtune_device_status(NULL, ...).
 *  - It allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 */
#define FT_NOALLOC_SCRATCH_BYTES (8u << 20)
ft_status fourtune_quantize_block16_noalloc(const void* x_dev, int32_t x_dtype, int64_t rows,
                                            int64_t cols, int64_t ld, const float* amax_or_null,
                                            const void* down_dev, int32_t r_down,
                                            float* down_out_dev, const ft_fp4* out,
                                            const ft_fp4* out_t, void* stream);

/*
 * Q(x) in group-wise 1x16 blocks: one UE4M3 scale per row and 16 consecutive columns, the
 * granularity FourTune compares its 16x16 blocks with (section 4.3, "Impact of
 * Quantization Granularity", Table 5).  Same two-level scaling and the same arithmetic per
 * element as fourtune_quantize_block16; forward use only (1x16 blocks do not transpose).
 *   x_dev : bf16 [rows, cols], row stride ld elements.
 *   out   : codes [rows, cols/2], scales [rows, cols/16] (one byte per group), g, and
 *           sf_mma (optional; the tensor-core layout, per row and 16 columns as always).
 * Shapes: rows % 128 == 0, cols % 64 == 0, ld % 8 == 0, else FT_ERR_SHAPE.  Workspace:
 * fourtune_quantize_workspace_bytes(rows, cols, 0).
 */
ft_status fourtune_quantize_1x16(const void* x_dev, int64_t rows, int64_t cols, int64_t ld,
                                 const float* amax_or_null, const ft_fp4* out, void* ws, size_t ws_bytes,
                                 void* stream);

/* Workspace bytes for fourtune_linear_fwd / fourtune_linear_bwd with M tokens. */
size_t fourtune_linear_workspace_bytes(const ft_linear* layer, int64_t M);

/*
 * Forward pass, Eq. (2): Y = GEMM4(Q(X), Q(R)) + X Ls_down^T Ls_up^T + s X A^T B^T.
 *   x_dev      : bf16 [M, K].
 *   amax_or_null : device float[1] = max|X| (see fourtune_quantize_block16) or NULL.
 *   y_dev      : bf16 [M, N], written.
 *   t_saved_dev: fp32 [M, r_s + r], written: X [Ls_down; A]^T, kept for the backward.
 * Shapes: M % 128 == 0, N % 256 == 0, K % 256 == 0.
 */
ft_status fourtune_linear_fwd(const ft_linear* layer, const void* x_dev, int64_t M,
                              const float* amax_or_null, void* y_dev, float* t_saved_dev,
                              void* ws, size_t ws_bytes, void* stream);

/*
 * fourtune_linear_fwd with X quantized group-wise 1x16 (fourtune_quantize_1x16) instead
 * of in 16x16 blocks: the Table 5 comparison, for forward-only use.  Arguments, shapes and
 * workspace as fourtune_linear_fwd.
 */
ft_status fourtune_linear_fwd_1x16(const ft_linear* layer, const void* x_dev, int64_t M,
                                   const float* amax_or_null, void* y_dev, float* t_saved_dev, void* ws,
                                   size_t ws_bytes, void* stream);

/*
 * Forward pass with GELU (tanh form) fused into the 4-bit GEMM's epilogue, for the first
 * linear of an MLP (section 3.3 "MLP Fusion": the FC1 GEMM is fused with what FC2's
 * quantization needs, so the activation is not read back and re-written by a separate
 * pass).
 *   p_dev      : bf16 [M, N], written: the layer output P (exactly fourtune_linear_fwd's y).
 *   h_dev      : bf16 [M, N], written: H = bf16(gelu_tanh(P)) evaluated in fp32 from the bf16
 *                P (the same bits as fourtune_gelu_tanh_fwd on p_dev).
 *   h_amax_dev : device float[1], written: max |H|.  Pass it as amax_or_null to the next
 *                layer's fourtune_linear_fwd, which then needs no pass of its own over H.
 *   The other arguments, shapes and the workspace are those of fourtune_linear_fwd.  P is
 *   what the backward's gelu' needs; H is the next layer's input (its forward and its dA).
 */
ft_status fourtune_linear_fwd_gelu(const ft_linear* layer, const void* x_dev, int64_t M,
                                   const float* amax_or_null, void* p_dev, void* h_dev,
                                   float* h_amax_dev, float* t_saved_dev, void* ws, size_t ws_bytes,
                                   void* stream);

/*
 * Backward pass, Eq. (3) and the adapter gradients of section 3.2.
 *   x_dev       : bf16 [M, K], the forward input.
 *   t_saved_dev : fp32 [M, r_s + r] from fourtune_linear_fwd.
 *   dy_dev      : bf16 [M, N], G = dL/dY.
 *   amax_or_null: device float[1] = max|G| or NULL.
 *   dx_dev      : bf16 [M, K], written: GEMM4(Q(G), Q(R)^T) + G Ls_up Ls_down + s G B A.
 *   da_dev      : fp32 [r, K], written (overwritten, not accumulated): s (G B)^T X.
 *   db_dev      : fp32 [N, r], written (overwritten, not accumulated): s G^T (X A^T).
 * Shapes as for the forward.  R and L_stab get no gradient (frozen).
 */
ft_status fourtune_linear_bwd(const ft_linear* layer, const void* x_dev, const float* t_saved_dev,
                              const void* dy_dev, int64_t M, const float* amax_or_null,
                              void* dx_dev, float* da_dev, float* db_dev, void* ws,
                              size_t ws_bytes, void* stream);

/*
 * Backward pass of an MLP's second linear with the GELU derivative fused into the dX
 * GEMM's epilogue (section 3.3 "MLP Fusion", backward side): instead of dX (= dH, the
 * gradient at the GELU output) it writes dP = bf16(bf16(dH) * gelu_tanh'(P)), the same bits
 * as fourtune_linear_bwd followed by fourtune_gelu_tanh_bwd, so dH is never stored.
 *   p_dev  : bf16 [M, K], the pre-activation P (p_dev of fourtune_linear_fwd_gelu).
 *   dp_dev : bf16 [M, K], written (in place of dx_dev).
 *   The other arguments (x_dev is this layer's input H), shapes and the workspace are those
 *   of fourtune_linear_bwd.
 */
ft_status fourtune_linear_bwd_gelu(const ft_linear* layer, const void* x_dev, const float* t_saved_dev,
                                   const void* dy_dev, int64_t M, const float* amax_or_null,
                                   const void* p_dev, void* dp_dev, float* da_dev, float* db_dev, void* ws,
                                   size_t ws_bytes, void* stream);

/*
 * Reads (synchronously, on `stream`) the device status word that the kernels of the
 * calls using workspace `ws` left behind since it was last read: FT_OK or
 * FT_ERR_TIMEOUT.  *status_out is a HOST pointer.  Clears the word.  ws == NULL reads
 * the status word of fourtune_quantize_block16_noalloc's fixed scratch array on the
 * current device instead.
 */
ft_status fourtune_device_status(void* ws, int32_t* status_out, void* stream);

/*
 * Failure-detection self-test: launches one kernel that waits, with the bounded wait
 * every pipelined kernel of this library uses, on an mbarrier that nothing completes;
 * after limit_ns nanoseconds (1 .. 1e9) it gives up and writes FT_ERR_TIMEOUT into the
 * status word at the start of `ws` (the same place fourtune_device_status reads).
 * The kernel then returns normally and the CUDA context stays usable.
 */
ft_status fourtune_selftest_bounded_wait(int64_t limit_ns, void* ws, void* stream);

/*
 * GELU (tanh form) between the MLP linears (section 3.3 "MLP Fusion" names GeLU):
 *   fwd: h = bf16(0.5 p (1 + tanh(sqrt(2/pi) (p + 0.044715 p^3))))
 *   bwd: dp = bf16(dh * gelu'(p))
 * p, h, dh, dp: bf16 device arrays of n elements (n % 8 == 0).
 */
ft_status fourtune_gelu_tanh_fwd(const void* p_dev, void* h_dev, int64_t n, void* stream);
ft_status fourtune_gelu_tanh_bwd(const void* p_dev, const void* dh_dev, void* dp_dev, int64_t n,
                                 void* stream);

/*
 * Codec access for exhaustive checks of the conversions the quantizer uses:
 * out[i] = E2M1 code (with sign) of v[i], or UE4M3 code of v[i] (v[i] >= 0), both
 * round-to-nearest-even with saturation.  v: fp32 device [n]; out: uint8 device [n].
 */
ft_status fourtune_encode_e2m1(const float* v_dev, int64_t n, uint8_t* out_dev, void* stream);
ft_status fourtune_encode_ue4m3(const float* v_dev, int64_t n, uint8_t* out_dev, void* stream);

/*
 * Instrumentation for benchmarks.
 * fourtune_launch_count: number of kernels this library has launched in this process.
 * fourtune_time_next_launch: records the caller's CUDA events (cudaEvent_t, created by
 *   the caller) on the launch stream immediately before and after the NEXT launch of the
 *   given kernel kind (FT_KERNEL_*), then forgets them.  Either event may be NULL.
 *   Returns FT_ERR_INVALID_ARG for an unknown kind.
 */
#define FT_KERNEL_GEMM 0      /* 4-bit GEMM with the low-rank tail (forward and dX) */
#define FT_KERNEL_QUANT 1     /* 16x16 block quantizer */
#define FT_KERNEL_AMAX 2      /* tensor max pass (the layer forward's: its prologue, which also builds the factors) */
#define FT_KERNEL_LOWRANK 3   /* low-rank split sum */
#define FT_KERNEL_LORA_DB 4   /* adapter gradient dB */
#define FT_KERNEL_LORA_DA 5   /* adapter gradient dA */
#define FT_KERNEL_KINDS 6
uint64_t fourtune_launch_count(void);
ft_status fourtune_time_next_launch(int32_t kernel, void* ev_before, void* ev_after);

#ifdef __cplusplus
}
#endif

#endif /* FOURTUNE_H_ */
