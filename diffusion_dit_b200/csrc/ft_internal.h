// Host-side declarations shared by the library's translation units (not public).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "fourtune.h"

namespace ft {

// Device address of fourtune_quantize_block16_noalloc's fixed scratch array on the
// current device and context, looked up on first use (ft_noalloc.cu).
ft_status noalloc_scratch(void** out);

// Instrumentation (ft_api.cu): every launcher calls before_launch(kind, stream) and
// after_launch(kind, stream) around its kernel launch.
enum KernelKind { K_GEMM = 0, K_QUANT = 1, K_AMAX = 2, K_LOWRANK = 3, K_LORA_DB = 4, K_LORA_DA = 5,
                  K_OTHER = 6 };
void before_launch(int kind, cudaStream_t stream);
void after_launch(int kind, cudaStream_t stream);

// Every kernel of the library is launched through launch_k with programmatic stream
// serialization: the next kernel on the stream may be scheduled while this one still
// runs (hiding launch latency and its prologue), and every kernel executes
// griddepcontrol.wait before its first global-memory access, so results are as if the
// kernels ran one after another.  Kernels call griddepcontrol.launch_dependents early.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                     Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// GEMM epilogue variants, one kernel instantiation each (the plain one carries no GELU code)
enum EpilogueKind { kEpiPlain = 0, kEpiGelu = 1, kEpiGeluBwd = 2 };

// The adapter-gradient kernel's CTA schedule over T tiles of 128 features: CTA b <
// full_tiles takes tile b over all tokens; CTA full_tiles + s * rem_tiles + i takes token
// range s (of rem_splits) of tile full_tiles + i.  CTA b writes partial slot b.
struct LoraSchedule {
    int full_tiles, rem_tiles, rem_splits, ctas;
};

// One split sum of the adapter gradients (run by lora_split_sums in ft_sidejobs.cuh):
//   out = s * sum over the tile's slots, in token order, of (D[f][j] + D[f][r + j])
// stored as out[f][j], or out[j][f] with transpose_out.  out == nullptr: no job.
struct LoraFinalizeJob {
    const float* partial;    // [slots][128][NBW]
    int full_tiles, rem_tiles, rem_splits, F, NBW, r;
    float s;
    bool transpose_out;
    float* out;
};

// The two split sums in a launch of their own (lora_split_sums on every thread).
cudaError_t launch_lora_grad_finalize(const LoraFinalizeJob& j0, const LoraFinalizeJob& j1, cudaStream_t stream);

struct GemmFp4Args {
    const uint8_t* sfa;     // tensor-core scale layout of A (rows M, cols K)
    const uint8_t* sfb;     // tensor-core scale layout of B (rows N, cols K)
    const float* ga;        // tensor factor of A
    const float* gb;        // tensor factor of B
    __nv_bfloat16* out;     // [M, ldo]
    int64_t ldo;
    int M, N, K;            // K: reduction length in elements (multiple of 256)
    int KL;                 // low-rank reduction length in bf16 elements (multiple of 16), 0 = none
    int* status;            // device status word
    // optional GELU epilogue: also store act = bf16(gelu_tanh(out)) (same layout as out,
    // through tmAct) and take max |act| into *act_amax (float bits, cleared beforehand)
    __nv_bfloat16* act_out;
    unsigned* act_amax;
    // optional GELU-backward epilogue: store bf16(bf16(out) * gelu_tanh'(gelu_in)) instead
    // of out, gelu_in bf16 with out's layout (the MLP's pre-activation P)
    const __nv_bfloat16* gelu_in;
    // optional side jobs for the epilogue warps, run before their first tile (they wait
    // for the first accumulator anyway): the adapter gradients' split sums
    LoraFinalizeJob side0, side1;
    // non-zero: tmB holds B^T untransposed ([K rows, N/2 bytes], box 256 rows), and the
    // scale warps transpose each tile in shared memory (ft_xpose.cuh); sfb is B's layout
    int xpose;
    // pair kernel: bit 0 set = A's scales from its compact 16x16-block grid through tmSA
    // (uint8 [M/16, K/16], box 16 x 8), bit 1 = B's through tmSB ([N/16, K/16], box 16 x 16);
    // a clear bit = that operand's tensor-core scale layout (sfa / sfb)
    int sfc;
    // pair kernel tile order: 0 = row bands fastest (consecutive tiles share B's panel and
    // sweep all of A), 1 = column tiles fastest (they share A's panel and sweep all of B)
    int n_inner;
};

// tmOut (and tmAct): bf16 [M, N] output, box 32 x 32, 64-byte swizzle.  tmB: 128 x 256
// (bytes x rows) with the 128-byte swizzle; with xpose, 128 bytes x 256 rows of B^T.
cudaError_t launch_gemm_fp4_lowrank(const CUtensorMap& tmA, const CUtensorMap& tmB,
                                    const CUtensorMap& tmLA, const CUtensorMap& tmLB,
                                    const CUtensorMap& tmOut, const CUtensorMap& tmAct,
                                    const GemmFp4Args& args, int num_sms, cudaStream_t stream);

// The same GEMM computed by CTA pairs (cta_group::2), 256 x 256 tiles; needs M % 256 == 0.
// tmB / tmLB boxes are 128 rows: each CTA of a pair loads half of the tile's N (with
// xpose, tmB's box is 64 bytes x 256 rows of B^T, 64-byte swizzle; without, 128 x 128 bytes).
cudaError_t launch_gemm_fp4_lowrank_pair(const CUtensorMap& tmA, const CUtensorMap& tmB,
                                         const CUtensorMap& tmLA, const CUtensorMap& tmLB,
                                         const CUtensorMap& tmOut, const CUtensorMap& tmAct,
                                         const CUtensorMap& tmSA, const CUtensorMap& tmSB,
                                         const GemmFp4Args& args, int num_sms, cudaStream_t stream);

// quantizer and helpers (ft_quant.cu)
// amax_out accumulates with atomicMax: it is cleared here unless slot_cleared (an earlier
// kernel of the same call cleared it).
cudaError_t launch_amax(const void* x, bool is_f32, int64_t rows, int64_t cols, int64_t ld,
                        float* amax_out, bool slot_cleared, int num_sms, cudaStream_t stream);
cudaError_t launch_quant_block16(const void* x, bool is_f32, int64_t rows, int64_t cols, int64_t ld,
                                 const float* amax, uint8_t* codes, uint8_t* scales, float* g_out,
                                 int num_sms, cudaStream_t stream);
cudaError_t launch_expand_scales(const uint8_t* scales, int64_t rows, int64_t cols, uint8_t* sf_mma,
                                 cudaStream_t stream);
cudaError_t launch_transpose_q(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols,
                               uint8_t* codes_t, uint8_t* scales_t, cudaStream_t stream);
cudaError_t launch_copy_scalar(const float* src, float* dst, cudaStream_t stream);
cudaError_t launch_encode_e2m1(const float* v, int64_t n, uint8_t* out, cudaStream_t stream);
cudaError_t launch_encode_ue4m3(const float* v, int64_t n, uint8_t* out, cudaStream_t stream);
cudaError_t launch_gelu_fwd(const __nv_bfloat16* p, __nv_bfloat16* h, int64_t n, cudaStream_t stream);
cudaError_t launch_gelu_bwd(const __nv_bfloat16* p, const __nv_bfloat16* dh, __nv_bfloat16* dp,
                            int64_t n, cudaStream_t stream);

cudaError_t launch_bounded_wait_selftest(uint64_t limit_ns, int* status, cudaStream_t stream);

// Fused quantizer + down-projection (ft_quant_fused.cu).
struct QuantDownArgs {
    int64_t rows, cols;      // input [rows, cols]; rows % 128 == 0, cols % 64 == 0
    int cols_per_split;      // columns per CTA slice (multiple of 64)
    int Rp;                  // down-projection width (multiple of 16, <= 256; 0 = none)
    uint32_t tmem_cols;      // TMEM columns to allocate: quant_down_tmem_cols(Rp)
    const float* amax;       // tensor max used for g
    uint8_t* codes;          // [rows, cols/2]
    uint8_t* scales;         // [rows/16, cols/16]
    uint8_t* sf_mma;         // tensor-core scale layout or null
    float* g_out;
    float* partial;          // [splits, rows, Rp] fp32
    int* status;
    int block_rows;          // 16: 16x16 blocks, scales [rows/16, cols/16]; 1: 1x16 groups, [rows, cols/16]
    // when set, the tensor max is max(amax_parts[0 .. amax_nparts)) instead of *amax
    const float* amax_parts;
    int amax_nparts;
};
int quant_down_splits(int64_t rows, int64_t cols, int num_sms);
uint32_t quant_down_tmem_cols(int Rp);  // room for the kernel's accumulators of Rp columns
size_t quant_down_smem_bytes(int Rp);
cudaError_t launch_quant_down(const CUtensorMap& tmX, const CUtensorMap& tmW, const QuantDownArgs& a,
                              int splits, cudaStream_t stream);

// Sums the split partials in a fixed order and emits out (fp32 [rows, R], may be null)
// and the 4-bit GEMM's low-rank operand cat (bf16 [rows, KL], may be null).
struct LowRankFinalizeArgs {
    const float* partial;    // [splits, rows, Rp]
    int splits;
    int64_t rows;
    int Rp, R, r_s;
    float s;
    const float* ga;
    const float* gb;
    float* out;
    __nv_bfloat16* cat;
    int KL;
    __nv_bfloat16* lora_cat;  // optional [rows, NBW] = [hi, lo, 0] of the LoRA columns (unscaled)
    int NBW;
};
cudaError_t launch_lowrank_finalize(const LowRankFinalizeArgs& a, cudaStream_t stream);

// Side jobs of the first kernel of a layer call (they depend only on the call's inputs):
// V' = [hi(V), lo(V), 0] (bf16 [M, NBW]) of the fp32 columns V = src[:, c0 : c0 + r]
// (row stride ld) for the adapter gradient dB, and clearing the tensor-max slot that the
// call's max kernel accumulates into.
struct PrologueExtras {
    const float* hilo_src = nullptr;
    int hilo_ld = 0, hilo_c0 = 0, hilo_r = 0, hilo_M = 0, hilo_NBW = 0;
    __nv_bfloat16* hilo_dst = nullptr;
    float* zero_slot = nullptr;
    float* zero_slot2 = nullptr;  // a second cleared max slot (the GELU epilogue's)
    // max |x| over a bf16 matrix [max_rows, max_cols] (row stride max_ld): every CTA of
    // the launch writes the max over its share to max_parts[blockIdx.x]
    // (kPrologueCtas entries, no clearing needed); the quantizer reduces them
    const __nv_bfloat16* max_src = nullptr;
    int64_t max_rows = 0, max_cols = 0, max_ld = 0;
    float* max_parts = nullptr;
};
constexpr int kPrologueCtas = 148 * 4;  // the factor kernel's grid
constexpr int kFactorCtas = 148;        // of which build the factors when the kernel also takes a max

// Build the concatenated low-rank factors used by the forward and backward GEMMs (and
// run the side jobs in `extra`, which may be null).  dn and upt get Rp rows (rows
// R..Rp-1 zero) so they can feed an MMA of width Rp.
cudaError_t launch_build_factors(const __nv_bfloat16* ls_down, const __nv_bfloat16* lora_a,
                                 const __nv_bfloat16* ls_up, const __nv_bfloat16* lora_b, int64_t N,
                                 int64_t K, int r_s, int r, int Rp, int KL, __nv_bfloat16* dn,
                                 __nv_bfloat16* upcat, __nv_bfloat16* upt, __nv_bfloat16* dntcat,
                                 const PrologueExtras* extra, cudaStream_t stream);

// adapter gradients on the tensor cores (ft_lora_grad.cu):
//   partial[split][f][c] = sum over the split's tokens m of P[m, f] V'[m, c]
struct LoraGradArgs {
    int64_t F;               // features of P [M, F] (multiple of 128)
    int chunks;              // 64-token chunks of P (M / 64)
    int full_tiles, rem_tiles, rem_splits;  // the CTA schedule (LoraSchedule)
    int NBW;                 // width of V' = [hi, lo, 0] (multiple of 64, <= 256)
    uint32_t tmem_cols;      // power of two >= max(32, NBW)
    float* partial;          // [ctas][128][NBW], slot b = CTA b
    int* status;
    // optional: max |P| over every element of P (each is read by exactly one CTA),
    // accumulated with atomicMax on the float's bits into a slot cleared beforehand
    unsigned* amax_out;
};
LoraSchedule lora_grad_schedule(int64_t M, int64_t F, int num_sms);
cudaError_t launch_lora_grad(const CUtensorMap& tmP, const CUtensorMap& tmV, const LoraGradArgs& a, int kind,
                             cudaStream_t stream);

}  // namespace ft
