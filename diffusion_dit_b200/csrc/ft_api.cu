// C ABI of the W4A4G4 triple-branch linear (declared in include/fourtune.h).
// Host side only: argument checks, workspace carving, TMA descriptors, launch order.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <atomic>
#include <mutex>

#include "fourtune.h"
#include "ft_internal.h"

namespace {

using ft::GemmFp4Args;

constexpr size_t kAlign = 256;

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct DeviceInfo {
    int device = -1;
    int num_sms = 0;
    int cc_major = 0;
};

ft_status device_info(DeviceInfo* out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FT_ERR_CUDA;
    static std::mutex mu;
    static DeviceInfo cache[64];
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64) return FT_ERR_CUDA;
    if (cache[dev].device != dev) {
        DeviceInfo d;
        d.device = dev;
        if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return FT_ERR_CUDA;
        if (cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
            return FT_ERR_CUDA;
        cache[dev] = d;
    }
    *out = cache[dev];
    if (out->cc_major != 10) return FT_ERR_UNSUPPORTED;
    return FT_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D row-major tensor map (128-byte swizzle unless told otherwise).
ft_status make_tmap(CUtensorMap* map, const void* base, CUtensorMapDataType dt, uint64_t inner_elems,
                    uint64_t rows, uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows,
                    CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
    auto fn = encode_fn();
    if (!fn) return FT_ERR_CUDA;
    cuuint64_t dims[2] = {inner_elems, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FT_OK : FT_ERR_CUDA;
}

ft_status cuda_status(cudaError_t e) { return e == cudaSuccess ? FT_OK : FT_ERR_CUDA; }

#define FT_TRY(expr)                          \
    do {                                      \
        ft_status _s = (expr);                \
        if (_s != FT_OK) return _s;           \
    } while (0)
#define FT_CUDA(expr) FT_TRY(cuda_status(expr))

// Width of the GEMMs' low-rank operands [hi, lo]: 2R rounded up to the bf16 MMA's K step.
int low_rank_width(int R) { return R == 0 ? 0 : static_cast<int>(align_up(2 * static_cast<size_t>(R), 16)); }

// Width of the tensor-core down-projection: the rank rounded up to the MMA's N step.
int padded_rank(int R) { return R == 0 ? 0 : static_cast<int>(align_up(static_cast<size_t>(R), 16)); }

uint32_t tmem_cols_for(int Rp) {
    uint32_t c = 32;
    while (c < static_cast<uint32_t>(Rp)) c <<= 1;
    return c;
}

// Upper bound of the column / token slices the fused quantizer and the adapter-gradient
// kernels use: one CTA per SM at most (the heuristics see at most kMaxSms SMs), and
// never more than 16 slices.
constexpr int kMaxSplits = 16;
constexpr int kMaxSms = 160;

size_t max_splits(int64_t units) {
    int64_t s = units > 0 ? kMaxSms / units : kMaxSplits;
    if (s < 1) s = 1;
    if (s > kMaxSplits) s = kMaxSplits;
    return static_cast<size_t>(s);
}

// Workspace of the layer calls.  Regions are 256-byte aligned.
struct LinearWs {
    size_t status, scal, amax_parts, qx_codes, qx_scales, qx_sf, dn, upcat, tcat, partial;
    size_t qg_codes, qg_scales, qg_sf, upt, dntcat, ucat, vcat, ucat_lora, gpartial_b, gpartial_a, total;
};

// Width of the adapter-gradient operand [hi, lo, 0]: 2r rounded up to 64.
int lora_width(int r) { return r == 0 ? 0 : static_cast<int>(align_up(2 * static_cast<size_t>(r), 64)); }

LinearWs linear_ws(int64_t M, int64_t N, int64_t K, int R, int r) {
    const int KL = low_rank_width(R);
    const int Rp = padded_rank(R);
    LinearWs w{};
    size_t o = 0;
    auto take = [&](size_t bytes) {
        size_t at = o;
        o = align_up(o + bytes, kAlign);
        return at;
    };
    w.status = take(16);
    w.scal = take(16 * sizeof(float));
    w.amax_parts = take(ft::kPrologueCtas * sizeof(float));
    w.qx_codes = take(static_cast<size_t>(M) * K / 2);
    w.qx_scales = take(static_cast<size_t>(M) * K / 16);  // 16x16 blocks use 1/16 of it, 1x16 groups all
    w.qx_sf = take(static_cast<size_t>(M) * K / 16);
    w.dn = take(static_cast<size_t>(Rp) * K * 2);
    w.upcat = take(static_cast<size_t>(N) * KL * 2);
    w.tcat = take(static_cast<size_t>(M) * KL * 2);
    w.partial = take(std::max(max_splits(M / 128), static_cast<size_t>(1)) * M * Rp * 4);
    w.qg_codes = take(static_cast<size_t>(M) * N / 2);
    w.qg_scales = take(static_cast<size_t>(M) * N / 256);
    w.qg_sf = take(static_cast<size_t>(M) * N / 16);
    w.upt = take(static_cast<size_t>(Rp) * N * 2);
    w.dntcat = take(static_cast<size_t>(K) * KL * 2);
    w.ucat = take(static_cast<size_t>(M) * KL * 2);
    w.vcat = take(static_cast<size_t>(M) * lora_width(r) * 2);
    w.ucat_lora = take(static_cast<size_t>(M) * lora_width(r) * 2);
    // the adapter gradients' partial slots: one per (CTA, tile it touched), at most
    // kMaxSms + tiles of [128 features][NBW] fp32
    w.gpartial_b = take((kMaxSms + N / 128) * 128 * static_cast<size_t>(lora_width(r)) * 4);  // dB's
    w.gpartial_a = take((kMaxSms + K / 128) * 128 * static_cast<size_t>(lora_width(r)) * 4);  // dA's
    w.total = o;
    return w;
}

// scal[] slots
enum { SC_AMAX_X = 0, SC_G_X = 1, SC_AMAX_G = 2, SC_G_G = 3 };

ft_status check_fp4(const ft_fp4& q, int64_t rows, int64_t cols, bool need_sf) {
    if (!q.codes || !q.scales || !q.g) return FT_ERR_INVALID_ARG;
    if (need_sf && !q.sf_mma) return FT_ERR_INVALID_ARG;
    if (q.rows != rows || q.cols != cols) return FT_ERR_SHAPE;
    if (!aligned16(q.codes) || !aligned16(q.scales) || (q.sf_mma && !aligned16(q.sf_mma)) ||
        (reinterpret_cast<uintptr_t>(q.g) & 3u))
        return FT_ERR_ALIGN;
    return FT_OK;
}

ft_status check_layer(const ft_linear* L) {
    if (!L) return FT_ERR_INVALID_ARG;
    if (L->N <= 0 || L->K <= 0 || L->r_s < 0 || L->r < 0) return FT_ERR_INVALID_ARG;
    if (L->r_s + L->r > 256 || L->r > 64) return FT_ERR_SHAPE;
    if (L->r_s % 8 || L->r % 8) return FT_ERR_SHAPE;  // factor rows move in 16-byte pieces
    if (L->N % 256 || L->K % 256) return FT_ERR_SHAPE;
    FT_TRY(check_fp4(L->qr, L->N, L->K, true));
    if (L->qr_t.codes) {
        FT_TRY(check_fp4(L->qr_t, L->K, L->N, true));
    } else {  // Q(R)^T transposed on the fly from Q(R)'s codes: only its scale layout is kept
        if (!L->qr_t.sf_mma || !L->qr_t.g) return FT_ERR_INVALID_ARG;
        if (L->qr_t.rows != L->K || L->qr_t.cols != L->N) return FT_ERR_SHAPE;
        if (!aligned16(L->qr_t.sf_mma) || (reinterpret_cast<uintptr_t>(L->qr_t.g) & 3u)) return FT_ERR_ALIGN;
    }
    if (L->r_s > 0 && (!L->ls_down || !L->ls_up)) return FT_ERR_INVALID_ARG;
    if (L->r > 0 && (!L->lora_a || !L->lora_b)) return FT_ERR_INVALID_ARG;
    if ((L->ls_down && !aligned16(L->ls_down)) || (L->ls_up && !aligned16(L->ls_up)) ||
        (L->lora_a && !aligned16(L->lora_a)) || (L->lora_b && !aligned16(L->lora_b)))
        return FT_ERR_ALIGN;
    return FT_OK;
}

const __nv_bfloat16* bf(const void* p) { return static_cast<const __nv_bfloat16*>(p); }
__nv_bfloat16* bfm(void* p) { return static_cast<__nv_bfloat16*>(p); }

// Quantize a bf16 [rows, cols] operand into (codes, scales, g, sf_mma) and, when
// Rp > 0, its down-projection partials x w^T (w: bf16 [Rp, cols]) in one fused kernel.
// Returns the number of column slices (partials) through *splits.
ft_status quantize_operand(const void* x, int64_t rows, int64_t cols, int64_t ld, const float* amax_or_null,
                           float* amax_slot, bool amax_slot_cleared, uint8_t* codes, uint8_t* scales, uint8_t* sf, float* g,
                           const void* w, int Rp, float* partial, int* splits, int* status,
                           const DeviceInfo& dev, cudaStream_t st, int block_rows = 16,
                           const float* amax_parts = nullptr) {
    const float* amax = amax_or_null;
    if (!amax && !amax_parts) {
        FT_CUDA(ft::launch_amax(x, false, rows, cols, ld, amax_slot, amax_slot_cleared, dev.num_sms, st));
        amax = amax_slot;
    }
    CUtensorMap tX, tW;
    FT_TRY(make_tmap(&tX, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, cols, rows, ld * 2, 64, 128));
    if (Rp > 0)
        FT_TRY(make_tmap(&tW, w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, cols, Rp, cols * 2, 64, Rp));
    else
        tW = tX;
    const int s = ft::quant_down_splits(rows, cols, dev.num_sms);
    ft::QuantDownArgs a{};
    a.rows = rows;
    a.cols = cols;
    a.cols_per_split = static_cast<int>(cols / s);
    a.Rp = Rp;
    a.tmem_cols = ft::quant_down_tmem_cols(Rp);
    a.amax = amax;
    a.codes = codes;
    a.scales = scales;
    a.sf_mma = sf;
    a.g_out = g;
    a.partial = partial;
    a.status = status;
    a.block_rows = block_rows;
    if (!amax_or_null && amax_parts) {  // the prologue's per-CTA maxima
        a.amax_parts = amax_parts;
        a.amax_nparts = ft::kPrologueCtas;
    }
    FT_CUDA(ft::launch_quant_down(tX, tW, a, s, st));
    *splits = s;
    return FT_OK;
}

// CTA pairs (256 x 256 tiles) when M allows, single CTAs (128 x 256) otherwise.
bool pair_gemm(int64_t M, const DeviceInfo& dev) { return (M % 256) == 0 && dev.num_sms >= 2; }

// One 4-bit GEMM with its low-rank tail: out[M, N] from A (M x K) and B (N x K); with
// act_out, also act_out = bf16(gelu_tanh(out)) and max |act_out| into *act_amax.  When
// b.codes is null, b_src holds B's codes transposed ([K, N/2] bytes: the stored Q(R) for
// the dX GEMM) and the GEMM transposes its tiles in shared memory; b.sf_mma is B's own.
// The pair kernel reads A's and B's scales from their compact 16x16-block grids when it
// has them (a_grid: A's [M/16, K/16] grid, or null for 1x16 groups; B's grid is b.scales
// unless B's codes are transposed on the fly), else from the tensor-core scale layouts
// (a_sf, b.sf_mma), which the one-CTA kernel always uses.
ft_status run_gemm(const uint8_t* a_codes, const uint8_t* a_sf, const uint8_t* a_grid, const float* ga,
                   const ft_fp4& b, const __nv_bfloat16* la, const __nv_bfloat16* lb, int KL, int64_t M,
                   int64_t N, int64_t K, void* out, int* status, const DeviceInfo& dev, cudaStream_t st,
                   void* act_out = nullptr, float* act_amax = nullptr, const void* gelu_in = nullptr,
                   const ft::LoraFinalizeJob* side = nullptr, const uint8_t* b_src = nullptr) {
    const bool pair = pair_gemm(M, dev);
    const uint32_t b_rows = pair ? 128 : 256;
    const bool xpose = b.codes == nullptr;
    if (xpose && (!b_src || act_out)) return FT_ERR_INVALID_ARG;
    const bool grid_a = pair && a_grid != nullptr;
    const bool grid_b = pair && !xpose && b.scales != nullptr;
    if ((!grid_a && !a_sf) || (!grid_b && !b.sf_mma)) return FT_ERR_INVALID_ARG;
    CUtensorMap tA, tB, tLA, tLB, tSA, tSB;
    FT_TRY(make_tmap(&tA, a_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / 2, M, K / 2, 128, 128));
    if (xpose)  // slabs of 256 rows of B^T by this CTA's b_rows columns (b_rows / 2 bytes)
        FT_TRY(make_tmap(&tB, b_src, CU_TENSOR_MAP_DATA_TYPE_UINT8, N / 2, K, N / 2, b_rows / 2, 256,
                         pair ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B));
    else
        FT_TRY(make_tmap(&tB, b.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / 2, N, K / 2, 128, b_rows));
    if (KL > 0) {
        FT_TRY(make_tmap(&tLA, la, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, KL, M, KL * 2, 64, 128));
        FT_TRY(make_tmap(&tLB, lb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, KL, N, KL * 2, 64, b_rows));
    } else {
        tLA = tA;
        tLB = tB;
    }
    // scale grids: uint8 [rows/16, cols/16]; a k step takes 16 block-columns of a CTA's 8
    // block-rows of A and of the pair tile's 16 block-rows of B (no swizzle)
    if (grid_a)
        FT_TRY(make_tmap(&tSA, a_grid, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / 16, M / 16, K / 16, 16, 8,
                         CU_TENSOR_MAP_SWIZZLE_NONE));
    else
        tSA = tA;
    if (grid_b)
        FT_TRY(make_tmap(&tSB, b.scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / 16, N / 16, K / 16, 16, 16,
                         CU_TENSOR_MAP_SWIZZLE_NONE));
    else
        tSB = tB;
    CUtensorMap tOut, tAct;
    FT_TRY(make_tmap(&tOut, out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, M, N * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B));
    if (act_out)
        FT_TRY(make_tmap(&tAct, act_out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, M, N * 2, 32, 32,
                         CU_TENSOR_MAP_SWIZZLE_64B));
    else
        tAct = tOut;
    GemmFp4Args g{};
    g.sfa = a_sf;
    g.sfb = b.sf_mma;
    g.ga = ga;
    g.gb = b.g;
    g.out = bfm(out);
    g.ldo = N;
    g.M = static_cast<int>(M);
    g.N = static_cast<int>(N);
    g.K = static_cast<int>(K);
    g.KL = KL;
    g.status = status;
    g.act_out = bfm(act_out);
    g.act_amax = reinterpret_cast<unsigned*>(act_amax);
    g.gelu_in = bf(gelu_in);
    if (side) {
        g.side0 = side[0];
        g.side1 = side[1];
    }
    g.xpose = xpose ? 1 : 0;
    g.sfc = (grid_a ? 1 : 0) | (grid_b ? 2 : 0);
    // The tiles that run at the same time share one operand's panels and together sweep all
    // of the other's: make the swept operand the smaller one (A is M x K codes, B N x K), so
    // that it stays in L2 between its sweeps instead of coming from HBM again.
    g.n_inner = N < M ? 1 : 0;
    if (pair)
        FT_CUDA(ft::launch_gemm_fp4_lowrank_pair(tA, tB, tLA, tLB, tOut, tAct, tSA, tSB, g, dev.num_sms, st));
    else
        FT_CUDA(ft::launch_gemm_fp4_lowrank(tA, tB, tLA, tLB, tOut, tAct, g, dev.num_sms, st));
    return FT_OK;
}

// Quantize workspace: status word, amax slot, the down factor padded to Rp rows, and
// the split partials of the down-projection.
struct QuantWs {
    size_t status, amax, down, partial, total;
};

QuantWs quant_ws(int64_t rows, int64_t cols, int r_down) {
    const int Rp = padded_rank(r_down);
    QuantWs w{};
    size_t o = 0;
    auto take = [&](size_t bytes) {
        size_t at = o;
        o = align_up(o + bytes, kAlign);
        return at;
    };
    w.status = take(16);
    w.amax = take(16);
    w.down = take(static_cast<size_t>(Rp) * cols * 2);
    w.partial = take(max_splits(rows / 128) * rows * Rp * 4);
    w.total = o;
    return w;
}

std::atomic<uint64_t> g_launches{0};
std::mutex g_ev_mu;
cudaEvent_t g_ev_before[FT_KERNEL_KINDS] = {};
cudaEvent_t g_ev_after[FT_KERNEL_KINDS] = {};

}  // namespace

namespace ft {

// Records a caller's timing event on the launch stream.  Inside a stream capture the
// record becomes an external event node of the graph, which is recorded at every
// replay and can be timed.
static void record_event(cudaEvent_t ev, cudaStream_t stream) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
        cudaEventRecordWithFlags(ev, stream, cudaEventRecordExternal);
    else
        cudaEventRecord(ev, stream);
}

void before_launch(int kind, cudaStream_t stream) {
    if (kind < 0 || kind >= FT_KERNEL_KINDS) return;
    std::lock_guard<std::mutex> lock(g_ev_mu);
    if (g_ev_before[kind]) {
        record_event(g_ev_before[kind], stream);
        g_ev_before[kind] = nullptr;
    }
}

void after_launch(int kind, cudaStream_t stream) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (kind < 0 || kind >= FT_KERNEL_KINDS) return;
    std::lock_guard<std::mutex> lock(g_ev_mu);
    if (g_ev_after[kind]) {
        record_event(g_ev_after[kind], stream);
        g_ev_after[kind] = nullptr;
    }
}

}  // namespace ft

extern "C" {

uint64_t fourtune_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

ft_status fourtune_time_next_launch(int32_t kernel, void* ev_before, void* ev_after) {
    if (kernel < 0 || kernel >= FT_KERNEL_KINDS) return FT_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(g_ev_mu);
    g_ev_before[kernel] = static_cast<cudaEvent_t>(ev_before);
    g_ev_after[kernel] = static_cast<cudaEvent_t>(ev_after);
    return FT_OK;
}

const char* fourtune_status_string(int s) {
    switch (s) {
        case FT_OK: return "ok";
        case FT_ERR_INVALID_ARG: return "invalid argument";
        case FT_ERR_SHAPE: return "unsupported shape";
        case FT_ERR_ALIGN: return "misaligned pointer";
        case FT_ERR_WORKSPACE: return "workspace too small";
        case FT_ERR_CUDA: return "CUDA error";
        case FT_ERR_UNSUPPORTED: return "device is not sm_100";
        case FT_ERR_TIMEOUT: return "device wait timed out";
        default: return "unknown status";
    }
}

size_t fourtune_quantize_workspace_bytes(int64_t rows, int64_t cols, int32_t r_down) {
    if (rows < 0 || cols < 0 || r_down < 0) return 0;
    return quant_ws(rows, cols, r_down).total;
}

ft_status fourtune_quantize_1x16(const void* x_dev, int64_t rows, int64_t cols, int64_t ld,
                                 const float* amax_or_null, const ft_fp4* out, void* ws, size_t ws_bytes,
                                 void* stream) {
    if (!x_dev || !out) return FT_ERR_INVALID_ARG;
    if (rows <= 0 || cols <= 0 || ld < cols) return FT_ERR_INVALID_ARG;
    if (rows % 128 || cols % 64 || ld % 8) return FT_ERR_SHAPE;
    FT_TRY(check_fp4(*out, rows, cols, false));
    if (!aligned16(x_dev)) return FT_ERR_ALIGN;
    const QuantWs qw = quant_ws(rows, cols, 0);
    if (!ws || ws_bytes < qw.total) return FT_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) % kAlign) return FT_ERR_ALIGN;
    DeviceInfo dev;
    FT_TRY(device_info(&dev));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* W = static_cast<uint8_t*>(ws);
    int splits = 1;
    return quantize_operand(x_dev, rows, cols, ld, amax_or_null, reinterpret_cast<float*>(W + qw.amax), false,
                            out->codes, out->scales, out->sf_mma, out->g, nullptr, 0,
                            reinterpret_cast<float*>(W + qw.partial), &splits,
                            reinterpret_cast<int*>(W + qw.status), dev, st, 1);
}

ft_status fourtune_quantize_block16(const void* x_dev, int32_t x_dtype, int64_t rows, int64_t cols,
                                    int64_t ld, const float* amax_or_null, const void* down_dev,
                                    int32_t r_down, float* down_out_dev, const ft_fp4* out,
                                    const ft_fp4* out_t, void* ws, size_t ws_bytes, void* stream) {
    if (!x_dev || !out || (x_dtype != FT_DTYPE_BF16 && x_dtype != FT_DTYPE_F32)) return FT_ERR_INVALID_ARG;
    if (rows <= 0 || cols <= 0 || ld < cols || r_down < 0 || r_down > 256) return FT_ERR_INVALID_ARG;
    if (rows % 16 || cols % 16 || ld % 8) return FT_ERR_SHAPE;
    if (r_down > 0 && (!down_dev || !down_out_dev || x_dtype != FT_DTYPE_BF16)) return FT_ERR_INVALID_ARG;
    FT_TRY(check_fp4(*out, rows, cols, false));
    const bool want_sf = out->sf_mma != nullptr;
    const bool fused_ok = x_dtype == FT_DTYPE_BF16 && rows % 128 == 0 && cols % 64 == 0;
    if (r_down > 0 && !fused_ok) return FT_ERR_SHAPE;
    if ((want_sf || out_t) && (rows % 128 || cols % 128)) return FT_ERR_SHAPE;
    if (out_t) FT_TRY(check_fp4(*out_t, cols, rows, true));
    if (!aligned16(x_dev) || (down_dev && !aligned16(down_dev)) || (down_out_dev && !aligned16(down_out_dev)))
        return FT_ERR_ALIGN;
    const QuantWs qw = quant_ws(rows, cols, r_down);
    if (!ws || ws_bytes < qw.total) return FT_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) % kAlign) return FT_ERR_ALIGN;
    DeviceInfo dev;
    FT_TRY(device_info(&dev));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* W = static_cast<uint8_t*>(ws);
    float* amax_slot = reinterpret_cast<float*>(W + qw.amax);
    int* status = reinterpret_cast<int*>(W + qw.status);
    const bool f32 = x_dtype == FT_DTYPE_F32;
    if (fused_ok) {
        const int Rp = padded_rank(r_down);
        ft::PrologueExtras ex;
        if (!amax_or_null) ex.zero_slot = amax_slot;
        if (Rp > 0)
            FT_CUDA(ft::launch_build_factors(bf(down_dev), nullptr, nullptr, nullptr, 0, cols, r_down, 0, Rp, 0,
                                             bfm(W + qw.down), nullptr, nullptr, nullptr, &ex, st));
        int splits = 1;
        float* partial = reinterpret_cast<float*>(W + qw.partial);
        FT_TRY(quantize_operand(x_dev, rows, cols, ld, amax_or_null, amax_slot, Rp > 0, out->codes, out->scales,
                                out->sf_mma, out->g, W + qw.down, Rp, partial, &splits, status, dev, st));
        if (Rp > 0) {
            ft::LowRankFinalizeArgs f{};
            f.partial = partial;
            f.splits = splits;
            f.rows = rows;
            f.Rp = Rp;
            f.R = r_down;
            f.r_s = r_down;
            f.s = 1.0f;
            f.out = down_out_dev;
            FT_CUDA(ft::launch_lowrank_finalize(f, st));
        }
    } else {
        const float* amax = amax_or_null;
        if (!amax) {
            FT_CUDA(ft::launch_amax(x_dev, f32, rows, cols, ld, amax_slot, false, dev.num_sms, st));
            amax = amax_slot;
        }
        FT_CUDA(ft::launch_quant_block16(x_dev, f32, rows, cols, ld, amax, out->codes, out->scales, out->g,
                                         dev.num_sms, st));
        if (want_sf) FT_CUDA(ft::launch_expand_scales(out->scales, rows, cols, out->sf_mma, st));
    }
    if (out_t) {
        FT_CUDA(ft::launch_transpose_q(out->codes, out->scales, rows, cols, out_t->codes, out_t->scales, st));
        FT_CUDA(ft::launch_copy_scalar(out->g, out_t->g, st));
        FT_CUDA(ft::launch_expand_scales(out_t->scales, cols, rows, out_t->sf_mma, st));
    }
    return FT_OK;
}

size_t fourtune_linear_workspace_bytes(const ft_linear* L, int64_t M) {
    if (!L || M <= 0) return 0;
    return linear_ws(M, L->N, L->K, L->r_s + L->r, L->r).total;
}

namespace {

// The forward of fourtune_linear_fwd; with h_dev also the GELU epilogue (h = bf16(gelu(y)),
// max |h| into *h_amax_dev).
ft_status linear_fwd_impl(const ft_linear* L, const void* x_dev, int64_t M, const float* amax_or_null,
                          void* y_dev, float* t_saved_dev, void* h_dev, float* h_amax_dev, void* ws,
                          size_t ws_bytes, void* stream, int x_block_rows = 16) {
    FT_TRY(check_layer(L));
    const int R = L->r_s + L->r;
    if (!x_dev || !y_dev || (R > 0 && !t_saved_dev) || M <= 0) return FT_ERR_INVALID_ARG;
    if (M % 128) return FT_ERR_SHAPE;
    if (!aligned16(x_dev) || !aligned16(y_dev) || (t_saved_dev && !aligned16(t_saved_dev))) return FT_ERR_ALIGN;
    const LinearWs w = linear_ws(M, L->N, L->K, R, L->r);
    if (!ws || ws_bytes < w.total) return FT_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) % kAlign) return FT_ERR_ALIGN;
    DeviceInfo dev;
    FT_TRY(device_info(&dev));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* W = static_cast<uint8_t*>(ws);
    float* scal = reinterpret_cast<float*>(W + w.scal);
    int* status = reinterpret_cast<int*>(W + w.status);
    const int64_t N = L->N, K = L->K;
    const int KL = low_rank_width(R);
    const int Rp = padded_rank(R);
    float* partial = reinterpret_cast<float*>(W + w.partial);

    // Eq. (2): the factors of this step ([Ls_down; A] and [Ls_up, B]; A, B train) and
    // max |X| in one prologue launch, then Q(X) fused with T = X [Ls_down; A]^T, then
    // the 4-bit GEMM with the up-projections in its accumulator.  The prologue leaves
    // one max per CTA, which the quantizer reduces (no cleared slot, no separate pass);
    // it also clears the GELU epilogue's max slot.
    ft::PrologueExtras ex;
    float* amax_parts = nullptr;
    if (!amax_or_null) {
        amax_parts = reinterpret_cast<float*>(W + w.amax_parts);
        ex.max_src = bf(x_dev);
        ex.max_rows = M;
        ex.max_cols = K;
        ex.max_ld = K;
        ex.max_parts = amax_parts;
    }
    if (h_dev) ex.zero_slot2 = h_amax_dev;
    if (R > 0 || amax_parts || h_dev)
        FT_CUDA(ft::launch_build_factors(bf(L->ls_down), bf(L->lora_a), bf(L->ls_up), bf(L->lora_b), N, K,
                                         L->r_s, L->r, Rp, KL, R > 0 ? bfm(W + w.dn) : nullptr,
                                         R > 0 ? bfm(W + w.upcat) : nullptr, nullptr, nullptr, &ex, st));
    int splits = 1;
    // the pair GEMM reads Q(X)'s compact block grid; 1x16 groups and the one-CTA GEMM need
    // the tensor-core scale layout
    const bool x_grid = pair_gemm(M, dev) && x_block_rows == 16;
    FT_TRY(quantize_operand(x_dev, M, K, K, amax_or_null, scal + SC_AMAX_X, R > 0, W + w.qx_codes, W + w.qx_scales,
                            x_grid ? nullptr : W + w.qx_sf, scal + SC_G_X, W + w.dn, Rp, partial, &splits, status,
                            dev, st, x_block_rows, amax_parts));
    if (R > 0) {
        ft::LowRankFinalizeArgs f{};
        f.partial = partial;
        f.splits = splits;
        f.rows = M;
        f.Rp = Rp;
        f.R = R;
        f.r_s = L->r_s;
        f.s = L->lora_scale;
        f.ga = scal + SC_G_X;
        f.gb = L->qr.g;
        f.out = t_saved_dev;
        f.cat = bfm(W + w.tcat);
        f.KL = KL;
        FT_CUDA(ft::launch_lowrank_finalize(f, st));
    }
    return run_gemm(W + w.qx_codes, x_grid ? nullptr : W + w.qx_sf, x_grid ? W + w.qx_scales : nullptr,
                    scal + SC_G_X, L->qr, bf(W + w.tcat), bf(W + w.upcat), KL, M, N, K, y_dev, status, dev, st,
                    h_dev, h_amax_dev);
}

}  // namespace

ft_status fourtune_linear_fwd(const ft_linear* L, const void* x_dev, int64_t M, const float* amax_or_null,
                              void* y_dev, float* t_saved_dev, void* ws, size_t ws_bytes, void* stream) {
    return linear_fwd_impl(L, x_dev, M, amax_or_null, y_dev, t_saved_dev, nullptr, nullptr, ws, ws_bytes, stream);
}

ft_status fourtune_linear_fwd_1x16(const ft_linear* L, const void* x_dev, int64_t M, const float* amax_or_null,
                                   void* y_dev, float* t_saved_dev, void* ws, size_t ws_bytes, void* stream) {
    return linear_fwd_impl(L, x_dev, M, amax_or_null, y_dev, t_saved_dev, nullptr, nullptr, ws, ws_bytes, stream,
                           1);
}

ft_status fourtune_linear_fwd_gelu(const ft_linear* L, const void* x_dev, int64_t M, const float* amax_or_null,
                                   void* p_dev, void* h_dev, float* h_amax_dev, float* t_saved_dev, void* ws,
                                   size_t ws_bytes, void* stream) {
    if (!h_dev || !h_amax_dev) return FT_ERR_INVALID_ARG;
    if (!aligned16(h_dev) || (reinterpret_cast<uintptr_t>(h_amax_dev) & 3u)) return FT_ERR_ALIGN;
    return linear_fwd_impl(L, x_dev, M, amax_or_null, p_dev, t_saved_dev, h_dev, h_amax_dev, ws, ws_bytes,
                           stream);
}

namespace {

// An upper bound on the slot loads one thread of `workers` makes in lora_split_sums over
// the two jobs: thread w takes blocks w, w + workers, ... (job 0's blocks first, then job
// 1's); a block of tile t adds rem_splits slots when t is a split tile, else one.  Each
// round of `workers` blocks counts the most slots any of its blocks adds.
double split_sum_rounds(const ft::LoraFinalizeJob& j0, const ft::LoraFinalizeJob& j1, int64_t workers) {
    const ft::LoraFinalizeJob* jobs[2] = {&j0, &j1};
    int64_t n[2];
    for (int k = 0; k < 2; ++k)
        n[k] = jobs[k]->out ? static_cast<int64_t>(jobs[k]->F / 4) * (jobs[k]->r / 4) : 0;
    const int64_t total = n[0] + n[1];
    double rounds = 0.0;
    for (int64_t lo = 0; lo < total; lo += workers) {
        const int64_t hi = std::min(total, lo + workers);  // this round's blocks [lo, hi)
        int most = 0;
        for (int k = 0, off = 0; k < 2; off += static_cast<int>(n[k]), ++k) {
            const int64_t a = std::max<int64_t>(lo, off) - off, b = std::min<int64_t>(hi, off + n[k]) - off;
            if (a >= b) continue;
            const ft::LoraFinalizeJob& j = *jobs[k];
            int slots = 1;
            if (j.rem_tiles > 0) {
                if (j.transpose_out) {
                    slots = j.rem_splits;  // blocks walk f fastest: every round meets a split tile
                } else {
                    const int64_t per_tile = 32 * static_cast<int64_t>(j.r / 4);  // blocks of one tile
                    if ((b - 1) / per_tile >= j.full_tiles) slots = j.rem_splits;
                }
            }
            most = std::max(most, slots);
        }
        rounds += most;
    }
    return rounds;
}

// The backward of fourtune_linear_bwd; with gelu_in, dx_dev receives bf16(dX * gelu'(gelu_in)).
ft_status linear_bwd_impl(const ft_linear* L, const void* x_dev, const float* t_saved_dev, const void* dy_dev,
                          int64_t M, const float* amax_or_null, void* dx_dev, float* da_dev, float* db_dev,
                          const void* gelu_in, void* ws, size_t ws_bytes, void* stream) {
    FT_TRY(check_layer(L));
    const int R = L->r_s + L->r;
    if (!x_dev || !dy_dev || !dx_dev || M <= 0) return FT_ERR_INVALID_ARG;
    if (L->r > 0 && (!t_saved_dev || !da_dev || !db_dev)) return FT_ERR_INVALID_ARG;
    if (M % 128) return FT_ERR_SHAPE;
    if (!aligned16(x_dev) || !aligned16(dy_dev) || !aligned16(dx_dev) ||
        (t_saved_dev && !aligned16(t_saved_dev)) || (da_dev && !aligned16(da_dev)) ||
        (db_dev && !aligned16(db_dev)))
        return FT_ERR_ALIGN;
    const LinearWs w = linear_ws(M, L->N, L->K, R, L->r);
    if (!ws || ws_bytes < w.total) return FT_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) % kAlign) return FT_ERR_ALIGN;
    DeviceInfo dev;
    FT_TRY(device_info(&dev));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t* W = static_cast<uint8_t*>(ws);
    float* scal = reinterpret_cast<float*>(W + w.scal);
    int* status = reinterpret_cast<int*>(W + w.status);
    const int64_t N = L->N, K = L->K;
    const int KL = low_rank_width(R);
    const int Rp = padded_rank(R);
    float* partial = reinterpret_cast<float*>(W + w.partial);

    // Eq. (3): dB (with max |G|), Q(G) fused with U = G [Ls_up, B], dA, then the dX GEMM
    // through Q(R)^T with U [Ls_down; A] in its accumulator.
    // The factor kernel also builds dB's operand V' = [hi, lo, 0] of T_lora (an input of
    // this call) and clears the tensor-max slot.
    ft::PrologueExtras ex;
    if (!amax_or_null) ex.zero_slot = scal + SC_AMAX_G;
    if (L->r > 0) {
        ex.hilo_src = t_saved_dev;
        ex.hilo_ld = R;
        ex.hilo_c0 = L->r_s;
        ex.hilo_r = L->r;
        ex.hilo_M = static_cast<int>(M);
        ex.hilo_NBW = lora_width(L->r);
        ex.hilo_dst = bfm(W + w.vcat);
    }
    if (R > 0)
        FT_CUDA(ft::launch_build_factors(bf(L->ls_down), bf(L->lora_a), bf(L->ls_up), bf(L->lora_b), N, K,
                                         L->r_s, L->r, Rp, KL, nullptr, nullptr, bfm(W + w.upt),
                                         bfm(W + w.dntcat), &ex, st));
    // Section 3.2 adapter gradients: dB = s G^T T_lora, dA = s U_lora^T X, on the tensor
    // cores, reading G and X straight (MN-major operands).  dB goes first: its kernel
    // reads every element of G once and also takes max |G| (into the slot the factor
    // kernel cleared), so Q(G) needs no separate pass over G; G is then still in L2.
    const int NBW = lora_width(L->r);
    ft::LoraGradArgs g{};
    g.NBW = NBW;
    g.tmem_cols = tmem_cols_for(NBW);
    g.status = status;
    const float* amax_g = amax_or_null;
    // dB's and dA's split sums run on the dX GEMM's epilogue warps, before its first tile
    ft::LoraFinalizeJob fin[2] = {};
    if (L->r > 0) {
        CUtensorMap tP, tV;
        FT_TRY(make_tmap(&tV, W + w.vcat, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, NBW, M, NBW * 2, 64, 64));
        FT_TRY(make_tmap(&tP, dy_dev, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, M, N * 2, 64, 64));
        const ft::LoraSchedule sc = ft::lora_grad_schedule(M, N, dev.num_sms);
        g.F = N;
        g.chunks = static_cast<int>(M / 64);
        g.full_tiles = sc.full_tiles;
        g.rem_tiles = sc.rem_tiles;
        g.rem_splits = sc.rem_splits;
        g.partial = reinterpret_cast<float*>(W + w.gpartial_b);
        if (!amax_or_null) {
            g.amax_out = reinterpret_cast<unsigned*>(scal + SC_AMAX_G);
            amax_g = scal + SC_AMAX_G;
        }
        FT_CUDA(ft::launch_lora_grad(tP, tV, g, ft::K_LORA_DB, st));
        g.amax_out = nullptr;
        fin[1] = ft::LoraFinalizeJob{g.partial, sc.full_tiles, sc.rem_tiles, sc.rem_splits, static_cast<int>(N), NBW,
                                     L->r, L->lora_scale, false, db_dev};
    }
    int splits = 1;
    const bool g_grid = pair_gemm(M, dev);  // the pair GEMM reads Q(G)'s compact block grid
    FT_TRY(quantize_operand(dy_dev, M, N, N, amax_g, scal + SC_AMAX_G, R > 0, W + w.qg_codes, W + w.qg_scales,
                            g_grid ? nullptr : W + w.qg_sf, scal + SC_G_G, W + w.upt, Rp, partial, &splits, status,
                            dev, st));
    if (R > 0) {
        ft::LowRankFinalizeArgs f{};
        f.partial = partial;
        f.splits = splits;
        f.rows = M;
        f.Rp = Rp;
        f.R = R;
        f.r_s = L->r_s;
        f.s = L->lora_scale;
        f.ga = scal + SC_G_G;
        f.gb = L->qr_t.g;
        f.out = nullptr;  // U itself is not needed: only its GEMM and dA operands
        f.cat = bfm(W + w.ucat);
        f.KL = KL;
        if (L->r > 0) {  // U_lora's hi/lo operand for dA, written by the same pass
            f.lora_cat = bfm(W + w.ucat_lora);
            f.NBW = NBW;
        }
        FT_CUDA(ft::launch_lowrank_finalize(f, st));
    }
    if (L->r > 0) {
        // dA over the input features k (V' = U_lora's hi/lo, written by the split sum)
        CUtensorMap tP, tV;
        FT_TRY(make_tmap(&tV, W + w.ucat_lora, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, NBW, M, NBW * 2, 64, 64));
        FT_TRY(make_tmap(&tP, x_dev, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, M, K * 2, 64, 64));
        const ft::LoraSchedule sc = ft::lora_grad_schedule(M, K, dev.num_sms);
        g.F = K;
        g.chunks = static_cast<int>(M / 64);
        g.full_tiles = sc.full_tiles;
        g.rem_tiles = sc.rem_tiles;
        g.rem_splits = sc.rem_splits;
        g.partial = reinterpret_cast<float*>(W + w.gpartial_a);
        FT_CUDA(ft::launch_lora_grad(tP, tV, g, ft::K_LORA_DA, st));
        fin[0] = ft::LoraFinalizeJob{g.partial, sc.full_tiles, sc.rem_tiles, sc.rem_splits, static_cast<int>(K), NBW,
                                     L->r, L->lora_scale, true, da_dev};
    }
    // dA's and dB's split sums: on the dX GEMM's epilogue warps when they fit in the time
    // those warps wait for their first accumulator (a k step of 256 takes ~0.42 us; a
    // thread's block of 4 x 4 outputs costs ~0.6 us per slot it adds: one round trip for
    // the slot's eight loads), else in a launch of their own before the GEMM.  Measured on
    // the FLUX single-stream linear2 (15 k steps in the first tile, ~5.4 us of sums): the
    // side path saves the launch and costs the GEMM ~3 us.
    bool side = false;
    if (L->r > 0) {
        // the dX GEMM's epilogue threads (32 per epilogue warp: 4 per CTA, 8 with the
        // GELU-backward epilogue; 148 CTAs, or fewer for a small grid)
        const bool pair = pair_gemm(M, dev);
        const int64_t gemm_ctas = pair ? 2 * std::min<int64_t>(dev.num_sms / 2, (M / 256) * (K / 256))
                                       : std::min<int64_t>(dev.num_sms, (M / 128) * (K / 256));
        const int64_t workers = gemm_ctas * 32 * (pair && gelu_in ? 8 : 4);
        const double cost_us = split_sum_rounds(fin[0], fin[1], workers) * 0.6;
        const double first_tile_us = (static_cast<double>(N) / 256.0 + (KL + 63) / 64) * 0.42;
        side = cost_us <= first_tile_us;
        if (!side) FT_CUDA(ft::launch_lora_grad_finalize(fin[0], fin[1], st));
    }
    // The dX GEMM goes last: the GEMM's operand and output traffic would evict G from L2.
    FT_TRY(run_gemm(W + w.qg_codes, g_grid ? nullptr : W + w.qg_sf, g_grid ? W + w.qg_scales : nullptr,
                    scal + SC_G_G, L->qr_t, bf(W + w.ucat), bf(W + w.dntcat), KL, M, K, N, dx_dev, status, dev, st,
                    nullptr, nullptr, gelu_in, side ? fin : nullptr, L->qr.codes));
    return FT_OK;
}

}  // namespace

ft_status fourtune_linear_bwd(const ft_linear* L, const void* x_dev, const float* t_saved_dev,
                              const void* dy_dev, int64_t M, const float* amax_or_null, void* dx_dev,
                              float* da_dev, float* db_dev, void* ws, size_t ws_bytes, void* stream) {
    return linear_bwd_impl(L, x_dev, t_saved_dev, dy_dev, M, amax_or_null, dx_dev, da_dev, db_dev, nullptr, ws,
                           ws_bytes, stream);
}

ft_status fourtune_linear_bwd_gelu(const ft_linear* L, const void* x_dev, const float* t_saved_dev,
                                   const void* dy_dev, int64_t M, const float* amax_or_null, const void* p_dev,
                                   void* dp_dev, float* da_dev, float* db_dev, void* ws, size_t ws_bytes,
                                   void* stream) {
    if (!p_dev) return FT_ERR_INVALID_ARG;
    if (!aligned16(p_dev)) return FT_ERR_ALIGN;
    return linear_bwd_impl(L, x_dev, t_saved_dev, dy_dev, M, amax_or_null, dp_dev, da_dev, db_dev, p_dev, ws,
                           ws_bytes, stream);
}

ft_status fourtune_selftest_bounded_wait(int64_t limit_ns, void* ws, void* stream) {
    if (!ws || limit_ns <= 0 || limit_ns > 1000000000LL) return FT_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(ws) % kAlign) return FT_ERR_ALIGN;
    DeviceInfo dev;
    FT_TRY(device_info(&dev));
    FT_CUDA(ft::launch_bounded_wait_selftest(static_cast<uint64_t>(limit_ns), static_cast<int*>(ws),
                                             static_cast<cudaStream_t>(stream)));
    return FT_OK;
}

ft_status fourtune_device_status(void* ws, int32_t* status_out, void* stream) {
    if (!status_out) return FT_ERR_INVALID_ARG;
    if (!ws) FT_TRY(ft::noalloc_scratch(&ws));  // the status of fourtune_quantize_block16_noalloc
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t v = 0;
    FT_CUDA(cudaMemcpyAsync(&v, ws, sizeof(int32_t), cudaMemcpyDeviceToHost, st));
    FT_CUDA(cudaStreamSynchronize(st));
    FT_CUDA(cudaMemsetAsync(ws, 0, sizeof(int32_t), st));
    *status_out = v;
    return FT_OK;
}

ft_status fourtune_gelu_tanh_fwd(const void* p_dev, void* h_dev, int64_t n, void* stream) {
    if (!p_dev || !h_dev || n < 0) return FT_ERR_INVALID_ARG;
    if (n % 8) return FT_ERR_SHAPE;
    if (!aligned16(p_dev) || !aligned16(h_dev)) return FT_ERR_ALIGN;
    if (n == 0) return FT_OK;
    DeviceInfo dev;
    FT_TRY(device_info(&dev));
    FT_CUDA(ft::launch_gelu_fwd(bf(p_dev), bfm(h_dev), n, static_cast<cudaStream_t>(stream)));
    return FT_OK;
}

ft_status fourtune_gelu_tanh_bwd(const void* p_dev, const void* dh_dev, void* dp_dev, int64_t n, void* stream) {
    if (!p_dev || !dh_dev || !dp_dev || n < 0) return FT_ERR_INVALID_ARG;
    if (n % 8) return FT_ERR_SHAPE;
    if (!aligned16(p_dev) || !aligned16(dh_dev) || !aligned16(dp_dev)) return FT_ERR_ALIGN;
    if (n == 0) return FT_OK;
    DeviceInfo dev;
    FT_TRY(device_info(&dev));
    FT_CUDA(ft::launch_gelu_bwd(bf(p_dev), bf(dh_dev), bfm(dp_dev), n, static_cast<cudaStream_t>(stream)));
    return FT_OK;
}

ft_status fourtune_encode_e2m1(const float* v_dev, int64_t n, uint8_t* out_dev, void* stream) {
    if (!v_dev || !out_dev || n < 0) return FT_ERR_INVALID_ARG;
    if (n == 0) return FT_OK;
    DeviceInfo dev;
    FT_TRY(device_info(&dev));
    FT_CUDA(ft::launch_encode_e2m1(v_dev, n, out_dev, static_cast<cudaStream_t>(stream)));
    return FT_OK;
}

ft_status fourtune_encode_ue4m3(const float* v_dev, int64_t n, uint8_t* out_dev, void* stream) {
    if (!v_dev || !out_dev || n < 0) return FT_ERR_INVALID_ARG;
    if (n == 0) return FT_OK;
    DeviceInfo dev;
    FT_TRY(device_info(&dev));
    FT_CUDA(ft::launch_encode_ue4m3(v_dev, n, out_dev, static_cast<cudaStream_t>(stream)));
    return FT_OK;
}

}  // extern "C"
