// hstu_api.cu -- host side of libhstu's C ABI (declared in include/hstu.h):
// argument validation, TMA tensor-map encoding, workspace carving and kernel
// launches. Every device kernel of the library is compiled in this one
// translation unit so they share the per-device error word.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "hstu.h"
#include "attn_bwd_simt.cuh"
#include "attn_bwd_tc.cuh"
#include "attn_simt.cuh"
#include "attn_tc.cuh"
#include "bias_prep.cuh"
#include "common.cuh"
#include "debug.cuh"
#include "gemm_tc.cuh"
#include "ln_gate.cuh"
#include "plan.cuh"
#include "quant_fp8.cuh"

using namespace hstu;

namespace {

constexpr int kMaxDevices = 64;

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// cuTensorMapEncodeTiled through the runtime's driver entry point, so the
// library does not link libcuda directly.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D bf16 tensor map over a row-major [rows, inner] view with the given row
// stride (bytes); 64 x 128 boxes with the 128-byte swizzle the UMMA
// descriptors expect.
bool make_tmap_bf16_box(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t rows,
                        uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows,
                        CUtensorMapSwizzle swizzle) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {row_stride_bytes};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// fp32 [rows, inner] with boxes of 16 x 32 (64-byte rows, 64-byte swizzle).
bool make_tmap_f32_16x32(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t rows,
                         uint64_t row_stride_bytes) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {row_stride_bytes};
    cuuint32_t box[2] = {16, 32};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Boxes of 128 E4M3 codes (128 bytes, 128-byte swizzle) x box_rows.
bool make_tmap_u8(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t rows,
                  uint64_t row_stride_bytes, uint32_t box_rows) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {row_stride_bytes};
    cuuint32_t box[2] = {128, box_rows};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Boxes of 64 columns (128 bytes, 128-byte swizzle) x box_rows: MMA operands.
bool make_tmap_bf16(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t rows,
                    uint64_t row_stride_bytes, uint32_t box_rows) {
    return make_tmap_bf16_box(tm, base, inner, rows, row_stride_bytes, 64, box_rows,
                              CU_TENSOR_MAP_SWIZZLE_128B);
}

// Raise a kernel's dynamic shared-memory limit once per device.
template <typename K>
bool ensure_smem(K kernel, int bytes, int* done_flags) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
    if (!done_flags[dev]) {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
            cudaSuccess)
            return false;
        done_flags[dev] = 1;
    }
    return true;
}

hstu_status_t launch_status() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

int max_tiles_of(int32_t max_seqlen) { return (max_seqlen + kTile - 1) / kTile; }

int64_t max_units_of(int32_t B, int64_t T, int32_t max_seqlen) {
    const int64_t by_tokens = T / kTile + B + 1;   // >= sum_b ceil(n_b / 128)
    const int64_t by_lengths = static_cast<int64_t>(B) * max_tiles_of(max_seqlen);
    return by_tokens < by_lengths ? by_tokens : by_lengths;
}

constexpr size_t kAttnWsHeader = 256;   // unit count (int at 0), item counters (2 ints at 16)

// attention workspace: [header][units: int4 x max_units][starts: uint4 x max_units]
// (the plan's part), then [window tables: H x DD x 3968 B][key summaries:
// 576 B x max_units] (built per run by the bias prep kernel)
size_t attn_units_bytes(int32_t B, int64_t T, int32_t max_seqlen) {
    return (static_cast<size_t>(max_units_of(B, T, max_seqlen)) * 16 + 255) / 256 * 256;
}

size_t attn_plan_bytes(int32_t B, int64_t T, int32_t max_seqlen) {
    return kAttnWsHeader + 2 * attn_units_bytes(B, T, max_seqlen);
}

// window tables of a run: P = num_pos (1 when there is no position term)
int attn_window_tables(int32_t P, int32_t max_seqlen) {
    return window_tables(P > 0 ? P : 1, max_tiles_of(max_seqlen));
}

size_t attn_tables_bytes(int32_t H, int32_t P, int32_t max_seqlen) {
    return static_cast<size_t>(H) * attn_window_tables(P, max_seqlen) * kWinBytes;
}

size_t attn_keys_bytes(int32_t B, int64_t T, int32_t max_seqlen) {
    return static_cast<size_t>(max_units_of(B, T, max_seqlen)) * sizeof(KeySummary);
}

int num_sms() {
    static int cached[kMaxDevices] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

// Grid for a kernel whose blocks stride over `blocks` units of work: at most
// as many blocks as fit on the device at once, so none waits for a second
// wave. `cache` holds the per-device count of resident blocks per SM.
template <typename K>
unsigned resident_grid(K kernel, int threads, int64_t blocks, int* cache) {
    int dev = 0;
    int per_sm = 1;
    if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < kMaxDevices) {
        if (cache[dev] == 0) {
            int n = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, 0) !=
                    cudaSuccess || n < 1)
                n = 1;
            cache[dev] = n;
        }
        per_sm = cache[dev];
    }
    const int64_t cap = static_cast<int64_t>(num_sms()) * per_sm;
    return static_cast<unsigned>(blocks < cap ? blocks : cap);
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool plan_sizes_ok(int32_t B, int64_t T, int32_t max_seqlen) {
    return B >= 0 && T >= 0 && T <= (int64_t{1} << 31) - 1 - 2 * kTile && max_seqlen >= 1 &&
           max_seqlen <= kMaxSeqlen;
}

struct AttnCall {
    hstu_dtype_t dtype;
    const void *q, *k, *v;
    int64_t qs, ks, vs;
    const int64_t* off;
    int32_t B;
    int64_t T;
    int32_t H, dqk, dv;
    const int64_t* ts;
    const float* pos;
    int32_t P;
    const float* tb;
    int32_t NB;
    int32_t max_seqlen;
    void* out;
    int64_t os;
    void* ws;
    size_t ws_bytes;
    cudaStream_t stream;
};

hstu_status_t validate_attn(const AttnCall& c) {
    if (c.dtype != HSTU_DTYPE_F32 && c.dtype != HSTU_DTYPE_BF16) return HSTU_ERR_INVALID_ARG;
    if (!plan_sizes_ok(c.B, c.T, c.max_seqlen)) return HSTU_ERR_INVALID_ARG;
    if (c.H < 1 || c.dqk < 1 || c.dv < 1) return HSTU_ERR_INVALID_ARG;
    if (c.B == 0 || c.T == 0) return HSTU_OK;
    if (!c.q || !c.k || !c.v || !c.out || !c.off) return HSTU_ERR_INVALID_ARG;
    if (c.qs < int64_t{c.H} * c.dqk || c.ks < int64_t{c.H} * c.dqk || c.vs < int64_t{c.H} * c.dv ||
        c.os < int64_t{c.H} * c.dv)
        return HSTU_ERR_INVALID_ARG;
    if (c.pos && c.P < 1) return HSTU_ERR_INVALID_ARG;
    if (c.tb && (c.NB < 1 || c.NB > kMaxTimeBuckets)) return HSTU_ERR_INVALID_ARG;
    if (c.dtype == HSTU_DTYPE_BF16) {
        if (c.dqk != c.dv || (c.dqk != 32 && c.dqk != 64 && c.dqk != 128))
            return HSTU_ERR_UNSUPPORTED;
        if (!aligned16(c.q) || !aligned16(c.k) || !aligned16(c.v) || !aligned16(c.out))
            return HSTU_ERR_INVALID_ARG;
        if (c.qs % 8 || c.ks % 8 || c.vs % 8 || c.os % 8) return HSTU_ERR_INVALID_ARG;
        if (!c.ws || c.ws_bytes < hstu_attn_workspace_bytes(c.B, c.T, c.max_seqlen, c.H,
                                                            c.pos ? c.P : 1))
            return HSTU_ERR_INVALID_ARG;
        if (!aligned16(c.ws)) return HSTU_ERR_INVALID_ARG;
    } else {
        if (c.dqk > 128 || c.dv > 128) return HSTU_ERR_UNSUPPORTED;
        if (c.H > 65535) return HSTU_ERR_UNSUPPORTED;
    }
    return HSTU_OK;
}

// Launch of the attention kernel as a programmatic dependent of the kernel
// before it in the stream (normally the plan): its set-up overlaps that
// kernel's tail, and it waits for it (griddepcontrol.wait) before reading the
// work list.
template <typename Kernel>
hstu_status_t launch_attn_pdl(Kernel kernel, unsigned grid, int threads, size_t smem,
                              cudaStream_t stream, const CUtensorMap& tq, const CUtensorMap& tk,
                              const CUtensorMap& tv, const AttnArgs& a) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(static_cast<unsigned>(threads));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, tq, tk, tv, a);
    return e == cudaSuccess ? HSTU_OK : HSTU_ERR_CUDA;
}

// The plan kernel: the longest-first work list into the workspace's plan part
// (and, for the backward, its item-order table: order_h = H).
hstu_status_t launch_plan(const int64_t* off, int32_t B, int64_t T, int32_t max_seqlen, void* ws,
                          cudaStream_t stream, int order_h = 0, int* order_tab = nullptr) {
    const int max_tiles = max_tiles_of(max_seqlen);
    const int64_t max_units = max_units_of(B, T, max_seqlen);
    uint8_t* w = static_cast<uint8_t*>(ws);
    size_t smem = static_cast<size_t>((3 * (max_tiles + 1) + 1) & ~1) * sizeof(int);
    if (B < kPlanSmemOffsets) smem += static_cast<size_t>(B + 1) * sizeof(int64_t);
    plan_kernel<<<1, 1024, smem, stream>>>(
        off, B, T, max_seqlen, max_tiles, static_cast<int>(max_units),
        reinterpret_cast<int4*>(w + kAttnWsHeader),
        reinterpret_cast<uint4*>(w + kAttnWsHeader + attn_units_bytes(B, T, max_seqlen)),
        reinterpret_cast<int*>(w), reinterpret_cast<int*>(w + 16), order_h, order_tab);
    return launch_status();
}

hstu_status_t run_attn(const AttnCall& c) {
    const hstu_status_t st = validate_attn(c);
    if (st != HSTU_OK || c.B == 0 || c.T == 0) return st;
    const bool use_time = c.ts != nullptr && c.tb != nullptr;
    const float inv_n = 1.0f / static_cast<float>(c.max_seqlen);
    if (c.dtype == HSTU_DTYPE_F32) {
        AttnF32Args a{static_cast<const float*>(c.q), c.qs, static_cast<const float*>(c.k), c.ks,
                      static_cast<const float*>(c.v), c.vs, c.off, c.B, c.T, c.H, c.dqk, c.dv,
                      use_time ? c.ts : nullptr, c.pos, c.P, use_time ? c.tb : nullptr,
                      use_time ? c.NB : 1, inv_n, static_cast<float*>(c.out), c.os};
        const dim3 grid(static_cast<unsigned>((c.T + 127) / 128), static_cast<unsigned>(c.H));
        const int dmax = c.dqk > c.dv ? c.dqk : c.dv;
        if (dmax <= 32) attn_fwd_f32_kernel<32><<<grid, 128, 0, c.stream>>>(a);
        else if (dmax <= 64) attn_fwd_f32_kernel<64><<<grid, 128, 0, c.stream>>>(a);
        else attn_fwd_f32_kernel<128><<<grid, 128, 0, c.stream>>>(a);
        return launch_status();
    }
    CUtensorMap tq, tk, tv;
    const uint64_t inner = static_cast<uint64_t>(c.H) * c.dqk;
    if (!make_tmap_bf16(&tq, c.q, inner, c.T, c.qs * 2, 128) ||
        !make_tmap_bf16(&tk, c.k, inner, c.T, c.ks * 2, 128) ||
        !make_tmap_bf16(&tv, c.v, inner, c.T, c.vs * 2, 128))
        return HSTU_ERR_CUDA;
    uint8_t* ws = static_cast<uint8_t*>(c.ws);
    const int P = c.pos ? c.P : 1;
    const int DD = attn_window_tables(P, c.max_seqlen);
    constexpr int G = kAttnGroups;
    const int64_t max_units = max_units_of(c.B, c.T, c.max_seqlen);
    uint4* ptab = reinterpret_cast<uint4*>(ws + attn_plan_bytes(c.B, c.T, c.max_seqlen));
    KeySummary* ksum = reinterpret_cast<KeySummary*>(
        ws + attn_plan_bytes(c.B, c.T, c.max_seqlen) + attn_tables_bytes(c.H, P, c.max_seqlen));
    // bias tables of this run (programmatic dependent of the plan)
    {
        const int64_t entries = static_cast<int64_t>(c.H) * DD * kWinEntries;
        const int table_blocks = static_cast<int>((entries + 127) / 128);
        BiasPrepArgs pa{c.pos, P, c.H, DD, ptab, reinterpret_cast<const int4*>(ws + kAttnWsHeader),
                        reinterpret_cast<const int*>(ws), static_cast<int>(max_units),
                        use_time ? c.ts : nullptr, c.T, ksum, table_blocks};
        const int64_t blocks = table_blocks + (use_time ? max_units : 0);
        if (blocks > 0x7fffffff) return HSTU_ERR_UNSUPPORTED;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(blocks));
        cfg.blockDim = dim3(128);
        cfg.stream = c.stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, bias_prep_kernel, pa) != cudaSuccess) return HSTU_ERR_CUDA;
    }
    AttnArgs a{reinterpret_cast<const int4*>(ws + kAttnWsHeader),
               reinterpret_cast<const int*>(ws),
               static_cast<int>(max_units),
               reinterpret_cast<int*>(ws + 16),
               reinterpret_cast<const uint4*>(ws + kAttnWsHeader +
                                              attn_units_bytes(c.B, c.T, c.max_seqlen)),
               ptab,
               DD,
               use_time ? ksum : nullptr,
               c.H,
               c.T,
               use_time ? c.ts : nullptr,
               c.pos,
               P,
               use_time ? c.tb : nullptr,
               use_time ? c.NB : 0,
               inv_n,
               static_cast<__nv_bfloat16*>(c.out),
               c.os};
    const int64_t items = max_units * c.H;
    if (items > 0x7fffffff) return HSTU_ERR_UNSUPPORTED;
    // persistent: one CTA per SM, work items dealt round-robin
    const unsigned grid = static_cast<unsigned>(items < num_sms() ? items : num_sms());
    static int smem_done32[kMaxDevices] = {0}, smem_done64[kMaxDevices] = {0},
               smem_done128[kMaxDevices] = {0};
    if (c.dqk == 32) {
        if (!ensure_smem(attn_fwd_bf16_kernel<32, G>, AttnSmem<32, G>::kAlloc,
                         smem_done32))
            return HSTU_ERR_CUDA;
        return launch_attn_pdl(attn_fwd_bf16_kernel<32, G>, grid,
                               AttnCfg<32, G>::kThreads, AttnSmem<32, G>::kAlloc,
                               c.stream, tq, tk, tv, a);
    }
    if (c.dqk == 64) {
        if (!ensure_smem(attn_fwd_bf16_kernel<64, G>, AttnSmem<64, G>::kAlloc,
                         smem_done64))
            return HSTU_ERR_CUDA;
        return launch_attn_pdl(attn_fwd_bf16_kernel<64, G>, grid,
                               AttnCfg<64, G>::kThreads, AttnSmem<64, G>::kAlloc,
                               c.stream, tq, tk, tv, a);
    }
    if (!ensure_smem(attn_fwd_bf16_kernel<128, G>, AttnSmem<128, G>::kAlloc,
                     smem_done128))
        return HSTU_ERR_CUDA;
    return launch_attn_pdl(attn_fwd_bf16_kernel<128, G>, grid,
                           AttnCfg<128, G>::kThreads, AttnSmem<128, G>::kAlloc,
                           c.stream, tq, tk, tv, a);
}

hstu_status_t plan_attn(const int64_t* off, int32_t B, int64_t T, int32_t max_seqlen, void* ws,
                        size_t ws_bytes, cudaStream_t stream) {
    if (!plan_sizes_ok(B, T, max_seqlen)) return HSTU_ERR_INVALID_ARG;
    if (B == 0 || T == 0) return HSTU_OK;
    if (!off || !ws || !aligned16(ws) || ws_bytes < attn_plan_bytes(B, T, max_seqlen))
        return HSTU_ERR_INVALID_ARG;
    return launch_plan(off, B, T, max_seqlen, ws, stream);
}

template <int EPI, int BN, bool FP8 = false>
hstu_status_t launch_gemm(unsigned grid, cudaStream_t stream, const CUtensorMap& ta,
                          const CUtensorMap& tb, const CUtensorMap& ty, const CUtensorMap& tr,
                          const GemmArgs& g) {
    constexpr int EW = GemmEpiWarps<EPI, FP8>::value;
    static int done[kMaxDevices] = {0};
    if (!ensure_smem(gemm_bf16_kernel<EPI, BN, FP8>, GemmSmem<BN, EW>::kAlloc, done))
        return HSTU_ERR_CUDA;
    gemm_bf16_kernel<EPI, BN, FP8>
        <<<grid, (EW + 2) * 32, GemmSmem<BN, EW>::kAlloc, stream>>>(ta, tb, ty, tr, g);
    return launch_status();
}

// y = epilogue(x W^T [* sx sw] + b): bf16 operands, or E4M3 codes with
// row scales (fp8)
hstu_status_t run_linear_any(bool fp8, const void* x, int64_t ldx, const float* sx, int64_t M,
                             int32_t K, const void* W, int64_t ldw, const float* sw, int32_t N,
                             const float* bias, hstu_epilogue_t epi, const void* residual,
                             int64_t ldr, void* y, int64_t ldy, cudaStream_t stream) {
    if (M < 0 || K < 1 || N < 1) return HSTU_ERR_INVALID_ARG;
    if (epi != HSTU_EPI_NONE && epi != HSTU_EPI_SILU && epi != HSTU_EPI_RESIDUAL)
        return HSTU_ERR_INVALID_ARG;
    if (K % (fp8 ? 128 : 64) || N % 128) return HSTU_ERR_UNSUPPORTED;
    if (M == 0) return HSTU_OK;
    if (M > (int64_t{1} << 31) - 256) return HSTU_ERR_UNSUPPORTED;
    if (!x || !W || !y) return HSTU_ERR_INVALID_ARG;
    if (fp8 && (!sx || !sw)) return HSTU_ERR_INVALID_ARG;
    const int ab = fp8 ? 16 : 8;     // elements per 16 bytes of an operand row
    if (ldx < K || ldw < K || ldy < N || ldx % ab || ldw % ab || ldy % 8) return HSTU_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(W) || !aligned16(y)) return HSTU_ERR_INVALID_ARG;
    if (epi == HSTU_EPI_RESIDUAL && (!residual || ldr < N || ldr % 8 || !aligned16(residual)))
        return HSTU_ERR_INVALID_ARG;
    // 128 x 256 output tiles when N allows (fewer operand bytes per FLOP),
    // else 128 x 128
    const int bn = N % 256 == 0 ? 256 : 128;
    // output and residual in 32 x 32 blocks (64-byte rows, 64-byte swizzle)
    CUtensorMap ta, tb, ty, tr;
    const bool maps_ok =
        fp8 ? make_tmap_u8(&ta, x, K, M, ldx, 128) &&
                  make_tmap_u8(&tb, W, K, N, ldw, static_cast<uint32_t>(bn))
            : make_tmap_bf16(&ta, x, K, M, ldx * 2, 128) &&
                  make_tmap_bf16(&tb, W, K, N, ldw * 2, static_cast<uint32_t>(bn));
    if (!maps_ok || !make_tmap_bf16_box(&ty, y, N, M, ldy * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
        return HSTU_ERR_CUDA;
    if (epi == HSTU_EPI_RESIDUAL) {
        if (!make_tmap_bf16_box(&tr, residual, N, M, ldr * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
            return HSTU_ERR_CUDA;
    } else {
        tr = ty;    // not read
    }
    GemmArgs g{M, N, K, sx, sw, bias, static_cast<const __nv_bfloat16*>(residual), ldr,
               static_cast<__nv_bfloat16*>(y), ldy};
    const int64_t tiles = (M + 127) / 128 * (N / bn);
    const unsigned grid = static_cast<unsigned>(tiles < num_sms() ? tiles : num_sms());
#define HSTU_GEMM_CASES(F8)                                                                   \
    if (bn == 256) {                                                                          \
        switch (epi) {                                                                        \
            case HSTU_EPI_NONE: return launch_gemm<0, 256, F8>(grid, stream, ta, tb, ty, tr, g); \
            case HSTU_EPI_SILU: return launch_gemm<1, 256, F8>(grid, stream, ta, tb, ty, tr, g); \
            default: return launch_gemm<2, 256, F8>(grid, stream, ta, tb, ty, tr, g);          \
        }                                                                                     \
    }                                                                                         \
    switch (epi) {                                                                            \
        case HSTU_EPI_NONE: return launch_gemm<0, 128, F8>(grid, stream, ta, tb, ty, tr, g);   \
        case HSTU_EPI_SILU: return launch_gemm<1, 128, F8>(grid, stream, ta, tb, ty, tr, g);   \
        default: return launch_gemm<2, 128, F8>(grid, stream, ta, tb, ty, tr, g);            \
    }
    if (fp8) {
        HSTU_GEMM_CASES(true)
    }
    HSTU_GEMM_CASES(false)
#undef HSTU_GEMM_CASES
}

hstu_status_t run_linear(const void* x, int64_t ldx, int64_t M, int32_t K, const void* W,
                         int64_t ldw, int32_t N, const float* bias, hstu_epilogue_t epi,
                         const void* residual, int64_t ldr, void* y, int64_t ldy,
                         cudaStream_t stream) {
    return run_linear_any(false, x, ldx, nullptr, M, K, W, ldw, nullptr, N, bias, epi, residual,
                          ldr, y, ldy, stream);
}

// Y = LayerNorm(A) * U (u given) or Y = LayerNorm(A) (u null, gate == false),
// as bf16 (quant == false) or as row-wise E4M3 codes of that bf16 result with
// row scales (quant == true)
hstu_status_t run_ln_gate_any(bool quant, bool gate, const void* a, int64_t lda, const void* u,
                              int64_t ldu, int64_t M, int32_t F, const float* gamma,
                              const float* beta, float eps, void* y, int64_t ldy, void* yq,
                              int64_t ldyq, float* ys, cudaStream_t stream) {
    if (M < 0 || F < 1 || !(eps >= 0.0f)) return HSTU_ERR_INVALID_ARG;
    if (F % 256 || F > 2048) return HSTU_ERR_UNSUPPORTED;
    if (M == 0) return HSTU_OK;
    if (!a || lda < F || lda % 8 || !aligned16(a)) return HSTU_ERR_INVALID_ARG;
    if (gate && (!u || ldu < F || ldu % 8 || !aligned16(u))) return HSTU_ERR_INVALID_ARG;
    if (quant ? (!yq || !ys || ldyq < F || ldyq % 16 || !aligned16(yq))
              : (!y || ldy < F || ldy % 8 || !aligned16(y)))
        return HSTU_ERR_INVALID_ARG;
    LnGateArgs args{static_cast<const __nv_bfloat16*>(a), lda, static_cast<const __nv_bfloat16*>(u),
                    ldu, M, gamma, beta, eps, static_cast<__nv_bfloat16*>(y), ldy,
                    static_cast<uint8_t*>(yq), ldyq, ys};
    // eight rows per block and pass; as many blocks as are resident at once,
    // each striding over the rows
    const int64_t blocks = (M + 7) / 8;
#define HSTU_LN_LAUNCH(NV, Q, GT)                                                       \
    {                                                                                   \
        static int occ[kMaxDevices] = {0};                                              \
        const unsigned grid = resident_grid(ln_gate_kernel<NV, Q, GT>, 256, blocks, occ); \
        ln_gate_kernel<NV, Q, GT><<<grid, 256, 0, stream>>>(args);                      \
        break;                                                                          \
    }
#define HSTU_LN_CASES(Q, GT)                     \
    switch (F / 256) {                           \
        case 1: HSTU_LN_LAUNCH(1, Q, GT)         \
        case 2: HSTU_LN_LAUNCH(2, Q, GT)         \
        case 3: HSTU_LN_LAUNCH(3, Q, GT)         \
        case 4: HSTU_LN_LAUNCH(4, Q, GT)         \
        case 5: HSTU_LN_LAUNCH(5, Q, GT)         \
        case 6: HSTU_LN_LAUNCH(6, Q, GT)         \
        case 7: HSTU_LN_LAUNCH(7, Q, GT)         \
        default: HSTU_LN_LAUNCH(8, Q, GT)        \
    }
    if (quant && gate) {
        HSTU_LN_CASES(true, true)
    } else if (quant) {
        HSTU_LN_CASES(true, false)
    } else if (gate) {
        HSTU_LN_CASES(false, true)
    } else {
        HSTU_LN_CASES(false, false)
    }
#undef HSTU_LN_CASES
#undef HSTU_LN_LAUNCH
    return launch_status();
}

hstu_status_t run_ln_gate(const void* a, int64_t lda, const void* u, int64_t ldu, int64_t M,
                          int32_t F, const float* gamma, const float* beta, float eps, void* y,
                          int64_t ldy, cudaStream_t stream) {
    return run_ln_gate_any(false, true, a, lda, u, ldu, M, F, gamma, beta, eps, y, ldy, nullptr,
                           0, nullptr, stream);
}

// bf16 layer workspace: [UVQK bf16][A bf16][Y bf16][LayerNorm(x) bf16][attention workspace]
struct LayerWs {
    size_t uvqk, attn, y, xn, plan, total;
};

LayerWs layer_ws(int64_t T, int32_t B, int32_t D, int32_t H, int32_t d, int32_t max_seqlen) {
    LayerWs w{};
    const size_t F = static_cast<size_t>(H) * d;
    w.uvqk = 0;
    w.attn = round_up(w.uvqk + static_cast<size_t>(T) * 4 * F * 2, 256);
    w.y = round_up(w.attn + static_cast<size_t>(T) * F * 2, 256);
    w.xn = round_up(w.y + static_cast<size_t>(T) * F * 2, 256);
    w.plan = round_up(w.xn + static_cast<size_t>(T) * D * 2, 256);
    // window tables for any num_pos: at most one per 128-token diagonal offset
    w.total = w.plan + hstu_attn_workspace_bytes(B, T, max_seqlen, H, 128 * max_tiles_of(max_seqlen));
    return w;
}

// FP8 layer workspace: [x codes T x D][x scales][UVQK bf16][A bf16]
// [Y codes T x F][Y scales][attention workspace]
struct LayerFp8Ws {
    size_t xq, sx, uvqk, attn, yq, sy, plan, total;
};

LayerFp8Ws layer_fp8_ws(int64_t T, int32_t B, int32_t D, int32_t H, int32_t d, int32_t max_seqlen) {
    LayerFp8Ws w{};
    const size_t F = static_cast<size_t>(H) * d, t = static_cast<size_t>(T);
    w.xq = 0;
    w.sx = round_up(w.xq + t * D, 256);
    w.uvqk = round_up(w.sx + t * 4, 256);
    w.attn = round_up(w.uvqk + t * 4 * F * 2, 256);
    w.yq = round_up(w.attn + t * F * 2, 256);
    w.sy = round_up(w.yq + t * F, 256);
    w.plan = round_up(w.sy + t * 4, 256);
    w.total = w.plan + hstu_attn_workspace_bytes(B, T, max_seqlen, H, 128 * max_tiles_of(max_seqlen));
    return w;
}

}  // namespace

extern "C" {

int32_t hstu_abi_version(void) { return HSTU_ABI_VERSION; }

const char* hstu_status_string(hstu_status_t s) {
    switch (s) {
        case HSTU_OK: return "ok";
        case HSTU_ERR_INVALID_ARG: return "invalid argument";
        case HSTU_ERR_UNSUPPORTED: return "unsupported configuration";
        case HSTU_ERR_CUDA: return "CUDA error";
        case HSTU_ERR_TIMEOUT: return "device pipeline wait timed out";
        case HSTU_ERR_BAD_INPUT: return "bad device input (offsets or lengths)";
    }
    return "unknown status";
}

hstu_status_t hstu_device_status(void* stream) {
    if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return HSTU_ERR_CUDA;
    unsigned int word = 0;
    if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word)) != cudaSuccess) return HSTU_ERR_CUDA;
    if (word != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess)
            return HSTU_ERR_CUDA;
    }
    if (word & kErrTimeout) return HSTU_ERR_TIMEOUT;
    if (word & kErrBadInput) return HSTU_ERR_BAD_INPUT;
    return HSTU_OK;
}

size_t hstu_attn_workspace_bytes(int32_t B, int64_t total_tokens, int32_t max_seqlen, int32_t H,
                                 int32_t num_pos) {
    if (!plan_sizes_ok(B, total_tokens, max_seqlen) || H < 1 || num_pos < 0) return 0;
    return attn_plan_bytes(B, total_tokens, max_seqlen) +
           attn_tables_bytes(H, num_pos > 0 ? num_pos : 1, max_seqlen) +
           attn_keys_bytes(B, total_tokens, max_seqlen);
}

hstu_status_t hstu_attn_plan(const int64_t* seq_offsets, int32_t B, int64_t total_tokens,
                             int32_t max_seqlen, void* workspace, size_t workspace_bytes,
                             void* stream) {
    return plan_attn(seq_offsets, B, total_tokens, max_seqlen, workspace, workspace_bytes,
                     as_stream(stream));
}

hstu_status_t hstu_attn_run(hstu_dtype_t dtype, const void* q, int64_t q_tok_stride,
                            const void* k, int64_t k_tok_stride, const void* v,
                            int64_t v_tok_stride, const int64_t* seq_offsets, int32_t B,
                            int64_t total_tokens, int32_t H, int32_t d_qk, int32_t d_v,
                            const int64_t* timestamps, const float* pos_bias, int32_t num_pos,
                            const float* time_bias, int32_t num_time_buckets, int32_t max_seqlen,
                            void* out, int64_t out_tok_stride, void* workspace,
                            size_t workspace_bytes, void* stream) {
    AttnCall c{dtype, q, k, v, q_tok_stride, k_tok_stride, v_tok_stride, seq_offsets, B,
               total_tokens, H, d_qk, d_v, timestamps, pos_bias, num_pos, time_bias,
               num_time_buckets, max_seqlen, out, out_tok_stride, workspace, workspace_bytes,
               as_stream(stream)};
    return run_attn(c);
}

hstu_status_t hstu_attn_fwd(hstu_dtype_t dtype, const void* q, int64_t q_tok_stride,
                            const void* k, int64_t k_tok_stride, const void* v,
                            int64_t v_tok_stride, const int64_t* seq_offsets, int32_t B,
                            int64_t total_tokens, int32_t H, int32_t d_qk, int32_t d_v,
                            const int64_t* timestamps, const float* pos_bias, int32_t num_pos,
                            const float* time_bias, int32_t num_time_buckets, int32_t max_seqlen,
                            void* out, int64_t out_tok_stride, void* workspace,
                            size_t workspace_bytes, void* stream) {
    AttnCall c{dtype, q, k, v, q_tok_stride, k_tok_stride, v_tok_stride, seq_offsets, B,
               total_tokens, H, d_qk, d_v, timestamps, pos_bias, num_pos, time_bias,
               num_time_buckets, max_seqlen, out, out_tok_stride, workspace, workspace_bytes,
               as_stream(stream)};
    hstu_status_t st = validate_attn(c);
    if (st != HSTU_OK || B == 0 || total_tokens == 0) return st;
    if (dtype == HSTU_DTYPE_BF16) {
        st = plan_attn(seq_offsets, B, total_tokens, max_seqlen, workspace, workspace_bytes,
                       as_stream(stream));
        if (st != HSTU_OK) return st;
    }
    return run_attn(c);
}

hstu_status_t hstu_debug_bias_indices(const int64_t* seq_offsets, int32_t B, int64_t total_tokens,
                                      const int64_t* timestamps, int32_t num_pos,
                                      int32_t num_time_buckets, int32_t* pos_idx_out,
                                      int32_t* bucket_out, void* stream) {
    if (B < 0 || total_tokens < 0 || num_pos < 1 || num_time_buckets < 1) return HSTU_ERR_INVALID_ARG;
    if (B == 0 || total_tokens == 0) return HSTU_OK;
    if (!seq_offsets || (bucket_out && !timestamps)) return HSTU_ERR_INVALID_ARG;
    bias_indices_kernel<<<B, 256, 0, as_stream(stream)>>>(seq_offsets, B, timestamps, num_pos,
                                                          num_time_buckets, pos_idx_out, bucket_out);
    return launch_status();
}

hstu_status_t hstu_debug_wait_timeout(int32_t wait_us, void* stream) {
    if (wait_us < 1 || wait_us > 100000) return HSTU_ERR_INVALID_ARG;
    int dev = 0, khz = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&khz, cudaDevAttrClockRate, dev) != cudaSuccess)
        return HSTU_ERR_CUDA;
    const long long limit = static_cast<long long>(wait_us) * (khz > 0 ? khz : 2000000) / 1000;
    wait_timeout_kernel<<<1, 32, 0, as_stream(stream)>>>(limit);
    return launch_status();
}

hstu_status_t hstu_linear_fwd(const void* x, int64_t ldx, int64_t M, int32_t K, const void* W,
                              int64_t ldw, int32_t N, const float* bias, hstu_epilogue_t epilogue,
                              const void* residual, int64_t ldr, void* y, int64_t ldy,
                              void* stream) {
    return run_linear(x, ldx, M, K, W, ldw, N, bias, epilogue, residual, ldr, y, ldy,
                      as_stream(stream));
}

hstu_status_t hstu_attn_bwd_f32(const float* q, const float* k, const float* v, const float* dout,
                                const int64_t* seq_offsets, int32_t B, int64_t total_tokens,
                                int32_t H, int32_t d_qk, int32_t d_v, const int64_t* timestamps,
                                const float* pos_bias, int32_t num_pos, const float* time_bias,
                                int32_t num_time_buckets, int32_t max_seqlen, float* dq, float* dk,
                                float* dv, float* dpos, float* dtime, void* stream) {
    if (!plan_sizes_ok(B, total_tokens, max_seqlen) || H < 1 || d_qk < 1 || d_v < 1)
        return HSTU_ERR_INVALID_ARG;
    if (d_qk > 128 || d_v > 128 || H > 65535) return HSTU_ERR_UNSUPPORTED;
    if (pos_bias && num_pos < 1) return HSTU_ERR_INVALID_ARG;
    const bool use_time = timestamps && time_bias;
    if (use_time && (num_time_buckets < 1 || num_time_buckets > kMaxTimeBuckets))
        return HSTU_ERR_INVALID_ARG;
    if ((pos_bias && !dpos) || (use_time && !dtime)) return HSTU_ERR_INVALID_ARG;
    if (B == 0 || total_tokens == 0) return HSTU_OK;
    if (!q || !k || !v || !dout || !seq_offsets || !dq || !dk || !dv) return HSTU_ERR_INVALID_ARG;
    cudaStream_t s = as_stream(stream);
    const int P = pos_bias ? num_pos : 0, NB = use_time ? num_time_buckets : 0;
    const size_t tab_bytes = static_cast<size_t>(P + NB) * sizeof(float);
    if (tab_bytes > 48 * 1024) return HSTU_ERR_UNSUPPORTED;     // shared-memory table partials
    if (pos_bias && cudaMemsetAsync(dpos, 0, static_cast<size_t>(H) * P * sizeof(float), s) != cudaSuccess)
        return HSTU_ERR_CUDA;
    if (use_time &&
        cudaMemsetAsync(dtime, 0, static_cast<size_t>(H) * NB * sizeof(float), s) != cudaSuccess)
        return HSTU_ERR_CUDA;
    AttnBwdArgs a{q, k, v, dout, seq_offsets, B, total_tokens, H, d_qk, d_v,
                  use_time ? timestamps : nullptr, pos_bias, P, use_time ? time_bias : nullptr, NB,
                  1.0f / static_cast<float>(max_seqlen), dq, dk, dv,
                  pos_bias ? dpos : nullptr, use_time ? dtime : nullptr};
    // four (token, head) warps per block
    if ((total_tokens + 3) / 4 > 0x7fffffff) return HSTU_ERR_UNSUPPORTED;
    const dim3 grid(static_cast<unsigned>((total_tokens + 3) / 4), static_cast<unsigned>(H));
    const int dmax = d_qk > d_v ? d_qk : d_v;
    if (dmax <= 32) {
        attn_bwd_q_kernel<32><<<grid, 128, tab_bytes, s>>>(a);
        attn_bwd_kv_kernel<32><<<grid, 128, 0, s>>>(a);
    } else if (dmax <= 64) {
        attn_bwd_q_kernel<64><<<grid, 128, tab_bytes, s>>>(a);
        attn_bwd_kv_kernel<64><<<grid, 128, 0, s>>>(a);
    } else {
        attn_bwd_q_kernel<128><<<grid, 128, tab_bytes, s>>>(a);
        attn_bwd_kv_kernel<128><<<grid, 128, 0, s>>>(a);
    }
    return launch_status();
}

// backward workspace: the plan's part, then its item-order table (four rows
// of max_tiles + 2 ints)
size_t attn_order_bytes(int32_t max_seqlen) {
    return round_up(static_cast<size_t>(4) * (max_tiles_of(max_seqlen) + 2) * sizeof(int), 256);
}

size_t hstu_attn_bwd_workspace_bytes(int32_t B, int64_t total_tokens, int32_t max_seqlen) {
    if (!plan_sizes_ok(B, total_tokens, max_seqlen)) return 0;
    return attn_plan_bytes(B, total_tokens, max_seqlen) + attn_order_bytes(max_seqlen);
}

hstu_status_t hstu_attn_bwd(hstu_dtype_t dtype, const void* q, int64_t q_stride, const void* k,
                            int64_t k_stride, const void* v, int64_t v_stride, const void* dout,
                            int64_t dout_stride, const int64_t* seq_offsets, int32_t B,
                            int64_t total_tokens, int32_t H, int32_t d, const int64_t* timestamps,
                            const float* pos_bias, int32_t num_pos, const float* time_bias,
                            int32_t num_time_buckets, int32_t max_seqlen, float* dq, float* dk,
                            float* dv, float* dpos, float* dtime, void* workspace,
                            size_t workspace_bytes, void* stream) {
    const int64_t T = total_tokens;
    if (dtype != HSTU_DTYPE_BF16 && dtype != HSTU_DTYPE_F32) return HSTU_ERR_INVALID_ARG;
    if (!plan_sizes_ok(B, T, max_seqlen) || H < 1 || d < 1) return HSTU_ERR_INVALID_ARG;
    if (dtype != HSTU_DTYPE_BF16 || (d != 64 && d != 128)) return HSTU_ERR_UNSUPPORTED;
    if (pos_bias && num_pos < 1) return HSTU_ERR_INVALID_ARG;
    const bool use_time = timestamps && time_bias;
    if (use_time && (num_time_buckets < 1 || num_time_buckets > kMaxTimeBuckets))
        return HSTU_ERR_INVALID_ARG;
    if ((pos_bias && !dpos) || (use_time && !dtime)) return HSTU_ERR_INVALID_ARG;
    cudaStream_t s = as_stream(stream);
    const int P = pos_bias ? num_pos : 0, NB = use_time ? num_time_buckets : 0;
    if (pos_bias && cudaMemsetAsync(dpos, 0, static_cast<size_t>(H) * P * sizeof(float), s) != cudaSuccess)
        return HSTU_ERR_CUDA;
    if (use_time &&
        cudaMemsetAsync(dtime, 0, static_cast<size_t>(H) * NB * sizeof(float), s) != cudaSuccess)
        return HSTU_ERR_CUDA;
    if (B == 0 || T == 0) return HSTU_OK;
    if (!q || !k || !v || !dout || !seq_offsets || !dq || !dk || !dv || !workspace)
        return HSTU_ERR_INVALID_ARG;
    const int64_t row = int64_t{H} * d;
    if (q_stride < row || k_stride < row || v_stride < row || dout_stride < row || q_stride % 8 ||
        k_stride % 8 || v_stride % 8 || dout_stride % 8)
        return HSTU_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(dq) ||
        !aligned16(dk) || !aligned16(dv) || !aligned16(workspace))
        return HSTU_ERR_INVALID_ARG;
    if (workspace_bytes < attn_plan_bytes(B, T, max_seqlen) + attn_order_bytes(max_seqlen))
        return HSTU_ERR_INVALID_ARG;
    if (cudaMemsetAsync(dq, 0, static_cast<size_t>(T) * row * sizeof(float), s) != cudaSuccess)
        return HSTU_ERR_CUDA;
    int* order_tab = reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) +
                                            attn_plan_bytes(B, T, max_seqlen));
    hstu_status_t st = launch_plan(seq_offsets, B, T, max_seqlen, workspace, s, H, order_tab);
    if (st != HSTU_OK) return st;
    CUtensorMap tq, tk, tv, tdo, tdq;
    if (!make_tmap_bf16(&tq, q, row, T, q_stride * 2, 128) ||
        !make_tmap_bf16(&tk, k, row, T, k_stride * 2, 128) ||
        !make_tmap_bf16(&tv, v, row, T, v_stride * 2, 128) ||
        !make_tmap_bf16(&tdo, dout, row, T, dout_stride * 2, 128) ||
        !make_tmap_f32_16x32(&tdq, dq, row, T, row * 4))
        return HSTU_ERR_CUDA;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    BwdArgs a{reinterpret_cast<const int4*>(ws + kAttnWsHeader), reinterpret_cast<const int*>(ws),
              static_cast<int>(max_units_of(B, T, max_seqlen)),
              reinterpret_cast<const uint4*>(ws + kAttnWsHeader + attn_units_bytes(B, T, max_seqlen)),
              H, T, use_time ? timestamps : nullptr, pos_bias, P > 0 ? P : 1,
              use_time ? time_bias : nullptr, NB > 0 ? NB : 1,
              1.0f / static_cast<float>(max_seqlen), dq, dk, dv, pos_bias ? dpos : nullptr,
              use_time ? dtime : nullptr, order_tab, max_tiles_of(max_seqlen)};
    const unsigned grid = static_cast<unsigned>(num_sms());
    if (d == 64) {
        static int done[kMaxDevices] = {0};
        if (!ensure_smem(attn_bwd_bf16_kernel<64>, BwdSmem<64>::kAlloc, done)) return HSTU_ERR_CUDA;
        attn_bwd_bf16_kernel<64><<<grid, BwdCfg<64>::kThreads, BwdSmem<64>::kAlloc, s>>>(
            tq, tk, tv, tdo, tdq, a);
    } else {
        static int done[kMaxDevices] = {0};
        if (!ensure_smem(attn_bwd_bf16_kernel<128>, BwdSmem<128>::kAlloc, done)) return HSTU_ERR_CUDA;
        attn_bwd_bf16_kernel<128><<<grid, BwdCfg<128>::kThreads, BwdSmem<128>::kAlloc, s>>>(
            tq, tk, tv, tdo, tdq, a);
    }
    return launch_status();
}

hstu_status_t hstu_quant_rows_e4m3(const void* x, int64_t ldx, int64_t M, int32_t K, void* codes,
                                   int64_t ldq, float* scales, void* stream) {
    if (M < 0 || K < 1) return HSTU_ERR_INVALID_ARG;
    if (K % 16) return HSTU_ERR_UNSUPPORTED;
    if (M == 0) return HSTU_OK;
    if (!x || !codes || !scales || ldx < K || ldq < K || ldx % 8 || ldq % 16 || !aligned16(x) ||
        !aligned16(codes))
        return HSTU_ERR_INVALID_ARG;
    if ((M + 7) / 8 > 0x7fffffff) return HSTU_ERR_UNSUPPORTED;
    QuantArgs a{static_cast<const __nv_bfloat16*>(x), ldx, M, K, static_cast<uint8_t*>(codes),
                ldq, scales};
    quant_rows_e4m3_kernel<<<static_cast<unsigned>((M + 7) / 8), 256, 0, as_stream(stream)>>>(a);
    return launch_status();
}

hstu_status_t hstu_linear_fp8_fwd(const void* xq, int64_t ldx, const float* x_scales, int64_t M,
                                  int32_t K, const void* wq, int64_t ldw, const float* w_scales,
                                  int32_t N, const float* bias, hstu_epilogue_t epilogue,
                                  const void* residual, int64_t ldr, void* y, int64_t ldy,
                                  void* stream) {
    return run_linear_any(true, xq, ldx, x_scales, M, K, wq, ldw, w_scales, N, bias, epilogue,
                          residual, ldr, y, ldy, as_stream(stream));
}

hstu_status_t hstu_layernorm_gate_fwd(const void* a, int64_t lda, const void* u, int64_t ldu,
                                      int64_t M, int32_t F, const float* gamma, const float* beta,
                                      float eps, void* y, int64_t ldy, void* stream) {
    return run_ln_gate(a, lda, u, ldu, M, F, gamma, beta, eps, y, ldy, as_stream(stream));
}

hstu_status_t hstu_layernorm_fwd(const void* a, int64_t lda, int64_t M, int32_t F,
                                 const float* gamma, const float* beta, float eps, void* y,
                                 int64_t ldy, void* stream) {
    return run_ln_gate_any(false, false, a, lda, nullptr, 0, M, F, gamma, beta, eps, y, ldy,
                           nullptr, 0, nullptr, as_stream(stream));
}

hstu_status_t hstu_layernorm_fp8_fwd(const void* a, int64_t lda, int64_t M, int32_t F,
                                     const float* gamma, const float* beta, float eps,
                                     void* codes, int64_t ldq, float* scales, void* stream) {
    return run_ln_gate_any(true, false, a, lda, nullptr, 0, M, F, gamma, beta, eps, nullptr, 0,
                           codes, ldq, scales, as_stream(stream));
}

size_t hstu_layer_workspace_bytes(int64_t total_tokens, int32_t B, int32_t D, int32_t H, int32_t d,
                                  int32_t max_seqlen) {
    if (total_tokens < 0 || D < 1 || H < 1 || d < 1 || !plan_sizes_ok(B, total_tokens, max_seqlen))
        return 0;
    return layer_ws(total_tokens, B, D, H, d, max_seqlen).total;
}

hstu_status_t hstu_layer_fwd(const void* x, int64_t total_tokens, int32_t D, const void* W1,
                             const float* b1, const void* W2, const float* b2,
                             const float* ln_gamma, const float* ln_beta, float ln_eps,
                             int32_t input_norm, const float* in_gamma, const float* in_beta,
                             const int64_t* seq_offsets, int32_t B, int32_t H, int32_t d,
                             const int64_t* timestamps, const float* pos_bias, int32_t num_pos,
                             const float* time_bias, int32_t num_time_buckets,
                             int32_t max_seqlen, void* out, void* workspace,
                             size_t workspace_bytes, void* stream) {
    const int64_t T = total_tokens;
    if (T < 0 || D < 1 || H < 1 || d < 1 || !plan_sizes_ok(B, T, max_seqlen))
        return HSTU_ERR_INVALID_ARG;
    const int32_t F = H * d;
    if (D % 128 || (d != 64 && d != 128) || F % 256 || F > 2048 || (4 * F) % 128)
        return HSTU_ERR_UNSUPPORTED;
    if (input_norm && (D % 256 || D > 2048)) return HSTU_ERR_UNSUPPORTED;
    if (T == 0 || B == 0) return HSTU_OK;
    if (!x || !W1 || !W2 || !out || !seq_offsets || !workspace) return HSTU_ERR_INVALID_ARG;
    const LayerWs w = layer_ws(T, B, D, H, d, max_seqlen);
    if (workspace_bytes < w.total || !aligned16(workspace)) return HSTU_ERR_INVALID_ARG;
    cudaStream_t s = as_stream(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    __nv_bfloat16* uvqk = reinterpret_cast<__nv_bfloat16*>(ws + w.uvqk);
    __nv_bfloat16* attn = reinterpret_cast<__nv_bfloat16*>(ws + w.attn);
    __nv_bfloat16* ygate = reinterpret_cast<__nv_bfloat16*>(ws + w.y);
    void* plan_ws = ws + w.plan;
    const size_t plan_bytes = workspace_bytes - w.plan;
    // 1. [LayerNorm(x) ->] f1 with the SiLU epilogue
    const void* xin = x;
    hstu_status_t st = HSTU_OK;
    if (input_norm) {
        __nv_bfloat16* xn = reinterpret_cast<__nv_bfloat16*>(ws + w.xn);
        st = run_ln_gate_any(false, false, x, D, nullptr, 0, T, D, in_gamma, in_beta, ln_eps, xn,
                             D, nullptr, 0, nullptr, s);
        if (st != HSTU_OK) return st;
        xin = xn;
    }
    st = run_linear(xin, D, T, D, W1, D, 4 * F, b1, HSTU_EPI_SILU, nullptr, 0, uvqk, 4 * F, s);
    if (st != HSTU_OK) return st;
    st = plan_attn(seq_offsets, B, T, max_seqlen, plan_ws, plan_bytes, s);
    if (st != HSTU_OK) return st;
    AttnCall c{HSTU_DTYPE_BF16, uvqk + 2 * F, uvqk + 3 * F, uvqk + F, 4 * F, 4 * F, 4 * F,
               seq_offsets, B, T, H, d, d, timestamps, pos_bias, num_pos, time_bias,
               num_time_buckets, max_seqlen, attn, F, plan_ws, plan_bytes, s};
    st = run_attn(c);
    if (st != HSTU_OK) return st;
    st = run_ln_gate(attn, F, uvqk, 4 * F, T, F, ln_gamma, ln_beta, ln_eps, ygate, F, s);
    if (st != HSTU_OK) return st;
    return run_linear(ygate, F, T, F, W2, F, D, b2, HSTU_EPI_RESIDUAL, x, D, out, D, s);
}

hstu_status_t hstu_layernorm_gate_fp8_fwd(const void* a, int64_t lda, const void* u, int64_t ldu,
                                          int64_t M, int32_t F, const float* gamma,
                                          const float* beta, float eps, void* codes,
                                          int64_t ldq, float* scales, void* stream) {
    return run_ln_gate_any(true, true, a, lda, u, ldu, M, F, gamma, beta, eps, nullptr, 0, codes,
                           ldq, scales, as_stream(stream));
}

size_t hstu_layer_fp8_workspace_bytes(int64_t total_tokens, int32_t B, int32_t D, int32_t H,
                                      int32_t d, int32_t max_seqlen) {
    if (total_tokens < 0 || D < 1 || H < 1 || d < 1 || !plan_sizes_ok(B, total_tokens, max_seqlen))
        return 0;
    return layer_fp8_ws(total_tokens, B, D, H, d, max_seqlen).total;
}

hstu_status_t hstu_layer_fp8_fwd(const void* x, int64_t total_tokens, int32_t D, const void* W1q,
                                 const float* w1_scales, const float* b1, const void* W2q,
                                 const float* w2_scales, const float* b2, const float* ln_gamma,
                                 const float* ln_beta, float ln_eps, int32_t input_norm,
                                 const float* in_gamma, const float* in_beta,
                                 const int64_t* seq_offsets,
                                 int32_t B, int32_t H, int32_t d, const int64_t* timestamps,
                                 const float* pos_bias, int32_t num_pos, const float* time_bias,
                                 int32_t num_time_buckets, int32_t max_seqlen, void* out,
                                 void* workspace, size_t workspace_bytes, void* stream) {
    const int64_t T = total_tokens;
    if (T < 0 || D < 1 || H < 1 || d < 1 || !plan_sizes_ok(B, T, max_seqlen))
        return HSTU_ERR_INVALID_ARG;
    const int32_t F = H * d;
    if (D % 128 || (d != 64 && d != 128) || F % 256 || F > 2048) return HSTU_ERR_UNSUPPORTED;
    if (input_norm && (D % 256 || D > 2048)) return HSTU_ERR_UNSUPPORTED;
    if (T == 0 || B == 0) return HSTU_OK;
    if (!x || !W1q || !w1_scales || !W2q || !w2_scales || !out || !seq_offsets || !workspace)
        return HSTU_ERR_INVALID_ARG;
    const LayerFp8Ws w = layer_fp8_ws(T, B, D, H, d, max_seqlen);
    if (workspace_bytes < w.total || !aligned16(workspace)) return HSTU_ERR_INVALID_ARG;
    cudaStream_t s = as_stream(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint8_t* xq = ws + w.xq;
    float* sx = reinterpret_cast<float*>(ws + w.sx);
    __nv_bfloat16* uvqk = reinterpret_cast<__nv_bfloat16*>(ws + w.uvqk);
    __nv_bfloat16* attn = reinterpret_cast<__nv_bfloat16*>(ws + w.attn);
    uint8_t* yq = ws + w.yq;
    float* sy = reinterpret_cast<float*>(ws + w.sy);
    void* plan_ws = ws + w.plan;
    const size_t plan_bytes = workspace_bytes - w.plan;
    // 1. x, or LayerNorm(x) in the same pass, -> E4M3 rows; f1 in FP8 with the
    // SiLU epilogue
    hstu_status_t st = input_norm ? run_ln_gate_any(true, false, x, D, nullptr, 0, T, D, in_gamma,
                                                    in_beta, ln_eps, nullptr, 0, xq, D, sx, s)
                                  : hstu_quant_rows_e4m3(x, D, T, D, xq, D, sx, stream);
    if (st != HSTU_OK) return st;
    st = run_linear_any(true, xq, D, sx, T, D, W1q, D, w1_scales, 4 * F, b1, HSTU_EPI_SILU,
                        nullptr, 0, uvqk, 4 * F, s);
    if (st != HSTU_OK) return st;
    // 2. attention (bf16)
    st = plan_attn(seq_offsets, B, T, max_seqlen, plan_ws, plan_bytes, s);
    if (st != HSTU_OK) return st;
    AttnCall c{HSTU_DTYPE_BF16, uvqk + 2 * F, uvqk + 3 * F, uvqk + F, 4 * F, 4 * F, 4 * F,
               seq_offsets, B, T, H, d, d, timestamps, pos_bias, num_pos, time_bias,
               num_time_buckets, max_seqlen, attn, F, plan_ws, plan_bytes, s};
    st = run_attn(c);
    if (st != HSTU_OK) return st;
    // 3. LayerNorm gate quantized to E4M3 rows in the same kernel
    st = run_ln_gate_any(true, true, attn, F, uvqk, 4 * F, T, F, ln_gamma, ln_beta, ln_eps,
                         nullptr, 0, yq, F, sy, s);
    if (st != HSTU_OK) return st;
    // 4. f2 in FP8 with the residual
    return run_linear_any(true, yq, F, sy, T, F, W2q, F, w2_scales, D, b2, HSTU_EPI_RESIDUAL, x,
                          D, out, D, s);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Attention without any allocation by the library or the caller.
//
// Some callers cannot allocate device memory at the moment they run the
// attention: an inference-engine plugin whose enqueue step must not call
// cudaMalloc (it can synchronise the device and can fail under memory
// pressure), or glue code that holds no allocator at all. For them the
// scratch that hstu_attn_fwd takes as `workspace` (the work list of the plan
// kernel) lives in this file-scope device array instead. Every GPU that loads
// the library holds it until the process exits.

static __device__ __align__(256) uint8_t g_noalloc_scratch[HSTU_NOALLOC_SCRATCH_BYTES];

namespace {

std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {nullptr};

// Device address of this device's scratch array. In host code the array's
// name only stands in for the symbol, so the address is looked up once per
// device, with that device current, and cached.
hstu_status_t noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HSTU_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
            return HSTU_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return HSTU_OK;
}

}  // namespace

extern "C" hstu_status_t hstu_attn_fwd_noalloc(
    hstu_dtype_t dtype, const void* q, int64_t q_tok_stride, const void* k, int64_t k_tok_stride,
    const void* v, int64_t v_tok_stride, const int64_t* seq_offsets, int32_t B,
    int64_t total_tokens, int32_t H, int32_t d_qk, int32_t d_v, const int64_t* timestamps,
    const float* pos_bias, int32_t num_pos, const float* time_bias, int32_t num_time_buckets,
    int32_t max_seqlen, void* out, int64_t out_tok_stride, void* stream) {
    void* scratch = nullptr;
    if (dtype == HSTU_DTYPE_BF16 && B > 0 && total_tokens > 0) {
        const size_t need = hstu_attn_workspace_bytes(B, total_tokens, max_seqlen, H,
                                                      pos_bias ? num_pos : 1);
        if (need == 0) return HSTU_ERR_INVALID_ARG;
        if (need > HSTU_NOALLOC_SCRATCH_BYTES) return HSTU_ERR_UNSUPPORTED;
        const hstu_status_t st = noalloc_scratch(&scratch);
        if (st != HSTU_OK) return st;
    }
    return hstu_attn_fwd(dtype, q, q_tok_stride, k, k_tok_stride, v, v_tok_stride, seq_offsets, B,
                         total_tokens, H, d_qk, d_v, timestamps, pos_bias, num_pos, time_bias,
                         num_time_buckets, max_seqlen, out, out_tok_stride, scratch,
                         scratch ? HSTU_NOALLOC_SCRATCH_BYTES : 0, stream);
}

