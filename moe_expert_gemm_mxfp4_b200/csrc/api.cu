// C ABI of the library (declared in include/mxfp4.h): argument validation,
// workspace carving, TMA tensor-map encoding and the launch sequence of each
// entry point.  No allocation, no host synchronization (except in
// mxfp4_get_device_status), no printing.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"


// Per-device status word written by kernels whose waits ran out of time.
__device__ unsigned g_mxfp4_status;

namespace {

thread_local int tl_last_cuda_error = 0;
thread_local void* const* tl_trace_events = nullptr;
thread_local int tl_trace_n = 0;

// Stage boundary i of a traced call (no-op unless tracing is on).
void trace_mark(int i, cudaStream_t s) {
    if (tl_trace_events && i < tl_trace_n && tl_trace_events[i])
        cudaEventRecord(static_cast<cudaEvent_t>(tl_trace_events[i]), s);
}

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    int sm_count = 0;
    int major = 0, minor = 0;
    unsigned* status = nullptr;
    bool ready = false;
};

std::mutex g_dev_mutex;
DeviceInfo g_dev[kMaxDevices];

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

mxfp4_status cuda_fail(cudaError_t e) {
    tl_last_cuda_error = static_cast<int>(e);
    return MXFP4_ERR_CUDA;
}

// Device properties and the status word's address, once per device.
mxfp4_status device_info(DeviceInfo** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return MXFP4_ERR_ARCH;
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    DeviceInfo& d = g_dev[dev];
    if (!d.ready) {
        if ((e = cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return cuda_fail(e);
        if (d.major == 10 && d.minor == 0) {
            void* p = nullptr;
            if ((e = cudaGetSymbolAddress(&p, g_mxfp4_status)) != cudaSuccess) return cuda_fail(e);
            d.status = static_cast<unsigned*>(p);
        }
        d.ready = true;
    }
    if (!(d.major == 10 && d.minor == 0)) return MXFP4_ERR_ARCH;
    *out = &d;
    return MXFP4_OK;
}

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Packed codes of G groups as a 3-D tensor {K/2 bytes, rows, G}; box {128, box_rows, 1}
// (128 B = 256 K values of each row per copy); 128-byte swizzle (conflict-free 16-B
// reads of one row per thread).
mxfp4_status encode_codes_map(CUtensorMap* m, const uint8_t* codes, int64_t K, int64_t rows,
                              int64_t G, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cuda_fail(cudaErrorNotSupported);
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows),
                                static_cast<cuuint64_t>(G)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(K / 2),
                                   static_cast<cuuint64_t>(rows * (K / 2))};
    const cuuint32_t box[3] = {128, static_cast<cuuint32_t>(box_rows), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(codes), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MXFP4_OK : cuda_fail(cudaErrorInvalidValue);
}

// bf16 activations {K, rows}; box {64, nt}; 128-byte swizzle (UMMA K-major SW128 layout).
mxfp4_status encode_act_map(CUtensorMap* m, const void* x, int64_t K, int64_t rows, int nt) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cuda_fail(cudaErrorNotSupported);
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K * 2)};
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(nt)};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MXFP4_OK : cuda_fail(cudaErrorInvalidValue);
}

// Packed E2M1 activation codes {K/2 bytes, rows}; box {128, nt} (256 K values per
// row); 128-byte swizzle (UMMA K-major SW128 layout of a 4-bit operand).
mxfp4_status encode_x4_map(CUtensorMap* m, const uint8_t* codes, int64_t K, int64_t rows, int nt) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cuda_fail(cudaErrorNotSupported);
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
    const cuuint32_t box[2] = {128, static_cast<cuuint32_t>(nt)};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MXFP4_OK : cuda_fail(cudaErrorInvalidValue);
}

// bf16 weights of G groups as a 3-D tensor {K, rows, G}; box {64, box_rows, 1}
// (128 B of K per row per copy); 128-byte swizzle (UMMA K-major SW128 layout).
mxfp4_status encode_w16_map(CUtensorMap* m, const void* w, int64_t K, int64_t rows, int64_t G, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cuda_fail(cudaErrorNotSupported);
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows),
                                static_cast<cuuint64_t>(G)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(K * 2), static_cast<cuuint64_t>(rows * K * 2)};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(w), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MXFP4_OK : cuda_fail(cudaErrorInvalidValue);
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Workspace of moe_mxfp4_mlp, carved in this order (256-byte aligned pieces).
struct MoeWs {
    int32_t* ids;
    float* weights;
    int32_t* counts;
    int32_t* offsets;
    int32_t* perm;
    int32_t* inv;
    float* w_sorted;
    void* route_tmp;
    void* x_sorted;   // W4A16: bf16 [P, H]
    void* h;          // bf16 [P, I]
    void* y_sorted;   // fp32 [P, H]
    // W4A4 only, the MXFP4 activations: x (codes [T, H/2], scales [T, H/32]), the
    // gathered rows (codes [P, H/2], scales [P, H/32]) and h (codes [P, I/2], scales
    // [P, I/32]).
    uint8_t* xq_codes;
    uint8_t* xq_scales;
    uint8_t* xs_codes;
    uint8_t* xs_scales;
    uint8_t* hq_codes;
    uint8_t* hq_scales;
    size_t bytes;
};

MoeWs carve_moe(void* base, int64_t T, int64_t H, int64_t I, int64_t E, int top_k, int mode) {
    const int64_t P = T * top_k;
    MoeWs w{};
    size_t off = 0;
    auto take = [&](size_t n) {
        void* p = base ? static_cast<uint8_t*>(base) + off : nullptr;
        off = align_up(off + n, 256);
        return p;
    };
    w.ids = static_cast<int32_t*>(take(P * 4));
    w.weights = static_cast<float*>(take(P * 4));
    w.counts = static_cast<int32_t*>(take(E * 4));
    w.offsets = static_cast<int32_t*>(take((E + 1) * 4));
    w.perm = static_cast<int32_t*>(take(P * 4));
    w.inv = static_cast<int32_t*>(take(P * 4));
    w.w_sorted = static_cast<float*>(take(P * 4));
    w.route_tmp = take(mx::route_tmp_bytes(T, E, top_k));
    if (mode == MXFP4_W4A4) {
        // scale arrays keep 16 readable bytes past their end (the GEMM's staging copy
        // rounds its byte range up to 16)
        w.xq_codes = static_cast<uint8_t*>(take(static_cast<size_t>(T) * H / 2));
        w.xq_scales = static_cast<uint8_t*>(take(static_cast<size_t>(T) * H / 32 + 16));
        w.xs_codes = static_cast<uint8_t*>(take(static_cast<size_t>(P) * H / 2));
        w.xs_scales = static_cast<uint8_t*>(take(static_cast<size_t>(P) * H / 32 + 16));
    } else {
        w.x_sorted = take(static_cast<size_t>(P) * H * 2);
    }
    w.h = take(static_cast<size_t>(P) * I * 2);
    if (mode == MXFP4_W4A4) {
        w.hq_codes = static_cast<uint8_t*>(take(static_cast<size_t>(P) * I / 2));
        w.hq_scales = static_cast<uint8_t*>(take(static_cast<size_t>(P) * I / 32 + 16));
    }
    w.y_sorted = take(static_cast<size_t>(P) * H * 4);
    w.bytes = off;
    return w;
}

int gemm_grid(const DeviceInfo* d, int64_t tile_bound) {
    int64_t g = tile_bound < d->sm_count ? tile_bound : d->sm_count;
    return static_cast<int>(g < 1 ? 1 : g);
}

// Operands of the experts' two grouped GEMMs (gate/up + SwiGLU, then down x the
// routing weight), all device memory.
struct ExpertsIO {
    const void* x_rows;       // W4A16: bf16 activation rows in expert-sorted order
    int64_t x_rows_n;         // rows of x_rows
    const uint8_t* xs_codes;  // W4A4: sorted activation rows as MXFP4 (codes, scales + 16 B)
    const uint8_t* xs_scales;
    const int32_t* offsets;   // [E + 1] sorted-row offsets of the experts
    const float* row_w;       // [P] routing weight of every sorted row
    void* h;                  // bf16 [P, I]
    uint8_t* hq_codes;        // W4A4: h as MXFP4
    uint8_t* hq_scales;
    void* y_sorted;           // fp32 [P, H] out
};

void trace_mark(int i, cudaStream_t s);

// The experts of one layer on their expert-sorted rows: h = bf16(SiLU(x W_g^T) * (x W_u^T)),
// then y = w * (h W_2^T) in fp32 (W4A4: x and h quantized to MXFP4 first).
mxfp4_status run_experts(DeviceInfo* d, int64_t P, int64_t H, int64_t I, int64_t E, mxfp4_mode mode,
                         const uint8_t* w13_codes, const uint8_t* w13_scales, const uint8_t* w2_codes,
                         const uint8_t* w2_scales, const ExpertsIO& io, cudaStream_t s) {
    const bool a4 = mode == MXFP4_W4A4;
    mxfp4_status st;
    cudaError_t e;
    const mx::TokenTiling tiling = a4 ? mx::pick_token_tiling_w4a4(P, E) : mx::pick_token_tiling(P, E);
    const int64_t tile_rows = static_cast<int64_t>(tiling.nt) * tiling.tt;
    const int64_t tok_tiles = (P + tile_rows - 1) / tile_rows + E;

    // gate/up projection with the SwiGLU epilogue -> h [P, I]
    CUtensorMap tw, tx;
    if ((st = encode_codes_map(&tw, w13_codes, H, 2 * I, E, a4 ? 16 : 64)) != MXFP4_OK) return st;
    st = a4 ? encode_x4_map(&tx, io.xs_codes, H, P, tiling.nt)
            : encode_act_map(&tx, io.x_rows, H, io.x_rows_n, tiling.nt);
    if (st != MXFP4_OK) return st;
    mx::GemmArgs a{};
    a.w_scales = w13_scales;
    a.x_scales = io.xs_scales;
    a.offsets = io.offsets;
    a.m_single = 0;
    a.G = static_cast<int>(E);
    a.K = static_cast<int>(H);
    a.rows_w = static_cast<int>(2 * I);
    a.I = static_cast<int>(I);
    a.n_ftiles = static_cast<int>(I / 64);
    a.out = io.h;
    a.out_ld = I;
    a.n_valid_feat = static_cast<int>(I);
    a.row_w = nullptr;
    a.status = d->status;
    const int grid1 = gemm_grid(d, tok_tiles * a.n_ftiles);
    e = a4      ? mx::launch_grouped_gemm_w4a4(mx::EPI_SWIGLU, tiling.nt, tw, tx, a, grid1, s)
                : mx::launch_grouped_gemm(mx::EPI_SWIGLU, tiling, tw, tx, a, grid1, s);
    if (e != cudaSuccess) return cuda_fail(e);

    trace_mark(2, s);
    if (a4) {   // h to MXFP4 (FLOOR rule, blocks along I)
        if ((e = mx::launch_quantize(io.h, 0, P, I, io.hq_codes, io.hq_scales, MXFP4_SCALE_FLOOR,
                                     d->sm_count, d->status, s)) != cudaSuccess)
            return cuda_fail(e);
    }

    // down projection, routing weight applied in fp32 -> y_sorted fp32 [P, H]
    if ((st = encode_codes_map(&tw, w2_codes, I, H, E, 128)) != MXFP4_OK) return st;
    st = a4 ? encode_x4_map(&tx, io.hq_codes, I, P, tiling.nt) : encode_act_map(&tx, io.h, I, P, tiling.nt);
    if (st != MXFP4_OK) return st;
    a.w_scales = w2_scales;
    a.x_scales = io.hq_scales;
    a.K = static_cast<int>(I);
    a.rows_w = static_cast<int>(H);
    a.I = 0;
    a.n_ftiles = static_cast<int>((H + 127) / 128);
    a.out = io.y_sorted;
    a.out_ld = H;
    a.n_valid_feat = static_cast<int>(H);
    a.row_w = io.row_w;
    const int grid2 = gemm_grid(d, tok_tiles * a.n_ftiles);
    e = a4      ? mx::launch_grouped_gemm_w4a4(mx::EPI_WEIGHTED, tiling.nt, tw, tx, a, grid2, s)
                : mx::launch_grouped_gemm(mx::EPI_WEIGHTED, tiling, tw, tx, a, grid2, s);
    if (e != cudaSuccess) return cuda_fail(e);
    trace_mark(3, s);
    return MXFP4_OK;
}

// Workspace of moe_mxfp4_experts: W4A4 sorted rows as MXFP4, h, W4A4 h as MXFP4.
struct ExpertsWs {
    uint8_t* xs_codes;
    uint8_t* xs_scales;
    void* h;
    uint8_t* hq_codes;
    uint8_t* hq_scales;
    size_t bytes;
};

ExpertsWs carve_experts(void* base, int64_t P, int64_t H, int64_t I, int mode) {
    ExpertsWs w{};
    size_t off = 0;
    auto take = [&](size_t n) {
        void* p = base ? static_cast<uint8_t*>(base) + off : nullptr;
        off = align_up(off + n, 256);
        return p;
    };
    if (mode == MXFP4_W4A4) {
        w.xs_codes = static_cast<uint8_t*>(take(static_cast<size_t>(P) * H / 2));
        w.xs_scales = static_cast<uint8_t*>(take(static_cast<size_t>(P) * H / 32 + 16));
    }
    w.h = take(static_cast<size_t>(P) * I * 2);
    if (mode == MXFP4_W4A4) {
        w.hq_codes = static_cast<uint8_t*>(take(static_cast<size_t>(P) * I / 2));
        w.hq_scales = static_cast<uint8_t*>(take(static_cast<size_t>(P) * I / 32 + 16));
    }
    w.bytes = off;
    return w;
}

}  // namespace

extern "C" {

const char* mxfp4_status_string(mxfp4_status s) {
    switch (s) {
        case MXFP4_OK: return "MXFP4_OK";
        case MXFP4_ERR_INVALID_ARG: return "MXFP4_ERR_INVALID_ARG";
        case MXFP4_ERR_UNSUPPORTED_SHAPE: return "MXFP4_ERR_UNSUPPORTED_SHAPE";
        case MXFP4_ERR_MISALIGNED: return "MXFP4_ERR_MISALIGNED";
        case MXFP4_ERR_ARCH: return "MXFP4_ERR_ARCH";
        case MXFP4_ERR_WORKSPACE: return "MXFP4_ERR_WORKSPACE";
        case MXFP4_ERR_CUDA: return "MXFP4_ERR_CUDA";
        case MXFP4_ERR_TIMEOUT: return "MXFP4_ERR_TIMEOUT";
    }
    return "MXFP4_ERR_UNKNOWN";
}

int mxfp4_last_cuda_error(void) { return tl_last_cuda_error; }

mxfp4_status mxfp4_selftest_wait_timeout(void* stream) {
    DeviceInfo* d = nullptr;
    mxfp4_status st = device_info(&d);
    if (st != MXFP4_OK) return st;
    cudaError_t e = mx::launch_selftest_wait_timeout(d->status, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MXFP4_OK : cuda_fail(e);
}

mxfp4_status mxfp4_selftest_mma_rate(int32_t kind, int32_t iters, double* flops, void* stream) {
    if ((kind != 0 && kind != 1) || iters <= 0 || iters > (1 << 20) || !flops) return MXFP4_ERR_INVALID_ARG;
    DeviceInfo* d = nullptr;
    mxfp4_status st = device_info(&d);
    if (st != MXFP4_OK) return st;
    *flops = mx::selftest_mma_flops(kind, iters, d->sm_count);
    cudaError_t e = mx::launch_selftest_mma_rate(kind, iters, d->sm_count, d->status,
                                                 static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MXFP4_OK : cuda_fail(e);
}

void mxfp4_set_trace_events(void* const* events, int n_events) {
    tl_trace_events = n_events > 0 ? events : nullptr;
    tl_trace_n = n_events > 0 ? n_events : 0;
}

mxfp4_status mxfp4_get_device_status(void* stream) {
    DeviceInfo* d = nullptr;
    mxfp4_status st = device_info(&d);
    if (st != MXFP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e);
    unsigned v = 0;
    if ((e = cudaMemcpyFromSymbolAsync(&v, g_mxfp4_status, sizeof v, 0, cudaMemcpyDeviceToHost, s)) != cudaSuccess)
        return cuda_fail(e);
    const unsigned zero = 0;
    if ((e = cudaMemcpyToSymbolAsync(g_mxfp4_status, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, s)) != cudaSuccess)
        return cuda_fail(e);
    if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return cuda_fail(e);
    return static_cast<mxfp4_status>(v);
}

mxfp4_status mxfp4_quantize(const void* x, mxfp4_in_dtype dt, int64_t rows, int64_t cols,
                            uint8_t* codes, uint8_t* scales, mxfp4_scale_rule rule, void* stream) {
    if (!x || !codes || !scales) return MXFP4_ERR_INVALID_ARG;
    if (rows <= 0 || cols <= 0) return MXFP4_ERR_INVALID_ARG;
    if (dt != MXFP4_IN_BF16 && dt != MXFP4_IN_F32) return MXFP4_ERR_INVALID_ARG;
    if (rule != MXFP4_SCALE_FLOOR && rule != MXFP4_SCALE_CEIL) return MXFP4_ERR_INVALID_ARG;
    if (cols % 32 != 0) return MXFP4_ERR_UNSUPPORTED_SHAPE;
    if (rows > (int64_t{1} << 40) / cols) return MXFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales)) return MXFP4_ERR_MISALIGNED;
    DeviceInfo* d = nullptr;
    mxfp4_status st = device_info(&d);
    if (st != MXFP4_OK) return st;
    cudaError_t e = mx::launch_quantize(x, dt == MXFP4_IN_F32, rows, cols, codes, scales,
                                        static_cast<int>(rule), d->sm_count, d->status,
                                        static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MXFP4_OK : cuda_fail(e);
}

mxfp4_status mxfp4_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t rows,
                              int64_t cols, void* out_bf16, void* stream) {
    if (!codes || !scales || !out_bf16) return MXFP4_ERR_INVALID_ARG;
    if (rows <= 0 || cols <= 0) return MXFP4_ERR_INVALID_ARG;
    if (cols % 32 != 0) return MXFP4_ERR_UNSUPPORTED_SHAPE;
    if (rows > (int64_t{1} << 40) / cols) return MXFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(codes) || !aligned16(scales) || !aligned16(out_bf16)) return MXFP4_ERR_MISALIGNED;
    DeviceInfo* d = nullptr;
    mxfp4_status st = device_info(&d);
    if (st != MXFP4_OK) return st;
    cudaError_t e = mx::launch_dequantize(codes, scales, rows, cols, out_bf16, d->sm_count,
                                          d->status, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MXFP4_OK : cuda_fail(e);
}

size_t mxfp4_gemm_workspace_size(int64_t M, int64_t K, int64_t N, mxfp4_mode mode) {
    (void)N;
    if (mode != MXFP4_W4A4 || M <= 0 || K <= 0) return 0;
    return align_up(static_cast<size_t>(M) * K / 2, 256) +
           align_up(static_cast<size_t>(M) * K / 32 + 16, 256);
}

int32_t mxfp4_token_tile_rows(int64_t rows, int64_t groups, mxfp4_mode mode) {
    if (rows < 1 || groups < 1 || rows >= (int64_t{1} << 62) || groups >= (int64_t{1} << 62)) return 0;
    if (mode == MXFP4_W4A16) return mx::pick_token_tiling(rows, groups).nt;
    if (mode == MXFP4_W4A4) return mx::pick_token_tiling_w4a4(rows, groups).nt;
    return 0;
}

mxfp4_status mxfp4_gemm(const void* x_bf16, int64_t M, int64_t K, const uint8_t* w_codes,
                        const uint8_t* w_scales, int64_t N, void* y_bf16, mxfp4_mode mode,
                        void* ws, size_t ws_bytes, void* stream) {
    if (!x_bf16 || !w_codes || !w_scales || !y_bf16) return MXFP4_ERR_INVALID_ARG;
    if (M <= 0 || K <= 0 || N <= 0) return MXFP4_ERR_INVALID_ARG;
    if (mode != MXFP4_W4A16 && mode != MXFP4_W4A4) return MXFP4_ERR_INVALID_ARG;
    if (K % 64 != 0) return MXFP4_ERR_UNSUPPORTED_SHAPE;
    if (M >= (int64_t{1} << 31) || N >= (int64_t{1} << 31) || K > mx::max_gemm_k() ||
        (mode == MXFP4_W4A4 && K > mx::max_gemm_k_w4a4()))
        return MXFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x_bf16) || !aligned16(w_codes) || !aligned16(w_scales) || !aligned16(y_bf16))
        return MXFP4_ERR_MISALIGNED;
    const size_t need = mxfp4_gemm_workspace_size(M, K, N, mode);
    if (need > 0 && (!ws || ws_bytes < need)) return MXFP4_ERR_WORKSPACE;
    if (ws && !aligned16(ws)) return MXFP4_ERR_MISALIGNED;
    DeviceInfo* d = nullptr;
    mxfp4_status st = device_info(&d);
    if (st != MXFP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const mx::TokenTiling tiling =
        mode == MXFP4_W4A4 ? mx::pick_token_tiling_w4a4(M, 1) : mx::pick_token_tiling(M, 1);
    CUtensorMap tw, tx;
    if ((st = encode_codes_map(&tw, w_codes, K, N, 1, 128)) != MXFP4_OK) return st;
    uint8_t* xq_codes = static_cast<uint8_t*>(ws);
    uint8_t* xq_scales = xq_codes ? xq_codes + align_up(static_cast<size_t>(M) * K / 2, 256) : nullptr;
    if (mode == MXFP4_W4A4) {   // activations to MXFP4 (FLOOR rule, blocks along K)
        cudaError_t e = mx::launch_quantize(x_bf16, 0, M, K, xq_codes, xq_scales, MXFP4_SCALE_FLOOR,
                                            d->sm_count, d->status, s);
        if (e != cudaSuccess) return cuda_fail(e);
        st = encode_x4_map(&tx, xq_codes, K, M, tiling.nt);
    } else {
        st = encode_act_map(&tx, x_bf16, K, M, tiling.nt);
    }
    if (st != MXFP4_OK) return st;
    mx::GemmArgs a{};
    a.w_scales = w_scales;
    a.offsets = nullptr;
    a.m_single = static_cast<int>(M);
    a.G = 1;
    a.K = static_cast<int>(K);
    a.rows_w = static_cast<int>(N);
    a.I = 0;
    a.n_ftiles = static_cast<int>((N + 127) / 128);
    a.out = y_bf16;
    a.out_ld = N;
    a.n_valid_feat = static_cast<int>(N);
    a.row_w = nullptr;
    a.status = d->status;
    a.x_scales = xq_scales;
    const int64_t tile_rows = static_cast<int64_t>(tiling.nt) * tiling.tt;
    const int64_t tiles = ((M + tile_rows - 1) / tile_rows) * a.n_ftiles;
    cudaError_t e = mode == MXFP4_W4A4
                        ? mx::launch_grouped_gemm_w4a4(mx::EPI_PLAIN, tiling.nt, tw, tx, a,
                                                       gemm_grid(d, tiles), s)
                            : mx::launch_grouped_gemm(mx::EPI_PLAIN, tiling, tw, tx, a,
                                                      gemm_grid(d, tiles), s);
    return e == cudaSuccess ? MXFP4_OK : cuda_fail(e);
}

static mxfp4_status check_route_args(const float* logits, int64_t T, int64_t E, int32_t top_k) {
    if (!logits) return MXFP4_ERR_INVALID_ARG;
    if (T <= 0 || E <= 0 || top_k <= 0) return MXFP4_ERR_INVALID_ARG;
    if (E > 256 || top_k > 8 || top_k > E) return MXFP4_ERR_UNSUPPORTED_SHAPE;
    if (T * top_k >= (int64_t{1} << 31)) return MXFP4_ERR_UNSUPPORTED_SHAPE;
    return MXFP4_OK;
}

size_t moe_mxfp4_route_workspace_size(int64_t T, int64_t E, int32_t top_k) {
    if (T <= 0 || E <= 0 || top_k <= 0) return 0;
    return align_up(mx::route_tmp_bytes(T, E, top_k), 256);
}

mxfp4_status moe_mxfp4_route(const float* router_logits, int64_t T, int64_t E, int32_t top_k,
                             int32_t* ids, float* weights, int32_t* counts, int32_t* offsets,
                             int32_t* perm, int32_t* inv, void* ws, size_t ws_bytes, void* stream) {
    mxfp4_status st = check_route_args(router_logits, T, E, top_k);
    if (st != MXFP4_OK) return st;
    if (!ids || !weights || !counts || !offsets || !perm || !inv) return MXFP4_ERR_INVALID_ARG;
    if (!aligned16(router_logits) || !aligned16(ids) || !aligned16(weights) || !aligned16(counts) ||
        !aligned16(offsets) || !aligned16(perm) || !aligned16(inv))
        return MXFP4_ERR_MISALIGNED;
    const size_t need = moe_mxfp4_route_workspace_size(T, E, top_k);
    if (!ws || ws_bytes < need) return MXFP4_ERR_WORKSPACE;
    if (!aligned16(ws)) return MXFP4_ERR_MISALIGNED;
    DeviceInfo* d = nullptr;
    if ((st = device_info(&d)) != MXFP4_OK) return st;
    cudaError_t e = mx::launch_route(router_logits, T, E, top_k, ids, weights, counts, offsets, perm,
                                     inv, nullptr, nullptr, ws, nullptr, 0, nullptr, nullptr, 0, nullptr,
                                     d->sm_count, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MXFP4_OK : cuda_fail(e);
}

mxfp4_status moe_mxfp4_route_project(const void* x_bf16, int64_t T, int64_t H, const void* w_router_bf16,
                                     int64_t E, int32_t top_k, int32_t* ids, float* weights,
                                     int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                                     float* logits_out, void* ws, size_t ws_bytes, void* stream) {
    if (!x_bf16 || !w_router_bf16 || !ids || !weights || !counts || !offsets || !perm || !inv)
        return MXFP4_ERR_INVALID_ARG;
    if (T <= 0 || H <= 0 || E <= 0 || top_k <= 0) return MXFP4_ERR_INVALID_ARG;
    if (E > 256 || top_k > 8 || top_k > E) return MXFP4_ERR_UNSUPPORTED_SHAPE;
    if (H % 64 != 0 || T * top_k >= (int64_t{1} << 31) || H >= (int64_t{1} << 31))
        return MXFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x_bf16) || !aligned16(w_router_bf16) || !aligned16(ids) || !aligned16(weights) ||
        !aligned16(counts) || !aligned16(offsets) || !aligned16(perm) || !aligned16(inv) ||
        (logits_out && !aligned16(logits_out)))
        return MXFP4_ERR_MISALIGNED;
    const size_t need = moe_mxfp4_route_workspace_size(T, E, top_k);
    if (!ws || ws_bytes < need) return MXFP4_ERR_WORKSPACE;
    if (!aligned16(ws)) return MXFP4_ERR_MISALIGNED;
    DeviceInfo* d = nullptr;
    mxfp4_status st = device_info(&d);
    if (st != MXFP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // x [T, H] in 128-token boxes; W_r [E, H] in one box of E rounded up to 16 rows
    // (the rows past E are the TMA's zero fill)
    CUtensorMap tx, tw;
    if ((st = encode_act_map(&tx, x_bf16, H, T, 128)) != MXFP4_OK) return st;
    if ((st = encode_act_map(&tw, w_router_bf16, H, E, static_cast<int>((E + 15) / 16 * 16))) != MXFP4_OK)
        return st;
    int32_t *chunk_counts, *local_rank;
    mx::route_tmp_split(ws, T, E, &chunk_counts, &local_rank);
    cudaError_t e = mx::launch_route_project(tx, tw, T, H, E, top_k, ids, weights, chunk_counts,
                                             local_rank, logits_out, d->sm_count, d->status, s);
    if (e != cudaSuccess) return cuda_fail(e);
    e = mx::launch_route_finish(T, E, top_k, ids, weights, counts, offsets, perm, inv, nullptr, nullptr,
                                ws, nullptr, 0, nullptr, nullptr, 0, nullptr, d->sm_count, s);
    return e == cudaSuccess ? MXFP4_OK : cuda_fail(e);
}

size_t moe_mxfp4_workspace_size(int64_t T, int64_t H, int64_t I, int64_t E, int32_t top_k,
                                mxfp4_mode mode) {
    if (T <= 0 || H <= 0 || I <= 0 || E <= 0 || top_k <= 0) return 0;
    return carve_moe(nullptr, T, H, I, E, top_k, mode).bytes;
}

mxfp4_status moe_mxfp4_mlp(const void* x_bf16, int64_t T, int64_t H, const float* router_logits,
                           int64_t E, int32_t top_k, const uint8_t* w13_codes,
                           const uint8_t* w13_scales, int64_t I, const uint8_t* w2_codes,
                           const uint8_t* w2_scales, void* out_bf16, mxfp4_mode mode, void* ws,
                           size_t ws_bytes, void* stream) {
    mxfp4_status st = check_route_args(router_logits, T, E, top_k);
    if (st != MXFP4_OK) return st;
    if (!x_bf16 || !w13_codes || !w13_scales || !w2_codes || !w2_scales || !out_bf16)
        return MXFP4_ERR_INVALID_ARG;
    if (H <= 0 || I <= 0) return MXFP4_ERR_INVALID_ARG;
    if (mode != MXFP4_W4A16 && mode != MXFP4_W4A4) return MXFP4_ERR_INVALID_ARG;
    if (H % 64 != 0 || I % 64 != 0) return MXFP4_ERR_UNSUPPORTED_SHAPE;
    if (H > mx::max_gemm_k() || I > mx::max_gemm_k()) return MXFP4_ERR_UNSUPPORTED_SHAPE;
    if (mode == MXFP4_W4A4 && (H > mx::max_gemm_k_w4a4() || I > mx::max_gemm_k_w4a4()))
        return MXFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x_bf16) || !aligned16(router_logits) || !aligned16(w13_codes) ||
        !aligned16(w13_scales) || !aligned16(w2_codes) || !aligned16(w2_scales) ||
        !aligned16(out_bf16))
        return MXFP4_ERR_MISALIGNED;
    const size_t need = moe_mxfp4_workspace_size(T, H, I, E, top_k, mode);
    if (!ws || ws_bytes < need) return MXFP4_ERR_WORKSPACE;
    if (!aligned16(ws)) return MXFP4_ERR_MISALIGNED;
    DeviceInfo* d = nullptr;
    if ((st = device_info(&d)) != MXFP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const MoeWs w = carve_moe(ws, T, H, I, E, top_k, mode);
    const int64_t P = T * top_k;
    cudaError_t e;

    trace_mark(0, s);
    const bool a4 = mode == MXFP4_W4A4;
    if (a4) {
        // W4A4: x to MXFP4 per token (FLOOR rule, blocks along H); the gather then
        // moves packed rows (H/2 code bytes + H/32 scale bytes) instead of bf16 rows
        if ((e = mx::launch_quantize(x_bf16, 0, T, H, w.xq_codes, w.xq_scales, MXFP4_SCALE_FLOOR,
                                     d->sm_count, d->status, s)) != cudaSuccess)
            return cuda_fail(e);
        e = mx::launch_route(router_logits, T, E, top_k, w.ids, w.weights, w.counts, w.offsets,
                             w.perm, w.inv, w.w_sorted, nullptr, w.route_tmp, w.xq_codes, H / 2,
                             w.xs_codes, w.xq_scales, H / 32, w.xs_scales, d->sm_count, s);
    } else {
        // W4A16: the routing's scatter also copies every token row to its expert-sorted
        // position (one 16-byte vector per lane, all loads before the stores)
        e = mx::launch_route(router_logits, T, E, top_k, w.ids, w.weights, w.counts, w.offsets,
                             w.perm, w.inv, w.w_sorted, nullptr, w.route_tmp, x_bf16, H * 2, w.x_sorted,
                             nullptr, 0, nullptr, d->sm_count, s);
    }
    if (e != cudaSuccess) return cuda_fail(e);

    trace_mark(1, s);
    ExpertsIO io{};
    io.x_rows = w.x_sorted;
    io.x_rows_n = P;
    io.xs_codes = w.xs_codes;
    io.xs_scales = w.xs_scales;
    io.offsets = w.offsets;
    io.row_w = w.w_sorted;
    io.h = w.h;
    io.hq_codes = w.hq_codes;
    io.hq_scales = w.hq_scales;
    io.y_sorted = w.y_sorted;
    if ((st = run_experts(d, P, H, I, E, mode, w13_codes, w13_scales, w2_codes, w2_scales, io, s)) != MXFP4_OK)
        return st;

    trace_mark(3, s);
    // deterministic combine in slot order
    if ((e = mx::launch_combine(w.y_sorted, w.inv, T, top_k, H, out_bf16, d->sm_count, s)) !=
        cudaSuccess)
        return cuda_fail(e);
    trace_mark(4, s);
    return MXFP4_OK;
}

mxfp4_status mxfp4_gather_rows(const void* src, int64_t n_src, int64_t row_bytes, const int32_t* idx,
                               int64_t n, int32_t div, void* dst, void* stream) {
    if (!src || !idx || !dst) return MXFP4_ERR_INVALID_ARG;
    if (n_src <= 0 || n <= 0 || row_bytes <= 0 || div <= 0) return MXFP4_ERR_INVALID_ARG;
    if (row_bytes % 4 != 0) return MXFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(src) || !aligned16(idx) || !aligned16(dst)) return MXFP4_ERR_MISALIGNED;
    DeviceInfo* d = nullptr;
    mxfp4_status st = device_info(&d);
    if (st != MXFP4_OK) return st;
    cudaError_t e = mx::launch_gather_rows(src, n_src, row_bytes, idx, n, div, dst, d->sm_count, d->status,
                                           static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MXFP4_OK : cuda_fail(e);
}

size_t moe_mxfp4_experts_workspace_size(int64_t P, int64_t H, int64_t I, int64_t E, mxfp4_mode mode) {
    (void)E;
    if (P <= 0 || H <= 0 || I <= 0) return 0;
    return carve_experts(nullptr, P, H, I, mode).bytes;
}

mxfp4_status moe_mxfp4_experts(const void* x_sorted_bf16, int64_t P, int64_t H, const int32_t* offsets,
                               int64_t E, const uint8_t* w13_codes, const uint8_t* w13_scales, int64_t I,
                               const uint8_t* w2_codes, const uint8_t* w2_scales, const float* row_w,
                               float* y_sorted, mxfp4_mode mode, void* ws, size_t ws_bytes, void* stream) {
    if (!x_sorted_bf16 || !offsets || !w13_codes || !w13_scales || !w2_codes || !w2_scales || !row_w ||
        !y_sorted)
        return MXFP4_ERR_INVALID_ARG;
    if (P <= 0 || H <= 0 || I <= 0 || E <= 0) return MXFP4_ERR_INVALID_ARG;
    if (mode != MXFP4_W4A16 && mode != MXFP4_W4A4) return MXFP4_ERR_INVALID_ARG;
    if (E > 256 || P >= (int64_t{1} << 31)) return MXFP4_ERR_UNSUPPORTED_SHAPE;
    if (H % 64 != 0 || I % 64 != 0) return MXFP4_ERR_UNSUPPORTED_SHAPE;
    if (H > mx::max_gemm_k() || I > mx::max_gemm_k()) return MXFP4_ERR_UNSUPPORTED_SHAPE;
    if (mode == MXFP4_W4A4 && (H > mx::max_gemm_k_w4a4() || I > mx::max_gemm_k_w4a4()))
        return MXFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x_sorted_bf16) || !aligned16(offsets) || !aligned16(w13_codes) || !aligned16(w13_scales) ||
        !aligned16(w2_codes) || !aligned16(w2_scales) || !aligned16(row_w) || !aligned16(y_sorted))
        return MXFP4_ERR_MISALIGNED;
    const size_t need = moe_mxfp4_experts_workspace_size(P, H, I, E, mode);
    if (!ws || ws_bytes < need) return MXFP4_ERR_WORKSPACE;
    if (!aligned16(ws)) return MXFP4_ERR_MISALIGNED;
    DeviceInfo* d = nullptr;
    mxfp4_status st = device_info(&d);
    if (st != MXFP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const ExpertsWs w = carve_experts(ws, P, H, I, mode);
    if (mode == MXFP4_W4A4) {
        cudaError_t e = mx::launch_quantize(x_sorted_bf16, 0, P, H, w.xs_codes, w.xs_scales, MXFP4_SCALE_FLOOR,
                                            d->sm_count, d->status, s);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    ExpertsIO io{};
    io.x_rows = x_sorted_bf16;
    io.x_rows_n = P;
    io.xs_codes = w.xs_codes;
    io.xs_scales = w.xs_scales;
    io.offsets = offsets;
    io.row_w = row_w;
    io.h = w.h;
    io.hq_codes = w.hq_codes;
    io.hq_scales = w.hq_scales;
    io.y_sorted = y_sorted;
    return run_experts(d, P, H, I, E, mode, w13_codes, w13_scales, w2_codes, w2_scales, io, s);
}

mxfp4_status moe_mxfp4_combine(const float* y_sorted, const int32_t* inv, int64_t T, int32_t top_k, int64_t H,
                               void* out_bf16, void* stream) {
    if (!y_sorted || !inv || !out_bf16) return MXFP4_ERR_INVALID_ARG;
    if (T <= 0 || H <= 0 || top_k <= 0) return MXFP4_ERR_INVALID_ARG;
    if (top_k > 8 || H % 8 != 0 || T * top_k >= (int64_t{1} << 31)) return MXFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(y_sorted) || !aligned16(inv) || !aligned16(out_bf16)) return MXFP4_ERR_MISALIGNED;
    DeviceInfo* d = nullptr;
    mxfp4_status st = device_info(&d);
    if (st != MXFP4_OK) return st;
    cudaError_t e = mx::launch_combine(y_sorted, inv, T, top_k, H, out_bf16, d->sm_count,
                                       static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MXFP4_OK : cuda_fail(e);
}

mxfp4_status moe_bf16_mlp(const void* x_bf16, int64_t T, int64_t H, const float* router_logits, int64_t E,
                          int32_t top_k, const void* w13_bf16, int64_t I, const void* w2_bf16, void* out_bf16,
                          void* ws, size_t ws_bytes, void* stream) {
    mxfp4_status st = check_route_args(router_logits, T, E, top_k);
    if (st != MXFP4_OK) return st;
    if (!x_bf16 || !w13_bf16 || !w2_bf16 || !out_bf16) return MXFP4_ERR_INVALID_ARG;
    if (H <= 0 || I <= 0) return MXFP4_ERR_INVALID_ARG;
    if (H % 64 != 0 || I % 64 != 0 || H >= (int64_t{1} << 31) || I >= (int64_t{1} << 31))
        return MXFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x_bf16) || !aligned16(router_logits) || !aligned16(w13_bf16) || !aligned16(w2_bf16) ||
        !aligned16(out_bf16))
        return MXFP4_ERR_MISALIGNED;
    const size_t need = moe_bf16_workspace_size(T, H, I, E, top_k);
    if (!ws || ws_bytes < need) return MXFP4_ERR_WORKSPACE;
    if (!aligned16(ws)) return MXFP4_ERR_MISALIGNED;
    DeviceInfo* d = nullptr;
    if ((st = device_info(&d)) != MXFP4_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const MoeWs w = carve_moe(ws, T, H, I, E, top_k, MXFP4_W4A16);
    const int64_t P = T * top_k;
    trace_mark(0, s);
    cudaError_t e = mx::launch_route(router_logits, T, E, top_k, w.ids, w.weights, w.counts, w.offsets, w.perm,
                                     w.inv, w.w_sorted, nullptr, w.route_tmp, x_bf16, H * 2, w.x_sorted, nullptr,
                                     0, nullptr, d->sm_count, s);
    if (e != cudaSuccess) return cuda_fail(e);
    trace_mark(1, s);
    const int nt = mx::pick_token_tiling_bf16w(P, E);
    const int64_t tok_tiles = (P + nt - 1) / nt + E;
    // gate/up with the SwiGLU epilogue: the weight tile in 16-row boxes (gate, up interleaved)
    CUtensorMap tw, tx;
    if ((st = encode_w16_map(&tw, w13_bf16, H, 2 * I, E, 16)) != MXFP4_OK) return st;
    if ((st = encode_act_map(&tx, w.x_sorted, H, P, nt)) != MXFP4_OK) return st;
    mx::GemmArgs a{};
    a.offsets = w.offsets;
    a.G = static_cast<int>(E);
    a.K = static_cast<int>(H);
    a.rows_w = static_cast<int>(2 * I);
    a.I = static_cast<int>(I);
    a.n_ftiles = static_cast<int>(I / 64);
    a.out = w.h;
    a.out_ld = I;
    a.n_valid_feat = static_cast<int>(I);
    a.status = d->status;
    if ((e = mx::launch_grouped_gemm_bf16w(mx::EPI_SWIGLU, nt, tw, tx, a, gemm_grid(d, tok_tiles * a.n_ftiles), s)) !=
        cudaSuccess)
        return cuda_fail(e);
    trace_mark(2, s);
    // down projection, routing weight applied in fp32
    if ((st = encode_w16_map(&tw, w2_bf16, I, H, E, 128)) != MXFP4_OK) return st;
    if ((st = encode_act_map(&tx, w.h, I, P, nt)) != MXFP4_OK) return st;
    a.K = static_cast<int>(I);
    a.rows_w = static_cast<int>(H);
    a.I = 0;
    a.n_ftiles = static_cast<int>((H + 127) / 128);
    a.out = w.y_sorted;
    a.out_ld = H;
    a.n_valid_feat = static_cast<int>(H);
    a.row_w = w.w_sorted;
    if ((e = mx::launch_grouped_gemm_bf16w(mx::EPI_WEIGHTED, nt, tw, tx, a, gemm_grid(d, tok_tiles * a.n_ftiles), s)) !=
        cudaSuccess)
        return cuda_fail(e);
    trace_mark(3, s);
    if ((e = mx::launch_combine(w.y_sorted, w.inv, T, top_k, H, out_bf16, d->sm_count, s)) != cudaSuccess)
        return cuda_fail(e);
    trace_mark(4, s);
    return MXFP4_OK;
}

size_t moe_bf16_workspace_size(int64_t T, int64_t H, int64_t I, int64_t E, int32_t top_k) {
    return moe_mxfp4_workspace_size(T, H, I, E, top_k, MXFP4_W4A16);
}

// ---------------------------------------------------------------- allocation-free MoE layer
// Scratch of moe_mxfp4_mlp_noalloc: a fixed array in device memory, set aside on every
// GPU that loads this library until the process exits.  Host code may not use the
// array's name as a device address; the address is looked up once per device below.
static __device__ __align__(256) unsigned char g_moe_noalloc_scratch[MXFP4_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_noalloc_mutex;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (queried on first use).
mxfp4_status noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return MXFP4_ERR_ARCH;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_moe_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e);
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return MXFP4_OK;
}
}  // namespace

mxfp4_status moe_mxfp4_mlp_noalloc(const void* x_bf16, int64_t T, int64_t H,
                                   const float* router_logits, int64_t E, int32_t top_k,
                                   const uint8_t* w13_codes, const uint8_t* w13_scales, int64_t I,
                                   const uint8_t* w2_codes, const uint8_t* w2_scales,
                                   void* out_bf16, mxfp4_mode mode, void* stream) {
    mxfp4_status st = check_route_args(router_logits, T, E, top_k);
    if (st != MXFP4_OK) return st;
    if (H <= 0 || I <= 0) return MXFP4_ERR_INVALID_ARG;
    if (moe_mxfp4_workspace_size(T, H, I, E, top_k, mode) > MXFP4_NOALLOC_SCRATCH_BYTES)
        return MXFP4_ERR_WORKSPACE;
    DeviceInfo* d = nullptr;
    if ((st = device_info(&d)) != MXFP4_OK) return st;
    void* ws = nullptr;
    if ((st = noalloc_scratch(&ws)) != MXFP4_OK) return st;
    // Every scratch byte a result depends on is written earlier in the same call, so
    // the previous call's leftovers need no clearing.  The one exception is read but
    // never used: in W4A4, the GEMM stages a token tile's scales with one bulk copy of
    // the 16-byte-aligned range that covers them, which takes in up to 16 bytes past
    // the end of an activation-scale array (the tail the carving keeps readable); no
    // kernel writes that tail, and the scale bytes past a tile's rows never reach an
    // MMA, so whatever an earlier call left there cannot change the output.
    return moe_mxfp4_mlp(x_bf16, T, H, router_logits, E, top_k, w13_codes, w13_scales, I,
                         w2_codes, w2_scales, out_bf16, mode, ws, MXFP4_NOALLOC_SCRATCH_BYTES,
                         stream);
}

}  // extern "C"
