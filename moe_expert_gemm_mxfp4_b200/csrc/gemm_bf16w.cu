// Grouped bf16-weight GEMM on sm_100a tensor cores: the comparison engine for the
// MXFP4 one.  The pages' fallback runs the same expert MLP on bf16 weights at about
// four times the memory (agentlenshq.com, "Transformers 4.40 performance upgrades
// for OpenAI GPT-OSS ...", sections "Native Support in transformers" and "Memory
// Savings"); this engine runs that layer on this GPU, so that the two weight formats
// are measured side by side on the same tiles and epilogues:
//     D_g = X_g . W_g^T,  W_g bf16 [rows_w, K],  fp32 accumulation,
//     PLAIN / SWIGLU / WEIGHTED epilogues of gemm_common.cuh.
//
// With no dequantization both operands go through TMA into shared memory (128B
// swizzle, the UMMA K-major layout) and the MMA is the all-shared-memory form:
// tcgen05.mma kind::f16, M = 128 weight rows, N = NT token rows (64, 128 or 256),
// K = 16.  For SWIGLU the weight tile is loaded as eight 16-row boxes (gate rows
// 16q.. at tile rows 32q.., up rows at 32q + 16..), the TMEM lane order the SwiGLU
// epilogue pairs by.  Roles (one persistent CTA per SM): warp 0 TMA producer, warp 1
// MMA issuer (one commit per stage releases it, one per tile hands the accumulator
// to the epilogue), warps 4-7 epilogue; accumulators double-buffered in TMEM.  Every
// wait is bounded (MXFP4_ERR_TIMEOUT in the status word).
#include "gemm_common.cuh"

namespace mx {

namespace {

using namespace gemm;

constexpr int kBThreads = 256;
constexpr int kBBK = 64;                       // K per stage
constexpr int kBWBytes = kBM * kBBK * 2;       // weight tile of a stage (16 KB)
constexpr int kBMaxStages = 8;
constexpr int kBSmemLimit = 227 * 1024;
constexpr int kBNumBars = 2 * kBMaxStages + 2 + 2 + 1;

struct BLayout {
    int stage_bytes, stages, bar_off, tstart_off, off_off, misc_off, total;
};

__host__ __device__ inline BLayout make_blayout(int nt) {
    BLayout L;
    L.stage_bytes = kBWBytes + nt * kBBK * 2;
    const int fixed = kBNumBars * 8 + 2 * (kMaxGroups + 1) * 4 + 16 + 1024;
    L.stages = (kBSmemLimit - fixed) / L.stage_bytes;
    if (L.stages > kBMaxStages) L.stages = kBMaxStages;
    L.bar_off = L.stages * L.stage_bytes;
    L.tstart_off = L.bar_off + kBNumBars * 8;
    L.off_off = L.tstart_off + (kMaxGroups + 1) * 4;
    L.misc_off = L.off_off + (kMaxGroups + 1) * 4;
    L.total = L.misc_off + 16 + 1024;   // + slack for the 1024-B alignment of the base
    return L;
}

template <int NT, int MODE>
__global__ void __launch_bounds__(kBThreads, 1)
grouped_bf16w_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                     const GemmArgs args) {
    constexpr uint32_t kTmemCols = 2 * NT < 32 ? 32 : 2 * NT;
    constexpr int CW = NT < 32 ? NT : 32;
    const BLayout Ly = make_blayout(NT);
    const int S = Ly.stages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Ly.bar_off);
    uint64_t* full = bars;                         // stage landed (TMA tx)
    uint64_t* empty = bars + kBMaxStages;          // stage consumed (MMA commit)
    uint64_t* accfull = bars + 2 * kBMaxStages;    // accumulators ready (MMA commit)
    uint64_t* accempty = accfull + 2;              // accumulators drained (128 epilogue threads)
    uint64_t* drain = accempty + 2;
    static_assert(2 * kBMaxStages + 2 + 2 + 1 == kBNumBars, "barrier block size");
    int* s_tstart = reinterpret_cast<int*>(smem + Ly.tstart_off);
    int* s_off = reinterpret_cast<int*>(smem + Ly.off_off);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + Ly.misc_off);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + Ly.misc_off + 4);
    volatile int* s_never = reinterpret_cast<volatile int*>(smem + Ly.misc_off + 8);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = args.offsets ? args.G : 1;

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accfull[b], 1);
            mbar_init(&accempty[b], 128);
        }
        mbar_init(drain, 1);
        *s_abort = 0;
        *s_never = 0;
        fence_mbar_init();
        prefetch_tmap(&tmap_w);
        prefetch_tmap(&tmap_x);
    }
    if (warp == 1) {
        tmem_alloc(s_tmem, kTmemCols);
        tmem_relinquish();
    }
    for (int i = tid; i <= G; i += kBThreads)
        s_off[i] = args.offsets ? args.offsets[i] : (i == 0 ? 0 : args.m_single);
    __syncthreads();
    if (tid == 0) {
        int acc = 0;
        for (int g = 0; g < G; ++g) {
            s_tstart[g] = acc;
            const int m = s_off[g + 1] - s_off[g];
            acc += ((m + NT - 1) / NT) * args.n_ftiles;
        }
        s_tstart[G] = acc;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;
    const int total_tiles = s_tstart[G];
    const int nk = args.K / kBBK;
    // CTAs start their K loop at different stages (fewer CTAs on the same lines at once)
    const int rot = static_cast<int>(blockIdx.x % static_cast<unsigned>(nk));

    if (warp == 0) {
        // ---------------- producer
        if (lane == 0) {
            RingPos c;
            int issued = 0;
            bool ok = true;
            const uint32_t bytes = static_cast<uint32_t>(Ly.stage_bytes);
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
                const TileInfo ti = decode_tile(t, s_tstart, s_off, G, NT);
                for (int i = 0; i < nk; ++i) {
                    const int ks = i + rot < nk ? i + rot : i + rot - nk;
                    if (!mbar_wait(&empty[c.idx], c.ph ^ 1, s_abort)) { ok = false; break; }
                    uint8_t* dst = smem + c.idx * Ly.stage_bytes;
                    mbar_arrive_expect_tx(&full[c.idx], bytes);
                    const int x = ks * kBBK;
                    if (MODE == EPI_SWIGLU) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            tma_load_3d(dst + (32 * q) * 128, &tmap_w, &full[c.idx], x, ti.f * 64 + 16 * q, ti.g);
                            tma_load_3d(dst + (32 * q + 16) * 128, &tmap_w, &full[c.idx], x,
                                        args.I + ti.f * 64 + 16 * q, ti.g);
                        }
                    } else {
                        tma_load_3d(dst, &tmap_w, &full[c.idx], x, ti.f * kBM, ti.g);
                    }
                    tma_load_2d(dst + kBWBytes, &tmap_x, &full[c.idx], x, ti.row0);
                    c.next(S);
                    ++issued;
                }
            }
            if (!ok) {
                *s_abort = 1;
                record_status(args.status, MXFP4_ERR_TIMEOUT);
                // let the copies already issued land before the CTA exits
                RingPos r;
                const int first = issued > S ? issued - S : 0;
                for (int i = 0; i < issued; ++i) {
                    if (i >= first) mbar_wait(&full[r.idx], r.ph, s_never);
                    r.next(S);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kBM, NT);
            RingPos c;
            int lt = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++lt) {
                const int b = lt & 1;
                if (!mbar_wait(&accempty[b], ((lt >> 1) & 1) ^ 1, s_abort)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + b * NT;
                for (int i = 0; i < nk; ++i) {
                    if (!mbar_wait(&full[c.idx], c.ph, s_abort)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t wa = smem_u32(smem + c.idx * Ly.stage_bytes);
                    const uint32_t xa = wa + kBWBytes;
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        mma_bf16_ss(d_tmem, sw128_desc(wa + 32 * j), sw128_desc(xa + 32 * j), idesc,
                                    (i | j) != 0 ? 1u : 0u);
                    tc_commit(&empty[c.idx]);
                    c.next(S);
                }
                if (!ok) break;
                tc_commit(&accfull[b]);
            }
            if (!ok) {
                *s_abort = 1;
                record_status(args.status, MXFP4_ERR_TIMEOUT);
            }
            // every MMA issued by this thread completes before TMEM is released
            tc_commit(drain);
            mbar_wait(drain, 0, s_never);
        }
    } else if (warp >= 4) {
        // ---------------- epilogue warpgroup (TMEM lane quarter q = warp & 3)
        const int q = warp & 3;
        int lt = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++lt) {
            const TileInfo ti = decode_tile(t, s_tstart, s_off, G, NT);
            const int b = lt & 1;
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&accfull[b], (lt >> 1) & 1, s_abort))) { ok = false; break; }
            tc_fence_after();
            const uint32_t t_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + b * NT;
            epilogue_tile<MODE, CW, NT>(args, ti, t_base, q, lane);
            tc_fence_before();
            mbar_arrive(&accempty[b]);
        }
        if (!ok) {
            *s_abort = 1;
            record_status(args.status, MXFP4_ERR_TIMEOUT);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

template <int NT, int MODE>
cudaError_t launch_b(const CUtensorMap& tw, const CUtensorMap& tx, const GemmArgs& a, int grid,
                     cudaStream_t stream) {
    const BLayout L = make_blayout(NT);
    if (L.stages < 2) return cudaErrorInvalidConfiguration;
    auto kern = grouped_bf16w_kernel<NT, MODE>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
    if (err != cudaSuccess) return err;
    kern<<<grid, kBThreads, L.total, stream>>>(tw, tx, a);
    return cudaGetLastError();
}

template <int MODE>
cudaError_t launch_b_mode(int nt, const CUtensorMap& tw, const CUtensorMap& tx, const GemmArgs& a, int grid,
                          cudaStream_t stream) {
    if (nt == 64) return launch_b<64, MODE>(tw, tx, a, grid, stream);
    if (nt == 128) return launch_b<128, MODE>(tw, tx, a, grid, stream);
    return launch_b<256, MODE>(tw, tx, a, grid, stream);
}

}  // namespace

// Token rows per work tile of the bf16-weight engine for `rows` rows over `groups`.
int pick_token_tiling_bf16w(int64_t rows, int64_t groups) {
    const int64_t avg = (rows + groups - 1) / (groups > 0 ? groups : 1);
    if (avg <= 64) return 64;
    if (avg <= 160) return 128;
    return 256;
}

// Host launcher.  `tmap_w` covers the bf16 weights as {K, rows_w, G} with box
// {64, 16 (SWIGLU) or 128, 1}; `tmap_x` the activations {K, rows} with box {64, nt};
// both 128B-swizzled.
cudaError_t launch_grouped_gemm_bf16w(int mode, int nt, const CUtensorMap& tmap_w, const CUtensorMap& tmap_x,
                                      const GemmArgs& args, int grid, cudaStream_t stream) {
    if (nt != 64 && nt != 128 && nt != 256) return cudaErrorInvalidValue;
    switch (mode) {
        case EPI_SWIGLU: return launch_b_mode<EPI_SWIGLU>(nt, tmap_w, tmap_x, args, grid, stream);
        case EPI_WEIGHTED: return launch_b_mode<EPI_WEIGHTED>(nt, tmap_w, tmap_x, args, grid, stream);
        default: return launch_b_mode<EPI_PLAIN>(nt, tmap_w, tmap_x, args, grid, stream);
    }
}

}  // namespace mx
