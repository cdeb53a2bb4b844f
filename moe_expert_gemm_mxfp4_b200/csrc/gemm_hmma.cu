// Grouped MXFP4-weight GEMM (W4A16) for small token groups (decode): the same
// operation and epilogues as gemm.cu,
//     D_g = X_g . dequant(W_g)^T,  fp32 accumulation,  PLAIN / SWIGLU / WEIGHTED,
// for groups of at most 32 activation rows, on the warp-level tensor-core MMA
// (mma.sync m16n8k16, bf16 operands, fp32 accumulators in registers).
//
// Why not tcgen05 here: with 8 to 32 token rows per expert the weights are used
// by only a few tokens, so the layer streams weights from HBM and the MMA work
// per weight byte is tiny.  A tcgen05.mma of N <= 64 costs about 45 cycles
// whatever its N, and 74 while dequantizing warps store into TMEM; with the
// weights as its 128-row A operand that caps the weight stream at about 0.67 of
// HBM, and a barrier wait in the issuing thread costs ~200 cycles more at N = 16
// (measured on this GPU).  mma.sync takes its A operand from registers, so the
// dequantized weights go from the LUT straight into A fragments: no TMEM, no
// shared-memory copy of the bf16 weights, no single issuing thread.
//
// Layout trick: the products of an MMA only need A and B to agree on which K
// element sits at each of the MMA's 16 K positions.  Thread (g = lane / 4, t =
// lane % 4) loads the 32-bit word t of a row's 16 code bytes (32 K values: K
// 8t .. 8t+7) and uses its bytes 0-1 as the A fragment of a first MMA and bytes
// 2-3 as that of a second one; it loads the same K range of its token row as one
// 16-byte vector (B fragments of both MMAs).  Each code byte dequantizes to one
// bf16x2 A register with the shared LUT of gemm.cu (one prmt, one ld.shared, one
// exact bf16x2 multiply by the block scale).
//
// Work tile: 128 weight rows x NT (16 or 32) token rows of one group.  Warp w
// (0..3) owns 32 weight rows as two m16 blocks; for SWIGLU block 0 holds gate
// features 16w .. 16w+15 of the tile and block 1 the matching up features, so each
// thread pairs gate and up in its own registers.  Warp 4 streams, per 256-wide K
// stage, the packed codes of the tile's rows (TMA, 128 B per row, 128B swizzle)
// and the stage's activation rows (TMA, four [NT x 64] bf16 boxes, 128B swizzle)
// into a ring, plus the tile's block scales (bulk copy, double-buffered).  Every
// wait is bounded (MXFP4_ERR_TIMEOUT in the status word).
#include "gemm_common.cuh"

namespace mx {

namespace {

using namespace gemm;

constexpr int kHWarps = 4;                        // compute warps
constexpr int kHThreads = (kHWarps + 1) * 32;     // + the producer warp
constexpr int kHSSK = 256;                        // K per stage
constexpr int kHCodeRow = kHSSK / 2;              // 128 code bytes per weight row per stage
constexpr int kHCodes = kBM * kHCodeRow;          // 16 KB
constexpr int kHMaxStages = 8;
constexpr int kHSmemLimit = 227 * 1024;
constexpr int kHWindowBase = 1024;                // shared-window address of dynamic smem
constexpr int kHLutOff = 65536 - kHWindowBase;    // LUT at window address 64 KB (see gemm.cu)
constexpr int kHLutBytes = 256 * 256;

struct HLayout {
    int stage_bytes, bar_off, tstart_off, off_off, misc_off, scales_off, scale_bytes;
    int n_lo, lo_off, n_hi, hi_off, total;
};

// Barriers, tables and the tile scales below the LUT, then as many stages as fit
// below it; the rest of the stages above it.
__host__ __device__ inline HLayout make_hlayout(int nt, int K) {
    HLayout L;
    L.stage_bytes = kHCodes + nt * kHSSK * 2;
    L.bar_off = 0;
    L.tstart_off = L.bar_off + (2 * kHMaxStages + 4 + 1) * 8;
    L.off_off = L.tstart_off + (kMaxGroups + 1) * 4;
    L.misc_off = L.off_off + (kMaxGroups + 1) * 4;
    L.scales_off = (L.misc_off + 16 + 127) / 128 * 128;
    L.scale_bytes = (kBM * (K / 32) + 127) / 128 * 128;
    L.lo_off = (L.scales_off + 2 * L.scale_bytes + 1023) / 1024 * 1024;
    L.n_lo = L.lo_off + L.stage_bytes <= kHLutOff ? (kHLutOff - L.lo_off) / L.stage_bytes : 0;
    L.hi_off = kHLutOff + kHLutBytes;
    L.n_hi = (kHSmemLimit - L.hi_off) / L.stage_bytes;
    if (L.n_lo + L.n_hi > kHMaxStages) L.n_hi = kHMaxStages - L.n_lo;
    L.total = L.hi_off + L.n_hi * L.stage_bytes;
    return L;
}

__device__ __forceinline__ uint32_t hbmul2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t hlds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint32_t hlds_u8(uint32_t addr) {
    uint16_t v;
    asm volatile("ld.shared.u8 %0, [%1];" : "=h"(v) : "r"(addr));
    return v;
}

// Code byte j of `w` -> bf16x2 of its two E2M1 values times 2^(S-127), exact: the
// LUT's magnitude pair times the bf16 scale (fast path S in [2, 254]; otherwise
// through fp32, where the products can be subnormal or NaN).
__device__ __forceinline__ uint32_t deq_byte(uint32_t w, int j, uint32_t S, uint32_t lut_lane) {
    if (S - 2u <= 252u)
        return hbmul2(hlds32(prmt(w, lut_lane, 0x7604u | (j << 4))), S * 0x00800080u);
    return dequant_byte_exact((w >> (8 * j)) & 0xFFu, e8m0_f32(S));
}

__device__ __forceinline__ void hmma16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int NT, int MODE>
__global__ void __launch_bounds__(kHThreads, 1)
grouped_w4a16_hmma_kernel(const __grid_constant__ CUtensorMap tmap_w,
                          const __grid_constant__ CUtensorMap tmap_x, const GemmArgs args) {
    constexpr int NTILES = NT / 8;
    constexpr int kActBox = NT * 128;            // one [NT x 64] bf16 box
    const HLayout Ly = make_hlayout(NT, args.K);
    const int S = Ly.n_lo + Ly.n_hi;
    extern __shared__ __align__(1024) uint8_t smem[];
    if (smem_u32(smem) != kHWindowBase) {         // the LUT addressing needs this base
        if (threadIdx.x == 0) record_status(args.status, MXFP4_ERR_CUDA);
        return;
    }
    auto stage_ptr = [&](int i) {
        return i < Ly.n_lo ? smem + Ly.lo_off + i * Ly.stage_bytes : smem + Ly.hi_off + (i - Ly.n_lo) * Ly.stage_bytes;
    };
    uint32_t* lut = reinterpret_cast<uint32_t*>(smem + kHLutOff);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Ly.bar_off);
    uint64_t* full = bars;                      // stage landed (TMA tx)
    uint64_t* empty = bars + kHMaxStages;       // stage read (4 compute warps)
    uint64_t* sfull = empty + kHMaxStages;      // tile scales staged (tx), double-buffered
    uint64_t* sempty = sfull + 2;               // tile scales released (4 compute warps)
    int* s_tstart = reinterpret_cast<int*>(smem + Ly.tstart_off);
    int* s_off = reinterpret_cast<int*>(smem + Ly.off_off);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + Ly.misc_off);
    volatile int* s_never = reinterpret_cast<volatile int*>(smem + Ly.misc_off + 4);
    uint8_t* scales = smem + Ly.scales_off;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = args.offsets ? args.G : 1;
    const int kb = args.K / 32;
    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kHWarps);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sfull[b], 1);
            mbar_init(&sempty[b], kHWarps);
        }
        *s_abort = 0;
        *s_never = 0;
        fence_mbar_init();
        prefetch_tmap(&tmap_w);
        prefetch_tmap(&tmap_x);
    }
    for (int i = tid; i <= G; i += kHThreads)
        s_off[i] = args.offsets ? args.offsets[i] : (i == 0 ? 0 : args.m_single);
    for (int i = tid; i < 256 * 32; i += kHThreads) {
        const uint32_t b = static_cast<uint32_t>(i >> 5);
        lut[(b << 6) | (i & 31)] = e2m1_bf16(b & 15u) | (e2m1_bf16(b >> 4) << 16);
    }
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
    __syncthreads();
    const int total_tiles = s_tstart[G];
    const int nss = (args.K + kHSSK - 1) / kHSSK;
    // CTAs start their tiles' K loop at different stages, so that CTAs reading the same
    // activation rows at the same time touch different lines
    const int rot = static_cast<int>(blockIdx.x % static_cast<unsigned>(nss));

    if (warp == kHWarps) {
        // ---------------- producer
        if (lane == 0) {
            int lt = 0, issued = 0, it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++lt) {
                const TileInfo ti = decode_tile(t, s_tstart, s_off, G, NT);
                const int sb = lt & 1;
                if (!mbar_wait(&sempty[sb], ((lt >> 1) & 1) ^ 1, s_abort)) { ok = false; break; }
                uint8_t* sdst = scales + sb * Ly.scale_bytes;
                const uint8_t* gsc = args.w_scales + static_cast<int64_t>(ti.g) * args.rows_w * kb;
                uint32_t tx = 0;
                if (MODE == EPI_SWIGLU) {
                    tx += stage_scales(sdst, gsc + static_cast<int64_t>(ti.f * 64) * kb, 64, kb, &sfull[sb]);
                    tx += stage_scales(sdst + 64 * kb, gsc + static_cast<int64_t>(args.I + ti.f * 64) * kb, 64, kb,
                                       &sfull[sb]);
                } else {
                    const int rows = min(kBM, args.rows_w - ti.f * kBM);
                    tx += stage_scales(sdst, gsc + static_cast<int64_t>(ti.f * kBM) * kb, rows, kb, &sfull[sb]);
                }
                mbar_arrive_expect_tx(&sfull[sb], tx);
                for (int si = 0; si < nss; ++si, ++it) {
                    const int ss = si + rot < nss ? si + rot : si + rot - nss;
                    const int s = it % S;
                    if (!mbar_wait(&empty[s], ((it / S) & 1) ^ 1, s_abort)) { ok = false; break; }
                    uint8_t* dst = stage_ptr(s);
                    mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(Ly.stage_bytes));
                    // codes: 128 B of each weight row (past K/2 the TMA fills zeros)
                    const int x = ss * kHCodeRow;
                    if (MODE == EPI_SWIGLU) {
                        tma_load_3d(dst, &tmap_w, &full[s], x, ti.f * 64, ti.g);
                        tma_load_3d(dst + 64 * kHCodeRow, &tmap_w, &full[s], x, args.I + ti.f * 64, ti.g);
                    } else {
                        tma_load_3d(dst, &tmap_w, &full[s], x, ti.f * kBM, ti.g);
                    }
                    // activations: NT rows from row0, four boxes of 64 K (past K: zeros)
#pragma unroll
                    for (int b = 0; b < 4; ++b)
                        tma_load_2d(dst + kHCodes + b * kActBox, &tmap_x, &full[s], ss * kHSSK + 64 * b, ti.row0);
                    ++issued;
                }
            }
            if (!ok) {
                *s_abort = 1;
                record_status(args.status, MXFP4_ERR_TIMEOUT);
                // let the copies already issued land before the CTA exits
                for (int i = issued > S ? issued - S : 0; i < issued; ++i)
                    mbar_wait(&full[i % S], (i / S) & 1, s_never);
                for (int l2 = lt - 1; l2 <= lt && l2 >= 0; ++l2)
                    mbar_wait(&sfull[l2 & 1], (l2 >> 1) & 1, s_never);
            }
        }
        return;
    }

    // ---------------- compute warps
    const int g = lane >> 2, t4 = lane & 3;
    const uint32_t lut_lane = smem_u32(lut) + lane * 4;
    // staged weight rows of this thread: block b, rows r and r + 8
    int srow[2];
    if (MODE == EPI_SWIGLU) {
        srow[0] = 16 * warp + g;          // gate features 16w + g (+8)
        srow[1] = 64 + 16 * warp + g;     // the matching up features
    } else {
        srow[0] = 32 * warp + g;
        srow[1] = 32 * warp + 16 + g;
    }
    int lt = 0, it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++lt) {
        const TileInfo ti = decode_tile(t, s_tstart, s_off, G, NT);
        // rows past the weight matrix (last feature tile) use scale 1.0 on their zero codes
        bool valid[2][2];
#pragma unroll
        for (int b = 0; b < 2; ++b)
#pragma unroll
            for (int h = 0; h < 2; ++h)
                valid[b][h] = MODE == EPI_SWIGLU || ti.f * kBM + srow[b] + 8 * h < args.rows_w;
        const int sb = lt & 1;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sfull[sb], (lt >> 1) & 1, s_abort))) { ok = false; break; }
        const uint32_t sc_base = smem_u32(scales + sb * Ly.scale_bytes);
        float acc[2][NTILES][4];
#pragma unroll
        for (int b = 0; b < 2; ++b)
#pragma unroll
            for (int n = 0; n < NTILES; ++n)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[b][n][i] = 0.f;
        for (int si = 0; si < nss; ++si, ++it) {
            const int ss = si + rot < nss ? si + rot : si + rot - nss;
            const int s = it % S;
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&full[s], (it / S) & 1, s_abort))) { ok = false; break; }
            const uint32_t cbase = smem_u32(stage_ptr(s));
            const uint32_t abase = cbase + kHCodes;
            const int nch = min(8, kb - ss * 8);          // 32-wide K blocks inside K
#pragma unroll 2
            for (int j = 0; j < nch; ++j) {
                const int kblk = ss * 8 + j;
                // A: code words (rows r, r + 8 of both blocks) and their block scales
                uint32_t w[2][2], S8[2][2];
#pragma unroll
                for (int b = 0; b < 2; ++b)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int r = srow[b] + 8 * h;
                        w[b][h] = hlds32(cbase + r * kHCodeRow + (((j ^ (r & 7)) << 4) | (t4 << 2)));
                        S8[b][h] = valid[b][h] ? hlds_u8(sc_base + r * kb + kblk) : 127u;
                    }
                uint32_t a[2][2][4];   // [block][mma of the pair][fragment register]
#pragma unroll
                for (int b = 0; b < 2; ++b)
#pragma unroll
                    for (int m = 0; m < 2; ++m) {
                        a[b][m][0] = deq_byte(w[b][0], 2 * m, S8[b][0], lut_lane);
                        a[b][m][1] = deq_byte(w[b][1], 2 * m, S8[b][1], lut_lane);
                        a[b][m][2] = deq_byte(w[b][0], 2 * m + 1, S8[b][0], lut_lane);
                        a[b][m][3] = deq_byte(w[b][1], 2 * m + 1, S8[b][1], lut_lane);
                    }
                // B: token rows n*8 + g, K 8t .. 8t+7 of this block (box j/2, chunk (j%2)*4 + t)
#pragma unroll
                for (int n = 0; n < NTILES; ++n) {
                    const int row = n * 8 + g;
                    const uint32_t c = static_cast<uint32_t>((j & 1) * 4 + t4);
                    const uint4 v = lds128(abase + (j >> 1) * kActBox + row * 128 + ((c ^ (row & 7)) << 4));
#pragma unroll
                    for (int b = 0; b < 2; ++b) {
                        hmma16816(acc[b][n], a[b][0][0], a[b][0][1], a[b][0][2], a[b][0][3], v.x, v.y);
                        hmma16816(acc[b][n], a[b][1][0], a[b][1][1], a[b][1][2], a[b][1][3], v.z, v.w);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
        if (!ok) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[sb]);
        // ---------------- epilogue: c0 (row g, token 2t), c1 (g, 2t+1), c2 (g+8, 2t), c3 (g+8, 2t+1)
#pragma unroll
        for (int n = 0; n < NTILES; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int tok = n * 8 + 2 * t4 + (i & 1);
                if (tok >= ti.mrows) continue;
                const int m = g + 8 * (i >> 1);
                const int64_t orow = static_cast<int64_t>(ti.row0 + tok) * args.out_ld;
                if (MODE == EPI_SWIGLU) {
                    const int feat = ti.f * 64 + 16 * warp + m;
                    store_bf16(args.out, orow + feat, silu_f32(acc[0][n][i]) * acc[1][n][i]);
                } else {
#pragma unroll
                    for (int b = 0; b < 2; ++b) {
                        const int feat = ti.f * kBM + 32 * warp + 16 * b + m;
                        if (feat < args.n_valid_feat) {
                            if (MODE == EPI_WEIGHTED)   // fp32 out: one rounding, in the combine
                                reinterpret_cast<float*>(args.out)[orow + feat] = acc[b][n][i] * args.row_w[ti.row0 + tok];
                            else
                                store_bf16(args.out, orow + feat, acc[b][n][i]);
                        }
                    }
                }
            }
    }
    if (!ok) {
        *s_abort = 1;
        record_status(args.status, MXFP4_ERR_TIMEOUT);
    }
}

template <int NT, int MODE>
cudaError_t launch_h(const CUtensorMap& tw, const CUtensorMap& tx, const GemmArgs& a, int grid,
                     cudaStream_t stream) {
    const HLayout L = make_hlayout(NT, a.K);
    if (L.n_lo + L.n_hi < 2) return cudaErrorInvalidConfiguration;
    auto kern = grouped_w4a16_hmma_kernel<NT, MODE>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
    if (err != cudaSuccess) return err;
    kern<<<grid, kHThreads, L.total, stream>>>(tw, tx, a);
    return cudaGetLastError();
}

template <int MODE>
cudaError_t launch_h_mode(int nt, const CUtensorMap& tw, const CUtensorMap& tx, const GemmArgs& a, int grid,
                          cudaStream_t stream) {
    return nt == 16 ? launch_h<16, MODE>(tw, tx, a, grid, stream) : launch_h<32, MODE>(tw, tx, a, grid, stream);
}

}  // namespace

// Token rows per work tile of the small-group engine (16 or 32), or 0 when the
// groups are too large for it (average rows per group above 32).
int pick_token_tiling_hmma(int64_t rows, int64_t groups) {
    const int64_t avg = (rows + groups - 1) / (groups > 0 ? groups : 1);
    if (avg <= 16) return 16;
    if (avg <= 32) return 32;
    return 0;
}

// Largest K the small-group engine takes (the tile scales share the space below
// the LUT with at least the ring's minimum).
bool hmma_fits_k(int64_t K) {
    if (K <= 0 || K % 64 != 0) return false;
    const HLayout a = make_hlayout(32, static_cast<int>(K));
    return a.n_lo + a.n_hi >= 2 && a.scales_off + 2 * a.scale_bytes <= kHLutOff;
}

// Host launcher.  `tmap_w` as for the tcgen05 engine (codes {K/2, rows_w, G}, box
// {128, 64 (SWIGLU) or 128, 1}, 128B swizzle); `tmap_x` the activations {K, rows}
// with box {64, nt} and 128B swizzle.
cudaError_t launch_grouped_gemm_hmma(int mode, int nt, const CUtensorMap& tmap_w, const CUtensorMap& tmap_x,
                                     const GemmArgs& args, int grid, cudaStream_t stream) {
    if (nt != 16 && nt != 32) return cudaErrorInvalidValue;
    switch (mode) {
        case EPI_SWIGLU: return launch_h_mode<EPI_SWIGLU>(nt, tmap_w, tmap_x, args, grid, stream);
        case EPI_WEIGHTED: return launch_h_mode<EPI_WEIGHTED>(nt, tmap_w, tmap_x, args, grid, stream);
        default: return launch_h_mode<EPI_PLAIN>(nt, tmap_w, tmap_x, args, grid, stream);
    }
}

}  // namespace mx
