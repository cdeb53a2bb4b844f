// Grouped MXFP4-weight GEMM (W4A16) on sm_100a tensor cores.
//
// Computes, for every group g (an expert) and its rows of activations
// X_g [m_g, K] (bf16, rows offsets[g] .. offsets[g+1] of one matrix),
//     D_g = X_g . dequant(W_g)^T          W_g = MXFP4 codes [rows_w, K/2] + E8M0 scales
// with fp32 accumulation, and applies one of three fused epilogues:
//   PLAIN     y = bf16(D)
//   SWIGLU    h = bf16(SiLU(D_gate) * D_up), W rows [0, I) gate and [I, 2I) up
//   WEIGHTED  y = w_row * D (fp32 out), w_row = the routing weight of the row
// (the gpt-oss expert MLP run on MXFP4 weights; agentlenshq.com, "Transformers
// 4.40 performance upgrades for OpenAI GPT-OSS ...", sections "What MXFP4 Is"
// and "Zero-Build Kernels from the Hub").
//
// Data flow (one persistent CTA per SM, 16 warps):
//   warp 0        TMA producer: per tile, the block scales of its 128 weight
//                 rows (bulk copy, double-buffered across tiles); per 64-wide K
//                 stage, the packed codes of the 128 rows (32 B per row,
//                 32B-swizzled) and the bf16 activation tile [NT x 64]
//                 (128B-swizzled) -> smem ring.
//   warps 4..11   two dequant warpgroups (alternate stages): each thread owns
//                 one weight row; codes -> bf16 through a 256-entry shared LUT
//                 (lane-replicated, conflict-free) times the block scale 2^(S-127)
//                 (exact bf16 product), stored with tcgen05.st into TMEM: the
//                 dequantized weights are the MMA's A operand and never touch
//                 shared memory.
//   warp 1        MMA issuer: tcgen05.mma kind::f16, M = 128 weight rows,
//                 N = NT tokens, K = 16 per instruction, A from TMEM, B from
//                 smem, D (fp32) in TMEM, double-buffered across tiles.
//   warps 12..15  epilogue: tcgen05.ld of the accumulator, fused epilogue,
//                 stores.
// TMEM: columns [0, 2*NT) the two accumulators, [256, 512) eight A slots.
// Every mbarrier wait is time-bounded (MXFP4_ERR_TIMEOUT in the status word).
#include "common.cuh"
#include "internal.h"

namespace mx {

namespace {

constexpr int kThreads = 512;
constexpr int kBM = 128;            // weight rows per tile (MMA M)
constexpr int kBK = 64;             // K per pipeline stage
constexpr int kASlots = 8;          // TMEM A-operand slots (32 columns each)
constexpr int kACol0 = 256;         // first TMEM column of the A slots
constexpr int kCodeBytes = kBM * kBK / 2;
constexpr int kLutBytes = 256 * 256;
constexpr int kMaxGroups = 256;
constexpr int kXbufBytes = 2 * 2 * 32 * 16 * 4;
constexpr int kSmemLimit = 227 * 1024;

template <int NT>
struct Cfg {
    static constexpr int kActBytes = NT * kBK * 2;
    static constexpr int kStageBytes = kCodeBytes + kActBytes;
    static constexpr int kMaxStages = NT == 16 ? 16 : (NT == 32 ? 12 : (NT == 64 ? 8 : 5));
    static_assert(kStageBytes % 1024 == 0, "stage must keep 1024-B alignment");
    static_assert(2 * NT <= kACol0, "accumulators overlap the A slots");
};

// Shared-memory layout, identical on host (sizing) and device.
struct Layout {
    int stages_off, scales_off, scale_bytes, xbuf_off, bar_off, tstart_off, off_off, misc_off, total;
};

__host__ __device__ inline Layout make_layout(int stage_bytes, int stages, int K) {
    Layout L;
    L.stages_off = kLutBytes;
    L.scales_off = L.stages_off + stages * stage_bytes;
    L.scale_bytes = ((kBM * (K / 32)) + 127) / 128 * 128;
    L.xbuf_off = L.scales_off + 2 * L.scale_bytes;
    L.bar_off = L.xbuf_off + kXbufBytes;
    const int n_bars = 2 * 16 + 2 * kASlots + 4 + 4 + 1;
    L.tstart_off = L.bar_off + n_bars * 8;
    L.off_off = L.tstart_off + (kMaxGroups + 1) * 4;
    L.misc_off = L.off_off + (kMaxGroups + 1) * 4;
    L.total = L.misc_off + 16 + 1024;   // + slack for the 1024-B alignment of the base
    return L;
}

__device__ __forceinline__ uint32_t bmul2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

// 16 code bytes (32 weights of one K block) -> 16 bf16x2 words.
// Fast path (S in [2, 254]): LUT value times 2^(S-127) as one bf16x2 multiply,
// exact because both factors and the product are normal bf16 numbers (or the
// product overflows to Inf, as round-to-nearest-even does).  Otherwise the
// exact fp32 route (subnormal results for S <= 1, NaN for S = 255).
// LUT entry (b, lane) sits at lut_base + b * 256 + lane * 4; lut_lane is
// lut_base + lane * 4 and prmt places code byte j of a word at bits 8..15.
__device__ __forceinline__ void dequant_block16(uint4 c, uint32_t S, uint32_t lut_lane,
                                                uint32_t* out) {
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
    if (S - 2u <= 252u) {
        const uint32_t sf = S * 0x00800080u;      // bf16x2 {2^(S-127), 2^(S-127)}
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t a = prmt(w[i], 0u, 0x4404u | (j << 4)) + lut_lane;
                out[4 * i + j] = bmul2(lds32(a), sf);
            }
        }
    } else {
        const float sc = e8m0_f32(S);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) out[4 * i + j] = dequant_byte_exact((w[i] >> (8 * j)) & 0xFFu, sc);
    }
}

__device__ __forceinline__ float silu_f32(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

__device__ __forceinline__ void store_bf16(void* out, int64_t idx, float v) {
    reinterpret_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(v);
}

struct TileInfo {
    int g, f, row0, mrows;
};

// Tile t -> (group, feature tile, first row, valid rows).  Tiles of a group are
// numbered feature-tile-major with the token tile fastest, so CTAs working at
// the same time share the weight tile (L2 reuse).
template <int NT>
__device__ __forceinline__ TileInfo decode_tile(int t, const int* s_tstart, const int* s_off, int G) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {                 // largest g with s_tstart[g] <= t
        const int mid = (lo + hi + 1) >> 1;
        if (s_tstart[mid] <= t) lo = mid; else hi = mid - 1;
    }
    TileInfo ti;
    ti.g = lo;
    const int m = s_off[lo + 1] - s_off[lo];
    const int mt = (m + NT - 1) / NT;
    const int local = t - s_tstart[lo];
    ti.f = local / mt;
    const int tt = local - ti.f * mt;
    ti.row0 = s_off[lo] + tt * NT;
    ti.mrows = min(NT, m - tt * NT);
    return ti;
}

// Copy `rows` consecutive rows of block scales (kb bytes each) from global to
// shared: the 16-byte multiple with one bulk copy (counted on `bar`), the tail
// with plain loads.  Returns the bulk byte count.
__device__ __forceinline__ uint32_t stage_scales(uint8_t* dst, const uint8_t* src, int rows, int kb,
                                                 uint64_t* bar) {
    const uint32_t bytes = static_cast<uint32_t>(rows * kb);
    const uint32_t bulk = bytes & ~15u;
    if (bulk) bulk_load(dst, src, bulk, bar);
    if (bulk < bytes) {
        for (uint32_t i = bulk; i < bytes; ++i) dst[i] = src[i];
        // order these generic-proxy writes before later bulk copies into the buffer
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    return bulk;
}

template <int NT, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
grouped_w4a16_kernel(const __grid_constant__ CUtensorMap tmap_w,
                     const __grid_constant__ CUtensorMap tmap_x, const GemmArgs args) {
    using C = Cfg<NT>;
    const int S_ = args.stages;
    const Layout Ly = make_layout(C::kStageBytes, S_, args.K);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint32_t* lut = reinterpret_cast<uint32_t*>(smem);
    uint8_t* stages = smem + Ly.stages_off;
    uint8_t* scales = smem + Ly.scales_off;
    float* xbuf = reinterpret_cast<float*>(smem + Ly.xbuf_off);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Ly.bar_off);
    uint64_t* full = bars;                 // [16] stage filled (TMA tx)
    uint64_t* empty = bars + 16;           // [16] stage consumed (MMA commit)
    uint64_t* afull = bars + 32;           // [8]  A slot written (128 dequant threads)
    uint64_t* aempty = afull + kASlots;    // [8]  A slot consumed (MMA commit)
    uint64_t* accfull = aempty + kASlots;  // [2]  accumulator ready (MMA commit)
    uint64_t* accempty = accfull + 2;      // [2]  accumulator drained (128 epilogue threads)
    uint64_t* sfull = accempty + 2;        // [2]  tile scales staged (tx)
    uint64_t* sempty = sfull + 2;          // [2]  tile scales no longer needed (MMA commit)
    uint64_t* drain = sempty + 2;
    int* s_tstart = reinterpret_cast<int*>(smem + Ly.tstart_off);
    int* s_off = reinterpret_cast<int*>(smem + Ly.off_off);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + Ly.misc_off);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + Ly.misc_off + 4);
    volatile int* s_never = reinterpret_cast<volatile int*>(smem + Ly.misc_off + 8);   // stays 0

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = args.offsets ? args.G : 1;
    const int kb = args.K / 32;            // scale bytes per weight row

    // ---------------- set-up
    if (tid == 0) {
        for (int s = 0; s < S_; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < kASlots; ++a) {
            mbar_init(&afull[a], 128);
            mbar_init(&aempty[a], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accfull[b], 1);
            mbar_init(&accempty[b], 128);
            mbar_init(&sfull[b], 1);
            mbar_init(&sempty[b], 1);
        }
        mbar_init(drain, 1);
        *s_abort = 0;
        *s_never = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmap_w);
        prefetch_tmap(&tmap_x);
    }
    if (warp == 1) {
        tmem_alloc(s_tmem, 512);
        tmem_relinquish();
    }
    for (int i = tid; i <= G; i += kThreads)
        s_off[i] = args.offsets ? args.offsets[i] : (i == 0 ? 0 : args.m_single);
    for (int i = tid; i < 256 * 32; i += kThreads) {
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
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;
    const int total_tiles = s_tstart[G];
    const int nk = args.K / kBK;

    if (warp == 0) {
        // ---------------- TMA producer
        if (lane == 0) {
            int kit = 0, lt = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++lt) {
                const TileInfo ti = decode_tile<NT>(t, s_tstart, s_off, G);
                // block scales of the tile's weight rows, in the smem row order of the codes
                const int sb = lt & 1;
                if (!mbar_wait(&sempty[sb], ((lt >> 1) & 1) ^ 1, s_abort)) { ok = false; break; }
                uint8_t* sdst = scales + sb * Ly.scale_bytes;
                const uint8_t* gsc = args.w_scales + static_cast<int64_t>(ti.g) * args.rows_w * kb;
                uint32_t tx = 0;
                if (MODE == EPI_SWIGLU) {
                    tx += stage_scales(sdst, gsc + static_cast<int64_t>(ti.f * 64) * kb, 64, kb, &sfull[sb]);
                    tx += stage_scales(sdst + 64 * kb, gsc + static_cast<int64_t>(args.I + ti.f * 64) * kb,
                                       64, kb, &sfull[sb]);
                } else {
                    const int rows = min(kBM, args.rows_w - ti.f * kBM);
                    tx += stage_scales(sdst, gsc + static_cast<int64_t>(ti.f * kBM) * kb, rows, kb, &sfull[sb]);
                }
                mbar_arrive_expect_tx(&sfull[sb], tx);
                for (int ks = 0; ks < nk; ++ks, ++kit) {
                    const int st = kit % S_;
                    const uint32_t ph = (kit / S_) & 1;
                    if (!mbar_wait(&empty[st], ph ^ 1, s_abort)) { ok = false; break; }
                    uint8_t* sb_ = stages + st * C::kStageBytes;
                    mbar_arrive_expect_tx(&full[st], C::kStageBytes);
                    if (MODE == EPI_SWIGLU) {
                        tma_load_3d(sb_, &tmap_w, &full[st], ks * 32, ti.f * 64, ti.g);
                        tma_load_3d(sb_ + 64 * 32, &tmap_w, &full[st], ks * 32, args.I + ti.f * 64, ti.g);
                    } else {
                        tma_load_3d(sb_, &tmap_w, &full[st], ks * 32, ti.f * kBM, ti.g);
                    }
                    tma_load_2d(sb_ + kCodeBytes, &tmap_x, &full[st], ks * kBK, ti.row0);
                }
            }
            if (!ok) {
                *s_abort = 1;
                record_status(args.status, MXFP4_ERR_TIMEOUT);
                // let the copies already issued land before the CTA exits
                const int n_inflight = kit < S_ ? kit : S_;
                for (int i = 1; i <= n_inflight; ++i) {
                    const int k2 = kit - i;
                    mbar_wait(&full[k2 % S_], (k2 / S_) & 1, s_never);
                }
                for (int i = 1; i <= 2 && i <= lt + 1; ++i) {
                    const int l2 = lt + 1 - i;
                    mbar_wait(&sfull[l2 & 1], (l2 >> 1) & 1, s_never);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kBM, NT);
            int kit = 0, lt = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++lt) {
                const int acc = lt & 1;
                if (!mbar_wait(&accempty[acc], ((lt >> 1) & 1) ^ 1, s_abort)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * NT;
                for (int ks = 0; ks < nk; ++ks, ++kit) {
                    const int st = kit % S_;
                    const int as = kit % kASlots;
                    if (!mbar_wait(&full[st], (kit / S_) & 1, s_abort) ||
                        !mbar_wait(&afull[as], (kit / kASlots) & 1, s_abort)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t b_base = smem_u32(stages + st * C::kStageBytes + kCodeBytes);
                    const uint32_t a_tmem = tmem_base + kACol0 + as * 32;
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        mma_bf16_ts(d_tmem, a_tmem + 8 * j, sw128_desc(b_base + 32 * j), idesc,
                                    (ks | j) != 0 ? 1u : 0u);
                    tc_commit(&empty[st]);
                    tc_commit(&aempty[as]);
                }
                if (!ok) break;
                tc_commit(&accfull[acc]);
                tc_commit(&sempty[lt & 1]);
            }
            if (!ok) {
                *s_abort = 1;
                record_status(args.status, MXFP4_ERR_TIMEOUT);
            }
            // wait for every MMA issued by this thread before TMEM is released
            tc_commit(drain);
            mbar_wait(drain, 0, s_never);
        }
    } else if (warp >= 4 && warp < 12) {
        // ---------------- dequant warpgroups
        const int d = (warp - 4) >> 2;        // 0 or 1: even or odd stages
        const int q = warp & 3;               // TMEM lane quarter
        const uint32_t lut_lane = smem_u32(lut) + lane * 4;
        int srow;
        if (MODE == EPI_SWIGLU) {
            const int half = q >> 1, up = q & 1;
            srow = up * 64 + half * 32 + lane;  // lanes: gate 0-31 | up 0-31 | gate 32-63 | up 32-63
        } else {
            srow = q * 32 + lane;
        }
        const uint32_t sw = (static_cast<uint32_t>(srow) >> 2) & 1u;
        int kit = 0, lt = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++lt) {
            const TileInfo ti = decode_tile<NT>(t, s_tstart, s_off, G);
            const bool valid = MODE == EPI_SWIGLU || ti.f * kBM + srow < args.rows_w;
            const uint32_t sc_row = smem_u32(scales + (lt & 1) * Ly.scale_bytes) + srow * kb;
            bool scales_ready = false;
            for (int ks = 0; ks < nk; ++ks, ++kit) {
                if ((kit & 1) != d) continue;
                const int st = kit % S_;
                const int as = kit % kASlots;
                bool got = mbar_wait(&full[st], (kit / S_) & 1, s_abort) &&
                           mbar_wait(&aempty[as], ((kit / kASlots) & 1) ^ 1, s_abort);
                if (!scales_ready)
                    got = got && mbar_wait(&sfull[lt & 1], (lt >> 1) & 1, s_abort);
                if (!__all_sync(0xFFFFFFFFu, got)) { ok = false; break; }
                scales_ready = true;
                tc_fence_after();
                const uint32_t sc = valid ? lds_u16(sc_row + 2 * ks) : 0x7F7Fu;
                const uint32_t row_addr = smem_u32(stages + st * C::kStageBytes) + srow * 32;
                const uint4 c0 = lds128(row_addr + ((0u ^ sw) << 4));
                const uint4 c1 = lds128(row_addr + ((1u ^ sw) << 4));
                uint32_t out[32];
                dequant_block16(c0, sc & 0xFFu, lut_lane, out);
                dequant_block16(c1, sc >> 8, lut_lane, out + 16);
                tmem_st_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + kACol0 + as * 32, out);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&afull[as]);
            }
        }
        if (!ok) {
            *s_abort = 1;
            record_status(args.status, MXFP4_ERR_TIMEOUT);
        }
    } else if (warp >= 12) {
        // ---------------- epilogue warpgroup
        const int q = warp & 3;
        int lt = 0, cc = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++lt) {
            const TileInfo ti = decode_tile<NT>(t, s_tstart, s_off, G);
            const int acc = lt & 1;
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&accfull[acc], (lt >> 1) & 1, s_abort))) { ok = false; break; }
            tc_fence_after();
            const uint32_t t_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * NT;
#pragma unroll 1
            for (int c = 0; c < NT / 16; ++c, ++cc) {
                uint32_t v[16];
                tmem_ld_x16(t_base + 16 * c, v);
                tmem_wait_ld();
                if (MODE == EPI_SWIGLU) {
                    const int pr = q >> 1, up = q & 1;
                    // [pair][buffer][n][lane]: lanes write consecutive words (no bank conflicts)
                    float* xb = xbuf + (pr * 2 + (cc & 1)) * 16 * 32 + lane;
                    if (!up) {
#pragma unroll
                        for (int n = 0; n < 16; ++n) xb[n * 32] = __uint_as_float(v[n]);
                    }
                    named_bar_sync(1 + pr, 64);
                    if (up) {
                        const int feat = ti.f * 64 + pr * 32 + lane;
#pragma unroll
                        for (int n = 0; n < 16; ++n) {
                            const int tok = 16 * c + n;
                            if (tok < ti.mrows) {
                                const float h = silu_f32(xb[n * 32]) * __uint_as_float(v[n]);
                                store_bf16(args.out, static_cast<int64_t>(ti.row0 + tok) * args.out_ld + feat, h);
                            }
                        }
                    }
                } else {
                    const int feat = ti.f * kBM + q * 32 + lane;
                    if (feat < args.n_valid_feat) {
#pragma unroll
                        for (int n = 0; n < 16; ++n) {
                            const int tok = 16 * c + n;
                            if (tok < ti.mrows) {
                                const int64_t idx = static_cast<int64_t>(ti.row0 + tok) * args.out_ld + feat;
                                const float val = __uint_as_float(v[n]);
                                if (MODE == EPI_WEIGHTED)   // fp32 out: one rounding, in the combine
                                    reinterpret_cast<float*>(args.out)[idx] = val * args.row_w[ti.row0 + tok];
                                else
                                    store_bf16(args.out, idx, val);
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&accempty[acc]);
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
        tmem_dealloc(tmem_base, 512);
    }
}

template <int NT, int MODE>
cudaError_t launch_nt(const CUtensorMap& tw, const CUtensorMap& tx, GemmArgs a, int grid,
                      cudaStream_t stream) {
    using C = Cfg<NT>;
    // deepest ring that fits next to the LUT, the scale buffers and the rest
    int stages = C::kMaxStages;
    while (stages > 2 && make_layout(C::kStageBytes, stages, a.K).total > kSmemLimit) --stages;
    const Layout L = make_layout(C::kStageBytes, stages, a.K);
    if (stages < 3 || L.total > kSmemLimit) return cudaErrorInvalidConfiguration;
    a.stages = stages;
    auto kern = grouped_w4a16_kernel<NT, MODE>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
    if (err != cudaSuccess) return err;
    kern<<<grid, kThreads, L.total, stream>>>(tw, tx, a);
    return cudaGetLastError();
}

template <int MODE>
cudaError_t launch_mode(int nt, const CUtensorMap& tw, const CUtensorMap& tx, const GemmArgs& a,
                        int grid, cudaStream_t stream) {
    switch (nt) {
        case 16: return launch_nt<16, MODE>(tw, tx, a, grid, stream);
        case 32: return launch_nt<32, MODE>(tw, tx, a, grid, stream);
        case 64: return launch_nt<64, MODE>(tw, tx, a, grid, stream);
        default: return launch_nt<128, MODE>(tw, tx, a, grid, stream);
    }
}

}  // namespace

int pick_token_tile(int64_t rows, int64_t groups) {
    const int64_t avg = (rows + groups - 1) / (groups > 0 ? groups : 1);
    if (avg <= 16) return 16;
    if (avg <= 32) return 32;
    if (avg <= 64) return 64;
    return 128;
}

// Largest K the kernel accepts (its tile's block scales must fit in shared memory
// next to a 3-stage ring at the largest token tile).
int64_t max_gemm_k() {
    int64_t k = 64;
    while (make_layout(Cfg<128>::kStageBytes, 3, static_cast<int>(k + 64)).total <= kSmemLimit) k += 64;
    return k;
}

// Host launcher.  `tmap_w` covers the codes as a 3-D tensor {K/2, rows_w, G}
// with box {32, 64 (SWIGLU) or 128, 1} and 32B swizzle; `tmap_x` covers the
// activations {K, rows} (bf16) with box {64, nt} and 128B swizzle.
cudaError_t launch_grouped_gemm(int mode, int nt, const CUtensorMap& tmap_w,
                                const CUtensorMap& tmap_x, const GemmArgs& args, int grid,
                                cudaStream_t stream) {
    switch (mode) {
        case EPI_SWIGLU: return launch_mode<EPI_SWIGLU>(nt, tmap_w, tmap_x, args, grid, stream);
        case EPI_WEIGHTED: return launch_mode<EPI_WEIGHTED>(nt, tmap_w, tmap_x, args, grid, stream);
        default: return launch_mode<EPI_PLAIN>(nt, tmap_w, tmap_x, args, grid, stream);
    }
}

}  // namespace mx
