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
// Work tile: 128 weight rows (the MMA's M side) x NT token rows (the N side).
// The weights are dequantized once per 64-wide K stage.  (The engine is written
// for TT token tiles per weight tile; every launch uses TT = 1.)
//
// Data flow (one persistent CTA per SM, 16 warps):
//   warp 0        codes producer: per tile the block scales of its 128 rows
//                 (bulk copy, double-buffered); per group of four K stages the
//                 packed codes (128 B per row, 128B-swizzled: rows this wide
//                 stream from HBM at full rate) -> a codes ring that the dequant
//                 warps release as soon as they have read it.
//   warp 2        activation producer: per K stage TT bf16 tiles [NT x 64]
//                 (128B-swizzled, the UMMA K-major layout) -> activation ring,
//                 released by the MMA.
//   warps 4..11   two dequant warpgroups (alternate stages): one weight row per
//                 thread; codes -> bf16 through a lane-replicated 256-entry
//                 shared LUT (one prmt forms an entry's address) times the block
//                 scale 2^(S-127) (exact bf16 product), stored with tcgen05.st
//                 into TMEM: the dequantized weights are the MMA's A operand and
//                 never touch shared memory.
//   warp 1        MMA issuer: tcgen05.mma kind::f16, M = 128, N = NT, K = 16,
//                 A from TMEM, B from shared memory, D (fp32) in TMEM.
//   warps 12..15  epilogue: tcgen05.ld of the accumulators, fused epilogue,
//                 stores.
// The MMA issuer waits once per group of four K stages: a wait between tcgen05
// operations costs the issuing thread about the latency of the MMAs in flight.
// TMEM: columns [0, 256) accumulators (TT*NT columns per buffer, double-buffered
// when they fit), [256, 512) eight 32-column A slots (two sets of four).
// Every mbarrier wait is time-bounded (MXFP4_ERR_TIMEOUT in the status word).
#include <cmath>

#include "gemm_common.cuh"

namespace mx {

namespace {

using namespace gemm;

constexpr int kThreads = 512;
constexpr int kBK = 64;             // K per pipeline stage
constexpr int kASlots = 8;          // at most 8 TMEM A-operand slots (32 columns each)
constexpr int kSub = 4;             // 64-wide K sub-stages per codes super-stage
constexpr int kCodeRowBytes = kSub * kBK / 2;          // 128 B of codes per weight row
constexpr int kCodeBytes = kBM * kCodeRowBytes;        // one codes super-stage (16 KB)
constexpr int kLutBytes = 256 * 256;   // 256 byte values x 256-B rows (32 lanes x bf16x2 used)
constexpr int kSmemLimit = 227 * 1024;
constexpr int kMaxRing = 16;
constexpr int kMaxCodeStages = 4;
// Small token tiles (decode) stream weights at a far higher rate per MMA: their codes
// ring takes the shared memory the activation ring leaves free (up to 8 x 16 KB in
// flight per SM keeps HBM busy at ~1.5 us of latency).
constexpr int kMaxCodeStagesLock = 8;

template <int NT, int TT>
struct Cfg {
    static constexpr int kActTile = NT * kBK * 2;          // one token tile of one K stage
    static constexpr int kActStage = TT * kActTile;
    static constexpr int kAccCols = TT * NT;               // TMEM columns of one accumulator set
    // K stages per MMA group (one barrier wait and one commit each): 4, or 2 when the
    // accumulators need more TMEM (NT = 192: two 192-column buffers + 4 A slots)
    static constexpr int kGrp = NT * TT > 128 && TT == 1 ? 2 : kSub;
    static constexpr int kACol = 512 - 2 * kGrp * 32;       // A slots: two sets of kGrp
    static constexpr int kAccBufs = 2 * kAccCols <= kACol ? 2 : 1;
    static constexpr int kTileRows = TT * NT;               // token rows of a work tile
    // NT <= 64 (decode): the activation ring holds whole groups (chunks of kSub
    // stages), each filled by one barrier and released by one MMA commit per group,
    // several groups ahead of the MMA (an activation tile's load latency exceeds a
    // group's MMA time at this N).  Otherwise the ring holds single stages.
    static constexpr bool kLock = NT <= 64;
    static constexpr int kActUnit = kLock ? kSub * kActStage : kActStage;   // bytes per ring slot
    static constexpr int kMaxActStages = kLock ? 4 : (TT == 1 ? (NT > 128 ? 4 : 5) : kSub);
    static constexpr int kChunk = kAccCols < 32 ? kAccCols : 32;   // epilogue columns per TMEM load
    static_assert(kActTile % 1024 == 0, "activation tiles must keep 1024-B alignment");
    static_assert(kAccCols <= kACol, "accumulators overlap the A slots");
    static_assert(!kLock || kGrp == kSub, "the chunked activation ring follows groups of kSub stages");
};

// Shared-memory layout, identical on host (sizing) and device.  Offsets count from
// the start of dynamic shared memory, whose shared-window address is 1024 (the
// window's first 1 KB is reserved and the kernel has no static shared memory; the
// kernel checks this).  The dequant LUT sits at window address 64 KB, so that the
// low 16 bits of an entry address are (code byte << 8) | (lane * 4) and one prmt
// builds it.  Below the LUT: barriers, tile tables, the tile scales and as many
// codes stages as fit; above it: the activation stages, then anything left over.
constexpr int kWindowBase = 1024;
constexpr int kLutOff = 65536 - kWindowBase;

struct Layout {
    int scales_off, scale_bytes, bar_off, tstart_off, off_off, misc_off;
    int n_codes_lo, codes_lo_off, acts_off, codes_hi_off, total;
};

__host__ __device__ inline Layout make_layout(int act_stage_bytes, int code_stages, int act_stages,
                                              int K) {
    Layout L;
    const int n_bars = 4 * kMaxRing + 2 * kASlots + 2 + 2 + 2 + 2 + 1;
    L.bar_off = 0;
    L.tstart_off = L.bar_off + n_bars * 8;
    L.off_off = L.tstart_off + (kMaxGroups + 1) * 4;
    L.misc_off = L.off_off + (kMaxGroups + 1) * 4;
    int lo = (L.misc_off + 16 + 127) / 128 * 128;
    int hi = kLutOff + kLutBytes;
    L.acts_off = hi;
    hi += act_stages * act_stage_bytes;
    L.scale_bytes = ((kBM * (K / 32)) + 127) / 128 * 128;
    if (lo + 2 * L.scale_bytes <= kLutOff) {
        L.scales_off = lo;
        lo += 2 * L.scale_bytes;
    } else {
        L.scales_off = hi;
        hi += 2 * L.scale_bytes;
    }
    lo = (lo + 1023) / 1024 * 1024;
    L.codes_lo_off = lo;
    L.n_codes_lo = lo < kLutOff ? (kLutOff - lo) / kCodeBytes : 0;
    if (L.n_codes_lo > code_stages) L.n_codes_lo = code_stages;
    hi = (hi + 1023) / 1024 * 1024;
    L.codes_hi_off = hi;
    hi += (code_stages - L.n_codes_lo) * kCodeBytes;
    L.total = hi;
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

// 16 code bytes (32 weights of one K block) -> 16 bf16x2 words.
// Fast path (S in [2, 254]): LUT value times 2^(S-127) as one bf16x2 multiply,
// exact because both factors and the product are normal bf16 numbers (or the
// product overflows to Inf, as round-to-nearest-even does).  Otherwise the
// exact fp32 route (subnormal results for S <= 1, NaN for S = 255).
// LUT entry (b, lane) sits at window address 65536 + b * 256 + lane * 4 (lane-
// replicated, so the 32 lanes of a warp hit 32 different banks whatever their
// bytes); lut_lane = 65536 + lane * 4 has a zero byte 1, and one prmt replaces that
// byte with code byte j of a word: the entry address in one instruction.
__device__ __forceinline__ void dequant_block16(uint4 c, uint32_t S, uint32_t lut_lane,
                                                uint32_t* out) {
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
    if (S - 2u <= 252u) {
        const uint32_t sf = S * 0x00800080u;      // bf16x2 {2^(S-127), 2^(S-127)}
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t a = prmt(w[i], lut_lane, 0x7604u | (j << 4));
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

template <int NT, int TT, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
grouped_w4a16_kernel(const __grid_constant__ CUtensorMap tmap_w,
                     const __grid_constant__ CUtensorMap tmap_x, const GemmArgs args) {
    using C = Cfg<NT, TT>;
    const int SC = args.code_stages, SA = args.act_stages;
    const Layout Ly = make_layout(C::kActUnit, SC, SA, args.K);
    extern __shared__ __align__(1024) uint8_t smem[];
    // the layout assumes dynamic shared memory at window address 1024 (see Layout)
    if (smem_u32(smem) != kWindowBase) {
        if (threadIdx.x == 0) record_status(args.status, MXFP4_ERR_CUDA);
        return;
    }
    uint32_t* lut = reinterpret_cast<uint32_t*>(smem + kLutOff);
    uint8_t* acts = smem + Ly.acts_off;
    auto codes_stage = [&](int i) {
        return i < Ly.n_codes_lo ? smem + Ly.codes_lo_off + i * kCodeBytes
                                 : smem + Ly.codes_hi_off + (i - Ly.n_codes_lo) * kCodeBytes;
    };
    uint8_t* scales = smem + Ly.scales_off;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Ly.bar_off);
    uint64_t* cfull = bars;                          // codes stage landed (TMA tx)
    uint64_t* cempty = bars + kMaxRing;              // codes super-stage read (256 dequant threads)
    uint64_t* xfull = bars + 2 * kMaxRing;           // activation stage landed (TMA tx)
    uint64_t* xempty = bars + 3 * kMaxRing;          // activation stage consumed (MMA commit)
    uint64_t* afull = bars + 4 * kMaxRing;           // A-slot set written (512 arrivals per group)
    uint64_t* aempty = afull + kASlots;              // A-slot set consumed (MMA commit)
    uint64_t* accfull = aempty + kASlots;            // accumulators ready (MMA commit)
    uint64_t* accempty = accfull + 2;                // accumulators drained (128 epilogue threads)
    uint64_t* sfull = accempty + 2;                  // tile scales staged (tx)
    uint64_t* sempty = sfull + 2;                    // tile scales released (MMA commit)
    uint64_t* drain = sempty + 2;
    int* s_tstart = reinterpret_cast<int*>(smem + Ly.tstart_off);
    int* s_off = reinterpret_cast<int*>(smem + Ly.off_off);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + Ly.misc_off);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + Ly.misc_off + 4);
    volatile int* s_never = reinterpret_cast<volatile int*>(smem + Ly.misc_off + 8);   // stays 0

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = args.offsets ? args.G : 1;
    const int kb = args.K / 32;            // scale bytes per weight row
    constexpr int NB = C::kAccBufs;

    // ---------------- set-up
    if (tid == 0) {
        for (int s = 0; s < SC; ++s) {
            mbar_init(&cfull[s], 1);
            mbar_init(&cempty[s], 256);   // both dequant warpgroups pass every super-stage
        }
        for (int s = 0; s < SA; ++s) {
            mbar_init(&xfull[s], 1);
            mbar_init(&xempty[s], 1);
        }
        for (int a = 0; a < kASlots; ++a) {
            mbar_init(&afull[a], 256 * C::kGrp / 2);   // per group: kGrp/2 arrivals x 256 dequant threads
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
    if (warp == 0 && lane == 0) prefetch_tmap(&tmap_w);
    if (warp == 2 && lane == 0) prefetch_tmap(&tmap_x);
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
            acc += ((m + C::kTileRows - 1) / C::kTileRows) * args.n_ftiles;
        }
        s_tstart[G] = acc;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;
    const int total_tiles = s_tstart[G];
    const int nk = args.K / kBK;                    // 64-wide K stages
    const int nss = (nk + kSub - 1) / kSub;         // codes super-stages
    // Every CTA walks the K super-stages of its tiles in a rotated order (starting at
    // blockIdx.x mod nss): CTAs that share a token tile then read different activation
    // lines at any moment instead of all hitting the same L2 lines together.
    const int rot = static_cast<int>(blockIdx.x % static_cast<unsigned>(nss));

    if (warp == 0) {
        // ---------------- codes (+ scales) producer
        if (lane == 0) {
            RingPos c;
            int lt = 0, issued = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++lt) {
                const TileInfo ti = decode_tile(t, s_tstart, s_off, G, C::kTileRows);
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
                // codes in super-stages of kSub K stages: 128 B of every weight row per
                // TMA box (row segments this wide stream from HBM at full rate); the tail
                // beyond K/2 bytes is zero-filled by the TMA and never dequantized
                for (int si = 0; si < nss; ++si) {
                    const int ss = si + rot < nss ? si + rot : si + rot - nss;
                    if (!mbar_wait(&cempty[c.idx], c.ph ^ 1, s_abort)) { ok = false; break; }
                    uint8_t* dst = codes_stage(c.idx);
                    mbar_arrive_expect_tx(&cfull[c.idx], kCodeBytes);
                    const int x = ss * kCodeRowBytes;
                    if (MODE == EPI_SWIGLU) {
                        tma_load_3d(dst, &tmap_w, &cfull[c.idx], x, ti.f * 64, ti.g);
                        tma_load_3d(dst + 64 * kCodeRowBytes, &tmap_w, &cfull[c.idx], x, args.I + ti.f * 64, ti.g);
                    } else {
                        tma_load_3d(dst, &tmap_w, &cfull[c.idx], x, ti.f * kBM, ti.g);
                    }
                    c.next(SC);
                    ++issued;
                }
            }
            if (!ok) {
                *s_abort = 1;
                record_status(args.status, MXFP4_ERR_TIMEOUT);
                // let the copies already issued land before the CTA exits
                RingPos r;
                const int first = issued > SC ? issued - SC : 0;
                for (int i = 0; i < issued; ++i) {
                    if (i >= first) mbar_wait(&cfull[r.idx], r.ph, s_never);
                    r.next(SC);
                }
                for (int l2 = lt - 1; l2 <= lt && l2 >= 0; ++l2)
                    mbar_wait(&sfull[l2 & 1], (l2 >> 1) & 1, s_never);
            }
        }
    } else if (warp == 2) {
        // ---------------- activation producer
        if (lane == 0) {
            RingPos x;             // kLock: ring of SA group chunks; else: ring of SA stages
            int issued = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
                const TileInfo ti = decode_tile(t, s_tstart, s_off, G, C::kTileRows);
                for (int si = 0; si < nss && ok; ++si) {
                    const int ss = si + rot < nss ? si + rot : si + rot - nss;
                    const int nsub = min(kSub, nk - ss * kSub);
                    if (C::kLock) {
                        // the group's stages in one chunk: one barrier, one release
                        if (!mbar_wait(&xempty[x.idx], x.ph ^ 1, s_abort)) { ok = false; break; }
                        mbar_arrive_expect_tx(&xfull[x.idx], nsub * C::kActStage);
                        for (int j = 0; j < nsub; ++j)
#pragma unroll
                            for (int tt = 0; tt < TT; ++tt)
                                tma_load_2d(acts + x.idx * C::kActUnit + j * C::kActStage + tt * C::kActTile,
                                            &tmap_x, &xfull[x.idx], (ss * kSub + j) * kBK, ti.row0 + tt * NT);
                        x.next(SA);
                        ++issued;
                    } else {
                        for (int j = 0; j < nsub; ++j) {
                            if (!mbar_wait(&xempty[x.idx], x.ph ^ 1, s_abort)) { ok = false; break; }
                            mbar_arrive_expect_tx(&xfull[x.idx], C::kActStage);
#pragma unroll
                            for (int tt = 0; tt < TT; ++tt)
                                tma_load_2d(acts + x.idx * C::kActStage + tt * C::kActTile, &tmap_x, &xfull[x.idx],
                                            (ss * kSub + j) * kBK, ti.row0 + tt * NT);
                            x.next(SA);
                            ++issued;
                        }
                    }
                }
            }
            if (!ok) {
                *s_abort = 1;
                record_status(args.status, MXFP4_ERR_TIMEOUT);
                // let the copies already issued land before the CTA exits
                RingPos r;
                const int first = issued > SA ? issued - SA : 0;
                for (int i = 0; i < issued; ++i) {
                    if (i >= first) mbar_wait(&xfull[r.idx], r.ph, s_never);
                    r.next(SA);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        // One barrier wait and one commit per group of kSub K stages: a wait issued
        // between tcgen05 operations stalls the issuing thread for roughly the latency
        // of the MMAs in flight, so it is paid once per group, not once per stage.
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kBM, NT);
            RingPos x, a;          // x: activation ring (chunks when kLock, else stages); a: A-slot sets
            int lt = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++lt) {
                const int b = NB == 2 ? (lt & 1) : 0;
                const uint32_t bph = NB == 2 ? ((lt >> 1) & 1) : (lt & 1);
                if (!mbar_wait(&accempty[b], bph ^ 1, s_abort)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + b * C::kAccCols;
                int ki = 0;
                for (int si = 0; si < nss && ok; ++si) {
                    const int ss = si + rot < nss ? si + rot : si + rot - nss;
                    const int nsub = min(kSub, nk - ss * kSub);
                    for (int g0 = 0; g0 < nsub; g0 += C::kGrp) {
                        const int ng = min(C::kGrp, nsub - g0);
                        if (!mbar_wait(&afull[a.idx], a.ph, s_abort)) { ok = false; break; }
                        tc_fence_after();
                        for (int j = 0; j < ng; ++j, ++ki) {
                            const uint32_t b_base = smem_u32(acts + x.idx * C::kActUnit +
                                                             (C::kLock ? j * C::kActStage : 0));
                            const uint32_t a_tmem = tmem_base + C::kACol + (a.idx * C::kGrp + j) * 32;
#pragma unroll
                            for (int tt = 0; tt < TT; ++tt)
#pragma unroll
                                for (int jj = 0; jj < 4; ++jj)
                                    mma_bf16_ts(d_tmem + tt * NT, a_tmem + 8 * jj,
                                                sw128_desc(b_base + tt * C::kActTile + 32 * jj), idesc,
                                                (ki | jj) != 0 ? 1u : 0u);
                            if (!C::kLock) {
                                tc_commit(&xempty[x.idx]);
                                x.next(SA);
                            }
                        }
                        tc_commit(&aempty[a.idx]);
                        a.next(2);
                        if (C::kLock) {
                            tc_commit(&xempty[x.idx]);
                            x.next(SA);
                        }
                    }
                }
                if (!ok) break;
                tc_commit(&accfull[b]);
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
            // smem rows 0-63 gate, 64-127 up; lane l of warp q: feature 16q + (l & 15),
            // gate for l < 16, up for l >= 16
            srow = (lane < 16 ? 0 : 64) + 16 * q + (lane & 15);
        } else {
            srow = q * 32 + lane;
        }
        const uint32_t sw = static_cast<uint32_t>(srow) & 7u;   // 128B swizzle: chunk ^= row % 8
        const uint32_t tmem_lane = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + C::kACol;
        RingPos c, a, xr;        // codes super-stages, A-slot sets, activation ring
        int kit = 0, lt = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++lt) {
            const TileInfo ti = decode_tile(t, s_tstart, s_off, G, C::kTileRows);
            const bool valid = MODE == EPI_SWIGLU || ti.f * kBM + srow < args.rows_w;
            const uint32_t sc_row = smem_u32(scales + (lt & 1) * Ly.scale_bytes) + srow * kb;
            for (int si = 0; si < nss && ok; ++si) {
                const int ss = si + rot < nss ? si + rot : si + rot - nss;
                const int nsub = min(kSub, nk - ss * kSub);
                // the super-stage's codes have landed, the tile's scales too
                bool got = mbar_wait(&cfull[c.idx], c.ph, s_abort);
                if (si == 0) got = got && mbar_wait(&sfull[lt & 1], (lt >> 1) & 1, s_abort);
                if (!__all_sync(0xFFFFFFFFu, got)) { ok = false; break; }
                const uint32_t row_addr = smem_u32(codes_stage(c.idx)) + srow * kCodeRowBytes;
                for (int g0 = 0; g0 < nsub; g0 += C::kGrp) {
                    const int ng = min(C::kGrp, nsub - g0);
                    // the group's A slots are free
                    if (!__all_sync(0xFFFFFFFFu, mbar_wait(&aempty[a.idx], a.ph ^ 1, s_abort))) { ok = false; break; }
                    tc_fence_after();
                    int done = 0;
                    int xs0 = 0, xs1 = 0;
                    uint32_t xph0 = 0, xph1 = 0;
                    for (int jg = 0; jg < ng; ++jg, ++kit) {
                        const int j = g0 + jg;    // stage within the super-stage
                        if ((kit & 1) == d) {
                            const int ks = ss * kSub + j;
                            const uint32_t sc = valid ? lds_u16(sc_row + 2 * ks) : 0x7F7Fu;
                            const uint4 c0 = lds128(row_addr + (((2u * j) ^ sw) << 4));
                            const uint4 c1 = lds128(row_addr + (((2u * j + 1u) ^ sw) << 4));
                            uint32_t out[32];
                            dequant_block16(c0, sc & 0xFFu, lut_lane, out);
                            dequant_block16(c1, sc >> 8, lut_lane, out + 16);
                            tmem_st_x32(tmem_lane + (a.idx * C::kGrp + jg) * 32, out);
                            const int xs = xr.idx;      // kLock: the group's chunk
                            const uint32_t xph = xr.ph;
                            if (done == 0) { xs0 = xs; xph0 = xph; } else { xs1 = xs; xph1 = xph; }
                            ++done;
                        }
                        if (!C::kLock) xr.next(SA);
                    }
                    // The MMA issuer waits for the whole group, so this thread signals its
                    // stages together at the end: one wait for all of its TMEM stores, and
                    // the activation tiles of its stages must have landed too.
                    tmem_wait_st();
                    bool landed = true;
                    if (done > 0) landed = mbar_wait(&xfull[xs0], xph0, s_abort);
                    if (done > 1) landed = landed && mbar_wait(&xfull[xs1], xph1, s_abort);
                    if (!__all_sync(0xFFFFFFFFu, landed)) { ok = false; break; }
                    tc_fence_before();
                    // every dequant thread arrives kGrp/2 times per group (the warpgroups
                    // alternate stages; short groups count the same)
#pragma unroll
                    for (int i2 = 0; i2 < C::kGrp / 2; ++i2) mbar_arrive(&afull[a.idx]);
                    a.next(2);
                    if (C::kLock) xr.next(SA);
                }
                if (!ok) break;
                mbar_arrive(&cempty[c.idx]);     // this warpgroup is done reading the codes
                c.next(SC);
            }
        }
        if (!ok) {
            *s_abort = 1;
            record_status(args.status, MXFP4_ERR_TIMEOUT);
        }
    } else if (warp >= 12) {
        // ---------------- epilogue warpgroup
        constexpr int CW = C::kChunk;
        const int q = warp & 3;
        int lt = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++lt) {
            const TileInfo ti = decode_tile(t, s_tstart, s_off, G, C::kTileRows);
            const int b = NB == 2 ? (lt & 1) : 0;
            const uint32_t bph = NB == 2 ? ((lt >> 1) & 1) : (lt & 1);
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&accfull[b], bph, s_abort))) { ok = false; break; }
            tc_fence_after();
            const uint32_t t_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + b * C::kAccCols;
            epilogue_tile<MODE, CW, C::kAccCols>(args, ti, t_base, q, lane);
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
        tmem_dealloc(tmem_base, 512);
    }
}

// Ring depths for a launch: the deepest rings that fit next to the LUT, the
// scale buffers and the rest (activation ring first, then the codes ring).
template <int NT, int TT>
bool ring_depths(int K, int* sc, int* sa, int* smem) {
    using C = Cfg<NT, TT>;
    // The activation ring must hold at least one whole group of kGrp stages: the MMA
    // issuer consumes a group only once all its stages are ready.
    int c = C::kLock ? kMaxCodeStagesLock : kMaxCodeStages, a = C::kMaxActStages;
    const int amin = C::kLock ? 2 : C::kGrp;   // two chunks, or one group of stages
    while (make_layout(C::kActUnit, c, a, K).total > kSmemLimit) {
        if (c > 2) --c;
        else if (a > amin) --a;
        else return false;
    }
    *sc = c;
    *sa = a;
    *smem = make_layout(C::kActUnit, c, a, K).total;
    return true;
}

template <int NT, int TT, int MODE>
cudaError_t launch_cfg(const CUtensorMap& tw, const CUtensorMap& tx, GemmArgs a, int grid,
                       cudaStream_t stream) {
    int sc = 0, sa = 0, smem = 0;
    if (!ring_depths<NT, TT>(a.K, &sc, &sa, &smem)) return cudaErrorInvalidConfiguration;
    a.code_stages = sc;
    a.act_stages = sa;
    auto kern = grouped_w4a16_kernel<NT, TT, MODE>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    kern<<<grid, kThreads, smem, stream>>>(tw, tx, a);
    return cudaGetLastError();
}

template <int MODE>
cudaError_t launch_mode(int nt, int tt, const CUtensorMap& tw, const CUtensorMap& tx,
                        const GemmArgs& a, int grid, cudaStream_t stream) {
    if (nt == 16) return launch_cfg<16, 1, MODE>(tw, tx, a, grid, stream);
    if (nt == 32) return launch_cfg<32, 1, MODE>(tw, tx, a, grid, stream);
    if (nt == 64) return launch_cfg<64, 1, MODE>(tw, tx, a, grid, stream);
    if (nt == 192) {
        int sc, sa, smem;
        if (ring_depths<192, 1>(a.K, &sc, &sa, &smem)) return launch_cfg<192, 1, MODE>(tw, tx, a, grid, stream);
    }
    (void)tt;   // one token tile per weight tile in every configuration
    return launch_cfg<128, 1, MODE>(tw, tx, a, grid, stream);
}

}  // namespace

// Token tiling for `rows` activation rows spread over `groups` groups: NT rows per
// MMA (16 .. 192).  Each token tile dequantizes the group's weight tiles once, and
// that, not the MMA width, bounds a tile's time (at NT <= 64 an MMA costs the same
// whatever its N).  So the cost of a tile grows only slowly with NT.  Measured on
// the decode- and 120b-shaped layers, relative to a 16-row tile: 1.0 (32), 1.04
// (64), 1.14 (128), 1.43 (192).  The launcher takes the NT with the least cost times
// tiles, counted for a group one standard deviation above the mean (routed counts
// spread about like the square root of the mean); ties go to the smaller tile.
TokenTiling pick_token_tiling(int64_t rows, int64_t groups) {
    const int64_t avg = (rows + groups - 1) / (groups > 0 ? groups : 1);
    const double hi = static_cast<double>(avg) + std::sqrt(static_cast<double>(avg));
    constexpr int kNt[5] = {16, 32, 64, 128, 192};
    constexpr double kCost[5] = {1.0, 1.0, 1.04, 1.14, 1.43};
    int best = 0;
    double best_cost = 0.0;
    for (int i = 0; i < 5; ++i) {
        const double c = kCost[i] * std::ceil(hi / kNt[i]);
        if (i == 0 || c < best_cost) {
            best = i;
            best_cost = c;
        }
    }
    return {kNt[best], 1};
}

// Largest K the kernel accepts: a tile's block scales must fit in shared memory
// next to the smallest rings of every configuration.
int64_t max_gemm_k() {
    int64_t k = 64;
    int sc, sa, smem;
    while (ring_depths<128, 1>(static_cast<int>(k + 64), &sc, &sa, &smem) &&
           ring_depths<64, 1>(static_cast<int>(k + 64), &sc, &sa, &smem) &&
           ring_depths<32, 1>(static_cast<int>(k + 64), &sc, &sa, &smem) &&
           ring_depths<16, 1>(static_cast<int>(k + 64), &sc, &sa, &smem))
        k += 64;
    return k;
}

// Host launcher.  `tmap_w` covers the codes as a 3-D tensor {K/2, rows_w, G}
// with box {128, 64 (SWIGLU) or 128, 1} and 128B swizzle; `tmap_x` covers the
// activations {K, rows} (bf16) with box {64, nt} and 128B swizzle.
cudaError_t launch_grouped_gemm(int mode, TokenTiling tiling, const CUtensorMap& tmap_w,
                                const CUtensorMap& tmap_x, const GemmArgs& args, int grid,
                                cudaStream_t stream) {
    switch (mode) {
        case EPI_SWIGLU:
            return launch_mode<EPI_SWIGLU>(tiling.nt, tiling.tt, tmap_w, tmap_x, args, grid, stream);
        case EPI_WEIGHTED:
            return launch_mode<EPI_WEIGHTED>(tiling.nt, tiling.tt, tmap_w, tmap_x, args, grid, stream);
        default:
            return launch_mode<EPI_PLAIN>(tiling.nt, tiling.tt, tmap_w, tmap_x, args, grid, stream);
    }
}

}  // namespace mx
