// Grouped W4A4 GEMM on sm_100a block-scaled tensor cores (tcgen05.mma kind::mxf4).
//
// Both operands are MXFP4 (agentlenshq.com, "Transformers 4.40 performance upgrades
// for OpenAI GPT-OSS ...", section "What MXFP4 Is": E2M1 values, one shared scale
// per 32 elements).  For every group g (an expert) with activation rows
// offsets[g] .. offsets[g+1] of one packed matrix X (codes [rows, K/2], E8M0 scales
// [rows, K/32]) and weights W_g (codes [rows_w, K/2], scales [rows_w, K/32]):
//     D_g = (X_g with its block scales) . (W_g with its block scales)^T
// in fp32, then the epilogues of the W4A16 engine (plain bf16, SwiGLU -> bf16 h,
// fp32 times the routing weight).  The tensor core applies the scales itself: a
// product of two E2M1 values times 2^(sa + sb) is exact and only the fp32
// accumulation rounds, so this equals the dot product of the dequantized operands
// up to summation order.
//
// Work tile: 128 weight rows (the MMA's M) x NT token rows (N); K in super-stages
// of 256 (128 bytes of codes per row, one 128B-swizzle row), four MMAs of K = 64.
//
// Roles (one persistent CTA per SM, 12 warps; warp 3 idles):
//   warp 0    weight producer: per tile the block scales of its 128 rows (bulk
//             copy, double-buffered); per super-stage the codes box -> stage ring.
//   warp 2    activation producer: per tile the block scales of its NT rows (bulk
//             copy of the covering 16-byte-aligned range, double-buffered); per
//             super-stage the activation codes box -> stage ring.
//   warps 8-11 scale builders: per super-stage each rewrites one operand's four
//             scales per row into the tensor core's scale-factor layout (per 4
//             scales of a 128-row block: row r at byte 16 (r % 32) + 4 (r / 32) + j),
//             waits for that operand's codes and marks its part of the stage ready.
//   warp 1    MMA issuer: per super-stage copies the four scale atoms to TMEM
//             (tcgen05.cp, ordered with its MMAs), issues the MMAs, and releases
//             the stage with one commit.
//   warps 4-7 epilogue (TMEM lane quarters 0-3).
// TMEM: accumulators [0, 2 NT) double-buffered, A scales at column 256 (4 columns
// per 4-scale chunk, two chunks), B scales at column 264.
#include "gemm_common.cuh"

namespace mx {

namespace {

using namespace gemm;

constexpr int kThreads4 = 384;
constexpr int kSSK = 256;                    // K per super-stage
constexpr int kRowBytes = kSSK / 2;          // codes bytes per row per super-stage
constexpr int kWBytes = kBM * kRowBytes;     // weight codes per stage (16 KB)
constexpr int kAtom = 512;                   // one scale atom: 128 rows x 4 scales
constexpr int kAtomsBytes = 4 * kAtom;       // A chunk 0, A chunk 1, B chunk 0, B chunk 1
constexpr int kMaxStages4 = 8;
constexpr int kSmemLimit4 = 227 * 1024;
constexpr uint32_t kSfaCol = 256, kSfbCol = 264;
// mbarriers: four per stage (codes of W, codes of X, ready, empty), six double
// buffers (tile scales of W and X full / empty, accumulators full / empty), drain.
constexpr int kNumBars4 = 4 * kMaxStages4 + 6 * 2 + 1;

struct Layout4 {
    int stage_bytes, x_off, atoms_off, wsc_off, wsc_bytes, xsc_off, xsc_bytes, bar_off, tstart_off,
        off_off, misc_off, total;
};

__host__ __device__ inline Layout4 make_layout4(int NT, int stages, int K) {
    Layout4 L;
    L.x_off = kWBytes;
    L.atoms_off = L.x_off + NT * kRowBytes;
    L.stage_bytes = L.atoms_off + kAtomsBytes;
    const int kb = K / 32;
    L.wsc_off = stages * L.stage_bytes;
    L.wsc_bytes = (kBM * kb + 127) / 128 * 128;
    L.xsc_off = L.wsc_off + 2 * L.wsc_bytes;
    L.xsc_bytes = (NT * kb + 32 + 127) / 128 * 128;   // + the 16-byte alignment shifts
    L.bar_off = L.xsc_off + 2 * L.xsc_bytes;
    const int n_bars = kNumBars4;
    L.tstart_off = L.bar_off + n_bars * 8;
    L.off_off = L.tstart_off + (kMaxGroups + 1) * 4;
    L.misc_off = L.off_off + (kMaxGroups + 1) * 4;
    L.total = L.misc_off + 32 + 1024;   // + slack for the 1024-B alignment of the base
    return L;
}

// Copies posted into a ring of up to 32 slots, waited for before the CTA exits
// when it leaves early (no bulk copy may land in shared memory after exit).
struct Posted {
    uint32_t mask = 0, ph = 0;
    __device__ __forceinline__ void post(int i, uint32_t parity) {
        mask |= 1u << i;
        ph = (ph & ~(1u << i)) | (parity << i);
    }
    __device__ __forceinline__ void drain(uint64_t* full, int n, volatile int* never) const {
        for (int i = 0; i < n; ++i)
            if ((mask >> i) & 1u) (void)mbar_wait(&full[i], (ph >> i) & 1u, never);
    }
};

// Four scale bytes of one row for K blocks k0 .. k0+3 (k0 even), 127 (= 1.0) past
// the row's kb blocks.  `row` is the shared-memory address of the row's scales
// (2-byte aligned: kb and the row offset are even).
__device__ __forceinline__ uint32_t scale_word(uint32_t row, int k0, int kb, bool valid) {
    if (!valid) return 0x7F7F7F7Fu;
    const uint32_t lo = k0 < kb ? lds_u16(row + k0) : 0x7F7Fu;
    const uint32_t hi = k0 + 2 < kb ? lds_u16(row + k0 + 2) : 0x7F7Fu;
    return lo | (hi << 16);
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

template <int NT, int MODE>
__global__ void __launch_bounds__(kThreads4, 1)
grouped_w4a4_kernel(const __grid_constant__ CUtensorMap tmap_w,
                    const __grid_constant__ CUtensorMap tmap_x, const GemmArgs args) {
    constexpr int kAccCols = NT;
    constexpr int kCW = NT < 32 ? NT : 32;
    const int S = args.code_stages;
    const Layout4 Ly = make_layout4(NT, S, args.K);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* wsc = smem + Ly.wsc_off;
    uint8_t* xsc = smem + Ly.xsc_off;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Ly.bar_off);
    uint64_t* wfull = bars;                          // weight codes landed (tx)
    uint64_t* xfull = bars + kMaxStages4;            // activation codes landed (tx)
    uint64_t* ready = bars + 2 * kMaxStages4;        // stage complete: codes + scale atoms
    uint64_t* empty = bars + 3 * kMaxStages4;        // stage consumed (MMA commit)
    uint64_t* sfull = bars + 4 * kMaxStages4;        // tile weight scales staged (tx)
    uint64_t* sempty = sfull + 2;                    // tile weight scales read (builder)
    uint64_t* xsfull = sempty + 2;                   // tile activation scales staged (tx)
    uint64_t* xsempty = xsfull + 2;                  // tile activation scales read (builder)
    uint64_t* accfull = xsempty + 2;                 // accumulators ready (MMA commit)
    uint64_t* accempty = accfull + 2;                // accumulators drained (128 epilogue threads)
    uint64_t* drain = accempty + 2;
    static_assert(4 * kMaxStages4 + 6 * 2 == kNumBars4 - 1, "barrier block size");
    int* s_tstart = reinterpret_cast<int*>(smem + Ly.tstart_off);
    int* s_off = reinterpret_cast<int*>(smem + Ly.off_off);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + Ly.misc_off);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + Ly.misc_off + 4);
    volatile int* s_never = reinterpret_cast<volatile int*>(smem + Ly.misc_off + 8);
    int* s_xshift = reinterpret_cast<int*>(smem + Ly.misc_off + 16);   // [2]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = args.offsets ? args.G : 1;
    const int kb = args.K / 32;

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&wfull[s], 1);
            mbar_init(&xfull[s], 1);
            mbar_init(&ready[s], 4);   // one arrival per scale-builder warp
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sfull[b], 1);
            mbar_init(&sempty[b], 2);    // the two weight-scale builders
            mbar_init(&xsfull[b], 1);
            mbar_init(&xsempty[b], 2);   // the two token-scale builders
            mbar_init(&accfull[b], 1);
            mbar_init(&accempty[b], 128);
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
    for (int i = tid; i <= G; i += kThreads4)
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
    const int nk = args.K / 64;                           // MMAs of K = 64 per tile
    const int nss = (args.K + kSSK - 1) / kSSK;           // super-stages per tile
    const int rot = static_cast<int>(blockIdx.x % static_cast<unsigned>(nss));
    auto ss_of = [&](int si) { return si + rot < nss ? si + rot : si + rot - nss; };

    if (warp == 0) {
        // ---------------- weight producer
        if (lane == 0) {
            RingPos c;
            Posted pc, ps;
            int lt = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++lt) {
                const TileInfo ti = decode_tile(t, s_tstart, s_off, G, NT);
                const int sb = lt & 1;
                if (!mbar_wait(&sempty[sb], ((lt >> 1) & 1) ^ 1, s_abort)) { ok = false; break; }
                uint8_t* sdst = wsc + sb * Ly.wsc_bytes;
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
                ps.post(sb, (lt >> 1) & 1);
                for (int si = 0; si < nss; ++si) {
                    const int ss = ss_of(si);
                    if (!mbar_wait(&empty[c.idx], c.ph ^ 1, s_abort)) { ok = false; break; }
                    uint8_t* dst = smem + c.idx * Ly.stage_bytes;
                    mbar_arrive_expect_tx(&wfull[c.idx], kWBytes);
                    const int x = ss * kRowBytes;
                    if (MODE == EPI_SWIGLU) {
                        // lane quarter q: gate features 16q.. (rows 32q..) and up (rows 32q+16..)
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            tma_load_3d(dst + (32 * q) * kRowBytes, &tmap_w, &wfull[c.idx], x,
                                        ti.f * 64 + 16 * q, ti.g);
                            tma_load_3d(dst + (32 * q + 16) * kRowBytes, &tmap_w, &wfull[c.idx], x,
                                        args.I + ti.f * 64 + 16 * q, ti.g);
                        }
                    } else {
                        tma_load_3d(dst, &tmap_w, &wfull[c.idx], x, ti.f * kBM, ti.g);
                    }
                    pc.post(c.idx, c.ph);
                    c.next(S);
                }
            }
            if (!ok) {
                *s_abort = 1;
                record_status(args.status, MXFP4_ERR_TIMEOUT);
                pc.drain(wfull, S, s_never);
                ps.drain(sfull, 2, s_never);
            }
        }
    } else if (warp == 2) {
        // ---------------- activation producer
        if (lane == 0) {
            RingPos c;
            Posted pc, ps;
            int lt = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++lt) {
                const TileInfo ti = decode_tile(t, s_tstart, s_off, G, NT);
                const int sb = lt & 1;
                if (!mbar_wait(&xsempty[sb], ((lt >> 1) & 1) ^ 1, s_abort)) { ok = false; break; }
                // scales of rows row0 .. row0+mrows-1 are one contiguous byte range; copy
                // the 16-byte-aligned range covering it (the buffer has 16 bytes of slack
                // past its end) and tell the builder where row0 starts
                const int64_t b0 = static_cast<int64_t>(ti.row0) * kb;
                const int64_t b1 = b0 + static_cast<int64_t>(ti.mrows) * kb;
                const int64_t a0 = b0 & ~int64_t{15};
                const uint32_t bytes = static_cast<uint32_t>(((b1 + 15) & ~int64_t{15}) - a0);
                s_xshift[sb] = static_cast<int>(b0 - a0);
                mbar_arrive_expect_tx(&xsfull[sb], bytes);   // release: s_xshift is seen by the builder
                bulk_load(xsc + sb * Ly.xsc_bytes, args.x_scales + a0, bytes, &xsfull[sb]);
                ps.post(sb, (lt >> 1) & 1);
                for (int si = 0; si < nss; ++si) {
                    const int ss = ss_of(si);
                    if (!mbar_wait(&empty[c.idx], c.ph ^ 1, s_abort)) { ok = false; break; }
                    mbar_arrive_expect_tx(&xfull[c.idx], NT * kRowBytes);
                    tma_load_2d(smem + c.idx * Ly.stage_bytes + Ly.x_off, &tmap_x, &xfull[c.idx],
                                ss * kRowBytes, ti.row0);
                    pc.post(c.idx, c.ph);
                    c.next(S);
                }
            }
            if (!ok) {
                *s_abort = 1;
                record_status(args.status, MXFP4_ERR_TIMEOUT);
                pc.drain(xfull, S, s_never);
                ps.drain(xsfull, 2, s_never);
            }
        }
    } else if (warp >= 8) {
        // ---------------- scale builders: warp 8 + (operand * 2 + h) writes the atom of
        // scales 4h .. 4h+3 of the super-stage for operand 0 (weights, A) or 1 (tokens, B)
        const int bw = warp - 8;
        const bool is_b = bw >= 2;
        const int h = bw & 1;
        RingPos c;
        int lt = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++lt) {
            const TileInfo ti = decode_tile(t, s_tstart, s_off, G, NT);
            const int sb = lt & 1;
            const uint32_t tph = (lt >> 1) & 1;
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(is_b ? &xsfull[sb] : &sfull[sb], tph, s_abort))) {
                ok = false;
                break;
            }
            // this lane's rows r = lane + 32 m1 (m1 = 0..3) of the operand
            uint32_t row[4];
            bool valid[4];
            const uint32_t base = is_b ? smem_u32(xsc + sb * Ly.xsc_bytes) + s_xshift[sb]
                                       : smem_u32(wsc + sb * Ly.wsc_bytes);
#pragma unroll
            for (int m1 = 0; m1 < 4; ++m1) {
                const int r = lane + 32 * m1;
                if (is_b) {
                    valid[m1] = r < ti.mrows;
                    row[m1] = base + r * kb;
                } else {
                    valid[m1] = MODE == EPI_SWIGLU || ti.f * kBM + r < args.rows_w;
                    row[m1] = base + (MODE == EPI_SWIGLU ? swiglu_staged_row(r) : r) * kb;
                }
            }
            for (int si = 0; si < nss; ++si) {
                const int ss = ss_of(si);
                if (!__all_sync(0xFFFFFFFFu, mbar_wait(&empty[c.idx], c.ph ^ 1, s_abort))) { ok = false; break; }
                const uint32_t atom = smem_u32(smem + c.idx * Ly.stage_bytes + Ly.atoms_off) + bw * kAtom;
                const int k0 = 8 * ss + 4 * h;
                sts128(atom + 16 * lane, scale_word(row[0], k0, kb, valid[0]),
                       scale_word(row[1], k0, kb, valid[1]), scale_word(row[2], k0, kb, valid[2]),
                       scale_word(row[3], k0, kb, valid[3]));
                // generic-proxy writes -> visible to the tensor core's (async-proxy) tcgen05.cp
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                const bool got = mbar_wait(is_b ? &xfull[c.idx] : &wfull[c.idx], c.ph, s_abort);
                if (!__all_sync(0xFFFFFFFFu, got)) { ok = false; break; }
                if (lane == 0) mbar_arrive(&ready[c.idx]);
                c.next(S);
            }
            if (!ok) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(is_b ? &xsempty[sb] : &sempty[sb]);
        }
        if (!ok) {
            *s_abort = 1;
            record_status(args.status, MXFP4_ERR_TIMEOUT);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            RingPos c;
            int lt = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++lt) {
                const int b = lt & 1;
                if (!mbar_wait(&accempty[b], ((lt >> 1) & 1) ^ 1, s_abort)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + b * kAccCols;
                int ki = 0;
                for (int si = 0; si < nss; ++si) {
                    const int ss = ss_of(si);
                    const int nsub = min(4, nk - 4 * ss);
                    if (!mbar_wait(&ready[c.idx], c.ph, s_abort)) { ok = false; break; }
                    tc_fence_after();
                    uint8_t* st = smem + c.idx * Ly.stage_bytes;
                    const uint32_t atoms = smem_u32(st + Ly.atoms_off);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        tmem_cp_32x128b_x4(tmem_base + kSfaCol + 4 * h, rows16_desc(atoms + h * kAtom));
                        tmem_cp_32x128b_x4(tmem_base + kSfbCol + 4 * h, rows16_desc(atoms + (2 + h) * kAtom));
                    }
                    const uint32_t wa = smem_u32(st), xa = smem_u32(st + Ly.x_off);
                    for (int kk = 0; kk < nsub; ++kk, ++ki) {
                        const uint32_t sf_id = (kk & 1) * 2;
                        const uint32_t h = kk >> 1;
                        mma_mxf4(d_tmem, sw128_desc(wa + 32 * kk), sw128_desc(xa + 32 * kk),
                                 idesc_mxf4(kBM, NT, sf_id),
                                 (tmem_base + kSfaCol + 4 * h) | (sf_id << 30),
                                 (tmem_base + kSfbCol + 4 * h) | (sf_id << 30), ki != 0 ? 1u : 0u);
                    }
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
            // wait for every tcgen05 operation issued by this thread before TMEM is released
            tc_commit(drain);
            mbar_wait(drain, 0, s_never);
        }
    } else if (warp >= 4) {   // warps 4-7
        // ---------------- epilogue warpgroup
        const int q = warp & 3;
        int lt = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++lt) {
            const TileInfo ti = decode_tile(t, s_tstart, s_off, G, NT);
            const int b = lt & 1;
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&accfull[b], (lt >> 1) & 1, s_abort))) { ok = false; break; }
            tc_fence_after();
            const uint32_t t_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + b * kAccCols;
            epilogue_tile<MODE, kCW, kAccCols>(args, ti, t_base, q, lane);
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

// Deepest stage ring that fits in shared memory (at least 2 stages).
bool stages4(int NT, int K, int* stages, int* smem) {
    for (int s = kMaxStages4; s >= 2; --s) {
        const Layout4 L = make_layout4(NT, s, K);
        if (L.total <= kSmemLimit4) {
            *stages = s;
            *smem = L.total;
            return true;
        }
    }
    return false;
}

template <int NT, int MODE>
cudaError_t launch4(const CUtensorMap& tw, const CUtensorMap& tx, GemmArgs a, int grid,
                    cudaStream_t stream) {
    int s = 0, smem = 0;
    if (!stages4(NT, a.K, &s, &smem)) return cudaErrorInvalidConfiguration;
    a.code_stages = s;
    a.act_stages = s;
    auto kern = grouped_w4a4_kernel<NT, MODE>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    kern<<<grid, kThreads4, smem, stream>>>(tw, tx, a);
    return cudaGetLastError();
}

template <int MODE>
cudaError_t launch4_mode(int nt, const CUtensorMap& tw, const CUtensorMap& tx, const GemmArgs& a,
                         int grid, cudaStream_t stream) {
    // nt must match the activation map's box rows (the stage expects nt * 128 bytes)
    if (nt == 16) return launch4<16, MODE>(tw, tx, a, grid, stream);
    if (nt == 32) return launch4<32, MODE>(tw, tx, a, grid, stream);
    if (nt == 64) return launch4<64, MODE>(tw, tx, a, grid, stream);
    if (nt == 128) return launch4<128, MODE>(tw, tx, a, grid, stream);
    return cudaErrorInvalidValue;
}

}  // namespace

// Token tiling of the W4A4 engine: NT rows per MMA (16..128) from the mean rows
// per group.
TokenTiling pick_token_tiling_w4a4(int64_t rows, int64_t groups) {
    const int64_t avg = (rows + groups - 1) / (groups > 0 ? groups : 1);
    if (avg <= 16) return {16, 1};
    if (avg <= 32) return {32, 1};
    if (avg <= 64) return {64, 1};
    return {128, 1};
}

int64_t max_gemm_k_w4a4() {
    int64_t k = 256;
    int s, smem;
    while (stages4(128, static_cast<int>(k + 64), &s, &smem)) k += 64;
    return k;
}

// Host launcher.  `tmap_w` covers the weight codes as {K/2, rows_w, G} with box
// {128, 16 (SWIGLU) or 128, 1}; `tmap_x` the activation codes {K/2, rows} with box
// {128, nt}; both with the 128-byte swizzle.  args.x_scales (row-major [rows, K/32])
// must have 16 readable bytes past its end.
cudaError_t launch_grouped_gemm_w4a4(int mode, int nt, const CUtensorMap& tmap_w,
                                     const CUtensorMap& tmap_x, const GemmArgs& args, int grid,
                                     cudaStream_t stream) {
    switch (mode) {
        case EPI_SWIGLU:
            return launch4_mode<EPI_SWIGLU>(nt, tmap_w, tmap_x, args, grid, stream);
        case EPI_WEIGHTED:
            return launch4_mode<EPI_WEIGHTED>(nt, tmap_w, tmap_x, args, grid, stream);
        default:
            return launch4_mode<EPI_PLAIN>(nt, tmap_w, tmap_x, args, grid, stream);
    }
}

}  // namespace mx
