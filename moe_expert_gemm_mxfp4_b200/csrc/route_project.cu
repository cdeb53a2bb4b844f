// Router projection fused with top-k routing on sm_100a tensor cores.
//
// For a block of 128 tokens: logits = x . W_r^T (x bf16 [T, H], router weights
// bf16 [E, H], fp32 accumulation) on tcgen05 kind::f16 with the tokens as the
// MMA's M side and the experts as N (E padded to a multiple of 16; the padding
// rows are the TMA's zero fill), the accumulator [128 tokens x E] in TMEM.  Then
// one thread per token reads its E logits from TMEM and keeps the running top-k
// in registers (larger logit first, lower expert id among equal logits, NaN below
// every number), takes the softmax over the k selected logits (fp32), and writes
// ids and weights.  The logits never reach global memory (unless the caller asks
// for a copy).  Last, each warp builds the per-expert counts and the pairs' stable
// ranks of two 8-token chunks at a time from warp match masks, in the format the
// routing's scan and scatter kernels take, so the rest of the routing is shared.
//
// The pages run the MoE layer's routing inside a downloadable MegaBlocks MoE kernel
// and name a top-k kernel (agentlenshq.com, "Transformers 4.40 performance upgrades
// for OpenAI GPT-OSS ...", section "Zero-Build Kernels from the Hub"); the router
// itself (a bias-free linear map, one logit per expert) is a reading.
//
// Roles (one CTA per 128 tokens, 4 warps): thread 0 streams the x and W_r tiles of
// each 64-wide K stage into a ring (TMA, 128B swizzle); thread 32 issues the MMAs
// and releases each stage with a commit; afterwards all 128 threads run the top-k
// epilogue.  Every wait is bounded (MXFP4_ERR_TIMEOUT in the status word); the
// pipeline's waits poll without suspending the thread (one CTA's K loop is a chain of
// such waits, so a late wake-up would cost each stage).
#include "common.cuh"
#include "internal.h"

namespace mx {

namespace {

constexpr int kRpTok = 128;        // tokens per CTA = TMEM lanes
constexpr int kRpThreads = 128;
constexpr int kRpBK = 64;          // K per stage (128 bytes of bf16 per row)
constexpr int kRpMaxStages = 12;   // ring depth: as many stages as fit (a K stage is a round trip to L2/HBM)
constexpr int kRpSmemLimit = 227 * 1024;
constexpr int kRpMaxTopK = 8;
constexpr int kRpMaxE = 256;
constexpr int kRpXTile = kRpTok * kRpBK * 2;     // 16 KB

struct RpLayout {
    int stages, stage_bytes, bar_off, ids_off, cnt_off, misc_off, total;
};

__host__ __device__ inline RpLayout rp_layout(int e_pad) {
    RpLayout L;
    L.stage_bytes = kRpXTile + e_pad * kRpBK * 2;
    const int fixed = (2 * kRpMaxStages + 1) * 8 + kRpTok * kRpMaxTopK * 4 + 4 * kRpMaxE * 4 + 16 + 1024;
    L.stages = (kRpSmemLimit - fixed) / L.stage_bytes;
    if (L.stages > kRpMaxStages) L.stages = kRpMaxStages;
    L.bar_off = L.stages * L.stage_bytes;
    L.ids_off = L.bar_off + (2 * kRpMaxStages + 1) * 8;
    L.cnt_off = L.ids_off + kRpTok * kRpMaxTopK * 4;
    L.misc_off = L.cnt_off + 4 * kRpMaxE * 4;
    L.total = L.misc_off + 16 + 1024;   // + slack for the 1024-B alignment of the base
    return L;
}

// Expert order: larger logit first, lower id among equal logits; NaN below every
// number, NaNs by id (the order of the routing kernel).
__device__ __forceinline__ bool rp_better(float v, int id, float bv, int bid) {
    const bool vn = v != v, bn = bv != bv;
    if (vn != bn) return bn;
    if (!vn && v != bv) return v > bv;
    return id < bid;
}

__global__ void __launch_bounds__(kRpThreads, 1)
route_project_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                     int T, int H, int E, int e_pad, int k, int32_t* __restrict__ ids,
                     float* __restrict__ weights, int32_t* __restrict__ chunk_counts,
                     int32_t* __restrict__ local_rank, float* __restrict__ logits_out, unsigned* status) {
    const RpLayout Ly = rp_layout(e_pad);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Ly.bar_off);
    const int NS = Ly.stages;
    uint64_t* full = bars;
    uint64_t* empty = bars + kRpMaxStages;
    uint64_t* done = bars + 2 * kRpMaxStages;
    int32_t* s_ids = reinterpret_cast<int32_t*>(smem + Ly.ids_off);
    int32_t* s_cnt = reinterpret_cast<int32_t*>(smem + Ly.cnt_off);    // [4 warps][kRpMaxE]
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + Ly.misc_off);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + Ly.misc_off + 4);
    volatile int* s_never = reinterpret_cast<volatile int*>(smem + Ly.misc_off + 8);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tok0 = blockIdx.x * kRpTok;
    const int nk = H / kRpBK;
    const uint32_t ncols = e_pad <= 32 ? 32 : e_pad <= 64 ? 64 : e_pad <= 128 ? 128 : 256;

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        *s_abort = 0;
        *s_never = 0;
        fence_mbar_init();
        prefetch_tmap(&tmap_x);
        prefetch_tmap(&tmap_w);
    }
    for (int i = tid; i < 4 * kRpMaxE; i += kRpThreads) s_cnt[i] = 0;
    if (warp == 1) {
        tmem_alloc(s_tmem, ncols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    bool ok = true;

    if (tid == 0) {
        // ---------------- producer: x rows tok0.. (past T: zero fill), W_r rows 0..e_pad-1
        const uint32_t bytes = static_cast<uint32_t>(Ly.stage_bytes);
        int issued = 0;
        for (int ks = 0; ks < nk; ++ks, ++issued) {
            const int s = ks % NS;
            const uint32_t ph = (ks / NS) & 1;
            if (!mbar_wait_spin(&empty[s], ph ^ 1, s_abort)) { ok = false; break; }
            uint8_t* st = smem + s * Ly.stage_bytes;
            mbar_arrive_expect_tx(&full[s], bytes);
            tma_load_2d(st, &tmap_x, &full[s], ks * kRpBK, tok0);
            tma_load_2d(st + kRpXTile, &tmap_w, &full[s], ks * kRpBK, 0);
        }
        if (!ok) {
            *s_abort = 1;
            record_status(status, MXFP4_ERR_TIMEOUT);
            for (int i = issued > NS ? issued - NS : 0; i < issued; ++i)
                mbar_wait(&full[i % NS], (i / NS) & 1, s_never);
        }
    } else if (tid == 32) {
        // ---------------- MMA issuer: D[128 x e_pad] += x_tile . W_tile^T, K = 16 per MMA
        const uint32_t idesc = idesc_bf16_f32(kRpTok, e_pad);
        for (int ks = 0; ks < nk; ++ks) {
            const int s = ks % NS;
            if (!mbar_wait_spin(&full[s], (ks / NS) & 1, s_abort)) { ok = false; break; }
            tc_fence_after();
            const uint32_t xa = smem_u32(smem + s * Ly.stage_bytes);
            const uint32_t wa = xa + kRpXTile;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                mma_bf16_ss(tmem, sw128_desc(xa + 32 * j), sw128_desc(wa + 32 * j), idesc,
                            (ks | j) != 0 ? 1u : 0u);
            tc_commit(&empty[s]);
        }
        if (!ok) {
            *s_abort = 1;
            record_status(status, MXFP4_ERR_TIMEOUT);
        }
        tc_commit(done);   // also drains every MMA issued before TMEM is released
    }
    __syncwarp();

    // ---------------- top-k epilogue: thread tid = token tok0 + tid (TMEM lane tid)
    // (waited for even after an abort: the MMAs in flight must finish before TMEM is
    // read or released, and the issuer commits `done` on every path)
    const bool got = mbar_wait_spin(done, 0, s_never);
    if (!__all_sync(0xFFFFFFFFu, got)) {
        *s_abort = 1;
        record_status(status, MXFP4_ERR_TIMEOUT);
    }
    tc_fence_after();
    const int t = tok0 + tid;
    float sel_v[kRpMaxTopK];
    int sel_id[kRpMaxTopK];
#pragma unroll
    for (int j = 0; j < kRpMaxTopK; ++j) {
        sel_v[j] = __uint_as_float(0x7FC00000u);   // NaN: below every number
        sel_id[j] = 0x7FFFFFFF;
    }
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    if (!*s_abort) {
        for (int c0 = 0; c0 < e_pad; c0 += 16) {
            uint32_t r[16];
            tmem_ld_x16(lane_base + c0, r);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int e = c0 + i;
                if (e >= E) break;
                float v = __uint_as_float(r[i]);
                if (logits_out && t < T) logits_out[static_cast<int64_t>(t) * E + e] = v;
                // insert (v, e) into the sorted top-k list if it beats the k-th entry
                int id = e;
#pragma unroll
                for (int j = 0; j < kRpMaxTopK; ++j) {
                    if (j < k && (sel_id[j] == 0x7FFFFFFF || rp_better(v, id, sel_v[j], sel_id[j]))) {
                        const float tv = sel_v[j];
                        const int ti = sel_id[j];
                        sel_v[j] = v;
                        sel_id[j] = id;
                        v = tv;
                        id = ti;
                    }
                }
            }
        }
    }
    if (*s_abort) {   // the result is void (status recorded), but later kernels index by these ids
#pragma unroll
        for (int j = 0; j < kRpMaxTopK; ++j) sel_id[j] = j;
    }
    tc_fence_before();
    // softmax over the k selected logits, fp32, slots in order
    float z[kRpMaxTopK], sum = 0.f;
#pragma unroll
    for (int j = 0; j < kRpMaxTopK; ++j) {
        z[j] = 0.f;
        if (j < k) {
            z[j] = expf(sel_v[j] - sel_v[0]);
            sum += z[j];
        }
    }
    if (t < T) {
#pragma unroll
        for (int j = 0; j < kRpMaxTopK; ++j) {
            if (j < k) {
                ids[static_cast<int64_t>(t) * k + j] = sel_id[j];
                weights[static_cast<int64_t>(t) * k + j] = z[j] / sum;
                s_ids[tid * k + j] = sel_id[j];
            }
        }
    }
    __syncthreads();

    // ---------------- per-8-token-chunk counts and stable ranks (warp w: chunks w, w+4, ...)
    int32_t* cnt = s_cnt + warp * kRpMaxE;
    for (int c = warp; c < kRpTok / 8; c += 4) {
        const int ct0 = tok0 + 8 * c;
        if (ct0 >= T) break;
        const int npairs = min(8, T - ct0) * k;     // at most 64
        const int32_t* pid = s_ids + 8 * c * k;
        // pass A: pairs lane; pass B: pairs 32 + lane
        const bool va = lane < npairs, vb = 32 + lane < npairs;
        const int ea = va ? pid[lane] : kRpMaxE + lane;
        const int eb = vb ? pid[32 + lane] : kRpMaxE + lane;
        const uint32_t lt = (1u << lane) - 1u;
        const uint32_t ma = __match_any_sync(0xFFFFFFFFu, ea);
        const uint32_t mb = __match_any_sync(0xFFFFFFFFu, eb);
        if (va && (ma & lt) == 0) cnt[ea] = __popc(ma);
        __syncwarp();
        const int64_t p0 = static_cast<int64_t>(ct0) * k;
        if (va) local_rank[p0 + lane] = __popc(ma & lt);
        if (vb) local_rank[p0 + 32 + lane] = __popc(mb & lt) + cnt[eb];
        __syncwarp();
        if (vb && (mb & lt) == 0) cnt[eb] += __popc(mb);
        __syncwarp();
        const int64_t chunk = ct0 / 8;
        for (int e = lane; e < E; e += 32) {
            chunk_counts[chunk * E + e] = cnt[e];
            cnt[e] = 0;
        }
        __syncwarp();
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, ncols);
    }
}

}  // namespace

int route_project_smem_bytes(int64_t E) {
    const int e_pad = static_cast<int>((E + 15) / 16 * 16);
    return rp_layout(e_pad).total;
}

cudaError_t launch_route_project(const CUtensorMap& tmap_x, const CUtensorMap& tmap_w, int64_t T,
                                 int64_t H, int64_t E, int top_k, int32_t* ids, float* weights,
                                 int32_t* chunk_counts, int32_t* local_rank, float* logits_out,
                                 unsigned* status, cudaStream_t stream) {
    const int e_pad = static_cast<int>((E + 15) / 16 * 16);
    const int smem = rp_layout(e_pad).total;
    cudaError_t e = cudaFuncSetAttribute(route_project_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = static_cast<unsigned>((T + kRpTok - 1) / kRpTok);
    route_project_kernel<<<grid, kRpThreads, smem, stream>>>(
        tmap_x, tmap_w, static_cast<int>(T), static_cast<int>(H), static_cast<int>(E), e_pad, top_k, ids,
        weights, chunk_counts, local_rank, logits_out, status);
    return cudaGetLastError();
}

}  // namespace mx
