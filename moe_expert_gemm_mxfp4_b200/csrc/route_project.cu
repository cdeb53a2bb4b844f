// Router projection fused with top-k routing on sm_100a tensor cores.
//
// For a block of 128 tokens: logits = x . W_r^T (x bf16 [T, H], router weights
// bf16 [E, H], fp32 accumulation) on tcgen05 kind::f16 with the tokens as the
// MMA's M side and the experts as N (E padded to a multiple of 16; the padding
// rows are the TMA's zero fill), the accumulator [128 tokens x E] in TMEM.  Then
// one thread per token takes the top-k of its E logits (larger logit first, lower
// expert id among equal logits, NaN below every number; as one sortable 64-bit key
// per expert, kept in a sorted register list by max/min swaps), the softmax over
// the k selected logits (fp32), and writes ids and weights.  The logits never reach
// global memory (unless the caller asks for a copy).  Last, each warp builds the
// per-expert counts and the pairs' stable ranks of two 8-token chunks at a time
// from warp match masks, in the format the routing's scan and scatter kernels
// take, so the rest of the routing is shared.
//
// The pages run the MoE layer's routing inside a downloadable MegaBlocks MoE kernel
// and name a top-k kernel (agentlenshq.com, "Transformers 4.40 performance upgrades
// for OpenAI GPT-OSS ...", section "Zero-Build Kernels from the Hub"); the router
// itself (a bias-free linear map, one logit per expert) is a reading.
//
// Roles: a thread-block cluster of CS CTAs (1 to 8, one 128-token tile; CS is
// chosen at launch so that the tiles times CS fill the SMs) splits the tile's K
// range: CTA r of the cluster takes K stages [r nk / CS, (r+1) nk / CS).  In each CTA
// (4 warps) thread 0 streams the x and W_r tiles of its stages into a ring (TMA,
// 128B swizzle) and thread 32 issues the MMAs into the CTA's own TMEM accumulator,
// releasing each stage with a commit.  Then CTAs 1..CS-1 copy their partial logits
// to shared memory (the ring, now idle), and after a cluster barrier CTA 0's 128
// threads (one per token) add them to its own, in rank order, through distributed
// shared memory: the sum is the same for every run.  CTA 0 alone runs the top-k
// epilogue; a second cluster barrier keeps the other CTAs' shared memory alive until
// it has read it.  Every mbarrier wait is bounded (MXFP4_ERR_TIMEOUT in the status
// word); the pipeline's waits poll without suspending the thread.
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

constexpr int kRpMaxCluster = 8;

struct RpLayout {
    int stages, stage_bytes, bar_off, ids_off, cnt_off, misc_off, total;
};

// want: the CTA's K stages (the ring needs no more).  The ring also holds the
// partial logits [128 x (e_pad + 4)] fp32 once the MMAs are done.
__host__ __device__ inline RpLayout rp_layout(int e_pad, int want) {
    RpLayout L;
    L.stage_bytes = kRpXTile + e_pad * kRpBK * 2;
    const int fixed = (2 * kRpMaxStages + 1) * 8 + kRpTok * kRpMaxTopK * 4 + 4 * kRpMaxE * 4 + 16 + 1024;
    int fit = (kRpSmemLimit - fixed) / L.stage_bytes;
    if (fit > kRpMaxStages) fit = kRpMaxStages;
    const int part_stages = (kRpTok * (e_pad + 4) * 4 + L.stage_bytes - 1) / L.stage_bytes;
    const int st = want > part_stages ? want : part_stages;
    L.stages = st < fit ? st : fit;
    L.bar_off = L.stages * L.stage_bytes;
    L.ids_off = L.bar_off + (2 * kRpMaxStages + 1) * 8;
    L.cnt_off = L.ids_off + kRpTok * kRpMaxTopK * 4;
    L.misc_off = L.cnt_off + 4 * kRpMaxE * 4;
    L.total = L.misc_off + 16 + 1024;   // + slack for the 1024-B alignment of the base
    return L;
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}
// Every thread of every CTA of the cluster; release/acquire at cluster scope.
__device__ __forceinline__ void cluster_barrier() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ float4 ld_cluster_f32x4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
    return v;
}

// Expert order: larger logit first, lower id among equal logits; NaN below every
// number, NaNs by id (the order of the routing kernel).  As one unsigned 64-bit key
// per (logit, expert): the high word orders the logits (a float's bits with the sign
// folded so that integer order is numeric order; -0 taken as +0, so that the two
// zeros tie; every NaN mapped to 0, below -inf), the low word is ~id (lower id
// larger).  A larger key is a better expert, so the running top-k is a sorted list
// kept by max/min swaps, with no branches.
__device__ __forceinline__ uint64_t rp_key(float v, int id) {
    uint32_t u = __float_as_uint(v);
    if (u == 0x80000000u) u = 0u;
    uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    if (v != v) ord = 0u;
    return (static_cast<uint64_t>(ord) << 32) | static_cast<uint32_t>(~id);
}
__device__ __forceinline__ float rp_key_value(uint64_t key) {
    const uint32_t ord = static_cast<uint32_t>(key >> 32);
    if (ord == 0u) return __uint_as_float(0x7FC00000u);
    return __uint_as_float((ord & 0x80000000u) ? (ord & 0x7FFFFFFFu) : ~ord);
}
__device__ __forceinline__ int rp_key_id(uint64_t key) { return static_cast<int>(~static_cast<uint32_t>(key)); }

// Insert a key into the sorted list sel[0..KM) (KM >= top_k; the worst key drops out).
// (The callers keep their loops rolled: this epilogue runs once per CTA, so its
// instructions come cold from L2 and a short body matters more than unrolling.)
template <int KM>
__device__ __forceinline__ void rp_insert(uint64_t key, uint64_t* sel) {
#pragma unroll
    for (int j = 0; j < KM; ++j) {
        const uint64_t hi = key > sel[j] ? key : sel[j];
        key = key > sel[j] ? sel[j] : key;
        sel[j] = hi;
    }
}

// The top-KM keys of one token's E logits (row `row` of shared memory).
template <int KM>
__device__ __forceinline__ void rp_topk_row(const float* row, int E, uint64_t* sel) {
#pragma unroll 1
    for (int e = 0; e < E; ++e) rp_insert<KM>(rp_key(row[e], e), sel);
}

__global__ void __launch_bounds__(kRpThreads, 1)
route_project_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                     int T, int H, int E, int e_pad, int k, int32_t* __restrict__ ids,
                     float* __restrict__ weights, int32_t* __restrict__ chunk_counts,
                     int32_t* __restrict__ local_rank, float* __restrict__ logits_out, unsigned* status) {
    const int nk = H / kRpBK;
    const int cs = static_cast<int>(cluster_size());
    const uint32_t rank = cluster_rank();
    // this CTA's K stages: [k0, k0 + nkc), at least one (the launch keeps cs <= nk)
    const int k0 = static_cast<int>(rank) * nk / cs;
    const int nkc = (static_cast<int>(rank) + 1) * nk / cs - k0;
    const RpLayout Ly = rp_layout(e_pad, (nk + cs - 1) / cs);
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
    const int tok0 = static_cast<int>(blockIdx.x) / cs * kRpTok;
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
        for (int i = 0; i < nkc; ++i, ++issued) {
            const int ks = k0 + i;
            const int s = i % NS;
            const uint32_t ph = (i / NS) & 1;
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
        for (int i = 0; i < nkc; ++i) {
            const int s = i % NS;
            if (!mbar_wait_spin(&full[s], (i / NS) & 1, s_abort)) { ok = false; break; }
            tc_fence_after();
            const uint32_t xa = smem_u32(smem + s * Ly.stage_bytes);
            const uint32_t wa = xa + kRpXTile;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                mma_bf16_ss(tmem, sw128_desc(xa + 32 * j), sw128_desc(wa + 32 * j), idesc,
                            (i | j) != 0 ? 1u : 0u);
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
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    // ---------------- every CTA: its partial logits -> shared memory (the idle ring),
    // row tid; the row stride keeps rows 16-byte aligned, so that the block is one
    // contiguous run of float4s for the cluster reduction below
    const int pld = e_pad + 4;
    float* s_part = reinterpret_cast<float*>(smem);
    float* my_row = s_part + tid * pld;
#pragma unroll 1
    for (int c0 = 0; c0 < e_pad; c0 += 16) {
        uint32_t r[16];
        tmem_ld_x16(lane_base + c0, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) my_row[c0 + i] = __uint_as_float(r[i]);
    }
    if (cs > 1) cluster_barrier();   // the partials are visible cluster-wide
    if (rank == 0) {
    // CTA 0 adds the other CTAs' partial blocks to its own, in rank order: thread i
    // owns float4s i, i + 128, ... of the block for every rank, so each logit's sum
    // is taken in the same order on every run; the reads of a warp are 512
    // contiguous bytes of the other CTA's shared memory
    if (cs > 1) {
        float4* blk = reinterpret_cast<float4*>(s_part);
        const int n4 = kRpTok * pld / 4;
        constexpr int kB = 8;   // remote loads in flight per thread
#pragma unroll 1
        for (int q = 1; q < cs; ++q) {
            const uint32_t src = map_to_rank(smem_u32(s_part), static_cast<uint32_t>(q));
#pragma unroll 1
            for (int i0 = tid; i0 < n4; i0 += kB * kRpThreads) {
                float4 v[kB];
#pragma unroll
                for (int b = 0; b < kB; ++b) {
                    const int i = i0 + b * kRpThreads;
                    v[b] = i < n4 ? ld_cluster_f32x4(src + 16u * static_cast<uint32_t>(i)) : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int b = 0; b < kB; ++b) {
                    const int i = i0 + b * kRpThreads;
                    if (i < n4) {
                        float4 a = blk[i];
                        a.x += v[b].x;
                        a.y += v[b].y;
                        a.z += v[b].z;
                        a.w += v[b].w;
                        blk[i] = a;
                    }
                }
            }
        }
        __syncthreads();   // every token's row is summed
    }
    if (logits_out && t < T) {
#pragma unroll 1
        for (int e = 0; e < E; ++e) logits_out[static_cast<int64_t>(t) * E + e] = my_row[e];
    }
    // running top-k: sel[0] the best; slots past k only ever hold worse keys
    uint64_t sel[kRpMaxTopK];
#pragma unroll
    for (int j = 0; j < kRpMaxTopK; ++j) sel[j] = 0;   // below every real key
    if (!*s_abort) {
        if (k <= 2) rp_topk_row<2>(my_row, E, sel);
        else if (k <= 4) rp_topk_row<4>(my_row, E, sel);
        else rp_topk_row<kRpMaxTopK>(my_row, E, sel);
    }
    float sel_v[kRpMaxTopK];
    int sel_id[kRpMaxTopK];
#pragma unroll
    for (int j = 0; j < kRpMaxTopK; ++j) {
        sel_v[j] = rp_key_value(sel[j]);
        sel_id[j] = rp_key_id(sel[j]);
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
    }   // rank == 0

    tc_fence_before();
    if (cs > 1) cluster_barrier();   // CTA 0 is done reading the others' shared memory
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, ncols);
    }
}

}  // namespace

// Cluster size for a launch: enough CTAs per token tile to fill the SMs (at most 8,
// a power of two, no more than the K stages), reduced while the GPU cannot hold a
// cluster of that size with its shared memory.
static int rp_cluster_size(int64_t T, int64_t H, int e_pad, int sm_count) {
    const int64_t ntiles = (T + kRpTok - 1) / kRpTok;
    const int64_t nk = H / kRpBK;
    int cs = 1;
    while (cs < kRpMaxCluster && 2 * cs <= nk && ntiles * 2 * cs <= sm_count) cs *= 2;
    if (e_pad > 64 && cs > 4) cs = 4;   // the sum reads (cs - 1) x e_pad partials per token
    return cs;
}

int route_project_smem_bytes(int64_t E, int64_t H, int cs) {
    const int e_pad = static_cast<int>((E + 15) / 16 * 16);
    const int nk = static_cast<int>(H / kRpBK);
    return rp_layout(e_pad, (nk + cs - 1) / cs).total;
}

cudaError_t launch_route_project(const CUtensorMap& tmap_x, const CUtensorMap& tmap_w, int64_t T,
                                 int64_t H, int64_t E, int top_k, int32_t* ids, float* weights,
                                 int32_t* chunk_counts, int32_t* local_rank, float* logits_out,
                                 int sm_count, unsigned* status, cudaStream_t stream) {
    const int e_pad = static_cast<int>((E + 15) / 16 * 16);
    const int64_t ntiles = (T + kRpTok - 1) / kRpTok;
    cudaError_t e = cudaSuccess;
    for (int cs = rp_cluster_size(T, H, e_pad, sm_count);; cs /= 2) {
        const RpLayout L = rp_layout(e_pad, static_cast<int>((H / kRpBK + cs - 1) / cs));
        if (L.stages * L.stage_bytes < kRpTok * (e_pad + 4) * 4) return cudaErrorInvalidConfiguration;
        const int smem = L.total;
        if ((e = cudaFuncSetAttribute(route_project_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
            cudaSuccess)
            return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(ntiles * cs), 1, 1);
        cfg.blockDim = dim3(kRpThreads, 1, 1);
        cfg.dynamicSmemBytes = static_cast<size_t>(smem);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = static_cast<unsigned>(cs);
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cs > 1) {
            int nclusters = 0;
            if (cudaOccupancyMaxActiveClusters(&nclusters, route_project_kernel, &cfg) != cudaSuccess ||
                nclusters < 1) {
                (void)cudaGetLastError();   // clear a refusal; try a smaller cluster
                continue;
            }
        }
        return cudaLaunchKernelEx(&cfg, route_project_kernel, tmap_x, tmap_w, static_cast<int>(T),
                                  static_cast<int>(H), static_cast<int>(E), e_pad, top_k, ids, weights,
                                  chunk_counts, local_rank, logits_out, status);
    }
}

}  // namespace mx
