// MoE routing for sm_100a: top-k + softmax, per-expert histogram with warp
// ballots, prefix sums, the expert-sorted permutation of (token, slot) pairs,
// the gather of token rows into that order, and the deterministic combine.
//
// The pages route MoE tokens through a downloadable MegaBlocks kernel and name
// a top-k kernel (agentlenshq.com, "Transformers 4.40 performance upgrades for
// OpenAI GPT-OSS ...", section "Zero-Build Kernels from the Hub"); the routing
// rule itself is a reading: top-k by (logit desc, expert id asc), softmax over
// the k selected logits, pairs p = t*k + j grouped by expert in ascending p.
//
// Kernels (one stream, no host synchronization):
//   route_topk_count  per 64-token chunk: top-k/softmax (one warp per token),
//                     then the chunk's per-expert counts and each pair's stable
//                     rank inside the chunk (warp multisplit by ballots over the
//                     bits of the expert id);
//   route_scan        per expert: exclusive scan of the chunk counts; counts,
//                     offsets (exclusive scan over experts);
//   route_scatter     position of every pair, perm / inv / sorted weights, and
//                     optionally the gather of its token row;
//   moe_combine       out[t] = bf16(sum_j y[inv[t*k + j]]), fp32 rows summed in slot order.
#include "common.cuh"
#include "internal.h"

namespace mx {

constexpr int kRouteTokPerCta = 64;
constexpr int kRouteThreads = 256;
constexpr int kMaxTopK = 8;
constexpr int kMaxExperts = 256;

namespace {

__device__ __forceinline__ bool better(float v, int id, float bv, int bid) {
    return v > bv || (v == bv && id < bid);
}

__global__ void __launch_bounds__(kRouteThreads)
route_topk_count_kernel(const float* __restrict__ logits, int T, int E, int k,
                        int32_t* __restrict__ ids, float* __restrict__ weights,
                        int32_t* __restrict__ chunk_counts, int32_t* __restrict__ local_rank) {
    __shared__ int32_t s_ids[kRouteTokPerCta * kMaxTopK];
    __shared__ int32_t s_seg[2 * (kRouteThreads / 32)][kMaxExperts];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int t0 = blockIdx.x * kRouteTokPerCta;
    const int ntok = min(kRouteTokPerCta, T - t0);

    for (int i = threadIdx.x; i < 2 * (kRouteThreads / 32) * kMaxExperts; i += blockDim.x)
        (&s_seg[0][0])[i] = 0;

    // ---- top-k + softmax, one warp per token
    for (int lt = wid; lt < ntok; lt += kRouteThreads / 32) {
        const int t = t0 + lt;
        float v[kMaxExperts / 32];
#pragma unroll
        for (int i = 0; i < kMaxExperts / 32; ++i) {
            const int e = lane + 32 * i;
            v[i] = e < E ? logits[static_cast<int64_t>(t) * E + e] : -INFINITY;
        }
        uint32_t taken = 0;
        float sel_v[kMaxTopK];
        int sel_id[kMaxTopK];
        for (int j = 0; j < k; ++j) {
            float bv = -INFINITY;
            int bid = 0x7FFFFFFF;
#pragma unroll
            for (int i = 0; i < kMaxExperts / 32; ++i) {
                const int e = lane + 32 * i;
                if (e < E && !((taken >> i) & 1u) && (bid == 0x7FFFFFFF || better(v[i], e, bv, bid))) {
                    bv = v[i];
                    bid = e;
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, o);
                const int oid = __shfl_xor_sync(0xFFFFFFFFu, bid, o);
                if (oid != 0x7FFFFFFF && (bid == 0x7FFFFFFF || better(ov, oid, bv, bid))) {
                    bv = ov;
                    bid = oid;
                }
            }
            if ((bid & 31) == lane) taken |= 1u << (bid >> 5);
            sel_v[j] = bv;
            sel_id[j] = bid;
        }
        if (lane == 0) {
            float z[kMaxTopK];
            float sum = 0.f;
            for (int j = 0; j < k; ++j) {
                z[j] = expf(sel_v[j] - sel_v[0]);
                sum += z[j];
            }
            for (int j = 0; j < k; ++j) {
                ids[static_cast<int64_t>(t) * k + j] = sel_id[j];
                weights[static_cast<int64_t>(t) * k + j] = z[j] / sum;
                s_ids[lt * k + j] = sel_id[j];
            }
        }
    }
    __syncthreads();

    // ---- per-chunk histogram and stable ranks (warp multisplit by ballots)
    const int npairs = ntok * k;
    int nbits = 0;
    while ((1 << nbits) < E) ++nbits;
    const uint32_t lt_mask = (1u << lane) - 1u;
    int my_e[2], my_rank[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int i = r * kRouteThreads + threadIdx.x;
        const bool valid = i < npairs;
        const int e = valid ? s_ids[i] : 0;
        uint32_t peers = __ballot_sync(0xFFFFFFFFu, valid);
        for (int b = 0; b < nbits; ++b) {
            const uint32_t bit = (e >> b) & 1;
            const uint32_t bal = __ballot_sync(0xFFFFFFFFu, bit);
            peers &= bit ? bal : ~bal;
        }
        my_e[r] = e;
        my_rank[r] = __popc(peers & lt_mask);
        if (valid && (peers & lt_mask) == 0) s_seg[r * (kRouteThreads / 32) + wid][e] = __popc(peers);
    }
    __syncthreads();
    const int nseg = 2 * (kRouteThreads / 32);
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0;
        for (int sg = 0; sg < nseg; ++sg) {
            const int c = s_seg[sg][e];
            s_seg[sg][e] = run;
            run += c;
        }
        chunk_counts[static_cast<int64_t>(blockIdx.x) * E + e] = run;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int i = r * kRouteThreads + threadIdx.x;
        if (i < npairs)
            local_rank[static_cast<int64_t>(t0) * k + i] =
                s_seg[r * (kRouteThreads / 32) + wid][my_e[r]] + my_rank[r];
    }
}

__global__ void __launch_bounds__(kMaxExperts)
route_scan_kernel(int32_t* __restrict__ chunk_counts, int n_chunks, int E,
                  int32_t* __restrict__ counts, int32_t* __restrict__ offsets) {
    __shared__ int32_t s[kMaxExperts];
    const int e = threadIdx.x;
    int total = 0;
    if (e < E) {
        for (int c = 0; c < n_chunks; ++c) {
            int32_t* p = chunk_counts + static_cast<int64_t>(c) * E + e;
            const int v = *p;
            *p = total;
            total += v;
        }
        counts[e] = total;
    }
    s[e] = e < E ? total : 0;
    __syncthreads();
    for (int o = 1; o < kMaxExperts; o <<= 1) {     // inclusive Hillis-Steele scan
        const int add = e >= o ? s[e - o] : 0;
        __syncthreads();
        s[e] += add;
        __syncthreads();
    }
    if (e < E) offsets[e + 1] = s[e];
    if (e == 0) offsets[0] = 0;
}

// One warp per pair: its sorted position, the routing tables and, if `x` is
// given, the copy of its token's row into the expert-sorted activation matrix.
__global__ void __launch_bounds__(kRouteThreads)
route_scatter_kernel(const int32_t* __restrict__ ids, const float* __restrict__ weights,
                     const int32_t* __restrict__ chunk_base, const int32_t* __restrict__ local_rank,
                     const int32_t* __restrict__ offsets, int64_t P, int k, int E,
                     int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                     float* __restrict__ w_sorted, const uint4* __restrict__ x, int64_t row_vec,
                     uint4* __restrict__ x_sorted) {
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t p = warp0; p < P; p += nwarps) {
        const int e = ids[p];
        const int64_t t = p / k;
        const int64_t chunk = t / kRouteTokPerCta;
        const int64_t pos = static_cast<int64_t>(offsets[e]) + chunk_base[chunk * E + e] + local_rank[p];
        if (lane == 0) {
            perm[pos] = static_cast<int32_t>(p);
            inv[p] = static_cast<int32_t>(pos);
            if (w_sorted) w_sorted[pos] = weights[p];
        }
        if (x) {
            const uint4* src = x + t * row_vec;
            uint4* dst = x_sorted + pos * row_vec;
            for (int64_t c = lane; c < row_vec; c += 32) dst[c] = __ldg(src + c);
        }
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 r = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&r);
}

// One warp per token; its k fp32 rows are summed in slot order j = 0..k-1 and
// rounded once to bf16.
__global__ void __launch_bounds__(kRouteThreads)
moe_combine_kernel(const float4* __restrict__ y_sorted, const int32_t* __restrict__ inv,
                   int64_t T, int k, int64_t row_vec8, uint4* __restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t t = warp0; t < T; t += nwarps) {
        int64_t rows[kMaxTopK];
        for (int j = 0; j < k; ++j) rows[j] = inv[t * k + j];
        for (int64_t c = lane; c < row_vec8; c += 32) {
            float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            for (int j = 0; j < k; ++j) {
                const float4* src = y_sorted + (rows[j] * row_vec8 + c) * 2;
                const float4 u = __ldcs(src), v = __ldcs(src + 1);
                a[0] += u.x; a[1] += u.y; a[2] += u.z; a[3] += u.w;
                a[4] += v.x; a[5] += v.y; a[6] += v.z; a[7] += v.w;
            }
            uint4 o;
            o.x = pack_bf16x2(a[0], a[1]);
            o.y = pack_bf16x2(a[2], a[3]);
            o.z = pack_bf16x2(a[4], a[5]);
            o.w = pack_bf16x2(a[6], a[7]);
            out[t * row_vec8 + c] = o;
        }
    }
}

}  // namespace

size_t route_tmp_bytes(int64_t T, int64_t E, int top_k) {
    const int64_t n_chunks = (T + kRouteTokPerCta - 1) / kRouteTokPerCta;
    return static_cast<size_t>(n_chunks * E + T * top_k) * sizeof(int32_t);
}

cudaError_t launch_route(const float* logits, int64_t T, int64_t E, int top_k, int32_t* ids,
                         float* weights, int32_t* counts, int32_t* offsets, int32_t* perm,
                         int32_t* inv, float* w_sorted, void* tmp, const void* x, int64_t H,
                         void* x_sorted, int sm_count, cudaStream_t stream) {
    const int64_t n_chunks = (T + kRouteTokPerCta - 1) / kRouteTokPerCta;
    int32_t* chunk_counts = static_cast<int32_t*>(tmp);
    int32_t* local_rank = chunk_counts + n_chunks * E;
    route_topk_count_kernel<<<static_cast<unsigned>(n_chunks), kRouteThreads, 0, stream>>>(
        logits, static_cast<int>(T), static_cast<int>(E), top_k, ids, weights, chunk_counts,
        local_rank);
    route_scan_kernel<<<1, kMaxExperts, 0, stream>>>(chunk_counts, static_cast<int>(n_chunks),
                                                     static_cast<int>(E), counts, offsets);
    const int64_t P = T * top_k;
    const int64_t warps_needed = P;
    int64_t grid = (warps_needed + kRouteThreads / 32 - 1) / (kRouteThreads / 32);
    const int64_t cap = static_cast<int64_t>(sm_count) * 8;
    if (grid > cap) grid = cap;
    route_scatter_kernel<<<static_cast<unsigned>(grid), kRouteThreads, 0, stream>>>(
        ids, weights, chunk_counts, local_rank, offsets, P, top_k, static_cast<int>(E), perm, inv,
        w_sorted, static_cast<const uint4*>(x), H / 8, static_cast<uint4*>(x_sorted));
    return cudaGetLastError();
}

cudaError_t launch_combine(const void* y_sorted, const int32_t* inv, int64_t T, int top_k,
                           int64_t H, void* out, int sm_count, cudaStream_t stream) {
    int64_t grid = (T + kRouteThreads / 32 - 1) / (kRouteThreads / 32);
    const int64_t cap = static_cast<int64_t>(sm_count) * 8;
    if (grid > cap) grid = cap;
    moe_combine_kernel<<<static_cast<unsigned>(grid), kRouteThreads, 0, stream>>>(
        static_cast<const float4*>(y_sorted), inv, T, top_k, H / 8, static_cast<uint4*>(out));
    return cudaGetLastError();
}

}  // namespace mx
