// MoE routing for sm_100a: top-k + softmax, per-expert histogram, prefix sums,
// the expert-sorted permutation of (token, slot) pairs, the gather of token rows
// into that order, and the deterministic combine.
//
// The pages route MoE tokens through a downloadable MegaBlocks kernel and name
// a top-k kernel (agentlenshq.com, "Transformers 4.40 performance upgrades for
// OpenAI GPT-OSS ...", section "Zero-Build Kernels from the Hub"); the routing
// rule itself is a reading: top-k by (logit desc, expert id asc), softmax over
// the k selected logits, pairs p = t*k + j grouped by expert in ascending p.
//
// Kernels (one stream, no host synchronization), sized for latency: every
// token, expert and output vector gets its own warp or thread, so that a decode
// step (tens of tokens) costs a few microseconds per launch.
//   route_topk     one warp per token: top-k and softmax; per CTA (a chunk of
//                  8 tokens, at most 64 pairs in two warps) the per-expert pair
//                  counts and each pair's rank among the chunk's pairs of its
//                  expert, from warp match masks and population counts;
//   route_scan     one CTA per expert: exclusive scan of its chunk counts ->
//                  per-chunk base ranks, and the expert's total;
//   route_scatter  offsets (exclusive scan over experts, recomputed per CTA in
//                  shared memory), the position of every pair, perm / inv /
//                  sorted weights / the token of every sorted row, and optionally
//                  the gather of token rows (the W4A4 layer's packed rows);
//   moe_combine    one thread per 8 output columns of a token:
//                  out[t] = bf16(sum_j y[inv[t*k + j]]), fp32, slot order.
#include "common.cuh"
#include "internal.h"

namespace mx {

constexpr int kRouteThreads = 256;
constexpr int kTokPerChunk = kRouteThreads / 32;   // one warp per token
constexpr int kMaxTopK = 8;
constexpr int kMaxExperts = 256;

namespace {

// Expert order: larger logit first, lower expert id among equal logits; a NaN logit
// ranks below every number (-inf included), NaNs among themselves by id.  This is a
// strict total order, so every lane of the butterfly below ends with the same pick.
__device__ __forceinline__ bool better(float v, int id, float bv, int bid) {
    const bool vn = v != v, bn = bv != bv;
    if (vn != bn) return bn;
    if (!vn && v != bv) return v > bv;
    return id < bid;
}

__global__ void __launch_bounds__(kRouteThreads)
route_topk_kernel(const float* __restrict__ logits, int T, int E, int k, int32_t* __restrict__ ids,
                  float* __restrict__ weights, int32_t* __restrict__ chunk_counts,
                  int32_t* __restrict__ local_rank) {
    static_assert(kTokPerChunk * kMaxTopK <= 64, "a chunk's pairs must fit in warps 0 and 1");
    __shared__ int32_t s_ids[kTokPerChunk * kMaxTopK];
    __shared__ int32_t s_cnt[kMaxExperts];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_cnt[e] = 0;
    const int t0 = blockIdx.x * kTokPerChunk;
    const int ntok = min(kTokPerChunk, T - t0);
    const int t = t0 + wid;
    if (wid < ntok) {
        float v[kMaxExperts / 32];
#pragma unroll
        for (int i = 0; i < kMaxExperts / 32; ++i) {
            const int e = lane + 32 * i;
            v[i] = e < E ? logits[static_cast<int64_t>(t) * E + e] : -INFINITY;
        }
        uint32_t taken = 0;
        float sel_v[kMaxTopK];
        int sel_id[kMaxTopK];
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) {
            sel_v[j] = -INFINITY;
            sel_id[j] = 0;
            if (j < k) {
                float bv = -INFINITY;
                int bid = 0x7FFFFFFF;
#pragma unroll
                for (int i = 0; i < kMaxExperts / 32; ++i) {
                    const int e = lane + 32 * i;
                    if (e < E && !((taken >> i) & 1u) &&
                        (bid == 0x7FFFFFFF || better(v[i], e, bv, bid))) {
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
                sel_v[j] = bv;   // uniform across the warp after the butterfly
                sel_id[j] = bid;
            }
        }
        // softmax over the k selected logits: lane j < k writes slot j
        float sum = 0.f, mine = 0.f;
        int my_id = 0;
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) {
            if (j < k) {
                const float z = expf(sel_v[j] - sel_v[0]);
                sum += z;
                if (lane == j) {
                    mine = z;
                    my_id = sel_id[j];
                }
            }
        }
        if (lane < k) {
            ids[static_cast<int64_t>(t) * k + lane] = my_id;
            weights[static_cast<int64_t>(t) * k + lane] = mine / sum;
            s_ids[wid * k + lane] = my_id;
        }
    }
    __syncthreads();
    // The chunk's pairs i = 0 .. ntok*k - 1 (ascending p, at most 64) sit one per
    // thread of warps 0 and 1.  Within a warp, the lanes holding the same expert are
    // one match mask: a pair's rank is the number of matching lanes below it, the
    // warp's count of that expert the mask's population.  Warp 1 adds warp 0's count.
    const int npairs = ntok * k;
    const int i = threadIdx.x;
    const bool valid = i < npairs;
    const int e = valid ? s_ids[i] : kMaxExperts + lane;   // out-of-range ids match no pair
    uint32_t m = 0;
    if (wid < 2) m = __match_any_sync(0xFFFFFFFFu, e);
    const uint32_t below = m & ((1u << lane) - 1u);
    const bool leader = below == 0;
    if (wid == 0 && valid && leader) s_cnt[e] = __popc(m);
    __syncthreads();
    if (valid) local_rank[static_cast<int64_t>(t0) * k + i] = __popc(below) + (wid == 1 ? s_cnt[e] : 0);
    __syncthreads();   // every rank has read warp 0's counts
    if (wid == 1 && valid && leader) s_cnt[e] += __popc(m);
    __syncthreads();
    for (int x = threadIdx.x; x < E; x += blockDim.x)
        chunk_counts[static_cast<int64_t>(blockIdx.x) * E + x] = s_cnt[x];
}

// Block-wide exclusive scan of one int per thread (blockDim.x == kRouteThreads);
// returns the thread's exclusive prefix and sets *total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* total) {
    __shared__ int s_warp[kRouteThreads / 32];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[wid] = x;
    __syncthreads();
    int base = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kRouteThreads / 32; ++w) {
        const int s = s_warp[w];
        if (w < wid) base += s;
        tot += s;
    }
    __syncthreads();   // s_warp may be reused by a later scan
    *total = tot;
    return base + x - v;
}

// One CTA per expert e: chunk_counts[c][e] <- exclusive prefix over chunks c;
// counts[e] <- total.  Each thread scans a contiguous run of chunks.
__global__ void __launch_bounds__(kRouteThreads)
route_scan_kernel(int32_t* __restrict__ chunk_counts, int n_chunks, int E,
                  int32_t* __restrict__ counts) {
    const int e = blockIdx.x;
    const int per = (n_chunks + kRouteThreads - 1) / kRouteThreads;
    const int c0 = threadIdx.x * per;
    const int c1 = min(n_chunks, c0 + per);
    int run = 0;
    for (int c = c0; c < c1; ++c) run += chunk_counts[static_cast<int64_t>(c) * E + e];
    int total;
    int base = block_exclusive_scan(run, &total);
    for (int c = c0; c < c1; ++c) {
        int32_t* p = chunk_counts + static_cast<int64_t>(c) * E + e;
        const int v = *p;
        *p = base;
        base += v;
    }
    if (threadIdx.x == 0) counts[e] = total;
}

// One warp per pair: its sorted position, the routing tables (perm, inv, the
// sorted routing weights and, if `row_tok` is given, the token of every sorted
// row, which a GEMM that gathers its activation rows itself reads) and, if `x` is
// given, the copy of its token's row into the expert-sorted activation matrix
// (row_vec 16-byte vectors per row); if `xs` is given, likewise for a second
// matrix of xs_row bytes per row (the block scales of MXFP4 activations).
// Every CTA first recomputes offsets (exclusive scan of counts over experts);
// CTA 0 also stores them.
__global__ void __launch_bounds__(kRouteThreads)
route_scatter_kernel(const int32_t* __restrict__ ids, const float* __restrict__ weights,
                     const int32_t* __restrict__ chunk_base, const int32_t* __restrict__ local_rank,
                     const int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int64_t P,
                     int k, int E, int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                     float* __restrict__ w_sorted, int32_t* __restrict__ row_tok,
                     const uint4* __restrict__ x, int64_t row_vec,
                     uint4* __restrict__ x_sorted, const uint8_t* __restrict__ xs, int64_t xs_row,
                     uint8_t* __restrict__ xs_sorted) {
    __shared__ int32_t s_off[kMaxExperts];
    {
        const int e = threadIdx.x;   // E <= kMaxExperts == blockDim.x
        const int c = e < E ? counts[e] : 0;
        int total;
        const int ex = block_exclusive_scan(c, &total);
        if (e < E) s_off[e] = ex;
        if (blockIdx.x == 0) {
            if (e < E) offsets[e] = ex;
            if (e == 0) offsets[E] = total;
        }
        __syncthreads();
    }
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t p = warp0; p < P; p += nwarps) {
        const int e = ids[p];
        const int64_t t = p / k;
        const int64_t chunk = t / kTokPerChunk;
        const int64_t pos = static_cast<int64_t>(s_off[e]) + chunk_base[chunk * E + e] + local_rank[p];
        if (lane == 0) {
            perm[pos] = static_cast<int32_t>(p);
            inv[p] = static_cast<int32_t>(pos);
            if (w_sorted) w_sorted[pos] = weights[p];
            if (row_tok) row_tok[pos] = static_cast<int32_t>(t);
        }
        if (x) {   // all of a lane's loads first, then its stores: 8 x 16 B in flight per lane
            const uint4* src = x + t * row_vec;
            uint4* dst = x_sorted + pos * row_vec;
            for (int64_t c0 = 0; c0 < row_vec; c0 += 32 * 8) {
                uint4 v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int64_t c = c0 + lane + 32 * u;
                    if (c < row_vec) v[u] = __ldg(src + c);
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int64_t c = c0 + lane + 32 * u;
                    if (c < row_vec) dst[c] = v[u];
                }
            }
        }
        if (xs) {
            const uint8_t* src = xs + t * xs_row;
            uint8_t* dst = xs_sorted + pos * xs_row;
            for (int64_t c = lane; c < xs_row; c += 32) dst[c] = __ldg(src + c);
        }
    }
}

// dst row i = src row idx[i] / div, for rows of row_vec vectors of type V (16-byte
// or 4-byte); one warp per row, all of a lane's loads issued before its stores.  An
// index outside the source leaves its row untouched and records
// MXFP4_ERR_INVALID_ARG in the status word.
template <typename V>
__global__ void __launch_bounds__(kRouteThreads)
gather_rows_kernel(const V* __restrict__ src, int64_t n_src, const int32_t* __restrict__ idx, int64_t n,
                   int div, int64_t row_vec, V* __restrict__ dst, unsigned* status) {
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t i = warp0; i < n; i += nwarps) {
        const int64_t r = __ldg(idx + i) / div;
        if (r < 0 || r >= n_src) {
            if (lane == 0) record_status(status, MXFP4_ERR_INVALID_ARG);
            continue;
        }
        const V* s = src + r * row_vec;
        V* d = dst + i * row_vec;
        for (int64_t c0 = 0; c0 < row_vec; c0 += 32 * 8) {
            V v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int64_t c = c0 + lane + 32 * u;
                if (c < row_vec) v[u] = __ldg(s + c);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int64_t c = c0 + lane + 32 * u;
                if (c < row_vec) d[c] = v[u];
            }
        }
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    __nv_bfloat162 r = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&r);
}

// One thread per 8 output columns of one token; the token's k fp32 rows are
// summed in slot order j = 0..k-1 and rounded once to bf16.
__global__ void __launch_bounds__(kRouteThreads)
moe_combine_kernel(const float4* __restrict__ y_sorted, const int32_t* __restrict__ inv,
                   int64_t T, int k, int64_t row_vec8, uint4* __restrict__ out) {
    const int64_t n = T * row_vec8;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
        const int64_t t = i / row_vec8, c = i - t * row_vec8;
        float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) {
            if (j < k) {
                const int64_t row = __ldg(inv + t * k + j);
                const float4* src = y_sorted + (row * row_vec8 + c) * 2;
                const float4 u = __ldcs(src), v = __ldcs(src + 1);
                a[0] += u.x; a[1] += u.y; a[2] += u.z; a[3] += u.w;
                a[4] += v.x; a[5] += v.y; a[6] += v.z; a[7] += v.w;
            }
        }
        uint4 o;
        o.x = pack_bf16x2(a[0], a[1]);
        o.y = pack_bf16x2(a[2], a[3]);
        o.z = pack_bf16x2(a[4], a[5]);
        o.w = pack_bf16x2(a[6], a[7]);
        out[i] = o;
    }
}

}  // namespace

size_t route_tmp_bytes(int64_t T, int64_t E, int top_k) {
    const int64_t n_chunks = (T + kTokPerChunk - 1) / kTokPerChunk;
    return static_cast<size_t>(n_chunks * E + T * top_k) * sizeof(int32_t);
}

void route_tmp_split(void* tmp, int64_t T, int64_t E, int32_t** chunk_counts, int32_t** local_rank) {
    const int64_t n_chunks = (T + kTokPerChunk - 1) / kTokPerChunk;
    *chunk_counts = static_cast<int32_t*>(tmp);
    *local_rank = *chunk_counts + n_chunks * E;
}

cudaError_t launch_route(const float* logits, int64_t T, int64_t E, int top_k, int32_t* ids,
                         float* weights, int32_t* counts, int32_t* offsets, int32_t* perm,
                         int32_t* inv, float* w_sorted, int32_t* row_tok, void* tmp, const void* x,
                         int64_t row_bytes, void* x_sorted, const void* xs, int64_t xs_row_bytes,
                         void* xs_sorted, int sm_count, cudaStream_t stream) {
    const int64_t n_chunks = (T + kTokPerChunk - 1) / kTokPerChunk;
    int32_t *chunk_counts, *local_rank;
    route_tmp_split(tmp, T, E, &chunk_counts, &local_rank);
    route_topk_kernel<<<static_cast<unsigned>(n_chunks), kRouteThreads, 0, stream>>>(
        logits, static_cast<int>(T), static_cast<int>(E), top_k, ids, weights, chunk_counts,
        local_rank);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_route_finish(T, E, top_k, ids, weights, counts, offsets, perm, inv, w_sorted, row_tok,
                               tmp, x, row_bytes, x_sorted, xs, xs_row_bytes, xs_sorted, sm_count, stream);
}

// The routing after top-k (chunk counts and ranks already in `tmp`): per-expert scan,
// offsets, permutation tables and the optional row copies.
cudaError_t launch_route_finish(int64_t T, int64_t E, int top_k, const int32_t* ids, const float* weights,
                                int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                                float* w_sorted, int32_t* row_tok, void* tmp, const void* x,
                                int64_t row_bytes, void* x_sorted, const void* xs, int64_t xs_row_bytes,
                                void* xs_sorted, int sm_count, cudaStream_t stream) {
    const int64_t n_chunks = (T + kTokPerChunk - 1) / kTokPerChunk;
    int32_t *chunk_counts, *local_rank;
    route_tmp_split(tmp, T, E, &chunk_counts, &local_rank);
    route_scan_kernel<<<static_cast<unsigned>(E), kRouteThreads, 0, stream>>>(
        chunk_counts, static_cast<int>(n_chunks), static_cast<int>(E), counts);
    const int64_t P = T * top_k;
    int64_t grid = (P + kRouteThreads / 32 - 1) / (kRouteThreads / 32);
    const int64_t cap = static_cast<int64_t>(sm_count) * 8;
    if (grid > cap) grid = cap;
    route_scatter_kernel<<<static_cast<unsigned>(grid), kRouteThreads, 0, stream>>>(
        ids, weights, chunk_counts, local_rank, counts, offsets, P, top_k, static_cast<int>(E),
        perm, inv, w_sorted, row_tok, static_cast<const uint4*>(x), row_bytes / 16,
        static_cast<uint4*>(x_sorted), static_cast<const uint8_t*>(xs), xs_row_bytes,
        static_cast<uint8_t*>(xs_sorted));
    return cudaGetLastError();
}

cudaError_t launch_gather_rows(const void* src, int64_t n_src, int64_t row_bytes, const int32_t* idx,
                               int64_t n, int div, void* dst, int sm_count, unsigned* status,
                               cudaStream_t stream) {
    int64_t grid = (n + kRouteThreads / 32 - 1) / (kRouteThreads / 32);
    const int64_t cap = static_cast<int64_t>(sm_count) * 8;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    if (row_bytes % 16 == 0)
        gather_rows_kernel<uint4><<<static_cast<unsigned>(grid), kRouteThreads, 0, stream>>>(
            static_cast<const uint4*>(src), n_src, idx, n, div, row_bytes / 16, static_cast<uint4*>(dst), status);
    else
        gather_rows_kernel<uint32_t><<<static_cast<unsigned>(grid), kRouteThreads, 0, stream>>>(
            static_cast<const uint32_t*>(src), n_src, idx, n, div, row_bytes / 4, static_cast<uint32_t*>(dst),
            status);
    return cudaGetLastError();
}

cudaError_t launch_combine(const void* y_sorted, const int32_t* inv, int64_t T, int top_k,
                           int64_t H, void* out, int sm_count, cudaStream_t stream) {
    const int64_t n = T * (H / 8);
    int64_t grid = (n + kRouteThreads - 1) / kRouteThreads;
    const int64_t cap = static_cast<int64_t>(sm_count) * 16;
    if (grid > cap) grid = cap;
    moe_combine_kernel<<<static_cast<unsigned>(grid), kRouteThreads, 0, stream>>>(
        static_cast<const float4*>(y_sorted), inv, T, top_k, H / 8, static_cast<uint4*>(out));
    return cudaGetLastError();
}

}  // namespace mx
