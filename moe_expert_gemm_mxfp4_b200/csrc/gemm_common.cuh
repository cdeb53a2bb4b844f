// Pieces shared by the two grouped-GEMM engines (gemm.cu: W4A16 on kind::f16 with
// weights dequantized into TMEM; gemm_mxf4.cu: W4A4 on kind::mxf4.block_scale):
// the work-tile decomposition over groups, ring positions, the block-scale
// staging copy and the fused epilogues.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace mx {
namespace gemm {

constexpr int kBM = 128;          // weight rows per work tile (the MMA's M)
constexpr int kMaxGroups = 256;

// Position in a ring of n slots with the parity of the slot's current use.
struct RingPos {
    int idx = 0;
    uint32_t ph = 0;
    __device__ __forceinline__ void next(int n) {
        if (++idx == n) {
            idx = 0;
            ph ^= 1u;
        }
    }
};

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

__device__ __forceinline__ float silu_f32(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

__device__ __forceinline__ void store_bf16(void* out, int64_t idx, float v) {
    reinterpret_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(v);
}

// Copy `rows` consecutive rows of block scales (kb bytes each) from global to
// shared: the 16-byte multiple with one bulk copy (counted on `bar`), the tail
// with plain loads.  Returns the bulk byte count.  `src` must be 16-byte aligned.
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

struct TileInfo {
    int g, f, row0, mrows;
};

// Work tile t -> (group, feature tile, first row, valid rows).  Tiles of a group
// are numbered feature-tile-major with the token tile fastest, so CTAs working at
// the same time share the weight tile (L2 reuse).  s_tstart[g] = first tile of
// group g; rows of group g are s_off[g] .. s_off[g+1].
__device__ __forceinline__ TileInfo decode_tile(int t, const int* s_tstart, const int* s_off, int G,
                                                int tile_rows) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {                 // largest g with s_tstart[g] <= t
        const int mid = (lo + hi + 1) >> 1;
        if (s_tstart[mid] <= t) lo = mid; else hi = mid - 1;
    }
    TileInfo ti;
    ti.g = lo;
    const int m = s_off[lo + 1] - s_off[lo];
    const int mt = (m + tile_rows - 1) / tile_rows;
    const int local = t - s_tstart[lo];
    ti.f = local / mt;
    const int tt = local - ti.f * mt;
    ti.row0 = s_off[lo] + tt * tile_rows;
    ti.mrows = min(tile_rows, m - tt * tile_rows);
    return ti;
}

// Accumulator lane of weight row `srow` of a SwiGLU tile and back: the tile holds
// gate features f*64 .. f*64+63 (staged rows 0-63) and the matching up features
// (staged rows 64-127); TMEM lane 32q + l carries feature 16q + (l & 15), gate for
// l < 16 and up for l >= 16, so that each warp of the epilogue pairs gate and up
// with one shuffle.
__host__ __device__ __forceinline__ int swiglu_staged_row(int lane_row) {
    const int q = lane_row >> 5, l = lane_row & 31;
    return (l < 16 ? 0 : 64) + 16 * q + (l & 15);
}

// Epilogue of one work tile, run by the four warps of an epilogue warpgroup (warp
// q reads TMEM lanes 32q .. 32q+31).  Accumulator column j is token row
// ti.row0 + j; `t_base` addresses column 0 of this warp's lanes.  CW columns per
// TMEM load, double-buffered in registers.
template <int MODE, int CW, int NCOLS>
__device__ __forceinline__ void epilogue_tile(const GemmArgs& args, const TileInfo& ti,
                                              uint32_t t_base, int q, int lane) {
    constexpr int NCH = NCOLS / CW;
    const bool lo = lane < 16;
    auto process = [&](const uint32_t* cur, int c) {
        if (MODE == EPI_SWIGLU) {
            // lanes < 16 finish columns [0, CW/2) of the chunk, lanes >= 16 columns
            // [CW/2, CW); each needs its partner's (lane ^ 16) gate or up value
            const int feat = ti.f * 64 + 16 * q + (lane & 15);
#pragma unroll
            for (int i = 0; i < CW / 2; ++i) {
                const uint32_t send = lo ? cur[CW / 2 + i] : cur[i];
                const float other = __uint_as_float(__shfl_xor_sync(0xFFFFFFFFu, send, 16));
                const float g = lo ? __uint_as_float(cur[i]) : other;
                const float u = lo ? other : __uint_as_float(cur[CW / 2 + i]);
                const int tok = c * CW + (lo ? i : CW / 2 + i);
                if (tok < ti.mrows)
                    store_bf16(args.out, static_cast<int64_t>(ti.row0 + tok) * args.out_ld + feat,
                               silu_f32(g) * u);
            }
        } else {
            const int feat = ti.f * kBM + q * 32 + lane;
            if (feat < args.n_valid_feat) {
#pragma unroll
                for (int n = 0; n < CW; ++n) {
                    const int tok = c * CW + n;
                    if (tok < ti.mrows) {
                        const int64_t idx = static_cast<int64_t>(ti.row0 + tok) * args.out_ld + feat;
                        const float val = __uint_as_float(cur[n]);
                        if (MODE == EPI_WEIGHTED)   // fp32 out: one rounding, in the combine
                            reinterpret_cast<float*>(args.out)[idx] = val * args.row_w[ti.row0 + tok];
                        else
                            store_bf16(args.out, idx, val);
                    }
                }
            }
        }
    };
    auto load = [&](uint32_t* dst, int c) {
        if (CW == 32) tmem_ld_x32(t_base + c * CW, dst); else tmem_ld_x16(t_base + c * CW, dst);
    };
    // two register buffers: the next chunk's TMEM load overlaps this chunk's work
    uint32_t v0[CW], v1[CW];
    load(v0, 0);
#pragma unroll 1
    for (int c = 0; c < NCH; c += 2) {
        tmem_wait_ld();
        if (c + 1 < NCH) load(v1, c + 1);
        process(v0, c);
        if (c + 1 < NCH) {
            tmem_wait_ld();
            if (c + 2 < NCH) load(v0, c + 2);
            process(v1, c + 1);
        }
    }
}

}  // namespace gemm
}  // namespace mx
