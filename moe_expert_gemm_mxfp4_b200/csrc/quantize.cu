// MXFP4 quantize / dequantize kernels for sm_100a (HBM-streaming).
//
// Format (agentlenshq.com, "Transformers 4.40 performance upgrades for OpenAI
// GPT-OSS ...", section "What MXFP4 Is"): E2M1 elements (1 sign, 2 exponent,
// 1 mantissa bit), 32 consecutive elements share one scale.  Encoding choices
// (E8M0 scale byte, round-to-nearest-even with saturation, low nibble = even
// element, Inf/NaN blocks -> scale 0xFF) are documented in include/mxfp4.h.
//
// Layout of the work: the input is treated as a flat array of 32-element blocks
// (cols % 32 == 0, so blocks never straddle rows).  One warp handles 32 blocks
// per step: 128-bit coalesced loads spread each block over 4 lanes (bf16) or 8
// lanes (fp32); the block amax is a shuffle reduction over those lanes; the
// scale is pure integer work on the amax bit pattern; |v| / 2^s is an exact
// power-of-two product in fp32 and the E2M1 rounding is the hardware
// cvt.rn.satfinite.e2m1x2.f32 (round-to-nearest-even, saturating at 6).  Codes
// are staged through shared memory so that each lane stores one whole block
// (16 bytes) with a 128-bit store.
#include "common.cuh"
#include "internal.h"

namespace mx {

namespace {

constexpr int kQThreads = 256;
constexpr int kWarpsPerCta = kQThreads / 32;

// Block exponent s from the amax magnitude bits of a bf16 block.
__device__ __forceinline__ int block_exp_bf16(uint32_t amax, int rule) {
    if (amax == 0) return -127;
    int e, gt;
    const uint32_t E = amax >> 7;
    if (E > 0) {
        e = static_cast<int>(E) - 127;
        gt = (amax & 0x7Fu) > 0x40u;          // significand > 1.5
    } else {                                  // subnormal: amax = m * 2^-133
        const int p = 31 - __clz(amax);
        e = p - 133;
        gt = (2u * amax) > (3u << p);
    }
    int s = e - 2 + ((rule == MXFP4_SCALE_CEIL) ? gt : 0);
    return s < -127 ? -127 : (s > 127 ? 127 : s);
}

// Block exponent s from the amax magnitude bits of an fp32 block.
__device__ __forceinline__ int block_exp_f32(uint32_t amax, int rule) {
    if (amax == 0) return -127;
    int e, gt;
    const uint32_t E = amax >> 23;
    if (E > 0) {
        e = static_cast<int>(E) - 127;
        gt = (amax & 0x7FFFFFu) > 0x400000u;
    } else {                                  // fp32 subnormal: amax = m * 2^-149
        const int p = 31 - __clz(amax);
        e = p - 149;
        gt = (2ull * amax) > (3ull << p);
    }
    int s = e - 2 + ((rule == MXFP4_SCALE_CEIL) ? gt : 0);
    return s < -127 ? -127 : (s > 127 ? 127 : s);
}

// 2^-s as fp32, s in [-127, 125] (exponent field 127 - s in [2, 254]).
__device__ __forceinline__ float inv_pow2(int s) {
    return __uint_as_float(static_cast<uint32_t>(127 - s) << 23);
}

// 8 magnitudes (already scaled) -> 4 packed E2M1 bytes; element 2i in the low nibble.
__device__ __forceinline__ uint32_t cvt_e2m1x8(float e0, float e1, float e2, float e3, float e4,
                                               float e5, float e6, float e7) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(e0), "f"(e1), "f"(e2), "f"(e3), "f"(e4), "f"(e5), "f"(e6), "f"(e7));
    return out;
}

__device__ __forceinline__ float bf16_mag(uint32_t h16) {
    return __uint_as_float((h16 & 0x7FFFu) << 16);
}

// Sign bits of the two bf16 halves of w at bits 3 and 7 of a code byte.
__device__ __forceinline__ uint32_t bf16x2_sign_nibbles(uint32_t w) {
    return ((w >> 12) & 0x8u) | ((w >> 24) & 0x80u);
}

// 8 bf16 elements (one uint4) -> 4 code bytes given the block multiplier 2^-s.
__device__ __forceinline__ uint32_t quant8_bf16(uint4 v, float mult) {
    uint32_t c = cvt_e2m1x8(bf16_mag(v.x) * mult, bf16_mag(v.x >> 16) * mult,
                            bf16_mag(v.y) * mult, bf16_mag(v.y >> 16) * mult,
                            bf16_mag(v.z) * mult, bf16_mag(v.z >> 16) * mult,
                            bf16_mag(v.w) * mult, bf16_mag(v.w >> 16) * mult);
    c |= bf16x2_sign_nibbles(v.x) | (bf16x2_sign_nibbles(v.y) << 8) |
         (bf16x2_sign_nibbles(v.z) << 16) | (bf16x2_sign_nibbles(v.w) << 24);
    return c;
}

__device__ __forceinline__ uint32_t amax8_bf16(uint4 v, uint32_t& nonfinite) {
    uint32_t m = 0;
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t lo = w[i] & 0x7FFFu, hi = (w[i] >> 16) & 0x7FFFu;
        nonfinite |= ((lo & 0x7F80u) == 0x7F80u) | ((hi & 0x7F80u) == 0x7F80u);
        m = max(m, max(lo, hi));
    }
    return m;
}

// Dequantize 8 codes (one 32-bit code word) with the block's scale byte -> 8 bf16.
__device__ __forceinline__ uint4 dequant8(uint32_t cw, uint32_t S) {
    const float sc = e8m0_f32(S);
    uint4 o;
    o.x = dequant_byte_exact(cw & 0xFFu, sc);
    o.y = dequant_byte_exact((cw >> 8) & 0xFFu, sc);
    o.z = dequant_byte_exact((cw >> 16) & 0xFFu, sc);
    o.w = dequant_byte_exact(cw >> 24, sc);
    return o;
}

// ---------------------------------------------------------------- bf16 -> MXFP4
// One warp step = 128 uint4 vectors = 32 blocks.  Lane l loads vectors
// 32j + l (j = 0..3); block 8j + l/4 therefore lives on lanes 4(l/4) .. +3.
// If `qdq_out` is set, the kernel writes the dequantized bf16 values instead of
// codes/scales (fake quantization for the W4A4 path).
__global__ void __launch_bounds__(kQThreads)
quantize_bf16_kernel(const uint4* __restrict__ x, int64_t n_blocks, uint4* __restrict__ codes,
                     uint8_t* __restrict__ scales, int rule, uint4* __restrict__ qdq_out) {
    __shared__ __align__(16) uint32_t s_codes[kWarpsPerCta][128];
    __shared__ uint8_t s_scales[kWarpsPerCta][32];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int64_t n_vec = n_blocks * 4;
    const int64_t n_steps = (n_blocks + 31) >> 5;
    const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t step = warp0; step < n_steps; step += nwarps) {
        const int64_t vbase = step * 128;
        uint4 v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t idx = vbase + 32 * j + lane;
            v[j] = idx < n_vec ? __ldcs(x + idx) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t nf = 0;
            uint32_t am = amax8_bf16(v[j], nf);
            am = max(am, __shfl_xor_sync(0xFFFFFFFFu, am, 1));
            am = max(am, __shfl_xor_sync(0xFFFFFFFFu, am, 2));
            nf |= __shfl_xor_sync(0xFFFFFFFFu, nf, 1);
            nf |= __shfl_xor_sync(0xFFFFFFFFu, nf, 2);
            const int s = block_exp_bf16(am, rule);
            const uint32_t cw = nf ? 0u : quant8_bf16(v[j], inv_pow2(s));
            const uint32_t S = nf ? 0xFFu : static_cast<uint32_t>(s + 127);
            if (qdq_out) {
                const int64_t idx = vbase + 32 * j + lane;
                if (idx < n_vec) qdq_out[idx] = dequant8(cw, S);
            } else {
                s_codes[wid][32 * j + lane] = cw;
                if ((lane & 3) == 0) s_scales[wid][8 * j + (lane >> 2)] = static_cast<uint8_t>(S);
            }
        }
        if (!qdq_out) {
            __syncwarp();
            const int64_t blk = step * 32 + lane;
            if (blk < n_blocks) {
                codes[blk] = reinterpret_cast<const uint4*>(s_codes[wid])[lane];
                scales[blk] = s_scales[wid][lane];
            }
            __syncwarp();
        }
    }
}

// ---------------------------------------------------------------- fp32 -> MXFP4
// One warp step = 256 uint4 vectors (4 fp32 each) = 32 blocks; a block spans 8 lanes.
__global__ void __launch_bounds__(kQThreads)
quantize_f32_kernel(const uint4* __restrict__ x, int64_t n_blocks, uint4* __restrict__ codes,
                    uint8_t* __restrict__ scales, int rule) {
    __shared__ __align__(16) uint16_t s_codes[kWarpsPerCta][256];
    __shared__ uint8_t s_scales[kWarpsPerCta][32];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int64_t n_vec = n_blocks * 8;
    const int64_t n_steps = (n_blocks + 31) >> 5;
    const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t step = warp0; step < n_steps; step += nwarps) {
        const int64_t vbase = step * 256;
#pragma unroll 2
        for (int j = 0; j < 8; ++j) {
            const int64_t idx = vbase + 32 * j + lane;
            const uint4 v = idx < n_vec ? __ldcs(x + idx) : make_uint4(0, 0, 0, 0);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            uint32_t am = 0, nf = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t m = w[i] & 0x7FFFFFFFu;
                nf |= (m & 0x7F800000u) == 0x7F800000u;
                am = max(am, m);
            }
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) {
                am = max(am, __shfl_xor_sync(0xFFFFFFFFu, am, o));
                nf |= __shfl_xor_sync(0xFFFFFFFFu, nf, o);
            }
            const int s = block_exp_f32(am, rule);
            const float mult = inv_pow2(s);
            uint32_t c;
            {
                uint32_t b;
                asm("{\n\t.reg .b8 b0, b1;\n\t"
                    "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
                    "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
                    "mov.b32 %0, {b0, b1, b1, b1};\n\t}"
                    : "=r"(b)
                    : "f"(__uint_as_float(w[0] & 0x7FFFFFFFu) * mult),
                      "f"(__uint_as_float(w[1] & 0x7FFFFFFFu) * mult),
                      "f"(__uint_as_float(w[2] & 0x7FFFFFFFu) * mult),
                      "f"(__uint_as_float(w[3] & 0x7FFFFFFFu) * mult));
                c = (b & 0xFFFFu) | ((w[0] >> 28) & 0x8u) | ((w[1] >> 24) & 0x80u) |
                    ((w[2] >> 20) & 0x800u) | ((w[3] >> 16) & 0x8000u);
            }
            s_codes[wid][32 * j + lane] = static_cast<uint16_t>(nf ? 0u : c);
            if ((lane & 7) == 0)
                s_scales[wid][4 * j + (lane >> 3)] = static_cast<uint8_t>(nf ? 0xFFu : s + 127);
        }
        __syncwarp();
        const int64_t blk = step * 32 + lane;
        if (blk < n_blocks) {
            codes[blk] = reinterpret_cast<const uint4*>(s_codes[wid])[lane];
            scales[blk] = s_scales[wid][lane];
        }
        __syncwarp();
    }
}

// ---------------------------------------------------------------- MXFP4 -> bf16
// One warp step = 128 chunks of 8 elements (4 code bytes -> 16 output bytes);
// lane l handles chunks 32j + l so that every load and store is coalesced.
__global__ void __launch_bounds__(kQThreads)
dequantize_kernel(const uint32_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                  int64_t n_chunks, uint4* __restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int64_t n_steps = (n_chunks + 127) >> 7;
    const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t step = warp0; step < n_steps; step += nwarps) {
        uint32_t cw[4], S[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t ch = step * 128 + 32 * j + lane;
            cw[j] = ch < n_chunks ? __ldcs(codes + ch) : 0u;
            S[j] = ch < n_chunks ? scales[ch >> 2] : 127u;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t ch = step * 128 + 32 * j + lane;
            if (ch < n_chunks) __stcs(out + ch, dequant8(cw[j], S[j]));
        }
    }
}

int grid_for(int64_t n_steps, int sm_count) {
    const int64_t per_cta = kWarpsPerCta;
    int64_t g = (n_steps + per_cta - 1) / per_cta;
    const int64_t cap = static_cast<int64_t>(sm_count) * 8;   // 8 CTAs of 256 threads per SM
    return static_cast<int>(g < cap ? (g < 1 ? 1 : g) : cap);
}

}  // namespace

cudaError_t launch_quantize(const void* x, int is_f32, int64_t rows, int64_t cols,
                            uint8_t* codes, uint8_t* scales, int rule, int sm_count,
                            cudaStream_t stream) {
    const int64_t n_blocks = rows * (cols / 32);
    const int64_t n_steps = (n_blocks + 31) / 32;
    const int grid = grid_for(n_steps, sm_count);
    if (is_f32)
        quantize_f32_kernel<<<grid, kQThreads, 0, stream>>>(
            reinterpret_cast<const uint4*>(x), n_blocks, reinterpret_cast<uint4*>(codes), scales,
            rule);
    else
        quantize_bf16_kernel<<<grid, kQThreads, 0, stream>>>(
            reinterpret_cast<const uint4*>(x), n_blocks, reinterpret_cast<uint4*>(codes), scales,
            rule, nullptr);
    return cudaGetLastError();
}

cudaError_t launch_qdq_bf16(const void* x, int64_t rows, int64_t cols, void* out, int sm_count,
                            cudaStream_t stream) {
    const int64_t n_blocks = rows * (cols / 32);
    const int64_t n_steps = (n_blocks + 31) / 32;
    quantize_bf16_kernel<<<grid_for(n_steps, sm_count), kQThreads, 0, stream>>>(
        reinterpret_cast<const uint4*>(x), n_blocks, nullptr, nullptr, MXFP4_SCALE_FLOOR,
        reinterpret_cast<uint4*>(out));
    return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t rows,
                              int64_t cols, void* out, int sm_count, cudaStream_t stream) {
    const int64_t n_chunks = rows * cols / 8;
    const int64_t n_steps = (n_chunks + 127) / 128;
    dequantize_kernel<<<grid_for(n_steps, sm_count), kQThreads, 0, stream>>>(
        reinterpret_cast<const uint32_t*>(codes), scales, n_chunks, reinterpret_cast<uint4*>(out));
    return cudaGetLastError();
}

}  // namespace mx
