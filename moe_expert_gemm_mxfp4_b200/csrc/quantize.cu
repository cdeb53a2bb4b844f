// MXFP4 quantize / dequantize kernels for sm_100a (HBM-streaming).
//
// Format (agentlenshq.com, "Transformers 4.40 performance upgrades for OpenAI
// GPT-OSS ...", section "What MXFP4 Is"): E2M1 elements (1 sign, 2 exponent,
// 1 mantissa bit), 32 consecutive elements share one scale.  Encoding choices
// (E8M0 scale byte, round-to-nearest-even with saturation, low nibble = even
// element, Inf/NaN blocks -> scale 0xFF) are documented in include/mxfp4.h.
//
// Layout of the work: the input is treated as a flat array of 32-element blocks
// (cols % 32 == 0, so blocks never straddle rows).
//   bf16 -> MXFP4 and MXFP4 -> bf16 stream with plain 128-bit (codes: 32-bit)
//   loads, non-allocating in L1: each warp of the grid takes 32-block units in a
//   grid-stride walk, two at a time, so that every lane has its loads of two
//   units in flight before it computes.
//   fp32 -> MXFP4 (weights, off the hot path) runs a ring of cp.async.bulk stages
//   per persistent CTA: one producer thread streams chunks of consecutive blocks
//   into shared memory (completion counted on an mbarrier per stage) and eight
//   consumer warps convert and release them.
// Quantize: each block is spread over 4 lanes (bf16) or 8 lanes (fp32); the block
// amax is a shuffle reduction over those lanes; the scale is pure integer work on
// the amax bit pattern; |v| / 2^s is an exact power-of-two product in fp32 and the
// E2M1 rounding is the hardware cvt.rn.satfinite.e2m1x2.f32 (round-to-nearest-even,
// saturating at 6).  Dequantize: the hardware E2M1 -> f16 conversion, a shift into
// a bf16 pattern and one exact bf16x2 multiply by the block scale per code pair.
#include "common.cuh"
#include "internal.h"

namespace mx {

namespace {


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

// 8 values (already scaled, signed) -> 4 packed E2M1 bytes; element 2i in the low
// nibble.  The conversion rounds to nearest even, saturates at 6 and keeps the sign
// of its input, zero results included (-0 and small negatives give code 8).
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

// The two bf16 halves of a word as fp32 (exact).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// 8 bf16 elements (one uint4) -> 4 code bytes given the block multiplier 2^-s
// (an exact power-of-two product in fp32).
__device__ __forceinline__ uint32_t quant8_bf16(uint4 v, float mult) {
    return cvt_e2m1x8(bf16_lo(v.x) * mult, bf16_hi(v.x) * mult, bf16_lo(v.y) * mult,
                      bf16_hi(v.y) * mult, bf16_lo(v.z) * mult, bf16_hi(v.z) * mult,
                      bf16_lo(v.w) * mult, bf16_hi(v.w) * mult);
}

__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Largest magnitude bit pattern (15 bits) of 8 bf16 elements.  As unsigned
// integers, magnitudes order like the values; Inf and NaN (0x7F80 and above)
// order above every finite value, so a block is non-finite iff its amax >= 0x7F80.
__device__ __forceinline__ uint32_t amax8_bf16(uint4 v) {
    const uint32_t m = max_u16x2(max_u16x2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
                                 max_u16x2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu));
    return max(m & 0xFFFFu, m >> 16);
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

__device__ __forceinline__ uint32_t bmul2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// 2 E2M1 codes (one byte, low nibble first) -> their values as f16x2, exactly.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
    uint32_t o;
    asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}" : "=r"(o) : "r"(byte));
    return o;
}

// Dequantize one code word (8 codes) with the block's scale byte S -> 8 bf16.
// An E2M1 value as f16 has a 1-bit mantissa; shifting the f16 magnitude right by 3
// (sign kept) gives the bf16 pattern of the same value times 2^-112, and one exact
// bf16x2 multiply by 2^(S-15) then gives value x 2^(S-127): exact for S in [2, 142]
// (normal operands and products).  Other S take the exact fp32 route.
__device__ __forceinline__ uint4 dequant8_alu(uint32_t cw, uint32_t S) {
    if (S - 2u > 140u) return dequant8(cw, S);
    const uint32_t sf = (S + 112u) * 0x00800080u;   // bf16x2 {2^(S-15), 2^(S-15)}
    uint32_t r[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t h = e2m1x2_to_f16x2((cw >> (8 * j)) & 0xFFu);
        r[j] = bmul2(((h & 0x7FFF7FFFu) >> 3) | (h & 0x80008000u), sf);
    }
    return make_uint4(r[0], r[1], r[2], r[3]);
}

// ---------------------------------------------------------------- bulk-copy ring
// Stage ring shared by the streaming kernels: full[i] completes when stage i's
// bulk copies have landed, empty[i] when all consumer warps have read it.
constexpr int kRingConsumerWarps = 8;
constexpr int kRingThreads = (kRingConsumerWarps + 1) * 32;   // + one producer warp
constexpr int kRingCtasPerSm = 2;
constexpr int kRingMaxStages = 8;
constexpr int kRingSmemBytes = 96 * 1024;                      // per CTA

struct Ring {
    uint64_t full[kRingMaxStages];
    uint64_t empty[kRingMaxStages];
    int abort;
};

__device__ __forceinline__ void ring_init(Ring& r, int n_stages, int consumer_warps = kRingConsumerWarps) {
    if (threadIdx.x == 0) {
        for (int i = 0; i < n_stages; ++i) {
            mbar_init(&r.full[i], 1);
            mbar_init(&r.empty[i], consumer_warps);
        }
        r.abort = 0;
        fence_mbar_init();
    }
    __syncthreads();
}

// Producer (one thread): for each chunk of this CTA wait for a free stage, then
// `issue(stage, chunk, bar)` posts the bulk copies (arrive.expect_tx + copies).
// On abort or timeout it stops issuing; before returning it waits (bounded) for
// every copy it posted, so that no copy lands in shared memory after exit.
template <class Issue>
__device__ __forceinline__ void ring_produce(Ring& r, int n_stages, int64_t n_chunks, Issue issue,
                                             unsigned* status) {
    int st = 0;
    uint32_t ph = 0;
    uint32_t posted = 0, last_ph = 0;   // bit i: stage i holds a copy posted in phase bit i of last_ph
    for (int64_t c = blockIdx.x; c < n_chunks; c += gridDim.x) {
        if (!mbar_wait(&r.empty[st], ph ^ 1u, &r.abort)) {
            if (!r.abort) record_status(status, MXFP4_ERR_TIMEOUT);
            r.abort = 1;
            break;
        }
        issue(st, c, &r.full[st]);
        posted |= 1u << st;
        last_ph = (last_ph & ~(1u << st)) | (ph << st);
        if (++st == n_stages) {
            st = 0;
            ph ^= 1u;
        }
    }
    if (r.abort) {
        int never = 0;
        for (int i = 0; i < n_stages; ++i)
            if ((posted >> i) & 1u) (void)mbar_wait(&r.full[i], (last_ph >> i) & 1u, &never);
    }
}

// Consumer side of one stage: wait until it is full (bounded).
__device__ __forceinline__ bool ring_wait_full(Ring& r, int st, uint32_t ph, unsigned* status) {
    if (mbar_wait(&r.full[st], ph, &r.abort)) return true;
    if (!r.abort) record_status(status, MXFP4_ERR_TIMEOUT);
    r.abort = 1;
    return false;
}

// Consumer warp done reading stage st.
__device__ __forceinline__ void ring_release(Ring& r, int st) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(&r.empty[st]);
}

// ---------------------------------------------------------------- bf16 -> MXFP4
// Plain 128-bit loads (no bulk-copy ring): warp u of the grid converts 32-block
// units u, u + n_warps, ... (2 KB of bf16 each, read as four fully coalesced
// 512-byte warp loads, non-allocating in L1), two units per iteration so that 8
// loads per lane are in flight.
__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// One 32-block unit held as v[j] = vector 32j + lane of the unit's 2 KB: block
// 8j + l/4 lives on lanes 4(l/4) .. +3, each lane writes the 4 code bytes of its
// vector (a warp store covers 128 contiguous bytes), and the 32 scale bytes are
// gathered by shuffles so that lane l stores block l's.
__device__ __forceinline__ void quant_unit_bf16(const uint4 (&v)[4], int64_t blk0, int64_t n_blocks, int lane,
                                                uint32_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                                int rule) {
    uint32_t mine = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint32_t am = amax8_bf16(v[j]);
        am = max(am, __shfl_xor_sync(0xFFFFFFFFu, am, 1));
        am = max(am, __shfl_xor_sync(0xFFFFFFFFu, am, 2));
        const bool nf = am >= 0x7F80u;
        const int s = block_exp_bf16(am, rule);
        const uint32_t cw = nf ? 0u : quant8_bf16(v[j], inv_pow2(s));
        const uint32_t S = nf ? 0xFFu : static_cast<uint32_t>(s + 127);
        const int64_t blk = blk0 + 8 * j + (lane >> 2);
        if (blk < n_blocks) __stcs(codes + blk0 * 4 + 32 * j + lane, cw);
        const uint32_t got = __shfl_sync(0xFFFFFFFFu, S, (lane & 7) * 4);
        if ((lane >> 3) == j) mine = got;
    }
    if (blk0 + lane < n_blocks) scales[blk0 + lane] = static_cast<uint8_t>(mine);
}

constexpr int kLsuThreads = 256;

__global__ void __launch_bounds__(kLsuThreads)
quantize_bf16_lsu_kernel(const uint4* __restrict__ x, int64_t n_blocks, uint32_t* __restrict__ codes,
                         uint8_t* __restrict__ scales, int rule) {
    const int lane = threadIdx.x & 31;
    const int64_t w0 = (static_cast<int64_t>(blockIdx.x) * kLsuThreads + threadIdx.x) >> 5;
    const int64_t nw = (static_cast<int64_t>(gridDim.x) * kLsuThreads) >> 5;
    const int64_t n_units = (n_blocks + 31) / 32;
    const int64_t n_vec = n_blocks * 4;   // 16-byte vectors of input
    for (int64_t u = w0; u < n_units; u += 2 * nw) {
        const int64_t u2 = u + nw;
        uint4 a[4], b[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t i = u * 128 + 32 * j + lane;
            a[j] = i < n_vec ? ld_stream(x + i) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t i = u2 * 128 + 32 * j + lane;
            b[j] = (u2 < n_units && i < n_vec) ? ld_stream(x + i) : make_uint4(0, 0, 0, 0);
        }
        quant_unit_bf16(a, u * 32, n_blocks, lane, codes, scales, rule);
        if (u2 < n_units) quant_unit_bf16(b, u2 * 32, n_blocks, lane, codes, scales, rule);
    }
}

// ---------------------------------------------------------------- fp32 -> MXFP4
constexpr int kChunkBlocks = 256;

// Chunk = 256 blocks (32 KB of fp32).  Consumer warp w converts blocks
// 32w .. 32w+31: step j (0..7) reads vectors 32j + l, i.e. block 4j + l/8, a
// block spanning 8 lanes; each lane produces 2 code bytes.
__global__ void __launch_bounds__(kRingThreads, kRingCtasPerSm)
quantize_f32_kernel(const uint8_t* __restrict__ x, int64_t n_blocks, uint16_t* __restrict__ codes,
                    uint8_t* __restrict__ scales, int rule, unsigned* status) {
    constexpr int kStageBytes = kChunkBlocks * 128;
    constexpr int kStages = kRingSmemBytes / kStageBytes;   // 3
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ Ring ring;
    ring_init(ring, kStages);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t n_chunks = (n_blocks + kChunkBlocks - 1) / kChunkBlocks;
    if (warp == kRingConsumerWarps) {
        if (lane == 0)
            ring_produce(ring, kStages, n_chunks, [&](int st, int64_t c, uint64_t* bar) {
                const int64_t nb = min(static_cast<int64_t>(kChunkBlocks), n_blocks - c * kChunkBlocks);
                const uint32_t bytes = static_cast<uint32_t>(nb * 128);
                mbar_arrive_expect_tx(bar, bytes);
                bulk_load(smem + st * kStageBytes, x + c * kStageBytes, bytes, bar);
            }, status);
        return;
    }
    int st = 0;
    uint32_t ph = 0;
    for (int64_t c = blockIdx.x; c < n_chunks; c += gridDim.x) {
        if (!ring_wait_full(ring, st, ph, status)) break;
        const uint4* src = reinterpret_cast<const uint4*>(smem + st * kStageBytes) + warp * 256;
        uint4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = src[32 * j + lane];
        ring_release(ring, st);
        const int64_t blk0 = c * kChunkBlocks + warp * 32;
        uint32_t mine = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            // magnitudes order like unsigned integers; Inf/NaN (>= 0x7F800000) above all
            uint32_t am = max(max(v[j].x & 0x7FFFFFFFu, v[j].y & 0x7FFFFFFFu),
                              max(v[j].z & 0x7FFFFFFFu, v[j].w & 0x7FFFFFFFu));
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) am = max(am, __shfl_xor_sync(0xFFFFFFFFu, am, o));
            const bool nf = am >= 0x7F800000u;
            const int s = block_exp_f32(am, rule);
            const float mult = inv_pow2(s);
            uint32_t cw;
            asm("{\n\t.reg .b8 b0, b1;\n\t"
                "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
                "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
                "mov.b32 %0, {b0, b1, b1, b1};\n\t}"
                : "=r"(cw)
                : "f"(__uint_as_float(v[j].x) * mult), "f"(__uint_as_float(v[j].y) * mult),
                  "f"(__uint_as_float(v[j].z) * mult), "f"(__uint_as_float(v[j].w) * mult));
            cw &= 0xFFFFu;
            const uint32_t S = nf ? 0xFFu : static_cast<uint32_t>(s + 127);
            const int64_t blk = blk0 + 4 * j + (lane >> 3);
            if (blk < n_blocks)
                __stcs(codes + blk0 * 8 + 32 * j + lane, static_cast<uint16_t>(nf ? 0u : cw));
            // block 4j + q (q = 0..3) lives on lanes 8q .. 8q+7; lane 4j + q takes its scale
            const uint32_t got = __shfl_sync(0xFFFFFFFFu, S, (lane & 3) * 8);
            if ((lane >> 2) == j) mine = got;
        }
        if (blk0 + lane < n_blocks) scales[blk0 + lane] = static_cast<uint8_t>(mine);
        if (++st == kStages) {
            st = 0;
            ph ^= 1u;
        }
    }
}

// ---------------------------------------------------------------- MXFP4 -> bf16
// Plain streaming loads, like the bf16 quantize: warp u of the grid expands 32-block
// units u, u + n_warps, ... two per iteration.  Lane l, step j (0..3) takes code word
// 32j + l of the unit (block 8j + l/4, whose scale byte lane 8j + l/4 loaded and a
// shuffle hands over) and stores output vector 32j + l: every warp access is a
// contiguous 128-byte (codes) or 512-byte (output) run.
constexpr int kDqThreads = 256;
constexpr int kDqUnits = 2;

__global__ void __launch_bounds__(kDqThreads, 8)
dequantize_kernel(const uint32_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                  int64_t n_blocks, uint4* __restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int64_t w0 = (static_cast<int64_t>(blockIdx.x) * kDqThreads + threadIdx.x) >> 5;
    const int64_t nw = (static_cast<int64_t>(gridDim.x) * kDqThreads) >> 5;
    const int64_t n_units = (n_blocks + 31) / 32;
    for (int64_t u = w0; u < n_units; u += kDqUnits * nw) {
        uint32_t cw[kDqUnits][4], sb[kDqUnits];
#pragma unroll
        for (int k = 0; k < kDqUnits; ++k) {
            const int64_t uk = u + k * nw;
            sb[k] = uk < n_units && uk * 32 + lane < n_blocks ? static_cast<uint32_t>(__ldcs(scales + uk * 32 + lane)) : 0u;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int64_t blk = uk * 32 + 8 * j + (lane >> 2);
                cw[k][j] = uk < n_units && blk < n_blocks ? __ldcs(codes + uk * 128 + 32 * j + lane) : 0u;
            }
        }
#pragma unroll
        for (int k = 0; k < kDqUnits; ++k) {
            const int64_t uk = u + k * nw;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t S = __shfl_sync(0xFFFFFFFFu, sb[k], 8 * j + (lane >> 2));
                const int64_t blk = uk * 32 + 8 * j + (lane >> 2);
                if (uk < n_units && blk < n_blocks) __stcs(out + uk * 128 + 32 * j + lane, dequant8_alu(cw[k][j], S));
            }
        }
    }
}

int ring_grid(int64_t n_chunks, int sm_count) {
    const int64_t cap = static_cast<int64_t>(sm_count) * kRingCtasPerSm;
    return static_cast<int>(n_chunks < cap ? (n_chunks < 1 ? 1 : n_chunks) : cap);
}

// Opt the kernel in to the ring's dynamic shared memory.  The attribute belongs to
// the current device's context, so it is set before every launch (a host-side call
// of about a microsecond) rather than cached, which stays right when the caller
// switches devices.
template <class K>
cudaError_t set_ring_smem(K kern) {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kRingSmemBytes);
}

}  // namespace

cudaError_t launch_quantize(const void* x, int is_f32, int64_t rows, int64_t cols,
                            uint8_t* codes, uint8_t* scales, int rule, int sm_count,
                            unsigned* status, cudaStream_t stream) {
    const int64_t n_blocks = rows * (cols / 32);
    const int grid = ring_grid((n_blocks + kChunkBlocks - 1) / kChunkBlocks, sm_count);
    cudaError_t e;
    if (is_f32) {
        if ((e = set_ring_smem(quantize_f32_kernel)) != cudaSuccess) return e;
        quantize_f32_kernel<<<grid, kRingThreads, kRingSmemBytes, stream>>>(
            static_cast<const uint8_t*>(x), n_blocks, reinterpret_cast<uint16_t*>(codes), scales,
            rule, status);
    } else {
        (void)status;
        const int64_t n_units = (n_blocks + 31) / 32;
        int64_t g = (n_units + 2 * (kLsuThreads / 32) - 1) / (2 * (kLsuThreads / 32));
        const int64_t cap = static_cast<int64_t>(sm_count) * 8;
        if (g > cap) g = cap;
        quantize_bf16_lsu_kernel<<<static_cast<unsigned>(g < 1 ? 1 : g), kLsuThreads, 0, stream>>>(
            static_cast<const uint4*>(x), n_blocks, reinterpret_cast<uint32_t*>(codes), scales, rule);
    }
    return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t rows,
                              int64_t cols, void* out, int sm_count, unsigned* status,
                              cudaStream_t stream) {
    (void)status;   // no waits in this kernel
    const int64_t n_blocks = rows * (cols / 32);
    const int64_t n_units = (n_blocks + 31) / 32;
    int64_t g = (n_units + kDqUnits * (kDqThreads / 32) - 1) / (kDqUnits * (kDqThreads / 32));
    const int64_t cap = static_cast<int64_t>(sm_count) * 16;   // two waves of 8 CTAs per SM
    if (g > cap) g = cap;
    dequantize_kernel<<<static_cast<unsigned>(g < 1 ? 1 : g), kDqThreads, 0, stream>>>(
        reinterpret_cast<const uint32_t*>(codes), scales, n_blocks, reinterpret_cast<uint4*>(out));
    return cudaGetLastError();
}

}  // namespace mx
