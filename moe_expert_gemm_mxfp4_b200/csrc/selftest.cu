// Failure-detection self-test: a wait that nothing satisfies.  The kernel's one
// thread waits on a fresh mbarrier with the library's bounded wait; when the wait
// limit passes it records MXFP4_ERR_TIMEOUT in the device status word and returns,
// which is how every kernel of the library reports a stalled pipeline.  Nothing
// faults, traps or hangs, so the context stays usable afterwards.
#include "common.cuh"
#include "internal.h"

namespace mx {

namespace {

__global__ void selftest_wait_timeout_kernel(unsigned* status) {
    __shared__ uint64_t bar;
    __shared__ int never;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);     // expects one arrival; none is ever made
    never = 0;
    fence_mbar_init();
    if (!mbar_wait(&bar, 0, &never)) record_status(status, MXFP4_ERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_selftest_wait_timeout(unsigned* status, cudaStream_t stream) {
    selftest_wait_timeout_kernel<<<1, 32, 0, stream>>>(status);
    return cudaGetLastError();
}

}  // namespace mx

// ---------------------------------------------------------------- tensor-pipe rate
// Peak-rate probe of the two MMA kinds the library's GEMMs use, for the roofline
// denominators: every CTA (one per SM) issues `iters` x 4 back-to-back
// tcgen05.mma of M = 128, N = 256 (the kind's full-rate shape) on operands that
// stay in shared memory, then waits (bounded) for their completion.  kind::f16:
// bf16 A and B, K = 16 per MMA; kind::mxf4: E2M1 A and B with E8M0 block scales
// (1.0) in TMEM, K = 64 per MMA.  Operands hold pseudo-random finite values, so
// the tensor pipe draws the power it does on real data.  The accumulator is never
// read: only the time of the launch matters.
namespace mx {

namespace {

constexpr int kRateN = 256;
constexpr int kRateThreads = 128;
// shared memory: A 128 rows x 128 B, B 256 rows x 128 B (128B-swizzled K-major
// tiles, any contents), then the barrier
constexpr int kRateA = 0, kRateB = 16384, kRateBar = 16384 + 32768;
// (more dynamic shared memory than two CTAs can share, so every SM runs exactly one
// CTA and no CTA waits for another's TMEM allocation)
constexpr int kRateSmem = 116 * 1024;
static_assert(kRateBar + 64 + 1024 <= kRateSmem, "probe layout");

__global__ void __launch_bounds__(kRateThreads, 1)
selftest_mma_rate_kernel(int kind, int iters, unsigned* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kRateBar);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + kRateBar + 16);
    volatile int* s_never = reinterpret_cast<volatile int*>(smem + kRateBar + 20);
    const int tid = threadIdx.x, warp = tid >> 5;
    // operands: bf16 values in +-[1, 2) (sign and mantissa from a hash), or any
    // E2M1 bytes (every 4-bit code is a finite value)
    uint32_t* w = reinterpret_cast<uint32_t*>(smem);
    for (int i = tid; i < kRateBar / 4; i += kRateThreads) {
        uint32_t h = static_cast<uint32_t>(i) * 2654435761u ^ (blockIdx.x * 40503u);
        h ^= h >> 15;
        h *= 2246822519u;
        w[i] = kind == 1 ? h : (h & 0x807F807Fu) | 0x3F803F80u;
    }
    if (tid == 0) {
        mbar_init(bar, 1);
        *s_never = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(s_tmem, 512);
        tmem_relinquish();
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // operands -> tensor core
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t base = *s_tmem;
    // kind::mxf4 block scales: 1.0 (byte 127) in columns 256..287 of every lane
    uint32_t v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = 0x7F7F7F7Fu;
    tmem_st_x32(base + (static_cast<uint32_t>(warp * 32) << 16) + 256, v);
    tmem_wait_st();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
        const uint32_t a_s = smem_u32(smem + kRateA), b_s = smem_u32(smem + kRateB);
        for (int r = 0; r < iters; ++r) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t acc = (r | j) != 0 ? 1u : 0u;
                if (kind == 1) {
                    const uint32_t sf_id = (j & 1) * 2, h = j >> 1;
                    mma_mxf4(base, sw128_desc(a_s + 32 * j), sw128_desc(b_s + 32 * j),
                             idesc_mxf4(128, kRateN, sf_id), (base + 256 + 4 * h) | (sf_id << 30),
                             (base + 264 + 4 * h) | (sf_id << 30), acc);
                } else {
                    mma_bf16_ss(base, sw128_desc(a_s + 32 * j), sw128_desc(b_s + 32 * j),
                                idesc_bf16_f32(128, kRateN), acc);
                }
            }
        }
        tc_commit(bar);
        if (!mbar_wait(bar, 0, s_never)) record_status(status, MXFP4_ERR_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(base, 512);
    }
}

}  // namespace

double selftest_mma_flops(int kind, int iters, int sm_count) {
    const double k = kind == 1 ? 64.0 : 16.0;
    return static_cast<double>(sm_count) * iters * 4 * 2.0 * 128 * kRateN * k;
}

cudaError_t launch_selftest_mma_rate(int kind, int iters, int sm_count, unsigned* status,
                                     cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(selftest_mma_rate_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kRateSmem);
    if (e != cudaSuccess) return e;
    selftest_mma_rate_kernel<<<sm_count, kRateThreads, kRateSmem, stream>>>(kind, iters, status);
    return cudaGetLastError();
}

}  // namespace mx
