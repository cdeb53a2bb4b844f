// Internal (non-exported) interface between the C ABI layer and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace mx {

enum EpiMode { EPI_PLAIN = 0, EPI_SWIGLU = 1, EPI_WEIGHTED = 2 };

// Arguments of the grouped W4A16 GEMM (see gemm.cu).
struct GemmArgs {
    const uint8_t* w_scales;   // [G, rows_w, K/32]
    const int32_t* offsets;    // [G+1] row offsets of each group, or nullptr (one group)
    int m_single;              // rows of the single group when offsets == nullptr
    int G;
    int K;
    int rows_w;                // weight rows per group
    int I;                     // SWIGLU: gate rows [0, I), up rows [I, 2I)
    int n_ftiles;              // feature tiles per group
    void* out;                 // output, row-major: bf16 (PLAIN, SWIGLU) or fp32 (WEIGHTED)
    int64_t out_ld;            // elements per output row
    int n_valid_feat;          // valid output columns
    const float* row_w;        // WEIGHTED: per-row scalar
    const uint8_t* x_scales;   // W4A4: activation block scales [rows, K/32] (+16 readable bytes)
    unsigned* status;          // device status word
    int code_stages;           // ring depths (set by launch_grouped_gemm)
    int act_stages;
};

// Token tiling of the grouped GEMM: NT token rows per MMA, TT token tiles per
// dequantized weight tile.
struct TokenTiling {
    int nt;
    int tt;
};

cudaError_t launch_quantize(const void* x, int is_f32, int64_t rows, int64_t cols,
                            uint8_t* codes, uint8_t* scales, int rule, int sm_count,
                            unsigned* status, cudaStream_t stream);
cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t rows,
                              int64_t cols, void* out, int sm_count, unsigned* status,
                              cudaStream_t stream);
cudaError_t launch_selftest_wait_timeout(unsigned* status, cudaStream_t stream);
double selftest_mma_flops(int kind, int iters, int sm_count);
cudaError_t launch_selftest_mma_rate(int kind, int iters, int sm_count, unsigned* status,
                                     cudaStream_t stream);
size_t route_tmp_bytes(int64_t T, int64_t E, int top_k);
cudaError_t launch_route(const float* logits, int64_t T, int64_t E, int top_k, int32_t* ids,
                         float* weights, int32_t* counts, int32_t* offsets, int32_t* perm,
                         int32_t* inv, float* w_sorted, int32_t* row_tok, void* tmp, const void* x,
                         int64_t row_bytes, void* x_sorted, const void* xs, int64_t xs_row_bytes,
                         void* xs_sorted, int sm_count, cudaStream_t stream);
cudaError_t launch_route_finish(int64_t T, int64_t E, int top_k, const int32_t* ids, const float* weights,
                                int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                                float* w_sorted, int32_t* row_tok, void* tmp, const void* x,
                                int64_t row_bytes, void* x_sorted, const void* xs, int64_t xs_row_bytes,
                                void* xs_sorted, int sm_count, cudaStream_t stream);
void route_tmp_split(void* tmp, int64_t T, int64_t E, int32_t** chunk_counts, int32_t** local_rank);
int route_project_smem_bytes(int64_t E, int64_t H, int cluster_size);
cudaError_t launch_route_project(const CUtensorMap& tmap_x, const CUtensorMap& tmap_w, int64_t T,
                                 int64_t H, int64_t E, int top_k, int32_t* ids, float* weights,
                                 int32_t* chunk_counts, int32_t* local_rank, float* logits_out,
                                 int sm_count, unsigned* status, cudaStream_t stream);
cudaError_t launch_gather_rows(const void* src, int64_t n_src, int64_t row_bytes, const int32_t* idx,
                               int64_t n, int div, void* dst, int sm_count, unsigned* status,
                               cudaStream_t stream);
cudaError_t launch_combine(const void* y_sorted, const int32_t* inv, int64_t T, int top_k,
                           int64_t H, void* out, int sm_count, cudaStream_t stream);
TokenTiling pick_token_tiling(int64_t rows, int64_t groups);
int64_t max_gemm_k();   // largest contraction length the grouped GEMM accepts

cudaError_t launch_grouped_gemm(int mode, TokenTiling tiling, const CUtensorMap& tmap_w,
                                const CUtensorMap& tmap_x, const GemmArgs& args, int grid,
                                cudaStream_t stream);
int pick_token_tiling_bf16w(int64_t rows, int64_t groups);   // 64, 128 or 256
cudaError_t launch_grouped_gemm_bf16w(int mode, int nt, const CUtensorMap& tmap_w, const CUtensorMap& tmap_x,
                                      const GemmArgs& args, int grid, cudaStream_t stream);
int64_t max_gemm_k_w4a4();   // largest contraction length the W4A4 engine accepts
TokenTiling pick_token_tiling_w4a4(int64_t rows, int64_t groups);
cudaError_t launch_grouped_gemm_w4a4(int mode, int nt, const CUtensorMap& tmap_w,
                                     const CUtensorMap& tmap_x, const GemmArgs& args, int grid,
                                     cudaStream_t stream);

}  // namespace mx
