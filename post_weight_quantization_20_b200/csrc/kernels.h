// Internal host-side entry points shared between the library's translation units.
#pragma once
#include "common.cuh"

namespace gptq {

// abi.cu: validation of a gptq_config shared by every entry point that takes one
gptq_status check_cfg(const gptq_config* cfg);
// abi.cu: polls of a pipeline's mbarrier wait before it gives up (the default
// unless gptq_debug_set_wait_limit has set another); passed to the tensor-core kernels
uint32_t pipeline_wait_limit();

// hessian.cu
gptq_status hessian_prescale(cudaStream_t st, float* H, int C, double alpha, bool overwrite);
gptq_status hessian_syrk_simt(cudaStream_t st, float* H, const void* X, int dt, int64_t m, int C,
                              int64_t ldx, float beta);
// hessian_tc.cu: returns GPTQ_ERR_UNSUPPORTED when the tensor-core path does not apply.
gptq_status hessian_syrk_tc(cudaStream_t st, float* H, const void* X, int dt, int64_t m, int C,
                            int64_t ldx, float beta, int32_t* status);

// prepare.cu
size_t prepare_ws_bytes(int64_t C);
gptq_status prepare_run(cudaStream_t st, const float* H, int C, const gptq_config& cfg, float* U,
                        int32_t* perm, void* ws, int32_t* status);

// sweep.cu
size_t quantize_ws_bytes(int64_t R, int64_t C, const gptq_config& cfg);
gptq_status quantize_run(cudaStream_t st, const void* W, int wdt, int R, int C, int64_t ldw,
                         const float* U, const int32_t* perm, const gptq_config& cfg,
                         uint8_t* codes, float* scales, float* zeros, int32_t* g_idx,
                         float* losses, void* ws, int32_t* status);

// tf32_split.cu: whether the tensor-core products apply (sm_100, C a multiple of
// 4, TMA available), and U split and transposed for them: hi[n][k] + lo[n][k] = U[k][n]
bool trailing_tc_supported(int C);
gptq_status split_tf32_t(cudaStream_t st, const float* U, int C, float* hi, float* lo);

// gemm_tc.cu: D[m][n] -= sum_k (Ahi + Alo)[m][k] (Bhi + Blo)[n][k] on tcgen05 (3xTF32,
// segmented fp32 accumulation) for m < M and n in [n_lo, n_hi); A is read from
// column a_k0 of an M x lda buffer, B from column b_k0 of a b_rows x ldb buffer (both
// K-major, lda and ldb multiples of 4); lower: only tiles with an entry on or below
// the diagonal (n_lo must be 0); K, a_k0 and b_k0 multiples of 32, 4 and 4
gptq_status gemm3_tf32(cudaStream_t st, float* D, int64_t ldd, int M, int n_lo, int n_hi, int K,
                       const float* Ahi, const float* Alo, int lda, int a_k0, const float* Bhi,
                       const float* Blo, int ldb, int b_rows, int b_k0, bool lower,
                       int32_t* status);

// selftest kernels (prepare.cu holds the grid-barrier one, next to the barrier)
gptq_status selftest_mbarrier(cudaStream_t st, int32_t* status);
gptq_status selftest_grid_barrier(cudaStream_t st, int32_t* status);

// dequant.cu: the stored form's product (sweep-order repack, dequantizing GEMV)
gptq_status repack_sweep_run(cudaStream_t st, const uint32_t* packed, int R, int C, int bits,
                             const int32_t* perm, uint32_t* out);
gptq_status dequant_matmul_run(cudaStream_t st, const void* X, int xdt, int M, int C, int64_t ldx,
                               const uint32_t* Qp, const float* scales, const float* zeros,
                               int bits, int g, const int32_t* perm, float* Y, int R,
                               int half_sums);

// pack.cu
gptq_status pack_run(cudaStream_t st, const uint8_t* codes, int64_t R, int64_t C, int bits,
                     uint32_t* packed);

}  // namespace gptq
