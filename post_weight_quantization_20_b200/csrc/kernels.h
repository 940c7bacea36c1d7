// Internal host-side entry points shared between the library's translation units.
#pragma once
#include "common.cuh"

namespace gptq {

// abi.cu: validation of a gptq_config shared by every entry point that takes one
gptq_status check_cfg(const gptq_config* cfg);

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

// trailing_tc.cu: W[:, e:cend] -= (Ehi + Elo)[:, kE0:kE0+K] * U[i0:i0+K, e:cend] on
// tcgen05 (3xTF32), with U given as its transposed split Ut_hi + Ut_lo
// (split_tf32_t) and the errors as column windows of rows x ldE buffers
bool trailing_tc_supported(int C);
gptq_status split_tf32_t(cudaStream_t st, const float* U, int C, float* hi, float* lo);
gptq_status trailing_update_tc(cudaStream_t st, float* Wk, int R, int C, int i0, int K, int e,
                               int cend, const float* Ehi, const float* Elo, int ldE, int kE0,
                               const float* Uthi, const float* Utlo, int32_t* status);

// selftest kernels (prepare.cu holds the grid-barrier one, next to the barrier)
gptq_status selftest_mbarrier(cudaStream_t st, int32_t* status);
gptq_status selftest_grid_barrier(cudaStream_t st, int32_t* status);

// pack.cu
gptq_status pack_run(cudaStream_t st, const uint8_t* codes, int64_t R, int64_t C, int bits,
                     uint32_t* packed);

}  // namespace gptq
