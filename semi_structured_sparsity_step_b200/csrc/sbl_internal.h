// sbl_internal.h -- host-side declarations shared by the library's .cu files
// (launchers called by the C ABI in sbl_api.cu).
#pragma once

#include <atomic>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

namespace sbl {

// ---- mask / gamma / ternary (mask_quant.cu)
constexpr int kGammaMaxBlocks = 592;  // 4 blocks of 256 threads per SM on 148 SMs
constexpr int kGammaLimbs = 10;       // 320-bit exact sum of |W| in units of 2^-133

struct GammaWorkspace {
  unsigned long long bucket[256];  // sum of 8-bit significands per biased exponent
  unsigned int ticket;             // blocks finished
  unsigned int zero_threshold;     // largest bf16 magnitude pattern with W_q = 0
  unsigned int pad[62];
  unsigned long long block_window[kGammaMaxBlocks];  // per-block window sums
};

size_t mask_quant_workspace_bytes();
// from_quantised: the mask is the top-N of |W_q| (an ablation), else of |W|.
cudaError_t launch_mask_quant(const void* W, int d_out, int d_in, int N, int M, int8_t* W_eff, void* W_eff_bf16,
                              uint8_t* mask_bits, float* gamma, void* workspace, cudaStream_t stream, int num_sms,
                              bool from_quantised = false);
// dW (.) M in place (the ablation without the Dual-STE).
cudaError_t launch_mask_grad(float* dW, const uint8_t* mask_bits, int d_out, int d_in, cudaStream_t stream,
                             int num_sms);

// The optimizer step (AdamW on the master weight) fused with the next weight
// step's gamma pass and a mask flip count, then the ternary pass.
struct AdamwParams {
  double lr, beta1, beta2, eps, weight_decay, max_norm;
  long long step;  // t >= 1
};
cudaError_t launch_adamw_step(void* W, float* W32, const float* dW, float* m, float* v, int d_out, int d_in, int N,
                              int M, const AdamwParams& hp, const double* grad_sqnorm, int8_t* W_eff,
                              void* W_eff_bf16, uint8_t* mask_bits, float* gamma, unsigned long long* flips,
                              void* workspace, cudaStream_t stream, int num_sms);
// *sumsq += sum of g^2 (fp64, deterministic for a given n).
cudaError_t launch_grad_sqnorm(const float* g, size_t n, double* sumsq, void* workspace, cudaStream_t stream);

// ---- activation quantiser (act_quant.cu)
cudaError_t launch_norm_act_quant(const void* X, const void* g, float eps, int T, int d_in, void* Xn, int8_t* Xq,
                                  float* amax, cudaStream_t stream, int num_sms);
cudaError_t launch_act_quant(const void* X, int T, int d_in, int8_t* Xq, float* amax, cudaStream_t stream,
                             int num_sms);

// ---- tensor-core GEMMs (gemm_tc.cu)
// 2-D tensor map of a row-major [rows, inner] uint32 matrix (row stride in
// bytes), box [box_rows, box_inner], no swizzle; out-of-range elements read 0.
bool make_tmap_u32(CUtensorMap* m, const void* base, unsigned long long inner, unsigned long long rows,
                   unsigned long long row_bytes, unsigned box_inner, unsigned box_rows);
// Same for a uint8 matrix, with the 128-byte swizzle or none.
bool make_tmap_u8(CUtensorMap* m, const void* base, unsigned long long inner, unsigned long long rows,
                  unsigned long long row_bytes, unsigned box_inner, unsigned box_rows, bool swizzle128);
extern std::atomic<int> g_gemm_variant;
cudaError_t launch_forward(const int8_t* Xq, const float* amax, const int8_t* W_eff, const float* gamma, int T,
                           int d_in, int d_out, float* Y, int32_t* acc, cudaStream_t stream, int num_sms,
                           uint32_t* err);
// One problem of a grouped forward (device pointers).
struct FwdProblemDev {
  const int8_t* Xq;
  const float* amax;
  const int8_t* W_eff;
  const float* gamma;
  int T, d_in, d_out;
  float* Y;
  int32_t* acc;
};
cudaError_t launch_forward_group(const FwdProblemDev* probs, int count, cudaStream_t stream, int num_sms,
                                 uint32_t* err);
cudaError_t launch_forward_packed(const int8_t* Xq, const float* amax, const uint8_t* packed, const float* gamma,
                                  int T, int d_in, int d_out, int N, int M, float* Y, int32_t* acc,
                                  cudaStream_t stream, int num_sms, uint32_t* err);
cudaError_t launch_backward(const void* dY, const void* X, const void* W_eff_bf16, const float* gamma, int T,
                            int d_in, int d_out, float* dX, float* dW, int accumulate_dW, cudaStream_t stream,
                            int num_sms, uint32_t* err);

// ---- 2:4 compressed weight and the sparse tensor-core forward (gemm_sp24.cu)
size_t sparse24_values_row_bytes(int d_in);
size_t sparse24_meta_offset(int d_out, int d_in);
size_t sparse24_bytes(int d_out, int d_in);
cudaError_t launch_compress24(const int8_t* W_eff, int d_out, int d_in, uint8_t* out, cudaStream_t stream,
                              int num_sms, uint32_t* err);
cudaError_t launch_forward_sparse24(const int8_t* Xq, const float* amax, const uint8_t* w24, const float* gamma,
                                   int T, int d_in, int d_out, float* Y, int32_t* acc, cudaStream_t stream,
                                   int num_sms, uint32_t* err);

// ---- packed format (pack_gemv.cu)
size_t packed_codes_row_bytes(int d_in, int N, int M);
size_t packed_index_row_bytes(int d_in, int M);
cudaError_t launch_unpack(const uint8_t* packed, int d_out, int d_in, int N, int M, int8_t* W_eff,
                          cudaStream_t stream, int num_sms);
cudaError_t launch_pack(const int8_t* W_eff, int d_out, int d_in, int N, int M, uint8_t* packed,
                        cudaStream_t stream, uint32_t* err);
struct GemvProblemDev {
  const uint8_t* packed;
  const int8_t* Xq;
  const float* amax;
  const float* gamma;
  float* Y;
  int d_in, d_out;
  size_t crow, irow;  // filled in by the launcher
  int rows;           // rows per work unit (16 or 8), filled in by the launcher
};
// Decode GEMV kernel: 0 = the default (the dense layout through gemv_tma.cu,
// the N:M formats through gemv_direct.cu), 1 = block-wide TMA tile ring
// (pack_gemv.cu), 2 = per-warp TMA rings in persistent blocks
// (gemv_direct.cu) for every format.
extern std::atomic<int> g_gemv_variant;
cudaError_t launch_gemv_group(const GemvProblemDev* probs, int count, int batch, int N, int M,
                              cudaStream_t stream, int num_sms, uint32_t* err, bool dense2);
// Failure-detection self-test: one bounded wait that runs out (selftest.cu).
cudaError_t launch_wait_timeout_selftest(uint64_t limit_ns, cudaStream_t stream, uint32_t* err);
cudaError_t launch_gemv_direct(const GemvProblemDev* probs, int count, int batch, int N, int M,
                               cudaStream_t stream, int num_sms, uint32_t* err, bool dense2);
// The dense 2-bit layout (also the codes plane of the 8:8 format) through
// per-warp TMA rings (gemv_tma.cu).
cudaError_t launch_gemv_dense_tma(const GemvProblemDev* probs, int count, int batch, cudaStream_t stream,
                                  int num_sms, uint32_t* err);
size_t dense2_row_bytes(int d_in);
cudaError_t launch_pack_dense2(const int8_t* W_eff, int d_out, int d_in, uint8_t* out, cudaStream_t stream,
                               int num_sms);
cudaError_t launch_gemv_packed(const int8_t* Xq, const float* amax, int batch, const uint8_t* packed,
                               const float* gamma, int d_in, int d_out, int N, int M, float* Y,
                               cudaStream_t stream, int num_sms, uint32_t* err);

}  // namespace sbl
