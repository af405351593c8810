// sbl_api.cu -- the C ABI declared in include/sbl.h: argument validation on
// the host, device capability checks, the latched device error word, and
// dispatch to the kernels' launchers.  Nothing here allocates device memory.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>
#include <vector>

#include "../../include/sbl.h"
#include "sbl_device.cuh"
#include "sbl_internal.h"

namespace sbl {

// Per-device error word, ORed by kernels (see sbl_device.cuh).
__device__ uint32_t g_sbl_error_word;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  bool supported = false;
  int num_sms = 0;
  uint32_t* err = nullptr;
};

DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

// Returns SBL_OK and fills *info for the current device.
sbl_status current_device(DeviceInfo** info) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SBL_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SBL_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return SBL_ERR_CUDA;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_sbl_error_word) != cudaSuccess) return SBL_ERR_CUDA;
    d.supported = (major == 10 && minor == 0);
    d.num_sms = sms;
    d.err = static_cast<uint32_t*>(p);
    d.ready = true;
  }
  *info = &d;
  return d.supported ? SBL_OK : SBL_ERR_UNSUPPORTED;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline sbl_status check_nm(int N, int M) {
  if (!(M == 4 || M == 8) || N < 1 || N > M) return SBL_ERR_INVALID_ARG;
  return SBL_OK;
}

// Shape rules shared by every entry point: d_in % 16 == 0 (16-byte rows of
// int8 for the tensor-memory loads), d_out % 8 == 0 (16-byte rows of bf16).
inline sbl_status check_dims(int d_in, int d_out) {
  if (d_in < 0 || d_out < 0) return SBL_ERR_SHAPE;
  if (d_in % 16 != 0 || d_out % 8 != 0) return SBL_ERR_SHAPE;
  return SBL_OK;
}

inline sbl_status from_cuda(cudaError_t e) { return e == cudaSuccess ? SBL_OK : SBL_ERR_CUDA; }

}  // namespace
}  // namespace sbl

using namespace sbl;

extern "C" {

const char* sbl_status_string(int status) {
  switch (status) {
    case SBL_OK: return "SBL_OK";
    case SBL_ERR_INVALID_ARG: return "SBL_ERR_INVALID_ARG";
    case SBL_ERR_SHAPE: return "SBL_ERR_SHAPE";
    case SBL_ERR_ALIGN: return "SBL_ERR_ALIGN";
    case SBL_ERR_UNSUPPORTED: return "SBL_ERR_UNSUPPORTED";
    case SBL_ERR_WORKSPACE: return "SBL_ERR_WORKSPACE";
    case SBL_ERR_TIMEOUT: return "SBL_ERR_TIMEOUT";
    case SBL_ERR_CUDA: return "SBL_ERR_CUDA";
    case SBL_ERR_DEVICE_CHECK: return "SBL_ERR_DEVICE_CHECK";
    default: return "SBL_ERR_UNKNOWN";
  }
}

int sbl_version(void) { return 100; }

sbl_status sbl_set_gemm_variant(int variant) {
  if (variant != 0 && variant != 1) return SBL_ERR_INVALID_ARG;
  g_gemm_variant = variant;
  return SBL_OK;
}

sbl_status sbl_set_gemv_variant(int variant) {
  if (variant < 0 || variant > 2) return SBL_ERR_INVALID_ARG;
  g_gemv_variant = variant;
  return SBL_OK;
}

sbl_status sbl_selftest_wait_timeout(unsigned limit_us, void* stream) {
  if (limit_us == 0u || limit_us > 1000000u) return SBL_ERR_INVALID_ARG;
  DeviceInfo* d = nullptr;
  const sbl_status st = current_device(&d);
  if (st != SBL_OK) return st;
  return from_cuda(launch_wait_timeout_selftest(static_cast<uint64_t>(limit_us) * 1000ull,
                                                static_cast<cudaStream_t>(stream), d->err));
}

sbl_status sbl_check(void* stream) {
  DeviceInfo* d = nullptr;
  sbl_status st = current_device(&d);
  if (st != SBL_OK) return st;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SBL_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, d->err, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return SBL_ERR_CUDA;
  if (word != 0) {
    const uint32_t zero = 0;
    if (cudaMemcpy(d->err, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return SBL_ERR_CUDA;
    if (word & kErrTimeout) return SBL_ERR_TIMEOUT;
    return SBL_ERR_DEVICE_CHECK;
  }
  return SBL_OK;
}

size_t sbl_mask_quant_workspace_bytes(int d_out, int d_in) {
  (void)d_out;
  (void)d_in;
  return mask_quant_workspace_bytes();
}

sbl_status sbl_mask_quant(const void* W, int d_out, int d_in, int N, int M, int8_t* W_eff, void* W_eff_bf16,
                          uint8_t* mask_bits, float* gamma, void* workspace, size_t workspace_bytes,
                          void* stream) {
  sbl_status st = check_nm(N, M);
  if (st != SBL_OK) return st;
  if (W == nullptr || W_eff == nullptr || gamma == nullptr || workspace == nullptr) return SBL_ERR_INVALID_ARG;
  if ((st = check_dims(d_in, d_out)) != SBL_OK) return st;
  const unsigned long long n = static_cast<unsigned long long>(d_out) * static_cast<unsigned long long>(d_in);
  if (n == 0 || n >= (1ull << 32) || d_in % M != 0) return SBL_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(W_eff) || !aligned16(W_eff_bf16) || !aligned16(mask_bits) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || (reinterpret_cast<uintptr_t>(gamma) & 3u) != 0)
    return SBL_ERR_ALIGN;
  if (workspace_bytes < mask_quant_workspace_bytes()) return SBL_ERR_WORKSPACE;
  DeviceInfo* d = nullptr;
  if ((st = current_device(&d)) != SBL_OK) return st;
  return from_cuda(launch_mask_quant(W, d_out, d_in, N, M, W_eff, W_eff_bf16, mask_bits, gamma, workspace,
                                     static_cast<cudaStream_t>(stream), d->num_sms));
}

sbl_status sbl_mask_quant_ex(const void* W, int d_out, int d_in, int N, int M, unsigned flags, int8_t* W_eff,
                             void* W_eff_bf16, uint8_t* mask_bits, float* gamma, void* workspace,
                             size_t workspace_bytes, void* stream) {
  if ((flags & ~static_cast<unsigned>(SBL_MASK_FROM_QUANTISED)) != 0u) return SBL_ERR_INVALID_ARG;
  sbl_status st = check_nm(N, M);
  if (st != SBL_OK) return st;
  if (W == nullptr || W_eff == nullptr || gamma == nullptr || workspace == nullptr) return SBL_ERR_INVALID_ARG;
  if ((st = check_dims(d_in, d_out)) != SBL_OK) return st;
  const unsigned long long n = static_cast<unsigned long long>(d_out) * static_cast<unsigned long long>(d_in);
  if (n == 0 || n >= (1ull << 32) || d_in % M != 0) return SBL_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(W_eff) || !aligned16(W_eff_bf16) || !aligned16(mask_bits) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || (reinterpret_cast<uintptr_t>(gamma) & 3u) != 0)
    return SBL_ERR_ALIGN;
  if (workspace_bytes < mask_quant_workspace_bytes()) return SBL_ERR_WORKSPACE;
  DeviceInfo* d = nullptr;
  if ((st = current_device(&d)) != SBL_OK) return st;
  return from_cuda(launch_mask_quant(W, d_out, d_in, N, M, W_eff, W_eff_bf16, mask_bits, gamma, workspace,
                                     static_cast<cudaStream_t>(stream), d->num_sms,
                                     (flags & SBL_MASK_FROM_QUANTISED) != 0u));
}

sbl_status sbl_mask_grad(float* dW, const uint8_t* mask_bits, int d_out, int d_in, void* stream) {
  sbl_status st = check_dims(d_in, d_out);
  if (st != SBL_OK) return st;
  if (d_out == 0 || d_in == 0) return SBL_OK;
  if (dW == nullptr || mask_bits == nullptr) return SBL_ERR_INVALID_ARG;
  if (!aligned16(dW) || !aligned16(mask_bits)) return SBL_ERR_ALIGN;
  DeviceInfo* d = nullptr;
  if ((st = current_device(&d)) != SBL_OK) return st;
  return from_cuda(launch_mask_grad(dW, mask_bits, d_out, d_in, static_cast<cudaStream_t>(stream), d->num_sms));
}

sbl_status sbl_grad_sqnorm(const float* dW, size_t n, double* sumsq, void* workspace, size_t workspace_bytes,
                           void* stream) {
  if (sumsq == nullptr || workspace == nullptr) return SBL_ERR_INVALID_ARG;
  if (n == 0) return SBL_OK;
  if (dW == nullptr) return SBL_ERR_INVALID_ARG;
  if (!aligned16(dW) || (reinterpret_cast<uintptr_t>(sumsq) & 7u) != 0 ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return SBL_ERR_ALIGN;
  if (workspace_bytes < mask_quant_workspace_bytes()) return SBL_ERR_WORKSPACE;
  DeviceInfo* d = nullptr;
  sbl_status st = current_device(&d);
  if (st != SBL_OK) return st;
  return from_cuda(launch_grad_sqnorm(dW, n, sumsq, workspace, static_cast<cudaStream_t>(stream)));
}

sbl_status sbl_adamw_step(void* W, float* W32, const float* dW, float* m, float* v, int d_out, int d_in, int N,
                          int M, double lr, double beta1, double beta2, double eps, double weight_decay,
                          long long step, const double* grad_sqnorm, double max_norm, int8_t* W_eff,
                          void* W_eff_bf16, uint8_t* mask_bits, float* gamma, unsigned long long* flips,
                          void* workspace, size_t workspace_bytes, void* stream) {
  sbl_status st = check_nm(N, M);
  if (st != SBL_OK) return st;
  if (W == nullptr || dW == nullptr || m == nullptr || v == nullptr || W_eff == nullptr || gamma == nullptr ||
      workspace == nullptr)
    return SBL_ERR_INVALID_ARG;
  if (flips != nullptr && mask_bits == nullptr) return SBL_ERR_INVALID_ARG;
  // hyperparameters (written so that NaN fails every test)
  if (!(step >= 1) || !(lr >= 0.0) || !(beta1 >= 0.0 && beta1 < 1.0) || !(beta2 >= 0.0 && beta2 < 1.0) ||
      !(eps > 0.0) || !(weight_decay >= 0.0) || (grad_sqnorm != nullptr && !(max_norm > 0.0)))
    return SBL_ERR_INVALID_ARG;
  if ((st = check_dims(d_in, d_out)) != SBL_OK) return st;
  const unsigned long long n = static_cast<unsigned long long>(d_out) * static_cast<unsigned long long>(d_in);
  if (n == 0 || n >= (1ull << 32) || d_in % M != 0) return SBL_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(W32) || !aligned16(dW) || !aligned16(m) || !aligned16(v) || !aligned16(W_eff) ||
      !aligned16(W_eff_bf16) || !aligned16(mask_bits) || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      (reinterpret_cast<uintptr_t>(gamma) & 3u) != 0 || (reinterpret_cast<uintptr_t>(grad_sqnorm) & 7u) != 0 ||
      (reinterpret_cast<uintptr_t>(flips) & 7u) != 0)
    return SBL_ERR_ALIGN;
  if (workspace_bytes < mask_quant_workspace_bytes()) return SBL_ERR_WORKSPACE;
  DeviceInfo* d = nullptr;
  if ((st = current_device(&d)) != SBL_OK) return st;
  const AdamwParams hp{lr, beta1, beta2, eps, weight_decay, max_norm, step};
  return from_cuda(launch_adamw_step(W, W32, dW, m, v, d_out, d_in, N, M, hp, grad_sqnorm, W_eff, W_eff_bf16,
                                     mask_bits, gamma, flips, workspace, static_cast<cudaStream_t>(stream),
                                     d->num_sms));
}

sbl_status sbl_act_quant(const void* X, int T, int d_in, int8_t* Xq, float* amax, void* stream) {
  if (T < 0 || d_in <= 0 || d_in % 16 != 0) return SBL_ERR_SHAPE;
  if (T == 0) return SBL_OK;
  if (X == nullptr || Xq == nullptr || amax == nullptr) return SBL_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Xq) || !aligned16(amax)) return SBL_ERR_ALIGN;
  DeviceInfo* d = nullptr;
  sbl_status st = current_device(&d);
  if (st != SBL_OK) return st;
  return from_cuda(launch_act_quant(X, T, d_in, Xq, amax, static_cast<cudaStream_t>(stream), d->num_sms));
}

sbl_status sbl_rmsnorm_act_quant(const void* X, const void* g, float eps, int T, int d_in, void* Xn, int8_t* Xq,
                                 float* amax, void* stream) {
  if (T < 0 || d_in <= 0 || d_in % 16 != 0) return SBL_ERR_SHAPE;
  if (T == 0) return SBL_OK;
  if (X == nullptr || g == nullptr || Xq == nullptr || amax == nullptr || !(eps > 0.0f)) return SBL_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(g) || !aligned16(Xn) || !aligned16(Xq) || !aligned16(amax)) return SBL_ERR_ALIGN;
  DeviceInfo* d = nullptr;
  sbl_status st = current_device(&d);
  if (st != SBL_OK) return st;
  return from_cuda(launch_norm_act_quant(X, g, eps, T, d_in, Xn, Xq, amax, static_cast<cudaStream_t>(stream),
                                         d->num_sms));
}

sbl_status sbl_forward(const int8_t* Xq, const float* amax, const int8_t* W_eff, const float* gamma, int T,
                       int d_in, int d_out, float* Y, int32_t* acc, void* stream) {
  sbl_status st = check_dims(d_in, d_out);
  if (st != SBL_OK) return st;
  if (T < 0) return SBL_ERR_SHAPE;
  if (T == 0 || d_out == 0) return SBL_OK;
  if (Xq == nullptr || amax == nullptr || W_eff == nullptr || gamma == nullptr || Y == nullptr)
    return SBL_ERR_INVALID_ARG;
  if (!aligned16(Xq) || !aligned16(amax) || !aligned16(W_eff) || !aligned16(Y) || !aligned16(acc) ||
      (reinterpret_cast<uintptr_t>(gamma) & 3u) != 0)
    return SBL_ERR_ALIGN;
  DeviceInfo* d = nullptr;
  if ((st = current_device(&d)) != SBL_OK) return st;
  return from_cuda(launch_forward(Xq, amax, W_eff, gamma, T, d_in, d_out, Y, acc, static_cast<cudaStream_t>(stream),
                                  d->num_sms, d->err));
}

sbl_status sbl_forward_group(const sbl_forward_problem* problems, int count, void* stream) {
  if (count < 0 || (count > 0 && problems == nullptr)) return SBL_ERR_INVALID_ARG;
  if (count == 0) return SBL_OK;
  std::vector<FwdProblemDev> dev;
  dev.reserve(static_cast<size_t>(count));
  for (int i = 0; i < count; ++i) {
    const sbl_forward_problem& q = problems[i];
    sbl_status st = check_dims(q.d_in, q.d_out);
    if (st != SBL_OK) return st;
    if (q.T < 0) return SBL_ERR_SHAPE;
    if (q.T == 0 || q.d_out == 0) continue;
    if (q.Xq == nullptr || q.amax == nullptr || q.W_eff == nullptr || q.gamma == nullptr || q.Y == nullptr)
      return SBL_ERR_INVALID_ARG;
    if (!aligned16(q.Xq) || !aligned16(q.amax) || !aligned16(q.W_eff) || !aligned16(q.Y) || !aligned16(q.acc) ||
        (reinterpret_cast<uintptr_t>(q.gamma) & 3u) != 0)
      return SBL_ERR_ALIGN;
    dev.push_back(FwdProblemDev{q.Xq, q.amax, q.W_eff, q.gamma, q.T, q.d_in, q.d_out, q.Y, q.acc});
  }
  if (dev.empty()) return SBL_OK;
  DeviceInfo* d = nullptr;
  const sbl_status st = current_device(&d);
  if (st != SBL_OK) return st;
  return from_cuda(launch_forward_group(dev.data(), static_cast<int>(dev.size()), static_cast<cudaStream_t>(stream),
                                        d->num_sms, d->err));
}

sbl_status sbl_forward_packed(const int8_t* Xq, const float* amax, const uint8_t* packed, const float* gamma,
                              int T, int d_in, int d_out, int N, int M, float* Y, int32_t* acc, void* stream) {
  sbl_status st = check_nm(N, M);
  if (st != SBL_OK) return st;
  if ((st = check_dims(d_in, d_out)) != SBL_OK) return st;
  if (T < 0 || d_in % M != 0) return SBL_ERR_SHAPE;
  if (T == 0 || d_out == 0) return SBL_OK;
  if (Xq == nullptr || amax == nullptr || packed == nullptr || gamma == nullptr || Y == nullptr)
    return SBL_ERR_INVALID_ARG;
  if (!aligned16(Xq) || !aligned16(amax) || !aligned16(packed) || !aligned16(Y) || !aligned16(acc) ||
      (reinterpret_cast<uintptr_t>(gamma) & 3u) != 0)
    return SBL_ERR_ALIGN;
  DeviceInfo* d = nullptr;
  if ((st = current_device(&d)) != SBL_OK) return st;
  return from_cuda(launch_forward_packed(Xq, amax, packed, gamma, T, d_in, d_out, N, M, Y, acc,
                                         static_cast<cudaStream_t>(stream), d->num_sms, d->err));
}

size_t sbl_compress24_bytes(int d_out, int d_in) {
  if (check_dims(d_in, d_out) != SBL_OK) return 0;
  return sparse24_bytes(d_out, d_in);
}

sbl_status sbl_compress24(const int8_t* W_eff, int d_out, int d_in, uint8_t* out, size_t out_bytes, void* stream) {
  sbl_status st = check_dims(d_in, d_out);
  if (st != SBL_OK) return st;
  if (d_out == 0 || d_in == 0) return SBL_OK;
  if (W_eff == nullptr || out == nullptr) return SBL_ERR_INVALID_ARG;
  if (!aligned16(W_eff) || !aligned16(out)) return SBL_ERR_ALIGN;
  if (out_bytes < sparse24_bytes(d_out, d_in)) return SBL_ERR_WORKSPACE;
  DeviceInfo* d = nullptr;
  if ((st = current_device(&d)) != SBL_OK) return st;
  return from_cuda(launch_compress24(W_eff, d_out, d_in, out, static_cast<cudaStream_t>(stream), d->num_sms,
                                     d->err));
}

sbl_status sbl_forward_sparse24(const int8_t* Xq, const float* amax, const uint8_t* w24, const float* gamma, int T,
                                int d_in, int d_out, float* Y, int32_t* acc, void* stream) {
  sbl_status st = check_dims(d_in, d_out);
  if (st != SBL_OK) return st;
  if (T < 0) return SBL_ERR_SHAPE;
  if (T == 0 || d_out == 0) return SBL_OK;
  if (Xq == nullptr || amax == nullptr || w24 == nullptr || gamma == nullptr || Y == nullptr)
    return SBL_ERR_INVALID_ARG;
  if (!aligned16(Xq) || !aligned16(amax) || !aligned16(w24) || !aligned16(Y) || !aligned16(acc) ||
      (reinterpret_cast<uintptr_t>(gamma) & 3u) != 0)
    return SBL_ERR_ALIGN;
  DeviceInfo* d = nullptr;
  if ((st = current_device(&d)) != SBL_OK) return st;
  return from_cuda(launch_forward_sparse24(Xq, amax, w24, gamma, T, d_in, d_out, Y, acc,
                                           static_cast<cudaStream_t>(stream), d->num_sms, d->err));
}

size_t sbl_backward_workspace_bytes(int T, int d_in, int d_out) {
  (void)T;
  (void)d_in;
  (void)d_out;
  return 0;
}

sbl_status sbl_backward(const void* dY, const void* X, const void* W_eff_bf16, const float* gamma, int T,
                        int d_in, int d_out, float* dX, float* dW, int accumulate_dW, void* workspace,
                        size_t workspace_bytes, void* stream) {
  (void)workspace;
  (void)workspace_bytes;
  sbl_status st = check_dims(d_in, d_out);
  if (st != SBL_OK) return st;
  if (T < 0) return SBL_ERR_SHAPE;
  if (dX == nullptr && dW == nullptr) return SBL_OK;
  if (T > 0 && dY == nullptr) return SBL_ERR_INVALID_ARG;
  if (dX != nullptr && (W_eff_bf16 == nullptr || gamma == nullptr)) return SBL_ERR_INVALID_ARG;
  if (dW != nullptr && T > 0 && X == nullptr) return SBL_ERR_INVALID_ARG;
  if (!aligned16(dY) || !aligned16(X) || !aligned16(W_eff_bf16) || !aligned16(dX) || !aligned16(dW) ||
      (reinterpret_cast<uintptr_t>(gamma) & 3u) != 0)
    return SBL_ERR_ALIGN;
  DeviceInfo* d = nullptr;
  if ((st = current_device(&d)) != SBL_OK) return st;
  return from_cuda(launch_backward(dY, X, W_eff_bf16, gamma, T, d_in, d_out, dX, dW, accumulate_dW,
                                   static_cast<cudaStream_t>(stream), d->num_sms, d->err));
}

size_t sbl_packed_bytes(int d_out, int d_in, int N, int M) {
  if (check_nm(N, M) != SBL_OK || check_dims(d_in, d_out) != SBL_OK || d_in % M != 0) return 0;
  return static_cast<size_t>(d_out) * (packed_codes_row_bytes(d_in, N, M) + packed_index_row_bytes(d_in, M));
}

sbl_status sbl_pack(const int8_t* W_eff, int d_out, int d_in, int N, int M, uint8_t* packed, size_t packed_bytes,
                    void* stream) {
  sbl_status st = check_nm(N, M);
  if (st != SBL_OK) return st;
  if ((st = check_dims(d_in, d_out)) != SBL_OK) return st;
  if (d_in % M != 0) return SBL_ERR_SHAPE;
  if (d_out == 0 || d_in == 0) return SBL_OK;
  if (W_eff == nullptr || packed == nullptr) return SBL_ERR_INVALID_ARG;
  if (!aligned16(W_eff) || !aligned16(packed)) return SBL_ERR_ALIGN;
  if (packed_bytes < sbl_packed_bytes(d_out, d_in, N, M)) return SBL_ERR_WORKSPACE;
  DeviceInfo* d = nullptr;
  if ((st = current_device(&d)) != SBL_OK) return st;
  return from_cuda(launch_pack(W_eff, d_out, d_in, N, M, packed, static_cast<cudaStream_t>(stream), d->err));
}

sbl_status sbl_unpack(const uint8_t* packed, int d_out, int d_in, int N, int M, int8_t* W_eff, void* stream) {
  sbl_status st = check_nm(N, M);
  if (st != SBL_OK) return st;
  if ((st = check_dims(d_in, d_out)) != SBL_OK) return st;
  if (d_in % M != 0) return SBL_ERR_SHAPE;
  if (d_out == 0 || d_in == 0) return SBL_OK;
  if (packed == nullptr || W_eff == nullptr) return SBL_ERR_INVALID_ARG;
  if (!aligned16(packed) || !aligned16(W_eff)) return SBL_ERR_ALIGN;
  DeviceInfo* d = nullptr;
  if ((st = current_device(&d)) != SBL_OK) return st;
  return from_cuda(launch_unpack(packed, d_out, d_in, N, M, W_eff, static_cast<cudaStream_t>(stream), d->num_sms));
}

sbl_status sbl_gemv_packed(const int8_t* Xq, const float* amax, int batch, const uint8_t* packed,
                           const float* gamma, int d_in, int d_out, int N, int M, float* Y, void* stream) {
  sbl_status st = check_nm(N, M);
  if (st != SBL_OK) return st;
  if ((st = check_dims(d_in, d_out)) != SBL_OK) return st;
  if (d_in % M != 0 || batch < 0 || batch > 16) return SBL_ERR_SHAPE;
  if (batch == 0 || d_out == 0) return SBL_OK;
  if (Xq == nullptr || amax == nullptr || packed == nullptr || gamma == nullptr || Y == nullptr)
    return SBL_ERR_INVALID_ARG;
  if (!aligned16(Xq) || !aligned16(amax) || !aligned16(packed) || !aligned16(Y) ||
      (reinterpret_cast<uintptr_t>(gamma) & 3u) != 0)
    return SBL_ERR_ALIGN;
  DeviceInfo* d = nullptr;
  if ((st = current_device(&d)) != SBL_OK) return st;
  return from_cuda(launch_gemv_packed(Xq, amax, batch, packed, gamma, d_in, d_out, N, M, Y,
                                      static_cast<cudaStream_t>(stream), d->num_sms, d->err));
}

sbl_status sbl_gemv_packed_group(const sbl_gemv_problem* problems, int count, int batch, int N, int M,
                                 void* stream) {
  sbl_status st = check_nm(N, M);
  if (st != SBL_OK) return st;
  if (count < 0 || batch < 0 || batch > 16) return SBL_ERR_SHAPE;
  if (count == 0 || batch == 0) return SBL_OK;
  if (problems == nullptr) return SBL_ERR_INVALID_ARG;
  std::vector<GemvProblemDev> dev(static_cast<size_t>(count));
  for (int i = 0; i < count; ++i) {
    const sbl_gemv_problem& p = problems[i];
    if ((st = check_dims(p.d_in, p.d_out)) != SBL_OK) return st;
    if (p.d_in % M != 0 || p.d_in == 0) return SBL_ERR_SHAPE;
    if (p.Xq == nullptr || p.amax == nullptr || p.packed == nullptr || p.gamma == nullptr || p.Y == nullptr)
      return SBL_ERR_INVALID_ARG;
    if (!aligned16(p.Xq) || !aligned16(p.amax) || !aligned16(p.packed) || !aligned16(p.Y) ||
        (reinterpret_cast<uintptr_t>(p.gamma) & 3u) != 0)
      return SBL_ERR_ALIGN;
    dev[i] = GemvProblemDev{p.packed, p.Xq, p.amax, p.gamma, p.Y, p.d_in, p.d_out, 0, 0, 0};
  }
  DeviceInfo* d = nullptr;
  if ((st = current_device(&d)) != SBL_OK) return st;
  return from_cuda(launch_gemv_group(dev.data(), count, batch, N, M, static_cast<cudaStream_t>(stream), d->num_sms,
                                     d->err, false));
}

size_t sbl_dense2_bytes(int d_out, int d_in) {
  if (check_dims(d_in, d_out) != SBL_OK) return 0;
  return static_cast<size_t>(d_out) * dense2_row_bytes(d_in);
}

sbl_status sbl_pack_dense2(const int8_t* W_eff, int d_out, int d_in, uint8_t* out, size_t out_bytes, void* stream) {
  sbl_status st = check_dims(d_in, d_out);
  if (st != SBL_OK) return st;
  if (d_out == 0 || d_in == 0) return SBL_OK;
  if (W_eff == nullptr || out == nullptr) return SBL_ERR_INVALID_ARG;
  if (!aligned16(W_eff) || !aligned16(out)) return SBL_ERR_ALIGN;
  if (out_bytes < sbl_dense2_bytes(d_out, d_in)) return SBL_ERR_WORKSPACE;
  DeviceInfo* d = nullptr;
  if ((st = current_device(&d)) != SBL_OK) return st;
  return from_cuda(launch_pack_dense2(W_eff, d_out, d_in, out, static_cast<cudaStream_t>(stream), d->num_sms));
}

sbl_status sbl_gemv_dense2_group(const sbl_gemv_problem* problems, int count, int batch, void* stream) {
  if (count < 0 || batch < 0 || batch > 16) return SBL_ERR_SHAPE;
  if (count == 0 || batch == 0) return SBL_OK;
  if (problems == nullptr) return SBL_ERR_INVALID_ARG;
  std::vector<GemvProblemDev> dev(static_cast<size_t>(count));
  sbl_status st = SBL_OK;
  for (int i = 0; i < count; ++i) {
    const sbl_gemv_problem& p = problems[i];
    if ((st = check_dims(p.d_in, p.d_out)) != SBL_OK) return st;
    if (p.d_in == 0) return SBL_ERR_SHAPE;
    if (p.Xq == nullptr || p.amax == nullptr || p.packed == nullptr || p.gamma == nullptr || p.Y == nullptr)
      return SBL_ERR_INVALID_ARG;
    if (!aligned16(p.Xq) || !aligned16(p.amax) || !aligned16(p.packed) || !aligned16(p.Y) ||
        (reinterpret_cast<uintptr_t>(p.gamma) & 3u) != 0)
      return SBL_ERR_ALIGN;
    dev[i] = GemvProblemDev{p.packed, p.Xq, p.amax, p.gamma, p.Y, p.d_in, p.d_out, 0, 0, 0};
  }
  DeviceInfo* d = nullptr;
  if ((st = current_device(&d)) != SBL_OK) return st;
  return from_cuda(launch_gemv_group(dev.data(), count, batch, 8, 8, static_cast<cudaStream_t>(stream), d->num_sms,
                                     d->err, true));
}

}  // extern "C"
