// m3_common.cuh -- shared definitions of the libm3 CUDA kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "../../include/m3.h"

namespace m3 {

// Everything a kernel needs, passed by value.  Layouts are those of include/m3.h.
struct Params {
  int64_t b, L;
  int H, P, N, R, G;
  int dtype;  // M3_BF16 / M3_F32 for x, B, C, y
  int angle_direct;  // 1: the step's rotation angle is theta itself (M3_FLAG_ANGLE_DIRECT)
  int raw_inputs;    // 1: B, C, dt, A, lam are raw projections, transformed in the load stage
  const void* x;
  const float* dt;
  const float* A;
  const float* lam;
  const void* B;
  const void* C;
  const float* theta;
  const float* bias_B;  // may be null
  const float* bias_C;  // may be null
  const float* W_x;     // may be null
  const float* W_o;     // may be null
  const float* D;       // may be null
  float* h;             // (b, H, N, P)
  float* carry_B;       // (b, H, R, N)
  float* carry_x;       // (b, H, P)
  void* y;
  int* status;          // device status word (M3_OK / M3_ERR_TIMEOUT)
};

// The block's front-end on raw projections (m3_frontend): the activations of the step, the
// decay and the trapezoid weight, and the eps of the B/C RMS norm.
constexpr float kBcNormEps = 1e-6f;
__device__ __forceinline__ float fe_softplus(float v) { return v > 20.0f ? v : log1pf(__expf(v)); }
__device__ __forceinline__ float fe_negexp(float v) { return -__expf(v); }
__device__ __forceinline__ float fe_sigmoid(float v) { return 1.0f / (1.0f + __expf(-v)); }

// Record a failure in the device status word (first failure wins).
__device__ __forceinline__ void set_status(int* word, int s) { atomicCAS(word, 0, s); }

template <bool BF16>
__device__ __forceinline__ float load_in(const void* base, int64_t i) {
  if constexpr (BF16) {
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[i]);
  } else {
    return reinterpret_cast<const float*>(base)[i];
  }
}

template <bool BF16>
__device__ __forceinline__ void store_out(void* base, int64_t i, float v) {
  if constexpr (BF16) {
    reinterpret_cast<__nv_bfloat16*>(base)[i] = __float2bfloat16_rn(v);
  } else {
    reinterpret_cast<float*>(base)[i] = v;
  }
}

// A value per CUDA device, filled once and then read without locking, safe for callers on
// several host threads: the first caller for a device runs `fill` under a mutex and publishes
// the value with a release store of `ready`; later callers see `ready` with an acquire load,
// so they never read a half-written value.  A fill that fails leaves the slot empty (it is
// retried by the next call).  Devices beyond kMaxDevices are reported as failures.
template <typename T>
class PerDevice {
 public:
  static constexpr int kMaxDevices = 64;
  template <typename F>
  bool get(int dev, T* out, F&& fill) {
    if (dev < 0 || dev >= kMaxDevices) return false;
    Slot& s = slots_[dev];
    if (!s.ready.load(std::memory_order_acquire)) {
      std::lock_guard<std::mutex> lock(mu_);
      if (!s.ready.load(std::memory_order_relaxed)) {
        T v{};
        if (!fill(&v)) return false;
        s.value = v;
        s.ready.store(true, std::memory_order_release);
      }
    }
    *out = s.value;
    return true;
  }

 private:
  struct Slot {
    std::atomic<bool> ready{false};
    T value{};
  };
  Slot slots_[kMaxDevices];
  std::mutex mu_;
};

// Largest dynamic shared memory size set so far on each device for one kernel: the attribute
// call runs under a mutex, and a size already set is seen through an acquire load.
class SmemAttr {
 public:
  template <typename Kernel>
  cudaError_t ensure(Kernel kernel, int bytes) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= PerDevice<int>::kMaxDevices) return cudaErrorInvalidDevice;
    if (set_[dev].load(std::memory_order_acquire) >= bytes) return cudaSuccess;
    std::lock_guard<std::mutex> lock(mu_);
    if (set_[dev].load(std::memory_order_relaxed) >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) set_[dev].store(bytes, std::memory_order_release);
    return e;
  }

 private:
  std::atomic<int> set_[PerDevice<int>::kMaxDevices] = {};
  std::mutex mu_;
};

// Launchers (defined in the kernel files); return cudaGetLastError() of the launch.
cudaError_t launch_scan_sequential(const Params& p, cudaStream_t stream);
// the chunk-parallel form of the sequential scan (segments summarised, folded, then scanned)
size_t seq_scan_workspace_bytes(const Params& p);
cudaError_t launch_scan_seq_chunked(const Params& p, void* ws, size_t ws_bytes, cudaStream_t stream);
bool decode_supported(const Params& p);                       // one-token kernel fits on chip
cudaError_t launch_decode(const Params& p, cudaStream_t stream);
bool decode_tc_supported(const Params& p);                    // tensor-core form (d_state = headdim = 128, bf16)
cudaError_t launch_decode_tc(const Params& p, cudaStream_t stream);
bool tc_scan_supported(const Params& p);
bool ws_scan_supported(const Params& p);  // the warp-specialised kernel (headdim 128) takes these dims
size_t tc_scan_workspace_bytes(const Params& p);  // scratch the chunked scan needs (0: none)
cudaError_t launch_scan_tc(const Params& p, void* workspace, size_t workspace_bytes, cudaStream_t stream);
struct SegInfo;
size_t scan_summary_workspace_bytes(const Params& p);  // scratch of the range summary's state pass
cudaError_t launch_scan_summary_pass(const Params& p, void* ws, size_t ws_bytes, SegInfo* sg, cudaStream_t stream);
cudaError_t launch_range_summary(const Params& p, void* ws, size_t ws_bytes, float* Z, float* logdec, double* angle,
                                 float* bp_first, float* carry_B, float* carry_x, cudaStream_t stream);
cudaError_t launch_state_fold(const Params& p, int nranges, const float* Z, const float* logdec, const double* angle,
                              const float* bp_first, const float* carry_B, const float* carry_x, cudaStream_t stream);
bool bwd_supported(const Params& p);
size_t scan_bwd_workspace_bytes(const Params& p);
cudaError_t launch_scan_bwd(const Params& p, const void* dy, const float* dh_final, void* dx, float* ddt, float* dA,
                            float* dlam, void* dB, void* dC, float* dtheta, float* dbias_B, float* dbias_C,
                            float* dW_x, float* dW_o, float* dD, float* dh0, float* dcarry_B, float* dcarry_x,
                            void* ws, size_t ws_bytes, cudaStream_t stream);
cudaError_t launch_output_norm(const Params& p, const void* z, const float* weight, float eps, void* out,
                               cudaStream_t stream);
cudaError_t launch_frontend(const Params& p, const void* Braw, const void* Craw, const float* dt_raw,
                            const float* A_raw, const float* lam_raw, void* B, void* C, float* dt, float* A,
                            float* lam, cudaStream_t stream);
cudaError_t launch_selftest_wait(int* status, unsigned long long limit_ns, cudaStream_t stream);

}  // namespace m3
