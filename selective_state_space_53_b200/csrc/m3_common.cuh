// m3_common.cuh -- shared definitions of the libm3 CUDA kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/m3.h"

namespace m3 {

// Everything a kernel needs, passed by value.  Layouts are those of include/m3.h.
struct Params {
  int64_t b, L;
  int H, P, N, R, G;
  int dtype;  // M3_BF16 / M3_F32 for x, B, C, y
  int angle_direct;  // 1: the step's rotation angle is theta itself (M3_FLAG_ANGLE_DIRECT)
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

// Launchers (defined in the kernel files); return cudaGetLastError() of the launch.
cudaError_t launch_scan_sequential(const Params& p, cudaStream_t stream);
bool decode_supported(const Params& p);                       // one-token kernel fits on chip
cudaError_t launch_decode(const Params& p, cudaStream_t stream);
bool decode_tc_supported(const Params& p);                    // tensor-core form (d_state = headdim = 128, bf16)
cudaError_t launch_decode_tc(const Params& p, cudaStream_t stream);
bool tc_scan_supported(const Params& p);
size_t tc_scan_workspace_bytes(const Params& p);  // scratch the chunked scan needs (0: none)
cudaError_t launch_scan_tc(const Params& p, void* workspace, size_t workspace_bytes, cudaStream_t stream);
cudaError_t launch_selftest_wait(int* status, unsigned long long limit_ns, cudaStream_t stream);

}  // namespace m3
