// m3_norm.cu -- the hybrid model's output norm (m3_output_norm).
//
// The Mamba-3 paper note (docsaid.org, section アーキテクチャ) removes the norm before the
// output projection in the pure Mamba-3 model and keeps it in the hybrid one.  The block's
// gate z is applied first when given, then each (batch, token, head) row of P values is
// RMS-normalised and scaled per channel:
//   v = y * silu(z)  (v = y without a gate),   out = weight[h] * v / sqrt(mean_p v^2 + eps).
// One warp per row (lanes take consecutive columns, so every load and store is coalesced), rows
// in a grid-stride loop; the kernel is bound by HBM: it reads y (and z) and writes out once.
#include "m3_common.cuh"

namespace m3 {
namespace {

constexpr int kNormWarps = 8;

template <bool BF16>
__global__ void __launch_bounds__(32 * kNormWarps)
    output_norm_kernel(int64_t rows, int H, int P, const void* y, const void* z, const float* weight, float eps,
                       void* out) {
  const int lane = threadIdx.x & 31;
  const int64_t stride = (int64_t)gridDim.x * kNormWarps;
  for (int64_t row = (int64_t)blockIdx.x * kNormWarps + (threadIdx.x >> 5); row < rows; row += stride) {
    const int64_t base = row * P;
    float v[8];
    float ss = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      v[i] = 0.0f;
      if (e < P) {
        float a = load_in<BF16>(y, base + e);
        if (z) {
          const float g = load_in<BF16>(z, base + e);
          a *= g / (1.0f + __expf(-g));
        }
        v[i] = a;
        ss = fmaf(a, a, ss);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float scale = rsqrtf(ss / (float)P + eps);
    const float* w = weight ? weight + (int64_t)(row % H) * P : nullptr;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      if (e < P) store_out<BF16>(out, base + e, v[i] * scale * (w ? w[e] : 1.0f));
    }
  }
}

}  // namespace

cudaError_t launch_output_norm(const Params& p, const void* z, const float* weight, float eps, void* out,
                               cudaStream_t stream) {
  const int64_t rows = p.b * p.L * p.H;
  int dev = 0, nsm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (rows + kNormWarps - 1) / kNormWarps;
  const int64_t cap = (int64_t)nsm * 16;  // 16 resident CTAs of 8 warps per SM: a full wave
  if (blocks > cap) blocks = cap;
  if (p.dtype == M3_BF16)
    output_norm_kernel<true><<<(unsigned)blocks, 32 * kNormWarps, 0, stream>>>(rows, p.H, p.P, p.y, z, weight, eps, out);
  else
    output_norm_kernel<false><<<(unsigned)blocks, 32 * kNormWarps, 0, stream>>>(rows, p.H, p.P, p.y, z, weight, eps, out);
  return cudaGetLastError();
}

}  // namespace m3
