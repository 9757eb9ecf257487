// m3_frontend.cu -- the block's front-end on raw projections (m3_frontend, M3_FLAG_RAW_INPUTS).
//
// The Mamba-3 block normalises B and C before they enter the core (the QK-norm-like BCNorm of
// the Cartesia blog and the docsaid note, section アーキテクチャ; the biases are added after it,
// inside the core) and parameterises the step, the decay and the trapezoid weight through
// softplus, -exp and sigmoid (section その1's discretisation):
//   B = B_raw / sqrt(mean_N B_raw^2 + 1e-6)  per (token, group, branch) row, likewise C,
//   dt = softplus(dt_raw),  A = -exp(A_raw),  lam = sigmoid(lam_raw).
// One warp per B or C row (coalesced columns, a shuffle reduction of the squares), then a
// grid-stride loop over the per-head scalars.  HBM-bound: every raw value is read once and every
// transformed value written once.
#include "m3_common.cuh"

namespace m3 {
namespace {

constexpr int kFeWarps = 8;

template <bool BF16>
__global__ void __launch_bounds__(32 * kFeWarps)
    frontend_kernel(int64_t rows, int N, const void* Braw, const void* Craw, void* Bout, void* Cout,
                    int64_t nscal, const float* dt_raw, const float* A_raw, const float* lam_raw, float* dt,
                    float* A, float* lam) {
  const int lane = threadIdx.x & 31;
  const int64_t wstride = (int64_t)gridDim.x * kFeWarps;
  for (int64_t w = (int64_t)blockIdx.x * kFeWarps + (threadIdx.x >> 5); w < 2 * rows; w += wstride) {
    const bool isC = w >= rows;
    const int64_t base = (isC ? w - rows : w) * N;
    const void* src = isC ? Craw : Braw;
    void* dst = isC ? Cout : Bout;
    float v[8];
    float ss = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      v[i] = e < N ? load_in<BF16>(src, base + e) : 0.0f;
      ss = fmaf(v[i], v[i], ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float sc = rsqrtf(ss / (float)N + kBcNormEps);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      if (e < N) store_out<BF16>(dst, base + e, v[i] * sc);
    }
  }
  const int64_t tstride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nscal; i += tstride) {
    dt[i] = fe_softplus(dt_raw[i]);
    A[i] = fe_negexp(A_raw[i]);
    lam[i] = fe_sigmoid(lam_raw[i]);
  }
}

}  // namespace

cudaError_t launch_frontend(const Params& p, const void* Braw, const void* Craw, const float* dt_raw,
                            const float* A_raw, const float* lam_raw, void* B, void* C, float* dt, float* A,
                            float* lam, cudaStream_t stream) {
  const int64_t rows = p.b * p.L * p.G * p.R;
  const int64_t nscal = p.b * p.L * p.H;
  int dev = 0, nsm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (2 * rows + kFeWarps - 1) / kFeWarps;
  const int64_t byscal = (nscal + 32 * kFeWarps - 1) / (32 * kFeWarps);
  if (byscal > blocks) blocks = byscal;
  if (blocks > (int64_t)nsm * 8) blocks = (int64_t)nsm * 8;
  if (blocks < 1) blocks = 1;
  if (p.dtype == M3_BF16)
    frontend_kernel<true><<<(unsigned)blocks, 32 * kFeWarps, 0, stream>>>(rows, p.N, Braw, Craw, B, C, nscal, dt_raw,
                                                                          A_raw, lam_raw, dt, A, lam);
  else
    frontend_kernel<false><<<(unsigned)blocks, 32 * kFeWarps, 0, stream>>>(rows, p.N, Braw, Craw, B, C, nscal, dt_raw,
                                                                           A_raw, lam_raw, dt, A, lam);
  return cudaGetLastError();
}

}  // namespace m3
