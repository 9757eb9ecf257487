// m3_shard.cu -- summaries of token ranges and the fold that chains them: the pieces of a
// sequence split across devices.
//
// The scan over a sequence splits into ranges combined associatively (IBM Mamba page,
// hardware-aware scan).  For the Mamba-3 recurrence (Mamba-3 paper note, docsaid.org, sections
// その1-その3) a range of tokens t0..t1 acts on the state entering it as
//   h_{t1} = e^{sum_t dt_t A_t} Rot(sum_t phi_t) h+ + Z,   h+ = h_{t0-1} + beta'_{t0} u_{t0-1},
// where Z is the range's end state from a fresh start (zero state, no previous token) and
// u_{t0-1} = sum_r (B_{t0-1,r} + bias_B[r]) (W_x[r] * x_{t0-1})^T comes from the token before
// the range (the carry).  A range summary is (Z, total log decay, total angle per pair, beta'
// of the first token, the carry of the last token); folding the summaries of ranges 0..k-1
// onto the sequence's initial state gives the state entering range k.
//
// range_summary_kernel combines the sub-segment summaries of the chunked state pass (each from
// a zero start, in its own rotated frame) into the range's Z in the true frame, and gathers the
// totals, beta' of the first token and the carry.  state_fold_kernel applies summaries to a
// state.  Both are plain SIMT kernels: one CTA per (batch, head), threads over (pair, column).
#include "m3_common.cuh"
#include "m3_scan_plan.cuh"

namespace m3 {
namespace {

constexpr int kShardThreads = 256;

template <bool BF16>
__global__ void __launch_bounds__(kShardThreads)
    range_summary_kernel(const Params p, const SegInfo sg, float* Z, float* logdec, double* angle, float* bp_first,
                         float* carry_B, float* carry_x) {
  const int bh = blockIdx.x;
  const int H = p.H, P = p.P, N = p.N, R = p.R, G = p.G;
  const int bi = bh / H, hi = bh % H, g = hi / (H / G);
  const int K2 = N / 2, ns = sg.nsub;
  const int64_t L = p.L;
  for (int idx = threadIdx.x; idx < K2 * P; idx += blockDim.x) {
    const int k = idx / P, pc = idx % P;
    float v0 = 0.0f, v1 = 0.0f;
    for (int s = 0; s < ns; ++s) {
      const int64_t sidx = (int64_t)bh * ns + s;
      const float dec = __expf(sg.ws_l[sidx]);
      const float* wh = sg.ws_h + sidx * N * P;
      const float a0 = fmaf(dec, v0, wh[(int64_t)(2 * k) * P + pc]);
      const float a1 = fmaf(dec, v1, wh[(int64_t)(2 * k + 1) * P + pc]);
      float sn, cn;
      sincosf((float)sg.ws_phi[sidx * K2 + k], &sn, &cn);
      v0 = cn * a0 - sn * a1;
      v1 = sn * a0 + cn * a1;
    }
    Z[((int64_t)bh * N + 2 * k) * P + pc] = v0;
    Z[((int64_t)bh * N + 2 * k + 1) * P + pc] = v1;
  }
  for (int k = threadIdx.x; k < K2; k += blockDim.x) {
    double tot = 0.0;
    for (int s = 0; s < ns; ++s) tot += sg.ws_phi[((int64_t)bh * ns + s) * K2 + k];
    tot -= 6.283185307179586 * rint(tot * 0.15915494309189535);
    angle[(int64_t)bh * K2 + k] = tot;
  }
  if (threadIdx.x == 0) {
    float ld = 0.0f;
    for (int s = 0; s < ns; ++s) ld += sg.ws_l[(int64_t)bh * ns + s];
    logdec[bh] = ld;
    const int64_t t0 = (int64_t)bi * L * H + hi;
    bp_first[bh] = (1.0f - p.lam[t0]) * p.dt[t0];
  }
  const int64_t tokl = (int64_t)bi * L + (L - 1);
  for (int i = threadIdx.x; i < R * N; i += blockDim.x)
    carry_B[(int64_t)bh * R * N + i] = load_in<BF16>(p.B, ((tokl * G + g) * R) * (int64_t)N + i);
  for (int i = threadIdx.x; i < P; i += blockDim.x)
    carry_x[(int64_t)bh * P + i] = load_in<BF16>(p.x, (tokl * H + hi) * (int64_t)P + i);
}

__global__ void __launch_bounds__(kShardThreads)
    state_fold_kernel(int64_t nbh, int H, int P, int N, int R, int nranges, const float* Z, const float* logdec,
                      const double* angle, const float* bp_first, const float* carry_B, const float* carry_x,
                      const float* bias_B, const float* W_x, float* h, float* state_cB, float* state_cx) {
  const int bh = blockIdx.x;
  const int hi = bh % H, K2 = N / 2;
  for (int idx = threadIdx.x; idx < K2 * P; idx += blockDim.x) {
    const int k = idx / P, pc = idx % P;
    float* hp0 = h + ((int64_t)bh * N + 2 * k) * P + pc;
    float* hp1 = hp0 + P;
    float h0 = *hp0, h1 = *hp1;
    for (int q = 0; q < nranges; ++q) {
      // the previous-token term of the range's first token: u of the token before the range
      const float* cb = q == 0 ? state_cB + (int64_t)bh * R * N : carry_B + ((int64_t)(q - 1) * nbh + bh) * R * N;
      const float* cx = q == 0 ? state_cx + (int64_t)bh * P : carry_x + ((int64_t)(q - 1) * nbh + bh) * P;
      float u0 = 0.0f, u1 = 0.0f;
      for (int r = 0; r < R; ++r) {
        const float xr = (W_x ? W_x[((int64_t)hi * R + r) * P + pc] : 1.0f) * cx[pc];
        const float b0 = cb[r * N + 2 * k] + (bias_B ? bias_B[((int64_t)hi * R + r) * N + 2 * k] : 0.0f);
        const float b1 = cb[r * N + 2 * k + 1] + (bias_B ? bias_B[((int64_t)hi * R + r) * N + 2 * k + 1] : 0.0f);
        u0 = fmaf(b0, xr, u0);
        u1 = fmaf(b1, xr, u1);
      }
      const int64_t qi = (int64_t)q * nbh + bh;
      const float bp = bp_first[qi];
      const float a0 = fmaf(bp, u0, h0), a1 = fmaf(bp, u1, h1);
      const float dec = __expf(logdec[qi]);
      float sn, cn;
      sincosf((float)angle[qi * K2 + k], &sn, &cn);
      const float* z = Z + (qi * N + 2 * k) * P + pc;
      h0 = fmaf(dec, cn * a0 - sn * a1, z[0]);
      h1 = fmaf(dec, sn * a0 + cn * a1, z[P]);
    }
    *hp0 = h0;
    *hp1 = h1;
  }
  if (nranges == 0) return;
  __syncthreads();  // every thread has read the state's carry
  const int64_t last = (int64_t)(nranges - 1) * nbh + bh;
  for (int i = threadIdx.x; i < R * N; i += blockDim.x) state_cB[(int64_t)bh * R * N + i] = carry_B[last * R * N + i];
  for (int i = threadIdx.x; i < P; i += blockDim.x) state_cx[(int64_t)bh * P + i] = carry_x[last * P + i];
}

}  // namespace

cudaError_t launch_range_summary(const Params& p, void* ws, size_t ws_bytes, float* Z, float* logdec, double* angle,
                                 float* bp_first, float* carry_B, float* carry_x, cudaStream_t stream) {
  SegInfo sg;
  cudaError_t e = launch_scan_summary_pass(p, ws, ws_bytes, &sg, stream);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)(p.b * p.H);
  if (p.dtype == M3_BF16)
    range_summary_kernel<true><<<grid, kShardThreads, 0, stream>>>(p, sg, Z, logdec, angle, bp_first, carry_B, carry_x);
  else
    range_summary_kernel<false><<<grid, kShardThreads, 0, stream>>>(p, sg, Z, logdec, angle, bp_first, carry_B, carry_x);
  return cudaGetLastError();
}

cudaError_t launch_state_fold(const Params& p, int nranges, const float* Z, const float* logdec, const double* angle,
                              const float* bp_first, const float* carry_B, const float* carry_x, cudaStream_t stream) {
  const int64_t nbh = p.b * p.H;
  state_fold_kernel<<<(unsigned)nbh, kShardThreads, 0, stream>>>(nbh, p.H, p.P, p.N, p.R, nranges, Z, logdec, angle,
                                                                 bp_first, carry_B, carry_x, p.bias_B, p.W_x, p.h,
                                                                 p.carry_B, p.carry_x);
  return cudaGetLastError();
}

}  // namespace m3
