// m3_scan_seq.cu -- token-sequential SIMT kernel of the Mamba-3 SSM core.
//
// One CTA per (batch, head).  The fp32 state h (N x P) lives in registers: each
// compute thread owns column quad p0..p0+3 of the rotation pairs (2k, 2k+1),
// k = kg, kg + KG, ...  Per token the CTA stages the biased B/C rows, the MIMO
// branches X_r = W_x[r] * x and the rotation table in shared memory, applies
//     h <- e^{dt A} Rot(dt theta) (h + (1 - lam) dt u_{t-1}) + lam dt u_t,
//     u = sum_r Bb_r X_r^T,
// (Mamba-3 paper note, docsaid.org: section その1 for the trapezoid rule,
// section その2 for the rotation, section その3 for the rank-R update) and reduces
// the R readouts Cb_r^T h over N across the CTA.
//
// It serves two entry points:
//   * m3_decode_step (L = 1): the state is streamed from and back to HBM with
//     128-bit loads/stores, all issued before any arithmetic; the kernel is
//     HBM-bound (8 bytes of state traffic per state element per token);
//   * m3_scan_fwd for fp32 inputs, shapes the tensor-core scan does not cover,
//     and M3_FLAG_SEQUENTIAL.
#include "m3_common.cuh"

namespace m3 {

namespace {

constexpr int kThreads = 256;

struct SeqShape {
  int PQ;  // column quads per row = P / 4
  int KG;  // pair groups = threads sharing one column quad
  int K;   // rotation pairs = N / 2
};

__host__ __device__ inline SeqShape seq_shape(int P, int N) {
  SeqShape s;
  s.PQ = P / 4;
  s.K = N / 2;
  int kg = kThreads / s.PQ;
  s.KG = kg < s.K ? kg : s.K;
  return s;
}

// Shared-memory plan (floats): two slots of biased B and of X (current / previous
// token), biased C, the rotation table, 4 coefficients, the readout partials.
struct SeqSmem {
  int bb0, bb1, cb, x0, x1, cs, coef, red, total;
};

__host__ __device__ inline SeqSmem seq_smem(int P, int N, int R, int KG) {
  SeqSmem m;
  int o = 0;
  m.bb0 = o; o += R * N;
  m.bb1 = o; o += R * N;
  m.cb = o;  o += R * N;
  m.x0 = o;  o += R * P;
  m.x1 = o;  o += R * P;
  m.cs = o;  o += N;          // (cos, sin) per pair
  m.coef = o; o += 4;
  o = (o + 3) & ~3;
  m.red = o; o += KG * R * P;
  m.total = o;
  return m;
}

template <int RT, int NK, bool BF16>
__global__ void __launch_bounds__(kThreads)
scan_seq_kernel(Params p) {
  extern __shared__ __align__(16) float sm[];
  const int tid = threadIdx.x;
  const int H = p.H, P = p.P, N = p.N, R = p.R, G = p.G;
  const int64_t L = p.L;
  const int bi = blockIdx.x / H, hi = blockIdx.x % H;
  const int g = hi / (H / G);
  const SeqShape sh = seq_shape(P, N);
  const SeqSmem ms = seq_smem(P, N, R, sh.KG);
  const int pq = tid % sh.PQ;
  const int kg = tid / sh.PQ;
  const bool active = kg < sh.KG;
  const int p0 = 4 * pq;

  float* const bbs[2] = {sm + ms.bb0, sm + ms.bb1};
  float* const xs[2] = {sm + ms.x0, sm + ms.x1};
  float* const cb = sm + ms.cb;
  float2* const cs = reinterpret_cast<float2*>(sm + ms.cs);
  float* const coef = sm + ms.coef;
  float* const red = sm + ms.red;

  float* hbase = p.h + ((int64_t)blockIdx.x * N) * P;
  float* cBb = p.carry_B + ((int64_t)blockIdx.x * R) * N;
  float* cxb = p.carry_x + (int64_t)blockIdx.x * P;
  const float* biasB = p.bias_B ? p.bias_B + (int64_t)hi * R * N : nullptr;
  const float* biasC = p.bias_C ? p.bias_C + (int64_t)hi * R * N : nullptr;
  const float* Wx = p.W_x ? p.W_x + (int64_t)hi * R * P : nullptr;
  const float* Wo = p.W_o ? p.W_o + (int64_t)hi * R * P : nullptr;
  const float Dh = p.D ? p.D[hi] : 0.0f;

  // ---- state into registers: all 128-bit loads issued first
  float4 h0[NK], h1[NK];
#pragma unroll
  for (int j = 0; j < NK; ++j) {
    const int k = kg + j * sh.KG;
    if (active && k < sh.K) {
      h0[j] = *reinterpret_cast<const float4*>(hbase + (int64_t)(2 * k) * P + p0);
      h1[j] = *reinterpret_cast<const float4*>(hbase + (int64_t)(2 * k + 1) * P + p0);
    } else {
      h0[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      h1[j] = h0[j];
    }
  }

  // ---- previous-token slot from the carry
  for (int i = tid; i < R * N; i += kThreads) bbs[1][i] = cBb[i] + (biasB ? biasB[i] : 0.0f);
  for (int i = tid; i < R * P; i += kThreads) xs[1][i] = cxb[i % P] * (Wx ? Wx[i] : 1.0f);

  int cur = 0;
  for (int64_t t = 0; t < L; ++t) {
    const int64_t tok = (int64_t)bi * L + t;
    // ---- stage token t
    {
      const int64_t bcoff = ((tok * G + g) * R) * (int64_t)N;
      for (int i = tid; i < R * N; i += kThreads) {
        bbs[cur][i] = load_in<BF16>(p.B, bcoff + i) + (biasB ? biasB[i] : 0.0f);
        cb[i] = load_in<BF16>(p.C, bcoff + i) + (biasC ? biasC[i] : 0.0f);
      }
      const int64_t xoff = (tok * H + hi) * (int64_t)P;
      for (int i = tid; i < R * P; i += kThreads)
        xs[cur][i] = load_in<BF16>(p.x, xoff + (i % P)) * (Wx ? Wx[i] : 1.0f);
      const float delta = p.dt[tok * H + hi];
      const float* th = p.theta + (tok * G + g) * (int64_t)(N / 2);
      for (int k = tid; k < N / 2; k += kThreads) {
        float s, c;
        sincosf(p.angle_direct ? th[k] : delta * th[k], &s, &c);
        cs[k] = make_float2(c, s);
      }
      if (tid == 0) {
        const float lm = p.lam[tok * H + hi];
        coef[0] = expf(delta * p.A[tok * H + hi]);  // alpha
        coef[1] = (1.0f - lm) * delta;             // beta'
        coef[2] = lm * delta;                      // gamma
      }
    }
    __syncthreads();

    // ---- state update and partial readouts
    if (active) {
      const float* bbc = bbs[cur];
      const float* bbp = bbs[cur ^ 1];
      const float* xc = xs[cur];
      const float* xp = xs[cur ^ 1];
      const float alpha = coef[0], bp = coef[1], gm = coef[2];
      float4 Xc[RT], Xp[RT];
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        if (r < R) {
          Xc[r] = *reinterpret_cast<const float4*>(xc + r * P + p0);
          Xp[r] = *reinterpret_cast<const float4*>(xp + r * P + p0);
        } else {
          Xc[r] = Xp[r] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      float Y[RT][4];
#pragma unroll
      for (int r = 0; r < RT; ++r) Y[r][0] = Y[r][1] = Y[r][2] = Y[r][3] = 0.0f;
#pragma unroll
      for (int j = 0; j < NK; ++j) {
        const int k = kg + j * sh.KG;
        if (k < sh.K) {
          float u0[4] = {0, 0, 0, 0}, u1[4] = {0, 0, 0, 0}, q0[4] = {0, 0, 0, 0}, q1[4] = {0, 0, 0, 0};
#pragma unroll
          for (int r = 0; r < RT; ++r) {
            if (r < R) {
              const float2 bc = *reinterpret_cast<const float2*>(bbc + r * N + 2 * k);
              const float2 bq = *reinterpret_cast<const float2*>(bbp + r * N + 2 * k);
              const float xc4[4] = {Xc[r].x, Xc[r].y, Xc[r].z, Xc[r].w};
              const float xp4[4] = {Xp[r].x, Xp[r].y, Xp[r].z, Xp[r].w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                u0[e] = fmaf(bc.x, xc4[e], u0[e]);
                u1[e] = fmaf(bc.y, xc4[e], u1[e]);
                q0[e] = fmaf(bq.x, xp4[e], q0[e]);
                q1[e] = fmaf(bq.y, xp4[e], q1[e]);
              }
            }
          }
          const float2 rc = cs[k];
          float a0[4] = {h0[j].x, h0[j].y, h0[j].z, h0[j].w};
          float a1[4] = {h1[j].x, h1[j].y, h1[j].z, h1[j].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float v0 = fmaf(bp, q0[e], a0[e]);
            const float v1 = fmaf(bp, q1[e], a1[e]);
            a0[e] = fmaf(alpha, rc.x * v0 - rc.y * v1, gm * u0[e]);
            a1[e] = fmaf(alpha, rc.y * v0 + rc.x * v1, gm * u1[e]);
          }
          h0[j] = make_float4(a0[0], a0[1], a0[2], a0[3]);
          h1[j] = make_float4(a1[0], a1[1], a1[2], a1[3]);
#pragma unroll
          for (int r = 0; r < RT; ++r) {
            if (r < R) {
              const float2 cc = *reinterpret_cast<const float2*>(cb + r * N + 2 * k);
#pragma unroll
              for (int e = 0; e < 4; ++e) Y[r][e] = fmaf(cc.x, a0[e], fmaf(cc.y, a1[e], Y[r][e]));
            }
          }
        }
      }
#pragma unroll
      for (int r = 0; r < RT; ++r)
        if (r < R)
          *reinterpret_cast<float4*>(red + (kg * R + r) * P + p0) = make_float4(Y[r][0], Y[r][1], Y[r][2], Y[r][3]);
    }
    __syncthreads();

    // ---- combine: y = sum_r W_o[r] * (sum over pair groups) + D x
    {
      const int64_t xoff = (tok * H + hi) * (int64_t)P;
      for (int pp = tid; pp < P; pp += kThreads) {
        float acc = 0.0f;
        for (int r = 0; r < R; ++r) {
          float s = 0.0f;
          for (int q = 0; q < sh.KG; ++q) s += red[(q * R + r) * P + pp];
          acc = fmaf(Wo ? Wo[r * P + pp] : 1.0f, s, acc);
        }
        acc = fmaf(Dh, load_in<BF16>(p.x, xoff + pp), acc);
        store_out<BF16>(p.y, xoff + pp, acc);
      }
    }
    cur ^= 1;
  }

  // ---- state and carry back
#pragma unroll
  for (int j = 0; j < NK; ++j) {
    const int k = kg + j * sh.KG;
    if (active && k < sh.K) {
      *reinterpret_cast<float4*>(hbase + (int64_t)(2 * k) * P + p0) = h0[j];
      *reinterpret_cast<float4*>(hbase + (int64_t)(2 * k + 1) * P + p0) = h1[j];
    }
  }
  if (L > 0) {
    const int64_t tok = (int64_t)bi * L + (L - 1);
    const int64_t bcoff = ((tok * G + g) * R) * (int64_t)N;
    for (int i = tid; i < R * N; i += kThreads) cBb[i] = load_in<BF16>(p.B, bcoff + i);
    const int64_t xoff = (tok * H + hi) * (int64_t)P;
    for (int i = tid; i < P; i += kThreads) cxb[i] = load_in<BF16>(p.x, xoff + i);
  }
}

template <int RT, int NK>
cudaError_t launch_rt_nk(const Params& p, size_t smem, cudaStream_t stream) {
  const dim3 grid((unsigned)(p.b * p.H));
  if (p.dtype == M3_BF16) {
    auto k = scan_seq_kernel<RT, NK, true>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<grid, kThreads, smem, stream>>>(p);
  } else {
    auto k = scan_seq_kernel<RT, NK, false>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<grid, kThreads, smem, stream>>>(p);
  }
  return cudaGetLastError();
}

template <int RT>
cudaError_t launch_rt(const Params& p, int nk, size_t smem, cudaStream_t stream) {
  switch (nk) {
    case 1: return launch_rt_nk<RT, 1>(p, smem, stream);
    case 2: return launch_rt_nk<RT, 2>(p, smem, stream);
    case 4: return launch_rt_nk<RT, 4>(p, smem, stream);
    case 8: return launch_rt_nk<RT, 8>(p, smem, stream);
    default: return launch_rt_nk<RT, 16>(p, smem, stream);
  }
}

}  // namespace

bool seq_scan_supported(int P, int N, int R) {
  if (P % 8 || N % 8 || P > 256 || N > 256 || R < 1 || R > 8) return false;
  const SeqShape sh = seq_shape(P, N);
  const int nk = (sh.K + sh.KG - 1) / sh.KG;
  return nk <= 16;
}

cudaError_t launch_scan_sequential(const Params& p, cudaStream_t stream) {
  if (p.b * p.H == 0) return cudaSuccess;
  const SeqShape sh = seq_shape(p.P, p.N);
  int nk = (sh.K + sh.KG - 1) / sh.KG;
  int nk2 = 1;
  while (nk2 < nk) nk2 *= 2;
  const size_t smem = sizeof(float) * (size_t)seq_smem(p.P, p.N, p.R, sh.KG).total;
  if (p.R <= 1) return launch_rt<1>(p, nk2, smem, stream);
  if (p.R <= 2) return launch_rt<2>(p, nk2, smem, stream);
  if (p.R <= 4) return launch_rt<4>(p, nk2, smem, stream);
  return launch_rt<8>(p, nk2, smem, stream);
}

}  // namespace m3
