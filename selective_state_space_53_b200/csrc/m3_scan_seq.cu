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
//
// With a workspace, m3_scan_fwd splits every sequence into segments walked in parallel (the scan
// combines associatively over token ranges: IBM page "Mamba モデルとは", hardware-aware scan):
// a first launch summarises segments 0..S-2 from a zero start (end state Z, total log decay,
// total angle per pair), seq_fold_kernel folds the summaries into the state entering each
// segment, h_k = e^{logdec} Rot(angle) (h_{k-1} + beta'_{t0} u_{t0-1}) + Z, and a second launch
// scans every segment from its entering state, writing y (and, for the last one, the final
// state and carry).
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

// Segments of the chunk-parallel form (nseg = 1: the whole sequence in one block).
struct SeqSegs {
  int nseg;          // segments per sequence
  int mode;          // 0: scan each segment from its entering state; 1: summaries of segments 0..nseg-2
  int64_t seg_len;   // tokens per segment (the last may be shorter)
  float* h_in;       // (b*H, nseg, N, P) state entering each segment (segments 1..nseg-1)
  float* Z;          // (nseg-1, b*H, N, P) end state of each summarised segment from a zero start
  float* logdec;     // (nseg-1, b*H) sum of dt A over the segment
  double* angle;     // (nseg-1, b*H, N/2) sum of the rotation angles, reduced mod 2 pi
};

template <int RT, int NK, bool BF16>
__global__ void __launch_bounds__(kThreads)
scan_seq_kernel(Params p, SeqSegs sgs) {
  extern __shared__ __align__(16) float sm[];
  const int tid = threadIdx.x;
  const int H = p.H, P = p.P, N = p.N, R = p.R, G = p.G;
  const int64_t L = p.L;
  const bool summary = sgs.mode == 1;
  const int nsg = summary ? sgs.nseg - 1 : sgs.nseg;  // blocks per sequence
  const int bh = blockIdx.x / nsg, seg = blockIdx.x % nsg;
  const int64_t t0 = (int64_t)seg * sgs.seg_len;
  const int64_t t1 = (t0 + sgs.seg_len < L) ? t0 + sgs.seg_len : L;
  const bool last = !summary && seg == sgs.nseg - 1;
  const int bi = bh / H, hi = bh % H;
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

  // the entering state: the sequence's for segment 0, the folded one after it, zero in a summary
  float* hstate = p.h + ((int64_t)bh * N) * P;
  const float* hbase = seg == 0 ? hstate : sgs.h_in + ((int64_t)bh * sgs.nseg + seg) * N * P;
  float* cBb = p.carry_B + ((int64_t)bh * R) * N;
  float* cxb = p.carry_x + (int64_t)bh * P;
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
    if (active && k < sh.K && !summary) {
      h0[j] = *reinterpret_cast<const float4*>(hbase + (int64_t)(2 * k) * P + p0);
      h1[j] = *reinterpret_cast<const float4*>(hbase + (int64_t)(2 * k + 1) * P + p0);
    } else {
      h0[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      h1[j] = h0[j];
    }
  }

  // ---- previous-token slot: the carry for segment 0, the token before the segment after it, none
  //      in a summary (a fresh start)
  if (summary) {
    for (int i = tid; i < R * N; i += kThreads) bbs[1][i] = 0.0f;
    for (int i = tid; i < R * P; i += kThreads) xs[1][i] = 0.0f;
  } else if (seg == 0) {
    for (int i = tid; i < R * N; i += kThreads) bbs[1][i] = cBb[i] + (biasB ? biasB[i] : 0.0f);
    for (int i = tid; i < R * P; i += kThreads) xs[1][i] = cxb[i % P] * (Wx ? Wx[i] : 1.0f);
  } else {
    const int64_t tp = (int64_t)bi * L + t0 - 1;
    for (int i = tid; i < R * N; i += kThreads)
      bbs[1][i] = load_in<BF16>(p.B, ((tp * G + g) * R) * (int64_t)N + i) + (biasB ? biasB[i] : 0.0f);
    for (int i = tid; i < R * P; i += kThreads)
      xs[1][i] = load_in<BF16>(p.x, (tp * H + hi) * (int64_t)P + (i % P)) * (Wx ? Wx[i] : 1.0f);
  }
  float ldsum = 0.0f;   // summary: sum of dt A (thread 0)
  double angsum = 0.0;  // summary: sum of the angles of pair tid (tid < N / 2)

  int cur = 0;
  for (int64_t t = t0; t < t1; ++t) {
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
        const float phi = p.angle_direct ? th[k] : delta * th[k];
        sincosf(phi, &s, &c);
        cs[k] = make_float2(c, s);
        if (summary) angsum += (double)phi;
      }
      if (tid == 0) {
        const float lm = p.lam[tok * H + hi];
        coef[0] = expf(delta * p.A[tok * H + hi]);  // alpha
        coef[1] = (1.0f - lm) * delta;             // beta'
        coef[2] = lm * delta;                      // gamma
        if (summary) ldsum += delta * p.A[tok * H + hi];
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
    if (!summary) {
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

  // ---- a summary: Z, the total log decay and angles; else the last segment: state and carry back
  if (summary) {
    const int64_t si = (int64_t)seg * (p.b * H) + bh;
    float* z = sgs.Z + si * N * P;
#pragma unroll
    for (int j = 0; j < NK; ++j) {
      const int k = kg + j * sh.KG;
      if (active && k < sh.K) {
        *reinterpret_cast<float4*>(z + (int64_t)(2 * k) * P + p0) = h0[j];
        *reinterpret_cast<float4*>(z + (int64_t)(2 * k + 1) * P + p0) = h1[j];
      }
    }
    if (tid == 0) sgs.logdec[si] = ldsum;
    if (tid < N / 2) sgs.angle[si * (N / 2) + tid] = angsum - 6.283185307179586 * rint(angsum * 0.15915494309189535);
    return;
  }
  if (!last) return;
#pragma unroll
  for (int j = 0; j < NK; ++j) {
    const int k = kg + j * sh.KG;
    if (active && k < sh.K) {
      *reinterpret_cast<float4*>(hstate + (int64_t)(2 * k) * P + p0) = h0[j];
      *reinterpret_cast<float4*>(hstate + (int64_t)(2 * k + 1) * P + p0) = h1[j];
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

// The state entering every segment s = 1..nseg-1: the sequence's state folded through the
// summaries of segments 0..s-1 (thread = one column of one rotation pair).  The previous-token
// term of segment s-1's first token t0 comes from the carry (s-1 = 0) or the input token t0 - 1.
template <bool BF16>
__global__ void __launch_bounds__(kThreads) seq_fold_kernel(const Params p, const SeqSegs sgs) {
  const int bh = blockIdx.x;
  const int H = p.H, P = p.P, N = p.N, R = p.R, G = p.G, K2 = N / 2;
  const int bi = bh / H, hi = bh % H, g = hi / (H / G);
  const int64_t L = p.L, nbh = p.b * H;
  for (int idx = threadIdx.x; idx < K2 * P; idx += blockDim.x) {
    const int k = idx / P, pc = idx % P;
    float h0 = p.h[((int64_t)bh * N + 2 * k) * P + pc], h1 = p.h[((int64_t)bh * N + 2 * k + 1) * P + pc];
    for (int s = 1; s < sgs.nseg; ++s) {
      const int64_t t0 = (int64_t)(s - 1) * sgs.seg_len;  // first token of the folded segment
      float u0 = 0.0f, u1 = 0.0f;
      for (int r = 0; r < R; ++r) {
        float b0, b1, xv;
        if (s == 1) {
          b0 = p.carry_B[((int64_t)bh * R + r) * N + 2 * k];
          b1 = p.carry_B[((int64_t)bh * R + r) * N + 2 * k + 1];
          xv = p.carry_x[(int64_t)bh * P + pc];
        } else {
          const int64_t tp = (int64_t)bi * L + t0 - 1;
          b0 = load_in<BF16>(p.B, ((tp * G + g) * R + r) * (int64_t)N + 2 * k);
          b1 = load_in<BF16>(p.B, ((tp * G + g) * R + r) * (int64_t)N + 2 * k + 1);
          xv = load_in<BF16>(p.x, (tp * H + hi) * (int64_t)P + pc);
        }
        if (p.bias_B) {
          b0 += p.bias_B[((int64_t)hi * R + r) * N + 2 * k];
          b1 += p.bias_B[((int64_t)hi * R + r) * N + 2 * k + 1];
        }
        const float xr = (p.W_x ? p.W_x[((int64_t)hi * R + r) * P + pc] : 1.0f) * xv;
        u0 = fmaf(b0, xr, u0);
        u1 = fmaf(b1, xr, u1);
      }
      const int64_t tf = ((int64_t)bi * L + t0) * H + hi;
      const float bp = (1.0f - p.lam[tf]) * p.dt[tf];
      const int64_t si = (int64_t)(s - 1) * nbh + bh;
      const float a0 = fmaf(bp, u0, h0), a1 = fmaf(bp, u1, h1);
      const float dec = __expf(sgs.logdec[si]);
      float sn, cn;
      sincosf((float)sgs.angle[si * K2 + k], &sn, &cn);
      const float* z = sgs.Z + (si * N + 2 * k) * P + pc;
      h0 = fmaf(dec, cn * a0 - sn * a1, z[0]);
      h1 = fmaf(dec, sn * a0 + cn * a1, z[P]);
      float* hi_ = sgs.h_in + (((int64_t)bh * sgs.nseg + s) * N + 2 * k) * P + pc;
      hi_[0] = h0;
      hi_[P] = h1;
    }
  }
}

template <int RT, int NK>
cudaError_t launch_rt_nk(const Params& p, const SeqSegs& sgs, size_t smem, cudaStream_t stream) {
  const int nsg = sgs.mode == 1 ? sgs.nseg - 1 : sgs.nseg;
  const dim3 grid((unsigned)(p.b * p.H * nsg));
  if (p.dtype == M3_BF16) {
    auto k = scan_seq_kernel<RT, NK, true>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<grid, kThreads, smem, stream>>>(p, sgs);
  } else {
    auto k = scan_seq_kernel<RT, NK, false>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<grid, kThreads, smem, stream>>>(p, sgs);
  }
  return cudaGetLastError();
}

template <int RT>
cudaError_t launch_rt(const Params& p, const SeqSegs& sgs, int nk, size_t smem, cudaStream_t stream) {
  switch (nk) {
    case 1: return launch_rt_nk<RT, 1>(p, sgs, smem, stream);
    case 2: return launch_rt_nk<RT, 2>(p, sgs, smem, stream);
    case 4: return launch_rt_nk<RT, 4>(p, sgs, smem, stream);
    case 8: return launch_rt_nk<RT, 8>(p, sgs, smem, stream);
    default: return launch_rt_nk<RT, 16>(p, sgs, smem, stream);
  }
}

cudaError_t launch_seq(const Params& p, const SeqSegs& sgs, cudaStream_t stream) {
  const SeqShape sh = seq_shape(p.P, p.N);
  int nk = (sh.K + sh.KG - 1) / sh.KG;
  int nk2 = 1;
  while (nk2 < nk) nk2 *= 2;
  const size_t smem = sizeof(float) * (size_t)seq_smem(p.P, p.N, p.R, sh.KG).total;
  if (p.R <= 1) return launch_rt<1>(p, sgs, nk2, smem, stream);
  if (p.R <= 2) return launch_rt<2>(p, sgs, nk2, smem, stream);
  if (p.R <= 4) return launch_rt<4>(p, sgs, nk2, smem, stream);
  return launch_rt<8>(p, sgs, nk2, smem, stream);
}

// Segments per sequence for the chunk-parallel form: enough blocks for two per SM, at least 32
// tokens per segment, at most 64 segments, and a workspace (entering states and summaries) of
// at most 12 MiB; 1 means the plain token-sequential walk.
constexpr size_t kSeqWsCap = size_t(12) << 20;
int seq_segments(const Params& p, int64_t* seg_len) {
  int dev = 0, nsm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int64_t nbh = p.b * p.H;
  int64_t s = nbh > 0 ? (2 * (int64_t)nsm + nbh - 1) / nbh : 1;
  if (s > p.L / 32) s = p.L / 32;
  if (s > 64) s = 64;
  const size_t per = 2 * (size_t)nbh * p.N * p.P * 4 + (size_t)nbh * (4 + 8 * (p.N / 2));
  while (s > 1 && per * (size_t)s > kSeqWsCap) --s;
  if (s < 2) {
    *seg_len = p.L;
    return 1;
  }
  *seg_len = (p.L + s - 1) / s;
  return (int)((p.L + *seg_len - 1) / *seg_len);
}

struct SeqWs {
  size_t h_in, z, ld, ang, total;
};
SeqWs seq_ws(const Params& p, int nseg) {
  const size_t nbh = (size_t)(p.b * p.H), np = (size_t)p.N * p.P;
  SeqWs w{};
  w.h_in = 0;
  w.z = (4 * nbh * nseg * np + 255) & ~(size_t)255;
  w.ld = w.z + ((4 * nbh * (nseg - 1) * np + 255) & ~(size_t)255);
  w.ang = w.ld + ((4 * nbh * (nseg - 1) + 255) & ~(size_t)255);
  w.total = w.ang + 8 * nbh * (nseg - 1) * (p.N / 2);
  return w;
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
  SeqSegs one{};
  one.nseg = 1;
  one.mode = 0;
  one.seg_len = p.L;
  return launch_seq(p, one, stream);
}

size_t seq_scan_workspace_bytes(const Params& p) {
  int64_t len = 0;
  const int nseg = seq_segments(p, &len);
  return nseg > 1 ? seq_ws(p, nseg).total : 0;
}

cudaError_t launch_scan_seq_chunked(const Params& p, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (p.b * p.H == 0) return cudaSuccess;
  int64_t len = 0;
  const int nseg = seq_segments(p, &len);
  if (nseg < 2) return launch_scan_sequential(p, stream);
  const SeqWs w = seq_ws(p, nseg);
  if (ws == nullptr || ws_bytes < w.total) return cudaErrorInvalidValue;
  char* b = static_cast<char*>(ws);
  SeqSegs sg{};
  sg.nseg = nseg;
  sg.seg_len = len;
  sg.h_in = reinterpret_cast<float*>(b + w.h_in);
  sg.Z = reinterpret_cast<float*>(b + w.z);
  sg.logdec = reinterpret_cast<float*>(b + w.ld);
  sg.angle = reinterpret_cast<double*>(b + w.ang);
  sg.mode = 1;
  cudaError_t e = launch_seq(p, sg, stream);
  if (e != cudaSuccess) return e;
  if (p.dtype == M3_BF16) seq_fold_kernel<true><<<(unsigned)(p.b * p.H), kThreads, 0, stream>>>(p, sg);
  else seq_fold_kernel<false><<<(unsigned)(p.b * p.H), kThreads, 0, stream>>>(p, sg);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  sg.mode = 0;
  return launch_seq(p, sg, stream);
}

}  // namespace m3
