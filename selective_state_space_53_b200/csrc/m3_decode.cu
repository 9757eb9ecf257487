// m3_decode.cu -- one-token decode update of the Mamba-3 SSM core (m3_decode_step).
//
// Decode reads and rewrites the whole fixed-size state every token (Mamba-3 paper note,
// docsaid.org, section その3: the step is memory-bound; MIMO rank R adds arithmetic per
// state byte).  One CTA per (batch, head):
//   * the fp32 state tile (N x P) is brought into shared memory by one bulk copy on the
//     TMA engine (cp.async.bulk, completion counted in bytes on an mbarrier), so no
//     registers hold loads in flight and two CTAs fit per SM;
//   * meanwhile the threads stage the token operands: biased B and C rows, the MIMO
//     branches X_r = W_x[r] * x_t and X'_r = W_x[r] * x_{t-1}, the rotation table;
//   * each thread then updates a 4-column quad of rotation pairs (2k, 2k+1),
//         h <- e^{dt A} Rot(dt theta) (h + (1 - lam) dt u_{t-1}) + lam dt u_t,
//     u = sum_r Bb_r X_r^T (section その1 trapezoid rule, section その2 rotation),
//     writes it straight back to HBM with 128-bit stores and accumulates the R readouts
//     Cb_r^T h, which are reduced over N through shared memory.
// The wait on the bulk copy is bounded by %globaltimer; a timeout sets M3_ERR_TIMEOUT.
#include "m3_common.cuh"

namespace m3 {
namespace {

constexpr int kThreads = 256;
constexpr unsigned long long kWaitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

struct DecShape {
  int PQ, KG, K;
};
__host__ __device__ inline DecShape dec_shape(int P, int N) {
  DecShape s;
  s.PQ = P / 4;
  s.K = N / 2;
  const int kg = kThreads / s.PQ;
  s.KG = kg < s.K ? kg : s.K;
  return s;
}

// shared-memory plan in floats; the state tile comes first (16-byte aligned for the copy)
struct DecSmem {
  int st, bb0, bb1, cb, x0, x1, cs, coef, red, mbar, total;
};
__host__ __device__ inline DecSmem dec_smem(int P, int N, int R, int KG) {
  DecSmem m;
  int o = 0;
  m.st = o;  o += N * P;
  m.bb0 = o; o += R * N;   // biased B of this token
  m.bb1 = o; o += R * N;   // biased B of the previous token (carry)
  m.cb = o;  o += R * N;
  m.x0 = o;  o += R * P;   // W_x * x_t
  m.x1 = o;  o += R * P;   // W_x * x_{t-1}
  m.cs = o;  o += N;       // (cos, sin) per pair
  m.coef = o; o += 4;
  o = (o + 3) & ~3;
  m.red = o; o += KG * R * P;
  o = (o + 3) & ~3;
  m.mbar = o; o += 4;
  m.total = o;
  return m;
}

template <int RT, bool BF16>
__global__ void __launch_bounds__(kThreads, 2) decode_kernel(Params p) {
  extern __shared__ __align__(16) float sm[];
  const int tid = threadIdx.x;
  const int H = p.H, P = p.P, N = p.N, R = p.R, G = p.G;
  const int bh = blockIdx.x;
  const int bi = bh / H, hi = bh % H;
  const int g = hi / (H / G);
  const DecShape sh = dec_shape(P, N);
  const DecSmem ms = dec_smem(P, N, R, sh.KG);
  float* st = sm + ms.st;
  float* bbc = sm + ms.bb0;
  float* bbp = sm + ms.bb1;
  float* cb = sm + ms.cb;
  float* xc = sm + ms.x0;
  float* xp = sm + ms.x1;
  float2* cs = reinterpret_cast<float2*>(sm + ms.cs);
  float* coef = sm + ms.coef;
  float* red = sm + ms.red;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + ms.mbar);

  float* hg = p.h + (int64_t)bh * N * P;
  float* cBg = p.carry_B + (int64_t)bh * R * N;
  float* cxg = p.carry_x + (int64_t)bh * P;
  const float* biasB = p.bias_B ? p.bias_B + (int64_t)hi * R * N : nullptr;
  const float* biasC = p.bias_C ? p.bias_C + (int64_t)hi * R * N : nullptr;
  const float* Wx = p.W_x ? p.W_x + (int64_t)hi * R * P : nullptr;
  const float* Wo = p.W_o ? p.W_o + (int64_t)hi * R * P : nullptr;

  // ---- state tile: one bulk copy HBM -> shared memory
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(bar)));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    const uint32_t bytes = (uint32_t)(N * P * 4);
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(st)),
        "l"(hg), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
  }

  // ---- token operands
  {
    const int64_t tok = bi;  // one token per sequence
    const int64_t bcoff = ((tok * G + g) * R) * (int64_t)N;
    for (int i = tid; i < R * N; i += kThreads) {
      const float bb = biasB ? biasB[i] : 0.0f;
      bbc[i] = load_in<BF16>(p.B, bcoff + i) + bb;
      bbp[i] = cBg[i] + bb;
      cb[i] = load_in<BF16>(p.C, bcoff + i) + (biasC ? biasC[i] : 0.0f);
    }
    const int64_t xoff = (tok * H + hi) * (int64_t)P;
    for (int i = tid; i < R * P; i += kThreads) {
      const float w = Wx ? Wx[i] : 1.0f;
      xc[i] = load_in<BF16>(p.x, xoff + (i % P)) * w;
      xp[i] = cxg[i % P] * w;
    }
    const float delta = p.dt[tok * H + hi];
    const float* th = p.theta + (tok * G + g) * (int64_t)(N / 2);
    for (int k = tid; k < N / 2; k += kThreads) {
      float s, c;
      sincosf(delta * th[k], &s, &c);
      cs[k] = make_float2(c, s);
    }
    if (tid == 0) {
      const float lm = p.lam[tok * H + hi];
      coef[0] = expf(delta * p.A[tok * H + hi]);
      coef[1] = (1.0f - lm) * delta;
      coef[2] = lm * delta;
    }
  }
  __syncthreads();
  // ---- wait for the state tile (bounded)
  {
    uint32_t done = 0;
    const uint64_t t0 = globaltimer();
    while (true) {
      asm volatile(
          "{\n .reg .pred q;\n mbarrier.try_wait.parity.shared::cta.b64 q, [%1], 0;\n selp.u32 %0, 1, 0, q;\n}\n"
          : "=r"(done)
          : "r"(smem_u32(bar))
          : "memory");
      if (done || globaltimer() - t0 > kWaitNs) break;
    }
    if (__syncthreads_or(!done)) {
      if (tid == 0) set_status(p.status, M3_ERR_TIMEOUT);
      return;
    }
  }

  const int pq = tid % sh.PQ;
  const int kg = tid / sh.PQ;
  const int p0 = 4 * pq;
  if (kg < sh.KG) {
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
#pragma unroll 2
    for (int k = kg; k < sh.K; k += sh.KG) {
      const float4 s0 = *reinterpret_cast<const float4*>(st + (2 * k) * P + p0);
      const float4 s1 = *reinterpret_cast<const float4*>(st + (2 * k + 1) * P + p0);
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
      const float ac = alpha * rc.x, as = alpha * rc.y;
      const float a0[4] = {s0.x, s0.y, s0.z, s0.w};
      const float a1[4] = {s1.x, s1.y, s1.z, s1.w};
      float n0[4], n1[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float v0 = fmaf(bp, q0[e], a0[e]);
        const float v1 = fmaf(bp, q1[e], a1[e]);
        n0[e] = fmaf(ac, v0, fmaf(-as, v1, gm * u0[e]));
        n1[e] = fmaf(as, v0, fmaf(ac, v1, gm * u1[e]));
      }
      *reinterpret_cast<float4*>(hg + (int64_t)(2 * k) * P + p0) = make_float4(n0[0], n0[1], n0[2], n0[3]);
      *reinterpret_cast<float4*>(hg + (int64_t)(2 * k + 1) * P + p0) = make_float4(n1[0], n1[1], n1[2], n1[3]);
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        if (r < R) {
          const float2 cc = *reinterpret_cast<const float2*>(cb + r * N + 2 * k);
#pragma unroll
          for (int e = 0; e < 4; ++e) Y[r][e] = fmaf(cc.x, n0[e], fmaf(cc.y, n1[e], Y[r][e]));
        }
      }
    }
#pragma unroll
    for (int r = 0; r < RT; ++r)
      if (r < R)
        *reinterpret_cast<float4*>(red + (kg * R + r) * P + p0) = make_float4(Y[r][0], Y[r][1], Y[r][2], Y[r][3]);
  }
  __syncthreads();
  // ---- y = sum_r W_o[r] * (sum over pair groups) + D x; new carry = this token's raw B, x
  {
    const int64_t xoff = ((int64_t)bi * H + hi) * P;
    const float Dh = p.D ? p.D[hi] : 0.0f;
    for (int pp = tid; pp < P; pp += kThreads) {
      float acc = 0.0f;
      for (int r = 0; r < R; ++r) {
        float s = 0.0f;
        for (int q = 0; q < sh.KG; ++q) s += red[(q * R + r) * P + pp];
        acc = fmaf(Wo ? Wo[r * P + pp] : 1.0f, s, acc);
      }
      const float xv = load_in<BF16>(p.x, xoff + pp);
      store_out<BF16>(p.y, xoff + pp, fmaf(Dh, xv, acc));
      cxg[pp] = xv;
    }
    const int64_t bcoff = (((int64_t)bi * G + g) * R) * (int64_t)N;
    for (int i = tid; i < R * N; i += kThreads) cBg[i] = load_in<BF16>(p.B, bcoff + i);
  }
}

template <int RT>
cudaError_t launch_rt(const Params& p, size_t smem, cudaStream_t stream) {
  const unsigned grid = (unsigned)(p.b * p.H);
  if (p.dtype == M3_BF16) {
    auto k = decode_kernel<RT, true>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<grid, kThreads, smem, stream>>>(p);
  } else {
    auto k = decode_kernel<RT, false>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<grid, kThreads, smem, stream>>>(p);
  }
  return cudaGetLastError();
}

size_t decode_smem_bytes(int P, int N, int R) {
  const DecShape sh = dec_shape(P, N);
  return sizeof(float) * (size_t)dec_smem(P, N, R, sh.KG).total;
}

}  // namespace

bool decode_supported(const Params& p) {
  return decode_smem_bytes(p.P, p.N, p.R) <= 200 * 1024;
}

cudaError_t launch_decode(const Params& p, cudaStream_t stream) {
  if (p.b * p.H == 0) return cudaSuccess;
  const size_t smem = decode_smem_bytes(p.P, p.N, p.R);
  if (p.R <= 1) return launch_rt<1>(p, smem, stream);
  if (p.R <= 2) return launch_rt<2>(p, smem, stream);
  if (p.R <= 4) return launch_rt<4>(p, smem, stream);
  return launch_rt<8>(p, smem, stream);
}

}  // namespace m3
