// m3_scan_bwd.cu -- backward pass of the Mamba-3 SSM core (m3_scan_bwd): the gradients of
// sum(dy * y) + sum(dh_final * h_final) with respect to every operand and the initial state.
//
// The forward step (Mamba-3 paper note, docsaid.org: section その1 for the trapezoid rule,
// section その2 for the rotation of state pairs, section その3 for the MIMO branches) is
//   y_t = sum_r W_o_r * (Cb_{t,r}^T h_t) + D x_t
//   h_t = alpha_t Rot(phi_t) z_t + gamma_t u_t,   z_t = h_{t-1} + beta'_t u_{t-1}
//   u_t = sum_r Bb_{t,r} X_{t,r}^T,  X_{t,r} = W_x_r * x_t,  Bb = B + bias_B, Cb = C + bias_C,
// and its reverse step, for g = dL/dh_t, is
//   dalpha = <g, Rot z>, dgamma = <g, u_t>, du_t = gamma g + beta'_{t+1} dz_{t+1},
//   dz = Rot^T (alpha g), dphi_k = <alpha g, dRot/dphi_k z>, dbeta' = <dz, u_{t-1}>,
//   dL/dh_{t-1} = dz,
// followed by the readout's and u_t's chain rules and the scalar chains of alpha, beta',
// gamma and phi through dt, A, lam and theta.
//
// One CTA per (batch, head) walks the tokens backwards (or 2 or 4 CTAs, each owning a slice of
// the columns p, when that fills more SMs: the columns evolve independently).  The fp32
// gradient g and u_t's share from the next token live in registers (a thread owns one column p
// and the rotation pairs k = grp, grp + KG, ...), the forward states come from a checkpointed
// recomputation: a first
// sweep stores the state before every K-th token in the workspace, and each block of K tokens
// is recomputed into the workspace before it is walked backwards (K about sqrt(L)).  Sums over
// the columns or rows of a token (the readout's and u_t's gradients, the rotation angles' and
// the scalars') are reduced with shared-memory atomics.  Gradients of operands shared by the
// heads of a group (B, C, theta) or by the batch (biases, W_x, W_o, D), and the sums over
// columns when several CTAs share a (batch, head), are added into global memory with atomics,
// after a first kernel has zeroed them.
#include "m3_common.cuh"

namespace m3 {
namespace {

constexpr int kBwdThreads = 512;

struct BwdArgs {
  const void* dy;        // (b, L, H, P), dtype of x
  const float* dh_final; // (b, H, N, P) or null
  void* dx;              // (b, L, H, P), dtype of x
  float *ddt, *dA, *dlam;          // (b, L, H)
  void *dB, *dC;                   // (b, L, G, R, N), dtype of x; fp32 accumulation buffers below
  float* dtheta;                   // (b, L, G, N/2)
  float *dbias_B, *dbias_C;        // (H, R, N) or null
  float *dW_x, *dW_o;              // (H, R, P) or null
  float* dD;                       // (H) or null
  float *dh0, *dcarry_B, *dcarry_x;  // (b, H, N, P), (b, H, R, N), (b, H, P)
  float *accB, *accC;              // fp32 (b, L, G, R, N) accumulators of dB, dC
  float* ckpt;                     // (b*H, nck + K, N, P) workspace of forward states
  int K;                           // tokens per recomputed block
  int nck;                         // blocks = ceil(L / K)
  int cs;                          // CTAs per (batch, head), each owning P / cs columns
};

struct BwdShape {
  int KG;   // pair groups (threads per column)
  int NK;   // pairs per thread
};

__host__ __device__ inline BwdShape bwd_shape(int P, int N) {
  BwdShape s;
  s.KG = kBwdThreads / P;
  if (s.KG > N / 2) s.KG = N / 2;
  s.NK = (N / 2 + s.KG - 1) / s.KG;
  return s;
}

// shared-memory plan (floats)
struct BwdSmem {
  int bb, bbp, cb, x, xp, xt, dyr, cs, red_cb, red_bb, red_x, red_y, red_phi, red_s, acc_bB, acc_bC, acc_wx,
      acc_wo, total;
};
__host__ __device__ inline BwdSmem bwd_smem(int P, int N, int R) {
  BwdSmem m;
  int o = 0;
  m.bb = o; o += R * N;
  m.bbp = o; o += R * N;
  m.cb = o; o += R * N;
  m.x = o; o += R * P;
  m.xp = o; o += R * P;
  m.xt = o; o += 2 * P;           // x_t and dy_t
  m.dyr = o; o += R * P;          // W_o_r * dy_t
  m.cs = o; o += N;               // (cos, sin) per pair
  m.red_cb = o; o += R * N;
  m.red_bb = o; o += R * N;
  m.red_x = o; o += R * P;
  m.red_y = o; o += R * P;
  m.red_phi = o; o += N / 2;
  m.red_s = o; o += 8;            // dalpha, dgamma, dbeta', sum dy x
  m.acc_bB = o; o += R * N;
  m.acc_bC = o; o += R * N;
  m.acc_wx = o; o += R * P;
  m.acc_wo = o; o += R * P;
  m.total = o;
  return m;
}

template <typename T>
__device__ __forceinline__ float ld(const void* base, int64_t i) {
  if constexpr (sizeof(T) == 2) return __bfloat162float(static_cast<const __nv_bfloat16*>(base)[i]);
  else return static_cast<const float*>(base)[i];
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Sums each of NV values (a power of two, 2..16) over the 32 lanes of a warp in a transposed
// butterfly: log2 NV steps each keep half of the values and add the partner lane's copy of them
// (offsets 16, 8, ...), then the lanes that hold the same value add theirs.  Lane l returns the
// total of value l / (32 / NV).
template <int NV>
__device__ __forceinline__ float warp_sum_n(float (&v)[NV], int lane) {
  int off = 16;
#pragma unroll
  for (int s = NV / 2; s >= 1; s >>= 1, off >>= 1) {
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const float give = up ? v[i] : v[i + s];
      const float keep = up ? v[i + s] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, give, off);
    }
  }
  float t = v[0];
#pragma unroll
  for (; off >= 1; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
  return t;
}

// The terms of one rotation pair (2 values per branch r < R <= RT: rows n0, n1) summed over the
// columns p into red[r N + n]: a warp butterfly when every lane of the warp holds this pair
// (wide), element atomics otherwise.
template <int RT>
__device__ __forceinline__ void pair_reduce(float (&v)[2 * RT], bool wide, int lane, int R, int N, int n0, int n1,
                                            float* red) {
  if (wide) {
    constexpr int span = 32 / (2 * RT);  // lanes that end with the same value
    const float tot = warp_sum_n<2 * RT>(v, lane);
    const int vi = lane / span, r = vi >> 1;
    if (lane % span == 0 && r < R) atomicAdd(&red[r * N + ((vi & 1) ? n1 : n0)], tot);
  } else {
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      if (r < R) {
        atomicAdd(&red[r * N + n0], v[2 * r]);
        atomicAdd(&red[r * N + n1], v[2 * r + 1]);
      }
    }
  }
}

// zero the fp32 gradient buffers that several CTAs add into
__global__ void bwd_zero_kernel(float* a, int64_t na, float* b, int64_t nb, float* c, int64_t nc, float* d,
                                int64_t nd, float* e, int64_t ne) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;; i += stride) {
    bool any = false;
    if (a && i < na) { a[i] = 0.0f; any = true; }
    if (b && i < nb) { b[i] = 0.0f; any = true; }
    if (c && i < nc) { c[i] = 0.0f; any = true; }
    if (d && i < nd) { d[i] = 0.0f; any = true; }
    if (e && i < ne) { e[i] = 0.0f; any = true; }
    if (!any && i >= na && i >= nb && i >= nc && i >= nd && i >= ne) break;
  }
}

// convert the fp32 accumulators of dB, dC to the storage type
template <typename T>
__global__ void bwd_store_kernel(const float* accB, const float* accC, void* dB, void* dC, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    if constexpr (sizeof(T) == 2) {
      static_cast<__nv_bfloat16*>(dB)[i] = __float2bfloat16_rn(accB[i]);
      static_cast<__nv_bfloat16*>(dC)[i] = __float2bfloat16_rn(accC[i]);
    } else {
      static_cast<float*>(dB)[i] = accB[i];
      static_cast<float*>(dC)[i] = accC[i];
    }
  }
}

template <typename T, int NK, int RT>
__global__ void __launch_bounds__(kBwdThreads) scan_bwd_kernel(const Params p, const BwdArgs q) {
  extern __shared__ __align__(16) float sm[];
  const int tid = threadIdx.x;
  const int H = p.H, P = p.P, N = p.N, R = p.R, G = p.G, K2 = N / 2;
  const int64_t L = p.L;
  // the columns of a state evolve independently (the rotation mixes rows): cs CTAs share a
  // (batch, head), CTA c owning columns c0 .. c0 + PL - 1; sums over columns are added up
  // across them with the global atomics that already sum over heads or the batch
  const int bh = blockIdx.x / q.cs, bi = bh / H, hi = bh % H, g = hi / (H / G);
  const int PL = P / q.cs, c0 = (blockIdx.x % q.cs) * PL;
  const BwdShape sh = bwd_shape(PL, N);
  const BwdSmem ms = bwd_smem(P, N, R);
  const int pc = c0 + tid % PL, grp = tid / PL;
  const bool active = grp < sh.KG;
  const bool wide = PL % 32 == 0;  // a warp's lanes are columns of one pair group
  float* const Bb = sm + ms.bb;
  float* const Bbp = sm + ms.bbp;
  float* const Cb = sm + ms.cb;
  float* const X = sm + ms.x;
  float* const Xp = sm + ms.xp;
  float* const xt = sm + ms.xt;
  float* const dyt = sm + ms.xt + P;
  float* const dYr = sm + ms.dyr;
  float2* const cs = reinterpret_cast<float2*>(sm + ms.cs);
  float* const red_cb = sm + ms.red_cb;
  float* const red_bb = sm + ms.red_bb;
  float* const red_x = sm + ms.red_x;
  float* const red_y = sm + ms.red_y;
  float* const red_phi = sm + ms.red_phi;
  float* const red_s = sm + ms.red_s;
  float* const acc_bB = sm + ms.acc_bB;
  float* const acc_bC = sm + ms.acc_bC;
  float* const acc_wx = sm + ms.acc_wx;
  float* const acc_wo = sm + ms.acc_wo;
  const float* biasB = p.bias_B ? p.bias_B + (int64_t)hi * R * N : nullptr;
  const float* biasC = p.bias_C ? p.bias_C + (int64_t)hi * R * N : nullptr;
  const float* Wx = p.W_x ? p.W_x + (int64_t)hi * R * P : nullptr;
  const float* Wo = p.W_o ? p.W_o + (int64_t)hi * R * P : nullptr;
  const float Dh = p.D ? p.D[hi] : 0.0f;
  const int64_t NP = (int64_t)N * P;
  float* ck = q.ckpt + (int64_t)bh * (q.nck + q.K) * NP;  // [nck] checkpoints, then [K] block states
  float* blk = ck + (int64_t)q.nck * NP;
  const float* cB0 = p.carry_B + (int64_t)bh * R * N;
  const float* cx0 = p.carry_x + (int64_t)bh * P;

  for (int i = tid; i < R * N; i += kBwdThreads) acc_bB[i] = acc_bC[i] = 0.0f;
  for (int i = tid; i < R * P; i += kBwdThreads) acc_wx[i] = acc_wo[i] = 0.0f;
  float accD = 0.0f;

  // stage token t's operands: Bb, Cb, X of t and Bbp, Xp of t - 1 (the carry at t = 0), its
  // coefficients and rotation table; returns (alpha, beta', gamma, dt, A, lam) through `co`
  auto stage = [&](int64_t t, float* co) {
    const int64_t tok = (int64_t)bi * L + t;
    const int64_t bco = ((tok * G + g) * R) * (int64_t)N;
    for (int i = tid; i < R * N; i += kBwdThreads) {
      const float bb = biasB ? biasB[i] : 0.0f;
      Bb[i] = ld<T>(p.B, bco + i) + bb;
      Cb[i] = ld<T>(p.C, bco + i) + (biasC ? biasC[i] : 0.0f);
      Bbp[i] = (t > 0 ? ld<T>(p.B, bco - (int64_t)G * R * N + i) : cB0[i]) + bb;
    }
    const int64_t xo = (tok * H + hi) * (int64_t)P;
    for (int i = tid; i < R * P; i += kBwdThreads) {
      const float w = Wx ? Wx[i] : 1.0f;
      X[i] = w * ld<T>(p.x, xo + i % P);
      Xp[i] = w * (t > 0 ? ld<T>(p.x, xo - (int64_t)H * P + i % P) : cx0[i % P]);
    }
    const float delta = p.dt[tok * H + hi], a = p.A[tok * H + hi], lm = p.lam[tok * H + hi];
    const float* th = p.theta + (tok * G + g) * (int64_t)K2;
    for (int k = tid; k < K2; k += kBwdThreads) {
      float sn, cn;
      sincosf(p.angle_direct ? th[k] : delta * th[k], &sn, &cn);
      cs[k] = make_float2(cn, sn);
    }
    co[0] = __expf(delta * a);
    co[1] = (1.0f - lm) * delta;
    co[2] = lm * delta;
    co[3] = delta;
    co[4] = a;
    co[5] = lm;
  };
  // one forward step of the owned elements: h <- alpha Rot (h + beta' u_{t-1}) + gamma u_t
  auto fwd_step = [&](float (&h0)[NK], float (&h1)[NK], const float* co) {
#pragma unroll
    for (int j = 0; j < NK; ++j) {
      const int k = grp + j * sh.KG;
      if (!active || k >= K2) continue;
      float u0 = 0.f, u1 = 0.f, q0 = 0.f, q1 = 0.f;
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        if (r < R) {
          const float2 b2 = *reinterpret_cast<const float2*>(Bb + r * N + 2 * k);
          const float2 bp2 = *reinterpret_cast<const float2*>(Bbp + r * N + 2 * k);
          const float xr = X[r * P + pc], xpr = Xp[r * P + pc];
          u0 = fmaf(b2.x, xr, u0);
          u1 = fmaf(b2.y, xr, u1);
          q0 = fmaf(bp2.x, xpr, q0);
          q1 = fmaf(bp2.y, xpr, q1);
        }
      }
      const float z0 = fmaf(co[1], q0, h0[j]), z1 = fmaf(co[1], q1, h1[j]);
      const float2 c = cs[k];
      h0[j] = fmaf(co[0], c.x * z0 - c.y * z1, co[2] * u0);
      h1[j] = fmaf(co[0], c.y * z0 + c.x * z1, co[2] * u1);
    }
  };
  auto store_state = [&](float* dst, const float (&h0)[NK], const float (&h1)[NK]) {
#pragma unroll
    for (int j = 0; j < NK; ++j) {
      const int k = grp + j * sh.KG;
      if (active && k < K2) {
        dst[(int64_t)(2 * k) * P + pc] = h0[j];
        dst[(int64_t)(2 * k + 1) * P + pc] = h1[j];
      }
    }
  };
  auto load_state = [&](const float* src, float (&h0)[NK], float (&h1)[NK]) {
#pragma unroll
    for (int j = 0; j < NK; ++j) {
      const int k = grp + j * sh.KG;
      h0[j] = h1[j] = 0.0f;
      if (active && k < K2) {
        h0[j] = src[(int64_t)(2 * k) * P + pc];
        h1[j] = src[(int64_t)(2 * k + 1) * P + pc];
      }
    }
  };

  // ---- sweep 1: checkpoints of the state before every block of K tokens
  float h0[NK], h1[NK];
  load_state(p.h + (int64_t)bh * NP, h0, h1);
  float co[6];
  for (int64_t t = 0; t < L; ++t) {
    if (t % q.K == 0) store_state(ck + (t / q.K) * NP, h0, h1);
    __syncthreads();
    stage(t, co);
    __syncthreads();
    fwd_step(h0, h1, co);
  }

  // ---- sweep 2: blocks backwards; g = dL/dh_t, dn = u_t's share from token t + 1
  float gr0[NK], gr1[NK], dn0[NK], dn1[NK];
#pragma unroll
  for (int j = 0; j < NK; ++j) {
    const int k = grp + j * sh.KG;
    gr0[j] = gr1[j] = dn0[j] = dn1[j] = 0.0f;
    if (q.dh_final && active && k < K2) {
      gr0[j] = q.dh_final[(int64_t)bh * NP + (int64_t)(2 * k) * P + pc];
      gr1[j] = q.dh_final[(int64_t)bh * NP + (int64_t)(2 * k + 1) * P + pc];
    }
  }
  for (int64_t c = q.nck - 1; c >= 0; --c) {
    const int64_t t0 = c * q.K;
    const int64_t t1 = (t0 + q.K < L) ? t0 + q.K : L;
    // recompute the block's states h_t (t0 <= t < t1) into blk[t - t0]
    load_state(ck + c * NP, h0, h1);
    for (int64_t t = t0; t < t1; ++t) {
      __syncthreads();
      stage(t, co);
      __syncthreads();
      fwd_step(h0, h1, co);
      store_state(blk + (t - t0) * NP, h0, h1);
    }
    for (int64_t t = t1 - 1; t >= t0; --t) {
      __syncthreads();  // the previous token's reductions have been consumed
      stage(t, co);
      const int64_t tok = (int64_t)bi * L + t;
      const int64_t xo = (tok * H + hi) * (int64_t)P;
      for (int i = tid; i < P; i += kBwdThreads) {
        xt[i] = ld<T>(p.x, xo + i);
        dyt[i] = ld<T>(q.dy, xo + i);
      }
      for (int i = tid; i < R * N; i += kBwdThreads) red_cb[i] = red_bb[i] = 0.0f;
      for (int i = tid; i < R * P; i += kBwdThreads) red_x[i] = red_y[i] = 0.0f;
      for (int i = tid; i < K2; i += kBwdThreads) red_phi[i] = 0.0f;
      if (tid < 8) red_s[tid] = 0.0f;
      __syncthreads();
      for (int i = tid; i < R * P; i += kBwdThreads) dYr[i] = (Wo ? Wo[i] : 1.0f) * dyt[i % P];
      __syncthreads();
      const float* ht = blk + (t - t0) * NP;
      const float* hp = t > t0 ? blk + (t - t0 - 1) * NP : ck + c * NP;
      const float alpha = co[0], bprime = co[1], gamma = co[2];
      float s_alpha = 0.f, s_gamma = 0.f, s_bp = 0.f;
      float px[RT], py[RT];  // partial dX and Y of this thread's column, per branch (R <= RT)
#pragma unroll
      for (int r = 0; r < RT; ++r) px[r] = py[r] = 0.0f;
#pragma unroll
      for (int j = 0; j < NK; ++j) {
        const int k = grp + j * sh.KG;
        if (!active || k >= K2) continue;
        const int n0 = 2 * k, n1 = 2 * k + 1;
        const float ht0 = ht[(int64_t)n0 * P + pc], ht1 = ht[(int64_t)n1 * P + pc];
        const float hp0 = hp[(int64_t)n0 * P + pc], hp1 = hp[(int64_t)n1 * P + pc];
        // readout: g += sum_r Cb_r dY_r^T; dCb_r += h_t dY_r (summed over the warp's columns
        // below); Y_r partial.  sv holds the pair's column terms: dCb (r, n0), (r, n1), then dBb
        float g0 = gr0[j], g1 = gr1[j];
        float sv[2 * RT];
#pragma unroll
        for (int r = 0; r < RT; ++r) {
          sv[2 * r] = sv[2 * r + 1] = 0.0f;
          if (r < R) {
            const float dy_r = dYr[r * P + pc];
            const float2 c2 = *reinterpret_cast<const float2*>(Cb + r * N + n0);
            g0 = fmaf(c2.x, dy_r, g0);
            g1 = fmaf(c2.y, dy_r, g1);
            sv[2 * r] = ht0 * dy_r;
            sv[2 * r + 1] = ht1 * dy_r;
            py[r] = fmaf(c2.x, ht0, fmaf(c2.y, ht1, py[r]));
          }
        }
        pair_reduce<RT>(sv, wide, tid & 31, R, N, n0, n1, red_cb);
        // step
        float u0 = 0.f, u1 = 0.f, q0 = 0.f, q1 = 0.f;
        float2 bbr[RT];  // Bb rows n0, n1 of each branch (reused by u_t's gradient below)
#pragma unroll
        for (int r = 0; r < RT; ++r) {
          bbr[r] = make_float2(0.f, 0.f);
          if (r < R) {
            bbr[r] = *reinterpret_cast<const float2*>(Bb + r * N + n0);
            const float2 bp2 = *reinterpret_cast<const float2*>(Bbp + r * N + n0);
            const float xr = X[r * P + pc], xpr = Xp[r * P + pc];
            u0 = fmaf(bbr[r].x, xr, u0);
            u1 = fmaf(bbr[r].y, xr, u1);
            q0 = fmaf(bp2.x, xpr, q0);
            q1 = fmaf(bp2.y, xpr, q1);
          }
        }
        const float z0 = fmaf(bprime, q0, hp0), z1 = fmaf(bprime, q1, hp1);
        const float2 cc = cs[k];
        const float m0 = cc.x * z0 - cc.y * z1, m1 = cc.y * z0 + cc.x * z1;
        s_alpha = fmaf(g0, m0, fmaf(g1, m1, s_alpha));
        s_gamma = fmaf(g0, u0, fmaf(g1, u1, s_gamma));
        const float du0 = fmaf(gamma, g0, dn0[j]), du1 = fmaf(gamma, g1, dn1[j]);
        const float dm0 = alpha * g0, dm1 = alpha * g1;
        const float dz0 = cc.x * dm0 + cc.y * dm1, dz1 = -cc.y * dm0 + cc.x * dm1;
        const float phi_t = dm0 * (-cc.y * z0 - cc.x * z1) + dm1 * (cc.x * z0 - cc.y * z1);
        if (wide) {
          const float ps = warp_sum(phi_t);
          if ((tid & 31) == 0) atomicAdd(&red_phi[k], ps);
        } else {
          atomicAdd(&red_phi[k], phi_t);
        }
        s_bp = fmaf(dz0, q0, fmaf(dz1, q1, s_bp));
        dn0[j] = bprime * dz0;
        dn1[j] = bprime * dz1;
        gr0[j] = dz0;
        gr1[j] = dz1;
        // u_t = sum_r Bb_r X_r^T
#pragma unroll
        for (int r = 0; r < RT; ++r) {
          sv[2 * r] = sv[2 * r + 1] = 0.0f;
          if (r < R) {
            const float xr = X[r * P + pc];
            sv[2 * r] = du0 * xr;
            sv[2 * r + 1] = du1 * xr;
            px[r] = fmaf(du0, bbr[r].x, fmaf(du1, bbr[r].y, px[r]));
          }
        }
        pair_reduce<RT>(sv, wide, tid & 31, R, N, n0, n1, red_bb);
      }
      if (active) {
#pragma unroll
        for (int r = 0; r < RT; ++r) {
          if (r < R) {
            atomicAdd(&red_x[r * P + pc], px[r]);
            atomicAdd(&red_y[r * P + pc], py[r]);
          }
        }
      }
      s_alpha = warp_sum(s_alpha);
      s_gamma = warp_sum(s_gamma);
      s_bp = warp_sum(s_bp);
      if ((tid & 31) == 0) {
        atomicAdd(&red_s[0], s_alpha);
        atomicAdd(&red_s[1], s_gamma);
        atomicAdd(&red_s[2], s_bp);
      }
      __syncthreads();
      // ---- gradients of token t
      for (int i = tid; i < R * N; i += kBwdThreads) {
        const int64_t o = ((tok * G + g) * R) * (int64_t)N + i;
        atomicAdd(&q.accC[o], red_cb[i]);
        atomicAdd(&q.accB[o], red_bb[i]);
        acc_bC[i] += red_cb[i];
        acc_bB[i] += red_bb[i];
      }
      for (int i = c0 + tid; i < c0 + PL; i += kBwdThreads) {
        float dxv = Dh * dyt[i];
        for (int r = 0; r < R; ++r) {
          dxv = fmaf(Wx ? Wx[r * P + i] : 1.0f, red_x[r * P + i], dxv);
          acc_wx[r * P + i] += red_x[r * P + i] * xt[i];
          acc_wo[r * P + i] += dyt[i] * red_y[r * P + i];
        }
        if constexpr (sizeof(T) == 2) static_cast<__nv_bfloat16*>(q.dx)[xo + i] = __float2bfloat16_rn(dxv);
        else static_cast<float*>(q.dx)[xo + i] = dxv;
        accD = fmaf(dyt[i], xt[i], accD);
      }
      const float delta = co[3], a = co[4], lm = co[5];
      const float* th = p.theta + (tok * G + g) * (int64_t)K2;
      float sdt = 0.0f;
      for (int k = tid; k < K2; k += kBwdThreads) {
        if (!p.angle_direct) sdt = fmaf(red_phi[k], th[k], sdt);
        atomicAdd(&q.dtheta[(tok * G + g) * (int64_t)K2 + k], red_phi[k] * (p.angle_direct ? 1.0f : delta));
      }
      sdt = warp_sum(sdt);
      if (K2 > 32) {  // more than one warp holds angle terms: gather them in red_s[4]
        if ((tid & 31) == 0 && tid < K2) atomicAdd(&red_s[4], sdt);
      }
      __syncthreads();
      if (tid == 0) {  // this CTA's columns' share (the scalars' gradients are linear in the sums)
        const float dth = K2 > 32 ? red_s[4] : sdt;
        const float da = red_s[0], dg = red_s[1], db = red_s[2];
        const float al = co[0];
        atomicAdd(&q.ddt[tok * H + hi], da * al * a + dg * lm + db * (1.0f - lm) + dth);
        atomicAdd(&q.dA[tok * H + hi], da * al * delta);
        atomicAdd(&q.dlam[tok * H + hi], (dg - db) * delta);
      }
    }
  }
  __syncthreads();
  // ---- the initial state: dh0 = g; the carry through u_{-1}
  store_state(q.dh0 + (int64_t)bh * NP, gr0, gr1);
  stage(0, co);  // Bbp, Xp = the carry's branches
  for (int i = tid; i < R * N; i += kBwdThreads) red_bb[i] = 0.0f;
  for (int i = tid; i < R * P; i += kBwdThreads) red_x[i] = 0.0f;
  __syncthreads();
  {
    float px[RT];
#pragma unroll
    for (int r = 0; r < RT; ++r) px[r] = 0.0f;
#pragma unroll
    for (int j = 0; j < NK; ++j) {
      const int k = grp + j * sh.KG;
      if (!active || k >= K2) continue;
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        if (r >= R) break;
        const float xr = Xp[r * P + pc];
        atomicAdd(&red_bb[r * N + 2 * k], dn0[j] * xr);
        atomicAdd(&red_bb[r * N + 2 * k + 1], dn1[j] * xr);
        px[r] = fmaf(dn0[j], Bbp[r * N + 2 * k], fmaf(dn1[j], Bbp[r * N + 2 * k + 1], px[r]));
      }
    }
    if (active) {
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        if (r >= R) break;
        atomicAdd(&red_x[r * P + pc], px[r]);
      }
    }
  }
  __syncthreads();
  for (int i = tid; i < R * N; i += kBwdThreads) {
    atomicAdd(&q.dcarry_B[(int64_t)bh * R * N + i], red_bb[i]);
    acc_bB[i] += red_bb[i];
  }
  for (int i = c0 + tid; i < c0 + PL; i += kBwdThreads) {
    float dcx = 0.0f;
    for (int r = 0; r < R; ++r) {
      dcx = fmaf(Wx ? Wx[r * P + i] : 1.0f, red_x[r * P + i], dcx);
      acc_wx[r * P + i] += red_x[r * P + i] * cx0[i];
    }
    q.dcarry_x[(int64_t)bh * P + i] = dcx;
  }
  // ---- per-head parameters, summed over the batch
  accD = warp_sum(accD);
  if ((tid & 31) == 0 && q.dD && tid < PL) atomicAdd(q.dD + hi, accD);
  __syncthreads();
  for (int i = tid; i < R * N; i += kBwdThreads) {
    if (q.dbias_B) atomicAdd(q.dbias_B + (int64_t)hi * R * N + i, acc_bB[i]);
    if (q.dbias_C) atomicAdd(q.dbias_C + (int64_t)hi * R * N + i, acc_bC[i]);
  }
  for (int i = tid; i < R * P; i += kBwdThreads) {
    if (q.dW_x) atomicAdd(q.dW_x + (int64_t)hi * R * P + i, acc_wx[i]);
    if (q.dW_o) atomicAdd(q.dW_o + (int64_t)hi * R * P + i, acc_wo[i]);
  }
}

template <typename T, int NK, int RT>
cudaError_t launch_bwd_nk(const Params& p, const BwdArgs& q, cudaStream_t stream) {
  const BwdSmem ms = bwd_smem(p.P, p.N, p.R);
  const size_t smem = sizeof(float) * (size_t)ms.total;
  auto k = scan_bwd_kernel<T, NK, RT>;
  if (smem > 48 * 1024) {
    static SmemAttr attr;
    cudaError_t e = attr.ensure(k, (int)smem);
    if (e != cudaSuccess) return e;
  }
  k<<<(unsigned)(p.b * p.H * q.cs), kBwdThreads, smem, stream>>>(p, q);
  return cudaGetLastError();
}

template <typename T, int RT>
cudaError_t launch_bwd_rt(const Params& p, const BwdArgs& q, cudaStream_t stream) {
  const int nk = bwd_shape(p.P / q.cs, p.N).NK;  // pairs per thread; the loops skip pairs past N/2
  if (nk <= 2) return launch_bwd_nk<T, 2, RT>(p, q, stream);
  if (nk <= 4) return launch_bwd_nk<T, 4, RT>(p, q, stream);
  if (nk <= 8) return launch_bwd_nk<T, 8, RT>(p, q, stream);
  return launch_bwd_nk<T, 16, RT>(p, q, stream);
}

template <typename T>
cudaError_t launch_bwd_t(const Params& p, const BwdArgs& q, cudaStream_t stream) {
  if (p.R <= 2) return launch_bwd_rt<T, 2>(p, q, stream);
  if (p.R <= 4) return launch_bwd_rt<T, 4>(p, q, stream);
  return launch_bwd_rt<T, 8>(p, q, stream);
}

}  // namespace

// CTAs per (batch, head): split the columns in two or four while the grid still fits one wave
// and every CTA keeps whole warps of columns
int bwd_col_split(const Params& p) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 1;
  for (int cs = 4; cs >= 2; cs /= 2)
    if (p.P % (32 * cs) == 0 && p.b * p.H * cs <= sms) return cs;
  return 1;
}

// tokens per recomputed block and the workspace the backward pass needs
int bwd_block(int64_t L) {
  int K = 1;
  while ((int64_t)K * K < L) ++K;
  return K;
}

size_t scan_bwd_workspace_bytes(const Params& p) {
  if (p.L <= 0) return 0;
  const int K = bwd_block(p.L);
  const int64_t nck = (p.L + K - 1) / K;
  const size_t nbh = (size_t)(p.b * p.H);
  const size_t states = nbh * (size_t)(nck + K) * p.N * p.P * 4;
  const size_t acc = 2 * (size_t)(p.b * p.L * p.G * p.R * p.N) * 4;
  return ((states + 255) & ~(size_t)255) + acc;
}

bool bwd_supported(const Params& p) {
  // at most 16 rotation pairs per thread (registers); headdim 256 with d_state >= 128 exceeds that
  return p.P <= kBwdThreads && p.R <= 8 && bwd_shape(p.P, p.N).NK <= 16 &&
         bwd_smem(p.P, p.N, p.R).total * 4 <= 200 * 1024;
}

cudaError_t launch_scan_bwd(const Params& p, const void* dy, const float* dh_final, void* dx, float* ddt, float* dA,
                            float* dlam, void* dB, void* dC, float* dtheta, float* dbias_B, float* dbias_C,
                            float* dW_x, float* dW_o, float* dD, float* dh0, float* dcarry_B, float* dcarry_x,
                            void* ws, size_t ws_bytes, cudaStream_t stream) {
  BwdArgs q;
  q.dy = dy; q.dh_final = dh_final; q.dx = dx; q.ddt = ddt; q.dA = dA; q.dlam = dlam; q.dB = dB; q.dC = dC;
  q.dtheta = dtheta; q.dbias_B = dbias_B; q.dbias_C = dbias_C; q.dW_x = dW_x; q.dW_o = dW_o; q.dD = dD;
  q.dh0 = dh0; q.dcarry_B = dcarry_B; q.dcarry_x = dcarry_x;
  q.K = bwd_block(p.L);
  q.nck = (int)((p.L + q.K - 1) / q.K);
  q.cs = bwd_col_split(p);
  const size_t nbh = (size_t)(p.b * p.H);
  const size_t states = nbh * (size_t)(q.nck + q.K) * p.N * p.P * 4;
  const int64_t nbc = p.b * p.L * p.G * p.R * p.N;
  if (ws_bytes < scan_bwd_workspace_bytes(p)) return cudaErrorInvalidValue;
  q.ckpt = static_cast<float*>(ws);
  q.accB = reinterpret_cast<float*>(static_cast<char*>(ws) + ((states + 255) & ~(size_t)255));
  q.accC = q.accB + nbc;
  // zero what several CTAs add into: the dB / dC accumulators, dtheta and the per-head sums
  bwd_zero_kernel<<<1024, 256, 0, stream>>>(q.accB, 2 * nbc, dtheta, p.b * p.L * p.G * (p.N / 2), dbias_B,
                                            dbias_B ? (int64_t)p.H * p.R * p.N : 0, dbias_C,
                                            dbias_C ? (int64_t)p.H * p.R * p.N : 0, nullptr, 0);
  bwd_zero_kernel<<<64, 256, 0, stream>>>(dW_x, dW_x ? (int64_t)p.H * p.R * p.P : 0, dW_o,
                                          dW_o ? (int64_t)p.H * p.R * p.P : 0, dD, dD ? p.H : 0, nullptr, 0,
                                          nullptr, 0);
  // the per-token scalars' gradients and dcarry_B are sums over columns, added by every CTA
  bwd_zero_kernel<<<256, 256, 0, stream>>>(ddt, p.b * p.L * p.H, dA, p.b * p.L * p.H, dlam, p.b * p.L * p.H,
                                           dcarry_B, p.b * p.H * p.R * p.N, nullptr, 0);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = p.dtype == M3_BF16 ? launch_bwd_t<__nv_bfloat16>(p, q, stream) : launch_bwd_t<float>(p, q, stream);
  if (e != cudaSuccess) return e;
  if (p.dtype == M3_BF16)
    bwd_store_kernel<__nv_bfloat16><<<1024, 256, 0, stream>>>(q.accB, q.accC, dB, dC, nbc);
  else
    bwd_store_kernel<float><<<1024, 256, 0, stream>>>(q.accB, q.accC, dB, dC, nbc);
  return cudaGetLastError();
}

}  // namespace m3
