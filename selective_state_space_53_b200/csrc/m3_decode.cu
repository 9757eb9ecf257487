// m3_decode.cu -- one-token decode update of the Mamba-3 SSM core (m3_decode_step).
//
// Decode reads and rewrites the whole fixed-size state every token (Mamba-3 paper note,
// docsaid.org, section その3: the step is memory-bound; MIMO rank R adds arithmetic per state
// byte).  Per (batch, head) unit and state row pair (2k, 2k+1):
//     h <- e^{dt A} Rot(dt theta) (h + (1 - lam) dt u_{t-1}) + lam dt u_t,
//     u = sum_r Bb_r X_r^T   (section その1 trapezoid rule, section その2 rotation, section その3 MIMO)
// and y = sum_r W_o[r] * (Cb_r^T h) + D x.  The kernel is persistent: each CTA walks a range of
// units, their state tiles streaming through a ring of shared-memory stages filled by the TMA
// engine (cp.async.bulk, completion counted in bytes on an mbarrier per stage) while the threads
// update the stage that has landed and write the new state straight to HBM.  Every wait is
// bounded by %globaltimer; a timeout sets M3_ERR_TIMEOUT in the device status word.
#include "m3_common.cuh"

namespace m3 {
namespace {

constexpr unsigned long long kWaitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------------ ring form
// Persistent form: each CTA takes a contiguous range of (batch, head) units, ordered head-major
// so that the per-head weights change at most a few times per CTA.  The CTA's threads form
// `teams` independent teams (named barriers, no CTA-wide synchronisation after set-up); team t
// walks units t, t + teams, ... of the range, so that while one team waits on a barrier or on
// its copies the others update theirs.  A unit's state tile is taken in `split` blocks of
// N / split rows (the readouts are summed over the blocks in shared memory), and each team
// keeps `stages` blocks in flight: while it updates one, the TMA engine brings the next blocks
// (state rows and raw token operands) into the team's ring of shared-memory stages.  The
// updated state goes straight from registers to HBM, so the copy engine only ever reads.

constexpr int kMaxStages = 6;
constexpr int kRingThreads = 512;
constexpr int kMaxTeams = 4;

struct RingPlan {
  int stages, split, teams, team_threads;
  uint32_t stage_bytes, team_bytes;
  // byte offsets inside a stage: state rows of the block, raw B_t, raw C_t, carry_B, raw x_t,
  // carry_x, theta_t, and the three per-unit scalars dt, A, lam
  uint32_t o_st, o_b, o_c, o_cb, o_x, o_cx, o_th, o_sc;
  // byte offsets (inside a team's region, after its stages) of the single-buffered arrays: the
  // block's biased B, C and the MIMO branches, the rotation table and coefficients, the weights
  // of the current head (bias_B, bias_C, W_x, W_o) and the per-pair-group partial readouts of
  // every block of the unit
  uint32_t o_bbc, o_bbp, o_cbb, o_xc, o_xp, o_xr, o_cs, o_coef, o_wb, o_wc, o_wx, o_wo, o_red, o_bar;
  uint32_t total;
};

// thread (pq, kg) of a team: columns 4 pq .. 4 pq + 3, rotation pairs kg, kg + KG, ... of the block
__host__ __device__ inline int ring_pq(int P) { return P / 4; }
__host__ __device__ inline int ring_kg(int P, int NB, int team_threads) {
  const int kg = team_threads / ring_pq(P);
  return kg < NB / 2 ? kg : NB / 2;
}

__host__ __device__ inline uint32_t pad16(uint32_t x) { return (x + 15u) & ~15u; }

// Layout of one team's region for `teams` teams sharing max_bytes; stages = 0 if none fits.
inline RingPlan ring_plan(int P, int N, int R, bool bf16, int split, int teams, int max_bytes) {
  const uint32_t esz = bf16 ? 2u : 4u;
  const int NB = N / split;
  RingPlan rp{};
  rp.split = split;
  rp.teams = teams;
  rp.team_threads = kRingThreads / teams;
  uint32_t o = 0;
  rp.o_st = o; o += pad16((uint32_t)NB * P * 4);
  rp.o_b = o;  o += pad16((uint32_t)R * N * esz);
  rp.o_c = o;  o += pad16((uint32_t)R * N * esz);
  rp.o_cb = o; o += pad16((uint32_t)R * N * 4);
  rp.o_x = o;  o += pad16((uint32_t)P * esz);
  rp.o_cx = o; o += pad16((uint32_t)P * 4);
  rp.o_th = o; o += pad16((uint32_t)N / 2 * 4);
  rp.o_sc = o; o += 16;
  rp.stage_bytes = (o + 127u) & ~127u;
  uint32_t f = 0;
  rp.o_bbc = f; f += pad16((uint32_t)R * NB * 4);
  rp.o_bbp = f; f += pad16((uint32_t)R * NB * 4);
  rp.o_cbb = f; f += pad16((uint32_t)R * NB * 4);
  rp.o_xc = f;  f += pad16((uint32_t)R * P * 4);
  rp.o_xp = f;  f += pad16((uint32_t)R * P * 4);
  rp.o_xr = f;  f += pad16((uint32_t)P * 4);
  rp.o_cs = f;  f += pad16((uint32_t)NB / 2 * 8);
  rp.o_coef = f; f += 16;
  rp.o_wb = f; f += pad16((uint32_t)R * N * 4);
  rp.o_wc = f; f += pad16((uint32_t)R * N * 4);
  rp.o_wx = f; f += pad16((uint32_t)R * P * 4);
  rp.o_wo = f; f += pad16((uint32_t)R * P * 4);
  rp.o_red = f; f += pad16((uint32_t)split * ring_kg(P, NB, rp.team_threads) * P * 4);
  rp.o_bar = f; f += 8 * kMaxStages;
  f = (f + 127u) & ~127u;
  const int room = max_bytes / teams - (int)f;
  int st = room > 0 ? room / (int)rp.stage_bytes : 0;
  rp.stages = st < kMaxStages ? st : kMaxStages;
  const uint32_t ring = (uint32_t)rp.stages * rp.stage_bytes;
  rp.o_bbc += ring; rp.o_bbp += ring; rp.o_cbb += ring; rp.o_xc += ring; rp.o_xp += ring;
  rp.o_xr += ring; rp.o_cs += ring; rp.o_coef += ring; rp.o_wb += ring; rp.o_wc += ring;
  rp.o_wx += ring; rp.o_wo += ring; rp.o_red += ring; rp.o_bar += ring;
  rp.team_bytes = ring + f;
  rp.total = rp.team_bytes * (uint32_t)teams;
  return rp;
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// named barrier of one team (id >= 1; id 0 is __syncthreads)
__device__ __forceinline__ void team_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// named barrier that also returns whether any thread of the team passed `pred` true
__device__ __forceinline__ bool team_sync_or(int id, int nthreads, bool pred) {
  uint32_t any;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(any)
      : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
      : "memory");
  return any != 0;
}

template <bool BF16>
__device__ __forceinline__ float stage_in(const unsigned char* base, int i) {
  if constexpr (BF16) {
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[i]);
  } else {
    return reinterpret_cast<const float*>(base)[i];
  }
}

// Position of a team in its walk: unit u (head-major: head hi, sequence bi) and block blk.
struct RingCursor {
  int64_t bi;
  int hi, blk;
  __device__ __forceinline__ void next(int split, int teams, int64_t nb) {
    if (++blk < split) return;
    blk = 0;
    bi += teams;
    while (bi >= nb) {
      bi -= nb;
      ++hi;
    }
  }
};

template <int RT, bool BF16>
__global__ void __launch_bounds__(kRingThreads, 1) decode_ring_kernel(Params p, RingPlan rp) {
  extern __shared__ __align__(128) unsigned char smem_cta[];
  const int TT = rp.team_threads;
  const int team = threadIdx.x / TT;
  const int tid = threadIdx.x % TT;
  const int bar_id = 1 + team;
  unsigned char* smem = smem_cta + (size_t)team * rp.team_bytes;
  const int H = p.H, P = p.P, N = p.N, R = p.R, G = p.G;
  const int SPL = rp.split;
  const int NB = N / SPL;  // state rows per block
  const int T = rp.teams;
  const int64_t nb = p.b;
  const int64_t U = nb * H;
  // this CTA's units [u0, u1); the team takes u0 + team, u0 + team + T, ..., each in SPL blocks
  const int64_t u0 = (int64_t)blockIdx.x * U / gridDim.x;
  const int64_t u1 = (int64_t)(blockIdx.x + 1) * U / gridDim.x;
  const int64_t nv = (u0 + team < u1 ? (u1 - u0 - team + T - 1) / T : 0) * SPL;
  const int S = rp.stages;
  constexpr uint32_t esz = BF16 ? 2u : 4u;
  const uint32_t sbase = smem_u32(smem);
  float* bbc = reinterpret_cast<float*>(smem + rp.o_bbc);
  float* bbp = reinterpret_cast<float*>(smem + rp.o_bbp);
  float* cbb = reinterpret_cast<float*>(smem + rp.o_cbb);
  float* xc = reinterpret_cast<float*>(smem + rp.o_xc);
  float* xp = reinterpret_cast<float*>(smem + rp.o_xp);
  float* xr = reinterpret_cast<float*>(smem + rp.o_xr);
  float2* cs = reinterpret_cast<float2*>(smem + rp.o_cs);
  float* coef = reinterpret_cast<float*>(smem + rp.o_coef);
  float* wb = reinterpret_cast<float*>(smem + rp.o_wb);
  float* wc = reinterpret_cast<float*>(smem + rp.o_wc);
  float* wx = reinterpret_cast<float*>(smem + rp.o_wx);
  float* wo = reinterpret_cast<float*>(smem + rp.o_wo);
  float* red = reinterpret_cast<float*>(smem + rp.o_red);
  const uint32_t bar0 = sbase + rp.o_bar;
  RingCursor first{0, 0, 0};
  if (nv > 0) {
    first.bi = (u0 + team) % nb;
    first.hi = (int)((u0 + team) / nb);
  }

  auto issue = [&](const RingCursor& c, int s) {
    const int g = c.hi / (H / G);
    const int64_t bh = c.bi * H + c.hi;
    const uint32_t st = sbase + (uint32_t)s * rp.stage_bytes;
    const uint32_t bar = bar0 + 8u * s;
    const uint32_t n_st = (uint32_t)NB * P * 4, n_b = (uint32_t)R * N * esz, n_cb = (uint32_t)R * N * 4;
    const uint32_t n_x = (uint32_t)P * esz, n_cx = (uint32_t)P * 4, n_th = (uint32_t)N / 2 * 4;
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
                 "r"(n_st + 2 * n_b + n_cb + n_x + n_cx + n_th)
                 : "memory");
    const int64_t bc = ((c.bi * G + g) * R) * (int64_t)N;
    bulk_g2s(st + rp.o_st, p.h + (bh * N + (int64_t)c.blk * NB) * P, n_st, bar);
    bulk_g2s(st + rp.o_b, static_cast<const unsigned char*>(p.B) + bc * esz, n_b, bar);
    bulk_g2s(st + rp.o_c, static_cast<const unsigned char*>(p.C) + bc * esz, n_b, bar);
    bulk_g2s(st + rp.o_cb, p.carry_B + bh * R * N, n_cb, bar);
    bulk_g2s(st + rp.o_x, static_cast<const unsigned char*>(p.x) + bh * P * esz, n_x, bar);
    bulk_g2s(st + rp.o_cx, p.carry_x + bh * P, n_cx, bar);
    bulk_g2s(st + rp.o_th, p.theta + (c.bi * G + g) * (N / 2), n_th, bar);
    // the three scalars: 4-byte asynchronous copies whose completion is the barrier's second arrival
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(st + rp.o_sc), "l"(p.dt + bh) : "memory");
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(st + rp.o_sc + 4), "l"(p.A + bh) : "memory");
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(st + rp.o_sc + 8), "l"(p.lam + bh) : "memory");
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
  };
  auto try_wait = [&](int s, uint32_t par) -> bool {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred q;\n mbarrier.try_wait.parity.shared::cta.b64 q, [%1], %2;\n selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(done)
        : "r"(bar0 + 8u * s), "r"(par)
        : "memory");
    return done != 0;
  };
  auto wait = [&](int s, uint32_t par) -> bool {
    if (try_wait(s, par)) return true;
    const uint64_t t0 = globaltimer();
    while (!try_wait(s, par)) {
      if (globaltimer() - t0 > kWaitNs) return false;
    }
    return true;
  };

  RingCursor ahead = first;  // the next block to issue (the team leader's)
  if (tid == 0) {
    for (int s = 0; s < S; ++s)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 2;" ::"r"(bar0 + 8u * s));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (int s = 0; s < S && s < nv; ++s) {
      issue(ahead, s);
      ahead.next(SPL, T, nb);
    }
  }
  __syncthreads();  // barriers initialised (the only CTA-wide synchronisation)

  const int PQ = ring_pq(P);
  const int KG = ring_kg(P, NB, TT);
  const int pq = tid % PQ;
  const int kg = tid / PQ;
  constexpr int CQ = 1;  // 4-column quads per thread (the compute below takes any count)
  int cur_h = -1;
  float Dh = 0.0f;
  uint32_t phases = 0;  // bit s: parity of the next completion of stage s
  int s = 0;
  bool ok = true;
  RingCursor cur = first;
  int64_t j = 0;
  for (; j < nv; ++j) {
    const uint32_t par = (phases >> s) & 1u;
    phases ^= 1u << s;
    const int blk = cur.blk;
    const bool last_blk = blk == SPL - 1;
    const int hi = cur.hi;
    const int64_t bh = cur.bi * H + hi;
    const unsigned char* stg = smem + (size_t)s * rp.stage_bytes;
    if (hi != cur_h) {  // weights of a new head (uniform: the whole team sees the same unit)
      cur_h = hi;
      team_sync(bar_id, TT);  // the previous block's update has read W_o
      const float* biasB = p.bias_B ? p.bias_B + (int64_t)hi * R * N : nullptr;
      const float* biasC = p.bias_C ? p.bias_C + (int64_t)hi * R * N : nullptr;
      const float* Wx = p.W_x ? p.W_x + (int64_t)hi * R * P : nullptr;
      const float* Wo = p.W_o ? p.W_o + (int64_t)hi * R * P : nullptr;
      for (int i = tid; i < R * N; i += TT) {
        wb[i] = biasB ? biasB[i] : 0.0f;
        wc[i] = biasC ? biasC[i] : 0.0f;
      }
      for (int i = tid; i < R * P; i += TT) {
        wx[i] = Wx ? Wx[i] : 1.0f;
        wo[i] = Wo ? Wo[i] : 1.0f;
      }
      Dh = p.D ? p.D[hi] : 0.0f;
      team_sync(bar_id, TT);
    }
    ok = wait(s, par);
    if (ok) {
      // ---- operands of this block
      const float* sc = reinterpret_cast<const float*>(stg + rp.o_sc);
      const float* cBs = reinterpret_cast<const float*>(stg + rp.o_cb);
      const float* cxs = reinterpret_cast<const float*>(stg + rp.o_cx);
      const float* ths = reinterpret_cast<const float*>(stg + rp.o_th);
      const int n0 = blk * NB;
      for (int i = tid; i < R * NB; i += TT) {
        const int r = i / NB, n = n0 + i % NB;
        const float bb = wb[r * N + n];
        bbc[i] = stage_in<BF16>(stg + rp.o_b, r * N + n) + bb;
        bbp[i] = cBs[r * N + n] + bb;
        cbb[i] = stage_in<BF16>(stg + rp.o_c, r * N + n) + wc[r * N + n];
      }
      for (int i = tid; i < R * P; i += TT) {
        const float w = wx[i];
        xc[i] = stage_in<BF16>(stg + rp.o_x, i % P) * w;
        xp[i] = cxs[i % P] * w;
      }
      const float delta = sc[0];
      for (int k = tid; k < NB / 2; k += TT) {
        float sn, cn;
        sincosf(p.angle_direct ? ths[n0 / 2 + k] : delta * ths[n0 / 2 + k], &sn, &cn);
        cs[k] = make_float2(cn, sn);
      }
      if (tid == 0) {
        const float lm = sc[2];
        coef[0] = expf(delta * sc[1]);
        coef[1] = (1.0f - lm) * delta;
        coef[2] = lm * delta;
      }
      if (last_blk) {
        // the unit's last block: every block's copy of the old carry has landed, so the new
        // carry (this token's raw B and x) may overwrite it
        float* cBg = p.carry_B + bh * R * N;
        float* cxg = p.carry_x + bh * P;
        for (int i = tid; i < R * N; i += TT) cBg[i] = stage_in<BF16>(stg + rp.o_b, i);
        for (int pp = tid; pp < P; pp += TT) {
          const float xv = stage_in<BF16>(stg + rp.o_x, pp);
          xr[pp] = xv;
          cxg[pp] = xv;
        }
      }
    }
    if (team_sync_or(bar_id, TT, !ok)) {
      ok = false;
      phases ^= 1u << s;  // block j's copies count as outstanding again
      break;
    }
    // ---- state update of the thread's 4 columns over its rotation pairs of the block
    if (kg < KG) {
      const float alpha = coef[0], bp = coef[1], gm = coef[2];
      const float* stt = reinterpret_cast<const float*>(stg + rp.o_st);
      float* hg = p.h + (bh * N + (int64_t)blk * NB) * P;
      int pc[CQ];
#pragma unroll
      for (int c = 0; c < CQ; ++c) pc[c] = 4 * pq + c * (P / CQ);
      float4 Xc[RT][CQ], Xp[RT][CQ];
      float Y[RT][CQ][4];
#pragma unroll
      for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int c = 0; c < CQ; ++c) {
          Y[r][c][0] = Y[r][c][1] = Y[r][c][2] = Y[r][c][3] = 0.0f;
          if (r < R) {
            Xc[r][c] = *reinterpret_cast<const float4*>(xc + r * P + pc[c]);
            Xp[r][c] = *reinterpret_cast<const float4*>(xp + r * P + pc[c]);
          } else {
            Xc[r][c] = Xp[r][c] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
#pragma unroll 2
      for (int k = kg; k < NB / 2; k += KG) {
        float4 s0[CQ], s1[CQ];
#pragma unroll
        for (int c = 0; c < CQ; ++c) {
          s0[c] = *reinterpret_cast<const float4*>(stt + (2 * k) * P + pc[c]);
          s1[c] = *reinterpret_cast<const float4*>(stt + (2 * k + 1) * P + pc[c]);
        }
        float u0v[CQ][4] = {}, u1v[CQ][4] = {}, q0[CQ][4] = {}, q1[CQ][4] = {};
#pragma unroll
        for (int r = 0; r < RT; ++r) {
          if (r < R) {
            const float2 bcv = *reinterpret_cast<const float2*>(bbc + r * NB + 2 * k);
            const float2 bqv = *reinterpret_cast<const float2*>(bbp + r * NB + 2 * k);
#pragma unroll
            for (int c = 0; c < CQ; ++c) {
              const float xc4[4] = {Xc[r][c].x, Xc[r][c].y, Xc[r][c].z, Xc[r][c].w};
              const float xp4[4] = {Xp[r][c].x, Xp[r][c].y, Xp[r][c].z, Xp[r][c].w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                u0v[c][e] = fmaf(bcv.x, xc4[e], u0v[c][e]);
                u1v[c][e] = fmaf(bcv.y, xc4[e], u1v[c][e]);
                q0[c][e] = fmaf(bqv.x, xp4[e], q0[c][e]);
                q1[c][e] = fmaf(bqv.y, xp4[e], q1[c][e]);
              }
            }
          }
        }
        const float2 rc = cs[k];
        const float ac = alpha * rc.x, as = alpha * rc.y;
        float n0[CQ][4], n1[CQ][4];
#pragma unroll
        for (int c = 0; c < CQ; ++c) {
          const float a0[4] = {s0[c].x, s0[c].y, s0[c].z, s0[c].w};
          const float a1[4] = {s1[c].x, s1[c].y, s1[c].z, s1[c].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float v0 = fmaf(bp, q0[c][e], a0[e]);
            const float v1 = fmaf(bp, q1[c][e], a1[e]);
            n0[c][e] = fmaf(ac, v0, fmaf(-as, v1, gm * u0v[c][e]));
            n1[c][e] = fmaf(as, v0, fmaf(ac, v1, gm * u1v[c][e]));
          }
          *reinterpret_cast<float4*>(hg + (int64_t)(2 * k) * P + pc[c]) =
              make_float4(n0[c][0], n0[c][1], n0[c][2], n0[c][3]);
          *reinterpret_cast<float4*>(hg + (int64_t)(2 * k + 1) * P + pc[c]) =
              make_float4(n1[c][0], n1[c][1], n1[c][2], n1[c][3]);
        }
#pragma unroll
        for (int r = 0; r < RT; ++r) {
          if (r < R) {
            const float2 cc = *reinterpret_cast<const float2*>(cbb + r * NB + 2 * k);
#pragma unroll
            for (int c = 0; c < CQ; ++c)
#pragma unroll
              for (int e = 0; e < 4; ++e) Y[r][c][e] = fmaf(cc.x, n0[c][e], fmaf(cc.y, n1[c][e], Y[r][c][e]));
          }
        }
      }
      // this pair group's part of sum_r W_o[r] * readout_r; summed over groups and blocks later
#pragma unroll
      for (int c = 0; c < CQ; ++c) {
        float o[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int r = 0; r < RT; ++r)
          if (r < R) {
            const float4 w4 = *reinterpret_cast<const float4*>(wo + r * P + pc[c]);
            o[0] = fmaf(w4.x, Y[r][c][0], o[0]);
            o[1] = fmaf(w4.y, Y[r][c][1], o[1]);
            o[2] = fmaf(w4.z, Y[r][c][2], o[2]);
            o[3] = fmaf(w4.w, Y[r][c][3], o[3]);
          }
        *reinterpret_cast<float4*>(red + (blk * KG + kg) * P + pc[c]) = make_float4(o[0], o[1], o[2], o[3]);
      }
    }
    team_sync(bar_id, TT);  // stage s is read; the block's readouts are in place
    if (tid == 0 && j + S < nv) {
      issue(ahead, s);
      ahead.next(SPL, T, nb);
    }
    if (last_blk) {
      // ---- y = sum_r W_o[r] * readout_r + D x, the readouts summed over groups and blocks
      const int nq = SPL * KG;
      for (int pp = tid; pp < P; pp += TT) {
        float acc0 = 0.0f, acc1 = 0.0f;
        int q = 0;
        for (; q + 1 < nq; q += 2) {
          acc0 += red[q * P + pp];
          acc1 += red[(q + 1) * P + pp];
        }
        if (q < nq) acc0 += red[q * P + pp];
        store_out<BF16>(p.y, bh * P + pp, fmaf(Dh, xr[pp], acc0 + acc1));
      }
    }
    s = (s + 1 == S) ? 0 : s + 1;
    cur.next(SPL, T, nb);
  }
  if (!ok) {
    // give up: wait (bounded) for the team's copies still in flight, then report
    if (tid == 0) {
      for (int64_t w = j; w < nv && w < j + S; ++w) {
        const int sw = (int)(w % S);
        wait(sw, (phases >> sw) & 1u);
      }
      set_status(p.status, M3_ERR_TIMEOUT);
    }
  }
}

struct DeviceLimits {
  int sms = 0, smem_optin = 0, smem_sm = 0;
};
// SM count and opt-in shared memory per block of the current device (cached per device).
DeviceLimits device_limits() {
  static PerDevice<DeviceLimits> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DeviceLimits{};
  DeviceLimits out{};
  cache.get(dev, &out, [dev](DeviceLimits* d) {
    int sms = 0, optin = 0, per_sm = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess)
      return false;
    d->sms = sms;
    d->smem_optin = optin;
    d->smem_sm = per_sm;
    return true;
  });
  return out;
}

template <int RT>
cudaError_t launch_ring_rt(const Params& p, const RingPlan& rp, unsigned grid, cudaStream_t stream) {
  if (p.dtype == M3_BF16) {
    auto k = decode_ring_kernel<RT, true>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rp.total);
    if (e != cudaSuccess) return e;
    k<<<grid, kRingThreads, rp.total, stream>>>(p, rp);
  } else {
    auto k = decode_ring_kernel<RT, false>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rp.total);
    if (e != cudaSuccess) return e;
    k<<<grid, kRingThreads, rp.total, stream>>>(p, rp);
  }
  return cudaGetLastError();
}

// The ring form needs two stages per team at least.  Preferred: the most teams (units in flight
// per CTA) whose threads each get a column quad, at the fewest row blocks per unit.
bool ring_plan_for(const Params& p, RingPlan* out) {
  const DeviceLimits d = device_limits();
  if (d.sms == 0) return false;
  const bool bf16 = p.dtype == M3_BF16;
  for (int teams = kMaxTeams; teams >= 1; teams /= 2) {
    if (kRingThreads / teams < ring_pq(p.P)) continue;
    for (int split = 1; split <= 4; split *= 2) {
      if (p.N % (2 * split) != 0 || (p.N / split) % 8 != 0) break;
      const RingPlan rp = ring_plan(p.P, p.N, p.R, bf16, split, teams, d.smem_optin);
      if (rp.stages >= 2) {
        *out = rp;
        return true;
      }
    }
  }
  return false;
}

}  // namespace

bool decode_supported(const Params& p) {
  if (decode_tc_supported(p)) return true;
  RingPlan rp;
  return ring_plan_for(p, &rp);
}

cudaError_t launch_decode(const Params& p, cudaStream_t stream) {
  if (p.b * p.H == 0) return cudaSuccess;
  if (decode_tc_supported(p)) return launch_decode_tc(p, stream);
  RingPlan rp;
  if (ring_plan_for(p, &rp)) {
    const int64_t units = p.b * p.H;
    const int64_t slots = device_limits().sms;
    const unsigned grid = (unsigned)(units < slots ? units : slots);
    if (p.R <= 1) return launch_ring_rt<1>(p, rp, grid, stream);
    if (p.R <= 2) return launch_ring_rt<2>(p, rp, grid, stream);
    if (p.R <= 4) return launch_ring_rt<4>(p, rp, grid, stream);
    return launch_ring_rt<8>(p, rp, grid, stream);
  }
  return cudaErrorInvalidConfiguration;  // callers check decode_supported first
}

}  // namespace m3
