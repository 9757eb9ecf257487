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
// walks units t, t + teams, ... of the range, so that while one team waits on a barrier the
// others update their units.  A unit's state tile is taken in `split` blocks of N / split rows,
// and each team keeps `stages` blocks in flight: while it updates one, the TMA engine brings the
// next blocks (state rows, the same rows of B, C and carry_B, and the token's x) into the team's
// ring of shared-memory stages.  One named barrier per block: the operands a block derives
// (biased B and C, rotation table, coefficients) alternate between two buffers, each thread
// sums its readout partial over the unit's blocks in registers, and the unit's output sum is
// written by half of the team during the next block's update.  The updated state goes straight
// from registers to HBM, so the copy engine only ever reads.

constexpr int kMaxStages = 6;
constexpr int kRingThreads = 512;
constexpr int kMaxTeams = 4;

struct RingPlan {
  int stages, split, teams, team_threads;
  uint32_t stage_bytes, team_bytes;
  // byte offsets inside a stage: state rows of the block and the same rows of raw B_t, raw C_t,
  // carry_B (R x NB each) and theta_t, raw x_t, carry_x, and the three per-unit scalars dt, A, lam
  uint32_t o_st, o_b, o_c, o_cb, o_x, o_cx, o_th, o_sc;
  // a block buffer (two per team, blocks alternate): the block's biased B_t, B_{t-1} and C_t,
  // the rotation table and the step's coefficients
  uint32_t blk_bytes, o_bbc, o_bbp, o_cbb, o_cs, o_coef;
  // a unit buffer (two per team, units alternate): the per-pair-group partial outputs of the unit
  uint32_t unit_bytes, o_red;
  // byte offsets inside a team's region, after its stages: the block and unit buffers, the
  // weights of the current head (bias_B, bias_C, W_x, W_o) and the stage barriers
  uint32_t o_blk, o_unit, o_wb, o_wc, o_wx, o_wo, o_bar;
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
  rp.o_b = o;  o += pad16((uint32_t)R * NB * esz);
  rp.o_c = o;  o += pad16((uint32_t)R * NB * esz);
  rp.o_cb = o; o += pad16((uint32_t)R * NB * 4);
  rp.o_x = o;  o += pad16((uint32_t)P * esz);
  rp.o_cx = o; o += pad16((uint32_t)P * 4);
  rp.o_th = o; o += pad16((uint32_t)NB / 2 * 4);
  rp.o_sc = o; o += 16;
  rp.stage_bytes = (o + 127u) & ~127u;
  o = 0;
  rp.o_bbc = o; o += pad16((uint32_t)R * NB * 4);
  rp.o_bbp = o; o += pad16((uint32_t)R * NB * 4);
  rp.o_cbb = o; o += pad16((uint32_t)R * NB * 4);
  rp.o_cs = o;  o += pad16((uint32_t)NB / 2 * 8);
  rp.o_coef = o; o += 16;
  rp.blk_bytes = o;
  o = 0;
  rp.o_red = o; o += pad16((uint32_t)ring_kg(P, NB, rp.team_threads) * P * 4);
  rp.unit_bytes = o;
  uint32_t f = 0;
  rp.o_blk = f;  f += 2 * rp.blk_bytes;
  rp.o_unit = f; f += 2 * rp.unit_bytes;
  rp.o_wb = f; f += pad16((uint32_t)R * N * 4);
  rp.o_wc = f; f += pad16((uint32_t)R * N * 4);
  rp.o_wx = f; f += pad16((uint32_t)R * P * 4);
  rp.o_wo = f; f += pad16((uint32_t)R * P * 4);
  rp.o_bar = f; f += 8 * kMaxStages;
  f = (f + 127u) & ~127u;
  const int room = max_bytes / teams - (int)f;
  int st = room > 0 ? room / (int)rp.stage_bytes : 0;
  rp.stages = st < kMaxStages ? st : kMaxStages;
  const uint32_t ring = (uint32_t)rp.stages * rp.stage_bytes;
  rp.o_blk += ring; rp.o_unit += ring; rp.o_bar += ring;
  rp.o_wb += ring; rp.o_wc += ring; rp.o_wx += ring; rp.o_wo += ring;
  rp.team_bytes = ring + f;
  rp.total = rp.team_bytes * (uint32_t)teams;
  return rp;
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// programmatic dependent launch: the next step's grid may start its set-up early; its first
// global access waits for this grid's completion
__device__ __forceinline__ void ring_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void ring_griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

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
    const uint32_t n_st = (uint32_t)NB * P * 4, n_b = (uint32_t)NB * esz, n_cb = (uint32_t)NB * 4;
    const uint32_t n_x = (uint32_t)P * esz, n_cx = (uint32_t)P * 4, n_th = (uint32_t)NB / 2 * 4;
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
                 "r"(n_st + (uint32_t)R * (2 * n_b + n_cb) + n_x + n_cx + n_th)
                 : "memory");
    const int n0 = c.blk * NB;
    const int64_t bc = ((c.bi * G + g) * R) * (int64_t)N + n0;  // row n0 of branch 0
    bulk_g2s(st + rp.o_st, p.h + (bh * N + n0) * P, n_st, bar);
    for (int r = 0; r < R; ++r) {
      bulk_g2s(st + rp.o_b + r * n_b, static_cast<const unsigned char*>(p.B) + (bc + (int64_t)r * N) * esz, n_b, bar);
      bulk_g2s(st + rp.o_c + r * n_b, static_cast<const unsigned char*>(p.C) + (bc + (int64_t)r * N) * esz, n_b, bar);
      bulk_g2s(st + rp.o_cb + r * n_cb, p.carry_B + (bh * R + r) * N + n0, n_cb, bar);
    }
    bulk_g2s(st + rp.o_x, static_cast<const unsigned char*>(p.x) + bh * P * esz, n_x, bar);
    bulk_g2s(st + rp.o_cx, p.carry_x + bh * P, n_cx, bar);
    bulk_g2s(st + rp.o_th, p.theta + (c.bi * G + g) * (N / 2) + n0 / 2, n_th, bar);
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
  ring_launch_dependents();
  if (tid == 0) {
    for (int s = 0; s < S; ++s)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 2;" ::"r"(bar0 + 8u * s));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  ring_griddep_wait();  // the previous step's state, carry and outputs are visible from here on
  if (tid == 0) {
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
  // y = sum_r W_o[r] * readout_r + D x of a finished unit: the partials of its pair groups
  // (D x rides in group 0's) summed, by the upper half of the team while the lower half starts
  // the next block's update
  auto finish_unit = [&](const unsigned char* ubuf, int64_t ybh, int lane0, int nlanes) {
    const float* red = reinterpret_cast<const float*>(ubuf + rp.o_red);
    const int nq = KG;
    for (int pp = tid - lane0; pp < P; pp += nlanes) {
      float acc0 = 0.0f, acc1 = 0.0f;
      int q = 0;
      for (; q + 1 < nq; q += 2) {
        acc0 += red[q * P + pp];
        acc1 += red[(q + 1) * P + pp];
      }
      if (q < nq) acc0 += red[q * P + pp];
      store_out<BF16>(p.y, ybh * P + pp, acc0 + acc1);
    }
  };
  float* wb = reinterpret_cast<float*>(smem + rp.o_wb);
  float* wc = reinterpret_cast<float*>(smem + rp.o_wc);
  float* wx = reinterpret_cast<float*>(smem + rp.o_wx);
  float* wo = reinterpret_cast<float*>(smem + rp.o_wo);
  int cur_h = -1;
  float Dh = 0.0f;
  uint32_t phases = 0;  // bit s: parity of the next completion of stage s
  int s = 0;
  bool ok = true;
  RingCursor cur = first;
  int ub = 0;            // unit buffer of the unit being updated
  bool pending = false;  // a finished unit whose y is still to be written
  int64_t pend_bh = 0;
  float oacc[4] = {0.f, 0.f, 0.f, 0.f};  // the thread's readout partial, summed over the unit's blocks
  const int half = TT / 2;
  const int pc = 4 * pq;  // the thread's first column
  int64_t j = 0;
  for (; j < nv; ++j) {
    const uint32_t par = (phases >> s) & 1u;
    phases ^= 1u << s;
    const int blk = cur.blk;
    const bool last_blk = blk == SPL - 1;
    const int hi = cur.hi;
    const int64_t bh = cur.bi * H + hi;
    const unsigned char* stg = smem + (size_t)s * rp.stage_bytes;
    unsigned char* bbuf = smem + rp.o_blk + (size_t)(j & 1) * rp.blk_bytes;
    unsigned char* ubuf = smem + rp.o_unit + (size_t)ub * rp.unit_bytes;
    float* bbc = reinterpret_cast<float*>(bbuf + rp.o_bbc);
    float* bbp = reinterpret_cast<float*>(bbuf + rp.o_bbp);
    float* cbb = reinterpret_cast<float*>(bbuf + rp.o_cbb);
    float2* cs = reinterpret_cast<float2*>(bbuf + rp.o_cs);
    float* coef = reinterpret_cast<float*>(bbuf + rp.o_coef);
    float* red = reinterpret_cast<float*>(ubuf + rp.o_red);
    if (hi != cur_h) {  // weights of a new head (uniform: the whole team sees the same unit)
      cur_h = hi;
      team_sync(bar_id, TT);  // every thread has finished the previous block's update (W_x, W_o)
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
      // ---- operands of this block (into the block buffer the previous block does not use)
      const float* sc = reinterpret_cast<const float*>(stg + rp.o_sc);
      const float* cBs = reinterpret_cast<const float*>(stg + rp.o_cb);
      const float* ths = reinterpret_cast<const float*>(stg + rp.o_th);
      const int n0 = blk * NB;
      // the block's rows of the new carry (this token's raw B): this block's copy of the old
      // rows has landed, and no other block reads them
      float* cBg = p.carry_B + bh * R * N + n0;
      for (int i = tid; i < R * NB; i += TT) {
        const int r = i / NB;
        const int rn = r * N + n0 + (i - r * NB);
        const float braw = stage_in<BF16>(stg + rp.o_b, i);
        const float bb = wb[rn];
        bbc[i] = braw + bb;
        bbp[i] = cBs[i] + bb;
        cbb[i] = stage_in<BF16>(stg + rp.o_c, i) + wc[rn];
        cBg[rn - n0] = braw;
      }
      const float delta = sc[0];
      // the rotation table from the team's last threads, the coefficients from its middle one,
      // so that the first warp (which issues the copies) carries no extra work
      for (int k = TT - 1 - tid; k < NB / 2; k += TT) {
        float sn, cn;
        sincosf(p.angle_direct ? ths[k] : delta * ths[k], &sn, &cn);
        cs[k] = make_float2(cn, sn);
      }
      if (tid == half) {
        const float lm = sc[2];
        coef[0] = expf(delta * sc[1]);
        coef[1] = (1.0f - lm) * delta;
        coef[2] = lm * delta;
      }
      if (last_blk) {
        // the unit's last block: every block's copy of the old carry_x has landed, so the new
        // one (this token's raw x) may overwrite it
        float* cxg = p.carry_x + bh * P;
        for (int pp = tid; pp < P; pp += TT) cxg[pp] = stage_in<BF16>(stg + rp.o_x, pp);
      }
    }
    if (team_sync_or(bar_id, TT, !ok)) {
      ok = false;
      phases ^= 1u << s;  // block j's copies count as outstanding again
      break;
    }
    // every thread is past the previous block's update: its stage may be refilled
    if (tid == 0 && j >= 1 && j - 1 + S < nv) {
      issue(ahead, s == 0 ? S - 1 : s - 1);
      ahead.next(SPL, T, nb);
    }
    if (pending) {
      if (tid >= half)
        finish_unit(smem + rp.o_unit + (size_t)(ub ^ 1) * rp.unit_bytes, pend_bh, half, TT - half);
      pending = false;
    }
    // ---- state update of the thread's 4 columns over its rotation pairs of the block
    if (kg < KG) {
      const float alpha = coef[0], bp = coef[1], gm = coef[2];
      const float* stt = reinterpret_cast<const float*>(stg + rp.o_st);
      float* hg = p.h + (bh * N + (int64_t)blk * NB) * P;
      // the MIMO branches of this column quad: X_r = W_x[r] x_t, X'_r = W_x[r] x_{t-1}
      float xq[4];
      if constexpr (BF16) {
        const uint2 raw = *reinterpret_cast<const uint2*>(stg + rp.o_x + 2 * pc);
        const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
        const float2 hi2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
        xq[0] = lo.x; xq[1] = lo.y; xq[2] = hi2.x; xq[3] = hi2.y;
      } else {
        const float4 v = *reinterpret_cast<const float4*>(stg + rp.o_x + 4 * pc);
        xq[0] = v.x; xq[1] = v.y; xq[2] = v.z; xq[3] = v.w;
      }
      const float4 cx4 = *reinterpret_cast<const float4*>(stg + rp.o_cx + 4 * pc);
      const float cq[4] = {cx4.x, cx4.y, cx4.z, cx4.w};
      float Xc[RT][4], Xp[RT][4], Y[RT][4];
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        const float4 w4 = r < R ? *reinterpret_cast<const float4*>(wx + r * P + pc) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float wq[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          Y[r][e] = 0.0f;
          Xc[r][e] = r < R ? xq[e] * wq[e] : 0.0f;
          Xp[r][e] = r < R ? cq[e] * wq[e] : 0.0f;
        }
      }
#pragma unroll 2
      for (int k = kg; k < NB / 2; k += KG) {
        const float4 s0 = *reinterpret_cast<const float4*>(stt + (2 * k) * P + pc);
        const float4 s1 = *reinterpret_cast<const float4*>(stt + (2 * k + 1) * P + pc);
        float u0v[4] = {}, u1v[4] = {}, q0[4] = {}, q1[4] = {};
#pragma unroll
        for (int r = 0; r < RT; ++r) {
          if (r < R) {
            const float2 bcv = *reinterpret_cast<const float2*>(bbc + r * NB + 2 * k);
            const float2 bqv = *reinterpret_cast<const float2*>(bbp + r * NB + 2 * k);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              u0v[e] = fmaf(bcv.x, Xc[r][e], u0v[e]);
              u1v[e] = fmaf(bcv.y, Xc[r][e], u1v[e]);
              q0[e] = fmaf(bqv.x, Xp[r][e], q0[e]);
              q1[e] = fmaf(bqv.y, Xp[r][e], q1[e]);
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
          n0[e] = fmaf(ac, v0, fmaf(-as, v1, gm * u0v[e]));
          n1[e] = fmaf(as, v0, fmaf(ac, v1, gm * u1v[e]));
        }
        *reinterpret_cast<float4*>(hg + (int64_t)(2 * k) * P + pc) = make_float4(n0[0], n0[1], n0[2], n0[3]);
        *reinterpret_cast<float4*>(hg + (int64_t)(2 * k + 1) * P + pc) = make_float4(n1[0], n1[1], n1[2], n1[3]);
#pragma unroll
        for (int r = 0; r < RT; ++r) {
          if (r < R) {
            const float2 cc = *reinterpret_cast<const float2*>(cbb + r * NB + 2 * k);
#pragma unroll
            for (int e = 0; e < 4; ++e) Y[r][e] = fmaf(cc.x, n0[e], fmaf(cc.y, n1[e], Y[r][e]));
          }
        }
      }
      // this pair group's part of sum_r W_o[r] * readout_r (+ D x in group 0), summed over the
      // unit's blocks in registers and over the pair groups when the unit's y is written
      if (blk == 0) {
#pragma unroll
        for (int e = 0; e < 4; ++e) oacc[e] = kg == 0 ? Dh * xq[e] : 0.0f;
      }
#pragma unroll
      for (int r = 0; r < RT; ++r)
        if (r < R) {
          const float4 w4 = *reinterpret_cast<const float4*>(wo + r * P + pc);
          oacc[0] = fmaf(w4.x, Y[r][0], oacc[0]);
          oacc[1] = fmaf(w4.y, Y[r][1], oacc[1]);
          oacc[2] = fmaf(w4.z, Y[r][2], oacc[2]);
          oacc[3] = fmaf(w4.w, Y[r][3], oacc[3]);
        }
      if (last_blk) *reinterpret_cast<float4*>(red + kg * P + pc) = make_float4(oacc[0], oacc[1], oacc[2], oacc[3]);
    }
    if (last_blk) {  // the unit's y is written during the next block's update
      pending = true;
      pend_bh = bh;
      ub ^= 1;
    }
    s = (s + 1 == S) ? 0 : s + 1;
    cur.next(SPL, T, nb);
  }
  if (ok) {
    team_sync(bar_id, TT);  // the last unit's readouts are in place
    if (pending) finish_unit(smem + rp.o_unit + (size_t)(ub ^ 1) * rp.unit_bytes, pend_bh, 0, TT);
  } else if (tid == 0) {
    // give up: wait (bounded) for the team's copies still in flight (blocks j .. j + S - 2, or
    // the first S when the first wait failed), then report
    const int64_t last = j == 0 ? S - 1 : j + S - 2;
    for (int64_t w = j; w <= last && w < nv; ++w) {
      const int sw = (int)(w % S);
      wait(sw, (phases >> sw) & 1u);
    }
    set_status(p.status, M3_ERR_TIMEOUT);
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

// launch with programmatic stream serialisation (the kernel waits on the previous grid before
// its first global access)
template <typename Kernel>
cudaError_t launch_ring_pdl(Kernel k, unsigned grid, size_t smem, cudaStream_t stream, const Params& p,
                            const RingPlan& rp) {
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kRingThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, p, rp);
}

template <int RT>
cudaError_t launch_ring_rt(const Params& p, const RingPlan& rp, unsigned grid, cudaStream_t stream) {
  return p.dtype == M3_BF16 ? launch_ring_pdl(decode_ring_kernel<RT, true>, grid, rp.total, stream, p, rp)
                            : launch_ring_pdl(decode_ring_kernel<RT, false>, grid, rp.total, stream, p, rp);
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
