// m3_scan_tc.cu -- chunked Mamba-3 prefill scan on the sm_100a tensor cores (TMA + tcgen05 + TMEM).
//
// A CTA walks one segment of one (batch, head) sequence in tiles of Q = 128 / R tokens, so
// that a tile has exactly 128 rows i = t * R + r (token t, MIMO branch r) -- the M of one
// tcgen05.mma.  The chunked form is exact (IBM Mamba page, SSD section: the scan splits into
// chunks combined associatively), so the tile length does not change the result; for R = 4
// it is the model's chunk of 32 tokens.
//
// Per tile, with Lc_t the tile-local cumulative sum of dt A (log decay) and Phi_t the
// cumulative rotation angle from the segment start (kept per pair in fp64, reduced mod 2 pi):
//   Bt_i = Rot(-Phi_t)(B_{t,r} + bias_B),  Ct_i = Rot(-Phi_t)(C_{t,r} + bias_C)
//     -- the rotation absorbed into B and C as a data-dependent RoPE (Mamba-3 paper note,
//        docsaid.org, section その2, statement 2);
//   S  = Ct Bt^T                                        (MMA1, 128 x 128, K = N)
//   S'[i,j] = S[i,j] e^{Lc_t - Lc_s} (gamma_s + [s<t] beta'_{s+1}) for s <= t, else 0
//     -- the trapezoid weights of section その1 (gamma = lam dt, beta' = (1 - lam) dt):
//        the input of token s enters h_s with gamma_s and h_{s+1} with beta'_{s+1};
//   Y  = S' X + diag(e^{Lc}) Ct h+                      (MMA2 + MMA3)
//     with X_i = W_x[r] * x_t (MIMO branches, section その3) and h+ the rotated-frame state
//     entering the tile (including the previous token's trapezoid term);
//   h+ <- e^{Lc_e} h+ + Xs^T Bt,  Xs_i = e^{Lc_e - Lc_t} (gamma_t + beta'_{t+1}) X_i   (MMA4)
//   y_t = sum_r W_o[r] * Y_{t,r} + D x_t.
// In the rotated frame the state update is a plain decay-and-add; the state is rotated back
// once, at the end of the sequence.
//
// Sequence splitting.  With few (batch, head) sequences the grid is b * H * nseg CTAs: a
// state-only pass (MODE_STATE: Bt, Xs, MMA4, state update) first runs segments 0..nseg-2, cut
// into m sub-segments each where free CTA slots allow, from a zero state and writes each
// sub-segment's end state, total log decay and total angle to the workspace; the full pass
// (MODE_FULL) then starts segment k from the combination of the summaries before it.  Both
// passes are the same chunk algebra; only the starting state differs.
//
// On chip: B and C tiles arrive by TMA (cp.async.bulk.tensor, 128-byte swizzle) directly in
// the canonical K-major UMMA layout and are rotated in place; x arrives by TMA into a staging
// buffer; Delta, A, lambda and theta are loaded into registers one tile ahead.  The next tile's
// loads are issued as soon as the buffers they overwrite are consumed, so they land while the
// current tile computes.  Accumulators S, Y, H and the
// fp32 state live in tensor memory; the masked S is written back into TMEM as bf16 pairs and
// consumed as the A operand of MMA2.
//
// Warp roles: all 8 warps stage tiles and run the epilogue (each its TMEM lane quarter, half
// the columns); thread 0 issues the TMA loads; warp 0 issues the MMAs (one elected lane) and
// commits them to an mbarrier, and builds the next tile's coefficients; warps 0-3 mask S
// while warps 4-7 update the state; all warps build the rotation tables.
// Every mbarrier wait is bounded by %globaltimer; a timeout sets M3_ERR_TIMEOUT in the device
// status word and the CTA frees its TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "m3_common.cuh"
#include "m3_ptx.cuh"
#include "m3_scan_plan.cuh"

namespace m3 {
namespace {

constexpr int kThreads = 256;
constexpr int kRows = 128;
constexpr unsigned long long kWaitNs = 2000000000ull;  // 2 s bound on any mbarrier wait
constexpr int MODE_FULL = 0, MODE_STATE = 1;
// Largest log-decay range of a tile that takes the pivot split.  The split scales X' rows by
// b_s = e^{m - Lc_s} <= e^{range / 2} and applies a_t only after S' X' has been summed in fp32,
// so the sum can reach Q R max|S| max|w x| e^{range / 2}; at 64 that is below 1e21 max|w x|,
// far from the fp32 limit (3.4e38) for any sane input.  Wider tiles take the exact path.
constexpr float kFastRange = 64.0f;

// ------------------------------------------------------------------ waits

// Bounded wait: false after kWaitNs without the phase completing.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > kWaitNs) return false;
  }
  return true;
}
// ------------------------------------------------------------------ configuration


template <int R, int N, int P, int MODE>
struct Cfg {
  static constexpr bool FULL = (MODE == MODE_FULL);
  static constexpr int Q = kRows / R;   // tokens per tile
  static constexpr int K2 = N / 2;      // rotation pairs
  static constexpr int TILE_N = kRows * N * 2;
  static constexpr int TILE_P = kRows * P * 2;
  static constexpr int TILE_H = P * N * 2;
  static constexpr int OFF_BT = 0;
  static constexpr int OFF_CT = OFF_BT + TILE_N;
  static constexpr int OFF_X = OFF_CT + (FULL ? TILE_N : 0);
  static constexpr int OFF_H = OFF_X + TILE_P;
  static constexpr int OFF_CS = OFF_H + (FULL ? TILE_H : 0);       // float2 [2][Q][K2]
  static constexpr int OFF_XSTG = OFF_CS + 2 * Q * K2 * 8;          // x staging [Q][P] bf16
  static constexpr int OFF_WX = OFF_XSTG + Q * P * 2;              // W_x [R][P]
  static constexpr int OFF_WO = OFF_WX + R * P * 4;                 // W_o [R][P]
  static constexpr int OFF_BASE = OFF_WO + R * P * 4;               // double [K2]
  static constexpr int SEGS = kThreads / K2;                        // angle prefix segments
  static constexpr int SEGLEN = (Q + SEGS - 1) / SEGS;
  static constexpr int OFF_SEGSUM = OFF_BASE + K2 * 8;              // float [SEGS][K2]
  static constexpr int TOKF = Q + 4;
  static constexpr int OFF_RAW = OFF_SEGSUM + SEGS * K2 * 4;        // float [2][4][TOKF]: dt, A, lam, (misc)
  static constexpr int OFF_REC = OFF_RAW + 2 * 4 * TOKF * 4;        // float4 [2][2][Q]
  static constexpr int OFF_SCAL = OFF_REC + 2 * 2 * Q * 16;         // float [2][8]
  static constexpr int OFF_MISC = OFF_SCAL + 2 * 8 * 4;
  static constexpr int BYTES = OFF_MISC + 64;
  static constexpr int SMEM = BYTES + 1024;  // slack for 1024-byte alignment
  // tensor memory columns
  static constexpr uint32_t TM_S = 0;
  static constexpr uint32_t TM_Y = 128;
  static constexpr uint32_t TM_H = 128 + P;
  static constexpr uint32_t TM_ST = (P == 64) ? TM_H : TM_H + N;  // P = 64: lanes 16-31 of H's columns
  static constexpr uint32_t TMEM_NEED = (P == 64) ? (TM_H + N) : (TM_ST + N);
  static constexpr uint32_t TMEM_COLS = TMEM_NEED <= 256 ? 256 : 512;
  static constexpr uint32_t ID_S = idesc_bf16(128, 128, false, false);
  static constexpr uint32_t ID_Y3 = idesc_bf16(128, P, false, false);
  static constexpr uint32_t ID_H = idesc_bf16(P, N, true, true);
  static constexpr uint32_t ID_Y2 = idesc_bf16(128, P, false, true);
  static constexpr int TX_B = kRows * N * 2;
  static constexpr int TX_X = Q * P * 2;
  static constexpr int NT = 256;  // threads that stage the B, C rows
};

// The decay inside a tile, e^{Lc_t - Lc_s}, is split around a pivot m (the middle of the
// tile's log-decay range) as a_t * b_s with a_t = e^{Lc_t - m}, b_s = e^{m - Lc_s}.  b_s and
// the trapezoid weight w_s = gamma_s + beta'_{s+1} go into X' = b_s w_s X, a_t is applied to
// the output rows, so the masked score matrix needs no exponentials: S' = S below the
// diagonal, S * gamma_s / w_s on it, 0 above.  The inter-chunk term e^{Lc_t} Ct h+ equals
// a_t Ct (e^m h+): the bf16 copy of the state is written pre-scaled by e^m, so that product
// accumulates into the same Y as S' X'.  The state update becomes H = X'^T Bt times the
// uniform factor e^{Le - m}.  When the range of Lc within a tile exceeds kFastRange the split
// could overflow fp32; such tiles take the exact path (m = 0, a_t = 1, b_s = 1, e^{Lc_t - Lc_s} per
// element, Ct rows scaled by e^{Lc_t} and Bt rows by e^{Le - Lc_t} in place).
// record A[t] = {Lc_t * log2 e, gamma_t / w_t, a_t, b_t w_t};  record B[t] = {e^{Lc_t},
// e^{Le - Lc_t}, 0, 0};  scalars {e^{Le}, Le, e^{Le - m} or 1, fast, e^m or 1, 0, 0, 0}

template <int R, int N, int P, int MODE>
__global__ void __launch_bounds__(kThreads, (P == 64 && N == 64) ? 2 : 1)
    scan_tc_kernel(const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmC,
                   const __grid_constant__ CUtensorMap tmX, const Params p, const SegInfo sg) {
  using C = Cfg<R, N, P, MODE>;
  constexpr bool FULL = C::FULL;
  constexpr int Q = C::Q;
  constexpr int K2 = C::K2;
  constexpr int NT = C::NT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = p.H, G = p.G;
  const int64_t L = p.L;
  // segment decomposition
  const int nseg_grid = FULL ? sg.nseg : sg.nsub;
  const int bh = blockIdx.x / nseg_grid;
  const int seg = blockIdx.x % nseg_grid;  // state pass: the sub-segment
  const int bi = bh / H, hi = bh % H;
  const int g = hi / (H / G);
  const int64_t ntiles_seq = (L + Q - 1) / Q;
  const int seg_len = FULL ? sg.seg_tiles : sg.sub_tiles;
  const int64_t j0 = (int64_t)seg * seg_len;
  const int64_t j1 = (j0 + seg_len < ntiles_seq) ? (j0 + seg_len) : ntiles_seq;
  const bool last_seg = (seg == sg.nseg - 1);
  const int64_t tok_base = (int64_t)bi * L;  // first token of this sequence (flattened b*L index)

  const uint32_t sBT = smem_u32(sm + C::OFF_BT), sCT = smem_u32(sm + C::OFF_CT);
  const uint32_t sX = smem_u32(sm + C::OFF_X), sH = smem_u32(sm + C::OFF_H);
  const uint32_t sXSTG = smem_u32(sm + C::OFF_XSTG);
  float2* csb = reinterpret_cast<float2*>(sm + C::OFF_CS);
  float* wx = reinterpret_cast<float*>(sm + C::OFF_WX);
  float* wo = reinterpret_cast<float*>(sm + C::OFF_WO);
  double* base = reinterpret_cast<double*>(sm + C::OFF_BASE);
  float* segsum = reinterpret_cast<float*>(sm + C::OFF_SEGSUM);
  float* raw = reinterpret_cast<float*>(sm + C::OFF_RAW);
  float4* recb = reinterpret_cast<float4*>(sm + C::OFF_REC);
  float* scalb = reinterpret_cast<float*>(sm + C::OFF_SCAL);
  uint64_t* mma_bar = reinterpret_cast<uint64_t*>(sm + C::OFF_MISC);
  uint64_t* load_bar = reinterpret_cast<uint64_t*>(sm + C::OFF_MISC + 8);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::OFF_MISC + 16);
  auto rawA = [&](int slot, int k) { return raw + (slot * 4 + k) * C::TOKF; };
  auto recA = [&](int slot) { return recb + (slot * 2) * Q; };
  auto recB = [&](int slot) { return recb + (slot * 2 + 1) * Q; };
  auto scal = [&](int slot) { return scalb + slot * 8; };
  auto cs = [&](int slot) { return csb + slot * Q * K2; };

  const __nv_bfloat16* xg = static_cast<const __nv_bfloat16*>(p.x);
  const __nv_bfloat16* Bg = static_cast<const __nv_bfloat16*>(p.B);
  __nv_bfloat16* yg = static_cast<__nv_bfloat16*>(p.y);
  const float Dh = (FULL && p.D) ? p.D[hi] : 0.0f;

  // ---- TMA loads of tile j (thread 0): x first (with the byte count of all), then B, C
  auto issue_x = [&](int64_t j) {
    const int tok = (int)(tok_base + j * Q);
    constexpr uint32_t tx = C::TX_B * (FULL ? 2 : 1) + C::TX_X;
    mbar_expect_tx(load_bar, tx);
    tma_load_3d(sXSTG, &tmX, 0, hi, tok, load_bar);
  };
  auto issue_bc = [&](int64_t j) {
    const int tok = (int)(tok_base + j * Q);
#pragma unroll
    for (int blk = 0; blk < N / 64; ++blk) {
      tma_load_4d(sBT + blk * (kRows * 128), &tmB, 64 * blk, 0, g, tok, load_bar);
      if constexpr (FULL) tma_load_4d(sCT + blk * (kRows * 128), &tmC, 64 * blk, 0, g, tok, load_bar);
    }
  };

  // ---- per-token coefficients and rotation angles, one tile ahead, through registers
  const int ak = tid % K2, aseg = tid / K2;
  float r_dt = 0.f, r_a = 0.f, r_lm = 0.f;
  float r_th[C::SEGLEN];
  auto load_coefs = [&](int64_t j) {
    const int64_t c0 = j * Q;
    if (tid < Q) {
      const int64_t t = c0 + tid;
      r_dt = r_a = r_lm = 0.0f;
      if (t < L) {
        const int64_t ti = (tok_base + t) * H + hi;
        r_dt = p.dt[ti];
        r_a = p.A[ti];
        r_lm = p.lam[ti];
      }
    } else if (tid == Q) {
      const int64_t t = c0 + Q;  // first token after the tile: its beta' weights the tile's last token
      r_dt = r_lm = 0.0f;
      if (t < L) {
        const int64_t ti = (tok_base + t) * H + hi;
        r_dt = p.dt[ti];
        r_lm = p.lam[ti];
      }
    }
#pragma unroll
    for (int e = 0; e < C::SEGLEN; ++e) {
      const int t = aseg * C::SEGLEN + e;
      r_th[e] = (t < Q && c0 + t < L) ? p.theta[((tok_base + c0 + t) * G + g) * K2 + ak] : 0.0f;
    }
  };
  auto store_coefs = [&](int slot) {
    if (tid < Q) {
      rawA(slot, 0)[tid] = r_dt;
      rawA(slot, 1)[tid] = r_a;
      rawA(slot, 2)[tid] = r_lm;
    } else if (tid == Q) {
      rawA(slot, 3)[0] = (1.0f - r_lm) * r_dt;
    }
  };
  // decay coefficients and per-token records of tile j into slot `slot` (warp 0; the raw
  // values of the tile must be in raw slot `slot`)
  auto coef_prep = [&](int64_t j, int slot) {
    const int nv = (int)((L - j * Q) < Q ? (L - j * Q) : Q);
    const float* dtA = rawA(slot, 0);
    const float* aA = rawA(slot, 1);
    const float* lmA = rawA(slot, 2);
    {
      constexpr int PER = (Q + 31) / 32;
      float loc[PER];
      float run = 0.0f;
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        const int t = lane * PER + e;
        run += (t < nv) ? dtA[t] * aA[t] : 0.0f;
        loc[e] = run;
      }
      float incl = run;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float nbv = __shfl_up_sync(kFull, incl, off);
        if (lane >= off) incl += nbv;
      }
      const float Le = __shfl_sync(kFull, incl, 31);
      const float excl = incl - run;
      float lmin = 0.0f, lmax = 0.0f;
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        loc[e] += excl;
        lmin = fminf(lmin, loc[e]);
        lmax = fmaxf(lmax, loc[e]);
      }
      // warp min / max in one redux each, on integer keys that order like the floats
      lmin = key_float(__reduce_min_sync(kFull, float_key(lmin)));
      lmax = key_float(__reduce_max_sync(kFull, float_key(lmax)));
      const bool fast = (lmax - lmin) <= kFastRange;
      const float m = fast ? 0.5f * (lmax + lmin) : 0.0f;
      const float bp_after = rawA(slot, 3)[0];
      float4* ra = recA(slot);
      float4* rb = recB(slot);
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        const int t = lane * PER + e;
        if (t < Q) {
          const float Lct = loc[e];
          const bool valid = t < nv;
          const float gm = valid ? lmA[t] * dtA[t] : 0.0f;
          const float bpn = (t + 1 < Q) ? ((t + 1 < nv) ? (1.0f - lmA[t + 1]) * dtA[t + 1] : 0.0f)
                                        : (valid ? bp_after : 0.0f);
          const float w = gm + bpn;
          const float dg = (w > 0.0f) ? __fdividef(gm, w) : 0.0f;
          const float at = fast ? __expf(Lct - m) : 1.0f;
          const float xs = fast ? __expf(m - Lct) * w : w;
          ra[t] = make_float4(Lct * 1.4426950408889634f, dg, at, xs);
          rb[t] = make_float4(__expf(Lct), __expf(Le - Lct), 0.0f, 0.0f);
        }
      }
      if (lane == 0) {
        float* sc = scal(slot);
        sc[0] = __expf(Le);
        sc[1] = Le;
        sc[2] = fast ? __expf(Le - m) : 1.0f;
        sc[3] = fast ? 1.0f : 0.0f;
        sc[4] = fast ? __expf(m) : 1.0f;
      }
    }
  };
  // rotation table of tile j into slot `slot` (all threads; the raw dt of the tile must be in
  // raw slot `slot` and its theta in r_th)
  auto angle_prep = [&](int64_t j, int slot) {
    const int nv = (int)((L - j * Q) < Q ? (L - j * Q) : Q);
    const float* dtA = rawA(slot, 0);
    float aloc[C::SEGLEN];
    {
      float run = 0.0f;
#pragma unroll
      for (int e = 0; e < C::SEGLEN; ++e) {
        const int t = aseg * C::SEGLEN + e;
        if (t < Q) run += (t < nv) ? (p.angle_direct ? r_th[e] : dtA[t] * r_th[e]) : 0.0f;
        aloc[e] = run;
      }
      segsum[aseg * K2 + ak] = run;
    }
    __syncthreads();
    double total = 0.0;
    {
      float aoff = 0.0f;
#pragma unroll
      for (int s = 0; s < C::SEGS; ++s)  // all loads issued together
        if (s < aseg) aoff += segsum[s * K2 + ak];
      if (aseg == 0) {
#pragma unroll
        for (int s = 0; s < C::SEGS; ++s) total += (double)segsum[s * K2 + ak];
      }
      aoff += (float)base[ak];
      float2* c2 = cs(slot);
#pragma unroll
      for (int e = 0; e < C::SEGLEN; ++e) {
        const int t = aseg * C::SEGLEN + e;
        if (t < Q) {
          float sn, cn;
          sincos_reduced(aoff + aloc[e], &sn, &cn);
          c2[t * K2 + ak] = make_float2(cn, sn);
        }
      }
    }
    __syncthreads();  // every thread has read base[] and segsum[]
    if (aseg == 0) {
      double nb = base[ak] + total;
      nb -= 6.283185307179586 * rint(nb * 0.15915494309189535);
      base[ak] = nb;
    }
  };

  // ---- setup
  if (warp == 0) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(mma_bar, 1);
    mbar_init(load_bar, 1);
    fence_mbar_init();
    if (j0 < j1) {  // the first tile's operands are in flight from the start
      issue_x(j0);
      issue_bc(j0);
    }
  }
  // every global load of the setup is issued before any of them is consumed
  constexpr int RPW = (R * P + kThreads - 1) / kThreads;
  float wxv[RPW], wov[RPW];
#pragma unroll
  for (int q = 0; q < RPW; ++q) {
    const int i = tid + q * kThreads;
    // branches p.R .. R-1 of the tile are zero padding: zero weights
    wxv[q] = i < p.R * P ? (p.W_x ? p.W_x[(int64_t)hi * p.R * P + i] : 1.0f) : 0.0f;
    wov[q] = i < p.R * P ? (p.W_o ? p.W_o[(int64_t)hi * p.R * P + i] : 1.0f) : 0.0f;
  }
  load_coefs(j0);
  const float* biasBg = p.bias_B ? p.bias_B + (int64_t)hi * p.R * N : nullptr;
  const float* biasCg = p.bias_C ? p.bias_C + (int64_t)hi * p.R * N : nullptr;
  // operand staging: B, C rows on all threads; x rows on warps 1-7 (warp 0 prepares the next
  // tile's coefficients meanwhile)
  const int xt = tid;
  constexpr int CHN = N / 8;
  constexpr int RPI = NT / CHN;  // rows per pass; a multiple of 8 and of R
  const int tch = xt % CHN;
  const int tr = (xt / CHN) % R;
  float bB[8], bC[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    bB[e] = (biasBg && tr < p.R) ? __ldg(biasBg + tr * N + tch * 8 + e) : 0.0f;
    bC[e] = (biasCg && tr < p.R) ? __ldg(biasCg + tr * N + tch * 8 + e) : 0.0f;
  }
#pragma unroll
  for (int q = 0; q < RPW; ++q) {
    const int i = tid + q * kThreads;
    if (i < R * P) {
      wx[i] = wxv[q];
      wo[i] = wov[q];
    }
  }
  for (int k = tid; k < K2; k += kThreads) base[k] = 0.0;
  store_coefs(0);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = __shfl_sync(kFull, *tmem_slot, 0);
  if (j0 < j1) {
    if (warp == 0) coef_prep(j0, 0);
    angle_prep(j0, 0);
  }
  if (j0 + 1 < j1) load_coefs(j0 + 1);

  // state warps: TMEM lane of accumulator row p (M = 128: lane = p; M = 64: rows in lanes
  // 0-15 of each quarter, and the state is kept in lanes 16-31 of the same columns)
  const int q4 = warp & 3;
  const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
  const bool state_warp = warp >= 4;
  const int prow = (P == 128) ? (32 * q4 + lane) : (16 * q4 + (lane & 15));
  const bool st_owner = (P == 128) || (lane >= 16);  // holds the fp32 state of row prow

  // ---- incoming rotated-frame state h+ of this segment
  //   nseg == 1 (full pass): h_{-1} + beta'_0 u_{-1} from the state / carry;
  //   state pass: zero (sub-segment 0 also writes the state's h+ to ws_init);
  //   full pass, segment k > 0: ws_init folded through the summaries of segments 0..k-1.
  // In the full pass every warp takes part (warp w: the TMEM lanes of quarter w & 3, half the
  // state columns), and the rotations of the folded segments come from a table that all
  // threads fill first (in the second rotation-table slot, unused until the first window).
  // segment seg of the full pass starts after sub-segments 0..nfold-1 of the state pass
  const int nfold = FULL ? seg * (sg.nseg > 1 ? sg.seg_tiles / sg.sub_tiles : 0) : 0;
  const bool fold_tab = FULL && sg.nseg > 1 && seg > 0 && nfold <= Q;
  float2* ftab = cs(1);
  if (fold_tab && j0 < j1) {
    for (int i = tid; i < nfold * K2; i += kThreads) {
      const int64_t sidx = (int64_t)bh * sg.nsub + i / K2;
      float sn, cn;
      sincosf((float)sg.ws_phi[sidx * K2 + i % K2], &sn, &cn);
      ftab[i] = make_float2(cn, sn);
    }
  }
  __syncthreads();
  const int c_lo = FULL ? (warp >> 2) * (N / 64) : 0;
  const int c_hi = FULL ? c_lo + N / 64 : N / 32;
  if ((FULL || state_warp) && j0 < j1) {
    const bool from_state = (sg.nseg == 1) || (!FULL && seg == 0 && sg.write_init);
    const float hscale = scal(0)[4];  // e^m of the first tile: the bf16 copy is pre-scaled
    float xprev[R];
    float bp0 = 0.0f;
    if (from_state) {
      bp0 = (1.0f - p.lam[tok_base * H + hi]) * p.dt[tok_base * H + hi];
#pragma unroll
      for (int r = 0; r < R; ++r) xprev[r] = wx[r * P + prow] * p.carry_x[(int64_t)bh * P + prow];
    }
    const float* h0 = p.h + (int64_t)bh * N * P;
    const float* cB = p.carry_B + (int64_t)bh * p.R * N;
#pragma unroll 1
    for (int c = c_lo; c < c_hi; ++c) {
      float v[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] = 0.0f;
      if (from_state) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int n = 32 * c + e;
          float u = 0.0f;
#pragma unroll
          for (int r = 0; r < R; ++r)
            if (r < p.R) u = fmaf(cB[r * N + n] + (biasBg ? __ldg(biasBg + r * N + n) : 0.0f), xprev[r], u);
          v[e] = fmaf(bp0, u, h0[(int64_t)n * P + prow]);
        }
        if (!FULL && sg.nseg > 1 && st_owner) {
          float* wi = sg.ws_init + (int64_t)bh * N * P;
#pragma unroll
          for (int e = 0; e < 32; ++e) wi[(int64_t)(32 * c + e) * P + prow] = v[e];
        }
        if constexpr (!FULL) {
          // the state pass summarises every sub-segment from a zero start; the incoming state
          // reaches later segments through the fold of ws_init in the full pass
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0.0f;
        }
      } else if (FULL) {
        const float* wi = sg.ws_init + (int64_t)bh * N * P;
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = wi[(int64_t)(32 * c + e) * P + prow];
        for (int k = 0; k < nfold; ++k) {
          const int64_t sidx = (int64_t)bh * sg.nsub + k;
          const float dec = __expf(sg.ws_l[sidx]);
          const float* wh = sg.ws_h + sidx * N * P;
          const double* ph = sg.ws_phi + sidx * K2;
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int n0 = 32 * c + 2 * e;
            float sn, cn;
            if (fold_tab) {
              const float2 t = ftab[k * K2 + n0 / 2];
              cn = t.x;
              sn = t.y;
            } else {
              sincosf((float)ph[n0 / 2], &sn, &cn);
            }
            const float a0 = fmaf(dec, v[2 * e], wh[(int64_t)n0 * P + prow]);
            const float a1 = fmaf(dec, v[2 * e + 1], wh[(int64_t)(n0 + 1) * P + prow]);
            v[2 * e] = cn * a0 - sn * a1;
            v[2 * e + 1] = sn * a0 + cn * a1;
          }
        }
      }
      uint32_t u32[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) u32[e] = __float_as_uint(v[e]);
      tmem_st32(tmem + lane_base + C::TM_ST + 32 * c, u32);
      if constexpr (FULL) {
        if (st_owner) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = hscale * v[8 * q + e];
            sts128(sH + sw128(prow, 4 * c + q, P * 128), pack8(f));
          }
        }
      }
    }
    tmem_wait_st();
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // state update ST <- e^{Le} ST + hs * H; with hnext > 0 also the bf16 copy hnext * ST
  auto state_update = [&](float Le_exp, float hs, float hnext) {
#pragma unroll 1
    for (int c = 0; c < N / 32; ++c) {
      uint32_t hv[32];
      float f[32];
      if constexpr (P == 64) {
        tmem_ld32(tmem + lane_base + C::TM_H + 32 * c, hv);  // lanes 0-15: H, lanes 16-31: state
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float hlow = __shfl_up_sync(kFull, __uint_as_float(hv[e]), 16);
          f[e] = (lane >= 16) ? fmaf(Le_exp, __uint_as_float(hv[e]), hs * hlow) : __uint_as_float(hv[e]);
          hv[e] = __float_as_uint(f[e]);
        }
        tmem_st32(tmem + lane_base + C::TM_ST + 32 * c, hv);
      } else {
        uint32_t sv[32];
        tmem_ld32(tmem + lane_base + C::TM_H + 32 * c, hv);
        tmem_ld32(tmem + lane_base + C::TM_ST + 32 * c, sv);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          f[e] = fmaf(Le_exp, __uint_as_float(sv[e]), hs * __uint_as_float(hv[e]));
          sv[e] = __float_as_uint(f[e]);
        }
        tmem_st32(tmem + lane_base + C::TM_ST + 32 * c, sv);
      }
      if (FULL && hnext > 0.0f && st_owner) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float f8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) f8[e] = hnext * f[8 * q + e];
          sts128(sH + sw128(prow, 4 * c + q, P * 128), pack8(f8));
        }
      }
    }
    tmem_wait_st();
  };

  // epilogue of tile j (warps 0-3): y_t = sum_r W_o[r] * a_t Y_{t,r} + D x_t
  auto epilogue = [&](int64_t j, int slot) {
    const int64_t c0 = j * Q;
    const int nv = (int)((L - c0) < Q ? (L - c0) : Q);
    const int i = 32 * q4 + lane;
    const int t = i / R, r = i % R;
    constexpr int W = 16 / R;
    const float at = recA(slot)[t].z;
    const int64_t yrow = ((tok_base + c0 + t) * H + hi) * P;
    const int c2_0 = (warp >> 2) * (P / 64);  // warps 0-3: columns [0, P/2); warps 4-7: [P/2, P)
#pragma unroll 1
    for (int c2 = c2_0; c2 < c2_0 + P / 64; ++c2) {
      uint32_t v2[32];  // two 16-column chunks per TMEM wait
      tmem_ld32(tmem + lane_base + C::TM_Y + 32 * c2, v2);
      tmem_wait_ld();
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int col0 = 32 * c2 + 16 * half;
        float f[16];
#pragma unroll
        for (int e4 = 0; e4 < 4; ++e4) {
          const float4 w4 = *reinterpret_cast<const float4*>(&wo[r * P + col0 + 4 * e4]);
          f[4 * e4] = (at * w4.x) * __uint_as_float(v2[16 * half + 4 * e4]);
          f[4 * e4 + 1] = (at * w4.y) * __uint_as_float(v2[16 * half + 4 * e4 + 1]);
          f[4 * e4 + 2] = (at * w4.z) * __uint_as_float(v2[16 * half + 4 * e4 + 2]);
          f[4 * e4 + 3] = (at * w4.w) * __uint_as_float(v2[16 * half + 4 * e4 + 3]);
        }
        // reduce over the R branches held by adjacent lanes: at each step a lane keeps the half of
        // its columns selected by one bit of r, moved to the front; lane r ends with columns
        // [r*W, r*W + W) of the sum in f[0..W)
#pragma unroll
        for (int m = R / 2, span = 8; m >= 1; m >>= 1, span >>= 1) {
          const bool upper = (r & m) != 0;
#pragma unroll
          for (int e = 0; e < span; ++e) {
            const float keep = upper ? f[e + span] : f[e];
            const float give = upper ? f[e] : f[e + span];
            f[e] = keep + __shfl_xor_sync(kFull, give, m);
          }
        }
        if (t < nv) {
          const int pc = col0 + r * W;
          if (p.D) {
#pragma unroll
            for (int e = 0; e < W; ++e) f[e] = fmaf(Dh, __bfloat162float(xg[yrow + pc + e]), f[e]);
          }
          if constexpr (W == 16) {
            uint4 o0 = make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]), pack_bf16(f[6], f[7]));
            uint4 o1 = make_uint4(pack_bf16(f[8], f[9]), pack_bf16(f[10], f[11]), pack_bf16(f[12], f[13]), pack_bf16(f[14], f[15]));
            *reinterpret_cast<uint4*>(yg + yrow + pc) = o0;
            *reinterpret_cast<uint4*>(yg + yrow + pc + 8) = o1;
          } else if constexpr (W == 8) {
            *reinterpret_cast<uint4*>(yg + yrow + pc) =
                make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]), pack_bf16(f[6], f[7]));
          } else if constexpr (W == 4) {
            *reinterpret_cast<uint2*>(yg + yrow + pc) = make_uint2(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]));
          } else {
            *reinterpret_cast<uint32_t*>(yg + yrow + pc) = pack_bf16(f[0], f[1]);
          }
        }
      }
    }
  };

  uint32_t mma_phase = 0, load_phase = 0;
  uint32_t y_phase = 0;    // barrier phase of the last MMA_B
  bool y_pending = false;  // a fast tile's MMA_B may still run: warps 0-3 wait before TM_Y / sX
  bool failed = false;
  float seg_logdec = 0.0f;
  for (int64_t j = j0; j < j1; ++j) {
    const int64_t c0 = j * Q;
    const int nv = (int)((L - c0) < Q ? (L - c0) : Q);
    const int par = (int)((j - j0) & 1);
    const bool has_next = j + 1 < j1;

    // ---- X (all warps): B, C rows of tile j; then, once MMA_B of tile j-1 is done, its
    //      epilogue (each warp: its TMEM lane quarter, half the columns); then the x rows of
    //      tile j (warps 1-7) and the coefficients of tile j+1 (warp 0)
    bool bad = false;
    if (has_next) store_coefs(par ^ 1);  // raw values of tile j+1 (loaded one window ago)
    bad = !mbar_wait(load_bar, load_phase);
    if (!bad) {
      {
        const bool fast = scal(par)[3] != 0.0f;
        const float2* csj = cs(par);
        const float4* rbj = recB(par);
        const int i0 = xt / CHN;
        const uint32_t off0 = (uint32_t)(tch >> 3) * (kRows * 128) + (uint32_t)i0 * 128u +
                              ((uint32_t)((tch & 7) ^ (i0 & 7)) << 4);  // i0 + k*RPI keeps i & 7
        // rows in groups of UG: all shared-memory loads of a group are issued before any store
        constexpr int NIT = kRows / RPI;
        constexpr int UG = NIT >= 2 ? 2 : 1;
#pragma unroll 1
        for (int it0 = 0; it0 < NIT; it0 += UG) {
          uint4 rb[UG], rc[UG];
          float4 w01[UG], w23[UG];
          int tt[UG];
          uint32_t offs[UG];
#pragma unroll
          for (int u = 0; u < UG; ++u) {
            const int i = i0 + (it0 + u) * RPI;
            tt[u] = i / R;
            offs[u] = off0 + (uint32_t)((it0 + u) * RPI) * 128u;
            const int tc = tt[u] < Q ? tt[u] : Q - 1;
            w01[u] = *reinterpret_cast<const float4*>(&csj[tc * K2 + tch * 4]);
            w23[u] = *reinterpret_cast<const float4*>(&csj[tc * K2 + tch * 4 + 2]);
            rb[u] = lds128(sBT + offs[u]);
            if constexpr (FULL) rc[u] = lds128(sCT + offs[u]);
          }
#pragma unroll
          for (int u = 0; u < UG; ++u) {
            const int t = tt[u];
            const bool valid = t < nv;
            const float wc[4] = {w01[u].x, w01[u].z, w23[u].x, w23[u].z};
            const float ws[4] = {w01[u].y, w01[u].w, w23[u].y, w23[u].w};
            if (!valid) {  // past the end of the sequence: zero rows
              sts128(sBT + offs[u], make_uint4(0, 0, 0, 0));
              if constexpr (FULL) sts128(sCT + offs[u], make_uint4(0, 0, 0, 0));
              continue;
            }
            {
              float f[8];
              unpack8(rb[u], f);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const float b0 = f[2 * q] + bB[2 * q], b1 = f[2 * q + 1] + bB[2 * q + 1];
                f[2 * q] = wc[q] * b0 + ws[q] * b1;  // Rot(-Phi)
                f[2 * q + 1] = wc[q] * b1 - ws[q] * b0;
              }
              if (!FULL && !fast) {  // state pass, exact tile: Bt rows * e^{Le - Lc_t}
                const float bsc = rbj[t].y;
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] *= bsc;
              }
              sts128(sBT + offs[u], pack8(f));
            }
            if constexpr (FULL) {
              float f[8];
              unpack8(rc[u], f);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const float d0 = f[2 * q] + bC[2 * q], d1 = f[2 * q + 1] + bC[2 * q + 1];
                f[2 * q] = wc[q] * d0 + ws[q] * d1;
                f[2 * q + 1] = wc[q] * d1 - ws[q] * d0;
              }
              sts128(sCT + offs[u], pack8(f));
            }
          }
        }
      }
    }
    if (FULL && y_pending && !bad) {
      bad = !mbar_wait(mma_bar, y_phase);
      tc_fence_after();
    }
    if (FULL && j > j0 && !bad) epilogue(j - 1, par ^ 1);
    // barrier 1: every thread has stored its raw values of tile j+1 and read the records of
    // tile j-1 (epilogue), whose slot coef_prep(j+1) overwrites; only warp 0 waits on it
    if (warp == 0) {
      named_bar_sync(1, kThreads);
      if (has_next) coef_prep(j + 1, par ^ 1);
    } else {
      named_bar_arrive(1, kThreads);
      if (!bad) {  // x rows on warps 1-7
        const float4* raj = recA(par);
        constexpr int CHP = P / 8;
        constexpr int NX = kThreads - 32;
        const int xi = tid - 32;
        const int xch = xi % CHP;  // fixed column chunk
        constexpr int TSTEP = NX / CHP;
        constexpr int XU = (Q / TSTEP) >= 2 ? 2 : 1;
#pragma unroll 1
        for (int t0 = xi / CHP; t0 < Q; t0 += XU * TSTEP) {
          uint4 xv[XU];
          float xsv[XU];
#pragma unroll
          for (int u = 0; u < XU; ++u) {
            const int t = t0 + u * TSTEP;
            const int tc = t < Q ? t : Q - 1;
            xv[u] = lds128(sXSTG + (uint32_t)(tc * P + xch * 8) * 2);
            xsv[u] = (t < nv) ? raj[tc].w : 0.0f;
          }
#pragma unroll
          for (int u = 0; u < XU; ++u) {
            const int t = t0 + u * TSTEP;
            if (t < Q) {
              float fx[8];
              unpack8(xv[u], fx);
#pragma unroll
              for (int e = 0; e < 8; ++e) fx[e] *= xsv[u];
#pragma unroll
              for (int rr = 0; rr < R; ++rr) {
                const int i = t * R + rr;
                const float4 w0 = *reinterpret_cast<const float4*>(&wx[rr * P + xch * 8]);
                const float4 w1 = *reinterpret_cast<const float4*>(&wx[rr * P + xch * 8 + 4]);
                const float xr[8] = {fx[0] * w0.x, fx[1] * w0.y, fx[2] * w0.z, fx[3] * w0.w,
                                     fx[4] * w1.x, fx[5] * w1.y, fx[6] * w1.z, fx[7] * w1.w};
                sts128(sX + sw128(i, xch, kRows * 128), pack8(xr));
              }
            }
          }
        }
      }
    }
    load_phase ^= 1;
    fence_async_smem();
    tc_fence_before();
    if (__syncthreads_or(bad)) {
      failed = true;
      break;
    }
    tc_fence_after();
    const bool fast = scal(par)[3] != 0.0f;
    if (tid == 0 && has_next) issue_x(j + 1);  // x staging is consumed

    // ---- MMA_A: S = Ct Bt^T; fast tiles also Y = Ct (e^m h+) and H = X'^T Bt
    if (warp == 0) {
      if constexpr (FULL) {
#pragma unroll
        for (int k = 0; k < N / 16; ++k) {
          const uint32_t koff = (uint32_t)(k >> 2) * (kRows * 128) + (uint32_t)(k & 3) * 32;
          mma_ss_w(tmem + C::TM_S, sdesc(sCT + koff, 16, 1024), sdesc(sBT + koff, 16, 1024), C::ID_S, k > 0);
        }
        if (fast) {
#pragma unroll
          for (int k = 0; k < N / 16; ++k) {
            const uint32_t aoff2 = (uint32_t)(k >> 2) * (kRows * 128) + (uint32_t)(k & 3) * 32;
            const uint32_t boff = (uint32_t)(k >> 2) * (P * 128) + (uint32_t)(k & 3) * 32;
            mma_ss_w(tmem + C::TM_Y, sdesc(sCT + aoff2, 16, 1024), sdesc(sH + boff, 16, 1024), C::ID_Y3, k > 0);
          }
        }
      }
      if (!FULL || fast) {
#pragma unroll
        for (int k = 0; k < kRows / 16; ++k)
          mma_ss_w(tmem + C::TM_H, sdesc(sX + k * 2048, kRows * 128, 1024), sdesc(sBT + k * 2048, kRows * 128, 1024),
                 C::ID_H, k > 0);
      }
      mma_commit_w(mma_bar);
    }
    // while the tensor cores run: next tile's coefficients and rotation table
    if (has_next) {
      angle_prep(j + 1, par ^ 1);
      if (j + 2 < j1) load_coefs(j + 2);
    }
    if (tid == 0 && !FULL) seg_logdec += scal(par)[1];
    {
      bool ok = true;
      if (tid == 0) ok = mbar_wait(mma_bar, mma_phase);
      mma_phase ^= 1;
      if (__syncthreads_or(!ok)) {
        failed = true;
        break;
      }
    }
    tc_fence_after();
    const float hnext = has_next ? scal(par ^ 1)[4] : 0.0f;  // bf16 state copy scale of tile j+1
    if (tid == 0 && has_next && (!FULL || fast)) issue_bc(j + 1);  // B (and C) are consumed

    // ---- D: mask S (warps 0-3) | state update or exact-tile rescaling (warps 4-7)
    if constexpr (FULL) {
      if (!state_warp) {
        const int i = 32 * warp + lane;
        const int t = i / R;
        const int t_lo = (32 * warp) / R, t_hi = (32 * warp + 31) / R;
        const float4* raj = recA(par);
        const float Lt2 = raj[t].x;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          const int s_lo = (32 * c) / R, s_hi = (32 * c + 31) / R;
          uint32_t o[16];
          if (s_lo > t_hi) {  // entirely above the diagonal
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] = 0u;
          } else {
            uint32_t v[32];
            tmem_ld32(tmem + lane_base + C::TM_S + 32 * c, v);
            tmem_wait_ld();
            if (fast && s_hi < t_lo) {  // entirely below the diagonal: S' = S
#pragma unroll
              for (int e = 0; e < 16; ++e) o[e] = pack_bf16(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
            } else {
              float f[32];
#pragma unroll
              for (int jj = 0; jj < 32 / R; ++jj) {
                const int s = s_lo + jj;
                const float4 rs = raj[s];
                float fac = (s < t) ? 1.0f : ((s == t) ? rs.y : 0.0f);
                if (!fast && s <= t) fac *= ex2_approx(Lt2 - rs.x);
#pragma unroll
                for (int rr = 0; rr < R; ++rr) f[jj * R + rr] = fac * __uint_as_float(v[jj * R + rr]);
              }
#pragma unroll
              for (int e = 0; e < 16; ++e) o[e] = pack_bf16(f[2 * e], f[2 * e + 1]);
            }
          }
          tmem_st16(tmem + lane_base + C::TM_S + 16 * c, o);
        }
        tmem_wait_st();
      } else if (fast) {
        state_update(scal(par)[0], scal(par)[2], hnext);
      } else {
        // exact tile: Ct rows * e^{Lc_t} and Bt rows * e^{Le - Lc_t}, in place (MMA1 has read them)
        const float4* rbj = recB(par);
        const int lt = tid - 128;
#pragma unroll 1
        for (int idx = lt; idx < kRows * CHN; idx += 128) {
          const int i = idx / CHN, ch = idx % CHN;
          const uint32_t off = sw128(i, ch, kRows * 128);
          const float4 rb = rbj[i / R];
          float f[8];
          unpack8(lds128(sBT + off), f);
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] *= rb.y;
          sts128(sBT + off, pack8(f));
          unpack8(lds128(sCT + off), f);
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] *= rb.x;
          sts128(sCT + off, pack8(f));
        }
      }
    } else {
      if (state_warp) state_update(scal(par)[0], scal(par)[2], 0.0f);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if constexpr (FULL) {
      // ---- MMA_B: [exact: Y = Ct' h+], Y += S' X', [exact: H = X'^T Bt']
      bool ok = true;
      if (warp == 0) {
        if (!fast) {
#pragma unroll
          for (int k = 0; k < N / 16; ++k) {
            const uint32_t aoff2 = (uint32_t)(k >> 2) * (kRows * 128) + (uint32_t)(k & 3) * 32;
            const uint32_t boff = (uint32_t)(k >> 2) * (P * 128) + (uint32_t)(k & 3) * 32;
            mma_ss_w(tmem + C::TM_Y, sdesc(sCT + aoff2, 16, 1024), sdesc(sH + boff, 16, 1024), C::ID_Y3, k > 0);
          }
        }
#pragma unroll
        for (int k = 0; k < kRows / 16; ++k)
          mma_ts_w(tmem + C::TM_Y, tmem + C::TM_S + 8 * k, sdesc(sX + k * 2048, kRows * 128, 1024), C::ID_Y2, 1);
        if (!fast) {
#pragma unroll
          for (int k = 0; k < kRows / 16; ++k)
            mma_ss_w(tmem + C::TM_H, sdesc(sX + k * 2048, kRows * 128, 1024),
                   sdesc(sBT + k * 2048, kRows * 128, 1024), C::ID_H, k > 0);
        }
        mma_commit_w(mma_bar);
        if (!fast && lane == 0) ok = mbar_wait(mma_bar, mma_phase);
      }
      y_phase = mma_phase;
      mma_phase ^= 1;
      // fast tile: MMA_B reads only TMEM S and sX, so warps 4-7 go on to the next tile's B, C
      // rows at once and warps 0-3 wait for it at the top of the next X phase
      y_pending = fast;
      if (!fast) {
        if (__syncthreads_or(!ok)) {
          failed = true;
          break;
        }
        tc_fence_after();
        if (tid == 0 && has_next) issue_bc(j + 1);
        if (state_warp) state_update(scal(par)[0], 1.0f, hnext);
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
      }
    }
  }
  if constexpr (FULL) {
    if (!failed && j0 < j1) {
      bool ok = true;
      if (y_pending) {
        ok = mbar_wait(mma_bar, y_phase);
        tc_fence_after();
      }
      if (ok)
        epilogue(j1 - 1, (int)((j1 - 1 - j0) & 1));
      else
        set_status(p.status, M3_ERR_TIMEOUT);
    }
  }

  // ---- results
  if (!failed && j0 < j1) {
    if constexpr (FULL) {
      if (last_seg) {
        // final state: rotate the segment-frame state back by the segment's total angle
        if (state_warp) {
          float* hout = p.h + (int64_t)bh * N * P;
#pragma unroll 1
          for (int c = 0; c < N / 32; ++c) {
            uint32_t sv[32];
            tmem_ld32(tmem + lane_base + C::TM_ST + 32 * c, sv);
            tmem_wait_ld();
            if (st_owner) {
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const int k = 16 * c + e;
                float sn, cn;
                sincosf((float)base[k], &sn, &cn);
                const float a0 = __uint_as_float(sv[2 * e]), a1 = __uint_as_float(sv[2 * e + 1]);
                hout[(int64_t)(2 * k) * P + prow] = cn * a0 - sn * a1;
                hout[(int64_t)(2 * k + 1) * P + prow] = sn * a0 + cn * a1;
              }
            }
          }
        } else {
          const int64_t tokl = tok_base + (L - 1);
          const int64_t bc = ((tokl * G + g) * p.R) * (int64_t)N;
          for (int i = tid; i < p.R * N; i += 128) p.carry_B[(int64_t)bh * p.R * N + i] = __bfloat162float(Bg[bc + i]);
          const int64_t xr = (tokl * H + hi) * (int64_t)P;
          for (int i = tid; i < P; i += 128) p.carry_x[(int64_t)bh * P + i] = __bfloat162float(xg[xr + i]);
        }
      }
    } else {
      // segment summary: end state (segment frame, zero start), total log decay, total angle
      const int64_t sidx = (int64_t)bh * sg.nsub + seg;
      if (state_warp) {
        float* wh = sg.ws_h + sidx * N * P;
#pragma unroll 1
        for (int c = 0; c < N / 32; ++c) {
          uint32_t sv[32];
          tmem_ld32(tmem + lane_base + C::TM_ST + 32 * c, sv);
          tmem_wait_ld();
          if (st_owner) {
#pragma unroll
            for (int e = 0; e < 32; ++e) wh[(int64_t)(32 * c + e) * P + prow] = __uint_as_float(sv[e]);
          }
        }
      }
      if (tid == 0) sg.ws_l[sidx] = seg_logdec;
      for (int k = tid; k < K2; k += kThreads) sg.ws_phi[sidx * K2 + k] = base[k];
    }
  }
  if (failed && tid == 0) set_status(p.status, M3_ERR_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  // the driver entry point is the same for every device; it is looked up once, under the
  // once-flag, so concurrent first calls neither race nor repeat the query
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

bool make_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const cuuint64_t* dims,
              const cuuint64_t* strides, const cuuint32_t* box, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return fn(m, dt, (cuuint32_t)rank, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            sw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Maps {
  CUtensorMap B, C, X;
};

// B and C tiles of Q tokens x RT branches: with RT above the operands' rank p.R the branch rows
// past p.R lie outside the tensor and the copy fills them with zeros.
bool make_maps(const Params& p, int Q, int RT, Maps* m) {
  const cuuint64_t toks = (cuuint64_t)(p.b * p.L);
  {
    const cuuint64_t dims[4] = {(cuuint64_t)p.N, (cuuint64_t)p.R, (cuuint64_t)p.G, toks};
    const cuuint64_t str[3] = {(cuuint64_t)p.N * 2, (cuuint64_t)p.R * p.N * 2, (cuuint64_t)p.G * p.R * p.N * 2};
    const cuuint32_t box[4] = {64, (cuuint32_t)RT, 1, (cuuint32_t)Q};
    if (!make_map(&m->B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, p.B, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return false;
    if (!make_map(&m->C, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, p.C, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return false;
  }
  {
    const cuuint64_t dims[3] = {(cuuint64_t)p.P, (cuuint64_t)p.H, toks};
    const cuuint64_t str[2] = {(cuuint64_t)p.P * 2, (cuuint64_t)p.H * p.P * 2};
    const cuuint32_t box[3] = {(cuuint32_t)p.P, 1, (cuuint32_t)Q};
    if (!make_map(&m->X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, p.x, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
      return false;
  }
  return true;
}

template <int R, int N, int P>
constexpr int ctas_per_sm() {
  return (P == 64 && N == 64) ? 2 : 1;
}

template <int R, int N, int P, int MODE>
cudaError_t launch_mode(const Maps& m, const Params& p, const SegInfo& sg, unsigned grid, cudaStream_t stream) {
  using Cf = Cfg<R, N, P, MODE>;
  auto k = scan_tc_kernel<R, N, P, MODE>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::SMEM);
  if (e != cudaSuccess) return e;
  k<<<grid, kThreads, Cf::SMEM, stream>>>(m.B, m.C, m.X, p, sg);
  return cudaGetLastError();
}

// Number of segments per sequence: enough CTAs to fill the SMs, at least 2 tiles each.
int plan_segments(int64_t nseq, int64_t ntiles, int per_sm) {
  int dev = 0, nsm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int64_t slots = (int64_t)nsm * per_sm;
  int64_t nseg = nseq >= slots ? 1 : slots / nseq;
  const int64_t maxseg = ntiles / 2;
  if (nseg > maxseg) nseg = maxseg;
  if (nseg < 1) nseg = 1;
  if (nseg > 64) nseg = 64;
  return (int)nseg;
}

// Sub-segments of the state pass: segments 0..nseg-2 are cut into m equal parts (m divides
// seg_tiles), as many as the free CTA slots allow, so that the state pass, which only has to
// produce each part's summary, runs in parallel too.
int plan_subsegments(int64_t nseq, int nseg, int seg_tiles, int per_sm) {
  int dev = 0, nsm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (nseg <= 1) return 1;
  const int64_t slots = (int64_t)nsm * per_sm;
  int64_t m = slots / (nseq * (nseg - 1));
  if (m > seg_tiles) m = seg_tiles;
  while (m > 1 && seg_tiles % m != 0) --m;
  return m < 1 ? 1 : (int)m;
}

struct SegPlan {
  int nseg, seg_tiles, nsub, sub_tiles;
};

template <int R, int N, int P>
size_t ws_bytes_for(const Params& p, SegPlan* out) {
  constexpr int Q = kRows / R;
  const int64_t ntiles = (p.L + Q - 1) / Q;
  const int64_t nseq = p.b * p.H;
  const int nseg = plan_segments(nseq, ntiles, ctas_per_sm<R, N, P>());
  const int seg_tiles = (int)((ntiles + nseg - 1) / nseg);
  const int nseg_eff = (int)((ntiles + seg_tiles - 1) / seg_tiles);
  const int m = plan_subsegments(nseq, nseg_eff, seg_tiles, ctas_per_sm<R, N, P>());
  if (out) *out = SegPlan{nseg_eff, seg_tiles, (nseg_eff - 1) * m, seg_tiles / m};
  if (nseg_eff <= 1) return 0;
  const size_t np = (size_t)N * P;
  const size_t s1 = (size_t)(nseg_eff - 1) * m;
  size_t bytes = 0;
  bytes += 4 * (size_t)nseq * np;                       // ws_init
  bytes += 4 * (size_t)nseq * s1 * np;                  // ws_h
  bytes = (bytes + 4 * (size_t)nseq * s1 + 255) & ~(size_t)255;   // ws_l, then align
  bytes += 8 * (size_t)nseq * s1 * (N / 2);             // ws_phi
  return bytes;
}

}  // namespace
bool ws_scan_supported(const Params& p);
cudaError_t launch_scan_ws(const CUtensorMap& tmB, const CUtensorMap& tmC, const CUtensorMap& tmX, const Params& p,
                           const SegInfo& sg, cudaStream_t stream);
cudaError_t launch_scan_ws_state(const CUtensorMap& tmB, const CUtensorMap& tmC, const CUtensorMap& tmX,
                                 const Params& p, const SegInfo& sg, cudaStream_t stream);
namespace {

// Summary of a whole range (sequence sharding): the state pass over every tile of the range,
// cut into sub-segments that fill the SMs, each summarised from a zero start.
template <int R, int N, int P>
SegInfo summary_plan(const Params& p) {
  constexpr int Q = kRows / R;
  int dev = 0, nsm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int64_t nseq = p.b * p.H;
  const int64_t ntiles = (p.L + Q - 1) / Q;
  const int64_t slots = (int64_t)nsm * ctas_per_sm<R, N, P>();
  int64_t m = slots / (nseq > 0 ? nseq : 1);
  if (m > ntiles / 2) m = ntiles / 2;  // at least two tiles per sub-segment
  if (m > 256) m = 256;
  if (m < 1) m = 1;
  SegInfo sg{};
  sg.sub_tiles = (int)((ntiles + m - 1) / m);
  sg.nsub = (int)((ntiles + sg.sub_tiles - 1) / sg.sub_tiles);
  sg.nseg = 2;  // the state pass reads only the sub-segment fields
  sg.seg_tiles = sg.nsub * sg.sub_tiles;
  sg.write_init = 0;
  return sg;
}

template <int R, int N, int P>
size_t summary_ws_for(const Params& p, SegInfo* sg) {
  *sg = summary_plan<R, N, P>(p);
  const size_t nseq = (size_t)(p.b * p.H), ns = (size_t)sg->nsub;
  size_t bytes = 4 * nseq * ns * (size_t)N * P;
  bytes = (bytes + 4 * nseq * ns + 255) & ~(size_t)255;
  return bytes + 8 * nseq * ns * (N / 2);
}

template <int R, int N, int P>
cudaError_t launch_summary_cfg(const Params& p, void* ws, size_t ws_bytes, SegInfo* sg_out, cudaStream_t stream) {
  constexpr int Q = kRows / R;
  SegInfo sg;
  const size_t need = summary_ws_for<R, N, P>(p, &sg);
  if (ws == nullptr || ws_bytes < need) return cudaErrorInvalidValue;
  const size_t nseq = (size_t)(p.b * p.H), ns = (size_t)sg.nsub;
  char* w = static_cast<char*>(ws);
  sg.ws_init = nullptr;
  sg.ws_h = reinterpret_cast<float*>(w);
  sg.ws_l = sg.ws_h + nseq * ns * N * P;
  sg.ws_phi = reinterpret_cast<double*>(w + ((4 * nseq * ns * (size_t)N * P + 4 * nseq * ns + 255) & ~(size_t)255));
  *sg_out = sg;
  Maps m;
  if (!make_maps(p, Q, R, &m)) return cudaErrorInvalidValue;
  if (ws_scan_supported(p)) return launch_scan_ws_state(m.B, m.C, m.X, p, sg, stream);
  return launch_mode<R, N, P, MODE_STATE>(m, p, sg, (unsigned)(nseq * ns), stream);
}

template <int R, int N, int P>
cudaError_t launch_cfg(const Params& p, void* ws, size_t ws_bytes, cudaStream_t stream) {
  constexpr int Q = kRows / R;
  SegPlan plan;
  const size_t need = ws_bytes_for<R, N, P>(p, &plan);
  if (need > ws_bytes || (need > 0 && ws == nullptr)) return cudaErrorInvalidValue;
  Maps m;
  if (!make_maps(p, Q, R, &m)) return cudaErrorInvalidValue;
  SegInfo sg;
  sg.nseg = plan.nseg;
  sg.seg_tiles = plan.seg_tiles;
  sg.nsub = plan.nsub;
  sg.sub_tiles = plan.sub_tiles;
  sg.ws_init = sg.ws_h = sg.ws_l = nullptr;
  sg.ws_phi = nullptr;
  sg.write_init = 1;
  const int64_t nseq = p.b * p.H;
  const int nseg = plan.nseg;
  if (nseg > 1) {
    const size_t np = (size_t)N * P;
    const size_t s1 = (size_t)plan.nsub;
    char* w = static_cast<char*>(ws);
    sg.ws_init = reinterpret_cast<float*>(w);
    sg.ws_h = sg.ws_init + (size_t)nseq * np;
    sg.ws_l = sg.ws_h + (size_t)nseq * s1 * np;
    size_t off = (4 * ((size_t)nseq * np + (size_t)nseq * s1 * np + (size_t)nseq * s1) + 255) & ~(size_t)255;
    sg.ws_phi = reinterpret_cast<double*>(w + off);
  }
  // headdim 128 with a rank the warp-specialised kernel covers: that kernel, same plan
  if (ws_scan_supported(p)) return launch_scan_ws(m.B, m.C, m.X, p, sg, stream);
  if (nseg > 1) {
    cudaError_t e = launch_mode<R, N, P, MODE_STATE>(m, p, sg, (unsigned)(nseq * plan.nsub), stream);
    if (e != cudaSuccess) return e;
  }
  return launch_mode<R, N, P, MODE_FULL>(m, p, sg, (unsigned)(nseq * nseg), stream);
}

template <int R, int N, int P>
constexpr bool fits() {
  return Cfg<R, N, P, MODE_FULL>::SMEM <= 227 * 1024;
}

template <int R>
cudaError_t launch_r(const Params& p, void* ws, size_t wsb, cudaStream_t s) {
  if (p.N == 64 && p.P == 64) return launch_cfg<R, 64, 64>(p, ws, wsb, s);
  if (p.N == 64 && p.P == 128) return launch_cfg<R, 64, 128>(p, ws, wsb, s);
  if (p.N == 128 && p.P == 64) return launch_cfg<R, 128, 64>(p, ws, wsb, s);
  return launch_cfg<R, 128, 128>(p, ws, wsb, s);
}

template <int R>
size_t ws_r(const Params& p) {
  if (p.N == 64 && p.P == 64) return ws_bytes_for<R, 64, 64>(p, nullptr);
  if (p.N == 64 && p.P == 128) return ws_bytes_for<R, 64, 128>(p, nullptr);
  if (p.N == 128 && p.P == 64) return ws_bytes_for<R, 128, 64>(p, nullptr);
  return ws_bytes_for<R, 128, 128>(p, nullptr);
}

template <int R>
bool fits_r(const Params& p) {
  if (p.N == 64 && p.P == 64) return fits<R, 64, 64>();
  if (p.N == 64 && p.P == 128) return fits<R, 64, 128>();
  if (p.N == 128 && p.P == 64) return fits<R, 128, 64>();
  return fits<R, 128, 128>();
}

template <int R>
size_t summary_ws_r(const Params& p) {
  SegInfo sg;
  if (p.N == 64 && p.P == 64) return summary_ws_for<R, 64, 64>(p, &sg);
  if (p.N == 64 && p.P == 128) return summary_ws_for<R, 64, 128>(p, &sg);
  if (p.N == 128 && p.P == 64) return summary_ws_for<R, 128, 64>(p, &sg);
  return summary_ws_for<R, 128, 128>(p, &sg);
}

template <int R>
cudaError_t launch_summary_r(const Params& p, void* ws, size_t wsb, SegInfo* sg, cudaStream_t s) {
  if (p.N == 64 && p.P == 64) return launch_summary_cfg<R, 64, 64>(p, ws, wsb, sg, s);
  if (p.N == 64 && p.P == 128) return launch_summary_cfg<R, 64, 128>(p, ws, wsb, sg, s);
  if (p.N == 128 && p.P == 64) return launch_summary_cfg<R, 128, 64>(p, ws, wsb, sg, s);
  return launch_summary_cfg<R, 128, 128>(p, ws, wsb, sg, s);
}

}  // namespace

size_t scan_summary_workspace_bytes(const Params& p) {
  switch (tile_rank(p.R)) {
    case 1: return summary_ws_r<1>(p);
    case 2: return summary_ws_r<2>(p);
    case 4: return summary_ws_r<4>(p);
    default: return summary_ws_r<8>(p);
  }
}

cudaError_t launch_scan_summary_pass(const Params& p, void* ws, size_t ws_bytes, SegInfo* sg, cudaStream_t stream) {
  switch (tile_rank(p.R)) {
    case 1: return launch_summary_r<1>(p, ws, ws_bytes, sg, stream);
    case 2: return launch_summary_r<2>(p, ws, ws_bytes, sg, stream);
    case 4: return launch_summary_r<4>(p, ws, ws_bytes, sg, stream);
    default: return launch_summary_r<8>(p, ws, ws_bytes, sg, stream);
  }
}

bool tc_scan_supported(const Params& p) {
  if (p.dtype != M3_BF16) return false;
  if (!((p.N == 64 || p.N == 128) && (p.P == 64 || p.P == 128))) return false;
  if (p.b * p.L > 0x7fffffffLL) return false;  // TMA token coordinate is 32-bit
  if (p.R < 1 || p.R > 8) return false;
  switch (tile_rank(p.R)) {  // ranks 3, 5, 6, 7 run padded to the next tile rank
    case 1: return fits_r<1>(p);
    case 2: return fits_r<2>(p);
    case 4: return fits_r<4>(p);
    default: return fits_r<8>(p);
  }
}

size_t tc_scan_workspace_bytes(const Params& p) {
  switch (tile_rank(p.R)) {
    case 1: return ws_r<1>(p);
    case 2: return ws_r<2>(p);
    case 4: return ws_r<4>(p);
    default: return ws_r<8>(p);
  }
}

cudaError_t launch_scan_tc(const Params& p, void* ws, size_t ws_bytes, cudaStream_t stream) {
  switch (tile_rank(p.R)) {
    case 1: return launch_r<1>(p, ws, ws_bytes, stream);
    case 2: return launch_r<2>(p, ws, ws_bytes, stream);
    case 4: return launch_r<4>(p, ws, ws_bytes, stream);
    default: return launch_r<8>(p, ws, ws_bytes, stream);
  }
}

}  // namespace m3
