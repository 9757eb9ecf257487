// m3_scan_tc.cu -- chunked Mamba-3 prefill scan on the sm_100a tensor cores (tcgen05 + TMEM).
//
// One CTA walks one (batch, head) sequence in tiles of Q = 128 / R tokens, so that a
// tile has exactly 128 rows i = t * R + r (token t, MIMO branch r) -- the M of one
// tcgen05.mma.  The chunked form is exact (the IBM Mamba page, SSD section: a
// selective scan can be cut into chunks whose results combine associatively), so
// the tile length does not change the result; for R = 4 it is the model's chunk of 32.
//
// Per tile, with Lc_t the tile-local cumulative sum of dt A (log decay) and Phi_t the
// cumulative rotation angle from the sequence start (kept per pair in fp64, reduced
// mod 2 pi, so that fp32 angles stay small):
//   Bt_i = Rot(-Phi_t)(B_{t,r} + bias_B),  Ct_i = Rot(-Phi_t)(C_{t,r} + bias_C)
//     -- the rotation absorbed into B and C as a data-dependent RoPE (Mamba-3 paper
//        note, docsaid.org, section その2, statement 2);
//   S  = Ct Bt^T                                     (MMA1, 128 x 128, K = N)
//   S'[i,j] = S[i,j] e^{Lc_t - Lc_s} (gamma_s + [s<t] beta'_{s+1}) for s <= t, else 0
//     -- the trapezoid weights of section その1 (gamma = lam dt, beta' = (1-lam) dt):
//        the input of token s enters h_s with gamma_s and h_{s+1} with beta'_{s+1};
//   Y  = (e^{Lc_t} Ct) h+  +  S' X                    (MMA3 + MMA2, K = N and K = 128)
//     with X_i = W_x[r] * x_t (MIMO branches, section その3), h+ the rotated-frame
//     state entering the tile (plus the trapezoid carry of its last token);
//   h+ <- e^{Lc_e} h+ + Xs^T Bt,  Xs_i = e^{Lc_e - Lc_t} (gamma_t + beta'_{t+1}) X_i
//                                                     (MMA4, state update, K = 128)
//   y_t = sum_r W_o[r] * Y_{t,r} + D x_t.
// Working in the rotated frame (Bt, Ct carry the rotation) leaves the state a
// plain decay-and-add; it is rotated back once at the end of the sequence.
//
// Data layout on chip: Bt, Ct, e^{Lc}Ct, X, Xs and the bf16 copy of h+ are bf16
// tiles in shared memory in the 128-byte-swizzled canonical UMMA layouts; the
// accumulators S, Y, H = Xs^T Bt and the fp32 state h+ live in tensor memory
// (columns 0, 128, 256, 384).  S is masked in place and consumed from TMEM as the
// A operand of MMA2 (bf16 packed two per column).
//
// Warp roles per tile: all 8 warps stage the tiles; thread 0 issues the MMAs and
// commits them to an mbarrier; warps 0-3 mask S while warps 4-7 update the state;
// all 8 warps run the epilogue (two column halves of Y).  Every mbarrier wait is
// bounded by %globaltimer; a timeout sets M3_ERR_TIMEOUT and the CTA releases its
// TMEM and returns.
#include "m3_common.cuh"

namespace m3 {
namespace {

constexpr int kThreads = 256;
constexpr int kRows = 128;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t TM_S = 0, TM_Y = 128, TM_H = 256, TM_ST = 384;
constexpr unsigned kFull = 0xffffffffu;
constexpr unsigned long long kWaitNs = 2000000000ull;  // 2 s bound on any mbarrier wait

// ------------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
               "r"(ncols));
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}
// Bounded wait: false after kWaitNs without the phase completing.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > kWaitNs) return false;
  }
  return true;
}

// D[tmem] (+)= A[smem] * B[smem]
__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
// D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d),
      "r"(a), "l"(b), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]),
        "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]),
        "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
      "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
      "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31]));
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::
          "r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 descriptor version 1).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: bf16 x bf16 -> fp32, dense.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ void unpack8(const uint4& w, float (&f)[8]) {
  f[0] = bf_lo(w.x); f[1] = bf_hi(w.x); f[2] = bf_lo(w.y); f[3] = bf_hi(w.y);
  f[4] = bf_lo(w.z); f[5] = bf_hi(w.z); f[6] = bf_lo(w.w); f[7] = bf_hi(w.w);
}
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  return make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]), pack_bf16(f[6], f[7]));
}
__device__ __forceinline__ void sts128(uint32_t addr, const uint4& v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// Byte offset of 16-byte chunk `ch` of row `row` in a 128B-swizzled tile whose rows are
// 128 bytes per 64-element block and whose blocks are `block_bytes` apart.
__device__ __forceinline__ uint32_t sw128(int row, int ch, uint32_t block_bytes) {
  return (uint32_t)(ch >> 3) * block_bytes + (uint32_t)row * 128u + ((uint32_t)((ch & 7) ^ (row & 7)) << 4);
}

// ------------------------------------------------------------------ configuration

template <int R, int N, int P>
struct Cfg {
  static constexpr int Q = kRows / R;  // tokens per tile
  static constexpr int K2 = N / 2;     // rotation pairs
  static constexpr int TILE_N = kRows * N * 2;
  static constexpr int TILE_P = kRows * P * 2;
  static constexpr int TILE_H = P * N * 2;
  static constexpr int OFF_BT = 0;
  static constexpr int OFF_CT = OFF_BT + TILE_N;
  static constexpr int OFF_C2 = OFF_CT + TILE_N;
  static constexpr int OFF_X = OFF_C2 + TILE_N;
  static constexpr int OFF_XS = OFF_X + TILE_P;
  static constexpr int OFF_H = OFF_XS + TILE_P;
  static constexpr int OFF_CS = OFF_H + TILE_H;  // float2 [Q][K2]
  static constexpr int OFF_BIASB = OFF_CS + Q * K2 * 8;
  static constexpr int OFF_BIASC = OFF_BIASB + R * N * 4;
  static constexpr int OFF_WX = OFF_BIASC + R * N * 4;
  static constexpr int OFF_WO = OFF_WX + R * P * 4;
  static constexpr int OFF_BASE = OFF_WO + R * P * 4;  // double [K2]
  static constexpr int TOKF = Q + 4;                    // floats per per-token array
  static constexpr int OFF_TOK = OFF_BASE + K2 * 8;     // 8 arrays of TOKF floats
  static constexpr int OFF_MISC = OFF_TOK + 8 * TOKF * 4;
  static constexpr int BYTES = OFF_MISC + 64;
  static constexpr int SMEM = BYTES + 1024;  // slack for 1024-byte alignment
  static constexpr int SEGS = kThreads / K2;  // angle prefix: segments per pair
  static constexpr int SEGLEN = (Q + SEGS - 1) / SEGS;
  static constexpr uint32_t ID_S = idesc_bf16(128, 128, false, false);
  static constexpr uint32_t ID_Y3 = idesc_bf16(128, P, false, false);
  static constexpr uint32_t ID_H = idesc_bf16(P, N, true, true);
  static constexpr uint32_t ID_Y2 = idesc_bf16(128, P, false, true);
};

// per-token array slots
enum { T_LA = 0, T_GAM = 1, T_BP = 2, T_LC = 3, T_DEC = 4, T_CW = 5, T_DT = 6, T_SCAL = 7 };

template <int R, int N, int P>
__global__ void __launch_bounds__(kThreads, 1) scan_tc_kernel(Params p) {
  using C = Cfg<R, N, P>;
  constexpr int Q = C::Q;
  constexpr int K2 = C::K2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = p.H, G = p.G;
  const int64_t L = p.L;
  const int bh = blockIdx.x;
  const int bi = bh / H, hi = bh % H;
  const int g = hi / (H / G);

  const uint32_t sBT = smem_u32(sm + C::OFF_BT), sCT = smem_u32(sm + C::OFF_CT), sC2 = smem_u32(sm + C::OFF_C2);
  const uint32_t sX = smem_u32(sm + C::OFF_X), sXS = smem_u32(sm + C::OFF_XS), sH = smem_u32(sm + C::OFF_H);
  float2* cs = reinterpret_cast<float2*>(sm + C::OFF_CS);
  float* biasB = reinterpret_cast<float*>(sm + C::OFF_BIASB);
  float* biasC = reinterpret_cast<float*>(sm + C::OFF_BIASC);
  float* wx = reinterpret_cast<float*>(sm + C::OFF_WX);
  float* wo = reinterpret_cast<float*>(sm + C::OFF_WO);
  double* base = reinterpret_cast<double*>(sm + C::OFF_BASE);
  float* tokf = reinterpret_cast<float*>(sm + C::OFF_TOK);
  float* la = tokf + T_LA * C::TOKF;
  float* gam = tokf + T_GAM * C::TOKF;
  float* bpv = tokf + T_BP * C::TOKF;
  float* Lc = tokf + T_LC * C::TOKF;
  float* dec0 = tokf + T_DEC * C::TOKF;
  float* cw = tokf + T_CW * C::TOKF;
  float* dtv = tokf + T_DT * C::TOKF;
  float* scal = tokf + T_SCAL * C::TOKF;  // [0] = e^{Lc_e}
  uint64_t* mbar = reinterpret_cast<uint64_t*>(sm + C::OFF_MISC);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::OFF_MISC + 8);

  const __nv_bfloat16* xg = static_cast<const __nv_bfloat16*>(p.x);
  const __nv_bfloat16* Bg = static_cast<const __nv_bfloat16*>(p.B);
  const __nv_bfloat16* Cg = static_cast<const __nv_bfloat16*>(p.C);
  __nv_bfloat16* yg = static_cast<__nv_bfloat16*>(p.y);
  const float Dh = p.D ? p.D[hi] : 0.0f;

  // ---- setup
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) mbar_init(mbar, 1);
  for (int i = tid; i < R * N; i += kThreads) {
    biasB[i] = p.bias_B ? p.bias_B[(int64_t)hi * R * N + i] : 0.0f;
    biasC[i] = p.bias_C ? p.bias_C[(int64_t)hi * R * N + i] : 0.0f;
  }
  for (int i = tid; i < R * P; i += kThreads) {
    wx[i] = p.W_x ? p.W_x[(int64_t)hi * R * P + i] : 1.0f;
    wo[i] = p.W_o ? p.W_o[(int64_t)hi * R * P + i] : 1.0f;
  }
  for (int k = tid; k < K2; k += kThreads) base[k] = 0.0;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // state warps: lanes of the P-row accumulators (M = 128: p = lane quarter * 32 + lane;
  // M = 64: rows 16 per quarter in lanes 0-15)
  const int q4 = warp & 3;
  const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
  const int prow = (P == 128) ? (32 * q4 + lane) : (16 * q4 + lane);
  const bool pvalid = (P == 128) || (lane < 16);
  const bool state_warp = warp >= 4;

  // ---- initial rotated-frame state h+ = h_{-1} + beta'_0 u_{-1} (angle 0 at the start)
  if (state_warp) {
    const int64_t tok0 = (int64_t)bi * L;
    const float bp0 = (1.0f - p.lam[tok0 * H + hi]) * p.dt[tok0 * H + hi];
    float xprev[R];
#pragma unroll
    for (int r = 0; r < R; ++r)
      xprev[r] = pvalid ? wx[r * P + prow] * p.carry_x[(int64_t)bh * P + prow] : 0.0f;
    const float* h0 = p.h + (int64_t)bh * N * P;
    const float* cB = p.carry_B + (int64_t)bh * R * N;
#pragma unroll 1
    for (int c = 0; c < N / 32; ++c) {
      uint32_t v[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int n = 32 * c + e;
        float u = 0.0f;
#pragma unroll
        for (int r = 0; r < R; ++r) u = fmaf(cB[r * N + n] + biasB[r * N + n], xprev[r], u);
        const float hv = pvalid ? fmaf(bp0, u, h0[(int64_t)n * P + prow]) : 0.0f;
        v[e] = __float_as_uint(hv);
      }
      tmem_st32(tmem + lane_base + TM_ST + 32 * c, v);
      if (pvalid) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(v[8 * q + e]);
          sts128(sH + sw128(prow, 4 * c + q, P * 128), pack8(f));
        }
      }
    }
    tmem_wait_st();
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  uint32_t phase = 0;
  bool failed = false;
  const int64_t ntiles = (L + Q - 1) / Q;
  for (int64_t j = 0; j < ntiles; ++j) {
    const int64_t c0 = j * Q;
    const int nv = (int)((L - c0) < Q ? (L - c0) : Q);

    // ---- A1: per-token coefficients (invalid tail tokens are identity steps)
    if (tid < Q) {
      const int t = tid;
      if (t < nv) {
        const int64_t ti = ((int64_t)bi * L + c0 + t) * H + hi;
        const float d = p.dt[ti], lm = p.lam[ti];
        la[t] = d * p.A[ti];
        gam[t] = lm * d;
        bpv[t] = (1.0f - lm) * d;
        dtv[t] = d;
      } else {
        la[t] = 0.0f;
        gam[t] = 0.0f;
        bpv[t] = 0.0f;
        dtv[t] = 0.0f;
      }
    } else if (tid == Q) {
      float nb = 0.0f;
      if (c0 + Q < L) {
        const int64_t ti = ((int64_t)bi * L + c0 + Q) * H + hi;
        nb = (1.0f - p.lam[ti]) * p.dt[ti];
      }
      bpv[Q] = nb;
    }
    __syncthreads();

    // ---- A2: cumulative log decay (warp 0) and angle partial sums (all threads)
    if (warp == 0) {
      constexpr int PER = (Q + 31) / 32;
      float loc[PER];
      float run = 0.0f;
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        const int t = lane * PER + e;
        run += (t < Q) ? la[t] : 0.0f;
        loc[e] = run;
      }
      float incl = run;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float nbv = __shfl_up_sync(kFull, incl, off);
        if (lane >= off) incl += nbv;
      }
      const float excl = incl - run;
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        const int t = lane * PER + e;
        if (t < Q) Lc[t] = excl + loc[e];
      }
      __syncwarp();
      const float Le = Lc[Q - 1];
      for (int t = lane; t < Q; t += 32) {
        dec0[t] = __expf(Lc[t]);
        cw[t] = __expf(Le - Lc[t]) * (gam[t] + bpv[t + 1]);
      }
      if (lane == 0) scal[0] = __expf(Le);
    }
    const int ak = tid % K2, aseg = tid / K2;
    {
      float run = 0.0f;
      const float* th = p.theta + (((int64_t)bi * L + c0) * G + g) * K2 + ak;
      for (int e = 0; e < C::SEGLEN; ++e) {
        const int t = aseg * C::SEGLEN + e;
        if (t < Q) {
          run += (t < nv) ? dtv[t] * th[(int64_t)t * G * K2] : 0.0f;
          cs[t * K2 + ak].x = run;
        }
      }
    }
    __syncthreads();
    float aoff = (float)base[ak];
    double total = 0.0;
    for (int s = 0; s < C::SEGS; ++s) {
      const int tend = ((s + 1) * C::SEGLEN < Q ? (s + 1) * C::SEGLEN : Q) - 1;
      if (s * C::SEGLEN < Q) {
        const float segsum = cs[tend * K2 + ak].x;
        if (s < aseg) aoff += segsum;
        total += (double)segsum;
      }
    }
    __syncthreads();
    for (int e = 0; e < C::SEGLEN; ++e) {
      const int t = aseg * C::SEGLEN + e;
      if (t < Q) {
        float sn, cn;
        sincosf(aoff + cs[t * K2 + ak].x, &sn, &cn);
        cs[t * K2 + ak] = make_float2(cn, sn);
      }
    }
    if (aseg == 0) {
      double nbse = base[ak] + total;
      nbse -= 6.283185307179586 * rint(nbse * 0.15915494309189535);
      base[ak] = nbse;
    }
    __syncthreads();

    // ---- B: stage the bf16 operand tiles (rows i = t * R + r)
    {
      constexpr int CHN = N / 8;
      for (int idx = tid; idx < kRows * CHN; idx += kThreads) {
        const int i = idx / CHN, ch = idx % CHN;
        const int t = i / R, r = i % R;
        uint4 ob = make_uint4(0, 0, 0, 0), oc = ob, oc2 = ob;
        if (t < nv) {
          const int64_t row = ((((int64_t)bi * L + c0 + t) * G + g) * R + r) * N + ch * 8;
          float fb[8], fc[8];
          unpack8(__ldg(reinterpret_cast<const uint4*>(Bg + row)), fb);
          unpack8(__ldg(reinterpret_cast<const uint4*>(Cg + row)), fc);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            fb[e] += biasB[r * N + ch * 8 + e];
            fc[e] += biasC[r * N + ch * 8 + e];
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 w = cs[t * K2 + ch * 4 + q];  // (cos Phi, sin Phi); apply Rot(-Phi)
            const float b0 = fb[2 * q], b1 = fb[2 * q + 1], d0 = fc[2 * q], d1 = fc[2 * q + 1];
            fb[2 * q] = w.x * b0 + w.y * b1;
            fb[2 * q + 1] = w.x * b1 - w.y * b0;
            fc[2 * q] = w.x * d0 + w.y * d1;
            fc[2 * q + 1] = w.x * d1 - w.y * d0;
          }
          ob = pack8(fb);
          oc = pack8(fc);
          const float dd = dec0[t];
#pragma unroll
          for (int e = 0; e < 8; ++e) fc[e] *= dd;
          oc2 = pack8(fc);
        }
        const uint32_t off = sw128(i, ch, kRows * 128);
        sts128(sBT + off, ob);
        sts128(sCT + off, oc);
        sts128(sC2 + off, oc2);
      }
      constexpr int CHP = P / 8;
      for (int idx = tid; idx < kRows * CHP; idx += kThreads) {
        const int i = idx / CHP, ch = idx % CHP;
        const int t = i / R, r = i % R;
        uint4 ox = make_uint4(0, 0, 0, 0), oxs = ox;
        if (t < nv) {
          const int64_t row = (((int64_t)bi * L + c0 + t) * H + hi) * P + ch * 8;
          float fx[8];
          unpack8(__ldg(reinterpret_cast<const uint4*>(xg + row)), fx);
#pragma unroll
          for (int e = 0; e < 8; ++e) fx[e] *= wx[r * P + ch * 8 + e];
          ox = pack8(fx);
          const float cwt = cw[t];
#pragma unroll
          for (int e = 0; e < 8; ++e) fx[e] *= cwt;
          oxs = pack8(fx);
        }
        const uint32_t off = sw128(i, ch, kRows * 128);
        sts128(sX + off, ox);
        sts128(sXS + off, oxs);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- C: MMA1 (S), MMA3 (Y = e^{Lc} Ct h+), MMA4 (H = Xs^T Bt)
    if (tid == 0) {
#pragma unroll
      for (int k = 0; k < N / 16; ++k) {
        const uint32_t koff = (uint32_t)(k >> 2) * (kRows * 128) + (uint32_t)(k & 3) * 32;
        mma_ss(tmem + TM_S, sdesc(sCT + koff, 16, 1024), sdesc(sBT + koff, 16, 1024), C::ID_S, k > 0);
      }
#pragma unroll
      for (int k = 0; k < N / 16; ++k) {
        const uint32_t aoff2 = (uint32_t)(k >> 2) * (kRows * 128) + (uint32_t)(k & 3) * 32;
        const uint32_t boff = (uint32_t)(k >> 2) * (P * 128) + (uint32_t)(k & 3) * 32;
        mma_ss(tmem + TM_Y, sdesc(sC2 + aoff2, 16, 1024), sdesc(sH + boff, 16, 1024), C::ID_Y3, k > 0);
      }
#pragma unroll
      for (int k = 0; k < kRows / 16; ++k) {
        mma_ss(tmem + TM_H, sdesc(sXS + k * 2048, kRows * 128, 1024), sdesc(sBT + k * 2048, kRows * 128, 1024),
               C::ID_H, k > 0);
      }
      mma_commit(mbar);
    }
    {
      const bool ok = mbar_wait(mbar, phase);
      phase ^= 1;
      if (__syncthreads_or(!ok)) {
        failed = true;
        break;
      }
    }
    tc_fence_after();

    // ---- D: mask S in TMEM (warps 0-3) | state update (warps 4-7)
    if (!state_warp) {
      const int i = 32 * warp + lane;
      const int t = i / R;
      const int t_hi = (32 * warp + 31) / R;
      const float Lt = Lc[t];
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[16];
        if ((32 * c) / R > t_hi) {
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] = 0u;
        } else {
          uint32_t v[32];
          tmem_ld32(tmem + lane_base + TM_S + 32 * c, v);
          tmem_wait_ld();
          float f[32];
#pragma unroll
          for (int jj = 0; jj < 32 / R; ++jj) {
            const int s = (32 * c) / R + jj;
            float fac = 0.0f;
            if (s <= t) fac = __expf(Lt - Lc[s]) * (gam[s] + (s < t ? bpv[s + 1] : 0.0f));
#pragma unroll
            for (int rr = 0; rr < R; ++rr) f[jj * R + rr] = fac * __uint_as_float(v[jj * R + rr]);
          }
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] = pack_bf16(f[2 * e], f[2 * e + 1]);
        }
        tmem_st16(tmem + lane_base + TM_S + 16 * c, o);
      }
      tmem_wait_st();
    } else {
      const float Le = scal[0];
#pragma unroll 1
      for (int c = 0; c < N / 32; ++c) {
        uint32_t hv[32], sv[32];
        tmem_ld32(tmem + lane_base + TM_H + 32 * c, hv);
        tmem_ld32(tmem + lane_base + TM_ST + 32 * c, sv);
        tmem_wait_ld();
        float f[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          f[e] = fmaf(Le, __uint_as_float(sv[e]), __uint_as_float(hv[e]));
          sv[e] = __float_as_uint(f[e]);
        }
        tmem_st32(tmem + lane_base + TM_ST + 32 * c, sv);
        if (pvalid) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float f8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f8[e] = f[8 * q + e];
            sts128(sH + sw128(prow, 4 * c + q, P * 128), pack8(f8));
          }
        }
      }
      tmem_wait_st();
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- E: MMA2 (Y += S' X), S' read from TMEM
    if (tid == 0) {
#pragma unroll
      for (int k = 0; k < kRows / 16; ++k)
        mma_ts(tmem + TM_Y, tmem + TM_S + 8 * k, sdesc(sX + k * 2048, kRows * 128, 1024), C::ID_Y2, 1);
      mma_commit(mbar);
    }
    {
      const bool ok = mbar_wait(mbar, phase);
      phase ^= 1;
      if (__syncthreads_or(!ok)) {
        failed = true;
        break;
      }
    }
    tc_fence_after();

    // ---- F: epilogue y_t = sum_r W_o[r] * Y_{t,r} + D x_t (all 8 warps, two column halves)
    {
      const int i = 32 * q4 + lane;
      const int t = i / R, r = i % R;
      const int half = warp >> 2;
      constexpr int PH = P / 2;
      constexpr int W = 16 / R;
      const int64_t yrow = (((int64_t)bi * L + c0 + t) * H + hi) * P;
#pragma unroll 1
      for (int c = 0; c < PH / 16; ++c) {
        const int col0 = half * PH + 16 * c;
        uint32_t v[16];
        tmem_ld16(tmem + lane_base + TM_Y + col0, v);
        tmem_wait_ld();
        float f[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) f[e] = wo[r * P + col0 + e] * __uint_as_float(v[e]);
#pragma unroll
        for (int m = 1; m < R; m <<= 1) {
#pragma unroll
          for (int e = 0; e < 16; ++e) f[e] += __shfl_xor_sync(kFull, f[e], m);
        }
        if (t < nv) {
          float outv[W];
#pragma unroll
          for (int e = 0; e < W; ++e) {
            float sel = f[e];
#pragma unroll
            for (int rr = 1; rr < R; ++rr)
              if (rr == r) sel = f[rr * W + e];
            outv[e] = sel;
          }
          const int pc = col0 + r * W;
          if (p.D) {
#pragma unroll
            for (int e = 0; e < W; ++e) outv[e] = fmaf(Dh, __bfloat162float(xg[yrow + pc + e]), outv[e]);
          }
#pragma unroll
          for (int e = 0; e < W; e += 2)
            *reinterpret_cast<uint32_t*>(yg + yrow + pc + e) = pack_bf16(outv[e], outv[e + 1]);
        }
      }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }

  // ---- final state: rotate the rotated-frame state back by the total angle; carry
  if (!failed) {
    if (state_warp) {
      float* hout = p.h + (int64_t)bh * N * P;
#pragma unroll 1
      for (int c = 0; c < N / 32; ++c) {
        uint32_t sv[32];
        tmem_ld32(tmem + lane_base + TM_ST + 32 * c, sv);
        tmem_wait_ld();
        if (pvalid) {
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
      const int64_t tokl = (int64_t)bi * L + (L - 1);
      const int64_t bc = ((tokl * G + g) * R) * (int64_t)N;
      for (int i = tid; i < R * N; i += 128) p.carry_B[(int64_t)bh * R * N + i] = __bfloat162float(Bg[bc + i]);
      const int64_t xr = (tokl * H + hi) * (int64_t)P;
      for (int i = tid; i < P; i += 128) p.carry_x[(int64_t)bh * P + i] = __bfloat162float(xg[xr + i]);
    }
  } else if (tid == 0) {
    set_status(p.status, M3_ERR_TIMEOUT);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int R, int N, int P>
cudaError_t launch_cfg(const Params& p, cudaStream_t stream) {
  using Cf = Cfg<R, N, P>;
  auto k = scan_tc_kernel<R, N, P>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::SMEM);
  if (e != cudaSuccess) return e;
  k<<<(unsigned)(p.b * p.H), kThreads, Cf::SMEM, stream>>>(p);
  return cudaGetLastError();
}

template <int R>
cudaError_t launch_r(const Params& p, cudaStream_t stream) {
  if (p.N == 64 && p.P == 64) return launch_cfg<R, 64, 64>(p, stream);
  if (p.N == 64 && p.P == 128) return launch_cfg<R, 64, 128>(p, stream);
  if (p.N == 128 && p.P == 64) return launch_cfg<R, 128, 64>(p, stream);
  return launch_cfg<R, 128, 128>(p, stream);
}

template <int R, int N, int P>
constexpr bool fits() {
  return Cfg<R, N, P>::SMEM <= 227 * 1024;
}

}  // namespace

bool tc_scan_supported(const Params& p) {
  if (p.dtype != M3_BF16) return false;
  if (!((p.N == 64 || p.N == 128) && (p.P == 64 || p.P == 128))) return false;
  switch (p.R) {
    case 1:
      return p.N == 64 ? (p.P == 64 ? fits<1, 64, 64>() : fits<1, 64, 128>())
                       : (p.P == 64 ? fits<1, 128, 64>() : fits<1, 128, 128>());
    case 2:
      return p.N == 64 ? (p.P == 64 ? fits<2, 64, 64>() : fits<2, 64, 128>())
                       : (p.P == 64 ? fits<2, 128, 64>() : fits<2, 128, 128>());
    case 4:
      return p.N == 64 ? (p.P == 64 ? fits<4, 64, 64>() : fits<4, 64, 128>())
                       : (p.P == 64 ? fits<4, 128, 64>() : fits<4, 128, 128>());
    case 8:
      return p.N == 64 ? (p.P == 64 ? fits<8, 64, 64>() : fits<8, 64, 128>())
                       : (p.P == 64 ? fits<8, 128, 64>() : fits<8, 128, 128>());
    default:
      return false;
  }
}

cudaError_t launch_scan_tc(const Params& p, cudaStream_t stream) {
  switch (p.R) {
    case 1: return launch_r<1>(p, stream);
    case 2: return launch_r<2>(p, stream);
    case 4: return launch_r<4>(p, stream);
    default: return launch_r<8>(p, stream);
  }
}

}  // namespace m3
