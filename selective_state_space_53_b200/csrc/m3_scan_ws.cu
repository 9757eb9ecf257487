// m3_scan_ws.cu -- warp-specialised chunked Mamba-3 prefill on the sm_100a tensor cores, for
// headdim P = 128 (the 1.5B-scale layer: d_state 128, MIMO rank 4).
//
// The chunk algebra is that of the other tensor-core scan (m3_scan_tc.cu): tiles of
// Q = 128 / R tokens, rows i = t R + r (token t, MIMO branch r), the rotation absorbed into B
// and C in a rotated frame (Mamba-3 paper note, docsaid.org, section その2, statement 2), the
// trapezoid weights gamma_s = lam_s dt_s and beta'_{s+1} = (1 - lam_{s+1}) dt_{s+1} (section
// その1) and the per-branch scales of the MIMO inputs and readouts (section その3).  The
// chunked form is exact (IBM Mamba page, SSD section), so the tile length does not change the
// result.  What differs is the layout of the products and the schedule.
//
// Transposed products.  With Lc_t the tile-local cumulative log decay and m a pivot in the
// middle of its range, a_t = e^{Lc_t - m}, b_s = e^{m - Lc_s}, w_s = gamma_s + beta'_{s+1}:
//   Ct_i = Rot(-Phi_t)(C_{t,r} + bias_C),   Bt_i = Rot(-Phi_t)(B_{t,r} + bias_B)
//   S   = Ct Bt^T                        (M = 128 rows i, N = 128 columns j, K = d_state)
//   S'  = S below the diagonal, S gamma/w on it, 0 above (masking only)
//   X'_s = b_s w_s W_x[r] x_t            (the column factor of the decay, per input row)
//   Y^T = hb^T Ct^T + X'^T S'^T          (M = P rows p, N = 128 columns i)
//   y_t[p] = a_t sum_r W_o[r,p] Y^T[p, tR + r] (+ D x_t[p])   (the row factor, in the epilogue)
//   ST <- ST + X'^T Bt                   (M = P, N = d_state, K = 128), ST pre-scaled by e^m
// with hb = bf16(e^m h+) the state entering the tile: the decay e^{Lc_t - Lc_s} w_s of the
// intra-chunk term is a_t b_s w_s, split between the input rows and the output columns, so the
// rotated operands carry no per-row factor.  The output has the head dimension p on the
// tensor-memory lanes, so the combine over r is a sum inside one thread; the uniform factor
// e^{Le - m} is applied once per tile to the state.  Tiles whose log-decay range exceeds 64 take
// an exact form instead: no pivot (X'_s = w_s W_x x_t, a_t = 1), the mask applies
// e^{Lc_t - Lc_s} per element, and after S has read them the rows of Ct and Bt are rescaled in
// place by e^{Lc_t} and e^{Le - Lc_t} for the inter-chunk and state products.  With the range at
// most 64 every factor a_t, b_s, e^{m}, e^{Le - m} lies within e^{+-32}.
//
// Warp roles, one warpgroup each (24 warps; every wait is an mbarrier wait that sleeps in the
// instruction, bounded by %globaltimer):
//   0      producer: TMA loads of the B and C tiles into two shared-memory stages, and of x
//   1      MMA issue (one elected lane): S, H, Y_inter, Y_intra; tensor-memory allocation
//   2      coefficients: decay cumsum, pivot, per-token scales, state scale factors
//   3      idle
//   4-11   rotation: cumulative angles and their sin/cos table; Bt, Ct rotated in place
//   12-15  mask: S from tensor memory -> S' (bf16, shared memory)
//   16-19  epilogue: Y^T from tensor memory -> y
//          (in the state pass, with N = 128 and plain inputs, warps 12-19 rotate B while warps 4-11
//          build the next tile's angle table)
//   20-23  state and inputs: the state rescale and its bf16 copy hb; X'^T into tensor memory
// The block is launched with 80 registers a thread; the control warpgroup gives some back and
// the rotation warpgroups take them (setmaxnreg), since the rotation holds the most live values.
// The tile pipeline per tile j (MMA order): H(j), Y_inter(j), Y_intra(j), S(j+1).  Each SIMT
// task has two MMAs' time between the commit that releases it and the MMA that needs it:
// state rescale SP(j+1) after Y_inter(j), before H(j+1); epilogue E(j) after Y_intra(j), before
// Y_inter(j+1); mask M(j+1) after S(j+1), before Y_intra(j+1); X'^T is double-buffered.
//
// Sequence splitting follows the shared segment plan (m3_scan_plan.cuh): a state pass
// (MODE 1: rotation of B only, X', H and the state rescale) summarises segments 0..nseg-2 from a
// zero start; the full pass starts each segment from the folded summaries.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cuda_fp16.h>

#include "m3_common.cuh"
#include "m3_ptx.cuh"
#include "m3_scan_plan.cuh"

namespace m3 {
namespace {

constexpr int WP = 128;  // head dim of this kernel
constexpr int W_PROD = 0, W_MMA = 1, W_COEF = 2, W_ROT = 4, N_ROT = 8, W_MASK = 12, W_EPI = 16, W_SPX = 20;
constexpr int WS_WARPS = 24;
constexpr int WS_THREADS = WS_WARPS * 32;
// registers a thread: at launch, and per warpgroup after the reallocation
constexpr int WS_REG_LAUNCH = 80, WS_REG_CTRL = 48, WS_REG_ROT = 96;
static_assert(128 * (WS_REG_CTRL + 2 * WS_REG_ROT + 3 * WS_REG_LAUNCH) <= WS_THREADS * WS_REG_LAUNCH,
              "the warpgroups' registers after setmaxnreg must fit the launch's total");
constexpr uint32_t WS_SLEEP_NS = 1000000;          // suspend-time hint of a wait (1 ms)
constexpr int WS_CS = 4;                          // coefficient record slots
constexpr float WS_FAST_RANGE = 64.0f;            // largest log-decay range of a pivot-split tile
constexpr unsigned long long WS_WAIT_NS = 2000000000ull;  // 2 s bound on any wait
constexpr int WS_FULL = 0, WS_STATE = 1;
constexpr uint32_t BAR_ROT = 1;                   // named barrier of the rotation warps
constexpr uint32_t BAR_SPX = 2;                   // named barrier of the state warps
constexpr uint32_t BAR_RH = 3;                    // rotation warps and their helpers (state pass)
constexpr int N_HELP = 8;                         // helper warps: the mask and epilogue groups

// barrier indices
enum {
  B_BCF = 0,    // [2] B/C tile of a stage landed (TMA bytes)
  B_BCE = 2,    // [2] stage free (MMA commit)
  B_CF = 4,     // [CS] coefficient records written
  B_CE = 8,     // [CS] coefficient records consumed
  B_ROT = 12,   // [2] Bt', Ct' of a stage rotated
  B_RESC = 14,  // exact tile: Bt', Ct' rescaled after S
  B_SF = 15,    // S in tensor memory (MMA commit)
  B_SPF = 16,   // S' in shared memory (mask warps)
  B_HF = 17,    // hb and the rescaled state ready (state warps)
  B_SPGO = 18,  // H and Y_inter done: state and hb may be rewritten (MMA commit)
  B_XPF = 19,   // [2] X'^T buffer written (state warps)
  B_XBF = 21,   // [2] X'^T buffer free (MMA commit)
  B_YF = 23,    // Y^T complete (MMA commit)
  B_YE = 24,    // Y^T read (epilogue warps)
  B_DRAIN = 25, // all MMAs complete (end of kernel)
  B_FIN = 26,   // final angles published (rotation warps)
  B_XF = 27,    // x of a tile landed (TMA bytes)
  B_XE = 28,    // the x slot consumed (state warps)
  NBAR = 29
};
static_assert(B_CE - B_CF == WS_CS && B_ROT - B_CE == WS_CS, "one pair of barriers per coefficient record slot");

template <int R, int N>
struct WsCfg {
  static constexpr int Q = 128 / R;
  static constexpr int K2 = N / 2;
  static constexpr int NKC = N / 8;                    // 16-byte chunks of a row
  static constexpr int KCW = NKC / N_ROT;              // chunks per rotation warp
  static constexpr int TILE_N = 128 * N * 2;           // a B or C tile, bytes
  static constexpr int BLK = 128 * 128;                // one 64-column block of a 128-row SW128 tile
  static constexpr int STAGE = 2 * TILE_N;             // B then C
  static constexpr int OFF_STAGE = 0;
  static constexpr int OFF_SP = OFF_STAGE + 2 * STAGE;           // S', 128 x 128 bf16
  static constexpr int OFF_HB = OFF_SP + 128 * 128 * 2;          // hb, 128 (p) x N bf16
  static constexpr int TAB_ROW = K2 * 4 + 16;                    // (cos, sin) of one token in bf16, padded
  static constexpr int OFF_TAB = OFF_HB + WP * N * 2;
  static constexpr int XSLOT = Q * WP * 2;                       // x of one tile, (token, p) bf16
  static constexpr int OFF_X = OFF_TAB + Q * TAB_ROW;            // one slot, TMA destination
  static constexpr int BIAS_ROW = NKC * 8 + 4;                   // floats of one (operand, branch) bias row, padded
  static constexpr int OFF_BIAS = OFF_X + XSLOT;                 // float [2][R][BIAS_ROW], staged pair layout
  static constexpr int SEGS = 256 / K2;                          // angle prefix segments
  static constexpr int SEGLEN = Q / SEGS;
  static constexpr int OFF_SEGSUM = OFF_BIAS + 2 * R * BIAS_ROW * 4;  // float [SEGS][K2]
  static constexpr int OFF_BASE = OFF_SEGSUM + SEGS * K2 * 4;    // double [K2]
  static constexpr int REC_SLOT = Q * 24 + 64;  // float4 rec[Q], float mult[Q], float ycol[Q], float scal[16]
  static constexpr int OFF_REC = OFF_BASE + K2 * 8;
  static constexpr int OFF_ROWSS = OFF_REC + WS_CS * REC_SLOT;    // float [2][128]: B, C row sums of squares
  static constexpr int OFF_BAR = OFF_ROWSS + 2 * 128 * 4;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int SMEM = BYTES + 1024;
  static constexpr uint32_t TM_S = 0, TM_Y = 128, TM_ST = 256, TM_XP = 256 + N;  // X'^T: two 64-column buffers
  static constexpr uint32_t TM_COLS = 512;
  static constexpr uint32_t ID_S = idesc_bf16(128, 128, false, false);
  static constexpr uint32_t ID_Y = idesc_bf16(WP, 128, false, false);
  static constexpr uint32_t ID_H = idesc_bf16(WP, N, false, true);
  static_assert(Q % SEGS == 0 && SEGLEN >= 1, "angle segments");
  static_assert(NKC % N_ROT == 0, "rotation chunks");
  static_assert(TM_XP + 128 <= TM_COLS, "tensor memory");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ bool ws_try(uint64_t* bar, uint32_t parity) {
  return mbar_try_wait_sleep(bar, parity, WS_SLEEP_NS);
}

// Wait for the phase of `parity` to complete; false (and the abort flag set) after WS_WAIT_NS,
// or false at once when another role has already aborted.
__device__ __forceinline__ bool ws_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (ws_try(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (!ws_try(bar, parity)) {
    if (*abort_flag) return false;
    if (globaltimer() - t0 > WS_WAIT_NS) {
      *abort_flag = 1;
      return false;
    }
  }
  return true;
}
// Wait bounded by time only (used to drain copies and MMAs in flight before the CTA exits).
__device__ __forceinline__ bool ws_wait_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!ws_try(bar, parity)) {
    if (globaltimer() - t0 > WS_WAIT_NS) return false;
  }
  return true;
}
// Phase bits of a set of barriers in one register: bit k is the parity the next wait on
// barrier k expects.
struct Phases {
  uint32_t bits = 0;
  __device__ __forceinline__ uint32_t operator[](int k) const { return (bits >> k) & 1u; }
  __device__ __forceinline__ void flip(int k) { bits ^= 1u << k; }
};

// Named barrier that also ORs a predicate over the participating threads: every thread gets
// the same answer, so a group decides together whether to stop.
__device__ __forceinline__ bool bar_any(uint32_t id, uint32_t nthreads, bool pred) {
  uint32_t out;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(out)
      : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
      : "memory");
  return out != 0;
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// cos, sin and -sin of the four rotation pairs k0..k0+3 of a 16-byte chunk, as f32x2 pairs
// (k0, k0+1) and (k0+2, k0+3), from the table's half-precision words (c_k0, c_k0+1),
// (s_k0, s_k0+1), (c_k0+2, c_k0+3), (s_k0+2, s_k0+3).
struct RotCS {
  uint64_t c01, s01, n01, c23, s23, n23;
};
__device__ __forceinline__ RotCS rot_cs(const uint4& w) {
  const float2 c01 = __half22float2(*reinterpret_cast<const __half2*>(&w.x));
  const float2 s01 = __half22float2(*reinterpret_cast<const __half2*>(&w.y));
  const float2 c23 = __half22float2(*reinterpret_cast<const __half2*>(&w.z));
  const float2 s23 = __half22float2(*reinterpret_cast<const __half2*>(&w.w));
  return {f2(c01.x, c01.y), f2(s01.x, s01.y), f2(-s01.x, -s01.y),
          f2(c23.x, c23.y), f2(s23.x, s23.y), f2(-s23.x, -s23.y)};
}
// Rot(-Phi)(n v + bias) on the 8 values of one 16-byte chunk (pair q in word q: first element in
// the low half), in fp32.  The first elements of two pairs share an f32x2 lane pair and the second
// elements another, so the rotation is four packed products per two pairs.  The bias comes in the
// same layout: be01 = (b0, b2), bo01 = (b1, b3), be23 = (b4, b6), bo23 = (b5, b7).
__device__ __forceinline__ uint4 rotate16(const uint4& raw, const RotCS& r, uint64_t n2, uint64_t be01,
                                          uint64_t bo01, uint64_t be23, uint64_t bo23) {
  const uint64_t v0a = f2_fma(n2, f2(bf_lo(raw.x), bf_lo(raw.y)), be01);
  const uint64_t v1a = f2_fma(n2, f2(bf_hi(raw.x), bf_hi(raw.y)), bo01);
  const uint64_t v0b = f2_fma(n2, f2(bf_lo(raw.z), bf_lo(raw.w)), be23);
  const uint64_t v1b = f2_fma(n2, f2(bf_hi(raw.z), bf_hi(raw.w)), bo23);
  const uint64_t o0a = f2_fma(r.c01, v0a, f2_mul(r.s01, v1a));  // c v0 + s v1
  const uint64_t o1a = f2_fma(r.c01, v1a, f2_mul(r.n01, v0a));  // c v1 - s v0
  const uint64_t o0b = f2_fma(r.c23, v0b, f2_mul(r.s23, v1b));
  const uint64_t o1b = f2_fma(r.c23, v1b, f2_mul(r.n23, v0b));
  float a0, a1, b0, b1, c0, c1, d0, d1;
  f2_split(o0a, a0, a1);
  f2_split(o1a, b0, b1);
  f2_split(o0b, c0, c1);
  f2_split(o1b, d0, d1);
  return make_uint4(pack_bf16(a0, b0), pack_bf16(a1, b1), pack_bf16(c0, d0), pack_bf16(c1, d1));
}
// Position of value j of a chunk in the staged bias layout (b0, b2, b1, b3, b4, b6, b5, b7).
__host__ __device__ constexpr int bias_pos(int j) { return (j & 4) | ((j & 1) << 1) | ((j >> 1) & 1); }
__device__ __forceinline__ uint4 scale_chunk(uint4 raw, float sc) {
  float f[8];
  unpack8(raw, f);
#pragma unroll
  for (int e = 0; e < 8; ++e) f[e] *= sc;
  return pack8(f);
}

// Row p of the bf16 state copy hb (K-major, 128-byte swizzle): the 32 values of column chunk c,
// scaled by fh.
__device__ __forceinline__ void hb_store_row(uint32_t sHB, int pc, int c, const uint32_t (&v)[32], float fh) {
  const uint64_t fh2 = f2(fh, fh);
#pragma unroll
  for (int qq = 0; qq < 4; ++qq) {
    const int ch = 4 * c + qq;
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float a, b;
      f2_split(f2_mul(fh2, f2(__uint_as_float(v[8 * qq + 2 * e]), __uint_as_float(v[8 * qq + 2 * e + 1]))), a, b);
      w[e] = pack_bf16(a, b);
    }
    const uint32_t off = (uint32_t)(ch >> 3) * (128 * 128) + (uint32_t)pc * 128u + ((uint32_t)((ch & 7) ^ (pc & 7)) << 4);
    sts128(sHB + off, make_uint4(w[0], w[1], w[2], w[3]));
  }
}

template <int R, int N, int MODE>
__global__ void __maxnreg__(WS_REG_LAUNCH)
    scan_ws_kernel(const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmC,
                   const __grid_constant__ CUtensorMap tmX, const Params p, const SegInfo sg) {
  using C = WsCfg<R, N>;
  constexpr bool FULL = (MODE == WS_FULL);
  constexpr int Q = C::Q, K2 = C::K2, BLK = C::BLK;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = p.H, G = p.G;
  const int RR = p.R;  // the operands' MIMO rank; branches RR .. R-1 of the tile are zero padding
  const int64_t L = p.L;
  const int nseg_grid = FULL ? sg.nseg : sg.nsub;
  const int bh = blockIdx.x / nseg_grid;
  const int seg = blockIdx.x % nseg_grid;
  const int bi = bh / H, hi = bh % H;
  const int g = hi / (H / G);
  const int64_t ntiles_seq = (L + Q - 1) / Q;
  const int seg_len = FULL ? sg.seg_tiles : sg.sub_tiles;
  const int64_t j0 = (int64_t)seg * seg_len;
  const int64_t j1 = (j0 + seg_len < ntiles_seq) ? (j0 + seg_len) : ntiles_seq;
  const int ntl = j1 > j0 ? (int)(j1 - j0) : 0;
  const int64_t tok_base = (int64_t)bi * L;
  const bool last_seg = FULL && (seg == sg.nseg - 1);

  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + C::OFF_MISC + 4);
  const uint32_t sStage = smem_u32(sm + C::OFF_STAGE);
  const uint32_t sSP = smem_u32(sm + C::OFF_SP), sHB = smem_u32(sm + C::OFF_HB);
  const uint32_t sXr = smem_u32(sm + C::OFF_X);
  auto sB = [&](int s) { return sStage + (uint32_t)(s * C::STAGE); };
  auto sC = [&](int s) { return sStage + (uint32_t)(s * C::STAGE + C::TILE_N); };
  auto recA = [&](int cs) { return reinterpret_cast<float4*>(sm + C::OFF_REC + cs * C::REC_SLOT); };
  auto mult = [&](int cs) { return reinterpret_cast<float*>(sm + C::OFF_REC + cs * C::REC_SLOT + Q * 16); };
  auto ycol = [&](int cs) { return reinterpret_cast<float*>(sm + C::OFF_REC + cs * C::REC_SLOT + Q * 20); };
  auto scal = [&](int cs) { return reinterpret_cast<float*>(sm + C::OFF_REC + cs * C::REC_SLOT + Q * 24); };
  double* base = reinterpret_cast<double*>(sm + C::OFF_BASE);
  float* rowss = reinterpret_cast<float*>(sm + C::OFF_ROWSS);
  float* segsum = reinterpret_cast<float*>(sm + C::OFF_SEGSUM);
  const __nv_bfloat16* xg = static_cast<const __nv_bfloat16*>(p.x);

  // ---- setup
  if (warp == W_MMA) {
    tmem_alloc(tmem_slot, C::TM_COLS);
    tmem_relinquish();
  }
  // In the state pass the mask and epilogue groups have no work of their own: with N = 128 and
  // plain inputs they rotate every tile's B, while the rotation group builds the angle tables one
  // tile ahead into two buffers (the second in the S' area, which the state pass does not use).
  // The two sides meet on BAR_RH once per tile ("table i complete and B of tile i in place"); the
  // buffer the rotation group fills next, for tile i + 1, was last read by the helpers for tile
  // i - 1, which they finished before reaching that barrier for tile i.
  const bool helpers = !FULL && !p.raw_inputs && C::NKC == 2 * N_ROT;
  if (tid == 0) {
    const int ce = FULL ? (N_ROT + 4 + 4 + 4 + 1) : (N_ROT + 4 + 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar[B_BCF + s], 1);
      mbar_init(&bar[B_BCE + s], 1);
      mbar_init(&bar[B_ROT + s], helpers ? N_HELP : N_ROT);
      mbar_init(&bar[B_XPF + s], 4);
      mbar_init(&bar[B_XBF + s], 1);
    }
    for (int c = 0; c < WS_CS; ++c) {
      mbar_init(&bar[B_CF + c], 1);
      mbar_init(&bar[B_CE + c], ce);
    }
    mbar_init(&bar[B_RESC], N_ROT);
    mbar_init(&bar[B_SF], 1);
    mbar_init(&bar[B_SPF], 4);
    mbar_init(&bar[B_HF], 4);
    mbar_init(&bar[B_SPGO], 1);
    mbar_init(&bar[B_YF], 1);
    mbar_init(&bar[B_YE], 4);
    mbar_init(&bar[B_DRAIN], 1);
    mbar_init(&bar[B_FIN], N_ROT);
    mbar_init(&bar[B_XF], 1);
    mbar_init(&bar[B_XE], 4);
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int k = tid; k < K2; k += WS_THREADS) base[k] = 0.0;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // State pass, N = 128, plain inputs: helper warp hw (0..7) of the mask and epilogue groups
  // rotates B chunks hw and hw + 8 of every tile, after the tile's BAR_RH barrier.
  auto rotate_help = [&]() {
    const int hw = warp - W_MASK;
    const float* biasB = reinterpret_cast<const float*>(sm + C::OFF_BIAS) + (lane % R) * C::BIAS_ROW;
    Phases ph_bcf;
    for (int i = 0; i < ntl; ++i) {
      const int s = i & 1;
      const int64_t c0 = (j0 + i) * Q;
      const int nv = (int)((L - c0) < Q ? (L - c0) : Q);
      const bool okb = ws_wait(&bar[B_BCF + s], ph_bcf[s], abort_flag);
      ph_bcf.flip(s);
      if (bar_any(BAR_RH, 32 * (N_ROT + N_HELP), !okb || *abort_flag)) break;  // table i complete
      const uint8_t* tb = s ? sm + C::OFF_SP : sm + C::OFF_TAB;
#pragma unroll 1
      for (int q = 0; q < 2; ++q) {
        const int kc = hw + N_ROT * q;
        const uint32_t cb = (uint32_t)(kc >> 3) * C::BLK + (uint32_t)lane * 128u + ((uint32_t)((kc & 7) ^ (lane & 7)) << 4);
        const float4 bBe = *reinterpret_cast<const float4*>(biasB + kc * 8);
        const float4 bBo = *reinterpret_cast<const float4*>(biasB + kc * 8 + 4);
        const uint64_t bB0 = f2(bBe.x, bBe.y), bB1 = f2(bBe.z, bBe.w), bB2 = f2(bBo.x, bBo.y), bB3 = f2(bBo.z, bBo.w);
        const uint8_t* tk = tb + kc * 16;
#pragma unroll 2
        for (int step = 0; step < 4; ++step) {
          const int t = (32 * step + lane) / R;
          const uint32_t off = cb + (uint32_t)step * 4096u;
          if (t < nv) {
            const RotCS rcs = rot_cs(*reinterpret_cast<const uint4*>(tk + t * C::TAB_ROW));
            sts128(sB(s) + off, rotate16(lds128(sB(s) + off), rcs, f2(1.0f, 1.0f), bB0, bB1, bB2, bB3));
          } else {
            sts128(sB(s) + off, make_uint4(0, 0, 0, 0));
          }
        }
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[B_ROT + s]);
    }
  };
  const int wg = warp >> 2;
  if (wg == 0) {
    regs_dec<WS_REG_CTRL>();
    if (ntl > 0) {
      if (warp == W_PROD) {
        // =============================================================== producer
        if (lane == 0) {
          Phases ph_e, ph_xe;
          int issued0 = 0, issued1 = 0, xissued = 0;
          for (int i = 0; i < ntl; ++i) {
            const int s = i & 1;
            const int tok = (int)(tok_base + (j0 + i) * Q);
            if (i >= 2) {
              if (!ws_wait(&bar[B_BCE + s], ph_e[s], abort_flag)) break;
              ph_e.flip(s);
            }
            mbar_expect_tx(&bar[B_BCF + s], FULL ? C::STAGE : C::TILE_N);
#pragma unroll
            for (int blk = 0; blk < N / 64; ++blk) {
              tma_load_4d(sB(s) + blk * BLK, &tmB, 64 * blk, 0, g, tok, &bar[B_BCF + s]);
              if constexpr (FULL) tma_load_4d(sC(s) + blk * BLK, &tmC, 64 * blk, 0, g, tok, &bar[B_BCF + s]);
            }
            if (s) ++issued1; else ++issued0;
            // x of the tile (for X'^T) into the slot, once the state warps have read the last one
            if (i >= 1) {
              if (!ws_wait(&bar[B_XE], ph_xe[0], abort_flag)) break;
              ph_xe.flip(0);
            }
            mbar_expect_tx(&bar[B_XF], C::XSLOT);
            tma_load_3d(sXr, &tmX, 0, hi, tok, &bar[B_XF]);
            ++xissued;
          }
          // every copy issued has landed before the CTA may exit
          if (issued0 > 0) ws_wait_drain(&bar[B_BCF + 0], (uint32_t)((issued0 - 1) & 1));
          if (issued1 > 0) ws_wait_drain(&bar[B_BCF + 1], (uint32_t)((issued1 - 1) & 1));
          if (xissued > 0) ws_wait_drain(&bar[B_XF], (uint32_t)((xissued - 1) & 1));
        }
      } else if (warp == W_COEF) {
        // =============================================================== coefficients
        constexpr int TPL = Q >= 32 ? Q / 32 : 1;  // tokens per lane
        float lrho_prev = 0.0f, seg_logdec = 0.0f;
        Phases ph_ce;
        for (int i = 0; i < ntl; ++i) {
          const int cs = i % WS_CS;
          const int64_t c0 = (j0 + i) * Q;
          const int nv = (int)((L - c0) < Q ? (L - c0) : Q);
          if (i >= WS_CS) {
            if (!ws_wait(&bar[B_CE + cs], ph_ce[cs], abort_flag)) break;
            ph_ce.flip(cs);
          }
          float dtv[TPL], av[TPL], lmv[TPL], loc[TPL];
          float run = 0.0f;
#pragma unroll
          for (int e = 0; e < TPL; ++e) {
            const int t = lane * TPL + e;
            const bool valid = t < nv && t < Q;
            const int64_t ti = (tok_base + c0 + t) * H + hi;
            dtv[e] = valid ? p.dt[ti] : 0.0f;
            av[e] = valid ? p.A[ti] : 0.0f;
            lmv[e] = valid ? p.lam[ti] : 0.0f;
            if (p.raw_inputs && valid) {  // the front-end, fused: the operands are raw projections
              dtv[e] = fe_softplus(dtv[e]);
              av[e] = fe_negexp(av[e]);
              lmv[e] = fe_sigmoid(lmv[e]);
            }
            run += dtv[e] * av[e];
            loc[e] = run;
          }
          float incl = run;
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) {
            const float o = __shfl_up_sync(kFull, incl, off);
            if (lane >= off) incl += o;
          }
          const float Le = __shfl_sync(kFull, incl, 31);
          const float excl = incl - run;
          float lmin = 0.0f, lmax = 0.0f;
#pragma unroll
          for (int e = 0; e < TPL; ++e) {
            loc[e] += excl;
            if (lane * TPL + e < Q) {
              lmin = fminf(lmin, loc[e]);
              lmax = fmaxf(lmax, loc[e]);
            }
          }
          lmin = key_float(__reduce_min_sync(kFull, float_key(lmin)));
          lmax = key_float(__reduce_max_sync(kFull, float_key(lmax)));
          const bool fast = (lmax - lmin) <= WS_FAST_RANGE;
          const float m = fast ? 0.5f * (lmax + lmin) : 0.0f;
          // beta' of the token after each token: the next lane's first token, or the token after the tile
          float bp_after = 0.0f;
          if (c0 + Q < L) {
            const int64_t ti = (tok_base + c0 + Q) * H + hi;
            const float la = p.raw_inputs ? fe_sigmoid(p.lam[ti]) : p.lam[ti];
            const float da = p.raw_inputs ? fe_softplus(p.dt[ti]) : p.dt[ti];
            bp_after = (1.0f - la) * da;
          }
          const float nxt_dt = __shfl_down_sync(kFull, dtv[0], 1);
          const float nxt_lm = __shfl_down_sync(kFull, lmv[0], 1);
          float4* ra = recA(cs);
          float* mu = mult(cs);
#pragma unroll
          for (int e = 0; e < TPL; ++e) {
            const int t = lane * TPL + e;
            if (t < Q) {
              const bool valid = t < nv;
              const float gm = lmv[e] * dtv[e];
              float bpn;
              if (t + 1 >= Q) bpn = valid ? bp_after : 0.0f;
              else if (e + 1 < TPL) bpn = (1.0f - lmv[e + 1]) * dtv[e + 1];
              else bpn = (1.0f - nxt_lm) * nxt_dt;  // invalid next tokens carry dt = 0
              const float w = gm + bpn;
              const float dg = (w > 0.0f) ? __fdividef(gm, w) : 0.0f;
              float xs, ys;  // factors of X' (input rows) and of the output columns
              if (fast) {
                xs = __expf(m - loc[e]) * w;
                ys = __expf(loc[e] - m);
              } else if (FULL) {
                xs = w;  // Bt rescaled by e^{Le - Lc_t} after S
                ys = 1.0f;
              } else {
                xs = __expf(Le - loc[e]) * w;  // state pass: no S, the final factor at once
                ys = 1.0f;
              }
              ra[t] = make_float4(loc[e], dg, xs, ys);
              mu[t] = valid ? (p.angle_direct ? 1.0f : dtv[e]) : 0.0f;
              ycol(cs)[t] = ys;
            }
          }
          // state scale factors: ST enters tile i as sigma ST_i (sigma = e^m, or e^{Le} on an exact
          // tile) and leaves it as rho ST_{i+1} (rho = e^{m - Le}, or 1 on an exact tile, whose H
          // operand already carries e^{Le - Lc_s})
          const float lsig = fast ? m : Le;
          const float lrho = fast ? (m - Le) : 0.0f;
          if (lane == 0) {
            float* sc = scal(cs);
            sc[0] = fast ? 1.0f : 0.0f;
            sc[1] = Le;
            sc[2] = m;
            sc[3] = __expf(m - lrho_prev);     // hb = bf16(f_h * tensor-memory state)
            sc[4] = __expf(lsig - lrho_prev);  // state before H = f_s * tensor-memory state
            sc[5] = __expf(-lrho);             // true state after the tile = this * tensor-memory state
            sc[6] = (float)nv;
          }
          lrho_prev = lrho;
          seg_logdec += Le;
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[B_CF + cs]);
        }
        if constexpr (!FULL) {
          if (lane == 0 && !*abort_flag) sg.ws_l[(int64_t)bh * sg.nsub + seg] = seg_logdec;
        }
      } else if (warp == W_MMA) {
        // =============================================================== MMA issue
        Phases ph_cf, ph_rot, ph_xpf;
        uint32_t ph_hf = 0, ph_resc = 0, ph_ye = 0, ph_spf = 0;
        bool issued = false, ok = true;
        auto kdesc = [&](uint32_t base_addr, int k) {  // K-major SW128 operand, K-step k of 16
          return sdesc(base_addr + (uint32_t)(k >> 2) * BLK + (uint32_t)(k & 3) * 32, 16, 1024);
        };
        if (FULL) {
          ok = ws_wait(&bar[B_ROT + 0], ph_rot[0], abort_flag);
          ph_rot.flip(0);
          if (ok) {
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < N / 16; ++k)
              mma_ss_w(tmem + C::TM_S, kdesc(sC(0), k), kdesc(sB(0), k), C::ID_S, k > 0);
            mma_commit_w(&bar[B_SF]);
            issued = true;
          }
        }
        for (int i = 0; ok && i < ntl; ++i) {
          const int cs = i % WS_CS, s = i & 1, xb = i & 1;
          if (!ws_wait(&bar[B_CF + cs], ph_cf[cs], abort_flag)) break;
          ph_cf.flip(cs);
          const bool fast = scal(cs)[0] != 0.0f;
          if (!ws_wait(&bar[B_HF], ph_hf, abort_flag)) break;
          ph_hf ^= 1;
          if (FULL && !fast) {
            if (!ws_wait(&bar[B_RESC], ph_resc, abort_flag)) break;
            ph_resc ^= 1;
          }
          if (!ws_wait(&bar[B_XPF + xb], ph_xpf[xb], abort_flag)) break;
          ph_xpf.flip(xb);
          if constexpr (!FULL) {  // the full pass waited for the rotation before S of this tile
            if (!ws_wait(&bar[B_ROT + s], ph_rot[s], abort_flag)) break;
            ph_rot.flip(s);
          }
          tc_fence_after();
          // H: ST += X'^T Bt'  (A = X'^T in tensor memory, B = Bt' MN-major)
#pragma unroll
          for (int k = 0; k < 128 / 16; ++k)
            mma_ts_w(tmem + C::TM_ST, tmem + C::TM_XP + 64 * xb + 8 * k,
                     sdesc(sB(s) + (uint32_t)k * 2048, BLK, 1024), C::ID_H, 1);
          issued = true;
          if constexpr (!FULL) {
            mma_commit_w(&bar[B_SPGO]);
            mma_commit_w(&bar[B_XBF + xb]);
            mma_commit_w(&bar[B_BCE + s]);
          } else {
            if (i > 0) {
              if (!ws_wait(&bar[B_YE], ph_ye, abort_flag)) break;
              ph_ye ^= 1;
              tc_fence_after();
            }
            // Y_inter: Y^T = hb Ct'^T  (A = hb K-major, B = Ct' K-major)
#pragma unroll
            for (int k = 0; k < N / 16; ++k)
              mma_ss_w(tmem + C::TM_Y, kdesc(sHB, k), kdesc(sC(s), k), C::ID_Y, k > 0);
            mma_commit_w(&bar[B_SPGO]);
            mma_commit_w(&bar[B_BCE + s]);
            if (!ws_wait(&bar[B_SPF], ph_spf, abort_flag)) break;
            ph_spf ^= 1;
            tc_fence_after();
            // Y_intra: Y^T += X'^T S'^T  (A = X'^T in tensor memory, B = S' K-major)
#pragma unroll
            for (int k = 0; k < 128 / 16; ++k)
              mma_ts_w(tmem + C::TM_Y, tmem + C::TM_XP + 64 * xb + 8 * k, kdesc(sSP, k), C::ID_Y, 1);
            mma_commit_w(&bar[B_YF]);
            mma_commit_w(&bar[B_XBF + xb]);
            if (i + 1 < ntl) {
              if (!ws_wait(&bar[B_ROT + (s ^ 1)], ph_rot[s ^ 1], abort_flag)) break;
              ph_rot.flip(s ^ 1);
              tc_fence_after();
#pragma unroll
              for (int k = 0; k < N / 16; ++k)
                mma_ss_w(tmem + C::TM_S, kdesc(sC(s ^ 1), k), kdesc(sB(s ^ 1), k), C::ID_S, k > 0);
              mma_commit_w(&bar[B_SF]);
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[B_CE + cs]);
        }
        if (issued) {  // every MMA issued has completed before tensor memory is released
          mma_commit_w(&bar[B_DRAIN]);
          ws_wait_drain(&bar[B_DRAIN], 0);
        }
      }
    }
  } else if (wg <= 2) {
    regs_inc<WS_REG_ROT>();
    if (ntl > 0) {
        // =============================================================== rotation
        const int rt = tid - 32 * W_ROT;
        const int wr = warp - W_ROT;
        const int ak = rt % K2, aseg = rt / K2;  // angles: pair ak over token segment aseg
        // rotation: chunks kc = wr + N_ROT q of rows 32 step + lane (the branch r = lane % R is fixed)
        const int rr = lane % R;
        // the biases of the head, staged once as fp32 in the pair layout of rotate16
        float* sbias = reinterpret_cast<float*>(sm + C::OFF_BIAS);
        for (int e = rt; e < 2 * R * N; e += 32 * N_ROT) {
          const int op = e / (R * N), rem = e % (R * N), r = rem / N, n = rem % N;
          const float* src = op ? p.bias_C : p.bias_B;
          sbias[(op * R + r) * C::BIAS_ROW + (n >> 3) * 8 + bias_pos(n & 7)] =
              (src && r < RR) ? src[((int64_t)hi * RR + r) * N + n] : 0.0f;
        }
        const float* biasB = sbias + rr * C::BIAS_ROW;
        const float* biasC = sbias + (R + rr) * C::BIAS_ROW;
        float thr[C::SEGLEN];
        auto load_theta = [&](int64_t j) {
          const int64_t t0 = j * Q + aseg * C::SEGLEN;  // first token of this thread's segment
          const float* th = p.theta + ((tok_base + t0) * G + g) * K2 + ak;
          const int nth = (int)(L - t0 < C::SEGLEN ? (L - t0 > 0 ? L - t0 : 0) : C::SEGLEN);
#pragma unroll
          for (int e = 0; e < C::SEGLEN; ++e) thr[e] = (e < nth) ? __ldg(th + e * G * K2) : 0.0f;
        };
        load_theta(j0);
        Phases ph_cf, ph_bcf;
        uint8_t* tab = sm + C::OFF_TAB;
        if (!FULL && helpers) {
          // ---- state pass with helpers: the angle tables only, one tile ahead of the rotation
          for (int i = 0; i < ntl; ++i) {
            const int cs = i % WS_CS, s = i & 1;
            const int64_t j = j0 + i;
            uint8_t* tb = s ? sm + C::OFF_SP : sm + C::OFF_TAB;
            const bool okw = ws_wait(&bar[B_CF + cs], ph_cf[cs], abort_flag);
            ph_cf.flip(cs);
            // a failed wait is carried to this tile's BAR_RH barrier, where everyone stops together
            // (the table is built regardless, from whatever the record holds); the previous tile's
            // segment sums were read before that tile's BAR_RH barrier
            double tot = 0.0;
            {
              const float* mu = mult(cs);
              float aloc[C::SEGLEN];
              float r2 = 0.0f;
#pragma unroll
              for (int e = 0; e < C::SEGLEN; ++e) {
                r2 = fmaf(mu[aseg * C::SEGLEN + e], thr[e], r2);
                aloc[e] = r2;
              }
              segsum[aseg * K2 + ak] = r2;
              named_bar_sync(BAR_ROT, 32 * N_ROT);
              float aoff = (float)base[ak];
#pragma unroll
              for (int s2 = 0; s2 < C::SEGS; ++s2) {
                const float v = segsum[s2 * K2 + ak];
                if (s2 < aseg) aoff += v;
                if (aseg == 0) tot += (double)v;
              }
#pragma unroll
              for (int e = 0; e < C::SEGLEN; ++e) {
                const int t = aseg * C::SEGLEN + e;
                float sn, cn;
                sincos_reduced(aoff + aloc[e], &sn, &cn);
                const float other = __shfl_xor_sync(kFull, (ak & 1) ? cn : sn, 1);
                const __half2 hv = (ak & 1) ? __floats2half2_rn(other, sn) : __floats2half2_rn(cn, other);
                *reinterpret_cast<__half2*>(tb + t * C::TAB_ROW + (ak >> 1) * 8 + (ak & 1) * 4) = hv;
              }
              if (i + 1 < ntl) load_theta(j + 1);
            }
            const bool okb = okw && ws_wait(&bar[B_BCF + s], ph_bcf[s], abort_flag);
            ph_bcf.flip(s);
            // table i complete, B of tile i in place: the helpers rotate it
            if (bar_any(BAR_RH, 32 * (N_ROT + N_HELP), !okb || *abort_flag)) break;
            if (aseg == 0) {
              double nb = base[ak] + tot;
              nb -= 6.283185307179586 * rint(nb * 0.15915494309189535);
              base[ak] = nb;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[B_CE + cs]);
          }
        } else
        for (int i = 0; i < ntl; ++i) {
          const int cs = i % WS_CS, s = i & 1;
          const int64_t j = j0 + i;
          const int64_t c0 = j * Q;
          const int nv = (int)((L - c0) < Q ? (L - c0) : Q);
          bool okw = ws_wait(&bar[B_CF + cs], ph_cf[cs], abort_flag);
          ph_cf.flip(cs);
          // the group stops together
          if (bar_any(BAR_ROT, 32 * N_ROT, !okw || *abort_flag)) break;
          const float* mu = mult(cs);
          const float4* ra = recA(cs);
          const float* sc = scal(cs);
          // ---- cumulative angles of the tile and their sin / cos
          float aloc[C::SEGLEN];
          {
            float r2 = 0.0f;
#pragma unroll
            for (int e = 0; e < C::SEGLEN; ++e) {
              r2 = fmaf(mu[aseg * C::SEGLEN + e], thr[e], r2);
              aloc[e] = r2;
            }
            segsum[aseg * K2 + ak] = r2;
          }
          named_bar_sync(BAR_ROT, 32 * N_ROT);
          double tot = 0.0;
          {
            float aoff = (float)base[ak];
#pragma unroll
            for (int s2 = 0; s2 < C::SEGS; ++s2) {
              const float v = segsum[s2 * K2 + ak];
              if (s2 < aseg) aoff += v;
              if (aseg == 0) tot += (double)v;
            }
#pragma unroll
            for (int e = 0; e < C::SEGLEN; ++e) {
              const int t = aseg * C::SEGLEN + e;
              float sn, cn;
              sincos_reduced(aoff + aloc[e], &sn, &cn);
              // per two pairs (k, k+1): half2 (c_k, c_k+1) then half2 (s_k, s_k+1); the lanes of
              // pairs k (even) and k+1 (odd) are neighbours
              const float other = __shfl_xor_sync(kFull, (ak & 1) ? cn : sn, 1);
              const __half2 hv = (ak & 1) ? __floats2half2_rn(other, sn) : __floats2half2_rn(cn, other);
              *reinterpret_cast<__half2*>(tab + t * C::TAB_ROW + (ak >> 1) * 8 + (ak & 1) * 4) = hv;
            }
          }
          if (i + 1 < ntl) load_theta(j + 1);
          // the angles needed no B or C: their copy lands meanwhile
          okw = ws_wait(&bar[B_BCF + s], ph_bcf[s], abort_flag);
          ph_bcf.flip(s);
          // table complete, base and segsum read, the tile's B and C in place
          if (bar_any(BAR_ROT, 32 * N_ROT, !okw || *abort_flag)) break;
          if (aseg == 0) {
            double nb = base[ak] + tot;
            nb -= 6.283185307179586 * rint(nb * 0.15915494309189535);
            base[ak] = nb;
          }
          if (p.raw_inputs) {
            // the fused B/C RMS norm: every row's sum of squares over N, from each warp's chunks
            rowss[rt] = 0.0f;
            named_bar_sync(BAR_ROT, 32 * N_ROT);
#pragma unroll 1
            for (int q = 0; q < C::KCW; ++q) {
              const int kc = wr + N_ROT * q;
              const uint32_t cb = (uint32_t)(kc >> 3) * BLK + (uint32_t)lane * 128u + ((uint32_t)((kc & 7) ^ (lane & 7)) << 4);
              for (int step = 0; step < 4; ++step) {
                const int row = 32 * step + lane;
                if (row / R >= nv) continue;
                float f[8], ss = 0.0f;
                unpack8(lds128(sB(s) + cb + step * 4096), f);
#pragma unroll
                for (int e = 0; e < 8; ++e) ss = fmaf(f[e], f[e], ss);
                atomicAdd(&rowss[row], ss);
                if constexpr (FULL) {
                  unpack8(lds128(sC(s) + cb + step * 4096), f);
                  ss = 0.0f;
#pragma unroll
                  for (int e = 0; e < 8; ++e) ss = fmaf(f[e], f[e], ss);
                  atomicAdd(&rowss[128 + row], ss);
                }
              }
            }
            named_bar_sync(BAR_ROT, 32 * N_ROT);
          }
          // ---- rotate Bt (and Ct) of the tile in place: lanes take 32 consecutive rows, the branch
          // r = lane % R and so the chunk's biases are fixed per thread
#pragma unroll 1
          for (int q = 0; q < C::KCW; ++q) {
            const int kc = wr + N_ROT * q;
            // row 32 step + lane, chunk kc: 128-byte swizzle with (row & 7) = (lane & 7)
            const uint32_t cb = (uint32_t)(kc >> 3) * BLK + (uint32_t)lane * 128u + ((uint32_t)((kc & 7) ^ (lane & 7)) << 4);
            const float4 bBe = *reinterpret_cast<const float4*>(biasB + kc * 8);
            const float4 bBo = *reinterpret_cast<const float4*>(biasB + kc * 8 + 4);
            const uint64_t bB0 = f2(bBe.x, bBe.y), bB1 = f2(bBe.z, bBe.w), bB2 = f2(bBo.x, bBo.y), bB3 = f2(bBo.z, bBo.w);
            uint64_t bC0 = 0, bC1 = 0, bC2 = 0, bC3 = 0;
            if constexpr (FULL) {
              const float4 bCe = *reinterpret_cast<const float4*>(biasC + kc * 8);
              const float4 bCo = *reinterpret_cast<const float4*>(biasC + kc * 8 + 4);
              bC0 = f2(bCe.x, bCe.y), bC1 = f2(bCe.z, bCe.w), bC2 = f2(bCo.x, bCo.y), bC3 = f2(bCo.z, bCo.w);
            }
            const uint8_t* tk = tab + kc * 16;
#pragma unroll 2
            for (int step = 0; step < 4; ++step) {
              const int row = 32 * step + lane;
              const int t = row / R;
              const uint32_t off = cb + (uint32_t)step * 4096u;
              if (t < nv) {
                float nb = 1.0f, nc = 1.0f;
                if (p.raw_inputs) {  // 1 / rms of the raw rows: the B/C norm, before the bias
                  nb = rsqrtf(rowss[row] * (1.0f / N) + kBcNormEps);
                  if constexpr (FULL) nc = rsqrtf(rowss[128 + row] * (1.0f / N) + kBcNormEps);
                }
                const RotCS rcs = rot_cs(*reinterpret_cast<const uint4*>(tk + t * C::TAB_ROW));
                const uint4 rb = lds128(sB(s) + off);
                uint4 rc;
                if constexpr (FULL) rc = lds128(sC(s) + off);
                sts128(sB(s) + off, rotate16(rb, rcs, f2(nb, nb), bB0, bB1, bB2, bB3));
                if constexpr (FULL) sts128(sC(s) + off, rotate16(rc, rcs, f2(nc, nc), bC0, bC1, bC2, bC3));
              } else {
                sts128(sB(s) + off, make_uint4(0, 0, 0, 0));
                if constexpr (FULL) sts128(sC(s) + off, make_uint4(0, 0, 0, 0));
              }
            }
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[B_ROT + s]);
          if (FULL && sc[0] == 0.0f) {
            // exact tile: after S has read them, Ct rows * e^{Lc_t} (inter-chunk product) and
            // Bt rows * e^{Le - Lc_t} (state product)
            const bool oks = ws_wait(&bar[B_SF], (uint32_t)(i & 1), abort_flag);
            if (bar_any(BAR_ROT, 32 * N_ROT, !oks || *abort_flag)) break;
            const float Le = sc[1];
#pragma unroll 1
            for (int q = 0; q < C::KCW; ++q) {
              const int kc = wr + N_ROT * q;
              const uint32_t cb = (uint32_t)(kc >> 3) * BLK + (uint32_t)lane * 128u + ((uint32_t)((kc & 7) ^ (lane & 7)) << 4);
              for (int step = 0; step < 4; ++step) {
                const int t = (32 * step + lane) / R;
                if (t >= nv) continue;
                const uint32_t off = cb + (uint32_t)step * 4096u;
                const float Lct = reinterpret_cast<const float*>(ra)[4 * t];
                sts128(sC(s) + off, scale_chunk(lds128(sC(s) + off), __expf(Lct)));
                sts128(sB(s) + off, scale_chunk(lds128(sB(s) + off), __expf(Le - Lct)));
              }
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar[B_RESC]);
          }
          if (lane == 0) mbar_arrive(&bar[B_CE + cs]);
        }
        // final angles of the segment: the full pass rotates the state back by them, the state
        // pass stores them in its summary
        named_bar_sync(BAR_ROT, 32 * N_ROT);
        if (!*abort_flag) {
          if constexpr (!FULL) {
            if (aseg == 0) sg.ws_phi[((int64_t)bh * sg.nsub + seg) * K2 + ak] = base[ak];
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[B_FIN]);
        }
    }
  } else if (wg == 3) {
    if (!FULL && helpers && ntl > 0) rotate_help();
    if (FULL && ntl > 0) {
        // =============================================================== mask
        const int q4 = warp & 3;
        const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
        const int row = 32 * q4 + lane;
        const int t = row / R;
        Phases ph_cf;
        for (int i = 0; i < ntl; ++i) {
          const int cs = i % WS_CS;
          if (!ws_wait(&bar[B_CF + cs], ph_cf[cs], abort_flag)) break;
          ph_cf.flip(cs);
          if (!ws_wait(&bar[B_SF], (uint32_t)(i & 1), abort_flag)) break;
          tc_fence_after();
          const float4* ra = recA(cs);
          const bool fast = scal(cs)[0] != 0.0f;
          const float* rf = reinterpret_cast<const float*>(ra);  // scalar reads of the records
          const float Lt2 = rf[4 * t] * 1.4426950408889634f;
          const float dgt = rf[4 * t + 1];
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t o[16];
            if (c > q4) {  // every column token is after every row token of this warp
#pragma unroll
              for (int e = 0; e < 16; ++e) o[e] = 0u;
            } else {
              uint32_t v[32];
              tmem_ld32(tmem + lane_base + C::TM_S + 32 * c, v);
              tmem_wait_ld();
              float f[32];
#pragma unroll
              for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(v[e]);
              if (!fast) {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                  const int st = (32 * c + e) / R;
                  f[e] = (st <= t) ? f[e] * ex2_approx(Lt2 - rf[4 * st] * 1.4426950408889634f) : 0.0f;
                }
              }
              if (c == q4) {  // the diagonal block: column token e / R against the row's lane / R
                const int lt = lane / R;
#pragma unroll
                for (int e = 0; e < 32; ++e) f[e] = (e / R < lt) ? f[e] : ((e / R == lt) ? f[e] * dgt : 0.0f);
              }
#pragma unroll
              for (int e = 0; e < 16; ++e) o[e] = pack_bf16(f[2 * e], f[2 * e + 1]);
            }
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
              const int ch = 4 * c + qq;
              const uint32_t off = (uint32_t)(ch >> 3) * BLK + (uint32_t)row * 128u +
                                   ((uint32_t)((ch & 7) ^ (row & 7)) << 4);
              sts128(sSP + off, make_uint4(o[4 * qq], o[4 * qq + 1], o[4 * qq + 2], o[4 * qq + 3]));
            }
          }
          fence_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&bar[B_SPF]);
            mbar_arrive(&bar[B_CE + cs]);
          }
        }
    }
  } else if (wg == 4) {
    if (!FULL && helpers && ntl > 0) rotate_help();
    if (FULL && ntl > 0) {
        // =============================================================== epilogue
        const int q4 = warp & 3;
        const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
        const int pc = 32 * q4 + lane;  // head-dim column of this thread
        float wo[R];
#pragma unroll
        for (int r = 0; r < R; ++r) wo[r] = r < RR ? (p.W_o ? p.W_o[((int64_t)hi * RR + r) * WP + pc] : 1.0f) : 0.0f;
        const float Dh = p.D ? p.D[hi] : 0.0f;
        __nv_bfloat16* yg = static_cast<__nv_bfloat16*>(p.y);
        constexpr int TPC = 16 / R;  // tokens per 16-column chunk
        const int64_t tstride = (int64_t)H * WP;  // elements between consecutive tokens of y and x
        Phases ph_cf;
        for (int i = 0; i < ntl; ++i) {
          const int cs = i % WS_CS;
          const int64_t c0 = (j0 + i) * Q;
          const int nv = (int)((L - c0) < Q ? (L - c0) : Q);
          if (!ws_wait(&bar[B_CF + cs], ph_cf[cs], abort_flag)) break;
          ph_cf.flip(cs);
          if (!ws_wait(&bar[B_YF], (uint32_t)(i & 1), abort_flag)) break;
          tc_fence_after();
          const float* yc = ycol(cs);
          const int64_t e0 = ((tok_base + c0) * H + hi) * (int64_t)WP + pc;
          __nv_bfloat16* yrow = yg + e0;
          const __nv_bfloat16* xrow = xg + e0;
          const bool plain = (nv == Q) && (p.D == nullptr);  // a full tile without the skip term
#pragma unroll 1
          for (int c = 0; c < 8; ++c) {
            uint32_t v[16];
            tmem_ld16(tmem + lane_base + C::TM_Y + 16 * c, v);
            float a[TPC];
#pragma unroll
            for (int u = 0; u < TPC; ++u) a[u] = yc[TPC * c + u];  // the column factors a_t
            tmem_wait_ld();
            if (c == 7) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&bar[B_YE]);
            }
            __nv_bfloat16* yp = yrow + (int64_t)(TPC * c) * tstride;
            if (plain) {
#pragma unroll
              for (int u = 0; u < TPC; ++u) {
                float acc = 0.0f;
#pragma unroll
                for (int r = 0; r < R; ++r) acc = fmaf(wo[r], __uint_as_float(v[u * R + r]), acc);
                *yp = __float2bfloat16_rn(a[u] * acc);
                yp += tstride;
              }
            } else {
#pragma unroll
              for (int u = 0; u < TPC; ++u) {
                const int t = TPC * c + u;
                if (t < nv) {
                  float acc = 0.0f;
#pragma unroll
                  for (int r = 0; r < R; ++r) acc = fmaf(wo[r], __uint_as_float(v[u * R + r]), acc);
                  const float dx = p.D ? Dh * __bfloat162float(xrow[t * tstride]) : 0.0f;
                  yp[u * tstride] = __float2bfloat16_rn(fmaf(a[u], acc, dx));
                }
              }
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[B_CE + cs]);
        }
    }
  } else {
    if (ntl > 0) {
        // =============================================================== state and inputs
        const int q4 = warp & 3;
        const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
        const int pc = 32 * q4 + lane;
        float wx[R];
#pragma unroll
        for (int r = 0; r < R; ++r) wx[r] = r < RR ? (p.W_x ? p.W_x[((int64_t)hi * RR + r) * WP + pc] : 1.0f) : 0.0f;
        Phases ph_cf, ph_xbf, ph_xf;
        constexpr int TPC = 32 / R;
        // X'^T of tile i: X'^T[p, tR + r] = W_x[r, p] x_t[p], bf16 pairs along the columns
        auto build_xp = [&](int i) -> bool {
          const int xb = i & 1, cs = i % WS_CS;
          if (i >= 2) {
            if (!ws_wait(&bar[B_XBF + xb], ph_xbf[xb], abort_flag)) return false;
            ph_xbf.flip(xb);
          }
          const int64_t c0 = (j0 + i) * Q;
          const int nv = (int)((L - c0) < Q ? (L - c0) : Q);
          // the tile's X' factors (the main loop waits for the same phase of this slot again)
          if (!ws_wait(&bar[B_CF + cs], ph_cf[cs], abort_flag)) return false;
          if (!ws_wait(&bar[B_XF], ph_xf[0], abort_flag)) return false;
          ph_xf.flip(0);
          tc_fence_after();
          const __nv_bfloat16* xs = reinterpret_cast<const __nv_bfloat16*>(sm + C::OFF_X);
          const float4* ra = recA(cs);
#pragma unroll 1
          for (int gq = 0; gq < 4; ++gq) {
            float xv[TPC];
#pragma unroll
            for (int u = 0; u < TPC; ++u) {
              const int t = TPC * gq + u;
              xv[u] = (t < nv) ? reinterpret_cast<const float*>(ra)[4 * t + 2] * __bfloat162float(xs[t * WP + pc]) : 0.0f;
            }
            uint32_t w[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int c2 = 2 * e;  // column pair (c2, c2 + 1) of this 32-column group
              w[e] = pack_bf16(wx[c2 % R] * xv[c2 / R], wx[(c2 + 1) % R] * xv[(c2 + 1) / R]);
            }
            tmem_st16(tmem + lane_base + C::TM_XP + 64 * xb + 16 * gq, w);
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&bar[B_XPF + xb]);
            mbar_arrive(&bar[B_XE]);  // the x slot is read
          }
          return true;
        };
        bool ok = build_xp(0);
        for (int i = 0; ok && i < ntl; ++i) {
          const int cs = i % WS_CS;
          if (!ws_wait(&bar[B_CF + cs], ph_cf[cs], abort_flag)) break;
          ph_cf.flip(cs);
          const float fh = scal(cs)[3], fs = scal(cs)[4];
          if (i == 0) {
            // the rotated-frame state entering the segment (h+: it includes the previous token's
            // trapezoid term beta'_0 u_{-1})
            const bool from_state = FULL ? (seg == 0) : false;
            const bool make_init = !FULL && seg == 0 && sg.write_init;
            const bool fold = FULL && seg > 0;
            const int nfold = fold ? seg * (sg.seg_tiles / sg.sub_tiles) : 0;
            float bp0 = 0.0f, xprev[R];
            if (from_state || make_init) {
              const float l0 = p.raw_inputs ? fe_sigmoid(p.lam[tok_base * H + hi]) : p.lam[tok_base * H + hi];
              const float d0 = p.raw_inputs ? fe_softplus(p.dt[tok_base * H + hi]) : p.dt[tok_base * H + hi];
              bp0 = (1.0f - l0) * d0;
#pragma unroll
              for (int r = 0; r < R; ++r) xprev[r] = wx[r] * p.carry_x[(int64_t)bh * WP + pc];
            }
            const float* h0 = p.h + (int64_t)bh * N * WP;
            const float* cB = p.carry_B + (int64_t)bh * RR * N;
            const float* bB = p.bias_B ? p.bias_B + (int64_t)hi * RR * N : nullptr;
#pragma unroll 1
            for (int c = 0; c < N / 32; ++c) {
              float v[32];
#pragma unroll
              for (int e = 0; e < 32; ++e) v[e] = 0.0f;
              if (from_state || make_init) {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                  const int n = 32 * c + e;
                  float u = 0.0f;
#pragma unroll
                  for (int r = 0; r < R; ++r)
                    if (r < RR) u = fmaf(cB[r * N + n] + (bB ? bB[r * N + n] : 0.0f), xprev[r], u);
                  v[e] = fmaf(bp0, u, h0[(int64_t)n * WP + pc]);
                }
                if (make_init) {
                  float* wi = sg.ws_init + (int64_t)bh * N * WP;
#pragma unroll
                  for (int e = 0; e < 32; ++e) wi[(int64_t)(32 * c + e) * WP + pc] = v[e];
#pragma unroll
                  for (int e = 0; e < 32; ++e) v[e] = 0.0f;  // the state pass starts from zero
                }
              } else if (fold) {
                const float* wi = sg.ws_init + (int64_t)bh * N * WP;
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] = wi[(int64_t)(32 * c + e) * WP + pc];
                for (int k = 0; k < nfold; ++k) {
                  const int64_t sidx = (int64_t)bh * sg.nsub + k;
                  const float dec = __expf(sg.ws_l[sidx]);
                  const float* wh = sg.ws_h + sidx * N * WP;
                  const double* ph = sg.ws_phi + sidx * K2;
#pragma unroll
                  for (int e = 0; e < 16; ++e) {
                    const int n0 = 32 * c + 2 * e;
                    float sn, cn;
                    sincosf((float)ph[n0 / 2], &sn, &cn);
                    const float a0 = fmaf(dec, v[2 * e], wh[(int64_t)n0 * WP + pc]);
                    const float a1 = fmaf(dec, v[2 * e + 1], wh[(int64_t)(n0 + 1) * WP + pc]);
                    v[2 * e] = cn * a0 - sn * a1;
                    v[2 * e + 1] = sn * a0 + cn * a1;
                  }
                }
              }
              uint32_t u32[32];
#pragma unroll
              for (int e = 0; e < 32; ++e) u32[e] = __float_as_uint(v[e]);
              if constexpr (FULL) hb_store_row(sHB, pc, c, u32, fh);
#pragma unroll
              for (int e = 0; e < 32; ++e) u32[e] = __float_as_uint(fs * v[e]);
              tmem_st32(tmem + lane_base + C::TM_ST + 32 * c, u32);
            }
          } else {
            if (!ws_wait(&bar[B_SPGO], (uint32_t)((i - 1) & 1), abort_flag)) break;
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < N / 32; ++c) {
              uint32_t u32[32];
              tmem_ld32(tmem + lane_base + C::TM_ST + 32 * c, u32);
              tmem_wait_ld();
              if constexpr (FULL) hb_store_row(sHB, pc, c, u32, fh);
#pragma unroll
              for (int e = 0; e < 16; ++e) {  // the rescale in f32x2 pairs, in place
                float a, b;
                f2_split(f2_mul(f2(fs, fs), f2(__uint_as_float(u32[2 * e]), __uint_as_float(u32[2 * e + 1]))), a, b);
                u32[2 * e] = __float_as_uint(a);
                u32[2 * e + 1] = __float_as_uint(b);
              }
              tmem_st32(tmem + lane_base + C::TM_ST + 32 * c, u32);
            }
          }
          tmem_wait_st();
          fence_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&bar[B_HF]);
            mbar_arrive(&bar[B_CE + cs]);
          }
          if (i + 1 < ntl) ok = build_xp(i + 1);
        }
        // ---- results: the state after the last tile
        bool go = ok && !*abort_flag && (!FULL || last_seg);
        if (go) go = ws_wait(&bar[B_SPGO], (uint32_t)((ntl - 1) & 1), abort_flag);
        if (FULL && go) go = ws_wait(&bar[B_FIN], 0, abort_flag);
        // the raw-input carry below synchronises the four state warps: they decide together
        if (FULL && last_seg && p.raw_inputs && bar_any(BAR_SPX, 128, !go)) go = false;
        if (go) {
          tc_fence_after();
          const float inv_rho = scal((ntl - 1) % WS_CS)[5];
          if constexpr (FULL) {
            // rotate back from the segment frame by the segment's total angle
            {
              float* hout = p.h + (int64_t)bh * N * WP;
#pragma unroll 1
              for (int c = 0; c < N / 32; ++c) {
                uint32_t sv[32];
                tmem_ld32(tmem + lane_base + C::TM_ST + 32 * c, sv);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                  const int k = 16 * c + e;
                  float sn, cn;
                  sincosf((float)base[k], &sn, &cn);
                  const float a0 = inv_rho * __uint_as_float(sv[2 * e]);
                  const float a1 = inv_rho * __uint_as_float(sv[2 * e + 1]);
                  hout[(int64_t)(2 * k) * WP + pc] = cn * a0 - sn * a1;
                  hout[(int64_t)(2 * k + 1) * WP + pc] = sn * a0 + cn * a1;
                }
              }
              // the carry: the last token's B (as the core used it: normalised when the operands are
              // raw) and raw x
              const int64_t tokl = tok_base + (L - 1);
              const __nv_bfloat16* Bg = static_cast<const __nv_bfloat16*>(p.B);
              const int64_t bc = ((tokl * G + g) * RR) * (int64_t)N;
              if (p.raw_inputs) {  // the rotation warps are done with rowss (B_FIN)
                if (pc < RR) rowss[pc] = 0.0f;
                named_bar_sync(BAR_SPX, 128);
                for (int k = pc; k < RR * N; k += WP) {
                  const float v = __bfloat162float(Bg[bc + k]);
                  atomicAdd(&rowss[k / N], v * v);
                }
                named_bar_sync(BAR_SPX, 128);
              }
              for (int k = pc; k < RR * N; k += WP) {
                float v = __bfloat162float(Bg[bc + k]);
                if (p.raw_inputs) v *= rsqrtf(rowss[k / N] * (1.0f / N) + kBcNormEps);
                p.carry_B[(int64_t)bh * RR * N + k] = v;
              }
              p.carry_x[(int64_t)bh * WP + pc] = __bfloat162float(xg[(tokl * H + hi) * (int64_t)WP + pc]);
            }
          } else {
            float* wh = sg.ws_h + ((int64_t)bh * sg.nsub + seg) * N * WP;
#pragma unroll 1
            for (int c = 0; c < N / 32; ++c) {
              uint32_t sv[32];
              tmem_ld32(tmem + lane_base + C::TM_ST + 32 * c, sv);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) wh[(int64_t)(32 * c + e) * WP + pc] = inv_rho * __uint_as_float(sv[e]);
            }
          }
        }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (tid == 0 && *abort_flag) set_status(p.status, M3_ERR_TIMEOUT);
  if (warp == W_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_COLS);
  }
}

}  // namespace

// ------------------------------------------------------------------ host side

bool ws_scan_supported(const Params& p) {
  if (p.dtype != M3_BF16 || p.P != WP || p.R < 1 || p.R > 8) return false;
  const int rt = tile_rank(p.R);
  if (p.N == 128) return rt == 4 || rt == 8;
  if (p.N == 64) return rt == 2 || rt == 4 || rt == 8;
  return false;
}

namespace {
template <int R, int N, int MODE>
cudaError_t launch_ws_mode(const CUtensorMap& tmB, const CUtensorMap& tmC, const CUtensorMap& tmX, const Params& p,
                           const SegInfo& sg, unsigned grid, cudaStream_t stream) {
  using Cf = WsCfg<R, N>;
  static SmemAttr attr;
  auto k = scan_ws_kernel<R, N, MODE>;
  cudaError_t e = attr.ensure(k, Cf::SMEM);
  if (e != cudaSuccess) return e;
  int per_sm = 0;  // one CTA must fit an SM (registers of the warps, rounded up, and shared memory)
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, WS_THREADS, Cf::SMEM);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorLaunchOutOfResources;
  k<<<grid, WS_THREADS, Cf::SMEM, stream>>>(tmB, tmC, tmX, p, sg);
  return cudaGetLastError();
}

template <int R, int N>
cudaError_t launch_ws_rn(const CUtensorMap& tmB, const CUtensorMap& tmC, const CUtensorMap& tmX, const Params& p,
                         const SegInfo& sg, cudaStream_t stream) {
  const int64_t nseq = p.b * p.H;
  if (sg.nseg > 1) {
    cudaError_t e = launch_ws_mode<R, N, WS_STATE>(tmB, tmC, tmX, p, sg, (unsigned)(nseq * sg.nsub), stream);
    if (e != cudaSuccess) return e;
  }
  return launch_ws_mode<R, N, WS_FULL>(tmB, tmC, tmX, p, sg, (unsigned)(nseq * sg.nseg), stream);
}
}  // namespace

cudaError_t launch_scan_ws_state(const CUtensorMap& tmB, const CUtensorMap& tmC, const CUtensorMap& tmX,
                                 const Params& p, const SegInfo& sg, cudaStream_t stream) {
  const unsigned grid = (unsigned)(p.b * p.H * sg.nsub);
  if (p.N == 128) return tile_rank(p.R) == 4 ? launch_ws_mode<4, 128, WS_STATE>(tmB, tmC, tmX, p, sg, grid, stream)
                                            : launch_ws_mode<8, 128, WS_STATE>(tmB, tmC, tmX, p, sg, grid, stream);
  switch (tile_rank(p.R)) {
    case 2: return launch_ws_mode<2, 64, WS_STATE>(tmB, tmC, tmX, p, sg, grid, stream);
    case 4: return launch_ws_mode<4, 64, WS_STATE>(tmB, tmC, tmX, p, sg, grid, stream);
    default: return launch_ws_mode<8, 64, WS_STATE>(tmB, tmC, tmX, p, sg, grid, stream);
  }
}

cudaError_t launch_scan_ws(const CUtensorMap& tmB, const CUtensorMap& tmC, const CUtensorMap& tmX, const Params& p,
                           const SegInfo& sg, cudaStream_t stream) {
  if (p.N == 128) return tile_rank(p.R) == 4 ? launch_ws_rn<4, 128>(tmB, tmC, tmX, p, sg, stream)
                                            : launch_ws_rn<8, 128>(tmB, tmC, tmX, p, sg, stream);
  switch (tile_rank(p.R)) {
    case 2: return launch_ws_rn<2, 64>(tmB, tmC, tmX, p, sg, stream);
    case 4: return launch_ws_rn<4, 64>(tmB, tmC, tmX, p, sg, stream);
    default: return launch_ws_rn<8, 64>(tmB, tmC, tmX, p, sg, stream);
  }
}

}  // namespace m3
