// m3_decode_tc.cu -- one-token decode on the tensor cores for d_state = headdim = 128, bf16 x/B/C.
//
// Same recurrence as m3_decode.cu (Mamba-3 paper note, docsaid.org, sections その1-その3):
//     h <- e^{dt A} Rot(phi) (h + (1 - lam) dt u_{t-1}) + lam dt u_t,   u = sum_r Bb_r X_r^T,
//     y = sum_r W_o[r] * (Cb_r^T h) + D x.
// Rotation acts on the state rows, so it commutes into the previous token's B:
//     h_new = alpha Rot(h) + Bcat Xcat^T,
//     Bcat = [gamma Bb_0 .. gamma Bb_{R-1} | alpha beta' Rot(Bb'_0) .. alpha beta' Rot(Bb'_{R-1})]  (N x 2R)
//     Xcat = [X_0 .. X_{R-1} | X'_0 .. X'_{R-1}]  (P x 2R),  X_r = W_x[r] x_t,  X'_r = W_x[r] x_{t-1}
// so the rank-2R update is one tcgen05.mma, D^T = Xcat Bcat^T (M = headdim 128, N = d_state 128,
// K = 16 >= 2R, bf16 operands, fp32 accumulator in tensor memory), and the R readouts are a
// second one, Y^T = h_new^T Cb (M = headdim, N = 16 >= R, K = d_state), from a bf16 copy of h_new.
// The threads do what is left per state element: h_new = alpha (c h_n -+ s h_n^1) + D[n][p] on
// the fp32 state (two FMAs), the bf16 copy for the readout, and the output sum over ranks.  Only
// the rank-2R increment and the readout see bf16 rounding; the carried state stays fp32.
//
// Persistent: one CTA per SM walks a contiguous range of (batch, head) units (head-major).  A
// producer warp streams their state tiles and token operands through two shared-memory stages
// (bulk copies on the TMA engine); the 16 compute warps update a tile in place, and the producer
// writes it back to HBM with one bulk store before refilling the stage, so neither the state
// loads nor the stores go through the threads' load/store path.  Every wait is bounded by
// %globaltimer; a timeout sets M3_ERR_TIMEOUT in the device status word, the CTA drains its
// copies, frees its tensor memory and returns.
#include "m3_common.cuh"

namespace m3 {
namespace {

__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Launch with programmatic stream serialisation (the kernels call griddepcontrol.wait before any
// global access).
template <typename Kernel, typename... Args>
cudaError_t launch_pdl(Kernel k, unsigned grid, unsigned block, size_t smem, cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, args...);
}

constexpr int kCT = 512;         // compute threads (16 warps)
constexpr int kT = kCT + 32;     // + one producer warp
constexpr int kN = 128;          // d_state
constexpr int kP = 128;          // headdim
constexpr int kStages = 2;
constexpr int kMaxR = 8;
constexpr unsigned kFull = 0xffffffffu;
constexpr unsigned long long kWaitNs = 2000000000ull;
// tensor memory: D^T in columns 0-127 (lane p, column n), the bf16 pairs of h_new^T in 128-191
// (lane p, column n / 2), Y^T in 192-207 (lane p, column r)
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColHB = 128, kColY = 192;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void sts128(uint32_t addr, const uint4& v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
// sin and cos after a two-constant Cody-Waite reduction of x to [-pi, pi] (2 pi split into an
// fp32 head and tail), then the hardware approximations on the reduced argument
__device__ __forceinline__ void sincos_reduced(float x, float* s, float* c) {
  const float n = rintf(x * 0.15915494309189535f);
  float r = fmaf(-n, 6.28318548202514648f, x);
  r = fmaf(-n, -1.7484555314695172e-7f, r);
  *s = __sinf(r);
  *c = __cosf(r);
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
// 16-byte chunk `ch` of row `row` in a 128-byte-swizzled tile: 128-byte rows per 64-element
// block, blocks `block_bytes` apart (TMA SWIZZLE_128B / UMMA SW128 layout)
__device__ __forceinline__ uint32_t sw128(int row, int ch, uint32_t block_bytes) {
  return (uint32_t)(ch >> 3) * block_bytes + (uint32_t)row * 128u + ((uint32_t)((ch & 7) ^ (row & 7)) << 4);
}
// shared-memory matrix descriptor, 128-byte swizzle (sm_100 descriptor version 1)
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// instruction descriptor, kind::f16: bf16 x bf16 -> fp32, dense
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// warp-collective: every lane executes, the lane elect.sync picks issues
__device__ __forceinline__ void mma_ss_w(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p, e;\n .reg .b32 r;\n elect.sync r|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void mma_ts_w(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p, e;\n .reg .b32 r;\n elect.sync r|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d),
      "r"(a), "l"(b), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void mma_commit_w(uint32_t bar) {
  asm volatile(
      "{\n .reg .pred e;\n .reg .b32 r;\n elect.sync r|e, 0xffffffff;\n"
      " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n}\n" ::"r"(bar)
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
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::
          "r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]));
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void bulk_s2g(void* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// barrier 1: the compute warps only (the producer warp never joins it)
__device__ __forceinline__ void compute_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory"); }
__device__ __forceinline__ bool compute_sync_or(bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, 1, %2, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(kCT)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// shared memory plan (bytes): the swizzled operand tiles first (1024-aligned), then the stages
struct TcPlan {
  uint32_t stage_bytes;
  uint32_t o_st, o_b, o_c, o_cb, o_x, o_cx, o_th, o_sc;  // inside a stage
  uint32_t o_bx;    // Bcat (k-chunks 0-1) and Xcat (k-chunks 2-3) of a 128-row SW128 K-major tile
  uint32_t o_cbt;   // bf16 Cb, K-major SW128 (16 rows r, 64-element blocks of n), one per stage
  uint32_t o_cs;    // rotation table of the unit, (alpha cos, alpha sin) per pair
  uint32_t o_xr;    // x_t of the unit, one copy per stage (read by the output after the stage is reused)
  uint32_t o_w;     // bias_B, bias_C, W_x, W_o of the current head, fp32
  uint32_t o_tm, o_bar, o_stage0;
  uint32_t total;
};

__host__ __device__ inline uint32_t pad16(uint32_t x) { return (x + 15u) & ~15u; }

inline TcPlan tc_plan(int R) {
  TcPlan t{};
  uint32_t f = 0;
  t.o_bx = f;  f += 128 * 128;
  t.o_cbt = f; f += kStages * 2 * 16 * 128;
  t.o_cs = f;  f += kN / 2 * 8;
  t.o_xr = f;  f += kStages * kP * 4;
  t.o_w = f;   f += 4u * (uint32_t)R * kN * 4;
  t.o_tm = f;  f += 16;
  t.o_bar = f; f += 8 * (2 * kStages + 2);
  t.o_stage0 = (f + 127u) & ~127u;
  uint32_t o = 0;
  t.o_st = o; o += kN * kP * 4;
  t.o_b = o;  o += pad16((uint32_t)R * kN * 2);
  t.o_c = o;  o += pad16((uint32_t)R * kN * 2);
  t.o_cb = o; o += pad16((uint32_t)R * kN * 4);
  t.o_x = o;  o += pad16((uint32_t)kP * 2);
  t.o_cx = o; o += pad16((uint32_t)kP * 4);
  t.o_th = o; o += pad16((uint32_t)kN / 2 * 4);
  t.o_sc = o; o += 16;
  t.stage_bytes = (o + 127u) & ~127u;
  t.total = t.o_stage0 + kStages * t.stage_bytes + 1024;  // slack for aligning the base to 1024 bytes
  return t;
}

template <int RT>
__global__ void __launch_bounds__(kT, 1) decode_tc_kernel(Params p, TcPlan tp) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = p.H, R = p.R, G = p.G;
  const int64_t nb = p.b;
  const int64_t U = nb * H;
  const int64_t u0 = (int64_t)blockIdx.x * U / gridDim.x;
  const int64_t u1 = (int64_t)(blockIdx.x + 1) * U / gridDim.x;
  const int64_t nu = u1 - u0;
  const uint32_t sbase = smem_u32(sm);
  const uint32_t full0 = sbase + tp.o_bar;            // stage landed (expect_tx + the scalar copies)
  const uint32_t empty0 = full0 + 8u * kStages;       // stage read and rewritten by the compute warps
  const uint32_t mma1_bar = empty0 + 8u * kStages;    // update MMA completion
  const uint32_t mma2_bar = mma1_bar + 8u;            // readout MMA completion
  float2* cs = reinterpret_cast<float2*>(sm + tp.o_cs);
  float* xr = reinterpret_cast<float*>(sm + tp.o_xr);
  float* wb = reinterpret_cast<float*>(sm + tp.o_w);
  float* wc = wb + R * kN;
  float* wx = wc + R * kN;
  float* wo = wx + R * kP;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + tp.o_tm);
  const uint32_t sBX = sbase + tp.o_bx, sCB = sbase + tp.o_cbt;
  const int hpg = H / G;

  auto try_wait = [&](uint32_t bar, uint32_t par) -> bool {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred q;\n mbarrier.try_wait.parity.shared::cta.b64 q, [%1], %2;\n selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(done)
        : "r"(bar), "r"(par)
        : "memory");
    return done != 0;
  };
  auto wait = [&](uint32_t bar, uint32_t par) -> bool {
    if (try_wait(bar, par)) return true;
    const uint64_t t0 = globaltimer();
    while (!try_wait(bar, par)) {
      if (globaltimer() - t0 > kWaitNs) return false;
    }
    return true;
  };

  // Programmatic dependent launch: the next decode step may start its set-up (tensor memory,
  // barriers) while this one runs; every global access of a step comes after its griddepcontrol.wait,
  // which returns once the previous kernel of the stream has finished and its writes are visible.
  griddep_launch_dependents();
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
  }
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 2;" ::"r"(full0 + 8u * s));
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(empty0 + 8u * s));
    }
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(mma1_bar));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(mma2_bar));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_wait();

  if (warp == kCT / 32) {
    // ---- producer: the state and token operands of unit j into stage j % 2, once the compute
    //      warps are done with unit j - 2 there and its new state has been stored from it
    if (lane == 0) {
      const uint32_t n_st = kN * kP * 4, n_b = (uint32_t)R * kN * 2, n_cb = (uint32_t)R * kN * 4;
      int64_t bl = u0 % nb, bs = u0 % nb;  // sequence and head of the next load and the next store
      int hl = (int)(u0 / nb), hs = (int)(u0 / nb);
      bool pok = true;
      int64_t j = 0;
      for (; j < nu + kStages; ++j) {
        const int st = (int)(j & 1);
        const uint32_t sst = sbase + tp.o_stage0 + (uint32_t)st * tp.stage_bytes;
        if (j >= kStages) {
          pok = wait(empty0 + 8u * st, (uint32_t)((j - kStages) >> 1) & 1u);
          if (!pok) break;
          bulk_s2g(p.h + (bs * H + hs) * (int64_t)(kN * kP), sst + tp.o_st, n_st);
          if (++bs == nb) { bs = 0; ++hs; }
        }
        if (j >= nu) continue;
        if (j >= kStages) bulk_wait_read();  // the store has read the stage
        const int g = hl / hpg;
        const int64_t bh = bl * H + hl;
        const uint32_t bar = full0 + 8u * st;
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
                     "r"(n_st + 2 * n_b + n_cb + kP * 2 + kP * 4 + kN / 2 * 4)
                     : "memory");
        const int64_t bc = ((bl * G + g) * R) * (int64_t)kN;
        bulk_g2s(sst + tp.o_st, p.h + bh * kN * kP, n_st, bar);
        bulk_g2s(sst + tp.o_b, static_cast<const __nv_bfloat16*>(p.B) + bc, n_b, bar);
        bulk_g2s(sst + tp.o_c, static_cast<const __nv_bfloat16*>(p.C) + bc, n_b, bar);
        bulk_g2s(sst + tp.o_cb, p.carry_B + bh * R * kN, n_cb, bar);
        bulk_g2s(sst + tp.o_x, static_cast<const __nv_bfloat16*>(p.x) + bh * kP, kP * 2, bar);
        bulk_g2s(sst + tp.o_cx, p.carry_x + bh * kP, kP * 4, bar);
        bulk_g2s(sst + tp.o_th, p.theta + (bl * G + g) * (kN / 2), kN / 2 * 4, bar);
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(sst + tp.o_sc), "l"(p.dt + bh) : "memory");
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(sst + tp.o_sc + 4), "l"(p.A + bh) : "memory");
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(sst + tp.o_sc + 8), "l"(p.lam + bh) : "memory");
        asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
        if (++bl == nb) { bl = 0; ++hl; }
      }
      if (!pok) {
        // the compute warps gave up: wait (bounded) for the last load issued into each stage
        const int64_t issued = j < nu ? j : nu;
        for (int64_t w = issued - kStages < 0 ? 0 : issued - kStages; w < issued; ++w)
          wait(full0 + 8u * (uint32_t)(w & 1), (uint32_t)(w >> 1) & 1u);
        set_status(p.status, M3_ERR_TIMEOUT);
      }
      bulk_wait_all();
    }
    __syncwarp();
  } else {
    // ---- compute warps.  Per unit: operands (warps 0-3 Bcat and the rotation table, 4-7 Xcat,
    //      8-11 Cb and the carry), the update MMA, the update (all), then warps 12-15 issue the
    //      readout MMA and write y while warps 0-11 go on to the next unit's operands
    const uint32_t tmem = __shfl_sync(kFull, *tmem_slot, 0);
    const int q4 = warp & 3;          // TMEM lane quarter: columns p = 32 q4 .. 32 q4 + 31
    const int rq = warp >> 2;         // state rows n = 32 rq .. 32 rq + 31 in the update
    const int pp = 32 * q4 + lane;
    const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
    constexpr uint32_t ID_UPD = idesc_bf16(kP, kN, false, false);  // D^T = Xcat Bcat^T
    constexpr uint32_t ID_RD = idesc_bf16(kP, 16, false, false);   // Y^T = h_new^T Cb
    constexpr int K2 = 2 * RT;                                      // columns of Bcat and Xcat in use
    // zero padding, written once: k-chunks 1 and 3 of the Bcat/Xcat tile when 2R <= 8, and the rows
    // r >= R of both Cb tiles
    if (K2 <= 8 && tid < 2 * kN) sts128(sBX + sw128(tid & 127, (tid >> 7) ? 3 : 1, 128 * 128), make_uint4(0, 0, 0, 0));
    for (int i = tid; i < kStages * (16 - RT) * 16; i += kCT) {
      const int st = i / ((16 - RT) * 16), rr = RT + (i / 16) % (16 - RT), nc = i & 15;
      sts128(sCB + (uint32_t)st * (2 * 16 * 128) + sw128(rr, nc, 16 * 128), make_uint4(0, 0, 0, 0));
    }

    int cur_h = -1;
    float Dh = 0.0f;
    bool ok = true, mfail = false;
    int64_t bi = u0 % nb;
    int hi = (int)(u0 / nb);
    for (int64_t j = 0; j < nu; ++j) {
      const int s = (int)(j & 1);
      const uint32_t par = (uint32_t)(j >> 1) & 1u, mpar = (uint32_t)j & 1u;
      const uint32_t sCBs = sCB + (uint32_t)s * (2 * 16 * 128);
      const int64_t bh = bi * H + hi;
      uint8_t* stg = sm + tp.o_stage0 + (size_t)s * tp.stage_bytes;
      float* hst = reinterpret_cast<float*>(stg + tp.o_st);
      if (hi != cur_h) {  // weights of a new head (uniform: every thread sees the same unit)
        cur_h = hi;
        compute_sync();  // the previous unit's output has read W_o
        const float* biasB = p.bias_B ? p.bias_B + (int64_t)hi * R * kN : nullptr;
        const float* biasC = p.bias_C ? p.bias_C + (int64_t)hi * R * kN : nullptr;
        const float* Wx = p.W_x ? p.W_x + (int64_t)hi * R * kP : nullptr;
        const float* Wo = p.W_o ? p.W_o + (int64_t)hi * R * kP : nullptr;
        for (int i = tid; i < R * kN; i += kCT) {
          wb[i] = biasB ? biasB[i] : 0.0f;
          wc[i] = biasC ? biasC[i] : 0.0f;
          wx[i] = Wx ? Wx[i] : 1.0f;
          wo[i] = Wo ? Wo[i] : 1.0f;
        }
        Dh = p.D ? p.D[hi] : 0.0f;
        compute_sync();
      }
      ok = wait(full0 + 8u * s, par);
      float hv[32];
      // ---- operands of the two MMAs (bf16), the rotation table, the new carry, and this
      //      thread's state rows
      if (ok) {
        const float* sc = reinterpret_cast<const float*>(stg + tp.o_sc);
        const float delta = sc[0], lm = sc[2];
        if (warp < 4) {
          // Bcat row n: gamma Bb_k for k < R, alpha beta' Rot(Bb'_{k-R}) for R <= k < 2R
          const __nv_bfloat16* Braw = reinterpret_cast<const __nv_bfloat16*>(stg + tp.o_b);
          const float* cBs = reinterpret_cast<const float*>(stg + tp.o_cb);
          const float* ths = reinterpret_cast<const float*>(stg + tp.o_th);
          const int n = tid, n0 = n & ~1;
          const float alpha = expf(delta * sc[1]);
          float sn, cn;
          sincos_reduced(p.angle_direct ? ths[n >> 1] : delta * ths[n >> 1], &sn, &cn);
          if ((n & 1) == 0) cs[n >> 1] = make_float2(alpha * cn, alpha * sn);
          const float gm = lm * delta, ab = alpha * (1.0f - lm) * delta;
          float fb[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) fb[k] = 0.0f;
#pragma unroll
          for (int k = 0; k < RT; ++k) {
            fb[k] = gm * (__bfloat162float(Braw[k * kN + n]) + wb[k * kN + n]);
            const float2 cv = *reinterpret_cast<const float2*>(cBs + k * kN + n0);
            const float2 bv = *reinterpret_cast<const float2*>(wb + k * kN + n0);
            const float v0 = cv.x + bv.x, v1 = cv.y + bv.y;
            fb[RT + k] = ab * ((n & 1) ? fmaf(sn, v0, cn * v1) : fmaf(cn, v0, -sn * v1));
          }
          sts128(sBX + sw128(n, 0, 128 * 128),
                 make_uint4(pack_bf16(fb[0], fb[1]), pack_bf16(fb[2], fb[3]), pack_bf16(fb[4], fb[5]),
                            pack_bf16(fb[6], fb[7])));
          if (K2 > 8)
            sts128(sBX + sw128(n, 1, 128 * 128),
                   make_uint4(pack_bf16(fb[8], fb[9]), pack_bf16(fb[10], fb[11]), pack_bf16(fb[12], fb[13]),
                              pack_bf16(fb[14], fb[15])));
        } else if (warp < 8) {
          // Xcat row p: W_x[k] x_t for k < R, W_x[k-R] x_{t-1} for R <= k < 2R; x_t for the output
          // and the new carry
          const __nv_bfloat16* xraw = reinterpret_cast<const __nv_bfloat16*>(stg + tp.o_x);
          const float* cxs = reinterpret_cast<const float*>(stg + tp.o_cx);
          const int row = tid - kP;
          const float xv = __bfloat162float(xraw[row]), cxv = cxs[row];
          float fx[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) fx[k] = 0.0f;
#pragma unroll
          for (int k = 0; k < RT; ++k) {
            const float w = wx[k * kP + row];
            fx[k] = w * xv;
            fx[RT + k] = w * cxv;
          }
          sts128(sBX + sw128(row, 2, 128 * 128),
                 make_uint4(pack_bf16(fx[0], fx[1]), pack_bf16(fx[2], fx[3]), pack_bf16(fx[4], fx[5]),
                            pack_bf16(fx[6], fx[7])));
          if (K2 > 8)
            sts128(sBX + sw128(row, 3, 128 * 128),
                   make_uint4(pack_bf16(fx[8], fx[9]), pack_bf16(fx[10], fx[11]), pack_bf16(fx[12], fx[13]),
                              pack_bf16(fx[14], fx[15])));
          xr[s * kP + row] = xv;
          p.carry_x[bh * kP + row] = xv;
        } else if (warp < 12) {
          // Cb rows r < R, eight elements of n per thread; the new carry: this token's raw B (the
          // old one is in the stage)
          const __nv_bfloat16* Braw = reinterpret_cast<const __nv_bfloat16*>(stg + tp.o_b);
          const __nv_bfloat16* Craw = reinterpret_cast<const __nv_bfloat16*>(stg + tp.o_c);
          const int t = tid - 2 * kP;
          if (t < 16 * RT) {
            const int r = t >> 4, nc = t & 15;
            const uint4 craw = *reinterpret_cast<const uint4*>(Craw + r * kN + 8 * nc);
            const float4 w0 = *reinterpret_cast<const float4*>(wc + r * kN + 8 * nc);
            const float4 w1 = *reinterpret_cast<const float4*>(wc + r * kN + 8 * nc + 4);
            const __nv_bfloat162* c2 = reinterpret_cast<const __nv_bfloat162*>(&craw);
            const float2 c01 = __bfloat1622float2(c2[0]), c23 = __bfloat1622float2(c2[1]);
            const float2 c45 = __bfloat1622float2(c2[2]), c67 = __bfloat1622float2(c2[3]);
            sts128(sCBs + sw128(r, nc, 16 * 128),
                   make_uint4(pack_bf16(c01.x + w0.x, c01.y + w0.y), pack_bf16(c23.x + w0.z, c23.y + w0.w),
                              pack_bf16(c45.x + w1.x, c45.y + w1.y), pack_bf16(c67.x + w1.z, c67.y + w1.w)));
          }
          float* cBg = p.carry_B + bh * R * kN;
#pragma unroll
          for (int k = 0; k < RT; ++k) cBg[k * kN + t] = __bfloat162float(Braw[k * kN + t]);
        }
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) hv[jj] = hst[(32 * rq + jj) * kP + pp];
      }
      fence_async_smem();
      tc_fence_before();
      if (compute_sync_or(!ok || mfail)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // ---- MMA 1: D^T = Xcat Bcat^T (one K = 16 step): TMEM lane p, column n.  Every thread waits
      //      for it; a timeout is reported at the update's barrier
      if (warp == 0) {
        mma_ss_w(tmem, sdesc(sBX + 32, 16, 1024), sdesc(sBX, 16, 1024), ID_UPD, 0);
        mma_commit_w(mma1_bar);
      }
      const bool okm = wait(mma1_bar, mpar);
      tc_fence_after();
      // ---- update: h_new[n][p] = alpha (c h_n -+ s h_n^1) + D[n][p]; thread = column p (TMEM lane)
      //      over rows 32 rq .. 32 rq + 31, a rotation pair in one thread.  The new state goes back
      //      into the stage in place (the producer stores the tile to HBM) and, as bf16 pairs,
      //      into tensor memory for the readout
      if (okm) {
        const int n0 = 32 * rq;
        uint32_t dv[32];
        tmem_ld32(tmem + lane_base + n0, dv);
        tmem_wait_ld();
        uint32_t hb[16];
        const float4* cs4 = reinterpret_cast<const float4*>(cs + n0 / 2);
#pragma unroll
        for (int jj = 0; jj < 16; jj += 2) {
          const float4 rc = cs4[jj / 2];  // (alpha cos, alpha sin) of pairs jj and jj + 1
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int i = jj + hh;
            const float ac = hh ? rc.z : rc.x, as = hh ? rc.w : rc.y;
            const float e0 = fmaf(ac, hv[2 * i], fmaf(-as, hv[2 * i + 1], __uint_as_float(dv[2 * i])));
            const float e1 = fmaf(as, hv[2 * i], fmaf(ac, hv[2 * i + 1], __uint_as_float(dv[2 * i + 1])));
            hst[(n0 + 2 * i) * kP + pp] = e0;
            hst[(n0 + 2 * i + 1) * kP + pp] = e1;
            hb[i] = pack_bf16(e0, e1);
          }
        }
        tmem_st16(tmem + lane_base + kColHB + n0 / 2, hb);
        tmem_wait_st();
      }
      fence_async_smem();
      tc_fence_before();
      if (compute_sync_or(!okm)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // the stage holds the new state and nothing reads it again: hand it to the producer
      if (tid == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(empty0 + 8u * s) : "memory");
      if (warp >= 12) {
        // ---- MMA 2: Y^T = h_new^T Cb (K = 128 in steps of 16, h_new^T from tensor memory)
        if (warp == 12) {
#pragma unroll
          for (int k = 0; k < kN / 16; ++k)
            mma_ts_w(tmem + kColY, tmem + kColHB + 8 * k,
                     sdesc(sCBs + (uint32_t)(k >> 2) * (16 * 128) + (uint32_t)(k & 3) * 32, 16, 1024), ID_RD,
                     k > 0);
          mma_commit_w(mma2_bar);
        }
        // ---- y[p] = sum_r W_o[r][p] Y^T[p][r] + D x[p] (TMEM lane p).  Cb has one tile per stage,
        //      and the next unit's barriers order these reads before anything else they read is
        //      rewritten; a timeout is reported at the next barrier
        mfail = !wait(mma2_bar, mpar);
        tc_fence_after();
        if (!mfail) {
          uint32_t yv[32];
          tmem_ld32(tmem + lane_base + kColY, yv);
          tmem_wait_ld();
          float acc = Dh * xr[s * kP + pp];
#pragma unroll
          for (int r = 0; r < RT; ++r) acc = fmaf(wo[r * kP + pp], __uint_as_float(yv[r]), acc);
          reinterpret_cast<__nv_bfloat16*>(p.y)[bh * kP + pp] = __float2bfloat16_rn(acc);
        }
      }
      if (++bi == nb) { bi = 0; ++hi; }
    }
    if (lane == 0 && (!ok || mfail)) set_status(p.status, M3_ERR_TIMEOUT);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_slot[0]), "r"(kTmemCols));
  }
}

// SM count and opt-in shared memory per block of the current device, queried once per device
struct TcDevice {
  int sms = 0, optin = 0;
};
TcDevice tc_device() {
  static PerDevice<TcDevice> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TcDevice{};
  TcDevice out{};
  cache.get(dev, &out, [dev](TcDevice* d) {
    int sms = 0, optin = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
      return false;
    d->sms = sms;
    d->optin = optin;
    return true;
  });
  return out;
}

template <int RT>
cudaError_t launch_tc_rt(const Params& p, const TcPlan& tp, unsigned grid, cudaStream_t stream) {
  static SmemAttr smem_set;
  auto k = decode_tc_kernel<RT>;
  cudaError_t e = smem_set.ensure(k, (int)tp.total);
  if (e != cudaSuccess) return e;
  e = launch_pdl(k, grid, kT, tp.total, stream, p, tp);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// ------------------------------------------------------------------ split form (few units)
// Few (batch, head) units leave most SMs idle in the persistent form.  Here a cluster of four CTAs
// takes one unit, each CTA 32 state rows: the rank-2R increment of its rows (D^T = Xcat
// Bcat_slice^T, M = 128, N = 32), their update, and their part of the readouts (Y^T =
// h_slice^T Cb_slice, K = 32).  The four partial outputs sum_r W_o[r] Y^T meet in CTA 0 through
// distributed shared memory; the new state goes straight from registers to HBM.
constexpr int kSplit = 4;                  // CTAs per unit (cluster size)
constexpr int kRows = kN / kSplit;         // state rows per CTA
constexpr int kST = 128;                   // threads per CTA: thread = column p
constexpr uint32_t kSplitTmemCols = 64;    // D^T 0-31, bf16 pairs of h_new^T 32-47, Y^T 48-63
constexpr uint32_t kSColHB = 32, kSColY = 48;
// The split form takes a decode call whose CTAs fit in one wave (kSplit x units <= SMs: batch 1 at
// 32 heads, 5.5 vs 6.8 us per step on B200); beyond that the persistent form is faster (batch 16:
// 15.3 vs 25.5 us).

struct SplitPlan {
  uint32_t o_x;     // Xcat: 128 rows, SW128 K-major (chunks 0-1 used)
  uint32_t o_b;     // Bcat of the slice: 32 rows, SW128 K-major
  uint32_t o_cb;    // Cb of the slice: 16 rows, SW128 K-major (the first 32 of 64 K-elements used)
  uint32_t o_st;    // state rows of the slice, fp32 [32][128]
  uint32_t o_braw, o_craw, o_cbold, o_xraw, o_cx, o_th;  // token operands of the unit
  uint32_t o_cs, o_yp, o_tm, o_bar;
  uint32_t total;
};

inline SplitPlan split_plan(int R) {
  SplitPlan t{};
  uint32_t f = 0;
  t.o_x = f;     f += 128 * 128;
  t.o_b = f;     f += kRows * 128;
  t.o_cb = f;    f += 16 * 128;
  t.o_st = f;    f += kRows * kP * 4;
  t.o_braw = f;  f += pad16((uint32_t)R * kN * 2);
  t.o_craw = f;  f += pad16((uint32_t)R * kN * 2);
  t.o_cbold = f; f += pad16((uint32_t)R * kN * 4);
  t.o_xraw = f;  f += pad16((uint32_t)kP * 2);
  t.o_cx = f;    f += pad16((uint32_t)kP * 4);
  t.o_th = f;    f += pad16((uint32_t)kN / 2 * 4);
  t.o_cs = f;    f += kRows / 2 * 8;
  t.o_yp = f;    f += kP * 4;
  t.o_tm = f;    f += 16;
  t.o_bar = f;   f += 16;
  t.total = f + 1024;  // slack for aligning the base to 1024 bytes
  return t;
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// a float of CTA `rank`'s shared memory at this CTA's shared address `addr`
__device__ __forceinline__ float ld_dsmem(uint32_t addr, uint32_t rank) {
  uint32_t ra;
  float v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(addr), "r"(rank));
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra) : "memory");
  return v;
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}

template <int RT>
__global__ void __cluster_dims__(kSplit, 1, 1) __launch_bounds__(kST, 1)
    decode_tc_split_kernel(Params p, SplitPlan sp) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = p.H, R = p.R, G = p.G;
  const uint32_t crank = cluster_rank();
  const int64_t nb = p.b;
  const int64_t u = blockIdx.x / kSplit;
  const int64_t bi = u % nb;
  const int hi = (int)(u / nb);
  const int g = hi / (H / G);
  const int64_t bh = bi * H + hi;
  const int n0 = kRows * (int)crank;  // first state row of this CTA
  const uint32_t sbase = smem_u32(sm);
  const uint32_t sX = sbase + sp.o_x, sB = sbase + sp.o_b, sC = sbase + sp.o_cb;
  const uint32_t full = sbase + sp.o_bar, mbar = full + 8;
  const float* hst = reinterpret_cast<const float*>(sm + sp.o_st);
  const __nv_bfloat16* Braw = reinterpret_cast<const __nv_bfloat16*>(sm + sp.o_braw);
  const __nv_bfloat16* Craw = reinterpret_cast<const __nv_bfloat16*>(sm + sp.o_craw);
  const float* cBs = reinterpret_cast<const float*>(sm + sp.o_cbold);
  const __nv_bfloat16* xraw = reinterpret_cast<const __nv_bfloat16*>(sm + sp.o_xraw);
  const float* cxs = reinterpret_cast<const float*>(sm + sp.o_cx);
  const float* ths = reinterpret_cast<const float*>(sm + sp.o_th);
  float2* cs = reinterpret_cast<float2*>(sm + sp.o_cs);
  float* yp = reinterpret_cast<float*>(sm + sp.o_yp);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + sp.o_tm);

  auto try_wait = [&](uint32_t bar, uint32_t par) -> bool {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred q;\n mbarrier.try_wait.parity.shared::cta.b64 q, [%1], %2;\n selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(done)
        : "r"(bar), "r"(par)
        : "memory");
    return done != 0;
  };
  auto wait = [&](uint32_t bar, uint32_t par) -> bool {
    if (try_wait(bar, par)) return true;
    const uint64_t t0 = globaltimer();
    while (!try_wait(bar, par)) {
      if (globaltimer() - t0 > kWaitNs) return false;
    }
    return true;
  };

  // programmatic dependent launch, as in the persistent form: set-up before the wait, every global
  // access after it
  griddep_launch_dependents();
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kSplitTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
  }
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(full));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(mbar));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  griddep_wait();
  if (tid == 0) {
    const uint32_t n_st = kRows * kP * 4, n_b = (uint32_t)R * kN * 2, n_cb = (uint32_t)R * kN * 4;
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(full),
                 "r"(n_st + 2 * n_b + n_cb + kP * 2 + kP * 4 + kN / 2 * 4)
                 : "memory");
    const int64_t bc = ((bi * G + g) * R) * (int64_t)kN;
    bulk_g2s(sbase + sp.o_st, p.h + (bh * kN + n0) * kP, n_st, full);
    bulk_g2s(sbase + sp.o_braw, static_cast<const __nv_bfloat16*>(p.B) + bc, n_b, full);
    bulk_g2s(sbase + sp.o_craw, static_cast<const __nv_bfloat16*>(p.C) + bc, n_b, full);
    bulk_g2s(sbase + sp.o_cbold, p.carry_B + bh * R * kN, n_cb, full);
    bulk_g2s(sbase + sp.o_xraw, static_cast<const __nv_bfloat16*>(p.x) + bh * kP, kP * 2, full);
    bulk_g2s(sbase + sp.o_cx, p.carry_x + bh * kP, kP * 4, full);
    bulk_g2s(sbase + sp.o_th, p.theta + (bi * G + g) * (kN / 2), kN / 2 * 4, full);
  }
  // per-unit scalars and this thread's weights while the copies land
  const float delta = __ldg(p.dt + bh), lm = __ldg(p.lam + bh);
  const float alpha = expf(delta * __ldg(p.A + bh));
  float wxr[RT], wor[RT];
#pragma unroll
  for (int k = 0; k < RT; ++k) {
    wxr[k] = p.W_x ? __ldg(p.W_x + ((int64_t)hi * R + k) * kP + tid) : 1.0f;
    wor[k] = p.W_o ? __ldg(p.W_o + ((int64_t)hi * R + k) * kP + tid) : 1.0f;
  }
  const float Dh = p.D ? __ldg(p.D + hi) : 0.0f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = (uint32_t)(32 * warp) << 16;

  bool ok = wait(full, 0);
  ok = !__syncthreads_or(!ok);
  float hv[kRows];
  if (ok) {
    // Xcat row p = tid: W_x[k] x_t for k < R, W_x[k-R] x_{t-1} for R <= k < 2R
    {
      const float xv = __bfloat162float(xraw[tid]), cxv = cxs[tid];
      float fx[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) fx[k] = 0.0f;
#pragma unroll
      for (int k = 0; k < RT; ++k) {
        fx[k] = wxr[k] * xv;
        fx[RT + k] = wxr[k] * cxv;
      }
      sts128(sX + sw128(tid, 0, 128 * 128),
             make_uint4(pack_bf16(fx[0], fx[1]), pack_bf16(fx[2], fx[3]), pack_bf16(fx[4], fx[5]), pack_bf16(fx[6], fx[7])));
      sts128(sX + sw128(tid, 1, 128 * 128),
             make_uint4(pack_bf16(fx[8], fx[9]), pack_bf16(fx[10], fx[11]), pack_bf16(fx[12], fx[13]),
                        pack_bf16(fx[14], fx[15])));
    }
    if (warp == 0) {
      // Bcat row n = n0 + lane: gamma Bb_k for k < R, alpha beta' Rot(Bb'_{k-R}) for R <= k < 2R
      const int n = n0 + lane, m = n & ~1;
      float sn, cn;
      sincos_reduced(p.angle_direct ? ths[n >> 1] : delta * ths[n >> 1], &sn, &cn);
      if ((lane & 1) == 0) cs[lane >> 1] = make_float2(alpha * cn, alpha * sn);
      const float gm = lm * delta, ab = alpha * (1.0f - lm) * delta;
      const float* bB = p.bias_B ? p.bias_B + (int64_t)hi * R * kN : nullptr;
      float fb[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) fb[k] = 0.0f;
#pragma unroll
      for (int k = 0; k < RT; ++k) {
        const float b0 = bB ? __ldg(bB + k * kN + m) : 0.0f, b1 = bB ? __ldg(bB + k * kN + m + 1) : 0.0f;
        const float bn = (n & 1) ? b1 : b0;
        fb[k] = gm * (__bfloat162float(Braw[k * kN + n]) + bn);
        const float v0 = cBs[k * kN + m] + b0, v1 = cBs[k * kN + m + 1] + b1;
        fb[RT + k] = ab * ((n & 1) ? fmaf(sn, v0, cn * v1) : fmaf(cn, v0, -sn * v1));
      }
      sts128(sB + sw128(lane, 0, kRows * 128),
             make_uint4(pack_bf16(fb[0], fb[1]), pack_bf16(fb[2], fb[3]), pack_bf16(fb[4], fb[5]), pack_bf16(fb[6], fb[7])));
      sts128(sB + sw128(lane, 1, kRows * 128),
             make_uint4(pack_bf16(fb[8], fb[9]), pack_bf16(fb[10], fb[11]), pack_bf16(fb[12], fb[13]),
                        pack_bf16(fb[14], fb[15])));
    } else if (warp == 1) {
      // Cb of the slice: rows r < 16 (zero for r >= R), chunks of 8 elements of n
      const float* bC = p.bias_C ? p.bias_C + (int64_t)hi * R * kN : nullptr;
      for (int it = lane; it < 16 * (kRows / 8); it += 32) {
        const int r = it / (kRows / 8), nc = it % (kRows / 8);
        float fc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int n = n0 + 8 * nc + e;
          fc[e] = r < R ? __bfloat162float(Craw[r * kN + n]) + (bC ? __ldg(bC + r * kN + n) : 0.0f) : 0.0f;
        }
        sts128(sC + sw128(r, nc, 16 * 128),
               make_uint4(pack_bf16(fc[0], fc[1]), pack_bf16(fc[2], fc[3]), pack_bf16(fc[4], fc[5]),
                          pack_bf16(fc[6], fc[7])));
      }
    }
#pragma unroll
    for (int j = 0; j < kRows; ++j) hv[j] = hst[j * kP + tid];
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // ---- MMA 1: D^T = Xcat Bcat_slice^T (M = 128, N = 32, K = 16)
  if (ok && warp == 0) {
    mma_ss_w(tmem, sdesc(sX, 16, 1024), sdesc(sB, 16, 1024), idesc_bf16(kP, kRows, false, false), 0);
    mma_commit_w(mbar);
  }
  bool okm = ok ? wait(mbar, 0) : false;
  tc_fence_after();
  if (okm) {
    uint32_t dv[32];
    tmem_ld32(tmem + lane_base, dv);
    tmem_wait_ld();
    float* hg = p.h + (bh * kN + n0) * kP + tid;
    const float4* cs4 = reinterpret_cast<const float4*>(cs);
    uint32_t hb[16];
#pragma unroll
    for (int jj = 0; jj < 16; jj += 2) {
      const float4 rc = cs4[jj / 2];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int i = jj + hh;
        const float ac = hh ? rc.z : rc.x, as = hh ? rc.w : rc.y;
        const float e0 = fmaf(ac, hv[2 * i], fmaf(-as, hv[2 * i + 1], __uint_as_float(dv[2 * i])));
        const float e1 = fmaf(as, hv[2 * i], fmaf(ac, hv[2 * i + 1], __uint_as_float(dv[2 * i + 1])));
        hg[(2 * i) * kP] = e0;
        hg[(2 * i + 1) * kP] = e1;
        hb[i] = pack_bf16(e0, e1);
      }
    }
    tmem_st16(tmem + lane_base + kSColHB, hb);
    tmem_wait_st();
  }
  tc_fence_before();
  okm = !__syncthreads_or(!okm);
  tc_fence_after();
  // ---- MMA 2: partial Y^T = h_slice^T Cb_slice (K = 32, h from tensor memory)
  if (okm && warp == 0) {
#pragma unroll
    for (int k = 0; k < kRows / 16; ++k)
      mma_ts_w(tmem + kSColY, tmem + kSColHB + 8 * k, sdesc(sC + 32 * k, 16, 1024), idesc_bf16(kP, 16, false, false),
               k > 0);
    mma_commit_w(mbar);
  }
  const bool okm2 = okm ? wait(mbar, 1) : false;
  tc_fence_after();
  if (okm2) {
    uint32_t yv[16];
    tmem_ld16(tmem + lane_base + kSColY, yv);
    tmem_wait_ld();
    float acc = 0.0f;
#pragma unroll
    for (int r = 0; r < RT; ++r) acc = fmaf(wor[r], __uint_as_float(yv[r]), acc);
    yp[tid] = acc;
  }
  const bool good = !__syncthreads_or(!okm2);
  // every CTA of the cluster has its copies landed and its partial output in place
  cluster_sync();
  if (good && crank == 0) {
    float acc = yp[tid] + Dh * __bfloat162float(xraw[tid]);
#pragma unroll
    for (uint32_t c = 1; c < kSplit; ++c) acc += ld_dsmem(smem_u32(yp + tid), c);
    reinterpret_cast<__nv_bfloat16*>(p.y)[bh * kP + tid] = __float2bfloat16_rn(acc);
  }
  if (good) {
    // the new carry, each CTA its slice (every CTA's copy of the old carry has landed)
    for (int i = tid; i < R * kRows; i += kST) {
      const int r = i / kRows, n = n0 + i % kRows;
      p.carry_B[bh * R * kN + r * kN + n] = __bfloat162float(Braw[r * kN + n]);
    }
    if (tid / kRows == (int)crank) p.carry_x[bh * kP + tid] = __bfloat162float(xraw[tid]);
  }
  if (!good && tid == 0) {
    wait(full, 0);  // copies still in flight land before the CTA leaves (bounded)
    set_status(p.status, M3_ERR_TIMEOUT);
  }
  // CTA 0 has read the other CTAs' partial outputs
  cluster_sync();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kSplitTmemCols));
  }
}

template <int RT>
cudaError_t launch_split_rt(const Params& p, const SplitPlan& sp, cudaStream_t stream) {
  static SmemAttr smem_set;
  auto k = decode_tc_split_kernel<RT>;
  cudaError_t e = smem_set.ensure(k, (int)sp.total);
  if (e != cudaSuccess) return e;
  e = launch_pdl(k, (unsigned)(p.b * p.H * kSplit), kST, sp.total, stream, p, sp);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Resident split CTAs per SM stay within the SM's tensor memory (512 columns), so that no
// allocation ever waits on a CTA that itself waits at a cluster barrier.
template <int RT>
bool split_fits(const SplitPlan& sp) {
  static PerDevice<bool> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  bool fits = false;
  cache.get(dev, &fits, [&sp](bool* v) {
    int per_sm = 0;
    auto k = decode_tc_split_kernel<RT>;
    *v = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sp.total) == cudaSuccess &&
         cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kST, sp.total) == cudaSuccess && per_sm >= 1 &&
         (uint32_t)per_sm * kSplitTmemCols <= 512;
    return true;
  });
  return fits;
}

cudaError_t launch_split(const Params& p, cudaStream_t stream, bool* used) {
  const SplitPlan sp = split_plan(p.R);
  *used = true;
  switch (p.R) {
#define M3_SPLIT_CASE(r) \
  case r:                \
    if (!split_fits<r>(sp)) break; \
    return launch_split_rt<r>(p, sp, stream);
    M3_SPLIT_CASE(1) M3_SPLIT_CASE(2) M3_SPLIT_CASE(3) M3_SPLIT_CASE(4)
    M3_SPLIT_CASE(5) M3_SPLIT_CASE(6) M3_SPLIT_CASE(7) M3_SPLIT_CASE(8)
#undef M3_SPLIT_CASE
    default: break;
  }
  *used = false;
  return cudaSuccess;
}

}  // namespace

bool decode_tc_supported(const Params& p) {
  if (!(p.dtype == M3_BF16 && p.N == kN && p.P == kP && p.R >= 1 && p.R <= kMaxR)) return false;
  const TcDevice d = tc_device();
  return d.sms > 0 && (int)tc_plan(p.R).total <= d.optin;
}

cudaError_t launch_decode_tc(const Params& p, cudaStream_t stream) {
  if (p.b * p.H == 0) return cudaSuccess;
  const int sms = tc_device().sms > 0 ? tc_device().sms : 148;
  const int64_t units = p.b * p.H;
  if (units * kSplit <= (int64_t)sms) {
    bool used = false;
    const cudaError_t e = launch_split(p, stream, &used);
    if (used) return e;
  }
  const unsigned grid = (unsigned)(units < sms ? units : sms);
  const TcPlan tp = tc_plan(p.R);
  switch (p.R) {
    case 1: return launch_tc_rt<1>(p, tp, grid, stream);
    case 2: return launch_tc_rt<2>(p, tp, grid, stream);
    case 3: return launch_tc_rt<3>(p, tp, grid, stream);
    case 4: return launch_tc_rt<4>(p, tp, grid, stream);
    case 5: return launch_tc_rt<5>(p, tp, grid, stream);
    case 6: return launch_tc_rt<6>(p, tp, grid, stream);
    case 7: return launch_tc_rt<7>(p, tp, grid, stream);
    default: return launch_tc_rt<8>(p, tp, grid, stream);
  }
}

}  // namespace m3
