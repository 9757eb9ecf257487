/*
 * m3.h -- C ABI of the B200-native Mamba-3 SSM layer core (libm3.so).
 *
 * The layer core is the exponential-trapezoidal selective scan with complex
 * (rotation / data-dependent RoPE) transitions and MIMO rank R, as described in
 * the Mamba-3 paper note (docsaid.org, "Mamba-3: Improved Sequence Modeling using
 * State Space Principles"):
 *   - section "その1 表現力の高い離散化": h_t = alpha_t h_{t-1} + beta_t B_{t-1}x_{t-1}
 *     + gamma_t B_t x_t with alpha = e^{dt A}, beta = (1-lam) dt e^{dt A}, gamma = lam dt;
 *   - section "その2 複素数の状態": complex A, i.e. a decay times 2x2 rotations of
 *     adjacent state pairs, equivalently a data-dependent RoPE of B and C;
 *   - section "その3 MIMO": R input branches and R readouts, rank <= R update.
 * Per (batch b, head h; group g = h / (H/G)) and token t:
 *   Bb_{t,r} = B[b,t,g,r,:] + bias_B[h,r,:],  Cb_{t,r} = C[b,t,g,r,:] + bias_C[h,r,:]
 *   X_{t,r} = W_x[h,r,:] * x[b,t,h,:],        u_t = sum_r Bb_{t,r} X_{t,r}^T   (N x P)
 *   h_t = e^{dt_t A_t} Rot(dt_t theta_t) (h_{t-1} + (1-lam_t) dt_t u_{t-1}) + lam_t dt_t u_t
 *   y[b,t,h,:] = sum_r W_o[h,r,:] * (Cb_{t,r}^T h_t) + D[h] x[b,t,h,:]
 * Rot rotates rows (2k, 2k+1) of the state by angle dt_t theta[b,t,g,k] (theta[b,t,g,k]
 * itself with M3_FLAG_ANGLE_DIRECT) with the matrix [[cos, -sin], [sin, cos]].
 *
 * Conventions for every entry point:
 *   - Tensor pointers are caller-owned DEVICE memory, contiguous row-major in the
 *     layouts below, 16-byte aligned.  The library never frees them.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL is
 *     the legacy default stream).  m3_scan_fwd and m3_decode_step allocate nothing
 *     and never synchronise the host.
 *   - Every call returns an m3_status; nothing throws across the ABI.  Argument
 *     errors are detected on the host before anything is launched.  A kernel
 *     that gives up a bounded wait records M3_ERR_TIMEOUT in a device status
 *     word, which m3_check() returns.
 *
 * Layouts (dtype: M3_BF16 or M3_F32 for x, B, C, y; fp32 for everything else):
 *   x, y          (b, L, H, P)        dt, A, lam   (b, L, H)
 *   B, C          (b, L, G, R, N)     theta        (b, L, G, N/2)
 *   bias_B/bias_C (H, R, N)  may be NULL (zero)
 *   W_x, W_o      (H, R, P)  may be NULL (all ones)
 *   D             (H)        may be NULL (no skip term)
 * State (m3_state): h (b, H, N, P) fp32, carry_B (b, H, R, N) fp32 (previous
 * token's raw B, before bias), carry_x (b, H, P) fp32 (previous token's raw x).
 * An all-zero state is a fresh sequence (no previous-token term at t = 0).
 */
#ifndef M3_H
#define M3_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  M3_OK = 0,
  M3_ERR_DIMS = -1,        /* bad sizes: N odd, G does not divide H, R/P/N out of range;
                              unknown flag bits */
  M3_ERR_DTYPE = -2,       /* dtype not M3_BF16 / M3_F32 */
  M3_ERR_ALIGN = -3,       /* a tensor pointer is not 16-byte aligned */
  M3_ERR_NULL = -4,        /* a required pointer is NULL */
  M3_ERR_WORKSPACE = -5,   /* workspace missing or smaller than m3_scan_workspace_size */
  M3_ERR_CUDA = -6,        /* a CUDA runtime call or kernel launch failed */
  M3_ERR_TIMEOUT = -7,     /* a kernel gave up a bounded wait (device status word) */
  M3_ERR_UNSUPPORTED = -8, /* valid dims that no kernel of this build handles */
  M3_ERR_STATE = -9        /* state was made for other dims, or buffer size mismatch */
} m3_status;

enum { M3_F32 = 0, M3_BF16 = 1 };

/* flags */
enum {
  M3_FLAG_SEQUENTIAL = 1u,   /* run the token-sequential SIMT scan even where the chunked
                                tensor-core scan applies (diagnostic / cross-check) */
  M3_FLAG_ANGLE_DIRECT = 2u, /* variant: theta is the rotation angle of the step itself,
                                phi_t = theta_t instead of dt_t * theta_t (the rotation
                                then no longer depends on the head's step size) */
  M3_FLAG_RAW_INPUTS = 4u    /* m3_scan_fwd: B, C, dt, A, lam are the block's raw projections;
                                the core applies the front-end of m3_frontend to them itself
                                (the workspace then also holds the transformed operands) */
};

typedef struct {
  int64_t b;      /* batch */
  int64_t L;      /* sequence length (ignored by m3_decode_step: one token) */
  int32_t H;      /* heads */
  int32_t P;      /* head dim (multiple of 8, <= 256) */
  int32_t N;      /* state dim d_state (even, multiple of 8, <= 256) */
  int32_t R;      /* MIMO rank (1..8) */
  int32_t G;      /* B/C/theta groups (divides H) */
  int32_t chunk;  /* chunk length of the model (0 = default 32).  The chunked scan is
                     exact, so this does not change the result; the kernel packs
                     128/R tokens per tensor-core tile whatever this value is. */
  int32_t dtype;  /* M3_BF16 or M3_F32: storage type of x, B, C, y */
  uint32_t flags; /* M3_FLAG_*; other bits: M3_ERR_DIMS */
} m3_dims;

typedef struct m3_state m3_state; /* opaque */

/* ---- state ------------------------------------------------------------- */

/* Bytes of device memory an m3_state for these dims holds (h + carry_B + carry_x). */
m3_status m3_state_bytes(const m3_dims* dims, size_t* out_bytes);

/* Allocate a zero-initialised state on the current device (cudaMallocAsync on
 * `stream`).  The library owns the memory; release it with m3_state_free. */
m3_status m3_state_alloc(const m3_dims* dims, void* stream, m3_state** out);

/* Wrap caller-owned device buffers (h, carry_B, carry_x in the layouts above) as a
 * state.  The library does not free them; m3_state_free releases only the handle. */
m3_status m3_state_wrap(const m3_dims* dims, float* h, float* carry_B, float* carry_x,
                        m3_state** out);

/* Release the handle (and the memory, if m3_state_alloc made it). */
m3_status m3_state_free(m3_state* state);

/* Device pointers of the three state tensors (any out pointer may be NULL). */
m3_status m3_state_tensors(const m3_state* state, float** h, float** carry_B, float** carry_x);

/* Copy the whole state (h, then carry_B, then carry_x, fp32) to / from a host
 * buffer of exactly m3_state_bytes bytes.  Synchronises `stream`. */
m3_status m3_state_copy_to_host(const m3_state* state, void* dst, size_t nbytes, void* stream);
m3_status m3_state_copy_from_host(m3_state* state, const void* src, size_t nbytes, void* stream);

/* ---- prefill (chunked scan) ------------------------------------------- */

/* Scratch bytes m3_scan_fwd needs for these dims (0 when it needs none).  For the chunked
 * tensor-core scan the workspace is required; for the token-sequential SIMT scan (fp32 inputs,
 * shapes outside the tensor-core tiles, M3_FLAG_SEQUENTIAL excepted) it lets the sequences be
 * split into segments scanned in parallel (summaries of the earlier segments folded into each
 * segment's entering state), and without it they are walked whole. */
m3_status m3_scan_workspace_size(const m3_dims* dims, size_t* out_bytes);

/* Run the layer core over L tokens of every sequence of the batch.
 * state: in = state before token 0 (fresh or carried), out = state after token
 * L-1 (h_{L-1} and the carry of token L-1).  y: (b, L, H, P) in dims->dtype.
 * workspace: device scratch of at least m3_scan_workspace_size bytes (may be NULL
 * when that size is 0, or on the sequential path, which then does not split the sequences).
 * L = 0 leaves the state unchanged and writes nothing.
 * Mamba-3 paper note, sections その1-その3 (recurrence above); the chunked form
 * follows the IBM Mamba page's SSD description (matrix form within a chunk,
 * state passed between chunks). */
m3_status m3_scan_fwd(const m3_dims* dims, const void* x, const float* dt, const float* A,
                      const float* lam, const void* B, const void* C, const float* theta,
                      const float* bias_B, const float* bias_C, const float* W_x,
                      const float* W_o, const float* D, m3_state* state, void* y,
                      void* workspace, size_t workspace_bytes, void* stream);

/* Same as m3_scan_fwd, for callers that cannot provide a workspace: a serving process
 * whose device memory is all reserved up front by an allocator it does not own, or a
 * plain C program with no device allocator of its own (a cudaMalloc mid-request may also
 * synchronise the device).  The paper has no counterpart; this is a property of the
 * library only.  The scratch m3_scan_fwd would take from `workspace` comes instead from
 * one fixed 16 MiB device array inside libm3, which every device that loads the library
 * holds until the process exits.  This call allocates nothing.  Dimensions whose scratch
 * (m3_scan_workspace_size) exceeds 16 MiB are rejected with M3_ERR_WORKSPACE.  All calls
 * share the array: calls whose kernels overlap on the GPU (several streams or host
 * threads) race and give wrong results; calls ordered on one stream are safe.  Nothing
 * needs clearing between calls (every scratch byte is written before it is read).  The
 * first call on a device, made with that device current, looks up the array's device
 * address (cudaGetSymbolAddress); make that first call before any stream capture. */
m3_status m3_scan_fwd_noalloc(const m3_dims* dims, const void* x, const float* dt, const float* A,
                              const float* lam, const void* B, const void* C, const float* theta,
                              const float* bias_B, const float* bias_C, const float* W_x,
                              const float* W_o, const float* D, m3_state* state, void* y,
                              void* stream);

/* ---- backward pass ----------------------------------------------------------- */

/* Gradients of the layer core: every pointer is caller-owned device memory in the layout of
 * the operand it belongs to.  dx, dB, dC in dims->dtype; everything else fp32. */
typedef struct {
  void* dx;          /* (b, L, H, P)                                  required */
  float* ddt;        /* (b, L, H)                                     required */
  float* dA;         /* (b, L, H)                                     required */
  float* dlam;       /* (b, L, H)                                     required */
  void* dB;          /* (b, L, G, R, N), summed over a group's heads  required */
  void* dC;          /* (b, L, G, R, N), summed over a group's heads  required */
  float* dtheta;     /* (b, L, G, N/2), summed over a group's heads   required */
  float* dbias_B;    /* (H, R, N), summed over batch and tokens       may be NULL (not computed) */
  float* dbias_C;    /* (H, R, N)                                     may be NULL */
  float* dW_x;       /* (H, R, P)                                     may be NULL */
  float* dW_o;       /* (H, R, P)                                     may be NULL */
  float* dD;         /* (H)                                           may be NULL */
  float* dh0;        /* (b, H, N, P): the initial state h             required */
  float* dcarry_B;   /* (b, H, R, N): the initial carry               required */
  float* dcarry_x;   /* (b, H, P)                                     required */
} m3_grads;

/* Scratch bytes m3_scan_bwd needs: the forward states it recomputes (one every ~sqrt(L)
 * tokens, plus one block of ~sqrt(L) states, per (batch, head)) and fp32 accumulators of dB
 * and dC. */
m3_status m3_scan_bwd_workspace_size(const m3_dims* dims, size_t* out_bytes);

/* Backward pass of m3_scan_fwd: the gradients of sum(dy * y) + sum(dh_final * h_L) with
 * respect to every operand and the initial state.  The operands are those the forward call
 * took; state0 is the state it started from (not modified).  dy: (b, L, H, P) in dims->dtype;
 * dh_final: (b, H, N, P) fp32 or NULL (zero).  Gradients whose operand was NULL (no bias, unit
 * weights, no skip term) are still the gradients at that value.  The chain rule is taken
 * through the recurrence of the Mamba-3 paper note (sections その1-その3) exactly as written
 * at the top of this header; the forward states are recomputed in fp32 from checkpoints.
 * L must be at least 1 (M3_ERR_DIMS otherwise).  Asynchronous on `stream`; allocates nothing. */
m3_status m3_scan_bwd(const m3_dims* dims, const void* x, const float* dt, const float* A,
                      const float* lam, const void* B, const void* C, const float* theta,
                      const float* bias_B, const float* bias_C, const float* W_x, const float* W_o,
                      const float* D, const m3_state* state0, const void* dy, const float* dh_final,
                      const m3_grads* grads, void* workspace, size_t workspace_bytes, void* stream);

/* ---- ranges of a sequence (sequence sharding) ---------------------------- */

/* A sequence split into consecutive token ranges (for instance one per device) runs as: every
 * range is summarised (m3_scan_summary), the summaries are exchanged, the state entering range k
 * is the sequence's initial state folded through the summaries of ranges 0..k-1
 * (m3_state_fold), and range k then runs m3_scan_fwd from that state.  The results equal one
 * m3_scan_fwd over the whole sequence.  The algebra: the scan combines associatively over
 * ranges (IBM page "Mamba モデルとは", hardware-aware scan); for the recurrence above a range
 * of tokens t0..t1 maps the state entering it to
 *   h_{t1} = e^{logdec} Rot(angle) (h_{t0-1} + bp_first u_{t0-1}) + Z,
 * logdec = sum_t dt_t A_t, angle_k = sum_t phi_{t,k}, bp_first = (1 - lam_{t0}) dt_{t0}, Z the
 * range's end state from a fresh start, u_{t0-1} = sum_r (carry_B_r + bias_B_r)(W_x_r * carry_x)^T
 * the previous-token term built from the carry of the token before the range (Mamba-3 paper
 * note, sections その1-その3). */

/* Scratch bytes m3_scan_summary needs (dims->L = the range's length, >= 1).  Ranges are
 * summarised by the chunked tensor-core state pass: bf16 with d_state and headdim in {64, 128}
 * and R in {1, 2, 4, 8} (R = 1 with d_state = headdim = 128 excepted); other dims give
 * M3_ERR_UNSUPPORTED. */
m3_status m3_scan_summary_workspace_size(const m3_dims* dims, size_t* out_bytes);

/* Summary of one range of every sequence of the batch (x, dt, A, lam, B, theta of the range in
 * the layouts above; bias_B, W_x may be NULL).  Outputs, caller-owned device memory:
 *   Z (b, H, N, P) fp32        the range's end state from a fresh start
 *   logdec (b, H) fp32         sum over the range of dt A
 *   angle (b, H, N/2) fp64     sum over the range of the rotation angles, reduced to [-pi, pi]
 *   bp_first (b, H) fp32       (1 - lam) dt of the range's first token
 *   carry_B (b, H, R, N) fp32, carry_x (b, H, P) fp32   the range's last token's raw B and x
 * workspace: at least m3_scan_summary_workspace_size bytes.  Asynchronous on `stream`. */
m3_status m3_scan_summary(const m3_dims* dims, const void* x, const float* dt, const float* A,
                          const float* lam, const void* B, const float* theta, const float* bias_B,
                          const float* W_x, float* Z, float* logdec, double* angle, float* bp_first,
                          float* carry_B, float* carry_x, void* workspace, size_t workspace_bytes,
                          void* stream);

/* Fold `nranges` range summaries (each array above with a leading nranges axis, ranges in
 * sequence order) onto `state`: in, the state entering range 0; out, the state entering range
 * nranges (h and the carry).  nranges = 0 leaves the state unchanged.  bias_B, W_x as for
 * m3_scan_fwd.  Asynchronous on `stream`. */
m3_status m3_state_fold(const m3_dims* dims, int32_t nranges, const float* Z, const float* logdec,
                        const double* angle, const float* bp_first, const float* carry_B,
                        const float* carry_x, const float* bias_B, const float* W_x,
                        m3_state* state, void* stream);

/* ---- decode (one token) ------------------------------------------------ */

/* Advance every sequence by one token.  Token inputs have L = 1 in the layouts
 * above: x_t (b, H, P), dt_t/A_t/lam_t (b, H), B_t/C_t (b, G, R, N),
 * theta_t (b, G, N/2); y_t (b, H, P).  dims->L is ignored.  Reads and rewrites the
 * state in place.  Same recurrence as m3_scan_fwd (section その3 of the paper note:
 * decode reads and writes the whole fixed-size state every token).
 * Precision: with bf16 inputs, d_state = headdim = 128 and R <= 8 the rank-2R state
 * increment and the R readouts run on the tensor cores with bf16 operands and fp32
 * accumulation (the carried state stays fp32); every other shape, and fp32 inputs,
 * compute in fp32 throughout.  Either way the result is within the bf16 tolerance of
 * the fp64 recurrence (max relative error 2e-2), or 1e-4 for fp32 inputs. */
m3_status m3_decode_step(const m3_dims* dims, const void* x_t, const float* dt_t,
                         const float* A_t, const float* lam_t, const void* B_t,
                         const void* C_t, const float* theta_t, const float* bias_B,
                         const float* bias_C, const float* W_x, const float* W_o,
                         const float* D, m3_state* state, void* y_t, void* stream);

/* ---- the block's front-end -------------------------------------------------------- */

/* The block's front-end on raw projections: B and C RMS-normalised over N per (token, group,
 * branch) row, B = B_raw / sqrt(mean_N B_raw^2 + 1e-6) (no weight; the biases are added later
 * by the core), dt = softplus(dt_raw), A = -exp(A_raw), lam = sigmoid(lam_raw) -- the B/C norm
 * of the Cartesia blog "Mamba-3" and the docsaid note (section アーキテクチャ) and the
 * parameterisation of the discretisation of section その1.  Raw and transformed tensors in the
 * layouts of m3_scan_fwd (B, C in dims->dtype; the others fp32); outputs may be the inputs.
 * m3_decode_step takes transformed operands: run this on the token first.  Asynchronous. */
m3_status m3_frontend(const m3_dims* dims, const void* B_raw, const void* C_raw, const float* dt_raw,
                      const float* A_raw, const float* lam_raw, void* B, void* C, float* dt, float* A,
                      float* lam, void* stream);

/* ---- the hybrid model's output norm ---------------------------------------------- */

/* The norm before the output projection that the Mamba-3 paper note (section アーキテクチャ)
 * removes in the pure Mamba-3 model and keeps in the hybrid one, with the block's gate z
 * applied first when given.  Per (batch, token, head) row of P values:
 *   v = y * silu(z)  (v = y when z is NULL),   out = weight[h] * v / sqrt(mean_p v^2 + eps).
 * y, z, out: (b, L, H, P) in dims->dtype (out may be y); weight: (H, P) fp32 or NULL (ones);
 * eps >= 0 (M3_ERR_DIMS otherwise).  Asynchronous on `stream`. */
m3_status m3_output_norm(const m3_dims* dims, const void* y, const void* z, const float* weight,
                         float eps, void* out, void* stream);

/* ---- status -------------------------------------------------------------- */

/* Synchronise `stream`, then return (and clear) the device status word:
 * M3_OK, M3_ERR_TIMEOUT, or M3_ERR_CUDA if the stream reports an error. */
m3_status m3_check(void* stream);

/* Diagnostic of the error path (no counterpart in the pages): launches one CTA that waits on
 * an mbarrier nothing arrives at, bounded by limit_ns (at most 10 s, else M3_ERR_DIMS) of
 * %globaltimer -- the same kind of bounded wait as every wait in the scan and decode kernels.
 * When the limit passes the kernel records M3_ERR_TIMEOUT in the device status word and
 * returns; the next m3_check() on `stream` returns M3_ERR_TIMEOUT and clears the word, and the
 * context stays usable.  Asynchronous on `stream`. */
m3_status m3_selftest_wait(uint64_t limit_ns, void* stream);

/* Static description of a status code. */
const char* m3_status_str(m3_status status);

/* Text of the last CUDA runtime error behind an M3_ERR_CUDA returned to this host thread
 * ("no CUDA error" if there was none).  The string is static. */
const char* m3_last_error(void);

/* Library version string. */
const char* m3_version(void);

#ifdef __cplusplus
}
#endif

#endif /* M3_H */
