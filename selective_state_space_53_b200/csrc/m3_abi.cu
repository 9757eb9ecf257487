// m3_abi.cu -- the extern "C" entry points of libm3 (declared in include/m3.h):
// argument validation, state handles, kernel dispatch, status codes.
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>

#include "m3_common.cuh"

namespace m3 {
__device__ int g_status = 0;
bool seq_scan_supported(int P, int N, int R);
}  // namespace m3

namespace {
// Device address of the status word, looked up once per device.
int* status_word() {
  static m3::PerDevice<int*> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  int* out = nullptr;
  const bool ok = cache.get(dev, &out, [](int** v) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, m3::g_status) != cudaSuccess) return false;
    *v = static_cast<int*>(ptr);
    return true;
  });
  return ok ? out : nullptr;
}
}  // namespace

struct m3_state {
  m3_dims dims;
  float* h;
  float* carry_B;
  float* carry_x;
  void* block;  // single allocation owned by the library (null when wrapped)
};

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The last CUDA error a call of this host thread met (m3_last_error reports it).
thread_local cudaError_t g_last_cuda = cudaSuccess;

m3_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return M3_OK;
  g_last_cuda = e;
  return M3_ERR_CUDA;
}

m3_status check_dims(const m3_dims* d) {
  if (!d) return M3_ERR_NULL;
  if (d->b < 0 || d->L < 0 || d->H < 1 || d->G < 1 || d->R < 1 || d->R > 8) return M3_ERR_DIMS;
  if (d->P < 8 || d->P > 256 || (d->P % 8) != 0) return M3_ERR_DIMS;
  if (d->N < 8 || d->N > 256 || (d->N % 8) != 0) return M3_ERR_DIMS;
  if ((d->H % d->G) != 0) return M3_ERR_DIMS;
  if (d->chunk < 0) return M3_ERR_DIMS;
  if (d->flags & ~(uint32_t)(M3_FLAG_SEQUENTIAL | M3_FLAG_ANGLE_DIRECT | M3_FLAG_RAW_INPUTS)) return M3_ERR_DIMS;
  if (d->dtype != M3_F32 && d->dtype != M3_BF16) return M3_ERR_DTYPE;
  if (d->b * (int64_t)d->H > (int64_t)0x7fffffff) return M3_ERR_DIMS;
  if (!m3::seq_scan_supported(d->P, d->N, d->R)) return M3_ERR_UNSUPPORTED;
  return M3_OK;
}

size_t state_bytes(const m3_dims* d) {
  const size_t bh = (size_t)d->b * d->H;
  return sizeof(float) * bh * ((size_t)d->N * d->P + (size_t)d->R * d->N + d->P);
}

bool same_state_dims(const m3_dims* a, const m3_dims* s) {
  return a->b == s->b && a->H == s->H && a->P == s->P && a->N == s->N && a->R == s->R;
}

// Validate the tensor operands shared by scan and decode.
m3_status check_operands(const m3_dims* d, const void* x, const float* dt, const float* A,
                         const float* lam, const void* B, const void* C, const float* theta,
                         const float* bias_B, const float* bias_C, const float* W_x,
                         const float* W_o, const float* D, const m3_state* state, const void* y,
                         bool tokens) {
  if (!state) return M3_ERR_NULL;
  if (!same_state_dims(d, &state->dims)) return M3_ERR_STATE;
  if (tokens) {
    const void* req[] = {x, dt, A, lam, B, C, theta, y};
    for (const void* q : req)
      if (!q) return M3_ERR_NULL;
  }
  const void* all[] = {x, dt, A, lam, B, C, theta, bias_B, bias_C, W_x, W_o, D, y,
                       state->h, state->carry_B, state->carry_x};
  for (const void* q : all)
    if (q && !aligned16(q)) return M3_ERR_ALIGN;
  return M3_OK;
}

m3::Params make_params(const m3_dims* d, int64_t L, const void* x, const float* dt,
                       const float* A, const float* lam, const void* B, const void* C,
                       const float* theta, const float* bias_B, const float* bias_C,
                       const float* W_x, const float* W_o, const float* D, m3_state* s,
                       void* y) {
  m3::Params p;
  p.b = d->b;
  p.L = L;
  p.H = d->H;
  p.P = d->P;
  p.N = d->N;
  p.R = d->R;
  p.G = d->G;
  p.dtype = d->dtype;
  p.angle_direct = (d->flags & M3_FLAG_ANGLE_DIRECT) ? 1 : 0;
  p.raw_inputs = (d->flags & M3_FLAG_RAW_INPUTS) ? 1 : 0;
  p.x = x;
  p.dt = dt;
  p.A = A;
  p.lam = lam;
  p.B = B;
  p.C = C;
  p.theta = theta;
  p.bias_B = bias_B;
  p.bias_C = bias_C;
  p.W_x = W_x;
  p.W_o = W_o;
  p.D = D;
  p.h = s ? s->h : nullptr;
  p.carry_B = s ? s->carry_B : nullptr;
  p.carry_x = s ? s->carry_x : nullptr;
  p.y = y;
  p.status = nullptr;
  return p;
}

// Raw inputs go through the warp-specialised scan's load stage directly (the front-end fused);
// every other kernel gets them transformed by m3_frontend into the workspace first.
bool fused_frontend(const m3_dims* dims) {
  if (!(dims->flags & M3_FLAG_RAW_INPUTS) || (dims->flags & M3_FLAG_SEQUENTIAL)) return false;
  m3::Params p = make_params(dims, dims->L, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                             nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr);
  return m3::tc_scan_supported(p) && m3::ws_scan_supported(p);
}

// Bytes of the scan's own scratch and, with M3_FLAG_RAW_INPUTS, where the transformed operands
// start in the workspace (after the scan's scratch, 256-byte aligned) and how many bytes they take.
struct WsLayout {
  size_t scan, fe_off, fe_bytes;
};

WsLayout ws_layout(const m3_dims* dims) {
  WsLayout w{0, 0, 0};
  if (dims->b * dims->L == 0) return w;
  m3::Params p = make_params(dims, dims->L, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                             nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr);
  if (!(dims->flags & M3_FLAG_SEQUENTIAL) && m3::tc_scan_supported(p)) w.scan = m3::tc_scan_workspace_bytes(p);
  else if (!(dims->flags & M3_FLAG_SEQUENTIAL)) w.scan = m3::seq_scan_workspace_bytes(p);  // segments in parallel
  if ((dims->flags & M3_FLAG_RAW_INPUTS) && !fused_frontend(dims)) {
    const size_t e = dims->dtype == M3_BF16 ? 2 : 4;
    const size_t nbc = (size_t)(dims->b * dims->L) * dims->G * dims->R * dims->N;
    const size_t nsc = (size_t)(dims->b * dims->L) * dims->H;
    w.fe_off = (w.scan + 255) & ~(size_t)255;
    w.fe_bytes = 2 * ((nbc * e + 255) & ~(size_t)255) + 3 * ((nsc * 4 + 255) & ~(size_t)255);
  }
  return w;
}

}  // namespace

extern "C" {

m3_status m3_state_bytes(const m3_dims* dims, size_t* out_bytes) {
  m3_status st = check_dims(dims);
  if (st != M3_OK) return st;
  if (!out_bytes) return M3_ERR_NULL;
  *out_bytes = state_bytes(dims);
  return M3_OK;
}

m3_status m3_state_alloc(const m3_dims* dims, void* stream, m3_state** out) {
  m3_status st = check_dims(dims);
  if (st != M3_OK) return st;
  if (!out) return M3_ERR_NULL;
  *out = nullptr;
  const size_t bytes = state_bytes(dims);
  void* block = nullptr;
  if (bytes > 0) {
    if (cudaMalloc(&block, bytes) != cudaSuccess) return M3_ERR_CUDA;
    if (cudaMemsetAsync(block, 0, bytes, (cudaStream_t)stream) != cudaSuccess) {
      cudaFree(block);
      return M3_ERR_CUDA;
    }
  }
  m3_state* s = new (std::nothrow) m3_state;
  if (!s) {
    cudaFree(block);
    return M3_ERR_CUDA;
  }
  const size_t bh = (size_t)dims->b * dims->H;
  s->dims = *dims;
  s->block = block;
  s->h = static_cast<float*>(block);
  s->carry_B = s->h + bh * dims->N * dims->P;
  s->carry_x = s->carry_B + bh * dims->R * dims->N;
  *out = s;
  return M3_OK;
}

m3_status m3_state_wrap(const m3_dims* dims, float* h, float* carry_B, float* carry_x,
                        m3_state** out) {
  m3_status st = check_dims(dims);
  if (st != M3_OK) return st;
  if (!out) return M3_ERR_NULL;
  *out = nullptr;
  if ((dims->b * dims->H > 0) && (!h || !carry_B || !carry_x)) return M3_ERR_NULL;
  if ((h && !aligned16(h)) || (carry_B && !aligned16(carry_B)) || (carry_x && !aligned16(carry_x)))
    return M3_ERR_ALIGN;
  m3_state* s = new (std::nothrow) m3_state;
  if (!s) return M3_ERR_CUDA;
  s->dims = *dims;
  s->block = nullptr;
  s->h = h;
  s->carry_B = carry_B;
  s->carry_x = carry_x;
  *out = s;
  return M3_OK;
}

m3_status m3_state_free(m3_state* state) {
  if (!state) return M3_ERR_NULL;
  m3_status st = M3_OK;
  if (state->block && cudaFree(state->block) != cudaSuccess) st = M3_ERR_CUDA;
  delete state;
  return st;
}

m3_status m3_state_tensors(const m3_state* state, float** h, float** carry_B, float** carry_x) {
  if (!state) return M3_ERR_NULL;
  if (h) *h = state->h;
  if (carry_B) *carry_B = state->carry_B;
  if (carry_x) *carry_x = state->carry_x;
  return M3_OK;
}

m3_status m3_state_copy_to_host(const m3_state* state, void* dst, size_t nbytes, void* stream) {
  if (!state || !dst) return M3_ERR_NULL;
  const m3_dims* d = &state->dims;
  const size_t bh = (size_t)d->b * d->H;
  const size_t nh = sizeof(float) * bh * d->N * d->P, nb = sizeof(float) * bh * d->R * d->N,
               nx = sizeof(float) * bh * d->P;
  if (nbytes != nh + nb + nx) return M3_ERR_STATE;
  cudaStream_t s = (cudaStream_t)stream;
  char* out = static_cast<char*>(dst);
  if (cudaMemcpyAsync(out, state->h, nh, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaMemcpyAsync(out + nh, state->carry_B, nb, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaMemcpyAsync(out + nh + nb, state->carry_x, nx, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return M3_ERR_CUDA;
  return M3_OK;
}

m3_status m3_state_copy_from_host(m3_state* state, const void* src, size_t nbytes, void* stream) {
  if (!state || !src) return M3_ERR_NULL;
  const m3_dims* d = &state->dims;
  const size_t bh = (size_t)d->b * d->H;
  const size_t nh = sizeof(float) * bh * d->N * d->P, nb = sizeof(float) * bh * d->R * d->N,
               nx = sizeof(float) * bh * d->P;
  if (nbytes != nh + nb + nx) return M3_ERR_STATE;
  cudaStream_t s = (cudaStream_t)stream;
  const char* in = static_cast<const char*>(src);
  if (cudaMemcpyAsync(state->h, in, nh, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(state->carry_B, in + nh, nb, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(state->carry_x, in + nh + nb, nx, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return M3_ERR_CUDA;
  return M3_OK;
}


m3_status m3_scan_workspace_size(const m3_dims* dims, size_t* out_bytes) {
  m3_status st = check_dims(dims);
  if (st != M3_OK) return st;
  if (!out_bytes) return M3_ERR_NULL;
  const WsLayout w = ws_layout(dims);
  *out_bytes = w.fe_bytes ? w.fe_off + w.fe_bytes : w.scan;
  return M3_OK;
}

m3_status m3_scan_fwd(const m3_dims* dims, const void* x, const float* dt, const float* A,
                      const float* lam, const void* B, const void* C, const float* theta,
                      const float* bias_B, const float* bias_C, const float* W_x,
                      const float* W_o, const float* D, m3_state* state, void* y,
                      void* workspace, size_t workspace_bytes, void* stream) {
  m3_status st = check_dims(dims);
  if (st != M3_OK) return st;
  const bool tokens = dims->b * dims->L > 0;
  st = check_operands(dims, x, dt, A, lam, B, C, theta, bias_B, bias_C, W_x, W_o, D, state, y,
                      tokens);
  if (st != M3_OK) return st;
  if (!tokens) return M3_OK;
  m3::Params p = make_params(dims, dims->L, x, dt, A, lam, B, C, theta, bias_B, bias_C, W_x, W_o,
                             D, state, y);
  const bool tc = !(dims->flags & M3_FLAG_SEQUENTIAL) && m3::tc_scan_supported(p);
  WsLayout w = ws_layout(dims);
  // the sequential kernel's segments are optional: without the workspace they asked for, the
  // sequences are walked whole, token by token (the front-end's part, if any, stays required)
  if (!tc && w.scan > 0 && (workspace == nullptr || workspace_bytes < (w.fe_bytes ? w.fe_off + w.fe_bytes : w.scan))) {
    const bool fe_fits = w.fe_bytes == 0 || (workspace != nullptr && workspace_bytes >= w.fe_bytes);
    if (fe_fits) {
      w.scan = 0;
      w.fe_off = 0;
    }
  }
  const size_t need = w.fe_bytes ? w.fe_off + w.fe_bytes : w.scan;
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return M3_ERR_WORKSPACE;
  if (need > 0 && !aligned16(workspace)) return M3_ERR_ALIGN;
  p.status = status_word();
  if (!p.status) return M3_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  if (w.fe_bytes) {
    // the front-end writes the transformed operands into the workspace after the scan's scratch
    char* fe = static_cast<char*>(workspace) + w.fe_off;
    const size_t e = dims->dtype == M3_BF16 ? 2 : 4;
    const size_t bc = ((size_t)(dims->b * dims->L) * dims->G * dims->R * dims->N * e + 255) & ~(size_t)255;
    const size_t sc = ((size_t)(dims->b * dims->L) * dims->H * 4 + 255) & ~(size_t)255;
    void* tB = fe;
    void* tC = fe + bc;
    float* tdt = reinterpret_cast<float*>(fe + 2 * bc);
    float* tA = reinterpret_cast<float*>(fe + 2 * bc + sc);
    float* tlam = reinterpret_cast<float*>(fe + 2 * bc + 2 * sc);
    if (m3::launch_frontend(p, B, C, dt, A, lam, tB, tC, tdt, tA, tlam, s) != cudaSuccess) return M3_ERR_CUDA;
    p.B = tB;
    p.C = tC;
    p.dt = tdt;
    p.A = tA;
    p.lam = tlam;
    p.raw_inputs = 0;
  }
  const cudaError_t e = tc                ? m3::launch_scan_tc(p, workspace, w.scan, s)
                        : w.scan > 0      ? m3::launch_scan_seq_chunked(p, workspace, w.scan, s)
                                          : m3::launch_scan_sequential(p, s);
  return cuda_status(e);
}

m3_status m3_decode_step(const m3_dims* dims, const void* x_t, const float* dt_t,
                         const float* A_t, const float* lam_t, const void* B_t,
                         const void* C_t, const float* theta_t, const float* bias_B,
                         const float* bias_C, const float* W_x, const float* W_o,
                         const float* D, m3_state* state, void* y_t, void* stream) {
  m3_status st = check_dims(dims);
  if (st != M3_OK) return st;
  if (dims->flags & M3_FLAG_RAW_INPUTS) return M3_ERR_UNSUPPORTED;  // m3_frontend on the token first
  const bool tokens = dims->b > 0;
  st = check_operands(dims, x_t, dt_t, A_t, lam_t, B_t, C_t, theta_t, bias_B, bias_C, W_x, W_o, D,
                      state, y_t, tokens);
  if (st != M3_OK) return st;
  if (!tokens) return M3_OK;
  m3::Params p = make_params(dims, 1, x_t, dt_t, A_t, lam_t, B_t, C_t, theta_t, bias_B, bias_C,
                             W_x, W_o, D, state, y_t);
  p.status = status_word();
  if (!p.status) return M3_ERR_CUDA;
  const cudaError_t e = m3::decode_supported(p) ? m3::launch_decode(p, (cudaStream_t)stream)
                                                : m3::launch_scan_sequential(p, (cudaStream_t)stream);
  return cuda_status(e);
}

m3_status m3_scan_bwd_workspace_size(const m3_dims* dims, size_t* out_bytes) {
  m3_status st = check_dims(dims);
  if (st != M3_OK) return st;
  if (!out_bytes) return M3_ERR_NULL;
  m3::Params p = make_params(dims, dims->L, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                             nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr);
  if (!m3::bwd_supported(p)) return M3_ERR_UNSUPPORTED;
  *out_bytes = m3::scan_bwd_workspace_bytes(p);
  return M3_OK;
}

m3_status m3_scan_bwd(const m3_dims* dims, const void* x, const float* dt, const float* A, const float* lam,
                      const void* B, const void* C, const float* theta, const float* bias_B, const float* bias_C,
                      const float* W_x, const float* W_o, const float* D, const m3_state* state0, const void* dy,
                      const float* dh_final, const m3_grads* gr, void* workspace, size_t workspace_bytes,
                      void* stream) {
  size_t need = 0;
  m3_status st = m3_scan_bwd_workspace_size(dims, &need);
  if (st != M3_OK) return st;
  if (!gr) return M3_ERR_NULL;
  if (dims->L < 1) return M3_ERR_DIMS;
  if (dims->flags & M3_FLAG_RAW_INPUTS) return M3_ERR_UNSUPPORTED;  // the backward pass of an empty scan is not defined here
  const bool tokens = dims->b * dims->L > 0;
  st = check_operands(dims, x, dt, A, lam, B, C, theta, bias_B, bias_C, W_x, W_o, D, state0, dy, tokens);
  if (st != M3_OK) return st;
  const void* req[] = {gr->dx, gr->ddt, gr->dA, gr->dlam, gr->dB, gr->dC, gr->dtheta, gr->dh0, gr->dcarry_B,
                       gr->dcarry_x};
  for (const void* q : req)
    if (!q) return M3_ERR_NULL;
  const void* all[] = {gr->dx, gr->ddt, gr->dA, gr->dlam, gr->dB, gr->dC, gr->dtheta, gr->dbias_B, gr->dbias_C,
                       gr->dW_x, gr->dW_o, gr->dD, gr->dh0, gr->dcarry_B, gr->dcarry_x, dh_final, workspace};
  for (const void* q : all)
    if (q && !aligned16(q)) return M3_ERR_ALIGN;
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return M3_ERR_WORKSPACE;
  if (dims->b * dims->H == 0) return M3_OK;
  m3::Params p = make_params(dims, dims->L, x, dt, A, lam, B, C, theta, bias_B, bias_C, W_x, W_o, D,
                             const_cast<m3_state*>(state0), nullptr);
  p.status = status_word();
  if (!p.status) return M3_ERR_CUDA;
  const cudaError_t e = m3::launch_scan_bwd(p, dy, dh_final, gr->dx, gr->ddt, gr->dA, gr->dlam, gr->dB, gr->dC,
                                            gr->dtheta, gr->dbias_B, gr->dbias_C, gr->dW_x, gr->dW_o, gr->dD,
                                            gr->dh0, gr->dcarry_B, gr->dcarry_x, workspace, workspace_bytes,
                                            (cudaStream_t)stream);
  return cuda_status(e);
}

m3_status m3_scan_summary_workspace_size(const m3_dims* dims, size_t* out_bytes) {
  m3_status st = check_dims(dims);
  if (st != M3_OK) return st;
  if (!out_bytes) return M3_ERR_NULL;
  if (dims->L < 1) return M3_ERR_DIMS;
  if (dims->flags & M3_FLAG_RAW_INPUTS) return M3_ERR_UNSUPPORTED;
  m3::Params p = make_params(dims, dims->L, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                             nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr);
  if (!m3::tc_scan_supported(p)) return M3_ERR_UNSUPPORTED;
  *out_bytes = m3::scan_summary_workspace_bytes(p);
  return M3_OK;
}

m3_status m3_scan_summary(const m3_dims* dims, const void* x, const float* dt, const float* A, const float* lam,
                          const void* B, const float* theta, const float* bias_B, const float* W_x, float* Z,
                          float* logdec, double* angle, float* bp_first, float* carry_B, float* carry_x,
                          void* workspace, size_t workspace_bytes, void* stream) {
  size_t need = 0;
  m3_status st = m3_scan_summary_workspace_size(dims, &need);
  if (st != M3_OK) return st;
  const void* req[] = {x, dt, A, lam, B, theta, Z, logdec, angle, bp_first, carry_B, carry_x, workspace};
  for (const void* q : req)
    if (!q) return M3_ERR_NULL;
  const void* all[] = {x, dt, A, lam, B, theta, bias_B, W_x, Z, logdec, angle, bp_first, carry_B, carry_x, workspace};
  for (const void* q : all)
    if (q && !aligned16(q)) return M3_ERR_ALIGN;
  if (workspace_bytes < need) return M3_ERR_WORKSPACE;
  if (dims->b * dims->H == 0) return M3_OK;
  // the state pass reads neither C nor a state: B stands in for C's tensor map
  m3::Params p = make_params(dims, dims->L, x, dt, A, lam, B, B, theta, bias_B, nullptr, W_x, nullptr, nullptr,
                             nullptr, nullptr);
  p.status = status_word();
  if (!p.status) return M3_ERR_CUDA;
  const cudaError_t e = m3::launch_range_summary(p, workspace, workspace_bytes, Z, logdec, angle, bp_first, carry_B,
                                                 carry_x, (cudaStream_t)stream);
  return cuda_status(e);
}

m3_status m3_state_fold(const m3_dims* dims, int32_t nranges, const float* Z, const float* logdec,
                        const double* angle, const float* bp_first, const float* carry_B, const float* carry_x,
                        const float* bias_B, const float* W_x, m3_state* state, void* stream) {
  m3_status st = check_dims(dims);
  if (st != M3_OK) return st;
  if (nranges < 0) return M3_ERR_DIMS;
  if (!state) return M3_ERR_NULL;
  if (!same_state_dims(dims, &state->dims)) return M3_ERR_STATE;
  if (nranges > 0) {
    const void* req[] = {Z, logdec, angle, bp_first, carry_B, carry_x};
    for (const void* q : req)
      if (!q) return M3_ERR_NULL;
  }
  const void* all[] = {Z, logdec, angle, bp_first, carry_B, carry_x, bias_B, W_x, state->h, state->carry_B,
                       state->carry_x};
  for (const void* q : all)
    if (q && !aligned16(q)) return M3_ERR_ALIGN;
  if (dims->b * dims->H == 0 || nranges == 0) return M3_OK;
  m3::Params p = make_params(dims, 1, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, bias_B, nullptr,
                             W_x, nullptr, nullptr, state, nullptr);
  const cudaError_t e = m3::launch_state_fold(p, nranges, Z, logdec, angle, bp_first, carry_B, carry_x,
                                              (cudaStream_t)stream);
  return cuda_status(e);
}

m3_status m3_frontend(const m3_dims* dims, const void* B_raw, const void* C_raw, const float* dt_raw,
                      const float* A_raw, const float* lam_raw, void* B, void* C, float* dt, float* A, float* lam,
                      void* stream) {
  m3_status st = check_dims(dims);
  if (st != M3_OK) return st;
  if (dims->b * dims->L == 0) return M3_OK;
  const void* req[] = {B_raw, C_raw, dt_raw, A_raw, lam_raw, B, C, dt, A, lam};
  for (const void* q : req) {
    if (!q) return M3_ERR_NULL;
    if (!aligned16(q)) return M3_ERR_ALIGN;
  }
  m3::Params p = make_params(dims, dims->L, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                             nullptr, nullptr, nullptr, nullptr, nullptr, nullptr);
  const cudaError_t e = m3::launch_frontend(p, B_raw, C_raw, dt_raw, A_raw, lam_raw, B, C, dt, A, lam,
                                            (cudaStream_t)stream);
  return cuda_status(e);
}

m3_status m3_output_norm(const m3_dims* dims, const void* y, const void* z, const float* weight, float eps,
                         void* out, void* stream) {
  m3_status st = check_dims(dims);
  if (st != M3_OK) return st;
  if (!(eps >= 0.0f)) return M3_ERR_DIMS;
  const bool rows = dims->b * dims->L * dims->H > 0;
  if (rows && (!y || !out)) return M3_ERR_NULL;
  const void* all[] = {y, z, weight, out};
  for (const void* q : all)
    if (q && !aligned16(q)) return M3_ERR_ALIGN;
  if (!rows) return M3_OK;
  m3::Params p = make_params(dims, dims->L, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                             nullptr, nullptr, nullptr, nullptr, nullptr, const_cast<void*>(y));
  const cudaError_t e = m3::launch_output_norm(p, z, weight, eps, out, (cudaStream_t)stream);
  return cuda_status(e);
}

m3_status m3_selftest_wait(uint64_t limit_ns, void* stream) {
  if (limit_ns > 10000000000ull) return M3_ERR_DIMS;
  int* st = status_word();
  if (!st) return M3_ERR_CUDA;
  return cuda_status(m3::launch_selftest_wait(st, (unsigned long long)limit_ns, (cudaStream_t)stream));
}

m3_status m3_check(void* stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return M3_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, m3::g_status, sizeof(int)) != cudaSuccess) return M3_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(m3::g_status, &zero, sizeof(int)) != cudaSuccess) return M3_ERR_CUDA;
  }
  return (m3_status)v;
}

const char* m3_status_str(m3_status status) {
  switch (status) {
    case M3_OK: return "ok";
    case M3_ERR_DIMS: return "bad dimensions";
    case M3_ERR_DTYPE: return "unsupported dtype";
    case M3_ERR_ALIGN: return "tensor pointer not 16-byte aligned";
    case M3_ERR_NULL: return "required pointer is NULL";
    case M3_ERR_WORKSPACE: return "workspace missing or too small";
    case M3_ERR_CUDA: return "CUDA error";
    case M3_ERR_TIMEOUT: return "a kernel gave up a bounded wait";
    case M3_ERR_UNSUPPORTED: return "dimensions not supported by this build";
    case M3_ERR_STATE: return "state does not match the dimensions";
  }
  return "unknown status";
}

const char* m3_last_error(void) { return g_last_cuda == cudaSuccess ? "no CUDA error" : cudaGetErrorString(g_last_cuda); }

const char* m3_version(void) { return "m3 0.1 (sm_100a)"; }

}  // extern "C"
