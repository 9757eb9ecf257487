// m3_noalloc.cu -- m3_scan_fwd_noalloc: the chunked prefill with its scratch in a fixed
// device array instead of a caller-provided workspace.
//
// Some callers cannot hand the library a workspace: a serving process that reserved all
// of its device memory up front for an allocator it does not control, or a plain C host
// program that links libm3 and has no device allocator of its own, and for which a
// cudaMalloc in the middle of a request could also synchronise the device.  For them the
// segment summaries that m3_scan_fwd keeps in its workspace live here, in one file-scope
// array of kScratchBytes.  Every device that loads the library holds that array until the
// process exits.  Calls share it: two calls whose kernels overlap on the GPU (on different
// streams, or on several host threads) race on its contents.  The scan overwrites every
// byte it reads before reading it, so the contents left by an earlier call never matter
// and nothing is cleared.
#include "m3_common.cuh"

// 16 MiB, sized for a 148-SM B200: there the segment planner asks for at most about 14 MiB
// (13.95 MiB, at 74 (batch, head) sequences with d_state = headdim = 128).  The planner fills
// the SMs, so on a part with more SMs the need grows with the SM count (about 16 MiB at 170
// SMs); dimensions that would need more than the array get M3_ERR_WORKSPACE.
static constexpr size_t kScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_scan_scratch[kScratchBytes];

namespace m3 {
namespace {

// Device address of g_scan_scratch for the current device, looked up on the first call
// made with that device current (host code cannot use the symbol itself as an address).
unsigned char* scratch_address() {
  static PerDevice<unsigned char*> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  unsigned char* out = nullptr;
  const bool ok = cache.get(dev, &out, [](unsigned char** v) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress((void**)&ptr, g_scan_scratch) != cudaSuccess) return false;
    *v = static_cast<unsigned char*>(ptr);
    return true;
  });
  return ok ? out : nullptr;
}

}  // namespace
}  // namespace m3

extern "C" m3_status m3_scan_workspace_size(const m3_dims* dims, size_t* out_bytes);
extern "C" m3_status m3_scan_fwd(const m3_dims* dims, const void* x, const float* dt, const float* A,
                                 const float* lam, const void* B, const void* C, const float* theta,
                                 const float* bias_B, const float* bias_C, const float* W_x, const float* W_o,
                                 const float* D, m3_state* state, void* y, void* workspace,
                                 size_t workspace_bytes, void* stream);

extern "C" m3_status m3_scan_fwd_noalloc(const m3_dims* dims, const void* x, const float* dt, const float* A,
                                         const float* lam, const void* B, const void* C, const float* theta,
                                         const float* bias_B, const float* bias_C, const float* W_x,
                                         const float* W_o, const float* D, m3_state* state, void* y,
                                         void* stream) {
  size_t need = 0;
  m3_status st = m3_scan_workspace_size(dims, &need);
  if (st != M3_OK) return st;
  if (need > kScratchBytes) return M3_ERR_WORKSPACE;
  void* ws = nullptr;
  if (need > 0) {
    ws = m3::scratch_address();
    if (!ws) return M3_ERR_CUDA;
  }
  return m3_scan_fwd(dims, x, dt, A, lam, B, C, theta, bias_B, bias_C, W_x, W_o, D, state, y, ws,
                     need > 0 ? kScratchBytes : 0, stream);
}
