// archead_logits_noalloc: archead_logits for callers that cannot allocate device memory.
//
// Some callers cannot let a library allocate: serving engines that reserve nearly all of
// the GPU's memory up front for their own pool (KV cache and activations) and account for
// every byte themselves, and latency-critical decode loops that must not enter an
// allocator between kernels.  This entry point runs the same prologue and residual
// kernels as archead_logits, but its temporary buffers (the FP16 copy of H and the rank
// products t) live in one file-scope device array of fixed size instead of the library's
// stream-ordered pool.  It calls no cudaMalloc, cudaFree or other allocating routine.
#include <mutex>

#include "archead_internal.cuh"

namespace archead {
namespace {

// The fixed scratch: every GPU that loads the library holds it until the process exits.
constexpr size_t kScratchBytes = 2u << 20;  // 2 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDev = 64;

struct NoAllocDevice {
  bool ready = false;
  unsigned char* scratch = nullptr;  // device address of g_noalloc_scratch on this device
  unsigned* err = nullptr;           // device address of the library's error word
};

std::mutex g_mu;
NoAllocDevice g_devs[kMaxDev];

// Set-up, once per device, with that device current: the host-side name of a __device__
// array is only a stand-in, so its device address comes from cudaGetSymbolAddress.
int device_setup(NoAllocDevice** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return ARCHEAD_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  NoAllocDevice& d = g_devs[dev];
  if (!d.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
      cudaGetLastError();  // do not leave the failure for the caller's next error check
      return ARCHEAD_ERR_CUDA;
    }
    unsigned* e = error_word_address();
    if (!e) {
      cudaGetLastError();
      return ARCHEAD_ERR_CUDA;
    }
    d.scratch = static_cast<unsigned char*>(p);
    d.err = e;
    d.ready = true;
  }
  *out = &d;
  return ARCHEAD_OK;
}

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace
}  // namespace archead

using namespace archead;

extern "C" int archead_logits_noalloc(const uint16_t* H, const archead_head* head, float* Y,
                                      int64_t N, int64_t V, int64_t D, int r_c, int r_r,
                                      int g, void* stream) {
  int rc = validate_head_args(head, N, V, D, r_c, r_r, g);
  if (rc) return rc;
  if (N == 0) return ARCHEAD_OK;
  if (!H || !Y) return ARCHEAD_ERR_NULLPTR;
  if (reinterpret_cast<uintptr_t>(H) % 16 || reinterpret_cast<uintptr_t>(Y) % 4)
    return ARCHEAD_ERR_ALIGN;
  const int64_t tb = residual_token_block(N);
  const int64_t Npad = (N + tb - 1) / tb * tb;
  // beyond the fixed scratch: rejected before any product is formed, so no size wraps
  const int64_t cap = (int64_t)kScratchBytes;
  if (D > cap / 2 || Npad > cap / 2 / D || N > cap / 4 / (r_c + r_r + 1))
    return ARCHEAD_ERR_SHAPE;
  const size_t hh_bytes = round256((size_t)Npad * D * 2);
  const size_t t_bytes = round256((size_t)N * (r_c + r_r + 1) * 4 + 16);  // t, token scales
  if (hh_bytes + t_bytes > kScratchBytes) return ARCHEAD_ERR_SHAPE;
  NoAllocDevice* d = nullptr;
  rc = device_setup(&d);
  if (rc) return rc;
  // Every scratch byte a kernel reads is written earlier in the same call (the FP16 copy
  // of H including its zero padding rows, then t and the token scales), so nothing needs
  // clearing between calls.
  __half* Hh = reinterpret_cast<__half*>(d->scratch);
  float* t = reinterpret_cast<float*>(d->scratch + hh_bytes);
  float* tsc = t + N * (r_c + r_r);
  Shapes s;
  s.N = N;
  s.V = V;
  s.D = D;
  s.r_c = r_c;
  s.r_r = r_r;
  s.g = g;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int launches = 0;
  cudaError_t e = launch_prologue(H, head, s, Npad, Hh, t, tsc, d->err, st, &launches);
  if (e == cudaSuccess)
    e = launch_residual_gemm(Hh, t, tsc, head, s, Y, nullptr, nullptr, nullptr, st, &launches, 0);
  return e == cudaSuccess ? ARCHEAD_OK : ARCHEAD_ERR_CUDA;
}
