// Window attention with pooled global memory for callers that cannot allocate
// device memory.
//
// basa_window_attn needs a caller-provided workspace for the pooled K/V tokens.
// Some callers have no way to provide one: an operator plugged into a host
// framework that owns all device memory and hands its operators no workspace,
// or a latency-critical serving path that reserves its memory at start-up and
// forbids cudaMalloc/cudaFree afterwards (both calls can block the host and
// cudaFree synchronises the device, stalling every stream).  This entry point
// keeps the pooled K/V scratch in a fixed device array that is part of the
// library itself, so a call needs no allocation at all.
//
// Cost and limits:
//  - every GPU on which the library's device code is loaded holds the array
//    (kNoAllocScratchBytes) until the process exits;
//  - a problem whose pooled K and V together need more than that is refused with
//    BASA_ERR_SCRATCH_LIMIT;
//  - all calls on a device share the array: two calls whose work overlaps on the
//    GPU (different streams, no ordering between them) race on it, so such calls
//    must be ordered by the caller.  The array keeps whatever the last call left;
//    nothing in it has to start at zero, because the pooling kernel overwrites
//    every byte a call reads before the attention kernel reads it.
#include <mutex>

#include "basa_internal.h"

namespace basa {
namespace {

constexpr size_t kNoAllocScratchBytes = 32u << 20;  // 32 MiB per device
constexpr int kMaxDevices = 64;

// Host code sees only a host-side stand-in of this array; its device address
// comes from cudaGetSymbolAddress (per device, below).
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mu;
// Device address of g_noalloc_scratch per device, and the id of the CUDA
// context it was resolved in: a new context on the device (after
// cudaDeviceReset, say) loads the module afresh, and the array may then sit
// at another address.
void* g_scratch_addr[kMaxDevices];
unsigned long long g_scratch_ctx[kMaxDevices];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current CUDA context (driver entry points,
// so the library links no driver library), or 0 if it cannot be read.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) == cudaSuccess &&
        qa == cudaDriverEntryPointSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) == cudaSuccess &&
        qb == cudaDriverEntryPointSuccess) {
      get_current = reinterpret_cast<CtxGetCurrentFn>(a);
      get_id = reinterpret_cast<CtxGetIdFn>(b);
    }
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the scratch array on the current device; resolved on the
// first call made with that device current, and again whenever the current
// context is not the one the cached address belongs to.
basa_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return BASA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return BASA_ERR_UNSUPPORTED;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (!g_scratch_addr[dev] || ctx == 0 || ctx != g_scratch_ctx[dev]) {
    // the lookup also makes the device's primary context current if the
    // runtime had not done so yet, so the context id is read after it
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr)
      return BASA_ERR_CUDA;
    g_scratch_addr[dev] = ptr;
    g_scratch_ctx[dev] = current_context_id();
  }
  *out = g_scratch_addr[dev];
  return BASA_OK;
}

bool misaligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

}  // namespace
}  // namespace basa

using namespace basa;

extern "C" basa_status basa_window_attn_noalloc(const void* q, const void* k, const void* v,
                                                void* out, float* lse, const basa_params* p,
                                                cudaStream_t stream) {
  NvtxRange nvtx("basa_window_attn_noalloc");
  Dims d;
  basa_status s = normalise(p, false, &d);
  if (s != BASA_OK) return s;
  if ((long long)d.B * d.H * d.N == 0) return BASA_OK;
  if (!q || !k || !v || !out) return BASA_ERR_INVALID_ARG;
  if (misaligned16(q) || misaligned16(k) || misaligned16(v) || misaligned16(out) ||
      (lse && misaligned16(lse)))
    return BASA_ERR_ALIGN;
  if (d.dtype == BASA_BF16) {  // refuse unsupported plans before launching anything
    TilePlan plan;
    if ((s = build_tile_plan(d, &plan)) != BASA_OK) return s;
  }
  const void* kp = nullptr;
  const void* vp = nullptr;
  if (d.P > 0) {
    const size_t es = d.dtype == BASA_BF16 ? 2 : 4;
    const size_t one = (((size_t)d.B * (size_t)d.P * (size_t)d.Hkv * (size_t)d.d * es) + 255) &
                       ~(size_t)255;
    if (2 * one > kNoAllocScratchBytes) return BASA_ERR_SCRATCH_LIMIT;
    void* base = nullptr;
    if ((s = scratch_address(&base)) != BASA_OK) return s;
    unsigned char* kpw = static_cast<unsigned char*>(base);
    unsigned char* vpw = kpw + one;
    if ((s = launch_pool(d, k, v, kpw, vpw, stream)) != BASA_OK) return s;
    kp = kpw;
    vp = vpw;
  }
  if (d.dtype == BASA_F32) return launch_simt(d, q, k, v, kp, vp, out, lse, stream);
  return launch_tc_static_params(d, false, q, k, v, kp, vp, out, lse, p->flags,
                                 p->wait_timeout_ms, stream, d.P > 0);
}
