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
void* g_scratch_addr[kMaxDevices];  // device address of g_noalloc_scratch, per device

// Device address of the scratch array on the current device; resolved once per
// device, on the first call made with that device current.
basa_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return BASA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return BASA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr)
      return BASA_ERR_CUDA;
    g_scratch_addr[dev] = ptr;
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
                                 p->wait_timeout_ms, stream);
}
