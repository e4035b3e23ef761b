// K/V mean pooling into global-memory tokens (forum review of the BASA paper,
// zhichai.net topic 178635722 reply 178634520, four-part method list: K/V
// pooled global memory).  Cells are pt x ph x pw boxes aligned to the grid
// origin; each pooled token is the plain mean of its cell's tokens.
//
// HBM-bound: every input byte is read once, every output byte written once.
// A CTA of 128 threads owns 128 consecutive 16-byte vectors of one pooled
// cell's H*d row (a cell's row splits over ceil(H*d*esize/2048) CTAs).  Each
// thread walks the cell's pt*ph*pw tokens eight at a time, issuing all sixteen
// 16-byte K and V loads of a batch before accumulating them in fp32, so that
// enough loads are in flight to cover HBM latency.  Consecutive threads read
// consecutive 16-byte pieces of a token row, so every warp load is coalesced.
// The walk over the cell keeps (row, column) counters and a running offset
// instead of dividing the token index, and bf16 pairs are widened by shifts
// and summed with packed fp32x2 adds: the kernel issues few enough
// instructions per byte to stay on the memory system's pace.
//
// Each CTA allows the next kernel in the stream to start as soon as its loads
// are issued (programmatic dependent launch); a dependent kernel that reads
// the pooled tokens waits for this grid's completion before doing so.
#include <cuda_bf16.h>

#include "basa_internal.h"

namespace basa {
namespace {

struct PoolArgs {
  const uint4* k;
  const uint4* v;
  uint4* kp;
  uint4* vp;
  int T, Hg, Wg, pt, ph, pw;
  int Pt, Ph, Pw;
  int vec_per_token;  // 16-byte vectors per token row of H*d values
  int vec_blocks;     // CTAs per pooled cell
  int P;              // pooled cells per batch
  float inv_count;
};

// fp32 pairs in one 64-bit register (the packed f32x2 arithmetic of sm_100).
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
  uint64_t d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}
__device__ __forceinline__ uint64_t f2add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float2 f2unpack(uint64_t v) {
  float2 f;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(f.x), "=f"(f.y) : "l"(v));
  return f;
}

// a[i] += the i-th bf16 pair of x, widened exactly (a bf16 value is the upper
// half of the fp32 value it stands for).
__device__ __forceinline__ void acc_bf16(uint64_t* a, const uint4& x) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
    a[i] = f2add(a[i], f2pack(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u)));
}

__device__ __forceinline__ uint4 pack_bf16(const uint64_t* a, float s) {
  uint4 r;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&r);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = f2unpack(a[i]);
    h[i] = __floats2bfloat162_rn(f.x * s, f.y * s);
  }
  return r;
}

__device__ __forceinline__ void allow_dependent_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

constexpr int kPoolThreads = 128;
constexpr int kPoolBatch = 8;  // tokens whose loads are issued together

template <bool kBf16>
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(PoolArgs a) {
  const int cell = blockIdx.x / a.vec_blocks;  // flattened (ct, cy, cx)
  const int vi = (blockIdx.x % a.vec_blocks) * kPoolThreads + threadIdx.x;
  const int b = blockIdx.y;
  if (vi >= a.vec_per_token) return;
  const int cx = cell % a.Pw, cy = (cell / a.Pw) % a.Ph, ct = cell / (a.Pw * a.Ph);
  const int ncell = a.pt * a.ph * a.pw;
  const long long vpt = a.vec_per_token;
  // the cell's tokens in (t, row, column) order: a running offset, advanced by
  // one token, at the end of a row of pw tokens to the next row of the cell,
  // and at the end of ph rows to the cell's next frame
  long long off =
      ((((long long)b * a.T + ct * a.pt) * a.Hg + cy * a.ph) * a.Wg + cx * a.pw) * vpt + vi;
  const long long next_row = (long long)(a.Wg - a.pw) * vpt;
  const long long next_frame = (long long)(a.Hg - a.ph) * a.Wg * vpt;
  int iw = 0, ih = 0;
  uint64_t ak[4], av[4];  // bf16: four fp32 pairs; fp32: the first two pairs
#pragma unroll
  for (int i = 0; i < 4; ++i) ak[i] = av[i] = f2pack(0.f, 0.f);
  for (int i0 = 0; i0 < ncell; i0 += kPoolBatch) {
    uint4 xk[kPoolBatch], xv[kPoolBatch];
#pragma unroll
    for (int u = 0; u < kPoolBatch; ++u) {
      if (i0 + u < ncell) {
        xk[u] = __ldcs(a.k + off);
        xv[u] = __ldcs(a.v + off);
        off += vpt;
        if (++iw == a.pw) {
          iw = 0;
          off += next_row;
          if (++ih == a.ph) {
            ih = 0;
            off += next_frame;
          }
        }
      }
    }
    if (i0 == 0) allow_dependent_launch();
#pragma unroll
    for (int u = 0; u < kPoolBatch; ++u) {
      if (i0 + u < ncell) {
        if (kBf16) {
          acc_bf16(ak, xk[u]);
          acc_bf16(av, xv[u]);
        } else {
          ak[0] = f2add(ak[0], f2pack(__uint_as_float(xk[u].x), __uint_as_float(xk[u].y)));
          ak[1] = f2add(ak[1], f2pack(__uint_as_float(xk[u].z), __uint_as_float(xk[u].w)));
          av[0] = f2add(av[0], f2pack(__uint_as_float(xv[u].x), __uint_as_float(xv[u].y)));
          av[1] = f2add(av[1], f2pack(__uint_as_float(xv[u].z), __uint_as_float(xv[u].w)));
        }
      }
    }
  }
  const long long o = ((long long)b * a.P + cell) * a.vec_per_token + vi;
  if (kBf16) {
    a.kp[o] = pack_bf16(ak, a.inv_count);
    a.vp[o] = pack_bf16(av, a.inv_count);
  } else {
    const float s = a.inv_count;
    const float2 k0 = f2unpack(ak[0]), k1 = f2unpack(ak[1]);
    const float2 v0 = f2unpack(av[0]), v1 = f2unpack(av[1]);
    a.kp[o] = make_uint4(__float_as_uint(k0.x * s), __float_as_uint(k0.y * s),
                         __float_as_uint(k1.x * s), __float_as_uint(k1.y * s));
    a.vp[o] = make_uint4(__float_as_uint(v0.x * s), __float_as_uint(v0.y * s),
                         __float_as_uint(v1.x * s), __float_as_uint(v1.y * s));
  }
}

}  // namespace

basa_status launch_pool(const Dims& d, const void* k, const void* v, void* kp, void* vp,
                        cudaStream_t stream) {
  PoolArgs a;
  a.k = static_cast<const uint4*>(k);
  a.v = static_cast<const uint4*>(v);
  a.kp = static_cast<uint4*>(kp);
  a.vp = static_cast<uint4*>(vp);
  a.T = d.T; a.Hg = d.Hg; a.Wg = d.Wg;
  a.pt = d.pt; a.ph = d.ph; a.pw = d.pw;
  a.Pt = d.T / d.pt; a.Ph = d.Hg / d.ph; a.Pw = d.Wg / d.pw;
  const int es = d.dtype == BASA_BF16 ? 2 : 4;
  a.vec_per_token = d.Hkv * d.d * es / 16;
  a.inv_count = 1.0f / (float)(d.pt * d.ph * d.pw);
  a.vec_blocks = (a.vec_per_token + kPoolThreads - 1) / kPoolThreads;
  a.P = (int)d.P;
  if (d.P * a.vec_blocks > 0x7fffffffLL || d.B > 65535) return BASA_ERR_UNSUPPORTED;
  dim3 grid((unsigned)(d.P * a.vec_blocks), (unsigned)d.B);
  if (d.dtype == BASA_BF16)
    pool_kernel<true><<<grid, kPoolThreads, 0, stream>>>(a);
  else
    pool_kernel<false><<<grid, kPoolThreads, 0, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? BASA_OK : BASA_ERR_CUDA;
}

}  // namespace basa
