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

__device__ __forceinline__ void acc_bf16(float* a, const uint4& x) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    a[2 * i] += f.x;
    a[2 * i + 1] += f.y;
  }
}

__device__ __forceinline__ uint4 pack_bf16(const float* a, float s) {
  uint4 r;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&r);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(a[2 * i] * s, a[2 * i + 1] * s);
  return r;
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
  constexpr int E = kBf16 ? 8 : 4;  // elements per 16-byte vector
  const int ncell = a.pt * a.ph * a.pw;
  float ak[E], av[E];
#pragma unroll
  for (int i = 0; i < E; ++i) ak[i] = av[i] = 0.f;
  for (int i0 = 0; i0 < ncell; i0 += kPoolBatch) {
    uint4 xk[kPoolBatch], xv[kPoolBatch];
#pragma unroll
    for (int u = 0; u < kPoolBatch; ++u) {
      const int i = i0 + u;
      if (i < ncell) {
        const int it = i / (a.ph * a.pw), ih = (i / a.pw) % a.ph, iw = i % a.pw;
        const long long row =
            (((long long)b * a.T + ct * a.pt + it) * a.Hg + cy * a.ph + ih) * a.Wg + cx * a.pw + iw;
        const long long off = row * a.vec_per_token + vi;
        xk[u] = __ldcs(a.k + off);
        xv[u] = __ldcs(a.v + off);
      }
    }
#pragma unroll
    for (int u = 0; u < kPoolBatch; ++u) {
      if (i0 + u < ncell) {
        if (kBf16) {
          acc_bf16(ak, xk[u]);
          acc_bf16(av, xv[u]);
        } else {
          const float* fk = reinterpret_cast<const float*>(&xk[u]);
          const float* fv = reinterpret_cast<const float*>(&xv[u]);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            ak[e] += fk[e];
            av[e] += fv[e];
          }
        }
      }
    }
  }
  const long long o = ((long long)b * a.P + cell) * a.vec_per_token + vi;
  if (kBf16) {
    a.kp[o] = pack_bf16(ak, a.inv_count);
    a.vp[o] = pack_bf16(av, a.inv_count);
  } else {
    uint4 rk, rv;
    float* fk = reinterpret_cast<float*>(&rk);
    float* fv = reinterpret_cast<float*>(&rv);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      fk[e] = ak[e] * a.inv_count;
      fv[e] = av[e] * a.inv_count;
    }
    a.kp[o] = rk;
    a.vp[o] = rv;
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
