// K/V mean pooling into global-memory tokens (forum review of the BASA paper,
// zhichai.net topic 178635722 reply 178634520, four-part method list: K/V
// pooled global memory).  Cells are pt x ph x pw boxes aligned to the grid
// origin; each pooled token is the plain mean of its cell's tokens.
//
// HBM-bound: every input byte is read once, every output byte written once.
// One CTA per (pooled cell, batch); each thread owns one 16-byte vector of the
// cell's H*d values and walks the cell's pt*ph*pw tokens with 16-byte loads
// (consecutive threads read consecutive 16-byte pieces of a token's H*d row, so
// every warp load is fully coalesced), accumulating in fp32.
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

template <bool kBf16>
__global__ void __launch_bounds__(512) pool_kernel(PoolArgs a) {
  const int cell = blockIdx.x;  // flattened (ct, cy, cx)
  const int b = blockIdx.y;
  const int cx = cell % a.Pw, cy = (cell / a.Pw) % a.Ph, ct = cell / (a.Pw * a.Ph);
  constexpr int E = kBf16 ? 8 : 4;  // elements per 16-byte vector
  for (int vi = threadIdx.x; vi < a.vec_per_token; vi += blockDim.x) {
    float ak[E], av[E];
#pragma unroll
    for (int i = 0; i < E; ++i) ak[i] = av[i] = 0.f;
    for (int i = 0; i < a.pt; ++i)
      for (int j = 0; j < a.ph; ++j) {
        const long long row =
            (((long long)b * a.T + ct * a.pt + i) * a.Hg + cy * a.ph + j) * a.Wg + cx * a.pw;
#pragma unroll 4
        for (int l = 0; l < a.pw; ++l) {
          const long long off = (row + l) * a.vec_per_token + vi;
          const uint4 xk = __ldcs(a.k + off);
          const uint4 xv = __ldcs(a.v + off);
          if (kBf16) {
            acc_bf16(ak, xk);
            acc_bf16(av, xv);
          } else {
            const float* fk = reinterpret_cast<const float*>(&xk);
            const float* fv = reinterpret_cast<const float*>(&xv);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              ak[e] += fk[e];
              av[e] += fv[e];
            }
          }
        }
      }
    const long long o = ((long long)b * gridDim.x + cell) * a.vec_per_token + vi;
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
  a.vec_per_token = d.H * d.d * es / 16;
  a.inv_count = 1.0f / (float)(d.pt * d.ph * d.pw);
  if (d.P > 0x7fffffffLL || d.B > 65535) return BASA_ERR_UNSUPPORTED;
  dim3 grid((unsigned)d.P, (unsigned)d.B);
  int threads = a.vec_per_token < 512 ? ((a.vec_per_token + 31) / 32) * 32 : 512;
  if (d.dtype == BASA_BF16)
    pool_kernel<true><<<grid, threads, 0, stream>>>(a);
  else
    pool_kernel<false><<<grid, threads, 0, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? BASA_OK : BASA_ERR_CUDA;
}

}  // namespace basa
