// fp32 shifted local window attention on CUDA cores ("BASA: Backend-Agnostic
// Sparse Attention for Fast High-Resolution Diffusion Transformers", zhichai.net
// topic 178635722, "The BASA Method"): each query attends to the tokens of its
// own cyclically shifted window (window id floor(((x - s) mod G) / w) per axis),
// plus the pooled global-memory tokens when they are given, under one softmax.
// Full attention is the same kernel with one window covering the grid.
//
// Exact fp32 arithmetic (fp32 FMA dot products, expf, fp32 accumulation), so
// the results stay within 1e-5 of an fp64 evaluation at the sizes this path
// serves.  One CTA of 128 threads handles a chunk of one window's queries for
// one (b, h); key/value rows of the window (then the pooled rows) are staged in
// shared memory 32 at a time.  Window members are addressed through the shift
// index math directly: no rolled copy of the grid is made.
#include <math.h>

#include "basa_internal.h"

namespace basa {
namespace {

constexpr int kThreads = 128;
constexpr int kKeyChunk = 32;

struct SimtArgs {
  const float* q;
  const float* k;
  const float* v;
  const float* kp;  // pooled [B, P, H, D] or null
  const float* vp;
  float* out;
  float* lse;       // [B, H, N] or null
  int B, H, T, Hg, Wg;
  int Hkv;          // K/V heads; query head h reads K/V head h / (H / Hkv)
  int wt, wh, ww, st, sh, sw;
  int nwt, nwh, nww;
  int Tp, Hgp, Wgp; // padded extents the windows wrap on (T, Hg, Wg unless padded);
                    // members at coordinates past T, Hg or Wg are padding: no token
  int m;            // window positions (tokens plus padding)
  int P;            // pooled tokens (0 = none)
  int n_qchunks;    // query chunks per window
  long long N;
  long long Nq;     // query rows per (b, h) when qsep (text queries)
  int qsep;         // 1: queries are rows [B, Nq, H, d] against the whole grid
  float scale;
};

__device__ __forceinline__ long long token_row(const SimtArgs& a, int b, int t, int y, int x) {
  return (((long long)b * a.T + t) * a.Hg + y) * a.Wg + x;
}

template <int D>
__global__ void __launch_bounds__(kThreads) simt_window_kernel(SimtArgs a) {
  constexpr int TPQ = D > 64 ? 2 : 1;  // threads per query
  constexpr int DPT = D / TPQ;         // head-dim elements per thread
  constexpr int QPC = kThreads / TPQ;  // queries per CTA
  constexpr int V4 = D / 4;            // float4 per row
  __shared__ float4 ks[kKeyChunk][V4];
  __shared__ float4 vs[kKeyChunk][V4];
  __shared__ int kok[kKeyChunk];  // key jj of the chunk is a token (not padding)

  long long u = blockIdx.x;
  const int qc = (int)(u % a.n_qchunks);
  u /= a.n_qchunks;
  const int nwin = a.nwt * a.nwh * a.nww;
  const int win = (int)(u % nwin);
  u /= nwin;
  const int h = (int)(u % a.H);
  const int b = (int)(u / a.H);
  const int hk = h / (a.H / a.Hkv);
  const int jw = win % a.nww, jh = (win / a.nww) % a.nwh, jt = win / (a.nww * a.nwh);
  const int ot = jt * a.wt + a.st, oh = jh * a.wh + a.sh, ow = jw * a.ww + a.sw;

  const int part = threadIdx.x % TPQ;
  const int lq = qc * QPC + threadIdx.x / TPQ;
  bool valid = a.qsep ? lq < a.Nq : lq < a.m;
  long long qrow = 0;
  long long qn = 0;
  float qr[DPT];
  if (valid && a.qsep) {  // a text query: its own row, the grid is one window
    qn = lq;
    qrow = (long long)b * a.Nq + lq;
    const float* qp = a.q + (qrow * a.H + h) * D + part * DPT;
#pragma unroll
    for (int c = 0; c < DPT; ++c) qr[c] = qp[c];
  } else if (valid) {
    const int lt = lq / (a.wh * a.ww), lh = (lq / a.ww) % a.wh, lw = lq % a.ww;
    const int t = (ot + lt) % a.Tp, y = (oh + lh) % a.Hgp, x = (ow + lw) % a.Wgp;
    valid = t < a.T && y < a.Hg && x < a.Wg;  // a padded position is no query
    qn = valid ? ((long long)t * a.Hg + y) * a.Wg + x : 0;
    qrow = valid ? token_row(a, b, t, y, x) : 0;
    const float* qp = a.q + (qrow * a.H + h) * D + part * DPT;
#pragma unroll
    for (int c = 0; c < DPT; ++c) qr[c] = valid ? qp[c] : 0.f;
  } else {
#pragma unroll
    for (int c = 0; c < DPT; ++c) qr[c] = 0.f;
  }

  float mrun = -INFINITY, l = 0.f;
  float acc[DPT];
#pragma unroll
  for (int c = 0; c < DPT; ++c) acc[c] = 0.f;

  const int nkeys = a.m + a.P;
  for (int k0 = 0; k0 < nkeys; k0 += kKeyChunk) {
    const int nk = nkeys - k0 < kKeyChunk ? nkeys - k0 : kKeyChunk;
    __syncthreads();
    for (int idx = threadIdx.x; idx < nk * V4; idx += kThreads) {
      const int jj = idx / V4, c4 = idx % V4;
      const int j = k0 + jj;
      const float4* kr;
      const float4* vr;
      if (j < a.m) {
        const int lt = j / (a.wh * a.ww), lh = (j / a.ww) % a.wh, lw = j % a.ww;
        const int t = (ot + lt) % a.Tp, y = (oh + lh) % a.Hgp, x = (ow + lw) % a.Wgp;
        const bool tok = t < a.T && y < a.Hg && x < a.Wg;
        if (c4 == 0) kok[jj] = tok ? 1 : 0;
        if (!tok) {  // padding: no key
          ks[jj][c4] = make_float4(0.f, 0.f, 0.f, 0.f);
          vs[jj][c4] = make_float4(0.f, 0.f, 0.f, 0.f);
          continue;
        }
        const long long row = token_row(a, b, t, y, x);
        kr = reinterpret_cast<const float4*>(a.k + (row * a.Hkv + hk) * D);
        vr = reinterpret_cast<const float4*>(a.v + (row * a.Hkv + hk) * D);
      } else {
        if (c4 == 0) kok[jj] = 1;
        const long long prow = (long long)b * a.P + (j - a.m);
        kr = reinterpret_cast<const float4*>(a.kp + (prow * a.Hkv + hk) * D);
        vr = reinterpret_cast<const float4*>(a.vp + (prow * a.Hkv + hk) * D);
      }
      ks[jj][c4] = kr[c4];
      vs[jj][c4] = vr[c4];
    }
    __syncthreads();
    float s[kKeyChunk];
    float cmax = -INFINITY;
#pragma unroll
    for (int jj = 0; jj < kKeyChunk; ++jj) {
      float dot = 0.f;
      const float* kr = reinterpret_cast<const float*>(&ks[jj][0]) + part * DPT;
#pragma unroll
      for (int c = 0; c < DPT; ++c) dot = fmaf(qr[c], kr[c], dot);
      if (TPQ == 2) dot += __shfl_xor_sync(0xffffffffu, dot, 1);
      s[jj] = (jj < nk && kok[jj]) ? dot * a.scale : -INFINITY;
      cmax = fmaxf(cmax, s[jj]);
    }
    const float mnew = fmaxf(mrun, cmax);
    if (mnew == -INFINITY) continue;  // every key so far is padding (same for every query)
    const float corr = expf(mrun - mnew);  // 0 on the first chunk
    l *= corr;
#pragma unroll
    for (int c = 0; c < DPT; ++c) acc[c] *= corr;
#pragma unroll
    for (int jj = 0; jj < kKeyChunk; ++jj) {
      if (jj < nk && kok[jj]) {
        const float p = expf(s[jj] - mnew);
        l += p;
        const float* vr = reinterpret_cast<const float*>(&vs[jj][0]) + part * DPT;
#pragma unroll
        for (int c = 0; c < DPT; ++c) acc[c] = fmaf(p, vr[c], acc[c]);
      }
    }
    mrun = mnew;
  }

  if (valid) {
    const float inv = 1.0f / l;
    float* op = a.out + (qrow * a.H + h) * D + part * DPT;
#pragma unroll
    for (int c = 0; c < DPT; c += 4)
      *reinterpret_cast<float4*>(op + c) =
          make_float4(acc[c] * inv, acc[c + 1] * inv, acc[c + 2] * inv, acc[c + 3] * inv);
    if (a.lse && part == 0) a.lse[((long long)b * a.H + h) * (a.qsep ? a.Nq : a.N) + qn] =
        mrun + logf(l);
  }
}

}  // namespace

basa_status launch_simt(const Dims& d, const void* q, const void* k, const void* v,
                        const void* kp, const void* vp, void* out, float* lse,
                        cudaStream_t stream) {
  SimtArgs a;
  a.q = static_cast<const float*>(q);
  a.k = static_cast<const float*>(k);
  a.v = static_cast<const float*>(v);
  a.kp = static_cast<const float*>(kp);
  a.vp = static_cast<const float*>(vp);
  a.out = static_cast<float*>(out);
  a.lse = lse;
  a.B = d.B; a.H = d.H; a.T = d.T; a.Hg = d.Hg; a.Wg = d.Wg;
  a.Hkv = d.Hkv;
  a.wt = d.wt; a.wh = d.wh; a.ww = d.ww;
  a.st = d.st; a.sh = d.sh; a.sw = d.sw;
  a.nwt = d.nwt; a.nwh = d.nwh; a.nww = d.nww;
  a.Tp = d.Tp > 0 ? d.Tp : d.T;
  a.Hgp = d.Hgp > 0 ? d.Hgp : d.Hg;
  a.Wgp = d.Wgp > 0 ? d.Wgp : d.Wg;
  const long long m = (long long)d.wt * d.wh * d.ww;
  if (m > (1LL << 30)) return BASA_ERR_UNSUPPORTED;
  a.m = (int)m;
  a.P = kp ? (int)d.P : 0;
  a.N = d.N;
  a.Nq = d.Nq;
  a.qsep = d.qsep;
  a.scale = d.scale;
  const int qpc = d.d > 64 ? kThreads / 2 : kThreads;
  const long long nq = d.qsep ? d.Nq : m;
  if (nq > (1LL << 30)) return BASA_ERR_UNSUPPORTED;
  a.n_qchunks = (int)((nq + qpc - 1) / qpc);
  const long long units = (long long)d.B * d.H * d.nwt * d.nwh * d.nww * a.n_qchunks;
  if (units > 0x7fffffffLL) return BASA_ERR_UNSUPPORTED;
  if (units == 0) return BASA_OK;
  switch (d.d) {
    case 32: simt_window_kernel<32><<<(unsigned)units, kThreads, 0, stream>>>(a); break;
    case 64: simt_window_kernel<64><<<(unsigned)units, kThreads, 0, stream>>>(a); break;
    case 128: simt_window_kernel<128><<<(unsigned)units, kThreads, 0, stream>>>(a); break;
    default: return BASA_ERR_UNSUPPORTED;
  }
  return cudaGetLastError() == cudaSuccess ? BASA_OK : BASA_ERR_CUDA;
}

}  // namespace basa
