// Backward of shifted local window attention on CUDA cores: dQ, dK, dV for an
// output gradient dO ("BASA: Backend-Agnostic Sparse Attention for Fast
// High-Resolution Diffusion Transformers", zhichai.net topic 178635722, "The
// BASA Method": each query attends to the keys of its own cyclically shifted
// window; the same pages' review names the dense-teacher adaptation that
// trains through this attention).
//
// With P_ij = exp(scale * q_i . k_j - lse_i) over the keys j of query i's
// window (lse from the forward pass), and D_i = dO_i . O_i:
//   dS_ij = P_ij (dO_i . v_j - D_i)
//   dQ_i  = scale * sum_j dS_ij k_j
//   dK_j  = scale * sum_i dS_ij q_i      (over the query heads sharing k_j)
//   dV_j  = sum_i P_ij dO_i
// Every key of a window is attended only by that window's queries, so each
// (b, K/V head, window) owns its dK, dV rows: no atomics.  Launches: D =
// rowsum(dO * O) into the caller's workspace (also used by the tensor-core
// backward); with pooled memory the pooled tokens' gradients, each summed over
// every query of its batch into fp32 buffers; dQ (a group of threads per query,
// the window's keys and then the pooled keys staged in shared memory); dK and
// dV (a group of threads per key, queries staged; d / 32 threads per row), each
// row adding its cell's pooled gradient divided by the cell size.  Arithmetic
// is fp32; bf16 inputs are widened on load and the gradients rounded once.
#include <cuda_bf16.h>
#include <math.h>

#include "basa_internal.h"

namespace basa {
namespace {

constexpr int kBwdThreads = 128;
constexpr int kChunk = 32;  // keys (or queries) staged per step

struct BwdArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* o;
  const void* dout;
  const float* lse;  // [B, H, N]
  float* dD;         // [B, H, N] workspace: dO . O
  void* dq;
  void* dk;
  void* dv;
  int B, H, Hkv, T, Hg, Wg;
  int wt, wh, ww, st, sh, sw, nwt, nwh, nww;
  int Tp, Hgp, Wgp; // padded extents the windows wrap on (T, Hg, Wg unless padded)
  int m;            // window positions (tokens plus padding)
  int n_chunks;     // query (or key) chunks per window
  long long N;
  float scale;
  // pooled global memory (P = 0: none)
  const void* kp;   // pooled K, V [B, P, Hkv, d] in the input dtype
  const void* vp;
  float* dkp;       // [B, P, Hkv, d] fp32: sum over the batch's queries of dS^T Q (no scale)
  float* dvp;       // [B, P, Hkv, d] fp32: sum of P^T dO
  long long P;
  int pt, ph, pw;
  int p_chunks;     // pooled key chunks
  float inv_count;  // 1 / (pt * ph * pw)
  // joint text tokens: the extra keys (kp, vp, P) are then the L text tokens,
  // not pooled cells, and the L text queries see every image and text token
  int joint;
  const void* qt;       // [B, L, H, d]
  const void* dout_t;
  const float* lse_t;   // [B, H, L]
  const float* dD_t;    // [B, H, L]: dout_t . out_t
  void* dqt;            // [B, L, H, d]
  void* dkt;            // [B, L, Hkv, d]
  void* dvt;
  int t_chunks;         // text query chunks
  const void* joint_out;  // out_t [B, L, H, d] (for D of the text rows)
};

template <bool BF16>
__device__ __forceinline__ float ld1(const void* base, long long i) {
  if (BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[i]);
  return reinterpret_cast<const float*>(base)[i];
}
template <bool BF16>
__device__ __forceinline__ void st1(void* base, long long i, float x) {
  if (BF16)
    reinterpret_cast<__nv_bfloat16*>(base)[i] = __float2bfloat16_rn(x);
  else
    reinterpret_cast<float*>(base)[i] = x;
}

// Flattened grid token of member j of window (jt, jh, jw), or -1 when the
// position is padding (past T, Hg or Wg on the padded axes).
__device__ __forceinline__ long long member(const BwdArgs& a, int jt, int jh, int jw, int j) {
  const int lt = j / (a.wh * a.ww), lh = (j / a.ww) % a.wh, lw = j % a.ww;
  int t = jt * a.wt + a.st + lt, y = jh * a.wh + a.sh + lh, x = jw * a.ww + a.sw + lw;
  t = t >= a.Tp ? t - a.Tp : t;
  y = y >= a.Hgp ? y - a.Hgp : y;
  x = x >= a.Wgp ? x - a.Wgp : x;
  if (t >= a.T || y >= a.Hg || x >= a.Wg) return -1;
  return ((long long)t * a.Hg + y) * a.Wg + x;
}

// Sum of x over the TPQ consecutive lanes that share one query (or key).
template <int TPQ>
__device__ __forceinline__ float lane_sum(float x) {
#pragma unroll
  for (int o = 1; o < TPQ; o <<= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// D = rowsum(dO * O) for every (b, n, h).  HBM-bound: LPR = d * esize / 16
// consecutive lanes read one row with 16-byte loads (a warp covers 32 / LPR
// whole rows, so every load instruction reads contiguous bytes), multiply in
// fp32 and add across their lanes.  Each warp issues the loads of kPrepGroups
// such row groups before it uses any, so that enough bytes are in flight, and
// splits the row index in 32-bit arithmetic when the rows fit.
constexpr int kPrepGroups = 4;
template <bool BF16, int D>
__global__ void __launch_bounds__(kBwdThreads) bwd_prep_kernel(BwdArgs a) {
  constexpr int LPR = D * (BF16 ? 2 : 4) / 16;  // lanes per row
  constexpr int RPW = 32 / LPR;                 // rows per warp and group
  constexpr int U = kPrepGroups;
  const long long rows = (long long)a.B * a.N * a.H;
  const long long warp = ((long long)blockIdx.x * kBwdThreads + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  const int sub = lane % LPR;
  uint4 x[U], y[U];
  long long r[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    r[u] = (warp * U + u) * RPW + lane / LPR;
    if (r[u] < rows) {
      x[u] = __ldcs(reinterpret_cast<const uint4*>(a.dout) + r[u] * LPR + sub);
      y[u] = __ldcs(reinterpret_cast<const uint4*>(a.o) + r[u] * LPR + sub);
    }
  }
  const bool small = rows <= 0xffffffffLL;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    float acc = 0.f;
    if (r[u] < rows) {
      if (BF16) {
        const __nv_bfloat162* hx = reinterpret_cast<const __nv_bfloat162*>(&x[u]);
        const __nv_bfloat162* hy = reinterpret_cast<const __nv_bfloat162*>(&y[u]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 fx = __bfloat1622float2(hx[i]), fy = __bfloat1622float2(hy[i]);
          acc = fmaf(fx.x, fy.x, acc);
          acc = fmaf(fx.y, fy.y, acc);
        }
      } else {
        acc = fmaf(__uint_as_float(x[u].x), __uint_as_float(y[u].x), acc);
        acc = fmaf(__uint_as_float(x[u].y), __uint_as_float(y[u].y), acc);
        acc = fmaf(__uint_as_float(x[u].z), __uint_as_float(y[u].z), acc);
        acc = fmaf(__uint_as_float(x[u].w), __uint_as_float(y[u].w), acc);
      }
    }
    acc = lane_sum<LPR>(acc);
    if (r[u] < rows && sub == 0) {
      long long h, n, b;
      if (small) {
        const uint32_t rr = (uint32_t)r[u], t = rr / (uint32_t)a.H;
        h = rr - t * (uint32_t)a.H;
        n = t % (uint32_t)a.N;
        b = t / (uint32_t)a.N;
      } else {
        h = r[u] % a.H;
        n = (r[u] / a.H) % a.N;
        b = r[u] / ((long long)a.H * a.N);
      }
      a.dD[(b * a.H + h) * a.N + n] = acc;
    }
  }
}

// dQ: one CTA per (b, h, window, query chunk); D / 32 threads per query.
// TEXTQ (joint): one CTA per (b, h, text query chunk); the keys are every
// image token and then every text token.
template <bool BF16, int D, bool TEXTQ>
__global__ void __launch_bounds__(kBwdThreads) bwd_dq_kernel(BwdArgs a) {
  constexpr int TPQ = D / 32;
  constexpr int DPT = D / TPQ;
  constexpr int QPC = kBwdThreads / TPQ;
  __shared__ float ks[kChunk][D];
  __shared__ float vs[kChunk][D];
  __shared__ int kok[kChunk];  // key jj of the chunk is a token (not padding)
  long long u = blockIdx.x;
  const int qc = (int)(u % (TEXTQ ? a.t_chunks : a.n_chunks));
  u /= (TEXTQ ? a.t_chunks : a.n_chunks);
  const int nwin = TEXTQ ? 1 : a.nwt * a.nwh * a.nww;
  const int win = (int)(u % nwin);
  u /= nwin;
  const int h = (int)(u % a.H);
  const int b = (int)(u / a.H);
  const int hk = h / (a.H / a.Hkv);
  const int jw = win % a.nww, jh = (win / a.nww) % a.nwh, jt = win / (a.nww * a.nwh);
  const int part = threadIdx.x % TPQ;
  const long long lq = (long long)qc * QPC + threadIdx.x / TPQ;
  const long long n = lq < (TEXTQ ? (long long)a.P : (long long)a.m)
                          ? (TEXTQ ? lq : member(a, jt, jh, jw, (int)lq)) : -1;
  const bool valid = n >= 0;  // padding and rows past the window are no query
  float qr[DPT], gr[DPT], acc[DPT];
  float lse = 0.f, dd = 0.f;
  long long qrow = 0;
  if (valid) {
    const long long nrows = TEXTQ ? (long long)a.P : a.N;
    qrow = (((long long)b * nrows + n) * a.H + h) * D + part * DPT;
    for (int c = 0; c < DPT; ++c) {
      qr[c] = ld1<BF16>(TEXTQ ? a.qt : a.q, qrow + c);
      gr[c] = ld1<BF16>(TEXTQ ? a.dout_t : a.dout, qrow + c);
    }
    lse = (TEXTQ ? a.lse_t : a.lse)[((long long)b * a.H + h) * nrows + n];
    dd = (TEXTQ ? a.dD_t : a.dD)[((long long)b * a.H + h) * nrows + n];
  } else {
    for (int c = 0; c < DPT; ++c) qr[c] = gr[c] = 0.f;
  }
  for (int c = 0; c < DPT; ++c) acc[c] = 0.f;
  // the window's keys (text queries: every image token), then the extra keys
  const long long nbase = TEXTQ ? a.N : (long long)a.m;
  const long long nkeys = nbase + a.P;
  for (long long k0 = 0; k0 < nkeys; k0 += kChunk) {
    const int nk = nkeys - k0 < kChunk ? (int)(nkeys - k0) : kChunk;
    __syncthreads();
    for (int idx = threadIdx.x; idx < nk * D; idx += kBwdThreads) {
      const int jj = idx / D, c = idx % D;
      const long long j = k0 + jj;
      if (j < nbase) {
        const long long kn = TEXTQ ? j : member(a, jt, jh, jw, (int)j);
        if (c == 0) kok[jj] = kn >= 0;
        if (kn < 0) {  // padding: no key
          ks[jj][c] = vs[jj][c] = 0.f;
          continue;
        }
        const long long off = (((long long)b * a.N + kn) * a.Hkv + hk) * D + c;
        ks[jj][c] = ld1<BF16>(a.k, off);
        vs[jj][c] = ld1<BF16>(a.v, off);
      } else {
        if (c == 0) kok[jj] = 1;
        const long long off = (((long long)b * a.P + (j - nbase)) * a.Hkv + hk) * D + c;
        ks[jj][c] = ld1<BF16>(a.kp, off);
        vs[jj][c] = ld1<BF16>(a.vp, off);
      }
    }
    __syncthreads();
    for (int jj = 0; jj < nk; ++jj) {
      float s = 0.f, dp = 0.f;
      for (int c = 0; c < DPT; ++c) {
        s = fmaf(qr[c], ks[jj][part * DPT + c], s);
        dp = fmaf(gr[c], vs[jj][part * DPT + c], dp);
      }
      s = lane_sum<TPQ>(s);
      dp = lane_sum<TPQ>(dp);
      const float pw = kok[jj] ? expf(s * a.scale - lse) : 0.f;
      const float ds = pw * (dp - dd);
      for (int c = 0; c < DPT; ++c) acc[c] = fmaf(ds, ks[jj][part * DPT + c], acc[c]);
    }
  }
  if (valid)
    for (int c = 0; c < DPT; ++c) st1<BF16>(TEXTQ ? a.dqt : a.dq, qrow + c, acc[c] * a.scale);
}

// dK, dV: one CTA per (b, K/V head, window, key chunk); the queries of every
// head of the group are staged in turn.  With pooled memory the row's share of
// its cell's pooled gradient (dkp, dvp / count) is added before the scale.
// POOL: the pooled tokens' gradients instead: one CTA per (b, K/V head, pooled
// key chunk), the queries being every token of the batch; fp32 sums to dkp, dvp.
template <bool BF16, int D, bool POOL>
__global__ void __launch_bounds__(kBwdThreads) bwd_dkv_kernel(BwdArgs a) {
  constexpr int TPQ = D / 32;
  constexpr int DPT = D / TPQ;
  constexpr int KPC = kBwdThreads / TPQ;
  __shared__ float qs[kChunk][D];
  __shared__ float gs[kChunk][D];
  __shared__ float ls[kChunk], ds_[kChunk];
  long long u = blockIdx.x;
  const int kc = (int)(u % (POOL ? a.p_chunks : a.n_chunks));
  u /= (POOL ? a.p_chunks : a.n_chunks);
  const int nwin = POOL ? 1 : a.nwt * a.nwh * a.nww;
  const int win = (int)(u % nwin);
  u /= nwin;
  const int hk = (int)(u % a.Hkv);
  const int b = (int)(u / a.Hkv);
  const int group = a.H / a.Hkv;
  const int jw = win % a.nww, jh = (win / a.nww) % a.nwh, jt = win / (a.nww * a.nwh);
  const int part = threadIdx.x % TPQ;
  const long long lk = (long long)kc * KPC + threadIdx.x / TPQ;
  const long long n_row = (!POOL && lk < a.m) ? member(a, jt, jh, jw, (int)lk) : 0;
  const bool valid = lk < (POOL ? a.P : a.m) && n_row >= 0;  // padding is no key
  float kr[DPT], vr[DPT], dk[DPT], dv[DPT];
  long long krow = 0;
  if (valid) {
    if (POOL) {
      krow = (((long long)b * a.P + lk) * a.Hkv + hk) * D + part * DPT;
    } else {
      krow = (((long long)b * a.N + n_row) * a.Hkv + hk) * D + part * DPT;
    }
    for (int c = 0; c < DPT; ++c) {
      kr[c] = ld1<BF16>(POOL ? a.kp : a.k, krow + c);
      vr[c] = ld1<BF16>(POOL ? a.vp : a.v, krow + c);
    }
  } else {
    for (int c = 0; c < DPT; ++c) kr[c] = vr[c] = 0.f;
  }
  for (int c = 0; c < DPT; ++c) dk[c] = dv[c] = 0.f;
  // Query sets: 0, the image queries that see these keys (the window's, or
  // every one for pooled / text keys); 1 (joint), the L text queries.
  for (int set = 0; set < (a.joint ? 2 : 1); ++set)
  for (int h = hk * group; h < (hk + 1) * group; ++h) {
    const long long nqry = set ? (long long)a.P : (POOL ? a.N : a.m);
    for (long long q0 = 0; q0 < nqry; q0 += kChunk) {
      const int nq = nqry - q0 < kChunk ? (int)(nqry - q0) : kChunk;
      __syncthreads();
      for (int idx = threadIdx.x; idx < nq * D; idx += kBwdThreads) {
        const int ii = idx / D, c = idx % D;
        if (set) {  // text query q0 + ii
          const long long n = q0 + ii;
          const long long off = (((long long)b * a.P + n) * a.H + h) * D + c;
          qs[ii][c] = ld1<BF16>(a.qt, off);
          gs[ii][c] = ld1<BF16>(a.dout_t, off);
          if (c == 0) {
            ls[ii] = a.lse_t[((long long)b * a.H + h) * a.P + n];
            ds_[ii] = a.dD_t[((long long)b * a.H + h) * a.P + n];
          }
          continue;
        }
        const long long n = POOL ? q0 + ii : member(a, jt, jh, jw, (int)(q0 + ii));
        if (n < 0) {  // padding: no query (weight exp(s - inf) = 0)
          qs[ii][c] = gs[ii][c] = 0.f;
          if (c == 0) {
            ls[ii] = INFINITY;
            ds_[ii] = 0.f;
          }
          continue;
        }
        const long long off = (((long long)b * a.N + n) * a.H + h) * D + c;
        qs[ii][c] = ld1<BF16>(a.q, off);
        gs[ii][c] = ld1<BF16>(a.dout, off);
        if (c == 0) {
          ls[ii] = a.lse[((long long)b * a.H + h) * a.N + n];
          ds_[ii] = a.dD[((long long)b * a.H + h) * a.N + n];
        }
      }
      __syncthreads();
      for (int ii = 0; ii < nq; ++ii) {
        float s = 0.f, dp = 0.f;
        for (int c = 0; c < DPT; ++c) {
          s = fmaf(qs[ii][part * DPT + c], kr[c], s);
          dp = fmaf(gs[ii][part * DPT + c], vr[c], dp);
        }
        s = lane_sum<TPQ>(s);
        dp = lane_sum<TPQ>(dp);
        const float pw = expf(s * a.scale - ls[ii]);
        const float dsv = pw * (dp - ds_[ii]);
        for (int c = 0; c < DPT; ++c) {
          dk[c] = fmaf(dsv, qs[ii][part * DPT + c], dk[c]);
          dv[c] = fmaf(pw, gs[ii][part * DPT + c], dv[c]);
        }
      }
    }
  }
  if (!valid) return;
  if (POOL && a.joint) {  // text keys: their final gradients
    for (int c = 0; c < DPT; ++c) {
      st1<BF16>(a.dkt, krow + c, dk[c] * a.scale);
      st1<BF16>(a.dvt, krow + c, dv[c]);
    }
    return;
  }
  if (POOL) {
    for (int c = 0; c < DPT; ++c) {
      a.dkp[krow + c] = dk[c];
      a.dvp[krow + c] = dv[c];
    }
    return;
  }
  if (a.P && !a.joint) {  // this token's share of its cell's pooled gradient
    const long long hw = (long long)a.Hg * a.Wg;
    const long long t = n_row / hw, y = (n_row / a.Wg) % a.Hg, x = n_row % a.Wg;
    const long long cell = ((t / a.pt) * (a.Hg / a.ph) + y / a.ph) * (a.Wg / a.pw) + x / a.pw;
    const long long po = (((long long)b * a.P + cell) * a.Hkv + hk) * D + part * DPT;
    for (int c = 0; c < DPT; ++c) {
      dk[c] = fmaf(a.inv_count, a.dkp[po + c], dk[c]);
      dv[c] = fmaf(a.inv_count, a.dvp[po + c], dv[c]);
    }
  }
  for (int c = 0; c < DPT; ++c) {
    st1<BF16>(a.dk, krow + c, dk[c] * a.scale);
    st1<BF16>(a.dv, krow + c, dv[c]);
  }
}

template <bool BF16, int D>
basa_status launch_bwd_typed(BwdArgs& a, const Dims& d, bool prep_only, cudaStream_t stream) {
  const long long rows = (long long)d.B * d.N * d.H;
  const long long nwin = (long long)d.nwt * d.nwh * d.nww;
  constexpr int per = kBwdThreads / (D / 32);  // queries (keys) per CTA
  a.n_chunks = (a.m + per - 1) / per;
  const long long dq_blocks = (long long)d.B * d.H * nwin * a.n_chunks;
  const long long dkv_blocks = (long long)d.B * d.Hkv * nwin * a.n_chunks;
  constexpr int rows_per_block =
      (kBwdThreads / 32) * (32 / (D * (BF16 ? 2 : 4) / 16)) * kPrepGroups;
  const long long prep_blocks = (rows + rows_per_block - 1) / rows_per_block;
  if (prep_blocks > 0x7fffffffLL || dq_blocks > 0x7fffffffLL) return BASA_ERR_UNSUPPORTED;
  bwd_prep_kernel<BF16, D><<<(unsigned)prep_blocks, kBwdThreads, 0, stream>>>(a);
  if (prep_only) return cudaGetLastError() == cudaSuccess ? BASA_OK : BASA_ERR_CUDA;
  if (a.joint) {  // D of the text rows: the prep kernel over [B, L, H] rows
    BwdArgs t = a;
    t.o = t.joint_out;
    t.dout = a.dout_t;
    t.dD = const_cast<float*>(a.dD_t);
    t.N = a.P;
    const long long trows = (long long)d.B * a.P * d.H;
    bwd_prep_kernel<BF16, D><<<(unsigned)((trows + rows_per_block - 1) / rows_per_block),
                               kBwdThreads, 0, stream>>>(t);
  }
  if (a.P) {  // the extra keys' gradients first: the window dK, dV add a pooled share
    a.p_chunks = (int)((a.P + per - 1) / per);
    const long long pool_blocks = (long long)d.B * d.Hkv * a.p_chunks;
    if (pool_blocks > 0x7fffffffLL) return BASA_ERR_UNSUPPORTED;
    bwd_dkv_kernel<BF16, D, true><<<(unsigned)pool_blocks, kBwdThreads, 0, stream>>>(a);
  }
  bwd_dq_kernel<BF16, D, false><<<(unsigned)dq_blocks, kBwdThreads, 0, stream>>>(a);
  if (a.joint) {  // the text queries' dq
    a.t_chunks = (int)((a.P + per - 1) / per);
    const long long tq_blocks = (long long)d.B * d.H * a.t_chunks;
    if (tq_blocks > 0x7fffffffLL) return BASA_ERR_UNSUPPORTED;
    bwd_dq_kernel<BF16, D, true><<<(unsigned)tq_blocks, kBwdThreads, 0, stream>>>(a);
  }
  bwd_dkv_kernel<BF16, D, false><<<(unsigned)dkv_blocks, kBwdThreads, 0, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? BASA_OK : BASA_ERR_CUDA;
}

basa_status launch_bwd_common(const Dims& d, const void* q, const void* k, const void* v,
                              const void* o, const void* dout, const float* lse, float* dD,
                              void* dq, void* dk, void* dv, const PoolGrads* pg, bool prep_only,
                              cudaStream_t stream, const JointGrads* jg = nullptr) {
  BwdArgs a;
  a.joint = 0;
  a.qt = a.dout_t = a.joint_out = nullptr;
  a.lse_t = a.dD_t = nullptr;
  a.dqt = a.dkt = a.dvt = nullptr;
  a.t_chunks = 0;
  a.kp = a.vp = nullptr;
  a.dkp = a.dvp = nullptr;
  a.P = 0;
  a.pt = a.ph = a.pw = 1;
  a.p_chunks = 0;
  a.inv_count = 1.0f;
  if (pg && d.P > 0) {
    a.kp = pg->kp; a.vp = pg->vp; a.dkp = pg->dkp; a.dvp = pg->dvp;
    a.P = d.P;
    a.pt = d.pt; a.ph = d.ph; a.pw = d.pw;
    a.inv_count = 1.0f / (float)(d.pt * d.ph * d.pw);
  }
  if (jg && jg->L > 0) {  // the text tokens are the extra keys; text queries see every token
    a.joint = 1;
    a.kp = jg->kt; a.vp = jg->vt;
    a.P = jg->L;
    a.qt = jg->qt; a.dout_t = jg->dout_t; a.joint_out = jg->out_t;
    a.lse_t = jg->lse_t; a.dD_t = jg->dD_t;
    a.dqt = jg->dqt; a.dkt = jg->dkt; a.dvt = jg->dvt;
  }
  a.q = q; a.k = k; a.v = v; a.o = o; a.dout = dout; a.lse = lse; a.dD = dD;
  a.dq = dq; a.dk = dk; a.dv = dv;
  a.B = d.B; a.H = d.H; a.Hkv = d.Hkv; a.T = d.T; a.Hg = d.Hg; a.Wg = d.Wg;
  a.wt = d.wt; a.wh = d.wh; a.ww = d.ww;
  a.st = d.st; a.sh = d.sh; a.sw = d.sw;
  a.nwt = d.nwt; a.nwh = d.nwh; a.nww = d.nww;
  a.Tp = d.Tp > 0 ? d.Tp : d.T;
  a.Hgp = d.Hgp > 0 ? d.Hgp : d.Hg;
  a.Wgp = d.Wgp > 0 ? d.Wgp : d.Wg;
  const long long m = (long long)d.wt * d.wh * d.ww;
  if (m > (1LL << 30)) return BASA_ERR_UNSUPPORTED;
  a.m = (int)m;
  a.N = d.N;
  a.scale = d.scale;
  const bool bf = d.dtype == BASA_BF16;
  switch (d.d) {
    case 32: return bf ? launch_bwd_typed<true, 32>(a, d, prep_only, stream) : launch_bwd_typed<false, 32>(a, d, prep_only, stream);
    case 64: return bf ? launch_bwd_typed<true, 64>(a, d, prep_only, stream) : launch_bwd_typed<false, 64>(a, d, prep_only, stream);
    case 128: return bf ? launch_bwd_typed<true, 128>(a, d, prep_only, stream) : launch_bwd_typed<false, 128>(a, d, prep_only, stream);
    default: return BASA_ERR_UNSUPPORTED;
  }
}

}  // namespace

basa_status launch_bwd(const Dims& d, const void* q, const void* k, const void* v,
                       const void* o, const void* dout, const float* lse, float* dD, void* dq,
                       void* dk, void* dv, const PoolGrads* pg, cudaStream_t stream) {
  return launch_bwd_common(d, q, k, v, o, dout, lse, dD, dq, dk, dv, pg, false, stream);
}

basa_status launch_bwd_joint(const Dims& d, const void* q, const void* k, const void* v,
                             const void* o, const void* dout, const float* lse, float* dD,
                             void* dq, void* dk, void* dv, const JointGrads& jg,
                             cudaStream_t stream) {
  return launch_bwd_common(d, q, k, v, o, dout, lse, dD, dq, dk, dv, nullptr, false, stream, &jg);
}

basa_status launch_bwd_prep(const Dims& d, const void* o, const void* dout, float* dD,
                            cudaStream_t stream) {
  return launch_bwd_common(d, nullptr, nullptr, nullptr, o, dout, nullptr, dD, nullptr, nullptr,
                           nullptr, nullptr, true, stream);
}

}  // namespace basa
