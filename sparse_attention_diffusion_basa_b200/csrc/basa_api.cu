// C ABI entry points: validation, shift normalisation, the bf16 window tile plan
// (shifted-window index math), TMA map encoding and dispatch to the kernels.
#include <math.h>
#include <string.h>

#include <mutex>

#include "basa_internal.h"

namespace basa {

static int floor_mod(long long a, int n) {
  long long r = a % n;
  return (int)(r < 0 ? r + n : r);
}

basa_status normalise(const basa_params* p, bool full, Dims* d, bool allow_fp8) {
  if (!p || !d) return BASA_ERR_INVALID_ARG;
  if (p->B < 0 || p->H < 0 || p->T < 0 || p->Hg < 0 || p->Wg < 0 || p->d <= 0)
    return BASA_ERR_INVALID_ARG;
  if (p->dtype != BASA_F32 && p->dtype != BASA_BF16 && p->dtype != BASA_FP8_E4M3)
    return BASA_ERR_INVALID_ARG;
  if (p->dtype == BASA_FP8_E4M3) {
    if (!allow_fp8 || p->d != 128) return BASA_ERR_UNSUPPORTED;
    if (p->pt != 0 || p->ph != 0 || p->pw != 0) return BASA_ERR_UNSUPPORTED;
  }
  const float dq = p->q_descale, dk = p->k_descale, dv = p->v_descale;
  if (!(dq >= 0.0f) || !(dk >= 0.0f) || !(dv >= 0.0f) || isinf(dq) || isinf(dk) || isinf(dv))
    return BASA_ERR_INVALID_ARG;
  if (!(p->scale >= 0.0f) || isinf(p->scale)) return BASA_ERR_INVALID_ARG;
  memset(d, 0, sizeof(*d));
  d->B = p->B; d->H = p->H; d->T = p->T; d->Hg = p->Hg; d->Wg = p->Wg; d->d = p->d;
  if (p->Hkv < 0 || (p->Hkv > 0 && p->H % p->Hkv != 0)) return BASA_ERR_INVALID_ARG;
  d->Hkv = p->Hkv > 0 ? p->Hkv : p->H;
  d->dtype = p->dtype;
  d->qk_descale = 1.0f;
  d->v_descale = 1.0f;
  if (p->dtype == BASA_FP8_E4M3) {
    d->qk_descale = (dq > 0.0f ? dq : 1.0f) * (dk > 0.0f ? dk : 1.0f);
    d->v_descale = dv > 0.0f ? dv : 1.0f;
  }
  d->N = (long long)p->T * p->Hg * p->Wg;
  d->Nq = d->N;
  d->scale = p->scale > 0.0f ? p->scale : 1.0f / sqrtf((float)p->d);
  if (p->dtype == BASA_F32) {
    if (p->d != 32 && p->d != 64 && p->d != 128) return BASA_ERR_UNSUPPORTED;
  } else if (p->dtype == BASA_BF16) {
    if (p->d != 64 && p->d != 128) return BASA_ERR_UNSUPPORTED;
  }
  if ((long long)p->B * p->H * d->N == 0) return BASA_OK;  // empty: valid no-op
  if (d->N > (1LL << 30) || (long long)p->B * p->T > (1LL << 30)) return BASA_ERR_UNSUPPORTED;
  if (full) {
    d->wt = p->T; d->wh = p->Hg; d->ww = p->Wg;
    d->st = d->sh = d->sw = 0;
    d->pt = d->ph = d->pw = 0;
  } else {
    if (p->wt <= 0 || p->wh <= 0 || p->ww <= 0) return BASA_ERR_INVALID_ARG;
    const bool pad = (p->flags & BASA_FLAG_PAD_GRID) != 0;
    if (!pad && (p->T % p->wt || p->Hg % p->wh || p->Wg % p->ww)) return BASA_ERR_SHAPE;
    if (p->wt > (1 << 20) || p->wh > (1 << 20) || p->ww > (1 << 20)) return BASA_ERR_UNSUPPORTED;
    d->wt = p->wt; d->wh = p->wh; d->ww = p->ww;
    d->st = floor_mod(p->st, p->wt);
    d->sh = floor_mod(p->sh, p->wh);
    d->sw = floor_mod(p->sw, p->ww);
    const bool none = p->pt == 0 && p->ph == 0 && p->pw == 0;
    if (!none) {
      if (p->pt <= 0 || p->ph <= 0 || p->pw <= 0) return BASA_ERR_INVALID_ARG;
      if (p->T % p->pt || p->Hg % p->ph || p->Wg % p->pw) return BASA_ERR_SHAPE;
      d->pt = p->pt; d->ph = p->ph; d->pw = p->pw;
      d->P = (long long)(p->T / p->pt) * (p->Hg / p->ph) * (p->Wg / p->pw);
    }
  }
  // windows per (padded) axis: ceil(G / w); the grid itself when w divides G
  d->nwt = (d->T + d->wt - 1) / d->wt;
  d->nwh = (d->Hg + d->wh - 1) / d->wh;
  d->nww = (d->Wg + d->ww - 1) / d->ww;
  d->Tp = d->nwt * d->wt; d->Hgp = d->nwh * d->wh; d->Wgp = d->nww * d->ww;
  d->padded = (d->Tp != d->T || d->Hgp != d->Hg || d->Wgp != d->Wg) ? 1 : 0;
  if ((long long)d->Tp * d->Hgp * d->Wgp > (1LL << 30) ||
      (long long)d->nwt * d->nwh * d->nww > (1LL << 30))
    return BASA_ERR_UNSUPPORTED;
  return BASA_OK;
}

// ---------------------------------------------------------------------------
// Tile plan: local boxes of whole window rows, split where the window wraps.
// ---------------------------------------------------------------------------
namespace {
struct Seg { int l0, n; };
int split(int l0, int n, int cut, Seg* out) {
  if (l0 < cut && cut < l0 + n) {
    out[0] = {l0, cut - l0};
    out[1] = {cut, l0 + n - cut};
    return 2;
  }
  out[0] = {l0, n};
  return 1;
}
}  // namespace

basa_status build_tile_plan(const Dims& d, TilePlan* plan) {
  memset(plan, 0, sizeof(*plan));
  if (d.ww > 128 || d.wh > 255 || d.wt > 255) return BASA_ERR_UNSUPPORTED;
  const int R = 128 / d.ww;  // window rows per tile, at most
  struct LocalTile { int t0, h0, bt, bh; } tiles[kMaxTiles];
  int nt = 0;
  for (int h0 = 0; h0 < d.wh; h0 += R) {
    const int c = d.wh - h0 < R ? d.wh - h0 : R;
    int g = 128 / (d.ww * c);
    if (g < 1) g = 1;
    for (int t0 = 0; t0 < d.wt; t0 += g) {
      if (nt >= kMaxTiles) return BASA_ERR_UNSUPPORTED;
      const int bt = d.wt - t0 < g ? d.wt - t0 : g;
      tiles[nt++] = {t0, h0, bt, c};
    }
  }
  plan->n_tiles = nt;
  for (int cls = 0; cls < kClasses; ++cls) {
    for (int ti = 0; ti < nt; ++ti) {
      const LocalTile& L = tiles[ti];
      Seg st[2], sh[2], sw[2];
      const int nst = (cls & 1) ? split(L.t0, L.bt, d.wt - d.st, st) : (st[0] = {L.t0, L.bt}, 1);
      const int nsh = (cls & 2) ? split(L.h0, L.bh, d.wh - d.sh, sh) : (sh[0] = {L.h0, L.bh}, 1);
      const int nsw = (cls & 4) ? split(0, d.ww, d.ww - d.sw, sw) : (sw[0] = {0, d.ww}, 1);
      int row = 0, nb = 0;
      for (int a = 0; a < nst; ++a)
        for (int b = 0; b < nsh; ++b)
          for (int c = 0; c < nsw; ++c) {
            const int rows = st[a].n * sh[b].n * sw[c].n;
            if (rows % 8 != 0) return BASA_ERR_UNSUPPORTED;
            int id = -1;
            for (int s = 0; s < plan->n_shapes; ++s)
              if (plan->shape_bt[s] == st[a].n && plan->shape_bh[s] == sh[b].n &&
                  plan->shape_bw[s] == sw[c].n)
                id = s;
            if (id < 0) {
              if (plan->n_shapes >= kMaxShapes) return BASA_ERR_UNSUPPORTED;
              id = plan->n_shapes++;
              plan->shape_bt[id] = (uint8_t)st[a].n;
              plan->shape_bh[id] = (uint8_t)sh[b].n;
              plan->shape_bw[id] = (uint8_t)sw[c].n;
            }
            plan->box[cls][ti][nb++] = box_pack(st[a].l0, sh[b].l0, sw[c].l0, id, row / 8);
            row += rows;
          }
      plan->nbox[cls][ti] = (uint8_t)nb;
      if (cls == 0) plan->tile_rows[ti] = (uint8_t)row;
    }
  }
  return BASA_OK;
}

// ---------------------------------------------------------------------------
// TMA map encoding through the driver entry point (no link against libcuda).
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

basa_status encode_map(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                       const uint64_t* strides_bytes, const uint32_t* box,
                       CUtensorMapDataType type) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return BASA_ERR_CUDA;
  cuuint64_t gd[5], gs[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
  CUresult r = fn(map, type, (cuuint32_t)rank, const_cast<void*>(base),
                  gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? BASA_OK : BASA_ERR_CUDA;
}

}  // namespace basa

using namespace basa;

static bool misaligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

static size_t pooled_bytes(const Dims& d) {
  const size_t es = d.dtype == BASA_BF16 ? 2 : 4;
  return align256((size_t)d.B * (size_t)d.P * (size_t)d.Hkv * (size_t)d.d * es);
}

extern "C" {

const char* basa_status_string(basa_status s) {
  switch (s) {
    case BASA_OK: return "ok";
    case BASA_ERR_INVALID_ARG: return "invalid argument";
    case BASA_ERR_SHAPE: return "window or pool cell does not divide the grid";
    case BASA_ERR_UNSUPPORTED: return "unsupported size for this dtype";
    case BASA_ERR_ALIGN: return "pointer not 16-byte aligned";
    case BASA_ERR_WORKSPACE: return "workspace missing";
    case BASA_ERR_CUDA: return "CUDA error";
    case BASA_ERR_TIMEOUT: return "device wait timed out";
    case BASA_ERR_SCRATCH_LIMIT: return "pooled K/V exceed the fixed no-alloc scratch";
    case BASA_ERR_CHECK: return "a checked kernel found an access outside its tensor";
  }
  return "unknown status";
}

int basa_version(void) { return 200; }

size_t basa_workspace_size(const basa_params* p) {
  Dims d;
  if (normalise(p, false, &d, true) != BASA_OK || d.P == 0) return 0;
  return 2 * pooled_bytes(d);
}

basa_status basa_pool_kv(const void* k, const void* v, void* kp, void* vp, const basa_params* p,
                         cudaStream_t stream) {
  NvtxRange nvtx("basa_pool_kv");
  Dims d;
  basa_status s = normalise(p, false, &d);
  if (s != BASA_OK) return s;
  if ((long long)d.B * d.H * d.N == 0) return BASA_OK;
  if (d.P == 0) return BASA_ERR_INVALID_ARG;
  if (!k || !v || !kp || !vp) return BASA_ERR_INVALID_ARG;
  if (misaligned(k) || misaligned(v) || misaligned(kp) || misaligned(vp)) return BASA_ERR_ALIGN;
  return launch_pool(d, k, v, kp, vp, stream);
}

static basa_status attn_common(const Dims& d, const void* q, const void* k, const void* v,
                               const void* kp, const void* vp, void* out, float* lse,
                               const basa_params* p, cudaStream_t stream, bool flat,
                               bool after_pool = false) {
  if (d.dtype == BASA_F32)
    return launch_simt(d, q, k, v, kp, vp, out, lse, stream);
  return launch_tc(d, flat, q, k, v, kp, vp, out, lse, p->flags, p->wait_timeout_ms, stream,
                   nullptr, after_pool);
}

static basa_status check_qkvo(const void* q, const void* k, const void* v, const void* out,
                              const float* lse) {
  if (!q || !k || !v || !out) return BASA_ERR_INVALID_ARG;
  if (misaligned(q) || misaligned(k) || misaligned(v) || misaligned(out) ||
      (lse && misaligned(lse)))
    return BASA_ERR_ALIGN;
  return BASA_OK;
}

basa_status basa_window_attn(const void* q, const void* k, const void* v, void* out, float* lse,
                             void* workspace, const basa_params* p, cudaStream_t stream) {
  NvtxRange nvtx("basa_window_attn");
  Dims d;
  basa_status s = normalise(p, false, &d, true);
  if (s != BASA_OK) return s;
  if ((long long)d.B * d.H * d.N == 0) return BASA_OK;
  if ((s = check_qkvo(q, k, v, out, lse)) != BASA_OK) return s;
  const void* kp = nullptr;
  const void* vp = nullptr;
  if (d.P > 0) {
    if (!workspace) return BASA_ERR_WORKSPACE;
    if (misaligned(workspace)) return BASA_ERR_ALIGN;
    char* ws = static_cast<char*>(workspace);
    void* kpw = ws;
    void* vpw = ws + pooled_bytes(d);
    if (d.dtype == BASA_BF16) {  // check the attention plan before launching anything
      TilePlan plan;
      if ((s = build_tile_plan(d, &plan)) != BASA_OK) return s;
    }
    if ((s = launch_pool(d, k, v, kpw, vpw, stream)) != BASA_OK) return s;
    kp = kpw;
    vp = vpw;
  }
  return attn_common(d, q, k, v, kp, vp, out, lse, p, stream, false, d.P > 0);
}

basa_status basa_window_attn_gm(const void* q, const void* k, const void* v, const void* kp,
                                const void* vp, void* out, float* lse, const basa_params* p,
                                cudaStream_t stream) {
  NvtxRange nvtx("basa_window_attn_gm");
  Dims d;
  basa_status s = normalise(p, false, &d);
  if (s != BASA_OK) return s;
  if ((long long)d.B * d.H * d.N == 0) return BASA_OK;
  if (d.P == 0) return BASA_ERR_INVALID_ARG;
  if ((s = check_qkvo(q, k, v, out, lse)) != BASA_OK) return s;
  if (!kp || !vp) return BASA_ERR_INVALID_ARG;
  if (misaligned(kp) || misaligned(vp)) return BASA_ERR_ALIGN;
  return attn_common(d, q, k, v, kp, vp, out, lse, p, stream, false);
}

// The text-query pass of a joint call: full attention of the L text queries
// over the N image and L text keys.
static basa_status joint_text_dims(const basa_params* p, int64_t L, Dims* dt) {
  basa_status s = normalise(p, true, dt);
  if (s != BASA_OK) return s;
  dt->P = L;
  dt->Nq = L;
  dt->qsep = 1;
  return BASA_OK;
}

size_t basa_joint_workspace_size(const basa_params* p, int64_t L) {
  Dims dt;
  if (L <= 0 || L > (1LL << 24) || joint_text_dims(p, L, &dt) != BASA_OK) return 0;
  if (dt.dtype != BASA_BF16 || (long long)dt.B * dt.H * dt.N == 0) return 0;
  return flat_split_bytes(dt, flat_split_count(dt, true));
}

basa_status basa_joint_attn(const void* q, const void* k, const void* v, const void* qt,
                            const void* kt, const void* vt, int64_t L, void* out, void* out_t,
                            float* lse, float* lse_t, void* workspace, const basa_params* p,
                            cudaStream_t stream) {
  NvtxRange nvtx("basa_joint_attn");
  Dims d;
  basa_status s = normalise(p, false, &d);
  if (s != BASA_OK) return s;
  if (d.pt || d.ph || d.pw) return BASA_ERR_UNSUPPORTED;  // text takes the global-memory slot
  if (L < 0) return BASA_ERR_INVALID_ARG;
  if (L > (1LL << 24)) return BASA_ERR_UNSUPPORTED;
  if ((long long)d.B * d.H * d.N == 0) return BASA_OK;
  if ((s = check_qkvo(q, k, v, out, lse)) != BASA_OK) return s;
  if (L == 0) return attn_common(d, q, k, v, nullptr, nullptr, out, lse, p, stream, false);
  if ((s = check_qkvo(qt, kt, vt, out_t, lse_t)) != BASA_OK) return s;
  // the text-query pass is validated before the image pass is launched
  Dims dt;
  if ((s = joint_text_dims(p, L, &dt)) != BASA_OK) return s;
  SplitK sk{1, nullptr, nullptr};
  if (d.dtype == BASA_BF16) {
    TilePlan plan;
    if ((s = build_tile_plan(d, &plan)) != BASA_OK) return s;
    const int n = workspace ? flat_split_count(dt, true) : 1;
    if (n > 1) {
      if (misaligned(workspace)) return BASA_ERR_ALIGN;
      const size_t o = align256((size_t)n * dt.B * dt.H * dt.Nq * dt.d * sizeof(float));
      sk.n = n;
      sk.part_o = static_cast<float*>(workspace);
      sk.part_ml = reinterpret_cast<float*>(static_cast<char*>(workspace) + o);
    }
  }
  // image queries: their window plus every text token
  d.P = L;
  if ((s = attn_common(d, q, k, v, kt, vt, out, lse, p, stream, false)) != BASA_OK) return s;
  // text queries: every image token plus every text token
  if (d.dtype == BASA_BF16)
    return launch_tc(dt, true, qt, k, v, kt, vt, out_t, lse_t, p->flags, p->wait_timeout_ms,
                     stream, &sk);
  return attn_common(dt, qt, k, v, kt, vt, out_t, lse_t, p, stream, true);
}

// Backward workspace: D = rowsum(dO * O) (fp32 [B, H, N]); with pooled memory
// also the pooled K, V (input dtype) and their gradients (fp32), [B, P, Hkv, d].
static size_t bwd_pooled_bytes(const Dims& d, size_t esize) {
  return align256((size_t)d.B * (size_t)d.P * (size_t)d.Hkv * (size_t)d.d * esize);
}

size_t basa_bwd_workspace_size(const basa_params* p) {
  Dims d;
  if (normalise(p, false, &d) != BASA_OK) return 0;
  size_t n = align256((size_t)d.B * (size_t)d.H * (size_t)d.N * sizeof(float));
  if (d.P) n += 2 * bwd_pooled_bytes(d, d.dtype == BASA_BF16 ? 2 : 4) + 2 * bwd_pooled_bytes(d, 4);
  return n;
}

basa_status basa_window_attn_bwd(const void* q, const void* k, const void* v, const void* out,
                                 const void* dout, const float* lse, void* dq, void* dk,
                                 void* dv, void* workspace, const basa_params* p,
                                 cudaStream_t stream) {
  NvtxRange nvtx("basa_window_attn_bwd");
  Dims d;
  basa_status s = normalise(p, false, &d);
  if (s != BASA_OK) return s;
  if ((long long)d.B * d.H * d.N == 0) return BASA_OK;
  if ((s = check_qkvo(q, k, v, out, lse)) != BASA_OK) return s;
  if ((s = check_qkvo(dout, dq, dk, dv, nullptr)) != BASA_OK) return s;
  if (!lse) return BASA_ERR_INVALID_ARG;
  if (!workspace) return BASA_ERR_WORKSPACE;
  if (misaligned(workspace)) return BASA_ERR_ALIGN;
  float* dD = static_cast<float*>(workspace);
  PoolGrads pg{nullptr, nullptr, nullptr, nullptr};
  if (d.P) {  // the pooled K, V the forward used, recomputed into the workspace
    char* w = static_cast<char*>(workspace) + align256((size_t)d.B * d.H * d.N * sizeof(float));
    const size_t pb = bwd_pooled_bytes(d, d.dtype == BASA_BF16 ? 2 : 4), pf = bwd_pooled_bytes(d, 4);
    void* kp = w;
    void* vp = w + pb;
    pg = PoolGrads{kp, vp, reinterpret_cast<float*>(w + 2 * pb),
                   reinterpret_cast<float*>(w + 2 * pb + pf)};
    if ((s = launch_pool(d, k, v, kp, vp, stream)) != BASA_OK) return s;
  }
  const PoolGrads* pgp = d.P ? &pg : nullptr;
  if (!(p->flags & BASA_FLAG_BWD_CUDA_CORES) && d.dtype == BASA_BF16 && (d.d == 64 || d.d == 128)) {
    s = launch_bwd_tc(d, q, k, v, out, dout, lse, dD, dq, dk, dv, pgp, p->wait_timeout_ms, stream);
    if (s != BASA_ERR_UNSUPPORTED) return s;  // outside the tensor-core path: CUDA cores
  }
  return launch_bwd(d, q, k, v, out, dout, lse, dD, dq, dk, dv, pgp, stream);
}

// D of the image rows, D of the text rows, and the text keys' fp32 dK, dV sums.
static size_t joint_bwd_parts(const Dims& d, int64_t L, size_t* off_dt, size_t* off_kp,
                              size_t* off_vp) {
  const size_t dd = align256((size_t)d.B * d.H * d.N * sizeof(float));
  const size_t dt = align256((size_t)d.B * d.H * (size_t)L * sizeof(float));
  const size_t kp = align256((size_t)d.B * (size_t)L * d.Hkv * d.d * sizeof(float));
  if (off_dt) *off_dt = dd;
  if (off_kp) *off_kp = dd + dt;
  if (off_vp) *off_vp = dd + dt + kp;
  return dd + dt + 2 * kp;
}

size_t basa_joint_bwd_workspace_size(const basa_params* p, int64_t L) {
  Dims d;
  if (L < 0 || L > (1LL << 24) || normalise(p, false, &d) != BASA_OK) return 0;
  return joint_bwd_parts(d, L, nullptr, nullptr, nullptr);
}

basa_status basa_joint_attn_bwd(const void* q, const void* k, const void* v, const void* qt,
                                const void* kt, const void* vt, int64_t L, const void* out,
                                const void* out_t, const void* dout, const void* dout_t,
                                const float* lse, const float* lse_t, void* dq, void* dk, void* dv,
                                void* dqt, void* dkt, void* dvt, void* workspace,
                                const basa_params* p, cudaStream_t stream) {
  NvtxRange nvtx("basa_joint_attn_bwd");
  Dims d;
  basa_status s = normalise(p, false, &d);
  if (s != BASA_OK) return s;
  if (d.pt || d.ph || d.pw) return BASA_ERR_UNSUPPORTED;  // text takes the global-memory slot
  if (L < 0) return BASA_ERR_INVALID_ARG;
  if (L > (1LL << 24)) return BASA_ERR_UNSUPPORTED;
  if ((long long)d.B * d.H * d.N == 0) return BASA_OK;
  if (L == 0)
    return basa_window_attn_bwd(q, k, v, out, dout, lse, dq, dk, dv, workspace, p, stream);
  if ((s = check_qkvo(q, k, v, out, lse)) != BASA_OK) return s;
  if ((s = check_qkvo(dout, dq, dk, dv, nullptr)) != BASA_OK) return s;
  if ((s = check_qkvo(qt, kt, vt, out_t, lse_t)) != BASA_OK) return s;
  if ((s = check_qkvo(dout_t, dqt, dkt, dvt, nullptr)) != BASA_OK) return s;
  if (!lse || !lse_t) return BASA_ERR_INVALID_ARG;
  if (!workspace) return BASA_ERR_WORKSPACE;
  if (misaligned(workspace)) return BASA_ERR_ALIGN;
  size_t off_dt, off_kp, off_vp;
  joint_bwd_parts(d, L, &off_dt, &off_kp, &off_vp);
  char* ws = static_cast<char*>(workspace);
  float* dD = reinterpret_cast<float*>(ws);
  float* dD_t = reinterpret_cast<float*>(ws + off_dt);
  const JointGrads jg{qt, kt, vt, out_t, dout_t, lse_t, dD_t, dqt, dkt, dvt, (long long)L};
  if (d.dtype == BASA_BF16 && !(p->flags & BASA_FLAG_BWD_CUDA_CORES)) {
    s = launch_bwd_tc_joint(d, q, k, v, out, dout, lse, dD, dq, dk, dv, jg,
                            reinterpret_cast<float*>(ws + off_kp),
                            reinterpret_cast<float*>(ws + off_vp), p->wait_timeout_ms, stream);
    if (s != BASA_ERR_UNSUPPORTED) return s;
  }
  return launch_bwd_joint(d, q, k, v, out, dout, lse, dD, dq, dk, dv, jg, stream);
}

basa_status basa_full_attn(const void* q, const void* k, const void* v, void* out, float* lse,
                           const basa_params* p, cudaStream_t stream) {
  NvtxRange nvtx("basa_full_attn");
  Dims d;
  basa_status s = normalise(p, true, &d, true);
  if (s != BASA_OK) return s;
  if ((long long)d.B * d.H * d.N == 0) return BASA_OK;
  if ((s = check_qkvo(q, k, v, out, lse)) != BASA_OK) return s;
  return attn_common(d, q, k, v, nullptr, nullptr, out, lse, p, stream, true);
}

basa_status basa_get_status(cudaStream_t stream) {
  return read_and_clear_status(stream);
}

basa_status basa_window_tiles(const basa_params* p, int32_t* n_windows, int32_t* n_tiles,
                              int32_t* rows, int64_t rows_capacity) {
  Dims d;
  basa_status s = normalise(p, false, &d, true);
  if (s != BASA_OK) return s;
  if (d.dtype == BASA_F32) return BASA_ERR_UNSUPPORTED;  // the tensor-core kernel's plan
  if ((long long)d.B * d.H * d.N == 0) return BASA_ERR_INVALID_ARG;
  TilePlan plan;
  if ((s = build_tile_plan(d, &plan)) != BASA_OK) return s;
  const int nwin = d.nwt * d.nwh * d.nww;
  if (n_windows) *n_windows = nwin;
  if (n_tiles) *n_tiles = plan.n_tiles;
  if (!rows) return BASA_OK;
  if (rows_capacity < (int64_t)nwin * plan.n_tiles * 128) return BASA_ERR_INVALID_ARG;
  for (int w = 0; w < nwin; ++w) {
    const int jw = w % d.nww, jh = (w / d.nww) % d.nwh, jt = w / (d.nww * d.nwh);
    const int cls = window_class(jt, jh, jw, d.nwt, d.nwh, d.nww, d.st, d.sh, d.sw);
    const int ot = jt * d.wt + d.st, oh = jh * d.wh + d.sh, ow = jw * d.ww + d.sw;
    for (int ti = 0; ti < plan.n_tiles; ++ti) {
      int32_t* r = rows + ((int64_t)w * plan.n_tiles + ti) * 128;
      for (int i = 0; i < 128; ++i) r[i] = -1;
      for (int bi = 0; bi < plan.nbox[cls][ti]; ++bi) {
        const uint32_t e = plan.box[cls][ti][bi];
        const int sid = box_shape(e);
        const int bt = plan.shape_bt[sid], bh = plan.shape_bh[sid], bw = plan.shape_bw[sid];
        const int gt = (ot + box_lt(e)) % d.Tp, gh = (oh + box_lh(e)) % d.Hgp,
                  gw = (ow + box_lw(e)) % d.Wgp;
        int row = box_row8(e) * 8;
        for (int a = 0; a < bt; ++a)
          for (int b = 0; b < bh; ++b)
            for (int c = 0; c < bw; ++c, ++row) {
              if (gt + a >= d.T || gh + b >= d.Hg || gw + c >= d.Wg) continue;  // padded
              r[row] = (int32_t)(((long long)(gt + a) * d.Hg + (gh + b)) * d.Wg + (gw + c));
            }
      }
    }
  }
  return BASA_OK;
}

}  // extern "C"
