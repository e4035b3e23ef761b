// Backward of bf16 shifted local window attention on the 5th-generation tensor
// cores (tcgen05 + TMEM + TMA) of sm_100a.
//
// The operation ("BASA: Backend-Agnostic Sparse Attention for Fast
// High-Resolution Diffusion Transformers", zhichai.net topic 178635722, "The
// BASA Method": every query attends to the keys of its own cyclically shifted
// window; the forum review of the same paper, reply 178634520, names the
// dense-teacher adaptation that trains through this attention).  With
// P = exp(scale * Q K^T - lse) over each query's window (lse from the forward
// pass) and D = rowsum(dO * O):
//   dP = dO V^T,  dS = P * (dP - D),
//   dQ = scale * dS K,  dK = scale * dS^T Q,  dV = P^T dO.
// A window key is seen only by the queries of its own window, so its gradient
// rows depend on one window alone and need no atomics.  Pooled global memory
// (the review's K/V-pooled tokens, the means of fixed cells) adds keys that
// every query of the batch sees: their gradients are summed over all queries
// (fp32 atomics) and reach each cell token divided by the cell size.
//
// One kernel template serves three modes of the same shape:
//   dQ (kModeDq): unit (b, h, window, query tile).  Fixed per unit: A0 = Q,
//       A1 = dO of the tile (and lse, D of its rows), copied from shared memory
//       into TMEM columns [384, 512) at unit start so that the slot refills a
//       whole unit ahead.  Step j over the window's key tiles, then the pooled
//       key tiles: B0 = K_j, B1 = V_j.
//   window dK, dV (kModeDkv): unit (b, K/V head, window, key tile).  Fixed per
//       unit: A0 = K, A1 = V of the tile.  Step over (query head of the group,
//       query tile): B0 = Q_i, B1 = dO_i (and lse, D of its rows).  With pooled
//       memory the epilogue adds the row's share of its cell's pooled gradient.
//   pooled dK, dV (kModePooled): unit (b, K/V head, pooled key tile, split of
//       the grid's query tiles); A0, A1 = pooled K, V; steps over flat query
//       tiles; the epilogue adds its sums into fp32 dkp, dvp with atomics.
// Per step the tensor core computes X = A0 B0^T and Y = A1 B1^T into TMEM
// (dQ: S and dP; dK, dV: S^T and dP^T).  The elementwise warps form P and dS in
// fp32 and write them back into TMEM as bf16 pairs over X (and Y), and the
// tensor core accumulates, with the bf16 operand read from TMEM,
//   dQ:  dQ += dS K_j                  (B0 read MN-major)
//   dKV: dV += P^T dO_i, dK += dS^T Q_i (B1, B0 read MN-major).
// TMEM columns: X [0, 128), Y [128, 256), accumulators from 256 (dQ: dQ, then
// Q and dO; dK, dV: dV, then dK).
//
// Persistent CTAs (one per SM, 384 threads):
//   warp 0       TMA loader of the step pairs through a two-slot ring (dKV:
//                with the lse and D of the step's queries);
//   warp 1       owns TMEM (512 columns) and issues the MMAs from one thread;
//   warp 2       TMA loader of the unit pair (dQ: with its rows' lse and D);
//   warps 4..11  two warpgroups, one per 64-column half of X and Y: the
//                elementwise stage, then the epilogue (scale, round to bf16,
//                warp-staged 16-byte stores to the window's token rows).
// Tiles, TMA boxes and the zero rows of partial tiles come from the forward's
// shifted-window tile plan.  Every mbarrier wait is bounded: on expiry the
// kernel raises its device status word, lets every role leave its loop, waits
// (bounded) for its own copies and MMAs in flight, frees TMEM and returns.
#include <cuda_bf16.h>
#include <math.h>
#include <string.h>

#include <new>

#include "basa_internal.h"
#include "tc_device.cuh"

namespace basa {
namespace {

constexpr int kBwdTcThreads = 384;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kTmemA = 384;  // dQ: TMEM columns of Q (64) and dO (64) as bf16 pairs

struct __align__(64) BwdTcParams {
  CUtensorMap qm[kMaxShapes];  // window boxes over q, rank 5: [d, H, Wg, Hg, B*T]
  CUtensorMap gm[kMaxShapes];  // the same over dout
  CUtensorMap km[kMaxShapes];  // over k: [d, Hkv, Wg, Hg, B*T]
  CUtensorMap vm[kMaxShapes];  // over v
  CUtensorMap fill;            // 8-row box over k's flat view, read out of bounds = zeros
  CUtensorMap kpf, vpf;        // pooled K, V: [d, Hkv, P, B], 128-row boxes
  CUtensorMap qf, gf;          // q and dout as flat rows: [d, H, N, B], 128-row boxes
  PlanImage plan;
  const float* lse;  // [B, H, N] natural-log log-sum-exp of the forward pass
  const float* dD;   // [B, H, N] rowsum(dout * out)
  __nv_bfloat16* dq;  // [B, N, H, d]
  __nv_bfloat16* dk;  // [B, N, Hkv, d]
  __nv_bfloat16* dv;
  unsigned long long timeout_ns;
  long long N;
  uint32_t n_units;
  int H, Hkv, group, T, Hg, Wg;
  int wt, wh, ww, st, sh, sw, nwt, nwh, nww;
  int n_windows, n_tiles, n_shapes;
  // unit decode divisors (set by the launcher): H, Hkv, n_tiles, n_windows,
  // nww, nwh, group, n_tt, n_pt, n_fsplits
  FastDiv fd_h, fd_hkv, fd_tiles, fd_windows, fd_nww, fd_nwh, fd_group, fd_tt, fd_pt, fd_fsplits;
  float scale, scale_log2;
  // pooled global memory (P = 0: none)
  float* dkp;  // [B, P, Hkv, d] fp32: sum over the batch's queries of dS^T Q (no scale)
  float* dvp;  // [B, P, Hkv, d] fp32: sum of P^T dO
  long long P;
  int n_pt;                      // pooled key tiles
  int n_fqt;                     // query tiles of the whole grid (flat rows)
  int fqt_per_split, n_fsplits;  // the pooled kernel's split of those query tiles
  int pt, ph, pw;
  float inv_count;               // 1 / (pt * ph * pw)
  long long q_elems, kv_elems;   // elements of dq and of dk, dv (checked build)
  // joint text + image (joint = 1): the L text tokens take the pooled slots
  // (kpf, vpf over kt, vt; dkp, dvp their fp32 sums; no share to the window
  // rows), their queries are n_tt more flat query tiles of the pooled and the
  // window dK, dV modes, and the text dQ mode walks every image key tile
  // (kf, vf) and then the text key tiles
  int joint;
  int n_tt;                      // text tiles (128 rows)
  long long L;
  CUtensorMap qtf, gtf;          // qt, dout_t as flat rows: [d, H, L, B]
  CUtensorMap kf, vf;            // k, v as flat rows: [d, Hkv, N, B]
  const float* lse_t;            // [B, H, L]
  const float* dD_t;             // [B, H, L]
  __nv_bfloat16* dqt;            // [B, L, H, d]
  long long qt_elems;            // elements of dqt (checked build)
};

// Kernel modes: the dQ kernel (window key tiles, then the pooled tiles), the
// window dK, dV kernel, and the pooled dK, dV kernel (a pooled key tile against
// a range of the grid's query tiles, summed into dkp, dvp).
constexpr int kModeDq = 0, kModeDkv = 1, kModePooled = 2, kModeDqText = 3;

// Shared memory: the unit pair, a two-slot ring of step pairs, 2 KB of output
// staging per epilogue warp, the per-row lse/D values of each ring slot (the dQ
// kernel keeps its unit's values in slot 0), barriers, the tile plan.
template <int D>
struct BwdSmem {
  static constexpr int kTile = (D / 64) * kHalf;
  static constexpr int a0 = 0;               // A0 | A1
  static constexpr int ring = 2 * kTile;     // slot s: B0 | B1 at ring + 2 s kTile
  static constexpr int stg = ring + 4 * kTile;
  static constexpr int rowv = stg + 8 * 2048;  // slot s: lse * log2(e) [128], D [128]
  static constexpr int bars = rowv + 2 * 1024;
  static constexpr int AFULL = 0, AEMPTY = 1, BFULL = 2, BEMPTY = 4, SFULL = 6, PFULL = 7,
                       OFULL = 8, DRAIN = 9, ATFULL = 10, ATFREE = 11, NBARS = 12;
  static constexpr int misc = bars + NBARS * 8;  // tmem slot, abort flag
  static constexpr int plan = misc + 64;
  static constexpr int bytes = plan + kPlanBytes;
  static constexpr int alloc = bytes + 1024;  // slack for 1024-byte alignment
};

enum BwdWaitSite : uint32_t {
  kBSiteLoadAEmpty = 101, kBSiteLoadBEmpty, kBSiteLoadDrainA, kBSiteLoadDrainB, kBSiteMmaAFull,
  kBSiteMmaBFull, kBSiteMmaPFull, kBSiteMmaDrain, kBSiteEwAFull, kBSiteEwBFull, kBSiteEwSFull,
  kBSiteEwOFull, kBSiteEwATFree
};

struct BwdUnit {
  WinAt w;
  int h;     // dQ: the query head; dKV: the first query head of the group
  int hk;    // the K/V head
  int tile;  // dQ: the query tile; dKV: the key tile; pooled: the pooled key tile
  int q0, nq;  // pooled: the unit's query tiles [q0, q0 + nq) of the grid
};

// Heads fastest, then the tile, the window and the batch (pooled: the K/V
// head, the pooled tile, the query-tile split, the batch).
template <int MODE>
__device__ __forceinline__ BwdUnit decode_bwd_unit(const BwdTcParams& p, uint32_t u) {
  constexpr bool KV = MODE == kModeDkv || MODE == kModePooled;
  BwdUnit U;
  if constexpr (MODE == kModeDqText) {  // (b, h, text tile): heads fastest
    const uint32_t r = p.fd_h.div(u);
    U.h = (int)(u - r * (uint32_t)p.H);
    U.hk = (int)p.fd_group.div((uint32_t)U.h);
    U.w.b = (int)p.fd_tt.div(r);
    U.tile = (int)(r - (uint32_t)U.w.b * (uint32_t)p.n_tt);
    U.w.cls = U.w.ot = U.w.oh = U.w.ow = 0;
    U.q0 = U.nq = 0;
    return U;
  }
  if constexpr (MODE == kModePooled) {
    const uint32_t r = p.fd_hkv.div(u);
    U.hk = (int)(u - r * (uint32_t)p.Hkv);
    U.h = U.hk * p.group;
    const uint32_t r2 = p.fd_pt.div(r);
    U.tile = (int)(r - r2 * (uint32_t)p.n_pt);
    U.w.b = (int)p.fd_fsplits.div(r2);
    const int sp = (int)(r2 - (uint32_t)U.w.b * (uint32_t)p.n_fsplits);
    U.w.cls = U.w.ot = U.w.oh = U.w.ow = 0;
    U.q0 = sp * p.fqt_per_split;
    const int left = p.n_fqt + (p.joint ? p.n_tt : 0) - U.q0;  // joint: image, then text tiles
    U.nq = left < p.fqt_per_split ? left : p.fqt_per_split;
    return U;
  }
  U.q0 = U.nq = 0;
  const uint32_t nh = (uint32_t)(KV ? p.Hkv : p.H);
  const uint32_t r = (KV ? p.fd_hkv : p.fd_h).div(u);
  const int head = (int)(u - r * nh);
  const uint32_t r2 = p.fd_tiles.div(r);
  U.tile = (int)(r - r2 * (uint32_t)p.n_tiles);
  const int b = (int)p.fd_windows.div(r2);
  const int win = (int)(r2 - (uint32_t)b * (uint32_t)p.n_windows);
  const uint32_t wr = p.fd_nww.div((uint32_t)win);
  const int jw = win - (int)wr * p.nww;
  const int jt = (int)p.fd_nwh.div(wr);
  const int jh = (int)wr - jt * p.nwh;
  U.w.cls = window_class(jt, jh, jw, p.nwt, p.nwh, p.nww, p.st, p.sh, p.sw);
  U.w.ot = jt * p.wt + p.st;
  U.w.oh = jh * p.wh + p.sh;
  U.w.ow = jw * p.ww + p.sw;
  U.w.b = b;
  if (KV) {
    U.hk = head;
    U.h = head * p.group;
  } else {
    U.h = head;
    U.hk = (int)p.fd_group.div((uint32_t)head);
  }
  return U;
}

// Query tiles per query head of a dK, dV unit: the window's (then, joint, the
// text tiles); pooled: the unit's range of the flat query tiles.
template <int MODE>
__device__ __forceinline__ int bwd_per_head(const BwdTcParams& p, const BwdUnit& U) {
  if constexpr (MODE == kModePooled) return U.nq;
  return p.n_tiles + (p.joint ? p.n_tt : 0);
}

// Steps of unit U: dQ, the window's key tiles then the pooled (text) tiles;
// text dQ, every image key tile then the text tiles; dKV, the group's query
// heads times the query tiles per head; pooled, the same over the unit's range.
template <int MODE>
__device__ __forceinline__ int bwd_steps(const BwdTcParams& p, const BwdUnit& U) {
  if constexpr (MODE == kModeDq) return p.n_tiles + p.n_pt;
  if constexpr (MODE == kModeDqText) return p.n_fqt + p.n_tt;
  return p.group * bwd_per_head<MODE>(p, U);
}

// lse * log2(e) and D of the 128 rows of query tile `tile` of head h into
// shared memory (dst[0..127], dst[128..255]); padding rows get +inf and 0, so
// that their probabilities and dS vanish.  Lane l handles rows l + 32 k.
__device__ __forceinline__ void write_row_values(const BwdTcParams& p, const PlanView& pv,
                                                 const WinAt& w, int tile, int h, float* dst,
                                                 int lane) {
#pragma unroll 1
  for (int k = 0; k < 4; ++k) {
    const int r = lane + 32 * k;
    const long long t = r < pv.rows[tile] ? window_row_token(pv, w, tile, r, p.T, p.Hg, p.Wg) : -1;
    float l2 = INFINITY, dd = 0.f;
    if (t >= 0) {
      const long long i = ((long long)w.b * p.H + h) * p.N + t;
      l2 = p.lse[i] * kLog2e;
      dd = p.dD[i];
    }
    dst[r] = l2;
    dst[128 + r] = dd;
  }
}

// The same for flat query tile i of the grid (rows 128 i .. 128 i + 127), or
// (text) of the text queries.
__device__ __forceinline__ void write_row_values_flat(const BwdTcParams& p, int b, int i, int h,
                                                      float* dst, int lane, bool text = false) {
  const long long nrows = text ? p.L : p.N;
  const float* lse = text ? p.lse_t : p.lse;
  const float* dD = text ? p.dD_t : p.dD;
#pragma unroll 1
  for (int k = 0; k < 4; ++k) {
    const int r = lane + 32 * k;
    const long long n = 128LL * i + r;
    float l2 = INFINITY, dd = 0.f;
    if (n < nrows) {
      const long long x = ((long long)b * p.H + h) * nrows + n;
      l2 = lse[x] * kLog2e;
      dd = dD[x];
    }
    dst[r] = l2;
    dst[128 + r] = dd;
  }
}

// Writes 64 bf16 columns (w: 32 packed pairs) of this lane's row to
// base[roff + col0 ...] (roff < 0: padding row, nothing written), through the
// warp's 2 KB staging block: each half of 32 columns is staged as 64-byte rows
// (16-byte chunks XOR-swizzled by row pair) and read back so that each store
// instruction writes 64 contiguous bytes of eight rows.
__device__ __forceinline__ void warp_store_row64(uint32_t stg, const uint32_t (&w)[32],
                                                 long long roff, __nv_bfloat16* base, int col0,
                                                 int lane, long long limit) {
#pragma unroll
  for (int ps = 0; ps < 2; ++ps) {
#pragma unroll
    for (int ch = 0; ch < 4; ++ch)
      st_shared_v4(stg + lane * 64 + ((ch ^ ((lane >> 1) & 3)) << 4), w[16 * ps + 4 * ch],
                   w[16 * ps + 4 * ch + 1], w[16 * ps + 4 * ch + 2], w[16 * ps + 4 * ch + 3]);
    __syncwarp();
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int rr = k * 8 + lane / 4, c = lane % 4;
      const uint4 val = ld_shared_v4(stg + rr * 64 + ((c ^ ((rr >> 1) & 3)) << 4));
      const long long t = __shfl_sync(0xffffffffu, roff, rr);
      if (t >= 0) {
        if (kChecked && t + col0 + ps * 32 + c * 8 + 8 > limit)
          check_failed(kCheckGradRow);
        else
          *reinterpret_cast<uint4*>(base + t + col0 + ps * 32 + c * 8) = val;
      }
    }
    __syncwarp();
  }
}

template <int D, int MODE>
__global__ void __launch_bounds__(kBwdTcThreads, 1)
    tc_bwd_kernel(const __grid_constant__ BwdTcParams p) {
  using S = BwdSmem<D>;
  constexpr int NH = D / 64;
  // dK, dV accumulators (window or pooled / text keys); else dQ (image or text queries)
  constexpr bool KV = MODE == kModeDkv || MODE == kModePooled;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + S::bars;
  auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::misc);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + S::misc + 4);
  float* rowv = reinterpret_cast<float*>(smem + S::rowv);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint64_t limit = p.timeout_ns;
  const PlanView pv = plan_to_smem(p.plan, smem + S::plan, p.n_tiles, threadIdx.x, kBwdTcThreads);
  if (threadIdx.x == 0) {
    mbar_init(BAR(S::AFULL), 33);  // lane 0's expect_tx + every lane after its row values
    // dKV: the MMA warp frees the unit pair; dQ: the elementwise threads, once
    // they have copied it into TMEM
    mbar_init(BAR(S::AEMPTY), KV ? 1 : 256);
    mbar_init(BAR(S::ATFULL), 256);  // dQ: the pair is in TMEM
    mbar_init(BAR(S::ATFREE), 1);    // dQ: the last X, Y MMAs of the unit have read it
    for (int s = 0; s < 2; ++s) {
      mbar_init(BAR(S::BFULL + s), 33);
      mbar_init(BAR(S::BEMPTY + s), 1);
    }
    mbar_init(BAR(S::SFULL), 1);
    mbar_init(BAR(S::PFULL), 256);
    mbar_init(BAR(S::OFULL), 1);
    mbar_init(BAR(S::DRAIN), 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) {
    for (int sid = 0; sid < p.n_shapes; ++sid) {
      prefetch_tmap(&p.qm[sid]); prefetch_tmap(&p.gm[sid]);
      prefetch_tmap(&p.km[sid]); prefetch_tmap(&p.vm[sid]);
    }
    prefetch_tmap(&p.fill);
    if (p.P) { prefetch_tmap(&p.kpf); prefetch_tmap(&p.vpf); }
    if (MODE == kModePooled) { prefetch_tmap(&p.qf); prefetch_tmap(&p.gf); }
    if (p.joint) { prefetch_tmap(&p.qtf); prefetch_tmap(&p.gtf); }
    if (MODE == kModeDqText) { prefetch_tmap(&p.kf); prefetch_tmap(&p.vf); }
  }

  if (warp == 0) {
    // ------------------------------------------------------------ step-pair loader
    uint32_t nb = 0, issued = 0, last_par = 0;
    bool ok = true;
    for (uint32_t u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
      const BwdUnit U = decode_bwd_unit<MODE>(p, u);
      const int n_steps = bwd_steps<MODE>(p, U);
      const int per_head = bwd_per_head<MODE>(p, U);
      for (int s = 0; s < n_steps && ok; ++s) {
        const uint32_t slot = nb & 1u, par = (nb >> 1) & 1u;
        if (!(ok = wait_warp(BAR(S::BEMPTY + slot), par ^ 1u, abort_flag, limit, kBSiteLoadBEmpty)))
          break;
        const uint32_t dst = sbase + S::ring + slot * 2 * S::kTile;
        const uint32_t bar = BAR(S::BFULL + slot);
        const int h = KV ? U.h + s / per_head : U.h;  // dKV: the step's query head
        const int tile = KV ? s % per_head : s;
        // pooled (joint): flat query tile U.q0 + tile, past the grid's tiles
        // a text tile; dKV (joint): query tiles past the window's are text tiles
        const int ftile = U.q0 + tile;
        const bool text_q = (MODE == kModePooled && ftile >= p.n_fqt) ||
                            (MODE == kModeDkv && tile >= p.n_tiles);
        const int ttile = MODE == kModePooled ? ftile - p.n_fqt : tile - p.n_tiles;
        if (lane == 0) {
          mbar_expect_tx(bar, 2 * S::kTile);
          if (text_q) {  // text query tile: Qt, dOt
#pragma unroll
            for (int hf = 0; hf < NH; ++hf) {
              tma_load_4d(dst + hf * kHalf, &p.qtf, bar, hf * 64, h, ttile * 128, U.w.b);
              tma_load_4d(dst + S::kTile + hf * kHalf, &p.gtf, bar, hf * 64, h, ttile * 128,
                          U.w.b);
            }
          } else if (MODE == kModePooled) {  // flat query tile U.q0 + tile of the grid
#pragma unroll
            for (int hf = 0; hf < NH; ++hf) {
              tma_load_4d(dst + hf * kHalf, &p.qf, bar, hf * 64, h, ftile * 128, U.w.b);
              tma_load_4d(dst + S::kTile + hf * kHalf, &p.gf, bar, hf * 64, h, ftile * 128,
                          U.w.b);
            }
          } else if (MODE == kModeDqText) {  // every image key tile, then the text tiles
            const bool img = tile < p.n_fqt;
            const int row = (img ? tile : tile - p.n_fqt) * 128;
#pragma unroll
            for (int hf = 0; hf < NH; ++hf) {
              tma_load_4d(dst + hf * kHalf, img ? &p.kf : &p.kpf, bar, hf * 64, U.hk, row, U.w.b);
              tma_load_4d(dst + S::kTile + hf * kHalf, img ? &p.vf : &p.vpf, bar, hf * 64, U.hk,
                          row, U.w.b);
            }
          } else if (!KV && tile >= p.n_tiles) {  // dQ: pooled key tile
#pragma unroll
            for (int hf = 0; hf < NH; ++hf) {
              tma_load_4d(dst + hf * kHalf, &p.kpf, bar, hf * 64, U.hk, (tile - p.n_tiles) * 128,
                          U.w.b);
              tma_load_4d(dst + S::kTile + hf * kHalf, &p.vpf, bar, hf * 64, U.hk,
                          (tile - p.n_tiles) * 128, U.w.b);
            }
          } else {
            load_window_tile<NH>(pv, KV ? p.qm : p.km, &p.fill, U.w, tile, KV ? h : U.hk, p.T,
                                 p.Hg, p.Wg, p.N, dst, bar);
            load_window_tile<NH>(pv, KV ? p.gm : p.vm, &p.fill, U.w, tile, KV ? h : U.hk, p.T,
                                 p.Hg, p.Wg, p.N, dst + S::kTile, bar);
          }
        }
        if (text_q)
          write_row_values_flat(p, U.w.b, ttile, h, rowv + slot * 256, lane, true);
        else if (MODE == kModePooled)
          write_row_values_flat(p, U.w.b, ftile, h, rowv + slot * 256, lane);
        else if (KV)
          write_row_values(p, pv, U.w, tile, h, rowv + slot * 256, lane);
        mbar_arrive(BAR(S::BFULL + slot));
        issued |= 1u << slot;
        last_par = (last_par & ~(1u << slot)) | (par << slot);
        ++nb;
      }
    }
    for (int s = 0; s < 2; ++s)  // every copy issued has landed before the CTA exits
      if (issued & (1u << s))
        wait_warp(BAR(S::BFULL + s), (last_par >> s) & 1u, abort_flag, limit, kBSiteLoadDrainB,
                  false);
  } else if (warp == 2) {
    // ------------------------------------------------------------ unit-pair loader
    uint32_t na = 0;
    bool ok = true;
    for (uint32_t u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
      const BwdUnit U = decode_bwd_unit<MODE>(p, u);
      if (!(ok = wait_warp(BAR(S::AEMPTY), (na & 1u) ^ 1u, abort_flag, limit, kBSiteLoadAEmpty)))
        break;
      const uint32_t dst = sbase + S::a0;
      if (lane == 0) {
        mbar_expect_tx(BAR(S::AFULL), 2 * S::kTile);
        if (MODE == kModePooled) {  // pooled key tile: Kp, Vp
#pragma unroll
          for (int hf = 0; hf < NH; ++hf) {
            tma_load_4d(dst + hf * kHalf, &p.kpf, BAR(S::AFULL), hf * 64, U.hk, U.tile * 128,
                        U.w.b);
            tma_load_4d(dst + S::kTile + hf * kHalf, &p.vpf, BAR(S::AFULL), hf * 64, U.hk,
                        U.tile * 128, U.w.b);
          }
        } else if (MODE == kModeDqText) {  // text query tile: Qt, dOt
#pragma unroll
          for (int hf = 0; hf < NH; ++hf) {
            tma_load_4d(dst + hf * kHalf, &p.qtf, BAR(S::AFULL), hf * 64, U.h, U.tile * 128,
                        U.w.b);
            tma_load_4d(dst + S::kTile + hf * kHalf, &p.gtf, BAR(S::AFULL), hf * 64, U.h,
                        U.tile * 128, U.w.b);
          }
        } else {
          load_window_tile<NH>(pv, KV ? p.km : p.qm, &p.fill, U.w, U.tile, KV ? U.hk : U.h, p.T,
                               p.Hg, p.Wg, p.N, dst, BAR(S::AFULL));
          load_window_tile<NH>(pv, KV ? p.vm : p.gm, &p.fill, U.w, U.tile, KV ? U.hk : U.h, p.T,
                               p.Hg, p.Wg, p.N, dst + S::kTile, BAR(S::AFULL));
        }
      }
      if (MODE == kModeDq) write_row_values(p, pv, U.w, U.tile, U.h, rowv, lane);
      if (MODE == kModeDqText) write_row_values_flat(p, U.w.b, U.tile, U.h, rowv, lane, true);
      mbar_arrive(BAR(S::AFULL));
      ++na;
    }
    if (na) wait_warp(BAR(S::AFULL), (na - 1) & 1u, abort_flag, limit, kBSiteLoadDrainA, false);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t IDX = idesc_bf16(128, false);  // X, Y: N = 128 rows of B, K-major
    constexpr uint32_t IDG = idesc_bf16(D, true);     // gradients: N = d, B MN-major
    uint32_t na = 0, nb = 0, pf = 0;
    bool ok = true;
    auto take_b = [&](uint32_t& slot) -> bool {
      slot = nb & 1u;
      const uint32_t par = (nb >> 1) & 1u;
      ++nb;
      if (!wait_warp(BAR(S::BFULL + slot), par, abort_flag, limit, kBSiteMmaBFull)) return false;
      tc_fence_after();
      return true;
    };
    // X = A0 B0^T into columns [0, 128), Y = A1 B1^T into [128, 256) (lane 0
    // only).  dKV reads A0, A1 from shared memory; dQ from TMEM columns
    // [384, 448) and [448, 512), where the elementwise threads copied them.
    auto mma_xy = [&](uint32_t slot) {
      const uint32_t a = sbase + S::a0;
      const uint32_t b = sbase + S::ring + slot * 2 * S::kTile;
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = t * S::kTile + (k / 4) * kHalf + (k % 4) * 32;
          if (KV)
            mma_bf16(tmem + t * 128, sdesc(a + off, 16, 1024), sdesc(b + off, 16, 1024), IDX,
                     k > 0 ? 1u : 0u);
          else
            mma_bf16_ts(tmem + t * 128, tmem + kTmemA + t * 64 + k * 8, sdesc(b + off, 16, 1024),
                        IDX, k > 0 ? 1u : 0u);
        }
    };
    // TMEM column of the bf16 operand for keys (or queries) 16 kk .. 16 kk + 15:
    // each elementwise warpgroup packs its 64 columns into the first 32 of them.
    auto opcol = [](int kk) -> uint32_t { return (uint32_t)(kk < 4 ? kk * 8 : 64 + (kk - 4) * 8); };
    // the gradient MMAs of one step (lane 0 only)
    auto mma_grad = [&](uint32_t slot, bool acc) {
      const uint32_t b = sbase + S::ring + slot * 2 * S::kTile;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t a1 = acc || kk > 0 ? 1u : 0u;
        if (KV) {
          // dV += P^T dO_i (P^T over X), dK += dS^T Q_i (dS^T over Y)
          mma_bf16_ts(tmem + 256, tmem + opcol(kk), sdesc(b + S::kTile + kk * 2048, kHalf, 1024),
                      IDG, a1);
          mma_bf16_ts(tmem + 256 + D, tmem + 128 + opcol(kk), sdesc(b + kk * 2048, kHalf, 1024),
                      IDG, a1);
        } else {
          // dQ += dS K_j (dS over X)
          mma_bf16_ts(tmem + 256, tmem + opcol(kk), sdesc(b + kk * 2048, kHalf, 1024), IDG, a1);
        }
      }
    };
    // The unit pair is read for the last time by the X, Y MMAs of the last
    // step: dKV then frees its shared-memory slot, dQ its TMEM copy.
    const int a_free = KV ? S::AEMPTY : S::ATFREE;
    for (uint32_t u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
      const BwdUnit U = decode_bwd_unit<MODE>(p, u);
      const int n_steps = bwd_steps<MODE>(p, U);
      if (!(ok = wait_warp(BAR(KV ? S::AFULL : S::ATFULL), na & 1u, abort_flag, limit,
                           kBSiteMmaAFull)))
        break;
      ++na;
      tc_fence_after();
      uint32_t slot;
      if (!(ok = take_b(slot))) break;
      if (lane == 0) {
        mma_xy(slot);
        if (n_steps == 1) mma_commit(BAR(a_free));
        mma_commit(BAR(S::SFULL));
      }
      __syncwarp();
      for (int s = 0; s < n_steps && ok; ++s) {
        // P and dS of step s in TMEM; for s = 0 this also orders the previous
        // unit's epilogue reads of the accumulators before the overwrite below.
        if (!(ok = wait_warp(BAR(S::PFULL), pf & 1u, abort_flag, limit, kBSiteMmaPFull))) break;
        ++pf;
        tc_fence_after();
        if (lane == 0) {
          mma_grad(slot, s > 0);
          mma_commit(BAR(S::BEMPTY + slot));
        }
        __syncwarp();
        if (s + 1 < n_steps) {
          if (!(ok = take_b(slot))) break;
          if (lane == 0) {
            mma_xy(slot);
            if (s + 2 == n_steps) mma_commit(BAR(a_free));
            mma_commit(BAR(S::SFULL));
          }
          __syncwarp();
        } else {
          if (lane == 0) mma_commit(BAR(S::OFULL));
          __syncwarp();
        }
      }
    }
    if (lane == 0) mma_commit(BAR(S::DRAIN));  // every MMA issued completes before TMEM is freed
    __syncwarp();
    wait_warp(BAR(S::DRAIN), 0u, abort_flag, limit, kBSiteMmaDrain, false);
  } else if (warp >= 4) {
    // ------------------------------------------------------------ elementwise + epilogue
    const int hc = (warp - 4) >> 2;  // 64-column half of X and Y
    const int q4 = warp & 3;         // TMEM lane quadrant
    const int r = q4 * 32 + lane;    // row of X, Y and the accumulators
    const uint32_t tl = (uint32_t)(q4 * 32) << 16;
    const uint32_t tX = tmem + tl + 64 * hc;
    const uint32_t tY = tmem + tl + 128 + 64 * hc;
    const uint32_t stg = sbase + S::stg + (uint32_t)(warp - 4) * 2048u;
    const float c = p.scale_log2;
    const uint64_t c2 = f2pack(c, c);
    uint32_t sf = 0, af = 0, atf = 0, nb = 0, of = 0;
    bool ok = true;
    // dQ: copies the unit pair from shared memory into TMEM (warpgroup hc
    // copies tile hc, Q or dO, both head-dim halves of its rows) and reads the
    // row's -lse*log2(e) and -D; then frees the shared-memory slot, so that
    // the next unit's pair is loaded a whole unit ahead.
    auto copy_a = [&](uint64_t& l2, uint64_t& d2) -> bool {
      if (!wait_warp(BAR(S::AFULL), af & 1u, abort_flag, limit, kBSiteEwAFull)) return false;
      ++af;
      if (!wait_warp(BAR(S::ATFREE), (atf & 1u) ^ 1u, abort_flag, limit, kBSiteEwATFree))
        return false;
      ++atf;
      tc_fence_after();
      const uint32_t src = sbase + S::a0 + hc * S::kTile;
#pragma unroll
      for (int hf = 0; hf < NH; ++hf) {
        uint32_t w[32];
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 v4 = ld_shared_v4(src + hf * kHalf + swz(r, ch));
          w[4 * ch] = v4.x;
          w[4 * ch + 1] = v4.y;
          w[4 * ch + 2] = v4.z;
          w[4 * ch + 3] = v4.w;
        }
        tmem_st32(tmem + tl + kTmemA + 64 * hc + 32 * hf, w);
      }
      l2 = f2pack(-rowv[r], -rowv[r]);
      d2 = f2pack(-rowv[128 + r], -rowv[128 + r]);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(BAR(S::AEMPTY));
      mbar_arrive(BAR(S::ATFULL));
      return true;
    };
    uint64_t nl2 = 0, nd2 = 0;  // dQ: -lse*log2(e) and -D of this thread's query row
    if (!KV && blockIdx.x < p.n_units) ok = copy_a(nl2, nd2);
    for (uint32_t u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
      const BwdUnit U = decode_bwd_unit<MODE>(p, u);
      const int n_steps = bwd_steps<MODE>(p, U);
      // the grid token (pooled: the pooled token) of this thread's gradient
      // row, found while the unit's first MMAs run
      long long tok;
      if (MODE == kModePooled)
        tok = 128LL * U.tile + r < p.P ? 128LL * U.tile + r : -1;
      else if (MODE == kModeDqText)
        tok = 128LL * U.tile + r < p.L ? 128LL * U.tile + r : -1;
      else
        tok = r < pv.rows[U.tile] ? window_row_token(pv, U.w, U.tile, r, p.T, p.Hg, p.Wg) : -1;
      for (int s = 0; s < n_steps; ++s) {
        const float* rv = rowv;
        if (KV) {
          const uint32_t slot = nb & 1u;
          if (!(ok = wait_warp(BAR(S::BFULL + slot), (nb >> 1) & 1u, abort_flag, limit,
                               kBSiteEwBFull)))
            break;
          ++nb;
          rv = rowv + slot * 256;
        }
        if (!(ok = wait_warp(BAR(S::SFULL), sf & 1u, abort_flag, limit, kBSiteEwSFull))) break;
        ++sf;
        tc_fence_after();
        // Two chunks of 32 columns; each chunk's bf16 pairs go over the 16
        // columns of X (and Y) that the chunk itself came from.
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t x[32], y[32];
          tmem_ld32(tX + 32 * cc, x);
          tmem_ld32(tY + 32 * cc, y);
          tmem_wait_ld(x);
          tmem_wait_ld(y);
          uint32_t wp[16], wd[16];  // bf16 pairs of P and dS for columns 2e, 2e + 1
          float lz = 0.f, lw = 0.f, gz = 0.f, gw = 0.f;  // dKV: the second pair of four columns
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            uint64_t l2 = nl2, d2 = nd2;
            if (KV) {  // lse*log2(e) and D of query columns 2e, 2e + 1 (loaded four at a time)
              if ((e % 2) == 0) {
                const int col = 64 * hc + 32 * cc + 2 * e;
                const uint4 L = ld_shared_v4(smem_u32(rv + col));
                const uint4 G = ld_shared_v4(smem_u32(rv + 128 + col));
                l2 = f2pack(-__uint_as_float(L.x), -__uint_as_float(L.y));
                d2 = f2pack(-__uint_as_float(G.x), -__uint_as_float(G.y));
                lz = __uint_as_float(L.z);
                lw = __uint_as_float(L.w);
                gz = __uint_as_float(G.z);
                gw = __uint_as_float(G.w);
              } else {
                l2 = f2pack(-lz, -lw);
                d2 = f2pack(-gz, -gw);
              }
            }
            const uint64_t t2 =
                f2fma(f2pack(__uint_as_float(x[2 * e]), __uint_as_float(x[2 * e + 1])), c2, l2);
            float t0, t1;
            f2unpack(t2, t0, t1);
            const uint64_t p2 = f2pack(ex2(t0), ex2(t1));
            const uint64_t g2 =
                f2add(f2pack(__uint_as_float(y[2 * e]), __uint_as_float(y[2 * e + 1])), d2);
            float p0, p1, g0, g1;
            f2unpack(p2, p0, p1);
            f2unpack(f2mul(g2, p2), g0, g1);
            wp[e] = pack_bf16(p0, p1);
            wd[e] = pack_bf16(g0, g1);
          }
          if (KV) {
            tmem_st16(tX + 16 * cc, wp);  // P^T
            tmem_st16(tY + 16 * cc, wd);  // dS^T
          } else {
            tmem_st16(tX + 16 * cc, wd);  // dS
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(BAR(S::PFULL));
      }
      if (!ok) break;
      uint64_t nl2n = 0, nd2n = 0;
      if (!KV && u + gridDim.x < p.n_units && !(ok = copy_a(nl2n, nd2n))) break;
      // epilogue: the accumulators of this unit -> bf16 -> token rows
      if (!(ok = wait_warp(BAR(S::OFULL), of & 1u, abort_flag, limit, kBSiteEwOFull))) break;
      ++of;
      tc_fence_after();
      if (MODE == kModePooled) {
        // warpgroup 0 adds its dV rows into dvp, warpgroup 1 its dK rows into
        // dkp: fp32 sums over the query-tile splits of the batch (no scale yet)
        float* dst = tok >= 0 ? (hc == 0 ? p.dvp : p.dkp) +
                                    (((long long)U.w.b * p.P + tok) * p.Hkv + U.hk) * D
                              : nullptr;
#pragma unroll
        for (int hf = 0; hf < NH; ++hf) {
          uint32_t o[2][32];
          tmem_ld32(tmem + tl + 256 + hc * D + hf * 64, o[0]);
          tmem_ld32(tmem + tl + 256 + hc * D + hf * 64 + 32, o[1]);
          tmem_wait_ld(o[0]);
          tmem_wait_ld(o[1]);
          if (dst) {
#pragma unroll
            for (int e = 0; e < 16; ++e)
              atomicAdd(reinterpret_cast<float4*>(dst + hf * 64 + 4 * e),
                        make_float4(__uint_as_float(o[e / 8][(4 * e) % 32]),
                                    __uint_as_float(o[e / 8][(4 * e) % 32 + 1]),
                                    __uint_as_float(o[e / 8][(4 * e) % 32 + 2]),
                                    __uint_as_float(o[e / 8][(4 * e) % 32 + 3])));
          }
        }
      } else if (KV) {
        // warpgroup 0 writes dV, warpgroup 1 writes dK (times the scale); with
        // pooled memory each row first adds its cell's pooled gradient / count
        const long long roff = tok >= 0 ? (((long long)U.w.b * p.N + tok) * p.Hkv + U.hk) * D : -1;
        __nv_bfloat16* base = hc == 0 ? p.dv : p.dk;
        const float mul = hc == 0 ? 1.0f : p.scale;
        const uint64_t m2 = f2pack(mul, mul);
        const float* share = nullptr;
        if (p.P && !p.joint && tok >= 0) {  // pooled cells only: text keys are their own rows
          const long long hw = (long long)p.Hg * p.Wg;
          const long long t = tok / hw, y = (tok / p.Wg) % p.Hg, x = tok % p.Wg;
          const long long cell =
              ((t / p.pt) * (p.Hg / p.ph) + y / p.ph) * (p.Wg / p.pw) + x / p.pw;
          if (kChecked && cell >= p.P)
            check_failed(kCheckPooledRow);
          else
            share = (hc == 0 ? p.dvp : p.dkp) + (((long long)U.w.b * p.P + cell) * p.Hkv + U.hk) * D;
        }
        const uint64_t ic2 = f2pack(p.inv_count, p.inv_count);
#pragma unroll
        for (int hf = 0; hf < NH; ++hf) {
          uint32_t o[2][32];
          tmem_ld32(tmem + tl + 256 + hc * D + hf * 64, o[0]);
          tmem_ld32(tmem + tl + 256 + hc * D + hf * 64 + 32, o[1]);
          tmem_wait_ld(o[0]);
          tmem_wait_ld(o[1]);
          if (share) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float2 sv = *reinterpret_cast<const float2*>(share + hf * 64 + 2 * e);
              float o0, o1;
              f2unpack(f2fma(f2pack(sv.x, sv.y), ic2,
                             f2pack(__uint_as_float(o[e / 16][(2 * e) % 32]),
                                    __uint_as_float(o[e / 16][(2 * e) % 32 + 1]))), o0, o1);
              o[e / 16][(2 * e) % 32] = __float_as_uint(o0);
              o[e / 16][(2 * e) % 32 + 1] = __float_as_uint(o1);
            }
          }
          uint32_t w[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            float o0, o1;
            f2unpack(f2mul(f2pack(__uint_as_float(o[e / 16][(2 * e) % 32]),
                                  __uint_as_float(o[e / 16][(2 * e) % 32 + 1])), m2), o0, o1);
            w[e] = pack_bf16(o0, o1);
          }
          warp_store_row64(stg, w, roff, base, hf * 64, lane, p.kv_elems);
        }
      } else if (hc < NH) {
        // warpgroup hc writes columns [64 hc, 64 hc + 64) of dQ (text: dQt), times the scale
        constexpr bool TQ = MODE == kModeDqText;
        const long long nrows = TQ ? p.L : p.N;
        const long long roff = tok >= 0 ? (((long long)U.w.b * nrows + tok) * p.H + U.h) * D : -1;
        const uint64_t m2 = f2pack(p.scale, p.scale);
        uint32_t o[2][32];
        tmem_ld32(tmem + tl + 256 + hc * 64, o[0]);
        tmem_ld32(tmem + tl + 256 + hc * 64 + 32, o[1]);
        tmem_wait_ld(o[0]);
        tmem_wait_ld(o[1]);
        uint32_t w[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          float o0, o1;
          f2unpack(f2mul(f2pack(__uint_as_float(o[e / 16][(2 * e) % 32]),
                                __uint_as_float(o[e / 16][(2 * e) % 32 + 1])), m2), o0, o1);
          w[e] = pack_bf16(o0, o1);
        }
        warp_store_row64(stg, w, roff, TQ ? p.dqt : p.dq, hc * 64, lane,
                         TQ ? p.qt_elems : p.q_elems);
      }
      tc_fence_before();  // the reads of the accumulators precede the next unit's MMAs
      nl2 = nl2n;
      nd2 = nd2n;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, int MODE>
basa_status launch_bwd_kernel(BwdTcParams* prm, long long units, cudaStream_t stream) {
  static_assert(BwdSmem<D>::alloc <= 232448, "shared memory plan exceeds 227 KB");
  const int smem = BwdSmem<D>::alloc;
  if (units > 0x7fffffffLL) return BASA_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(tc_bwd_kernel<D, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem) != cudaSuccess)
    return BASA_ERR_CUDA;
  prm->n_units = (uint32_t)units;
  prm->fd_h = FastDiv(prm->H);
  prm->fd_hkv = FastDiv(prm->Hkv);
  prm->fd_tiles = FastDiv(prm->n_tiles);
  prm->fd_windows = FastDiv(prm->n_windows);
  prm->fd_nww = FastDiv(prm->nww);
  prm->fd_nwh = FastDiv(prm->nwh);
  prm->fd_group = FastDiv(prm->group);
  prm->fd_tt = FastDiv(prm->n_tt);
  prm->fd_pt = FastDiv(prm->n_pt);
  prm->fd_fsplits = FastDiv(prm->n_fsplits);
  const long long grid = persistent_grid(units);
  tc_bwd_kernel<D, MODE><<<(unsigned)grid, kBwdTcThreads, smem, stream>>>(*prm);
  return cudaGetLastError() == cudaSuccess ? BASA_OK : BASA_ERR_CUDA;
}

// The three kernels in order: the pooled tokens' gradients (when P), dQ, then
// the window dK, dV (which add each row's share of the pooled gradients).
template <int D>
basa_status launch_bwd_all(BwdTcParams* prm, const Dims& d, long long per, cudaStream_t stream) {
  basa_status st;
  if (d.P) {
    const size_t bytes = (size_t)d.B * d.P * d.Hkv * d.d * sizeof(float);
    if (cudaMemsetAsync(prm->dkp, 0, bytes, stream) != cudaSuccess ||
        cudaMemsetAsync(prm->dvp, 0, bytes, stream) != cudaSuccess)
      return BASA_ERR_CUDA;
    const long long pooled_units = (long long)d.B * d.Hkv * prm->n_pt * prm->n_fsplits;
    if ((st = launch_bwd_kernel<D, kModePooled>(prm, pooled_units, stream)) != BASA_OK) return st;
  }
  if ((st = launch_bwd_kernel<D, kModeDq>(prm, (long long)d.B * d.H * per, stream)) != BASA_OK)
    return st;
  return launch_bwd_kernel<D, kModeDkv>(prm, (long long)d.B * d.Hkv * per, stream);
}

// Text keys' gradients from their fp32 sums: dkt = scale * dkp, dvt = dvp,
// rounded to bf16 once ([B, L, Hkv, d], four elements per thread).
__global__ void __launch_bounds__(256) text_grad_round_kernel(const float* dkp, const float* dvp,
                                                              __nv_bfloat16* dkt,
                                                              __nv_bfloat16* dvt, float scale,
                                                              long long n4) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  const float4 a = reinterpret_cast<const float4*>(dkp)[i];
  const float4 b = reinterpret_cast<const float4*>(dvp)[i];
  uint2 ka, vb;
  ka.x = pack_bf16(a.x * scale, a.y * scale);
  ka.y = pack_bf16(a.z * scale, a.w * scale);
  vb.x = pack_bf16(b.x, b.y);
  vb.y = pack_bf16(b.z, b.w);
  reinterpret_cast<uint2*>(dkt)[i] = ka;
  reinterpret_cast<uint2*>(dvt)[i] = vb;
}

// The joint backward's launches: D of the image and text rows, the text keys'
// dK, dV (over the image and the text queries, summed into dkp, dvp), the
// image dQ (window then text keys), the text dQ (every key), the window dK, dV
// (window then text queries), and the rounding of the text keys' gradients.
template <int D>
basa_status launch_bwd_joint_all(BwdTcParams* prm, const Dims& d, long long per,
                                 const JointGrads& jg, float* dkp, float* dvp,
                                 cudaStream_t stream) {
  basa_status st;
  const size_t n = (size_t)d.B * jg.L * d.Hkv * d.d;
  if (cudaMemsetAsync(dkp, 0, n * sizeof(float), stream) != cudaSuccess ||
      cudaMemsetAsync(dvp, 0, n * sizeof(float), stream) != cudaSuccess)
    return BASA_ERR_CUDA;
  const long long text_key_units = (long long)d.B * d.Hkv * prm->n_pt * prm->n_fsplits;
  if ((st = launch_bwd_kernel<D, kModePooled>(prm, text_key_units, stream)) != BASA_OK) return st;
  if ((st = launch_bwd_kernel<D, kModeDq>(prm, (long long)d.B * d.H * per, stream)) != BASA_OK)
    return st;
  if ((st = launch_bwd_kernel<D, kModeDqText>(prm, (long long)d.B * d.H * prm->n_tt, stream)) !=
      BASA_OK)
    return st;
  if ((st = launch_bwd_kernel<D, kModeDkv>(prm, (long long)d.B * d.Hkv * per, stream)) != BASA_OK)
    return st;
  const long long n4 = (long long)(n / 4);
  text_grad_round_kernel<<<(unsigned)((n4 + 255) / 256), 256, 0, stream>>>(
      dkp, dvp, static_cast<__nv_bfloat16*>(jg.dkt), static_cast<__nv_bfloat16*>(jg.dvt),
      d.scale, n4);
  return cudaGetLastError() == cudaSuccess ? BASA_OK : BASA_ERR_CUDA;
}

basa_status build_and_launch_bwd(BwdTcParams* prm, const Dims& d, const TilePlan& plan,
                                 const void* q, const void* k, const void* v, const void* out,
                                 const void* dout, const float* lse, float* dD, void* dq,
                                 void* dk, void* dv, const PoolGrads* pg, uint32_t timeout_ms,
                                 cudaStream_t stream, const JointGrads* jg = nullptr,
                                 float* jdkp = nullptr, float* jdvp = nullptr) {
  basa_status st;
  const uint64_t D = (uint64_t)d.d, H = (uint64_t)d.H, Hk = (uint64_t)d.Hkv;
  if ((st = pack_plan_image(plan, &prm->plan)) != BASA_OK) return st;
  const uint64_t qdims[5] = {D, H, (uint64_t)d.Wg, (uint64_t)d.Hg, (uint64_t)d.B * d.T};
  const uint64_t qstr[4] = {D * 2, H * D * 2, (uint64_t)d.Wg * H * D * 2,
                            (uint64_t)d.Hg * d.Wg * H * D * 2};
  const uint64_t kdims[5] = {D, Hk, (uint64_t)d.Wg, (uint64_t)d.Hg, (uint64_t)d.B * d.T};
  const uint64_t kstr[4] = {D * 2, Hk * D * 2, (uint64_t)d.Wg * Hk * D * 2,
                            (uint64_t)d.Hg * d.Wg * Hk * D * 2};
  for (int s = 0; s < plan.n_shapes; ++s) {
    const uint32_t box[5] = {64, 1, plan.shape_bw[s], plan.shape_bh[s], plan.shape_bt[s]};
    if ((st = encode_map(&prm->qm[s], q, 5, qdims, qstr, box)) != BASA_OK) return st;
    if ((st = encode_map(&prm->gm[s], dout, 5, qdims, qstr, box)) != BASA_OK) return st;
    if ((st = encode_map(&prm->km[s], k, 5, kdims, kstr, box)) != BASA_OK) return st;
    if ((st = encode_map(&prm->vm[s], v, 5, kdims, kstr, box)) != BASA_OK) return st;
  }
  {
    const uint64_t fdims[4] = {D, Hk, (uint64_t)d.N, (uint64_t)d.B};
    const uint64_t fstr[3] = {D * 2, Hk * D * 2, (uint64_t)d.N * Hk * D * 2};
    const uint32_t box8[4] = {64, 1, 8, 1};
    if ((st = encode_map(&prm->fill, k, 4, fdims, fstr, box8)) != BASA_OK) return st;
  }
  if (d.P) {  // pooled K, V tiles; q and dout as flat 128-row tiles for the pooled kernel
    const uint64_t pdims[4] = {D, Hk, (uint64_t)d.P, (uint64_t)d.B};
    const uint64_t pstr[3] = {D * 2, Hk * D * 2, (uint64_t)d.P * Hk * D * 2};
    const uint64_t fqdims[4] = {D, H, (uint64_t)d.N, (uint64_t)d.B};
    const uint64_t fqstr[3] = {D * 2, H * D * 2, (uint64_t)d.N * H * D * 2};
    const uint32_t box128[4] = {64, 1, 128, 1};
    if ((st = encode_map(&prm->kpf, pg->kp, 4, pdims, pstr, box128)) != BASA_OK) return st;
    if ((st = encode_map(&prm->vpf, pg->vp, 4, pdims, pstr, box128)) != BASA_OK) return st;
    if ((st = encode_map(&prm->qf, q, 4, fqdims, fqstr, box128)) != BASA_OK) return st;
    if ((st = encode_map(&prm->gf, dout, 4, fqdims, fqstr, box128)) != BASA_OK) return st;
    prm->dkp = pg->dkp;
    prm->dvp = pg->dvp;
    prm->P = d.P;
    prm->n_pt = (int)((d.P + 127) / 128);
    prm->n_fqt = (int)((d.N + 127) / 128);
    // split the grid's query tiles so that the pooled kernel has about four
    // units per SM
    const long long base = (long long)d.B * d.Hkv * prm->n_pt;
    long long n = (4LL * tc_sm_count() + base - 1) / base;
    if (n > prm->n_fqt) n = prm->n_fqt;
    if (n < 1) n = 1;
    prm->fqt_per_split = (int)((prm->n_fqt + n - 1) / n);
    prm->n_fsplits = (prm->n_fqt + prm->fqt_per_split - 1) / prm->fqt_per_split;
    prm->pt = d.pt; prm->ph = d.ph; prm->pw = d.pw;
    prm->inv_count = 1.0f / (float)(d.pt * d.ph * d.pw);
  }
  if (jg) {  // text tokens in the pooled slots, text queries as flat tiles, flat image K, V
    const uint64_t L = (uint64_t)jg->L;
    const uint64_t tkdims[4] = {D, Hk, L, (uint64_t)d.B};
    const uint64_t tkstr[3] = {D * 2, Hk * D * 2, L * Hk * D * 2};
    const uint64_t tqdims[4] = {D, H, L, (uint64_t)d.B};
    const uint64_t tqstr[3] = {D * 2, H * D * 2, L * H * D * 2};
    const uint64_t fqdims[4] = {D, H, (uint64_t)d.N, (uint64_t)d.B};
    const uint64_t fqstr[3] = {D * 2, H * D * 2, (uint64_t)d.N * H * D * 2};
    const uint64_t fkdims[4] = {D, Hk, (uint64_t)d.N, (uint64_t)d.B};
    const uint64_t fkstr[3] = {D * 2, Hk * D * 2, (uint64_t)d.N * Hk * D * 2};
    const uint32_t box128[4] = {64, 1, 128, 1};
    if ((st = encode_map(&prm->kpf, jg->kt, 4, tkdims, tkstr, box128)) != BASA_OK) return st;
    if ((st = encode_map(&prm->vpf, jg->vt, 4, tkdims, tkstr, box128)) != BASA_OK) return st;
    if ((st = encode_map(&prm->qtf, jg->qt, 4, tqdims, tqstr, box128)) != BASA_OK) return st;
    if ((st = encode_map(&prm->gtf, jg->dout_t, 4, tqdims, tqstr, box128)) != BASA_OK) return st;
    if ((st = encode_map(&prm->qf, q, 4, fqdims, fqstr, box128)) != BASA_OK) return st;
    if ((st = encode_map(&prm->gf, dout, 4, fqdims, fqstr, box128)) != BASA_OK) return st;
    if ((st = encode_map(&prm->kf, k, 4, fkdims, fkstr, box128)) != BASA_OK) return st;
    if ((st = encode_map(&prm->vf, v, 4, fkdims, fkstr, box128)) != BASA_OK) return st;
    prm->joint = 1;
    prm->L = jg->L;
    prm->P = jg->L;
    prm->n_tt = (int)((jg->L + 127) / 128);
    prm->n_pt = prm->n_tt;
    prm->n_fqt = (int)((d.N + 127) / 128);
    prm->dkp = jdkp;
    prm->dvp = jdvp;
    prm->lse_t = jg->lse_t;
    prm->dD_t = jg->dD_t;
    prm->dqt = static_cast<__nv_bfloat16*>(jg->dqt);
    prm->qt_elems = (long long)d.B * jg->L * d.H * d.d;
    // split the image and text query tiles so that the text keys' kernel has
    // about four units per SM
    const int nq = prm->n_fqt + prm->n_tt;
    const long long base = (long long)d.B * d.Hkv * prm->n_pt;
    long long n = (4LL * tc_sm_count() + base - 1) / base;
    if (n > nq) n = nq;
    if (n < 1) n = 1;
    prm->fqt_per_split = (int)((nq + n - 1) / n);
    prm->n_fsplits = (nq + prm->fqt_per_split - 1) / prm->fqt_per_split;
    prm->pt = prm->ph = prm->pw = 1;
    prm->inv_count = 1.0f;
  }
  prm->lse = lse;
  prm->dD = dD;
  prm->q_elems = (long long)d.B * d.N * d.H * d.d;
  prm->kv_elems = (long long)d.B * d.N * d.Hkv * d.d;
  prm->dq = static_cast<__nv_bfloat16*>(dq);
  prm->dk = static_cast<__nv_bfloat16*>(dk);
  prm->dv = static_cast<__nv_bfloat16*>(dv);
  prm->timeout_ns = (unsigned long long)(timeout_ms ? timeout_ms : 2000u) * 1000000ull;
  prm->N = d.N;
  prm->H = d.H; prm->Hkv = d.Hkv; prm->group = d.H / d.Hkv;
  prm->T = d.T; prm->Hg = d.Hg; prm->Wg = d.Wg;
  prm->wt = d.wt; prm->wh = d.wh; prm->ww = d.ww;
  prm->st = d.st; prm->sh = d.sh; prm->sw = d.sw;
  prm->nwt = d.nwt; prm->nwh = d.nwh; prm->nww = d.nww;
  prm->n_windows = d.nwt * d.nwh * d.nww;
  prm->n_tiles = plan.n_tiles;
  prm->n_shapes = plan.n_shapes;
  prm->scale = d.scale;
  prm->scale_log2 = d.scale * kLog2e;
  const long long per = (long long)prm->n_windows * plan.n_tiles;
  // D = rowsum(dout * out) (joint: also of the text rows), then the gradient kernels
  if ((st = launch_bwd_prep(d, out, dout, dD, stream)) != BASA_OK) return st;
  if (jg) {
    Dims dt = d;
    dt.N = jg->L;
    if ((st = launch_bwd_prep(dt, jg->out_t, jg->dout_t, jg->dD_t, stream)) != BASA_OK) return st;
    return d.d == 64 ? launch_bwd_joint_all<64>(prm, d, per, *jg, jdkp, jdvp, stream)
                     : launch_bwd_joint_all<128>(prm, d, per, *jg, jdkp, jdvp, stream);
  }
  return d.d == 64 ? launch_bwd_all<64>(prm, d, per, stream)
                   : launch_bwd_all<128>(prm, d, per, stream);
}

}  // namespace

basa_status launch_bwd_tc(const Dims& d, const void* q, const void* k, const void* v,
                          const void* out, const void* dout, const float* lse, float* dD,
                          void* dq, void* dk, void* dv, const PoolGrads* pg, uint32_t timeout_ms,
                          cudaStream_t stream) {
  // padded grids: the CUDA-core kernels (these kernels do not mask padded rows)
  if (d.dtype != BASA_BF16 || (d.d != 64 && d.d != 128) || d.qsep || (d.P && !pg) || d.padded)
    return BASA_ERR_UNSUPPORTED;
  TilePlan plan;
  basa_status st = build_tile_plan(d, &plan);  // before any launch
  if (st != BASA_OK) return st;
  BwdTcParams* prm = new (std::nothrow) BwdTcParams;
  if (!prm) return BASA_ERR_INVALID_ARG;
  memset(prm, 0, sizeof(*prm));
  st = build_and_launch_bwd(prm, d, plan, q, k, v, out, dout, lse, dD, dq, dk, dv, pg, timeout_ms,
                            stream);
  delete prm;
  return st;
}

basa_status launch_bwd_tc_joint(const Dims& d, const void* q, const void* k, const void* v,
                                const void* out, const void* dout, const float* lse, float* dD,
                                void* dq, void* dk, void* dv, const JointGrads& jg, float* dkp,
                                float* dvp, uint32_t timeout_ms, cudaStream_t stream) {
  if (d.dtype != BASA_BF16 || (d.d != 64 && d.d != 128) || d.qsep || d.P || d.padded ||
      jg.L <= 0 || !dkp || !dvp)
    return BASA_ERR_UNSUPPORTED;
  TilePlan plan;
  basa_status st = build_tile_plan(d, &plan);  // before any launch
  if (st != BASA_OK) return st;
  BwdTcParams* prm = new (std::nothrow) BwdTcParams;
  if (!prm) return BASA_ERR_INVALID_ARG;
  memset(prm, 0, sizeof(*prm));
  st = build_and_launch_bwd(prm, d, plan, q, k, v, out, dout, lse, dD, dq, dk, dv, nullptr,
                            timeout_ms, stream, &jg, dkp, dvp);
  delete prm;
  return st;
}

cudaError_t take_bwd_status(cudaStream_t stream, unsigned int* status, unsigned int* where) {
  return tc_take_status(stream, status, where);
}

}  // namespace basa
