// bf16 shifted local window attention on the 5th-generation tensor cores
// (tcgen05 + TMEM) of sm_100a.
//
// The operation ("BASA: Backend-Agnostic Sparse Attention for Fast
// High-Resolution Diffusion Transformers", zhichai.net topic 178635722, "The
// BASA Method"; forum review of the same paper, reply 178634520, four-part
// method list): every query attends to the keys of its own cyclically shifted
// window, plus the K/V-pooled global-memory tokens when they are given, under
// one softmax.  Full attention is "flat" mode: 128-token tiles of the whole
// grid, each query tile against every key tile.
//
// Work unit: (b, h, window, pair of 128-query tiles).  Persistent CTAs (one
// per SM) walk the units, heads fastest.  Inside a CTA the warps specialise:
//   warp 0        TMA loader of the K and V tiles, through a 4-slot ring (boxes
//                 from the shifted-window tile plan; a tile that crosses a
//                 wrapped border is fetched as up to 8 boxes, so no rolled copy
//                 of the grid is ever made);
//   warp 2        TMA loader of the two query tiles of each unit;
//   warp 1        owns TMEM (512 columns) and issues the MMAs from one thread:
//                 S_i = Q_i K_j^T into TMEM, and O_i += P_i V_j with P_i read
//                 from TMEM; the two query tiles alternate so that one tile's
//                 exponentials overlap the other tile's MMAs;
//   warps 4..7    softmax + epilogue for query tile 0 of the unit,
//   warps 8..11   the same for query tile 1.
// Each softmax thread owns one query row: it reads its 128 logits from TMEM,
// keeps the running max and sum in fp32 (base-2 exponentials with the scale
// folded in), writes the bf16 probabilities P back into TMEM over its logits,
// and rescales its O row in TMEM when the max grows by more than 2^8.  The
// epilogue divides by the sum and rounds to bf16.  Window passes stage the
// tile in shared memory and store it with TMA boxes that mirror the load
// boxes: with at most two key tiles per window (3-slot ring) both 64-column
// halves of both query tiles have their own staging blocks, so the warps move
// on to the next unit while the stores drain, and only the next unit's
// epilogue waits for the staging to have been read; otherwise one half at a
// time.  Flat passes and padded grids instead have each warp stage its 32 rows
// and write them back with 16-byte stores that cover whole 128-byte row
// segments.
//
// A flat pass with few units (the text queries of a joint call) can split its
// key tiles into ranges (template parameter kSplit): each split-unit writes its
// unnormalised fp32 output and per-row (max, sum) to the caller's workspace and
// split_combine_kernel merges them.
//
// Every mbarrier wait is bounded (wall-clock limit from the call); on expiry the
// kernel raises the device status word, lets every role leave its loop, waits
// (bounded) for its own copies and MMAs in flight, frees TMEM and returns.  The
// PTX wrappers, the bounded waits and the tile-plan helpers shared with the
// backward kernels are in tc_device.cuh.
#include <cuda_bf16.h>
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <new>

#include "basa_internal.h"
#include "tc_device.cuh"

namespace basa {

namespace {

constexpr int kThreads = 384;

struct __align__(64) TcParams {
  CUtensorMap qm[kMaxShapes];  // window boxes, rank 5: [d, H, Wg, Hg, B*T]
  CUtensorMap km[kMaxShapes];
  CUtensorMap vm[kMaxShapes];
  CUtensorMap om[kMaxShapes];
  CUtensorMap qf, kf, vf, of;  // flat 128-row tiles, rank 4: [d, H, N, B]
  CUtensorMap kpf, vpf;        // pooled 128-row tiles, rank 4: [d, H, P, B]
  CUtensorMap fill;            // 8-row box over k's flat view, read out of bounds = zeros
  PlanImage plan;             // compact tile plan, copied to shared memory at start
  float* lse;
  __nv_bfloat16* out;  // [B, T, Hg, Wg, H, d]
  int warp_stores;  // output by warp-staged 16-byte stores (1) or by TMA boxes (0)
  uint32_t n_units;
  long long N;   // key tokens of the grid per (b, h)
  long long Nq;  // query (and output) tokens per (b, h): N, or the text length
  unsigned long long timeout_ns;
  int B, H, T, Hg, Wg;
  int group;  // query heads per K/V head
  // unit decode divisors: H, n_pairs, n_windows, nww, nwh, group
  FastDiv fd_h, fd_pairs, fd_windows, fd_nww, fd_nwh, fd_group;
  int wt, wh, ww, st, sh, sw, nwt, nwh, nww;
  int Tp, Hgp, Wgp;  // padded extents the window origins wrap on (T, Hg, Wg unless padded)
  int padded;        // 1: padded positions exist and are masked
  int n_windows;
  int n_shapes;
  int n_qt;   // query tiles per window (flat: per (b, h))
  int n_pairs;
  int n_wkt;  // key tiles from the window (flat: from the grid)
  int n_pkt;  // pooled key tiles
  int P;
  int flat;
  uint32_t flags;
  float scale_log2;
  // Split key range (flat mode): units_per_split units per split; split s
  // covers key tiles [s * kt_per_split, ...).  With part_o set, each unit
  // writes its unnormalised fp32 output and its (max, sum) per row there
  // instead of the output, for a separate combine.
  int n_splits;
  int kt_per_split;
  uint32_t units_per_split;
  float* part_o;   // [n_splits, B, H, Nq, d]
  float* part_ml;  // [n_splits, B, H, Nq, 2]: base-2 running max, sum
  float v_scale;   // e4m3 inputs: the V descale factor, applied in the epilogue
};

// Two e4m3 values (lower byte first) as a bf16 pair.  Exact: every e4m3 value
// (3 mantissa bits, exponents 2^-9 .. 2^8) is a bf16 value.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t two) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)two, __NV_E4M3);
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
  return pack_bf16(f.x, f.y);
}

// Widens one e4m3 V tile (128 rows of D bytes, 128-byte swizzled rows) into the
// bf16 layout the P.V MMA reads (D / 64 halves of 128 rows x 128 bytes, same
// swizzle).  One warp; each lane converts 16-byte chunks of 16 values.
template <int D>
__device__ __forceinline__ void widen_v_tile(uint32_t src, uint32_t dst, int lane) {
  static_assert(D == 128, "e4m3 tiles have 128-byte rows");
#pragma unroll 4
  for (int it = 0; it < 32; ++it) {
    const int item = it * 32 + lane;
    const int r = item >> 3, c = item & 7;
    const uint4 x = ld_shared_v4(src + r * 128 + ((c ^ (r & 7)) << 4));
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint32_t o[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      o[2 * e] = e4m3x2_to_bf16x2(w[e] & 0xffffu);
      o[2 * e + 1] = e4m3x2_to_bf16x2(w[e] >> 16);
    }
    const uint32_t half = dst + (uint32_t)(c >> 2) * kHalf + r * 128;
    const int c2 = 2 * (c & 3);
    st_shared_v4(half + ((c2 ^ (r & 7)) << 4), o[0], o[1], o[2], o[3]);
    st_shared_v4(half + (((c2 + 1) ^ (r & 7)) << 4), o[4], o[5], o[6], o[7]);
  }
}


// Rescale O only when a tile's row max exceeds the reference max by more than
// 2^kLazyRescale; until then the stale reference is kept (P stays <= 2^8).
constexpr float kLazyRescale = 8.0f;

// Sites recorded by the first wait that gives up (host debug output only).
enum WaitSite : uint32_t {
  kSiteLoadKvEmpty = 1, kSiteLoadQEmpty, kSiteLoadDrainKv, kSiteLoadDrainQ, kSiteMmaQFull,
  kSiteMmaKvFull, kSiteMmaSFree, kSiteMmaPFull, kSiteMmaDrain, kSiteSmxSFull, kSiteSmxPvDone,
  kSiteSmxPvLast, kSiteSmxOStaged, kSiteSmxOFree
};


// ---------------------------------------------------------------------------
// Work-unit decoding
// ---------------------------------------------------------------------------
struct Unit {
  int b, h, hk, pair, cls, ot, oh, ow, nq;  // hk: the K/V head of query head h
  int split, j0, nk;                        // key tiles [j0, j0 + nk)
  int holes;                                // the window holds padded positions
};

// Window mode walks the heads fastest: concurrently running CTAs then read the
// same tokens for all heads, so each token's H*d row (a few DRAM pages) is
// fetched as a whole.  Full-attention mode walks the query-tile pairs fastest,
// so the CTAs in flight share one (b, h)'s K and V through L2.
template <bool kSplit>
__device__ __forceinline__ Unit decode_unit(const TcParams& p, uint32_t u) {
  Unit U;
  if constexpr (kSplit) {
    const int n_kt = p.n_wkt + p.n_pkt;
    U.split = (int)(u / p.units_per_split);
    u %= p.units_per_split;
    U.j0 = U.split * p.kt_per_split;
    const int left = n_kt - U.j0;
    U.nk = left < p.kt_per_split ? left : p.kt_per_split;
  }
  if (p.flat) {
    const uint32_t r = p.fd_pairs.div(u);
    U.pair = (int)(u - r * (uint32_t)p.n_pairs);
    U.b = (int)p.fd_h.div(r);
    U.h = (int)(r - (uint32_t)U.b * (uint32_t)p.H);
    U.cls = 0;
    U.ot = U.oh = U.ow = 0;
    U.holes = 0;
  } else {
    uint32_t r = p.fd_h.div(u);
    U.h = (int)(u - r * (uint32_t)p.H);
    uint32_t r2 = p.fd_pairs.div(r);
    U.pair = (int)(r - r2 * (uint32_t)p.n_pairs);
    U.b = (int)p.fd_windows.div(r2);
    const int win = (int)(r2 - (uint32_t)U.b * (uint32_t)p.n_windows);
    const uint32_t wr = p.fd_nww.div((uint32_t)win);
    const int jw = win - (int)wr * p.nww;
    const int jt = (int)p.fd_nwh.div(wr);
    const int jh = (int)wr - jt * p.nwh;
    U.cls = window_class(jt, jh, jw, p.nwt, p.nwh, p.nww, p.st, p.sh, p.sw);
    U.ot = jt * p.wt + p.st;
    U.oh = jh * p.wh + p.sh;
    U.ow = jw * p.ww + p.sw;
    // An axis's window [o, o + w) on the padded axis (o < Gp, wrapping at Gp)
    // meets the padding [G, Gp) exactly when Gp > G and o + w > G.
    U.holes = p.padded && ((p.Tp > p.T && U.ot + p.wt > p.T) ||
                           (p.Hgp > p.Hg && U.oh + p.wh > p.Hg) ||
                           (p.Wgp > p.Wg && U.ow + p.ww > p.Wg));
  }
  const int left = p.n_qt - 2 * U.pair;
  U.nq = left < 2 ? left : 2;
  U.hk = (int)p.fd_group.div((uint32_t)U.h);
  return U;
}


// Valid rows of key tile j (rows past them are zero-filled and masked).
__device__ __forceinline__ int key_valid(const TcParams& p, const PlanView& pv, int j) {
  if (j >= p.n_wkt) {  // extra keys: pooled cells or text tokens
    const int left = p.P - 128 * (j - p.n_wkt);
    return left < 128 ? left : 128;
  }
  if (p.flat) {
    const long long left = p.N - 128LL * j;
    return left < 128 ? (int)left : 128;
  }
  return pv.rows[j];
}
__device__ __forceinline__ int query_valid(const TcParams& p, const PlanView& pv, int qt) {
  if (p.flat) {
    const long long left = p.Nq - 128LL * qt;
    return left < 128 ? (int)left : 128;
  }
  return pv.rows[qt];
}


// kind: 0 = q, 1 = k, 2 = v.  Loads one 128-row tile (all head-dim halves) into
// shared memory at dst and signals bar with the transaction bytes.
template <int D, bool kF8 = false>
__device__ __forceinline__ void load_tile(const TcParams& p, const PlanView& pv, int kind,
                                          const Unit& U, int tile, uint32_t dst, uint32_t bar) {
  constexpr int NH = kF8 ? D / 128 : D / 64;  // 128-byte boxes per row (coordinate 0 for e4m3)
  if (kind != 0 && tile >= p.n_wkt) {  // extra keys: pooled global memory or text tokens
    const CUtensorMap* m = kind == 1 ? &p.kpf : &p.vpf;
#pragma unroll
    for (int hf = 0; hf < NH; ++hf)
      tma_load_4d(dst + hf * kHalf, m, bar, hf * 64, U.hk, (tile - p.n_wkt) * 128, U.b);
    return;
  }
  const int head = kind == 0 ? U.h : U.hk;
  if (p.flat) {
    const CUtensorMap* m = kind == 0 ? &p.qf : kind == 1 ? &p.kf : &p.vf;
#pragma unroll
    for (int hf = 0; hf < NH; ++hf) tma_load_4d(dst + hf * kHalf, m, bar, hf * 64, head, tile * 128, U.b);
    return;
  }
  const CUtensorMap* maps = kind == 0 ? p.qm : kind == 1 ? p.km : p.vm;
  load_window_tile<NH>(pv, maps, &p.fill, WinAt{U.cls, U.ot, U.oh, U.ow, U.b}, tile, head, p.T,
                       p.Tp, p.Hgp, p.Wgp, p.N, dst, bar);
}

// Stores d-half hf of query tile qt from a 128-row x 64-column staging block
// (128-byte swizzled) with TMA boxes that mirror the load boxes.  Never used on
// a padded grid (its calls take the warp-staged stores, which skip padded rows).
template <int D>
__device__ __forceinline__ void store_half(const TcParams& p, const PlanView& pv, const Unit& U,
                                           int qt, int hf, uint32_t src) {
  if (p.flat) {
    tma_store_4d(&p.of, src, hf * 64, U.h, qt * 128, U.b);
    return;
  }
  const int b0 = pv.first(U.cls, qt), nb = pv.count(U.cls, qt);
#pragma unroll 1
  for (int bi = 0; bi < nb; ++bi) {
    const uint32_t e = pv.entries[b0 + bi];
    const int sid = box_shape(e);
    const int gt = wrap(U.ot + box_lt(e), p.T);
    const int gh = wrap(U.oh + box_lh(e), p.Hg);
    const int gw = wrap(U.ow + box_lw(e), p.Wg);
    if constexpr (kChecked) {
      const int bt = pv.bt[sid], bh = pv.bh[sid], bw = pv.bw[sid];
      if (sid >= kMaxShapes || gt + bt > p.T || gh + bh > p.Hg || gw + bw > p.Wg ||
          box_row8(e) * 8 + bt * bh * bw > 128) {
        check_failed(kCheckStoreBox);
        continue;
      }
    }
    tma_store_5d(&p.om[sid], src + box_row8(e) * 1024, hf * 64, U.h, gw, gh, U.b * p.T + gt);
  }
}

// Flattened grid index of the token held in row r of query tile qt.
__device__ __forceinline__ long long row_token(const TcParams& p, const PlanView& pv,
                                               const Unit& U, int qt, int r) {
  if (p.flat) return 128LL * qt + r;
  return window_row_token(pv, WinAt{U.cls, U.ot, U.oh, U.ow, U.b}, qt, r, p.Tp, p.Hgp, p.Wgp,
                          p.T, p.Hg, p.Wg);
}

// Bit r of word r / 32: row r of key tile j of U's window holds a token (not a
// padded position, not a row past the tile).  Warp-collective.
__device__ __forceinline__ uint4 key_token_mask(const TcParams& p, const PlanView& pv, const Unit& U,
                                             int j, int lane) {
  uint32_t w[4];
#pragma unroll
  for (int cc = 0; cc < 4; ++cc)
    w[cc] = __ballot_sync(0xffffffffu, row_token(p, pv, U, j, cc * 32 + lane) >= 0);
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Shared-memory plan: the unit's two 128-row query tiles, output staging (one
// 64-column block per query tile, or both halves of both query tiles with the
// 3-slot ring), and a ring of K/V tiles.  The probabilities P
// never touch shared memory: they are written into TMEM over their logits and
// read from there by the P.V MMA.
template <int D, int kRing, bool kF8 = false>
struct Smem {
  // Q/K/V tile bytes: 128 rows of D bf16 (D / 64 swizzled halves), or of D e4m3
  static constexpr int kTile = kF8 ? (D / 128) * kHalf : (D / 64) * kHalf;
  static constexpr int kVbf = (D / 64) * kHalf;   // one V tile widened to bf16 (e4m3 only)
  static constexpr int NS = kRing;                // K/V ring slots
  // 3-slot ring (windows of at most two key tiles): room to stage both output
  // halves of both query tiles, so the TMA stores of a unit need no wait
  static constexpr bool kFullStg = kRing == 3 && !kF8 && D == 128;
  static constexpr int q0 = 0;
  static constexpr int stg0 = 2 * kTile;
  static constexpr int ring0 = stg0 + (kFullStg ? 4 : 2) * kHalf;
  static constexpr int vbf0 = ring0 + NS * kTile;
  static constexpr int bars = vbf0 + (kF8 ? 2 * kVbf : 0);
  // barrier indices (VBFULL, VBEMPTY: the two widened V buffers, e4m3 only)
  static constexpr int QFULL = 0, QEMPTY = 2, SFULL = 4, PFULL = 6, OFULL = 8, STAGED = 10,
                       STGFREE = 12, DRAIN = 14, KVFULL = 15, KVEMPTY = 15 + NS,
                       VBFULL = 15 + 2 * NS, VBEMPTY = 17 + 2 * NS,
                       NBARS = 15 + 2 * NS + (kF8 ? 4 : 0);
  static_assert(VBEMPTY == VBFULL + 2, "two widened V buffers");
  static constexpr int misc = bars + NBARS * 8;  // tmem slot, abort flag
  static constexpr int plan = misc + 64;         // compact tile plan (kPlanBytes)
  static constexpr int bytes = plan + kPlanBytes;
  static constexpr int alloc = bytes + 1024;     // slack for 1024-byte alignment
};

// Schedule of one unit (query tiles i = 0, 1 against key tiles j = 0..n-1).
// TMEM columns: S_0 | S_1 | O_0 | O_1 (128 each); P_i is written as bf16 pairs
// over the first 64 columns of S_i.  The MMA warp issues S_0(0), S_1(0), then
// per key tile j: O_0 += P_0(j) V_j, S_0(j+1), O_1 += P_1(j) V_j, S_1(j+1).
// The tensor core executes one thread's MMAs in issue order, so S_i(j+1) only
// overwrites P_i(j) after the P.V MMA that reads it.  The two query tiles
// alternate: while softmax 0 exponentiates S_0(j+1), the tensor core runs
// P_1(j) V_j and S_1(j+1), and the other way round, so the exponentials of one
// tile overlap the MMAs of the other.
template <int D, int kRing, bool kSplit, bool kF8 = false>
__global__ void __launch_bounds__(kThreads, 1) tc_attn_kernel(const __grid_constant__ TcParams p) {
  using S = Smem<D, kRing, kF8>;
  constexpr int NS = S::NS;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + S::bars;
  auto BAR = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::misc);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + S::misc + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint64_t limit = p.timeout_ns;

  // the compact tile plan, from the parameter block into shared memory
  const PlanView pv = plan_to_smem(p.plan, smem + S::plan, p.n_qt, threadIdx.x, kThreads);
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR(S::QFULL + i), 1);
      mbar_init(BAR(S::QEMPTY + i), 1);
      mbar_init(BAR(S::SFULL + i), 1);
      mbar_init(BAR(S::PFULL + i), 128);
      mbar_init(BAR(S::OFULL + i), 1);
      mbar_init(BAR(S::STAGED + i), 128);
      mbar_init(BAR(S::STGFREE + i), 1);
    }
    mbar_init(BAR(S::DRAIN), 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(BAR(S::KVFULL + s), 1);
      mbar_init(BAR(S::KVEMPTY + s), 1);
    }
    if constexpr (kF8) {
      for (int b = 0; b < 2; ++b) {
        mbar_init(BAR(S::VBFULL + b), 1);
        mbar_init(BAR(S::VBEMPTY + b), 1);
      }
    }
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
  const int n_kt = p.n_wkt + p.n_pkt;
  // Key tiles of unit U: [kbeg, kend); without a split, every key tile.
  auto kbeg = [&](const Unit& U) -> int {
    if constexpr (kSplit) return U.j0; else return 0;
  };
  auto kcount = [&](const Unit& U) -> int {
    if constexpr (kSplit) return U.nk; else return n_kt;
  };
  // Pull every tensor map this launch uses into the TMA descriptor cache.
  if (threadIdx.x == 0) {
    if (p.flat) {
      prefetch_tmap(&p.qf); prefetch_tmap(&p.kf); prefetch_tmap(&p.vf); prefetch_tmap(&p.of);
    } else {
      for (int sid = 0; sid < p.n_shapes; ++sid) {
        prefetch_tmap(&p.qm[sid]); prefetch_tmap(&p.km[sid]);
        prefetch_tmap(&p.vm[sid]); prefetch_tmap(&p.om[sid]);
      }
      prefetch_tmap(&p.fill);
    }
    if (p.n_pkt) { prefetch_tmap(&p.kpf); prefetch_tmap(&p.vpf); }
  }

  const bool withhold = (p.flags & BASA_FLAG_TEST_WITHHOLD_LOADS) != 0;
  if (warp == 0) {
    // ------------------------------------------------------------ K/V loader
    // The whole warp walks the schedule and waits; lane 0 issues the copies.
    // Ring order per unit: K_0, V_0, K_1, V_1, ... (the MMA warp's order).
    if (!withhold) {
      uint32_t kv = 0;
      uint32_t issued_mask = 0, last_par = 0;
      bool ok = true, dep_done = false;
      for (uint32_t u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
        const Unit U = decode_unit<kSplit>(p, u);
        for (int j = kbeg(U); j < kbeg(U) + kcount(U) && ok; ++j) {
          if (j >= p.n_wkt && !dep_done) {
            // extra keys may be pooled by the kernel this one was launched as a
            // dependent of: wait for that grid (returns at once otherwise)
            grid_dependency_wait();
            dep_done = true;
          }
          for (int kind = 1; kind <= 2 && ok; ++kind) {
            const uint32_t slot = kv % NS, par = (kv / NS) & 1u;
            if (!(ok = wait_warp(BAR(S::KVEMPTY + slot), par ^ 1u, abort_flag, limit,
                                 kSiteLoadKvEmpty)))
              break;
            if (lane == 0) {
              mbar_expect_tx(BAR(S::KVFULL + slot), S::kTile);
              load_tile<D, kF8>(p, pv, kind, U, j, sbase + S::ring0 + slot * S::kTile,
                                BAR(S::KVFULL + slot));
            }
            __syncwarp();
            issued_mask |= 1u << slot;
            last_par = (last_par & ~(1u << slot)) | (par << slot);
            ++kv;
          }
        }
      }
      // Drain: wait (bounded, regardless of an abort) until every copy issued has landed.
      for (int s = 0; s < NS; ++s)
        if (issued_mask & (1u << s))
          wait_warp(BAR(S::KVFULL + s), (last_par >> s) & 1u, abort_flag, limit,
                    kSiteLoadDrainKv, false);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ query loader
    // Q_i of the next unit is fetched as soon as the last S MMA of the current
    // unit has read Q_i.
    if (!withhold) {
      uint32_t qn[2] = {0u, 0u};
      uint32_t q_issued = 0, q_last = 0;
      bool ok = true;
      for (uint32_t u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
        const Unit U = decode_unit<kSplit>(p, u);
        for (int i = 0; i < U.nq && ok; ++i) {
          if (!(ok = wait_warp(BAR(S::QEMPTY + i), (qn[i] & 1u) ^ 1u, abort_flag, limit,
                               kSiteLoadQEmpty)))
            break;
          if (lane == 0) {
            mbar_expect_tx(BAR(S::QFULL + i), S::kTile);
            load_tile<D, kF8>(p, pv, 0, U, 2 * U.pair + i, sbase + S::q0 + i * S::kTile,
                              BAR(S::QFULL + i));
          }
          __syncwarp();
          q_issued |= 1u << i;
          q_last = (q_last & ~(1u << i)) | ((qn[i] & 1u) << i);
          ++qn[i];
        }
        __syncwarp();
      }
      for (int i = 0; i < 2; ++i)
        if (q_issued & (1u << i))
          wait_warp(BAR(S::QFULL + i), (q_last >> i) & 1u, abort_flag, limit, kSiteLoadDrainQ,
                    false);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp walks the schedule and waits; lane 0 issues MMAs and commits.
    constexpr uint32_t IDS = kF8 ? idesc_e4m3(128) : idesc_bf16(128, false);
    constexpr uint32_t IDO = idesc_bf16(D, true);
    uint32_t qf[2] = {0u, 0u}, pfull[2] = {0u, 0u};
    uint32_t kv = 0, vbn = 0;
    bool ok = true;
    auto take_slot = [&](uint32_t& slot) -> bool {
      slot = kv % NS;
      const uint32_t par = (kv / NS) & 1u;
      ++kv;
      if (!wait_warp(BAR(S::KVFULL + slot), par, abort_flag, limit, kSiteMmaKvFull)) return false;
      tc_fence_after();
      return true;
    };
    auto release = [&](uint32_t slot) {
      if (lane == 0) mma_commit(BAR(S::KVEMPTY + slot));
      __syncwarp();
    };
    // V_j for P.V: its ring slot (bf16), or (e4m3) the widened bf16 copy that
    // warp 3 makes, whose ring slot warp 3 releases; vref = slot or buffer.
    auto take_v = [&](uint32_t& vaddr, uint32_t& vref) -> bool {
      if constexpr (kF8) {
        ++kv;
        vref = vbn & 1u;
        const uint32_t par = (vbn >> 1) & 1u;
        ++vbn;
        if (!wait_warp(BAR(S::VBFULL + vref), par, abort_flag, limit, kSiteMmaKvFull)) return false;
        tc_fence_after();
        vaddr = sbase + S::vbf0 + vref * S::kVbf;
        return true;
      } else {
        if (!take_slot(vref)) return false;
        vaddr = sbase + S::ring0 + vref * S::kTile;
        return true;
      }
    };
    auto release_v = [&](uint32_t vref) {
      if constexpr (kF8) {
        if (lane == 0) mma_commit(BAR(S::VBEMPTY + vref));
        __syncwarp();
      } else {
        release(vref);
      }
    };
    // S_i = Q_i K^T (lane 0 only)
    auto mma_s = [&](int i, uint32_t kslot) {
      const uint32_t qa = sbase + S::q0 + i * S::kTile;
      const uint32_t ka = sbase + S::ring0 + kslot * S::kTile;
      if constexpr (kF8) {  // 32 e4m3 (32 bytes) per step along the 128-byte rows
#pragma unroll
        for (int k = 0; k < D / 32; ++k) {
          const uint32_t off = (k / 4) * kHalf + (k % 4) * 32;
          mma_e4m3(tmem + i * 128, sdesc(qa + off, 16, 1024), sdesc(ka + off, 16, 1024), IDS,
                   k > 0 ? 1u : 0u);
        }
      } else {
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k / 4) * kHalf + (k % 4) * 32;
          mma_bf16(tmem + i * 128, sdesc(qa + off, 16, 1024), sdesc(ka + off, 16, 1024), IDS,
                   k > 0 ? 1u : 0u);
        }
      }
    };
    // O_i (+)= P_i V, P_i from TMEM (8 columns per 16 keys) (lane 0 only)
    auto mma_pv = [&](int i, uint32_t va, bool accumulate) {
#pragma unroll
      for (int k = 0; k < 8; ++k)
        mma_bf16_ts(tmem + 256 + i * 128, tmem + i * 128 + k * 8,
                    sdesc(va + k * 2048, kHalf, 1024), IDO, (accumulate || k > 0) ? 1u : 0u);
    };
    // A unit's coordinates take a chain of dependent divisions (by reciprocal
    // multipliers) to decode: the next unit's are decoded while this unit's
    // exponentials run.
    Unit Un = decode_unit<kSplit>(p, blockIdx.x);
    for (uint32_t u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
      const Unit U = Un;
      uint32_t kslot;
      if (!(ok = take_slot(kslot))) break;
      for (int i = 0; i < U.nq && ok; ++i) {
        if (!(ok = wait_warp(BAR(S::QFULL + i), qf[i] & 1u, abort_flag, limit, kSiteMmaQFull)))
          break;
        ++qf[i];
        tc_fence_after();
        if (lane == 0) {
          mma_s(i, kslot);
          mma_commit(BAR(S::SFULL + i));
          if (kcount(U) == 1) mma_commit(BAR(S::QEMPTY + i));  // Q_i read for the last time
        }
        __syncwarp();
      }
      if (!ok) break;
      release(kslot);
      if (u + gridDim.x < p.n_units) Un = decode_unit<kSplit>(p, u + gridDim.x);
      for (int j = 0; j < kcount(U) && ok; ++j) {
        const bool next = j + 1 < kcount(U);
        uint32_t vaddr, vref;
        if (!(ok = take_v(vaddr, vref))) break;
        if (next && !(ok = take_slot(kslot))) break;
        for (int i = 0; i < U.nq && ok; ++i) {
          // P_i(j) in TMEM and O_i rescaled; for j = 0 this also orders the
          // previous unit's epilogue reads of O_i before the overwrite below.
          if (!(ok = wait_warp(BAR(S::PFULL + i), pfull[i] & 1u, abort_flag, limit,
                               kSiteMmaPFull)))
            break;
          ++pfull[i];
          tc_fence_after();
          if (lane == 0) {
            mma_pv(i, vaddr, j > 0);
            if (next) {
              mma_s(i, kslot);
              mma_commit(BAR(S::SFULL + i));
              if (j + 2 == kcount(U)) mma_commit(BAR(S::QEMPTY + i));  // Q_i read for the last time
            } else {
              mma_commit(BAR(S::OFULL + i));
            }
          }
          __syncwarp();
        }
        if (!ok) break;
        release_v(vref);
        if (next) release(kslot);
      }
    }
    // Drain: every MMA issued has completed before TMEM is released.
    if (lane == 0) mma_commit(BAR(S::DRAIN));
    __syncwarp();
    wait_warp(BAR(S::DRAIN), 0u, abort_flag, limit, kSiteMmaDrain, false);
  } else if (warp == 3) {
    // ------------------------------------------------------------ V widening (e4m3)
    // Walks the K/V ring in the loader's order; each V tile is widened to bf16
    // into one of two buffers for the P.V MMA (whose operands must both be
    // bf16), then its ring slot is handed back to the loader.
    if constexpr (kF8) {
      if (!withhold) {
        uint32_t kv = 0, vbn = 0;
        bool ok = true;
        for (uint32_t u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
          const Unit U = decode_unit<kSplit>(p, u);
          for (int j = kbeg(U); j < kbeg(U) + kcount(U) && ok; ++j) {
            ++kv;  // K_j
            const uint32_t slot = kv % NS, par = (kv / NS) & 1u;
            ++kv;
            const uint32_t b = vbn & 1u, bpar = (vbn >> 1) & 1u;
            ++vbn;
            if (!(ok = wait_warp(BAR(S::KVFULL + slot), par, abort_flag, limit, kSiteMmaKvFull)))
              break;
            if (!(ok = wait_warp(BAR(S::VBEMPTY + b), bpar ^ 1u, abort_flag, limit,
                                 kSiteMmaKvFull)))
              break;
            tc_fence_after();
            widen_v_tile<D>(sbase + S::ring0 + slot * S::kTile, sbase + S::vbf0 + b * S::kVbf,
                            lane);
            fence_proxy_async();  // the generic stores, before the tensor core reads them
            __syncwarp();
            if (lane == 0) {
              mbar_arrive(BAR(S::VBFULL + b));
              mbar_arrive(BAR(S::KVEMPTY + slot));
            }
            __syncwarp();
          }
        }
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax + epilogue
    const int i = (warp - 4) / 4;      // query tile slot of the unit
    const int q4 = warp & 3;           // TMEM lane quadrant
    const int r = q4 * 32 + lane;      // query row owned by this thread
    const uint32_t tl = (uint32_t)(q4 * 32) << 16;
    const uint32_t tS = tmem + tl + i * 128;
    const uint32_t tO = tmem + tl + 256 + i * 128;
    const uint32_t stg = sbase + S::stg0 + i * kHalf;  // output staging, 128 x 64, swizzled
    uint32_t sfull = 0, ofull = 0, staged = 0, stgfree = 0;
    const bool leader = (warp % 4 == 0) && lane == 0;
    bool stg_busy = false;  // a TMA store may still be reading the staging block
    const float c = p.scale_log2;
    bool ok = true;
    // next unit decoded while this unit's last P.V MMA runs
    Unit Un = decode_unit<kSplit>(p, blockIdx.x);
    for (uint32_t u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
      const Unit U = Un;
      const bool more = u + gridDim.x < p.n_units;
      if (i >= U.nq) {
        if (more) Un = decode_unit<kSplit>(p, u + gridDim.x);
        continue;
      }
      const int qt = 2 * U.pair + i;
      float m = -INFINITY, l = 0.f;
      for (int j = kbeg(U); j < kbeg(U) + kcount(U); ++j) {
        if (!(ok = wait_warp(BAR(S::SFULL + i), sfull & 1u, abort_flag, limit, kSiteSmxSFull)))
          break;
        ++sfull;
        tc_fence_after();
        uint32_t s[4][32];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) tmem_ld32(tS + cc * 32, s[cc]);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) tmem_wait_ld(s[cc]);
        const int kvalid = key_valid(p, pv, j);
        if (kvalid < 128) {  // padding keys of a partial tile
#pragma unroll
          for (int cc = 0; cc < 4; ++cc)
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (cc * 32 + e >= kvalid) s[cc][e] = __float_as_uint(-INFINITY);
        }
        if (U.holes && j < p.n_wkt) {  // keys at padded positions of this window
          const uint4 ok4 = key_token_mask(p, pv, U, j, lane);
          const uint32_t okw[4] = {ok4.x, ok4.y, ok4.z, ok4.w};
#pragma unroll
          for (int cc = 0; cc < 4; ++cc)
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (!((okw[cc] >> e) & 1u)) s[cc][e] = __float_as_uint(-INFINITY);
        }
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            mx0 = max3(mx0, __uint_as_float(s[cc][e]), __uint_as_float(s[cc][e + 1]));
            mx1 = max3(mx1, __uint_as_float(s[cc][e + 2]), __uint_as_float(s[cc][e + 3]));
          }
        const float mtile = fmaxf(mx0, mx1) * c;
        float alpha = 1.0f;
        if (mtile > m + kLazyRescale) {  // first tile (m = -inf) or a large jump
          alpha = ex2(m - mtile);
          m = mtile;
        }
        const uint64_t c2 = f2pack(c, c);
        // every key so far masked (a tile of padded positions): P = 0, not NaN
        const float mneg = m == -INFINITY ? 0.f : -m;
        const uint64_t nm2 = f2pack(mneg, mneg);
        uint64_t rsa = f2pack(0.f, 0.f), rsb = rsa;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t pk[16];  // P as bf16 pairs of keys (2e, 2e + 1) of this 32-key chunk
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint64_t x2 = f2fma(f2pack(__uint_as_float(s[cc][2 * e]),
                                             __uint_as_float(s[cc][2 * e + 1])), c2, nm2);
            float a0, a1;
            f2unpack(x2, a0, a1);
            const uint64_t p2 = f2pack(ex2(a0), ex2(a1));
            if (e & 1) rsb = f2add(rsb, p2); else rsa = f2add(rsa, p2);
            float p0, p1;
            f2unpack(p2, p0, p1);
            pk[e] = pack_bf16(p0, p1);
          }
          tmem_st16(tS + cc * 16, pk);  // over logits already read
        }
        float ra0, ra1, rb0, rb1;
        f2unpack(rsa, ra0, ra1);
        f2unpack(rsb, rb0, rb1);
        l = l * alpha + ((ra0 + ra1) + (rb0 + rb1));
        // O_i is stable here: S_i(j) was issued after P_i(j-1) V_{j-1}, so its
        // completion covers that MMA.  tcgen05.ld/st are warp-collective: the
        // whole warp rescales if any of its rows needs it.
        if (j > kbeg(U) && __any_sync(0xffffffffu, alpha < 1.0f)) {
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(tO + cc * 32, o);
            tmem_wait_ld(o);
            const uint64_t a2 = f2pack(alpha, alpha);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              float o0, o1;
              f2unpack(f2mul(f2pack(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), a2), o0, o1);
              o[e] = __float_as_uint(o0);
              o[e + 1] = __float_as_uint(o1);
            }
            tmem_st32(tO + cc * 32, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(BAR(S::PFULL + i));
      }
      if (!ok) break;
      if (more) Un = decode_unit<kSplit>(p, u + gridDim.x);
      // epilogue: O / l -> bf16 -> staging -> stores
      if (!(ok = wait_warp(BAR(S::OFULL + i), ofull & 1u, abort_flag, limit, kSiteSmxPvLast)))
        break;
      ++ofull;
      tc_fence_after();
      if constexpr (kSplit) {
        // Split key range: this split's unnormalised fp32 output and its
        // (max, sum) in base 2, for the combine kernel.
        const bool valid = r < query_valid(p, pv, qt);
        const long long row =
            (((long long)U.split * p.B + U.b) * p.H + U.h) * p.Nq + 128LL * qt + r;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + cc * 32, o);
          tmem_wait_ld(o);
          if (valid) {
            float4* dst = reinterpret_cast<float4*>(p.part_o + row * D + cc * 32);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = make_float4(__uint_as_float(o[4 * e]), __uint_as_float(o[4 * e + 1]),
                                   __uint_as_float(o[4 * e + 2]), __uint_as_float(o[4 * e + 3]));
          }
        }
        if (valid) *reinterpret_cast<float2*>(p.part_ml + 2 * row) = make_float2(m, l);
        tc_fence_before();  // the reads of O_i precede the next unit's first P.V MMA
        continue;
      }
      float inv = 1.0f / l;
      if constexpr (kF8) inv = p.v_scale / l;
      const uint64_t inv2 = f2pack(inv, inv);
      if (p.warp_stores) {
        // Warp-staged stores: each warp converts its 32 rows one 64-column half
        // at a time into its own 4 KB of shared memory (128-byte rows, 16-byte
        // chunks XOR-swizzled by row), then reads them back so that each 16-byte
        // store instruction writes four whole 128-byte row segments.
        const uint32_t wst = sbase + S::stg0 + (uint32_t)(warp - 4) * 4096u;
        const long long tok = r < query_valid(p, pv, qt) ? row_token(p, pv, U, qt, r) : -1;
#pragma unroll
        for (int hf = 0; hf < D / 64; ++hf) {
          uint32_t o[2][32];
          tmem_ld32(tO + hf * 64, o[0]);
          tmem_ld32(tO + hf * 64 + 32, o[1]);
          tmem_wait_ld(o[0]);
          tmem_wait_ld(o[1]);
          uint32_t w[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            float o0, o1;
            f2unpack(f2mul(f2pack(__uint_as_float(o[e / 16][(2 * e) % 32]),
                                  __uint_as_float(o[e / 16][(2 * e) % 32 + 1])), inv2), o0, o1);
            w[e] = pack_bf16(o0, o1);
          }
#pragma unroll
          for (int ch = 0; ch < 8; ++ch)
            st_shared_v4(wst + lane * 128 + ((ch ^ (lane & 7)) << 4), w[4 * ch], w[4 * ch + 1],
                         w[4 * ch + 2], w[4 * ch + 3]);
          __syncwarp();
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int rr = k * 4 + lane / 8, c = lane % 8;
            const uint4 val = ld_shared_v4(wst + rr * 128 + ((c ^ (rr & 7)) << 4));
            const long long t = __shfl_sync(0xffffffffu, tok, rr);
            if (t >= 0) {
              if (kChecked && t >= p.Nq)
                check_failed(kCheckOutRow);
              else
                *reinterpret_cast<uint4*>(p.out + (((long long)U.b * p.Nq + t) * p.H + U.h) * D +
                                          hf * 64 + c * 8) = val;
            }
          }
          __syncwarp();
        }
      }
      if constexpr (S::kFullStg) {
        if (!p.warp_stores) {
          const uint32_t stg2 = sbase + S::stg0 + (uint32_t)i * 2u * kHalf;
          if (stg_busy) {  // the previous unit's stores have read the staging blocks
            if (leader) {
              bulk_wait_read0();
              mbar_arrive(BAR(S::STGFREE + i));
            }
            if (!(ok = wait_warp(BAR(S::STGFREE + i), stgfree & 1u, abort_flag, limit,
                                 kSiteSmxOFree)))
              break;
            ++stgfree;
          }
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            uint32_t o[2][32];
            tmem_ld32(tO + hf * 64, o[0]);
            tmem_ld32(tO + hf * 64 + 32, o[1]);
            tmem_wait_ld(o[0]);
            tmem_wait_ld(o[1]);
            uint32_t w[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              float o0, o1;
              f2unpack(f2mul(f2pack(__uint_as_float(o[e / 16][(2 * e) % 32]),
                                    __uint_as_float(o[e / 16][(2 * e) % 32 + 1])), inv2), o0, o1);
              w[e] = pack_bf16(o0, o1);
            }
#pragma unroll
            for (int ch = 0; ch < 8; ++ch)
              st_shared_v4(stg2 + hf * kHalf + swz(r, ch), w[4 * ch], w[4 * ch + 1],
                           w[4 * ch + 2], w[4 * ch + 3]);
          }
          fence_proxy_async();
          mbar_arrive(BAR(S::STAGED + i));
          if (leader &&
              wait_bounded(BAR(S::STAGED + i), staged & 1u, abort_flag, limit, kSiteSmxOStaged)) {
            store_half<D>(p, pv, U, qt, 0, stg2);
            store_half<D>(p, pv, U, qt, 1, stg2 + kHalf);
            bulk_commit();
          }
          ++staged;
          stg_busy = true;
        }
      }
#pragma unroll
      for (int hf = 0; hf < ((p.warp_stores || S::kFullStg) ? 0 : D / 64); ++hf) {
        uint32_t o[2][32];
        tmem_ld32(tO + hf * 64, o[0]);
        tmem_ld32(tO + hf * 64 + 32, o[1]);
        tmem_wait_ld(o[0]);
        tmem_wait_ld(o[1]);
        uint32_t w[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          float o0, o1;
          f2unpack(f2mul(f2pack(__uint_as_float(o[e / 16][(2 * e) % 32]),
                                __uint_as_float(o[e / 16][(2 * e) % 32 + 1])), inv2), o0, o1);
          w[e] = pack_bf16(o0, o1);
        }
        if (stg_busy) {  // the previous store out of this block has read it
          if (!(ok = wait_warp(BAR(S::STGFREE + i), stgfree & 1u, abort_flag, limit,
                               kSiteSmxOFree)))
            break;
          ++stgfree;
        }
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)  // 8 output columns per 16-byte chunk
          st_shared_v4(stg + swz(r, ch), w[4 * ch], w[4 * ch + 1], w[4 * ch + 2], w[4 * ch + 3]);
        fence_proxy_async();
        mbar_arrive(BAR(S::STAGED + i));
        if (leader) {
          if (wait_bounded(BAR(S::STAGED + i), staged & 1u, abort_flag, limit, kSiteSmxOStaged)) {
            store_half<D>(p, pv, U, qt, hf, stg);
            bulk_commit();
            bulk_wait_read0();
          }
          mbar_arrive(BAR(S::STGFREE + i));
        }
        ++staged;
        stg_busy = true;
      }
      if (!ok) break;
      tc_fence_before();  // the reads of O_i precede the next unit's first P.V MMA
      if (p.lse && r < query_valid(p, pv, qt)) {
        const long long n = row_token(p, pv, U, qt, r);
        if (kChecked && n >= p.Nq)
          check_failed(kCheckLseRow);
        else if (n >= 0)
          p.lse[((long long)U.b * p.H + U.h) * p.Nq + n] = (m + __log2f(l)) * 0.69314718055994531f;
      }
    }
  }

  if (warp >= 4 && (warp % 4 == 0) && lane == 0) bulk_wait_all0();  // stores issued
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, int kRing, bool kSplit = false, bool kF8 = false>
basa_status launch_impl(TcParams* prm, cudaStream_t stream, bool dependent) {
  const int smem = Smem<D, kRing, kF8>::alloc;
  static_assert(Smem<D, kRing, kF8>::alloc <= 232448, "shared memory plan exceeds 227 KB");
  if (cudaFuncSetAttribute(tc_attn_kernel<D, kRing, kSplit, kF8>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return BASA_ERR_CUDA;
  // balanced rounds for a few units per SM (flux1024: 44.1 against 45.8 us);
  // one CTA per SM for many (flux2048, 11 units per SM: 116.4 against 118.0 us)
  const long long grid = persistent_grid(prm->n_units, 4);
  // dependent: launched as the programmatic dependent of the kernel before it
  // on the stream (the pooling), so that its start overlaps that kernel's tail
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, tc_attn_kernel<D, kRing, kSplit, kF8>, *prm) != cudaSuccess)
    return BASA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? BASA_OK : BASA_ERR_CUDA;
}

}  // namespace

namespace {

// Fills *prm (zeroed by the caller) for one call and launches the kernel.
basa_status build_and_launch(TcParams* prm, const Dims& d, bool flat, const void* q,
                             const void* k, const void* v, const void* kp, const void* vp,
                             void* out, float* lse, uint32_t flags, uint32_t timeout_ms,
                             cudaStream_t stream, const SplitK* sk, bool after_pool) {
  basa_status st = BASA_OK;
  const uint64_t D = (uint64_t)d.d;
  const uint64_t H = (uint64_t)d.H;
  const uint64_t Hk = (uint64_t)d.Hkv;
  prm->B = d.B; prm->H = d.H; prm->T = d.T; prm->Hg = d.Hg; prm->Wg = d.Wg;
  prm->group = d.H / d.Hkv;
  prm->wt = d.wt; prm->wh = d.wh; prm->ww = d.ww;
  prm->st = d.st; prm->sh = d.sh; prm->sw = d.sw;
  prm->nwt = d.nwt; prm->nwh = d.nwh; prm->nww = d.nww;
  prm->Tp = flat ? d.T : d.Tp;
  prm->Hgp = flat ? d.Hg : d.Hgp;
  prm->Wgp = flat ? d.Wg : d.Wgp;
  prm->padded = flat ? 0 : d.padded;
  prm->N = d.N;
  prm->Nq = d.Nq;
  prm->lse = lse;
  prm->out = static_cast<__nv_bfloat16*>(out);


  prm->flags = flags;
  prm->timeout_ns = (unsigned long long)(timeout_ms ? timeout_ms : 2000u) * 1000000ull;
  prm->scale_log2 = d.scale * d.qk_descale * 1.4426950408889634f;
  prm->v_scale = d.v_descale;
  // e4m3 inputs: one-byte elements, 128-element (128-byte) boxes per row; the
  // output stays bf16 with 64-element boxes
  const bool f8 = d.dtype == BASA_FP8_E4M3;
  const uint64_t es = f8 ? 1 : 2;
  const uint32_t inner = f8 ? 128 : 64;
  const CUtensorMapDataType ity =
      f8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  prm->flat = flat ? 1 : 0;
  prm->P = kp ? (int)d.P : 0;
  bool dep = false;  // launched as the dependent of the pooling kernel
  TilePlan plan;
  if (!flat && (st = build_tile_plan(d, &plan)) != BASA_OK) goto done;  // before any driver call
  // flat [d, H, N, B] views (full attention tiles; the fill source); the query
  // and output views hold Nq tokens (the text length for text queries)
  {
    const uint64_t dims[4] = {D, Hk, (uint64_t)d.N, (uint64_t)d.B};  // k, v (and the fill)
    const uint64_t strides[3] = {D * es, Hk * D * es, (uint64_t)d.N * Hk * D * es};
    const uint64_t qdims[4] = {D, H, (uint64_t)d.Nq, (uint64_t)d.B};
    const uint64_t qstrides[3] = {D * es, H * D * es, (uint64_t)d.Nq * H * D * es};
    const uint64_t ostrides[3] = {D * 2, H * D * 2, (uint64_t)d.Nq * H * D * 2};
    const uint32_t box128[4] = {inner, 1, 128, 1};
    const uint32_t obox128[4] = {64, 1, 128, 1};
    const uint32_t box8[4] = {inner, 1, 8, 1};
    if (flat) {
      if ((st = encode_map(&prm->qf, q, 4, qdims, qstrides, box128, ity)) != BASA_OK) goto done;
      if ((st = encode_map(&prm->kf, k, 4, dims, strides, box128, ity)) != BASA_OK) goto done;
      if ((st = encode_map(&prm->vf, v, 4, dims, strides, box128, ity)) != BASA_OK) goto done;
      if ((st = encode_map(&prm->of, out, 4, qdims, ostrides, obox128)) != BASA_OK) goto done;
    } else {
      if ((st = encode_map(&prm->fill, k, 4, dims, strides, box8, ity)) != BASA_OK) goto done;
    }
  }
  if (kp && f8) { st = BASA_ERR_UNSUPPORTED; goto done; }
  if (kp) {  // extra keys (pooled cells or text tokens) [d, Hkv, P, B]
    const uint64_t pdims[4] = {D, Hk, (uint64_t)d.P, (uint64_t)d.B};
    const uint64_t pstr[3] = {D * 2, Hk * D * 2, (uint64_t)d.P * Hk * D * 2};
    const uint32_t box128[4] = {64, 1, 128, 1};
    if ((st = encode_map(&prm->kpf, kp, 4, pdims, pstr, box128)) != BASA_OK) goto done;
    if ((st = encode_map(&prm->vpf, vp, 4, pdims, pstr, box128)) != BASA_OK) goto done;
  }
  if (flat) {
    const long long nt = (d.N + 127) / 128;
    const long long nqt = (d.Nq + 127) / 128;
    if (nt > (1LL << 24) || nqt > (1LL << 24)) { st = BASA_ERR_UNSUPPORTED; goto done; }
    prm->n_qt = (int)nqt;
    prm->n_wkt = (int)nt;
    prm->n_pkt = kp ? (int)((d.P + 127) / 128) : 0;
    prm->n_windows = 1;
    prm->n_pairs = (prm->n_qt + 1) / 2;
    const long long units = (long long)d.B * d.H * prm->n_pairs;
    if (units > 0x7fffffffLL) { st = BASA_ERR_UNSUPPORTED; goto done; }
    prm->n_units = (uint32_t)units;
    if (sk && sk->n > 1) {  // split key range, partials to the caller's workspace
      const int n_kt = prm->n_wkt + prm->n_pkt;
      prm->n_splits = sk->n;
      prm->kt_per_split = (n_kt + sk->n - 1) / sk->n;
      if ((long long)(sk->n - 1) * prm->kt_per_split >= n_kt || units * sk->n > 0x7fffffffLL) {
        st = BASA_ERR_INVALID_ARG;
        goto done;
      }
      prm->units_per_split = (uint32_t)units;
      prm->n_units = (uint32_t)(units * sk->n);
      prm->part_o = sk->part_o;
      prm->part_ml = sk->part_ml;
    }
  } else {
    if ((st = pack_plan_image(plan, &prm->plan)) != BASA_OK) goto done;
    const uint64_t dims[5] = {D, H, (uint64_t)d.Wg, (uint64_t)d.Hg, (uint64_t)d.B * d.T};
    const uint64_t strides[4] = {D * es, H * D * es, (uint64_t)d.Wg * H * D * es,
                                 (uint64_t)d.Hg * d.Wg * H * D * es};
    const uint64_t ostrides[4] = {D * 2, H * D * 2, (uint64_t)d.Wg * H * D * 2,
                                  (uint64_t)d.Hg * d.Wg * H * D * 2};
    const uint64_t kdims[5] = {D, Hk, (uint64_t)d.Wg, (uint64_t)d.Hg, (uint64_t)d.B * d.T};
    const uint64_t kstrides[4] = {D * es, Hk * D * es, (uint64_t)d.Wg * Hk * D * es,
                                  (uint64_t)d.Hg * d.Wg * Hk * D * es};
    for (int s = 0; s < plan.n_shapes; ++s) {
      const uint32_t box[5] = {inner, 1, plan.shape_bw[s], plan.shape_bh[s], plan.shape_bt[s]};
      const uint32_t obox[5] = {64, 1, plan.shape_bw[s], plan.shape_bh[s], plan.shape_bt[s]};
      if ((st = encode_map(&prm->qm[s], q, 5, dims, strides, box, ity)) != BASA_OK) goto done;
      if ((st = encode_map(&prm->km[s], k, 5, kdims, kstrides, box, ity)) != BASA_OK) goto done;
      if ((st = encode_map(&prm->vm[s], v, 5, kdims, kstrides, box, ity)) != BASA_OK) goto done;
      if ((st = encode_map(&prm->om[s], out, 5, dims, ostrides, obox)) != BASA_OK) goto done;
    }
    prm->n_shapes = plan.n_shapes;
    prm->n_qt = plan.n_tiles;
    prm->n_wkt = plan.n_tiles;
    prm->n_pkt = kp ? (int)((d.P + 127) / 128) : 0;
    prm->n_windows = d.nwt * d.nwh * d.nww;
    prm->n_pairs = (prm->n_qt + 1) / 2;
    const long long units = (long long)d.B * d.H * prm->n_windows * prm->n_pairs;
    if (units > 0x7fffffffLL) { st = BASA_ERR_UNSUPPORTED; goto done; }
    prm->n_units = (uint32_t)units;
  }
  prm->fd_h = FastDiv(prm->H);
  prm->fd_pairs = FastDiv(prm->n_pairs);
  prm->fd_windows = FastDiv(prm->n_windows);
  prm->fd_nww = FastDiv(prm->nww);
  prm->fd_nwh = FastDiv(prm->nwh);
  prm->fd_group = FastDiv(prm->group);
  // Output path: TMA store boxes for windows (both halves staged at once when
  // the window has at most two key tiles and no extra keys), against the
  // warp-staged stores: flux2048 117.6 -> 104.8 us, flux1024 44.2 -> 38.3 us,
  // flux2048_gm4 attention 546 -> 521 us.  Warp-staged stores for flat passes;
  // a padded grid always takes them too (they skip padded rows).
  prm->warp_stores = (flat || prm->padded) ? 1 : 0;
  // K/V ring depth: windows of at most two key tiles and no extra keys stream
  // each K/V tile once per unit and ran faster with 3 slots in flight than with
  // 4; everything else reuses K/V tiles from L2 and runs faster with 4.
  // Split key range: its own instantiation, so that the window kernels carry
  // none of its code.
  // launched as the pooling kernel's dependent only when it reads pooled tiles
  dep = after_pool && prm->n_pkt > 0;
  if (f8) {  // d = 128, no extra keys, no split (checked by the entry points)
    if (d.d != 128 || prm->n_splits > 1 || prm->n_pkt) { st = BASA_ERR_UNSUPPORTED; goto done; }
    st = launch_impl<128, 4, false, true>(prm, stream, dep);
  } else if (prm->n_splits > 1)
    st = d.d == 64 ? launch_impl<64, 8, true>(prm, stream, dep)
                   : launch_impl<128, 4, true>(prm, stream, dep);
  else if (d.d == 64)
    st = launch_impl<64, 8>(prm, stream, dep);
  else if (!flat && prm->n_wkt + prm->n_pkt <= 2)
    st = launch_impl<128, 3>(prm, stream, dep);
  else
    st = launch_impl<128, 4>(prm, stream, dep);
  if (st == BASA_OK && prm->n_splits > 1) st = launch_split_combine(d, *sk, out, lse, stream);
done:
  return st;
}

// Parameter block of the entry points that allocate nothing: one static block,
// used under a lock (the launch copies it, so it is free again on return).
TcParams g_static_params;
std::mutex g_static_params_mu;

}  // namespace

basa_status launch_tc(const Dims& d, bool flat, const void* q, const void* k, const void* v,
                      const void* kp, const void* vp, void* out, float* lse, uint32_t flags,
                      uint32_t timeout_ms, cudaStream_t stream, const SplitK* sk,
                      bool after_pool) {
  TcParams* prm = new (std::nothrow) TcParams;
  if (!prm) return BASA_ERR_INVALID_ARG;
  memset(prm, 0, sizeof(*prm));
  const basa_status st =
      build_and_launch(prm, d, flat, q, k, v, kp, vp, out, lse, flags, timeout_ms, stream, sk,
                       after_pool);
  delete prm;
  return st;
}

basa_status launch_tc_static_params(const Dims& d, bool flat, const void* q, const void* k,
                                    const void* v, const void* kp, const void* vp, void* out,
                                    float* lse, uint32_t flags, uint32_t timeout_ms,
                                    cudaStream_t stream, bool after_pool) {
  std::lock_guard<std::mutex> lock(g_static_params_mu);
  memset(&g_static_params, 0, sizeof(g_static_params));
  return build_and_launch(&g_static_params, d, flat, q, k, v, kp, vp, out, lse, flags,
                          timeout_ms, stream, nullptr, after_pool);
}

namespace {

// Merges the split partials of every (b, h, query row): with M = max_s m_s and
// w_s = 2^(m_s - M), out = sum_s w_s O_s / sum_s w_s l_s (rounded to bf16) and
// lse = (M + log2 sum_s w_s l_s) ln 2.  One warp per row, D / 32 columns per lane.
template <int D>
__global__ void __launch_bounds__(256) split_combine_kernel(const float* po, const float* pml,
                                                            __nv_bfloat16* out, float* lse,
                                                            int n_splits, int H, long long Nq,
                                                            long long rows) {
  constexpr int C = D / 32;
  const long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  if (w >= rows) return;
  float M = -INFINITY;
  for (int sp = 0; sp < n_splits; ++sp) M = fmaxf(M, pml[2 * (sp * rows + w)]);
  float den = 0.f, acc[C];
#pragma unroll
  for (int e = 0; e < C; ++e) acc[e] = 0.f;
  for (int sp = 0; sp < n_splits; ++sp) {
    const long long row = sp * rows + w;
    const float ws = ex2(pml[2 * row] - M);
    den = fmaf(ws, pml[2 * row + 1], den);
    const float* src = po + row * D + lane * C;
#pragma unroll
    for (int e = 0; e < C; ++e) acc[e] = fmaf(ws, src[e], acc[e]);
  }
  const float inv = 1.0f / den;
  const long long n = w % Nq, bh = w / Nq, h = bh % H, b = bh / H;
  __nv_bfloat16* dst = out + ((b * Nq + n) * H + h) * D + lane * C;
#pragma unroll
  for (int e = 0; e < C; ++e) dst[e] = __float2bfloat16_rn(acc[e] * inv);
  if (lse && lane == 0) lse[w] = (M + __log2f(den)) * 0.69314718055994531f;
}

}  // namespace

int flat_split_count(const Dims& d, bool extra_keys) {
  const long long nqt = (d.Nq + 127) / 128;
  const long long units = (long long)d.B * d.H * ((nqt + 1) / 2);
  const long long n_kt = (d.N + 127) / 128 + (extra_keys ? (d.P + 127) / 128 : 0);
  const int sm = tc_sm_count();
  if (units <= 0 || 2 * units > sm) return 1;
  long long n = sm / units;
  if (n > n_kt / 4) n = n_kt / 4;  // at least four key tiles per split
  if (n < 2) return 1;
  const long long per = (n_kt + n - 1) / n;
  return (int)((n_kt + per - 1) / per);
}

size_t flat_split_bytes(const Dims& d, int n_splits) {
  if (n_splits <= 1) return 0;
  const size_t rows = (size_t)n_splits * d.B * d.H * d.Nq;
  const size_t o = (rows * d.d * sizeof(float) + 255) & ~(size_t)255;
  return o + ((rows * 2 * sizeof(float) + 255) & ~(size_t)255);
}

basa_status launch_split_combine(const Dims& d, const SplitK& sk, void* out, float* lse,
                                 cudaStream_t stream) {
  const long long rows = (long long)d.B * d.H * d.Nq;
  const long long blocks = (rows * 32 + 255) / 256;
  if (blocks > 0x7fffffffLL) return BASA_ERR_UNSUPPORTED;
  if (d.d == 64)
    split_combine_kernel<64><<<(unsigned)blocks, 256, 0, stream>>>(
        sk.part_o, sk.part_ml, static_cast<__nv_bfloat16*>(out), lse, sk.n, d.H, d.Nq, rows);
  else
    split_combine_kernel<128><<<(unsigned)blocks, 256, 0, stream>>>(
        sk.part_o, sk.part_ml, static_cast<__nv_bfloat16*>(out), lse, sk.n, d.H, d.Nq, rows);
  return cudaGetLastError() == cudaSuccess ? BASA_OK : BASA_ERR_CUDA;
}

basa_status read_and_clear_status(cudaStream_t stream) {
  unsigned int v = 0, where = 0, vb = 0, whereb = 0;
  if (tc_take_status(stream, &v, &where) != cudaSuccess) return BASA_ERR_CUDA;
  if (take_bwd_status(stream, &vb, &whereb) != cudaSuccess) return BASA_ERR_CUDA;
  if (v | vb) {
    if (getenv("BASA_DEBUG"))
      fprintf(stderr, "basa: device status %u at site %u (backward: %u at %u)\n", v, where, vb,
              whereb);
    return ((v | vb) & 2u) ? BASA_ERR_CHECK : BASA_ERR_TIMEOUT;
  }
  return cudaGetLastError() == cudaSuccess ? BASA_OK : BASA_ERR_CUDA;
}

}  // namespace basa
