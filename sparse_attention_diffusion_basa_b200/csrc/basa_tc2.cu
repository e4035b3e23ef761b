// bf16 shifted window attention for windows of 256 tokens (the FLUX 16 x 16
// windows) on pairs of SMs: tcgen05 MMAs of cta_group::2 over a cluster of two
// CTAs.
//
// The operation is the one of basa_tc.cu ("BASA: Backend-Agnostic Sparse
// Attention for Fast High-Resolution Diffusion Transformers", zhichai.net topic
// 178635722, "The BASA Method"): every query attends to the keys of its own
// cyclically shifted window under one softmax.
//
// Why a CTA pair.  At m = 256 the work is HBM-bound: every (window, head) unit
// reads its Q, K and V once (192 KB in bf16 at d = 128) and writes its output.
// One CTA per SM has room for one unit's tiles only, so the next unit's loads
// can start only as the current unit's compute releases its slots, and the
// kernel runs at about half the memory bandwidth.  A pair of SMs running the
// 2-SM MMA (M = 256: each CTA holds its own 128-query tile; the B operand is
// split between the two shared memories along N) keeps a unit at 96 KB per
// SM: its query tile (32 KB), half of each key tile's rows (2 x 16 KB), half
// of each value tile's head-dim columns (2 x 16 KB).  That leaves room for two
// units per SM, so a unit's loads are issued a whole unit ahead.
//
// Layout of a unit (b, h, window).  The window's tile plan has four 64-row
// tiles (whole window rows).  Query tile r (rows of plan tiles 2r, 2r + 1)
// belongs to CTA r of the pair.  Key tile j (plan tiles 2j, 2j + 1): CTA r
// holds the K rows of plan tile 2j + r, so S_j = Q K_j^T comes out in every
// CTA's TMEM as 128 query rows x 128 keys (plan tile 2j, then 2j + 1); and
// CTA r holds head-dim columns [64 r, 64 r + 64) of V for all 128 keys of the
// tile, so O = P V comes out as 128 query rows x 128 columns in each CTA.
//
// Per unit: the leader (CTA rank 0) issues S_0 and S_1 as soon as both CTAs'
// Q and K halves have landed (into TMEM columns [0, 128) and [128, 256)); the
// softmax warpgroup of each CTA takes the exact max over its row's 256 logits,
// writes the bf16 probabilities over the first 64 columns of S_0 and S_1 and
// signals the leader, which issues O_x = P_0 V_0 + P_1 V_1 into the unit's
// output buffer x = u mod 2 (TMEM columns [256 + 128 x, ...)); the epilogue
// divides by the row sum and stores 16-byte chunks.  Shared-memory slots and
// output buffers alternate between units, so unit u + 1's loads, its S MMAs
// and unit u's epilogue overlap.
//
// Warps of each CTA: 0 loads (Q, K half, V half), 1 owns TMEM and (leader)
// issues the MMAs, 3 (second CTA) forwards the arrival of that CTA's tiles to
// the leader, 4..7 softmax + epilogue.  Every wait is bounded; on expiry a CTA
// raises the device status word, leaves its loops, waits (bounded) for its own
// loads, meets its peer at the cluster barrier, frees TMEM and returns.
#include <cuda_bf16.h>
#include <math.h>
#include <string.h>

#include <mutex>
#include <new>

#include "basa_internal.h"
#include "tc_device.cuh"

namespace basa {
namespace {

constexpr int kPairThreads = 256;
constexpr int kQB = 2 * kHalf;        // query tile: 128 rows x 2 head-dim halves
constexpr int kKHalfB = 64 * 128;     // 64 key rows x 64 head-dim columns
constexpr int kKB = 2 * kKHalfB;      // K rows of one plan tile, both halves
constexpr int kVB = kHalf;            // 128 keys x 64 head-dim columns

struct __align__(64) PairParams {
  CUtensorMap qm[kMaxShapes];  // window boxes, rank 5: [d, H, Wg, Hg, B*T]
  CUtensorMap km[kMaxShapes];
  CUtensorMap vm[kMaxShapes];
  PlanImage plan;              // 64-row tiles; tiles 2i, 2i + 1 form 128-row tile i
  float* lse;
  __nv_bfloat16* out;          // [B, T, Hg, Wg, H, d]
  uint32_t n_units;
  long long N;
  unsigned long long timeout_ns;
  int B, H, T, Hg, Wg, group;
  int wt, wh, ww, st, sh, sw, nwt, nwh, nww;
  int n_windows, n_shapes;
  uint32_t flags;
  float scale_log2;
};

// Shared memory of one CTA: two slots of (Q, K halves of key tiles 0 and 1),
// two slots of (V halves of key tiles 0 and 1), 4 KB of output staging per
// softmax warp, barriers, the tile plan.
struct PairSmem {
  static constexpr int q0 = 0;                       // slot x: q0 + x kQB
  static constexpr int k0 = 2 * kQB;                 // slot x, tile j: k0 + (2x + j) kKB
  static constexpr int v0 = k0 + 4 * kKB;            // slot x, tile j: v0 + (2x + j) kVB
  static constexpr int stg0 = v0 + 4 * kVB;
  static constexpr int bars = stg0 + 4 * 4096;
  // QKF, VF: this CTA's Q+K, V slot landed; QKE, VE: slot free (MMA commit,
  // both CTAs); PQK, PVF: (leader) the second CTA's slot landed; SF: both S
  // tiles of the unit in TMEM; PF: (leader) P_j written by all 8 softmax warps
  // of the pair; OF: O_x complete; OR: (leader) O_x read by all 8 epilogue warps
  static constexpr int QKF = 0, VF = 2, QKE = 4, VE = 6, PQK = 8, PVF = 10, SF = 12, PF = 13,
                       OF = 15, OR = 17, DRAIN = 19, NBARS = 20;
  static constexpr int misc = bars + NBARS * 8;      // tmem slot, abort flag
  static constexpr int plan = misc + 64;
  static constexpr int bytes = plan + kPlanBytes;
  static constexpr int alloc = bytes + 1024;         // slack for 1024-byte alignment
};

enum PairSite : uint32_t {
  kPSiteLoadEmpty = 301, kPSiteLoadDrain, kPSiteFwd, kPSiteMmaFull, kPSiteMmaPeer, kPSiteMmaP,
  kPSiteMmaOFree, kPSiteMmaDrain, kPSiteSmxS, kPSiteSmxO
};

// ---------------------------------------------------------------------------
// Cluster and CTA-pair PTX
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_count() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// All threads of both CTAs.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
// Address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
// try_wait with cluster-scope acquire (barriers that the other CTA arrives on).
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __noinline__ bool wait_slow_cluster(uint32_t bar, uint32_t parity,
                                               volatile uint32_t* abort_flag, uint64_t limit_ns,
                                               uint32_t site, bool honour_abort) {
  const long long c0 = clock64();
  const long long climit = (long long)(limit_ns * 2ull);
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((it & 63u) == 0u) {
      if (honour_abort && *abort_flag) return false;
      if (clock64() - c0 > climit) {
        *abort_flag = 1u;
        atomicCAS(&g_basa_where, 0u, site);
        atomicOr(&g_basa_status, 1u);
        return false;
      }
    }
  }
}
__device__ __forceinline__ bool wait_warp_cluster(uint32_t bar, uint32_t parity,
                                                  volatile uint32_t* abort_flag,
                                                  uint64_t limit_ns, uint32_t site,
                                                  bool honour_abort = true) {
  bool ok = mbar_try_wait_cluster(bar, parity);
  if (!ok) ok = wait_slow_cluster(bar, parity, abort_flag, limit_ns, site, honour_abort);
  return __all_sync(0xffffffffu, ok);
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t slot_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// D (+)= A B over the CTA pair: A (M = 256) K-major in both shared memories.
__device__ __forceinline__ void mma_pair_ss(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
// The same with A read from both CTAs' TMEM.
__device__ __forceinline__ void mma_pair_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t b,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrives on the barrier at `bar`'s offset in both CTAs once every MMA this
// thread issued before has completed.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar), "h"((uint16_t)3)
      : "memory");
}
// Instruction descriptor of kind::f16 for the pair: bf16 A and B, fp32 D,
// A K-major, B K-major or MN-major, M = 256, N = n.
__host__ __device__ constexpr uint32_t idesc_pair(int n, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
}

// ---------------------------------------------------------------------------
struct PairUnit {
  WinAt w;
  int h, hk;
};
__device__ __forceinline__ PairUnit decode_pair_unit(const PairParams& p, uint32_t u) {
  PairUnit U;
  U.h = (int)(u % (uint32_t)p.H);
  const uint32_t r = u / (uint32_t)p.H;
  const int win = (int)(r % (uint32_t)p.n_windows);
  U.w.b = (int)(r / (uint32_t)p.n_windows);
  const int jw = win % p.nww, jh = (win / p.nww) % p.nwh, jt = win / (p.nww * p.nwh);
  U.w.cls = window_class(jt, jh, jw, p.nwt, p.nwh, p.nww, p.st, p.sh, p.sw);
  U.w.ot = jt * p.wt + p.st;
  U.w.oh = jh * p.wh + p.sh;
  U.w.ow = jw * p.ww + p.sw;
  U.hk = p.group == 1 ? U.h : U.h / p.group;
  return U;
}

// Loads head-dim halves [h0, h0 + nh) of 64-row plan tile `tile` of window w
// (its boxes through maps) to dst; half hf lands at dst + (hf - h0) * half_bytes,
// box rows at + row8 * 1024.  Signals bar with the transaction bytes.
__device__ __forceinline__ void load_plan_tile(const PlanView& pv, const CUtensorMap* maps,
                                               const WinAt& w, int tile, int head, int T,
                                               int Hg, int Wg, int h0, int nh, uint32_t half_bytes,
                                               uint32_t dst, uint32_t bar) {
  const int b0 = pv.first(w.cls, tile), nb = pv.count(w.cls, tile);
#pragma unroll 1
  for (int bi = 0; bi < nb; ++bi) {
    const uint32_t e = pv.entries[b0 + bi];
    const int sid = box_shape(e);
    const int gt = wrap(w.ot + box_lt(e), T);
    const int gh = wrap(w.oh + box_lh(e), Hg);
    const int gw = wrap(w.ow + box_lw(e), Wg);
    if constexpr (kChecked) {  // inside the grid and inside the 64-row tile
      const int bt = pv.bt[sid], bh = pv.bh[sid], bw = pv.bw[sid];
      if (sid >= kMaxShapes || gt + bt > T || gh + bh > Hg || gw + bw > Wg ||
          box_row8(e) * 8 + bt * bh * bw > 64) {
        check_failed(kCheckLoadBox);
        continue;
      }
    }
    const uint32_t d0 = dst + box_row8(e) * 1024;
#pragma unroll 1
    for (int hf = h0; hf < h0 + nh; ++hf)
      tma_load_5d(d0 + (hf - h0) * half_bytes, &maps[sid], bar, hf * 64, head, gw, gh,
                  w.b * T + gt);
  }
}

__global__ void __launch_bounds__(kPairThreads, 1)
    tc_attn_pair_kernel(const __grid_constant__ PairParams p) {
  using S = PairSmem;
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
  const uint32_t rank = cluster_rank();    // = query tile of the unit
  const bool leader = rank == 0;
  const uint32_t cid = cluster_id(), ncl = cluster_count();

  const PlanView pv = plan_to_smem(p.plan, smem + S::plan, 4, threadIdx.x, kPairThreads);
  if (threadIdx.x == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(BAR(S::QKF + x), 1);
      mbar_init(BAR(S::VF + x), 1);
      mbar_init(BAR(S::QKE + x), 1);
      mbar_init(BAR(S::VE + x), 1);
      mbar_init(BAR(S::PQK + x), 1);
      mbar_init(BAR(S::PVF + x), 1);
      mbar_init(BAR(S::PF + x), 8);
      mbar_init(BAR(S::OF + x), 1);
      mbar_init(BAR(S::OR + x), 8);
    }
    mbar_init(BAR(S::SF), 1);
    mbar_init(BAR(S::DRAIN), 1);
    *abort_flag = 0u;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers and TMEM exist before any cross-CTA use
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) {
    for (int sid = 0; sid < p.n_shapes; ++sid) {
      prefetch_tmap(&p.qm[sid]); prefetch_tmap(&p.km[sid]); prefetch_tmap(&p.vm[sid]);
    }
  }
  const bool withhold = (p.flags & BASA_FLAG_TEST_WITHHOLD_LOADS) != 0;

  if (warp == 0) {
    // ------------------------------------------------------------ loader
    if (!withhold) {
      uint32_t n = 0, nqk = 0, nv = 0;  // units walked; Q+K and V loads issued
      bool ok = true;
      for (uint32_t u = cid; u < p.n_units && ok; u += ncl, ++n) {
        const PairUnit U = decode_pair_unit(p, u);
        const uint32_t x = n & 1u, par = ((n >> 1) & 1u) ^ 1u;
        // Q (plan tiles 2 rank, 2 rank + 1) and this CTA's K rows of both key tiles
        if (!(ok = wait_warp(BAR(S::QKE + x), par, abort_flag, limit, kPSiteLoadEmpty))) break;
        if (lane == 0) {
          const uint32_t bar = BAR(S::QKF + x);
          mbar_expect_tx(bar, kQB + 2 * kKB);
          const uint32_t q = sbase + S::q0 + x * kQB;
          for (int t = 0; t < 2; ++t)
            load_plan_tile(pv, p.qm, U.w, 2 * (int)rank + t, U.h, p.T, p.Hg, p.Wg, 0, 2, kHalf,
                           q + t * 64 * 128, bar);
          for (int j = 0; j < 2; ++j)
            load_plan_tile(pv, p.km, U.w, 2 * j + (int)rank, U.hk, p.T, p.Hg, p.Wg, 0, 2, kKHalfB,
                           sbase + S::k0 + (2 * x + j) * kKB, bar);
        }
        __syncwarp();
        ++nqk;
        // this CTA's head-dim half of V for both key tiles (all 128 keys each)
        if (!(ok = wait_warp(BAR(S::VE + x), par, abort_flag, limit, kPSiteLoadEmpty))) break;
        if (lane == 0) {
          const uint32_t bar = BAR(S::VF + x);
          mbar_expect_tx(bar, 2 * kVB);
          for (int j = 0; j < 2; ++j)
            for (int t = 0; t < 2; ++t)
              load_plan_tile(pv, p.vm, U.w, 2 * j + t, U.hk, p.T, p.Hg, p.Wg, (int)rank, 1, 0,
                             sbase + S::v0 + (2 * x + j) * kVB + t * 64 * 128, bar);
        }
        __syncwarp();
        ++nv;
      }
      // Drain: the last loads issued into each slot have landed (bounded,
      // regardless of an abort).
      for (uint32_t k = nqk > 2 ? nqk - 2 : 0; k < nqk; ++k)
        wait_warp(BAR(S::QKF + (k & 1u)), (k >> 1) & 1u, abort_flag, limit, kPSiteLoadDrain,
                  false);
      for (uint32_t k = nv > 2 ? nv - 2 : 0; k < nv; ++k)
        wait_warp(BAR(S::VF + (k & 1u)), (k >> 1) & 1u, abort_flag, limit, kPSiteLoadDrain, false);
    }
  } else if (warp == 3 && !leader) {
    // ------------------------------------------------------------ forwarder
    // Tells the leader (whose MMAs read this CTA's shared memory) that this
    // CTA's tiles of a unit have landed.
    if (!withhold) {
      const uint32_t pqk = peer_addr(BAR(S::PQK), 0), pvf = peer_addr(BAR(S::PVF), 0);
      uint32_t n = 0;
      bool ok = true;
      for (uint32_t u = cid; u < p.n_units && ok; u += ncl, ++n) {
        const uint32_t x = n & 1u, par = (n >> 1) & 1u;
        if (!(ok = wait_warp_cluster(BAR(S::QKF + x), par, abort_flag, limit, kPSiteFwd))) break;
        if (lane == 0) mbar_arrive_cluster(pqk + 8u * x);
        __syncwarp();
        if (!(ok = wait_warp_cluster(BAR(S::VF + x), par, abort_flag, limit, kPSiteFwd))) break;
        if (lane == 0) mbar_arrive_cluster(pvf + 8u * x);
        __syncwarp();
      }
    }
  } else if (warp == 1 && leader) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t IDS = idesc_pair(128, false);  // S = Q K^T: N = 128 keys
    constexpr uint32_t IDO = idesc_pair(128, true);   // O = P V: N = 128 head-dim columns
    uint32_t n = 0;
    bool ok = true;
    for (uint32_t u = cid; u < p.n_units && ok; u += ncl, ++n) {
      const uint32_t x = n & 1u, par = (n >> 1) & 1u;
      if (!(ok = wait_warp(BAR(S::QKF + x), par, abort_flag, limit, kPSiteMmaFull))) break;
      if (!(ok = wait_warp_cluster(BAR(S::PQK + x), par, abort_flag, limit, kPSiteMmaPeer)))
        break;
      tc_fence_after();
      if (lane == 0) {
        // S_j = Q K_j^T into columns [128 j, 128 j + 128), 16 head-dim values per step
        const uint32_t qa = sbase + S::q0 + x * kQB;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const uint32_t ka = sbase + S::k0 + (2 * x + j) * kKB;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mma_pair_ss(tmem + 128 * j,
                        sdesc(qa + (k / 4) * kHalf + (k % 4) * 32, 16, 1024),
                        sdesc(ka + (k / 4) * kKHalfB + (k % 4) * 32, 16, 1024), IDS,
                        k > 0 ? 1u : 0u);
        }
        mma_commit_pair(BAR(S::SF));
        mma_commit_pair(BAR(S::QKE + x));
      }
      __syncwarp();
      if (!(ok = wait_warp(BAR(S::VF + x), par, abort_flag, limit, kPSiteMmaFull))) break;
      if (!(ok = wait_warp_cluster(BAR(S::PVF + x), par, abort_flag, limit, kPSiteMmaPeer)))
        break;
      // O_x was last read by the epilogue of unit n - 2
      if (n >= 2 && !(ok = wait_warp_cluster(BAR(S::OR + x), ((n - 2) >> 1) & 1u, abort_flag,
                                             limit, kPSiteMmaOFree)))
        break;
#pragma unroll 1
      for (int j = 0; j < 2 && ok; ++j) {
        if (!(ok = wait_warp_cluster(BAR(S::PF + j), n & 1u, abort_flag, limit, kPSiteMmaP)))
          break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t va = sbase + S::v0 + (2 * x + j) * kVB;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mma_pair_ts(tmem + 256 + 128 * x, tmem + 128 * j + 8 * k,
                        sdesc(va + k * 2048, kHalf, 1024), IDO, (j > 0 || k > 0) ? 1u : 0u);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) {
        mma_commit_pair(BAR(S::OF + x));
        mma_commit_pair(BAR(S::VE + x));
      }
      __syncwarp();
    }
    // Drain: every MMA issued has completed before TMEM is released.
    if (lane == 0) mma_commit_pair(BAR(S::DRAIN));
    __syncwarp();
    wait_warp(BAR(S::DRAIN), 0u, abort_flag, limit, kPSiteMmaDrain, false);
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax + epilogue
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;  // query row of this CTA's tile
    const uint32_t tl = (uint32_t)(q4 * 32) << 16;
    const uint32_t wst = sbase + S::stg0 + (uint32_t)(warp - 4) * 4096u;
    // barriers of the leader that this warp arrives on (lane 0)
    const uint32_t pf = leader ? BAR(S::PF) : peer_addr(BAR(S::PF), 0);
    const uint32_t orl = leader ? BAR(S::OR) : peer_addr(BAR(S::OR), 0);
    auto arrive_leader = [&](uint32_t addr) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          mbar_arrive(addr);
        else
          mbar_arrive_cluster(addr);
      }
      __syncwarp();
    };
    const float c = p.scale_log2;
    const uint64_t c2 = f2pack(c, c);
    uint32_t n = 0;
    bool ok = true;
    for (uint32_t u = cid; u < p.n_units && ok; u += ncl, ++n) {
      const PairUnit U = decode_pair_unit(p, u);
      const uint32_t x = n & 1u;
      if (!(ok = wait_warp(BAR(S::SF), n & 1u, abort_flag, limit, kPSiteSmxS))) break;
      tc_fence_after();
      // exact row max over both key tiles
      uint32_t s[4][32];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) tmem_ld32(tmem + tl + 128 + cc * 32, s[cc]);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) tmem_wait_ld(s[cc]);
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc)
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          mx0 = max3(mx0, __uint_as_float(s[cc][e]), __uint_as_float(s[cc][e + 1]));
          mx1 = max3(mx1, __uint_as_float(s[cc][e + 2]), __uint_as_float(s[cc][e + 3]));
        }
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) tmem_ld32(tmem + tl + cc * 32, s[cc]);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) tmem_wait_ld(s[cc]);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc)
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          mx0 = max3(mx0, __uint_as_float(s[cc][e]), __uint_as_float(s[cc][e + 1]));
          mx1 = max3(mx1, __uint_as_float(s[cc][e + 2]), __uint_as_float(s[cc][e + 3]));
        }
      const float m = fmaxf(mx0, mx1) * c;
      const uint64_t nm2 = f2pack(-m, -m);
      float l = 0.f;
      // P_j = 2^(s c - m) as bf16 pairs over the first 64 columns of S_j
#pragma unroll 1
      for (int j = 0; j < 2; ++j) {
        if (j == 1) {
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) tmem_ld32(tmem + tl + 128 + cc * 32, s[cc]);
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) tmem_wait_ld(s[cc]);
        }
        uint64_t rsa = f2pack(0.f, 0.f), rsb = rsa;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t pk[16];
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
          tmem_st16(tmem + tl + 128 * j + cc * 16, pk);
        }
        float ra0, ra1, rb0, rb1;
        f2unpack(rsa, ra0, ra1);
        f2unpack(rsb, rb0, rb1);
        l += (ra0 + ra1) + (rb0 + rb1);
        tmem_wait_st();
        arrive_leader(pf + 8u * j);
      }
      // epilogue: O_x / l -> bf16 -> warp-staged 16-byte stores of whole 128-byte segments
      if (!(ok = wait_warp(BAR(S::OF + x), (n >> 1) & 1u, abort_flag, limit, kPSiteSmxO))) break;
      tc_fence_after();
      uint32_t o[4][32];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) tmem_ld32(tmem + tl + 256 + 128 * x + cc * 32, o[cc]);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) tmem_wait_ld(o[cc]);
      arrive_leader(orl + 8u * x);  // O_x read: the unit after next may overwrite it
      const float inv = 1.0f / l;
      const uint64_t inv2 = f2pack(inv, inv);
      // rows 0..63 come from plan tile 2 rank, rows 64..127 from 2 rank + 1
      const int tile = 2 * (int)rank + (r >> 6);
      const long long tok = window_row_token(pv, U.w, tile, r & 63, p.T, p.Hg, p.Wg);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t w[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          float o0, o1;
          f2unpack(f2mul(f2pack(__uint_as_float(o[2 * hf + e / 16][(2 * e) % 32]),
                                __uint_as_float(o[2 * hf + e / 16][(2 * e) % 32 + 1])), inv2),
                   o0, o1);
          w[e] = pack_bf16(o0, o1);
        }
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
          st_shared_v4(wst + lane * 128 + ((ch ^ (lane & 7)) << 4), w[4 * ch], w[4 * ch + 1],
                       w[4 * ch + 2], w[4 * ch + 3]);
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int rr = k * 4 + lane / 8, cc = lane % 8;
          const uint4 val = ld_shared_v4(wst + rr * 128 + ((cc ^ (rr & 7)) << 4));
          const long long t = __shfl_sync(0xffffffffu, tok, rr);
          if (t >= 0) {
            if (kChecked && t >= p.N)
              check_failed(kCheckOutRow);
            else
              *reinterpret_cast<uint4*>(p.out + (((long long)U.w.b * p.N + t) * p.H + U.h) * 128 +
                                        hf * 64 + cc * 8) = val;
          }
        }
        __syncwarp();
      }
      if (p.lse && tok >= 0) {
        if (kChecked && tok >= p.N)
          check_failed(kCheckLseRow);
        else
          p.lse[((long long)U.w.b * p.H + U.h) * p.N + tok] = (m + __log2f(l)) * 0.69314718055994531f;
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync();  // neither CTA leaves while the other may still use its memory
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace

// Windows the CTA-pair kernel takes: bf16, d = 128, no extra keys, no padded
// grid, and a 256-token window whose 64-row tile plan has four full tiles.
bool pair_kernel_applies(const Dims& d, bool extra_keys, TilePlan* plan64) {
  if (d.dtype != BASA_BF16 || d.d != 128 || extra_keys || d.padded) return false;
  if ((long long)d.wt * d.wh * d.ww != 256) return false;
  if (build_tile_plan(d, plan64, 64) != BASA_OK || plan64->n_tiles != 4) return false;
  for (int t = 0; t < 4; ++t)
    if (plan64->tile_rows[t] != 64) return false;
  return true;
}

namespace {

// Fills *prm (zeroed by the caller) and launches the pair kernel.
basa_status pair_build_and_launch(PairParams* prm, const Dims& d, const TilePlan& plan,
                                  const void* q, const void* k, const void* v, void* out,
                                  float* lse, uint32_t flags, uint32_t timeout_ms,
                                  cudaStream_t stream) {
  basa_status st = BASA_OK;
  const uint64_t D = 128, H = (uint64_t)d.H, Hk = (uint64_t)d.Hkv;
  prm->B = d.B; prm->H = d.H; prm->T = d.T; prm->Hg = d.Hg; prm->Wg = d.Wg;
  prm->group = d.H / d.Hkv;
  prm->wt = d.wt; prm->wh = d.wh; prm->ww = d.ww;
  prm->st = d.st; prm->sh = d.sh; prm->sw = d.sw;
  prm->nwt = d.nwt; prm->nwh = d.nwh; prm->nww = d.nww;
  prm->N = d.N;
  prm->lse = lse;
  prm->out = static_cast<__nv_bfloat16*>(out);
  prm->flags = flags;
  prm->timeout_ns = (unsigned long long)(timeout_ms ? timeout_ms : 2000u) * 1000000ull;
  prm->scale_log2 = d.scale * 1.4426950408889634f;
  prm->n_windows = d.nwt * d.nwh * d.nww;
  prm->n_shapes = plan.n_shapes;
  const long long units = (long long)d.B * d.H * prm->n_windows;
  if (units > 0x7fffffffLL) st = BASA_ERR_UNSUPPORTED;
  if (st == BASA_OK) st = pack_plan_image(plan, &prm->plan);
  if (st == BASA_OK) {
    prm->n_units = (uint32_t)units;
    const uint64_t dims[5] = {D, H, (uint64_t)d.Wg, (uint64_t)d.Hg, (uint64_t)d.B * d.T};
    const uint64_t strides[4] = {D * 2, H * D * 2, (uint64_t)d.Wg * H * D * 2,
                                 (uint64_t)d.Hg * d.Wg * H * D * 2};
    const uint64_t kdims[5] = {D, Hk, (uint64_t)d.Wg, (uint64_t)d.Hg, (uint64_t)d.B * d.T};
    const uint64_t kstrides[4] = {D * 2, Hk * D * 2, (uint64_t)d.Wg * Hk * D * 2,
                                  (uint64_t)d.Hg * d.Wg * Hk * D * 2};
    for (int s = 0; s < plan.n_shapes && st == BASA_OK; ++s) {
      const uint32_t box[5] = {64, 1, plan.shape_bw[s], plan.shape_bh[s], plan.shape_bt[s]};
      if ((st = encode_map(&prm->qm[s], q, 5, dims, strides, box)) != BASA_OK) break;
      if ((st = encode_map(&prm->km[s], k, 5, kdims, kstrides, box)) != BASA_OK) break;
      st = encode_map(&prm->vm[s], v, 5, kdims, kstrides, box);
    }
  }
  if (st == BASA_OK) {
    const int smem = PairSmem::alloc;
    static_assert(PairSmem::alloc <= 232448, "shared memory plan exceeds 227 KB");
    if (cudaFuncSetAttribute(tc_attn_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess) {
      st = BASA_ERR_CUDA;
    } else {
      cudaLaunchConfig_t cfg = {};
      cfg.blockDim = dim3(kPairThreads);
      cfg.dynamicSmemBytes = (size_t)smem;
      cfg.stream = stream;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      // as many clusters as can be resident at once (each walks units)
      cfg.gridDim = dim3((unsigned)(2 * tc_sm_count()));
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, tc_attn_pair_kernel, &cfg) != cudaSuccess ||
          clusters < 1)
        clusters = tc_sm_count() / 2;
      if ((long long)clusters > units) clusters = (int)units;
      cfg.gridDim = dim3((unsigned)(2 * clusters));
      if (cudaLaunchKernelEx(&cfg, tc_attn_pair_kernel, *prm) != cudaSuccess ||
          cudaGetLastError() != cudaSuccess)
        st = BASA_ERR_CUDA;
    }
  }
  return st;
}

// Parameter block of the entry points that allocate nothing (see basa_tc.cu).
PairParams g_pair_static_params;
std::mutex g_pair_static_mu;

}  // namespace

basa_status launch_tc_pair(const Dims& d, const TilePlan& plan, const void* q, const void* k,
                           const void* v, void* out, float* lse, uint32_t flags,
                           uint32_t timeout_ms, cudaStream_t stream, bool static_params) {
  if (static_params) {
    std::lock_guard<std::mutex> lock(g_pair_static_mu);
    memset(&g_pair_static_params, 0, sizeof(g_pair_static_params));
    return pair_build_and_launch(&g_pair_static_params, d, plan, q, k, v, out, lse, flags,
                                 timeout_ms, stream);
  }
  PairParams* prm = new (std::nothrow) PairParams;
  if (!prm) return BASA_ERR_INVALID_ARG;
  memset(prm, 0, sizeof(*prm));
  const basa_status st =
      pair_build_and_launch(prm, d, plan, q, k, v, out, lse, flags, timeout_ms, stream);
  delete prm;
  return st;
}

cudaError_t take_pair_status(cudaStream_t stream, unsigned int* status, unsigned int* where) {
  return tc_take_status(stream, status, where);
}

}  // namespace basa
