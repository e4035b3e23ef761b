// Device helpers shared by the tcgen05 kernels of the library: PTX wrappers for
// mbarriers, TMA (cp.async.bulk.tensor), TMEM allocation and access, tcgen05.mma
// of kind::f16 with shared-memory descriptors, packed fp32x2 arithmetic, the
// bounded mbarrier waits, and the view of the compact tile plan in shared
// memory.  Everything here has internal linkage: each translation unit that
// includes this header gets its own copy, including its own device status word
// (the library is built without relocatable device code), which
// tc_take_status() reads and clears from the host.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <math.h>

#include "basa_internal.h"

namespace basa {
namespace {

__device__ unsigned int g_basa_status;  // bit 0: a device wait timed out
__device__ unsigned int g_basa_where;   // site of the first wait that gave up

constexpr int kHalf = 128 * 128;  // bytes of one 64-wide head-dim half of a 128-row tile

// Division by a launch constant d >= 1 without the integer-divide sequence
// (Granlund and Montgomery, "Division by Invariant Integers using
// Multiplication", PLDI 1994): with l = ceil(log2 d) and the 33-bit multiplier
// 2^32 + m = ceil(2^(32 + l) / d), n / d = (umulhi(n, m) + n) >> l for every
// 32-bit n.  d < 1 is taken as 1.
struct FastDiv {
  uint32_t d, m, l;
  FastDiv() = default;
  explicit FastDiv(int dv) {
    d = dv > 1 ? (uint32_t)dv : 1u;
    l = 0;
    while ((1ull << l) < d) ++l;
    m = (uint32_t)(((1ull << 32) * ((1ull << l) - d)) / d + 1);
  }
  __device__ __forceinline__ uint32_t div(uint32_t n) const {
    return (uint32_t)(((uint64_t)__umulhi(n, m) + n) >> l);
  }
};

// Checked build (compiled with BASA_CHECKED): the kernels verify every TMA box
// and every output index against their tensors before the access; a failed
// check skips the access, sets bit 1 of the device status word and records its
// site (codes from 200).  A skipped load leaves its barrier short, so the
// consumer's bounded wait then ends the kernel cleanly as well.
#ifdef BASA_CHECKED
constexpr bool kChecked = true;
#else
constexpr bool kChecked = false;
#endif
enum CheckSite : uint32_t {
  kCheckLoadBox = 200, kCheckStoreBox, kCheckOutRow, kCheckLseRow, kCheckGradRow, kCheckPooledRow
};
__device__ __noinline__ void check_failed(uint32_t site) {
  atomicCAS(&g_basa_where, 0u, site);
  atomicOr(&g_basa_status, 2u);
}

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
      : "memory");
}
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
__device__ __forceinline__ void tma_store_5d(const CUtensorMap* map, uint32_t src, int c0, int c1,
                                             int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.global.shared::cta.tile.bulk_group"
      " [%0, {%2, %3, %4, %5, %6}], [%1];" ::"l"(reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
      : "memory");
}
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, uint32_t src, int c0, int c1,
                                             int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group"
      " [%0, {%2, %3, %4, %5}], [%1];" ::"l"(reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
// Programmatic dependent launch: waits until the grid this one was launched
// as a dependent of has completed and its writes are visible (returns at once
// for a grid launched without that dependency).
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all0() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t slot_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 layout: start
// address >> 4 in bits 0-13, leading byte offset >> 4 in 16-29, stride byte
// offset >> 4 in 32-45, descriptor version 1 in 46-47, swizzle mode 2 in 61-63).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor of kind::f16: bf16 A and B, fp32 accumulator, A K-major,
// B K-major or MN-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc_bf16(int n, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}
__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
// The same with the A operand (M x K, K-major) read from TMEM: two 16-bit
// elements per 32-bit column, lower half first.
__device__ __forceinline__ void mma_bf16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t b,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Instruction descriptor of kind::f8f6f4 with e4m3 A and B (format code 0),
// fp32 accumulator, both K-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc_e4m3(int n) {
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}
// D (+)= A B^T with A, B e4m3 in shared memory (K = 32 per instruction).
__device__ __forceinline__ void mma_e4m3(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

#define TMEM_REGS32(r)                                                                         \
  "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),         \
      "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), \
      "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),           \
      "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),           \
      "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
#define TMEM_INREGS32(r)                                                                          \
  "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),         \
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),          \
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),        \
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),        \
      "r"(r[29]), "r"(r[30]), "r"(r[31])
#define TMEM_RWREGS32(r)                                                                         \
  "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),           \
      "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),   \
      "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),             \
      "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]),             \
      "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])

// 32 consecutive fp32 columns of this thread's TMEM lane; the values are valid
// only after tmem_wait_ld, which takes them as operands so that no use can be
// scheduled before it.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : TMEM_REGS32(r)
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" : TMEM_RWREGS32(r)::"memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31, %32};" ::"r"(taddr),
      TMEM_INREGS32(r)
      : "memory");
}
// 16 consecutive 32-bit columns of this thread's lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
// Packed pairs of fp32 (f32x2 arithmetic of sm_100).
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
  uint64_t d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}
// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` inside a 128-byte
// swizzled, 1024-byte-aligned block of rows.
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// ---------------------------------------------------------------------------
// Bounded waits.  `abort_flag` lives in shared memory; any role that gives up
// raises it so that the others leave their loops promptly.  The poll loop is
// tight (try_wait itself sleeps until the phase completes or a short hardware
// limit passes); the abort flag and the bound, in SM cycles (2 per ns of the
// limit, so at least the limit at clocks up to 2 GHz), are checked every 64
// polls.  The first wait that gives up records its site in g_basa_where.
// ---------------------------------------------------------------------------

__device__ __noinline__ bool wait_slow(uint32_t bar, uint32_t parity,
                                       volatile uint32_t* abort_flag, uint64_t limit_ns,
                                       uint32_t site, bool honour_abort) {
  const long long c0 = clock64();
  const long long climit = (long long)(limit_ns * 2ull);
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
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
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity,
                                             volatile uint32_t* abort_flag, uint64_t limit_ns,
                                             uint32_t site, bool honour_abort = true) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_slow(bar, parity, abort_flag, limit_ns, site, honour_abort);
}
// Warp-uniform variant: every lane waits, and the warp proceeds only if all did.
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity,
                                          volatile uint32_t* abort_flag, uint64_t limit_ns,
                                          uint32_t site, bool honour_abort = true) {
  const bool ok = wait_bounded(bar, parity, abort_flag, limit_ns, site, honour_abort);
  return __all_sync(0xffffffffu, ok);
}

// The tile plan as seen from shared memory.  Image layout (bytes): per (class,
// tile) a 16-bit word (first box << 4 | box count); per tile its valid rows;
// per box shape its t, row and column extents; then the packed box entries.
struct PlanView {
  const uint16_t* idx;
  const uint8_t* rows;
  const uint8_t* bt;
  const uint8_t* bh;
  const uint8_t* bw;
  const uint32_t* entries;
  int n_tiles;
  __device__ __forceinline__ int first(int cls, int tile) const { return idx[cls * n_tiles + tile] >> 4; }
  __device__ __forceinline__ int count(int cls, int tile) const { return idx[cls * n_tiles + tile] & 15; }
};

// x mod G for 0 <= x < 2G: a window origin (below G) plus an offset inside the
// window (below w <= G).
__device__ __forceinline__ int wrap(int x, int G) { return x >= G ? x - G : x; }

// ---------------------------------------------------------------------------
// The compact tile plan.  The host packs the plan of build_tile_plan into an
// image that travels in the kernel's parameter block; each CTA copies it into
// shared memory.  Image layout (bytes): per (class, tile) a 16-bit word (first
// box << 4 | box count); per tile its valid rows; per box shape its t, row and
// column extents; then the packed 32-bit box entries.
// ---------------------------------------------------------------------------
constexpr int kPlanBytes = 1536;  // shared-memory room for the compact tile plan
constexpr int kPlanWords = kPlanBytes / 4;

struct PlanImage {
  uint32_t words[kPlanWords];
  int n_words;
  int off_rows, off_bt, off_bh, off_bw, off_entries;  // byte offsets inside words
};

inline basa_status pack_plan_image(const TilePlan& plan, PlanImage* out) {
  const int T = plan.n_tiles, NSh = plan.n_shapes;
  uint8_t* img = reinterpret_cast<uint8_t*>(out->words);
  const int off_rows = 2 * kClasses * T;
  const int off_bt = off_rows + T, off_bh = off_bt + NSh, off_bw = off_bh + NSh;
  const int off_entries = (off_bw + NSh + 3) & ~3;
  int n = 0;
  for (int c = 0; c < kClasses; ++c)
    for (int t = 0; t < T; ++t) n += plan.nbox[c][t];
  const int total = off_entries + 4 * n;
  if (total > kPlanBytes || n >= 4096) return BASA_ERR_UNSUPPORTED;
  uint16_t* idx = reinterpret_cast<uint16_t*>(img);
  uint32_t* entries = reinterpret_cast<uint32_t*>(img + off_entries);
  int e = 0;
  for (int c = 0; c < kClasses; ++c)
    for (int t = 0; t < T; ++t) {
      idx[c * T + t] = (uint16_t)((e << 4) | plan.nbox[c][t]);
      for (int b = 0; b < plan.nbox[c][t]; ++b) entries[e++] = plan.box[c][t][b];
    }
  for (int t = 0; t < T; ++t) img[off_rows + t] = plan.tile_rows[t];
  for (int s2 = 0; s2 < NSh; ++s2) {
    img[off_bt + s2] = plan.shape_bt[s2];
    img[off_bh + s2] = plan.shape_bh[s2];
    img[off_bw + s2] = plan.shape_bw[s2];
  }
  out->n_words = (total + 3) / 4;
  out->off_rows = off_rows;
  out->off_bt = off_bt;
  out->off_bh = off_bh;
  out->off_bw = off_bw;
  out->off_entries = off_entries;
  return BASA_OK;
}

// Copies the image into shared memory (all threads of the CTA take part) and
// returns its view; the caller synchronises the CTA before the first use.
__device__ __forceinline__ PlanView plan_to_smem(const PlanImage& im, uint8_t* dst, int n_tiles,
                                                 int tid, int nthreads) {
  uint32_t* d32 = reinterpret_cast<uint32_t*>(dst);
  for (int w = tid; w < im.n_words; w += nthreads) d32[w] = im.words[w];
  PlanView pv;
  pv.idx = reinterpret_cast<const uint16_t*>(dst);
  pv.rows = dst + im.off_rows;
  pv.bt = dst + im.off_bt;
  pv.bh = dst + im.off_bh;
  pv.bw = dst + im.off_bw;
  pv.entries = reinterpret_cast<const uint32_t*>(dst + im.off_entries);
  pv.n_tiles = n_tiles;
  return pv;
}

// Position of one window: its wrap class, its origin on the grid (window index
// times window size plus the shift, below the grid size) and its batch.
struct WinAt {
  int cls, ot, oh, ow, b;
};

// Loads tile `tile` of window w for one head: each box of the plan through
// maps[box shape] (rank 5: [d, heads, Wg, Hg, B*T]; NH head-dim halves of 64),
// then the rows past the tile's tokens as zeros, read out of bounds through
// `fill` (8-row boxes).  Signals bar with the transaction bytes.  Tp, Hgp, Wgp
// are the padded extents the window origins wrap on (the grid's own unless it
// is padded); rows at padded positions read zeros (rows, columns: out of the
// map's bounds) or another frame (t: the map merges B and T) and are masked by
// the caller.
template <int NH>
__device__ __forceinline__ void load_window_tile(const PlanView& pv, const CUtensorMap* maps,
                                                 const CUtensorMap* fill, const WinAt& w,
                                                 int tile, int head, int T, int Tp, int Hgp,
                                                 int Wgp, long long N, uint32_t dst,
                                                 uint32_t bar) {
  const int b0 = pv.first(w.cls, tile), nb = pv.count(w.cls, tile);
#pragma unroll 1
  for (int bi = 0; bi < nb; ++bi) {
    const uint32_t e = pv.entries[b0 + bi];
    const int sid = box_shape(e);
    const int gt = wrap(w.ot + box_lt(e), Tp);
    const int gh = wrap(w.oh + box_lh(e), Hgp);
    const int gw = wrap(w.ow + box_lw(e), Wgp);
    if constexpr (kChecked) {  // the box lies inside the padded grid and the 128-row tile
      const int bt = pv.bt[sid], bh = pv.bh[sid], bw = pv.bw[sid];
      if (sid >= kMaxShapes || gt < 0 || gh < 0 || gw < 0 || gt + bt > Tp || gh + bh > Hgp ||
          gw + bw > Wgp || box_row8(e) * 8 + bt * bh * bw > 128) {
        check_failed(kCheckLoadBox);
        continue;
      }
    }
    const uint32_t d0 = dst + box_row8(e) * 1024;
#pragma unroll
    for (int hf = 0; hf < NH; ++hf)
      tma_load_5d(d0 + hf * kHalf, &maps[sid], bar, hf * 64, head, gw, gh, w.b * T + gt);
  }
#pragma unroll 1
  for (int r = pv.rows[tile]; r < 128; r += 8) {
#pragma unroll
    for (int hf = 0; hf < NH; ++hf)
      tma_load_4d(dst + hf * kHalf + r * 128, fill, bar, hf * 64, 0, (int)N, 0);
  }
}
template <int NH>
__device__ __forceinline__ void load_window_tile(const PlanView& pv, const CUtensorMap* maps,
                                                 const CUtensorMap* fill, const WinAt& w,
                                                 int tile, int head, int T, int Hg, int Wg,
                                                 long long N, uint32_t dst, uint32_t bar) {
  load_window_tile<NH>(pv, maps, fill, w, tile, head, T, T, Hg, Wg, N, dst, bar);
}

// Flattened grid index of the token in row r of tile `tile` of window w, or -1
// for a row past the tile's tokens or at a padded position (a coordinate at or
// past the grid's extent T, Hg, Wg; origins wrap on the padded Tp, Hgp, Wgp).
__device__ __forceinline__ long long window_row_token(const PlanView& pv, const WinAt& w,
                                                      int tile, int r, int Tp, int Hgp, int Wgp,
                                                      int T, int Hg, int Wg) {
  const int b0 = pv.first(w.cls, tile), nb = pv.count(w.cls, tile);
#pragma unroll 1
  for (int bi = 0; bi < nb; ++bi) {
    const uint32_t e = pv.entries[b0 + bi];
    const int sid = box_shape(e);
    const int bt = pv.bt[sid], bh = pv.bh[sid], bw = pv.bw[sid];
    const int r0 = box_row8(e) * 8;
    if (r >= r0 && r < r0 + bt * bh * bw) {
      const int idx = r - r0;
      const int it = idx / (bh * bw), ih = (idx / bw) % bh, iw = idx % bw;
      const int gt = wrap(w.ot + box_lt(e), Tp) + it;
      const int gh = wrap(w.oh + box_lh(e), Hgp) + ih;
      const int gw = wrap(w.ow + box_lw(e), Wgp) + iw;
      if (gt >= T || gh >= Hg || gw >= Wg) return -1;
      return ((long long)gt * Hg + gh) * Wg + gw;
    }
  }
  return -1;
}
__device__ __forceinline__ long long window_row_token(const PlanView& pv, const WinAt& w,
                                                      int tile, int r, int T, int Hg, int Wg) {
  return window_row_token(pv, w, tile, r, T, Hg, Wg, T, Hg, Wg);
}

// SMs of the current device (the persistent grids launch one CTA per SM).
inline int tc_sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 1;
}

// CTAs of a persistent grid over `units` work units.  Up to `max_rounds`
// units per CTA: as few CTAs as keep the number of units per CTA at its
// minimum, ceil(units / SMs), so that every CTA walks the same number of units
// (384 units on 148 SMs: 128 CTAs of 3 units, not 88 CTAs of 3 and 60 of 2).
// Beyond that, one CTA per SM: with many units per CTA the uneven last round
// costs less than the bandwidth of the SMs a balanced grid leaves idle.
inline long long persistent_grid(long long units, long long max_rounds = 1LL << 40) {
  const long long sms = tc_sm_count();
  if (units <= 0) return 1;
  const long long rounds = (units + sms - 1) / sms;
  if (rounds > max_rounds) return units < sms ? units : sms;
  return (units + rounds - 1) / rounds;
}

// Reads this translation unit's device status word after synchronising the
// stream; returns the status bits and the first give-up site and clears both.
inline cudaError_t tc_take_status(cudaStream_t stream, unsigned int* status, unsigned int* where) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  *status = 0;
  *where = 0;
  if ((e = cudaMemcpyFromSymbol(status, g_basa_status, sizeof(*status))) != cudaSuccess) return e;
  if (*status) {
    if ((e = cudaMemcpyFromSymbol(where, g_basa_where, sizeof(*where))) != cudaSuccess) return e;
    const unsigned int zero = 0;
    if ((e = cudaMemcpyToSymbol(g_basa_status, &zero, sizeof(zero))) != cudaSuccess) return e;
    if ((e = cudaMemcpyToSymbol(g_basa_where, &zero, sizeof(zero))) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace
}  // namespace basa
