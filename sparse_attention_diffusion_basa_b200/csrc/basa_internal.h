// Internal declarations shared by the host API and the kernels of the library.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <nvtx3/nvToolsExt.h>

#include "basa.h"

namespace basa {

// An NVTX range over one library call, so that profilers show each call's
// launches under its name (a pointer check when no tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// ---------------------------------------------------------------------------
// Normalised call description (after validation).
// ---------------------------------------------------------------------------
struct Dims {
  int B, H, T, Hg, Wg, d;
  int Hkv;            // K/V heads (H for plain multi-head attention)
  int wt, wh, ww;     // window
  int st, sh, sw;     // shift reduced to [0, w)
  int pt, ph, pw;     // pool cell; 0 = none
  int nwt, nwh, nww;  // windows per axis (of the padded axes)
  int Tp, Hgp, Wgp;   // padded extents: nw * w (the grid itself unless it is padded)
  int padded;         // 1: some axis is padded (BASA_FLAG_PAD_GRID and w does not divide G)
  long long N;        // tokens per (b, h)
  long long P;        // extra (pooled or text) key tokens per (b, h); 0 = none
  long long Nq;       // query tokens per (b, h): N, or the text length for text queries
  int qsep;           // 1: queries are separate rows [B, Nq, H, d] (text queries)
  float scale;
  int dtype;
  float qk_descale;   // e4m3: q_descale * k_descale (1 otherwise), folded into the logit scale
  float v_descale;    // e4m3: applied to the output (1 otherwise)
};

// Validates p and fills d.  `full` = one window covering the grid, no shift,
// no pool (full attention).  allow_fp8: the entry point takes e4m3 inputs
// (otherwise BASA_FP8_E4M3 is BASA_ERR_UNSUPPORTED).
basa_status normalise(const basa_params* p, bool full, Dims* d, bool allow_fp8 = false);

// ---------------------------------------------------------------------------
// Tile plan of the bf16 tensor-core kernel (shifted-window index math).
//
// A window of wt x wh x ww tokens is cut into local boxes ("tiles") of whole
// window rows: rows of width ww, grouped into chunks of at most 128/ww rows
// along the window's row axis, and chunks of one row count stacked over t.
// Each tile holds at most 128 tokens.  When a window wraps around the grid
// border on an axis (only the last window on an axis with a non-zero shift
// does), a tile is split along that axis into the part before the border and
// the part after it; each part is one TMA box.  The wrap pattern of a window
// is its "class": bit 0 = wraps in t, bit 1 = in rows, bit 2 = in columns.
// ---------------------------------------------------------------------------
constexpr int kMaxShapes = 16;  // distinct box shapes per call
constexpr int kMaxTiles = 32;   // tiles per window
constexpr int kMaxBoxes = 8;    // boxes per tile (2 per wrapped axis)
constexpr int kClasses = 8;

// One TMA box of a tile: local start of the box inside the window, its shape id
// and its first shared-memory row / 8.  Packed in 32 bits:
// [0,8) lt  [8,16) lh  [16,24) lw  [24,28) shape  [28,32) row8.
__host__ __device__ inline uint32_t box_pack(int lt, int lh, int lw, int shape, int row8) {
  return (uint32_t)lt | ((uint32_t)lh << 8) | ((uint32_t)lw << 16) | ((uint32_t)shape << 24) |
         ((uint32_t)row8 << 28);
}
__host__ __device__ inline int box_lt(uint32_t e) { return (int)(e & 0xff); }
__host__ __device__ inline int box_lh(uint32_t e) { return (int)((e >> 8) & 0xff); }
__host__ __device__ inline int box_lw(uint32_t e) { return (int)((e >> 16) & 0xff); }
__host__ __device__ inline int box_shape(uint32_t e) { return (int)((e >> 24) & 0xf); }
__host__ __device__ inline int box_row8(uint32_t e) { return (int)(e >> 28); }

struct TilePlan {
  int n_tiles;
  int n_shapes;
  uint8_t shape_bt[kMaxShapes], shape_bh[kMaxShapes], shape_bw[kMaxShapes];
  uint8_t tile_rows[kMaxTiles];                 // valid rows of each tile (same in every class)
  uint8_t nbox[kClasses][kMaxTiles];
  uint32_t box[kClasses][kMaxTiles][kMaxBoxes];
};

// Builds the plan for window (wt, wh, ww) with shifts already reduced to [0, w).
// Returns BASA_ERR_UNSUPPORTED when the bounds of the bf16 kernel are exceeded.
basa_status build_tile_plan(const Dims& d, TilePlan* plan);

// Window class (wrap bits) of window (jt, jh, jw).
__host__ __device__ inline int window_class(int jt, int jh, int jw, int nwt, int nwh, int nww,
                                            int st, int sh, int sw) {
  return ((st != 0 && jt == nwt - 1) ? 1 : 0) | ((sh != 0 && jh == nwh - 1) ? 2 : 0) |
         ((sw != 0 && jw == nww - 1) ? 4 : 0);
}

// ---------------------------------------------------------------------------
// Launchers (defined next to their kernels).
// ---------------------------------------------------------------------------
basa_status launch_pool(const Dims& d, const void* k, const void* v, void* kp, void* vp,
                        cudaStream_t stream);

// fp32 CUDA-core window attention (window mode; full attention = one window).
basa_status launch_simt(const Dims& d, const void* q, const void* k, const void* v,
                        const void* kp, const void* vp, void* out, float* lse,
                        cudaStream_t stream);

// Split key range of a flat launch: n splits; the partial outputs (fp32
// [n, B, H, Nq, d]) and per-row (max, sum) ([n, B, H, Nq, 2]) in caller memory.
struct SplitK {
  int n;
  float* part_o;
  float* part_ml;
};

// bf16 tcgen05 window / full attention.  flat = full attention over the grid.
// sk (flat only, nullable): split the key range and combine the partials.
// after_pool: the kernel just launched on `stream` is the pooling of kp, vp;
// the attention kernel is then launched as its programmatic dependent, so
// that its start overlaps the pooling's tail (it waits for the pooling grid
// before it loads a pooled tile).
basa_status launch_tc(const Dims& d, bool flat, const void* q, const void* k, const void* v,
                      const void* kp, const void* vp, void* out, float* lse, uint32_t flags,
                      uint32_t timeout_ms, cudaStream_t stream, const SplitK* sk = nullptr,
                      bool after_pool = false);

// Splits that keep a flat launch's grid full when it has fewer than half as
// many units as SMs (1 = no split); the workspace bytes they need; the
// combine kernel (bf16 out [B, Nq, H, d], lse [B, H, Nq] nullable).
int flat_split_count(const Dims& d, bool extra_keys);
size_t flat_split_bytes(const Dims& d, int n_splits);
basa_status launch_split_combine(const Dims& d, const SplitK& sk, void* out, float* lse,
                                 cudaStream_t stream);

// Pooled global memory in the backward: the pooled K, V (as the forward used
// them, in the input dtype) and fp32 buffers for the pooled tokens' gradients,
// all [B, P, Hkv, d].
struct PoolGrads {
  const void* kp;
  const void* vp;
  float* dkp;
  float* dvp;
};

// Joint text + image backward: the text tokens' tensors ([B, L, H or Hkv, d];
// lse_t [B, H, L]) and the workspace for their D = rowsum(dout_t * out_t).
struct JointGrads {
  const void* qt;
  const void* kt;
  const void* vt;
  const void* out_t;
  const void* dout_t;
  const float* lse_t;
  float* dD_t;
  void* dqt;
  void* dkt;
  void* dvt;
  long long L;
};

// Joint backward on CUDA cores (fp32 arithmetic): D of the image and text rows,
// the text keys' gradients over every query, dQ of the image queries (window
// and text keys) and of the text queries (every key), then the image keys' dK,
// dV over their window's queries and every text query.
basa_status launch_bwd_joint(const Dims& d, const void* q, const void* k, const void* v,
                             const void* o, const void* dout, const float* lse, float* dD,
                             void* dq, void* dk, void* dv, const JointGrads& jg,
                             cudaStream_t stream);

// Backward of window attention on CUDA cores: D = rowsum(dO * O) into dD, the
// pooled tokens' gradients (pg, nullable), then dQ, then dK and dV.
basa_status launch_bwd(const Dims& d, const void* q, const void* k, const void* v,
                       const void* o, const void* dout, const float* lse, float* dD, void* dq,
                       void* dk, void* dv, const PoolGrads* pg, cudaStream_t stream);

// D = rowsum(dO * O) alone (fp32 [B, H, N] into dD).
basa_status launch_bwd_prep(const Dims& d, const void* o, const void* dout, float* dD,
                            cudaStream_t stream);

// bf16 backward on the tensor cores (d = 64 or 128, window mode): D into dD,
// then dQ, then dK and dV.  BASA_ERR_UNSUPPORTED, before any launch, when the
// shape is outside the tile plan's bounds.
basa_status launch_bwd_tc(const Dims& d, const void* q, const void* k, const void* v,
                          const void* out, const void* dout, const float* lse, float* dD,
                          void* dq, void* dk, void* dv, const PoolGrads* pg, uint32_t timeout_ms,
                          cudaStream_t stream);

// bf16 joint text + image backward on the tensor cores: D of the image rows
// into dD and of the text rows into jg.dD_t, the text keys' fp32 sums in dkp,
// dvp ([B, L, Hkv, d] each), then every gradient.  BASA_ERR_UNSUPPORTED,
// before any launch, outside the tensor-core kernels' bounds.
basa_status launch_bwd_tc_joint(const Dims& d, const void* q, const void* k, const void* v,
                                const void* out, const void* dout, const float* lse, float* dD,
                                void* dq, void* dk, void* dv, const JointGrads& jg, float* dkp,
                                float* dvp, uint32_t timeout_ms, cudaStream_t stream);

// The same launch with its parameter block in static storage (no host heap use);
// calls are serialised by a lock held until the launch has copied the block.
basa_status launch_tc_static_params(const Dims& d, bool flat, const void* q, const void* k,
                                    const void* v, const void* kp, const void* vp, void* out,
                                    float* lse, uint32_t flags, uint32_t timeout_ms,
                                    cudaStream_t stream, bool after_pool = false);

// Device status word helpers.  read_and_clear_status (basa_tc.cu) synchronises
// the stream and reads and clears the status words of every kernel file;
// take_bwd_status does that for the tensor-core backward's own word.
basa_status read_and_clear_status(cudaStream_t stream);
cudaError_t take_bwd_status(cudaStream_t stream, unsigned int* status, unsigned int* where);

// Encodes a tiled TMA map (128-byte swizzle) through the driver entry point.
basa_status encode_map(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                       const uint64_t* strides_bytes, const uint32_t* box,
                       CUtensorMapDataType type = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);

}  // namespace basa
