/*
 * basa.h — C ABI of the shifted local window attention library for NVIDIA B200
 * (sm_100a).
 *
 * The operation.  Tokens of a Diffusion Transformer lie on a 2D image or 3D video
 * latent grid.  Shifted local window attention replaces full visual
 * self-attention: the grid is cut into fixed windows, the window partition is
 * moved by a per-block shift, and each token attends only to the tokens of its
 * own shifted window ("BASA: Backend-Agnostic Sparse Attention for Fast
 * High-Resolution Diffusion Transformers", zhichai.net topic 178635722,
 * sections "Summary" and "The BASA Method").  Optionally every query also
 * attends to a small set of K/V mean-pooled "global memory" tokens (forum
 * review of the same paper, zhichai.net topic 178635722 reply 178634520, the
 * four-part method list).  Full attention, the quadratic baseline the same
 * pages compare against, is the case of one window covering the whole grid.
 *
 * Readings taken where the pages give no formula:
 *   - on each axis of size G with window w and shift s, coordinate x lies in
 *     window floor(((x - s) mod G) / w): windows wrap cyclically at the border
 *     and no extra mask is applied; s is reduced mod w;
 *   - pooled cells are non-overlapping pt x ph x pw boxes aligned to the
 *     unshifted origin; pooled K/V are plain means; window keys and pooled keys
 *     share one softmax, with no count correction;
 *   - softmax scale defaults to 1/sqrt(d).
 *
 * Layout.  q, k, v and out are dense row-major [B, T, Hg, Wg, H, d] arrays
 * (batch, time, grid rows, grid columns, heads, head dim) in device memory,
 * all of the same dtype.  A 2D grid has T = 1.  Pooled tensors are dense
 * [B, T/pt, Hg/ph, Wg/pw, H, d] arrays of the same dtype.  The optional lse
 * output is a dense fp32 [B, H, T*Hg*Wg] array holding the natural-log
 * log-sum-exp of each query's scaled logits.
 *
 * Ownership.  The caller allocates and owns every buffer, including the
 * workspace.  No entry point allocates device or host memory, keeps a pointer
 * after it returns, or synchronises the stream (except basa_get_status).
 *
 * Ordering.  All device work is enqueued on the given stream, in order.
 *
 * Errors.  Arguments are validated synchronously before anything is launched;
 * on an error nothing is enqueued and a status code is returned.  A launch
 * failure returns BASA_ERR_CUDA.  Every wait inside the kernels is bounded in
 * time; a wait that runs out makes the kernel stop early and sets a device
 * status word that basa_get_status reports as BASA_ERR_TIMEOUT.  The library
 * never aborts the process and never traps on the device.
 *
 * Supported sizes.
 *   fp32 (BASA_F32): d in {32, 64, 128}; any window that divides the grid.
 *     Exact fp32 arithmetic on CUDA cores (no reduced-precision tensor math).
 *   bf16 (BASA_BF16): d in {64, 128}; window width ww <= 128; the window is
 *     cut into tiles of whole rows of width ww, and every TMA box of a tile
 *     (a piece of a tile that does not cross a wrapped border) must hold a
 *     multiple of 8 tokens; at most 32 tiles (about 4096 tokens) per window;
 *     at most 16 distinct box shapes per call.  Sizes outside these bounds
 *     return BASA_ERR_UNSUPPORTED.  Tensor cores (tcgen05) with fp32
 *     accumulation and an fp32 softmax; probabilities are rounded to bf16
 *     before they multiply V; outputs are rounded to bf16.
 *   All pointers 16-byte aligned.  B * H * T * Hg * Wg == 0 is a valid no-op.
 */
#ifndef BASA_H_
#define BASA_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define BASA_API __attribute__((visibility("default")))
#else
#define BASA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum basa_status {
  BASA_OK = 0,
  BASA_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad dtype value */
  BASA_ERR_SHAPE = 2,       /* window or pool cell does not divide the grid */
  BASA_ERR_UNSUPPORTED = 3, /* head dim, window or box plan outside the bounds above */
  BASA_ERR_ALIGN = 4,       /* a pointer is not 16-byte aligned */
  BASA_ERR_WORKSPACE = 5,   /* workspace missing when global memory is requested */
  BASA_ERR_CUDA = 6,        /* CUDA runtime or driver error at launch */
  BASA_ERR_TIMEOUT = 7,     /* a bounded wait inside a kernel ran out */
  BASA_ERR_SCRATCH_LIMIT = 8, /* basa_window_attn_noalloc: pooled K/V exceed its fixed scratch */
  BASA_ERR_CHECK = 9          /* checked build (BASA_CHECKED) only: a kernel found a TMA box or
                                 an output index outside its tensor and skipped the access */
} basa_status;

/* Element types.  BASA_FP8_E4M3: q, k, v as OCP e4m3 bytes (basa_window_attn
 * and basa_full_attn only, d = 128, no pool cell), each tensor's values scaled
 * by its descale factor in basa_params; the output is bf16 [B, T, Hg, Wg, H, d]
 * and lse fp32.  Q K^T runs on e4m3 tensor-core MMAs; V is widened to bf16 in
 * shared memory (exactly) for the bf16 P.V MMA.  Other entry points return
 * BASA_ERR_UNSUPPORTED for it. */
typedef enum basa_dtype { BASA_F32 = 0, BASA_BF16 = 1, BASA_FP8_E4M3 = 2 } basa_dtype;

/* Flag bits for basa_params.flags. */
#define BASA_FLAG_PAD_GRID 0x4u            /* grids that a window size does not divide: each
                                              axis is padded at its far end to the next
                                              multiple of the window, the shift rolls the
                                              padded axis (window of coordinate x:
                                              floor(((x - s) mod Gp) / w)), and padded
                                              positions are neither queries nor keys.  The
                                              pages give no rule for such grids; this is the
                                              usual shifted-window padding.  Without the flag
                                              such a grid is BASA_ERR_SHAPE.  Pool cells must
                                              still divide the grid.  The backward runs on
                                              CUDA cores for padded grids. */
#define BASA_FLAG_TEST_WITHHOLD_LOADS 0x1u /* the bf16 kernel's loader issues nothing,
                                              so its first wait runs out (tests the
                                              timeout path); output is not written */
#define BASA_FLAG_BWD_CUDA_CORES 0x2u      /* basa_window_attn_bwd: take the fp32 CUDA-core
                                              kernels for bf16 too (comparison and tests) */

typedef struct basa_params {
  int32_t B, H;        /* batch, heads */
  int32_t T, Hg, Wg;   /* grid: time (1 for images), rows, columns */
  int32_t d;           /* head dim */
  int32_t wt, wh, ww;  /* window size per axis (t, rows, columns) */
  int32_t st, sh, sw;  /* window-partition shift per axis; any integer, reduced mod window */
  int32_t pt, ph, pw;  /* pooled cell size per axis; all 0 = no global memory */
  float scale;         /* softmax scale on q.k; 0 selects 1/sqrt(d) */
  int32_t dtype;       /* basa_dtype of q, k, v, out and pooled tensors */
  uint32_t flags;      /* 0, or BASA_FLAG_* bits */
  uint32_t wait_timeout_ms; /* bound on each device wait; 0 selects 2000 ms */
  int32_t Hkv;         /* K/V heads (grouped-query attention); 0 selects H.  H must be a
                          multiple of Hkv; query head h reads K/V head h / (H / Hkv).
                          k, v and pooled / text K/V then have Hkv heads, q and out H. */
  float q_descale, k_descale, v_descale; /* BASA_FP8_E4M3 only: the value of an element is
                          its e4m3 value times its tensor's factor (0 selects 1); other
                          dtypes ignore them */
} basa_params;

/* Human-readable name of a status code (static string). */
BASA_API const char* basa_status_string(basa_status s);

/* Library ABI version (major * 100 + minor). */
BASA_API int basa_version(void);

/*
 * Bytes of workspace basa_window_attn needs for params p: room for pooled K and
 * pooled V (each [B, P, H, d] of p->dtype, 256-byte aligned), or 0 when p asks
 * for no global memory.  Returns 0 for invalid params.
 */
BASA_API size_t basa_workspace_size(const basa_params* p);

/*
 * K/V mean pooling into global-memory tokens (forum review of the BASA paper,
 * zhichai.net topic 178635722 reply 178634520, four-part method list: K/V
 * pooled global memory).  kp[b, c, h, :] = mean of k over the tokens of cell c
 * (cells of pt x ph x pw aligned to the grid origin); the same for v into vp.
 * Accumulates in fp32, stores in p->dtype (round to nearest even for bf16).
 * k, v: [B, T, Hg, Wg, H, d]; kp, vp: [B, T/pt, Hg/ph, Wg/pw, H, d].
 */
BASA_API basa_status basa_pool_kv(const void* k, const void* v, void* kp, void* vp,
                         const basa_params* p, cudaStream_t stream);

/*
 * Shifted local window attention ("BASA: Backend-Agnostic Sparse Attention for
 * Fast High-Resolution Diffusion Transformers", zhichai.net topic 178635722,
 * "The BASA Method").  out[b, x, h, :] = softmax over the keys of x's shifted
 * window (plus, when p asks for global memory, the pooled keys) of
 * scale * q[b, x, h, :] . k[b, y, h, :], applied to v.
 * If p asks for global memory, pooled K/V are first computed into
 * `workspace` (basa_workspace_size(p) bytes) on the same stream; otherwise
 * workspace may be NULL.  lse may be NULL.
 */
BASA_API basa_status basa_window_attn(const void* q, const void* k, const void* v, void* out,
                             float* lse, void* workspace, const basa_params* p,
                             cudaStream_t stream);

/*
 * Shifted local window attention with caller-supplied pooled global memory
 * kp, vp ([B, T/pt, Hg/ph, Wg/pw, H, d], e.g. from basa_pool_kv).  The same
 * operation as basa_window_attn without the pooling step; p must ask for global
 * memory (pt, ph, pw >= 1).
 */
BASA_API basa_status basa_window_attn_gm(const void* q, const void* k, const void* v,
                                const void* kp, const void* vp, void* out, float* lse,
                                const basa_params* p, cudaStream_t stream);

/*
 * Joint text + image attention of an MM-DiT block (FLUX-style double-stream
 * attention) with the visual self-attention replaced by shifted windows.  The
 * pages ("BASA: Backend-Agnostic Sparse Attention for Fast High-Resolution
 * Diffusion Transformers", zhichai.net topic 178635722, "The BASA Method") say
 * the method replaces the *visual* self-attention; the reading taken here for
 * the text tokens of a joint block:
 *   - image query p attends to Win(p) plus all L text tokens, one softmax;
 *   - text query attends to all N image tokens plus all L text tokens.
 * q, k, v, out: image tokens [B, T, Hg, Wg, H, d]; qt, kt, vt, out_t: text
 * tokens [B, L, H, d]; lse / lse_t: fp32 [B, H, N] / [B, H, L], or NULL.  Same
 * dtype for all, 16-byte aligned.  p gives the window and shift; its pool cell
 * must be (0, 0, 0) (text tokens take the place of the global memory), else
 * BASA_ERR_UNSUPPORTED.  L = 0 is plain window attention (text pointers
 * unused).  Two launches on `stream`: the image queries, then the text queries
 * (plus a combine launch when the text pass is split, see
 * basa_joint_workspace_size; workspace may be NULL).  Validation happens before
 * the first launch.  The caller owns every buffer.
 */
BASA_API basa_status basa_joint_attn(const void* q, const void* k, const void* v,
                                     const void* qt, const void* kt, const void* vt, int64_t L,
                                     void* out, void* out_t, float* lse, float* lse_t,
                                     void* workspace, const basa_params* p,
                                     cudaStream_t stream);

/*
 * Bytes of workspace basa_joint_attn can use for L text tokens, or 0.  The
 * text-query pass has few work units (B * H * ceil(L / 256)); when they would
 * leave most SMs idle and a workspace of this size (16-byte aligned) is given,
 * the pass splits its key range over the SMs, writes fp32 partial outputs and
 * per-row (max, sum) there, and merges them in one more launch.  With a NULL
 * workspace the pass runs unsplit.  0 for fp32, for invalid params, and when
 * no split is chosen on the current device.
 */
BASA_API size_t basa_joint_workspace_size(const basa_params* p, int64_t L);

/*
 * Backward of shifted window attention, with or without pooled global memory:
 * the gradients dq, dk, dv of basa_window_attn's output for the output
 * gradient dout.  The
 * dense-teacher adaptation on the pages ("BASA: Backend-Agnostic Sparse
 * Attention for Fast High-Resolution Diffusion Transformers", zhichai.net topic
 * 178635722, forum review reply 178634520) trains through this attention.
 * With P the softmax weights of each query over its window (recomputed from q,
 * k and the forward's lse) and D_i = dout_i . out_i:
 *   dS_ij = P_ij (dout_i . v_j - D_i),  dq_i = scale sum_j dS_ij k_j,
 *   dk_j = scale sum_i dS_ij q_i,  dv_j = sum_i P_ij dout_i.
 * q, out, dout, dq: [B, T, Hg, Wg, H, d]; k, v, dk, dv: [B, T, Hg, Wg, Hkv, d]
 * (query heads of one group add into the shared dk, dv); lse: fp32 [B, H, N]
 * from the forward call; workspace: basa_bwd_workspace_size(p) bytes, 16-byte
 * aligned.  With a pool cell in p the pooled tokens join every query's keys as
 * in the forward: their K, V are recomputed into the workspace, their gradients
 * (summed over every query of the batch) reach dq and flow back to each cell
 * token's dk, dv divided by the cell size.  bf16 with d = 64 or 128 runs on the
 * tensor cores: fp32 logits, exponentials and accumulators, with P and dS
 * rounded to bf16 as the operands of their MMAs, and the gradients rounded
 * once.  fp32 (and bf16 windows beyond the tensor-core tile plan's bounds, or
 * with BASA_FLAG_BWD_CUDA_CORES) runs in fp32 on CUDA cores.  Launches on
 * `stream` only; nothing is allocated.
 */
BASA_API size_t basa_bwd_workspace_size(const basa_params* p);

/*
 * Backward of joint text + image attention (basa_joint_attn): the gradients of
 * both outputs for the output gradients dout (image) and dout_t (text).  Image
 * query i's keys are its shifted window and the L text tokens, text query t's
 * keys are every image and text token; per query row dS = P (dP - D) with
 * D = dout . out, and every key's dk, dv sum over all the queries that see it
 * (the text keys over every image and text query).  Image tensors
 * [B, T, Hg, Wg, H or Hkv, d], text tensors [B, L, H or Hkv, d]; lse, lse_t from
 * the forward call; workspace: basa_joint_bwd_workspace_size(p, L) bytes,
 * 16-byte aligned.  bf16 (d = 64 or 128, grids the window divides): tensor
 * cores, with P and dS rounded to bf16 as MMA operands and the text keys' sums
 * in fp32; fp32, or BASA_FLAG_BWD_CUDA_CORES, or shapes outside those bounds:
 * fp32 arithmetic on CUDA cores.  Gradients rounded once.  L = 0 is basa_window_attn_bwd.  A pool cell in p gives
 * BASA_ERR_UNSUPPORTED.  Launches on `stream` only; nothing is allocated.
 */
BASA_API size_t basa_joint_bwd_workspace_size(const basa_params* p, int64_t L);
BASA_API basa_status basa_joint_attn_bwd(const void* q, const void* k, const void* v,
                                         const void* qt, const void* kt, const void* vt,
                                         int64_t L, const void* out, const void* out_t,
                                         const void* dout, const void* dout_t, const float* lse,
                                         const float* lse_t, void* dq, void* dk, void* dv,
                                         void* dqt, void* dkt, void* dvt, void* workspace,
                                         const basa_params* p, cudaStream_t stream);
BASA_API basa_status basa_window_attn_bwd(const void* q, const void* k, const void* v,
                                          const void* out, const void* dout, const float* lse,
                                          void* dq, void* dk, void* dv, void* workspace,
                                          const basa_params* p, cudaStream_t stream);

/*
 * Full softmax attention over all T*Hg*Wg tokens: the same kernels with one
 * window covering the whole grid (the quadratic baseline of the BASA pages).
 * Window, shift and pool fields of p are ignored.
 */
BASA_API basa_status basa_full_attn(const void* q, const void* k, const void* v, void* out,
                           float* lse, const basa_params* p, cudaStream_t stream);

/*
 * basa_window_attn without any device allocation.  There is no counterpart on
 * the pages that describe the method; this exists for callers that cannot
 * allocate device memory, such as an operator inside a host framework that owns
 * all device memory and gives its operators no workspace, or a latency-critical
 * serving path that reserves memory at start-up and forbids cudaMalloc/cudaFree
 * (which can block the host and, for cudaFree, synchronise the device).
 *
 * Same operation, arguments and layouts as basa_window_attn, minus the
 * workspace: the pooled K/V tokens go to a fixed 32 MiB scratch array inside
 * the library's device code.
 *  - Every GPU that loads the library's device code holds that array until the
 *    process exits.
 *  - If pooled K and V together need more than 32 MiB (each [B, P, Hkv, d] of
 *    p->dtype, Hkv = p->Hkv or H when it is 0, rounded up to 256 bytes), the
 *    call returns BASA_ERR_SCRATCH_LIMIT and enqueues nothing.
 *  - The first call with a given device current looks up the array's device
 *    address (cudaGetSymbolAddress) and caches it together with the id of the
 *    current CUDA context; that first call should be made before any stream
 *    capture begins.  A call in a new context on the same device (after
 *    cudaDeviceReset, for instance) looks the address up again, so it too
 *    should come before any capture in that context.
 *  - All calls on a device share the array: calls whose work overlaps on the
 *    GPU (e.g. on unordered streams) race on it and must be ordered by the
 *    caller.  Nothing in it needs to start at zero: each call overwrites every
 *    byte it reads.
 *  - The call makes no device or host heap allocation.
 */
BASA_API basa_status basa_window_attn_noalloc(const void* q, const void* k, const void* v,
                                              void* out, float* lse, const basa_params* p,
                                              cudaStream_t stream);

/*
 * Test and diagnostics only: synchronises `stream`, then reports and clears the
 * device status word of the current device.  BASA_ERR_TIMEOUT if a kernel
 * wait ran out since the last call, BASA_ERR_CUDA on a pending CUDA error,
 * else BASA_OK.
 */
BASA_API basa_status basa_get_status(cudaStream_t stream);

/*
 * Host-only description of the bf16 kernel's window tiling (no GPU needed).
 * *n_windows = windows per (b, h) and *n_tiles = 128-row tiles per window.
 * If rows != NULL it receives [n_windows][n_tiles][128] int32 entries: the
 * flattened grid index (t * Hg + y) * Wg + x of the token that row r of the
 * tile holds in shared memory, or -1 for a padding row (past the tile's
 * tokens, or a padded position with BASA_FLAG_PAD_GRID).  Only the grid,
 * window, shift and flags fields and d/dtype of p are read; shapes outside the bf16 bounds
 * return BASA_ERR_UNSUPPORTED.  rows_capacity is the number of int32 entries
 * rows can hold.
 */
BASA_API basa_status basa_window_tiles(const basa_params* p, int32_t* n_windows, int32_t* n_tiles,
                              int32_t* rows, int64_t rows_capacity);

#ifdef __cplusplus
}
#endif

#endif /* BASA_H_ */
