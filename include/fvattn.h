/*
 * fvattn.h -- C ABI of libfvattn.so: adaptive block-sparse self-attention over
 * 3D video latent tokens, for NVIDIA B200 (sm_100a).
 *
 * The path (pages: "VSA" digest, section 3; "FVAttn" digest, sections 00/02;
 * "DFSAttn" digest, sections 1 and 3; "Causal-RoPE SP" digest, sections
 * 2.2-2.3):
 *   1. tokens of a T x Hg x W latent grid are grouped into 4x4x4 tiles
 *      (64 tokens), in raster-cube or 3D Hilbert order;
 *   2. optionally, a 3D rotary position encoding is applied to Q and K;
 *   3. Q and K are mean-pooled per tile;
 *   4. a coarse pooled Q K^T gives a softmax over key tiles per query tile;
 *   5. per (batch, head, query tile) the key tiles are selected by top-p
 *      cumulative mass with a k_min floor;
 *   6. the fine stage runs softmax attention of each query token over the
 *      tokens of its tile's selected key tiles only.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Tensors.  q, k, v, out are [B, H, N, d] row-major (d fastest), N = T*Hg*W;
 *   lse is [B, H, N] float32.  dtype FVATTN_BF16 (bf16 storage, fp32
 *   accumulation, bf16 tensor-core operands) or FVATTN_F32 (fp32 throughout).
 *   Natural layout: token n = (t*Hg + h)*W + w.  Tiled layout: token rows
 *   permuted so that tile j (in the chosen order) occupies rows 64j..64j+63,
 *   as produced by fvattn_tile_reorder.  Tile ids always follow the order.
 * Pointers.  Every tensor, block-list and workspace pointer is a DEVICE
 *   pointer owned by the caller; the library never allocates or frees device
 *   memory and keeps no pointer after a call returns.  Shapes, rope and
 *   cache structs are HOST pointers read during the call.  Device pointers
 *   must be 16-byte aligned; the workspace 256-byte aligned.
 * Execution.  Calls enqueue kernels on the given stream and return without
 *   synchronising (except fvattn_get_device_status).  Calls that share a
 *   workspace must not overlap in time.
 * Outputs.  out must not overlap q, k or v: with RoPE enabled the forward
 *   calls first write the rotated Q into out (each query row where its
 *   output row goes) and the fine stage overwrites it with the output; the
 *   rotated K goes to the workspace.
 * Errors.  Argument, shape and capacity errors are detected on the host and
 *   returned before anything is enqueued.  A failed launch returns
 *   FVATTN_ERR_CUDA.  Errors found by a kernel (an out-of-range block index,
 *   a wait that hit its iteration cap) set a status word in the workspace,
 *   read with fvattn_get_device_status; kernels never trap.
 * Limits.  grid extents multiples of the tile (4,4,4), each <= 4096;
 *   d = 128 for BF16 (tensor-core fine stage), d in {32, 64, 128} for F32;
 *   nT = N/64 <= 4096; B*H*N*d < 2^31.
 */
#ifndef FVATTN_H
#define FVATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* fvattn_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  FVATTN_OK = 0,
  FVATTN_ERR_INVALID_ARG = -1,     /* null pointer, bad enum, top_p NaN, misaligned pointer */
  FVATTN_ERR_SHAPE = -2,           /* grid not a multiple of the tile, bad head_dim, too large */
  FVATTN_ERR_DTYPE = -3,
  FVATTN_ERR_CAPACITY = -4,        /* blocks.cap < nT */
  FVATTN_ERR_CUDA = -5,            /* a CUDA runtime/driver call failed */
  FVATTN_ERR_CACHE_MISMATCH = -6,  /* reuse_mask with a cache filled for another shape */
  FVATTN_ERR_DEVICE = -7,          /* a kernel set the device status word */
  FVATTN_ERR_WORKSPACE = -8,       /* ws_bytes smaller than fvattn_workspace_size */
  FVATTN_ERR_UNSUPPORTED = -9      /* device is not sm_100, or a combination not built */
} fvattn_status;

typedef enum { FVATTN_F32 = 0, FVATTN_BF16 = 1 } fvattn_dtype;
typedef enum { FVATTN_ORDER_RASTER_CUBE = 0, FVATTN_ORDER_HILBERT = 1 } fvattn_order;
typedef enum { FVATTN_LAYOUT_NATURAL = 0, FVATTN_LAYOUT_TILED = 1 } fvattn_layout;

typedef struct { int32_t T, H, W; } fvattn_dims;   /* latent grid (frames, height, width) */
typedef struct { int32_t t, h, w; } fvattn_tile;   /* tile edge per axis; only 4,4,4 is supported */

/* 3D rotary encoding ("Causal-RoPE SP" digest, sections 2.2-2.3): head dims
 * split into groups of dt, dh, dw (dt+dh+dw == d, each even) for the t, h,
 * w axes; in a group of size da, dims (2j, 2j+1) rotate by pos*base^(-2j/da),
 * pos the token's integer grid coordinate on that axis.  Pooling uses the
 * rotated values in fp32; the fine stage uses them rounded to the dtype. */
typedef struct { int32_t enabled, dt, dh, dw; float base; } fvattn_rope;

typedef struct {
  int32_t batch, heads, head_dim;
  fvattn_dims grid;
  fvattn_tile tile;
  fvattn_dtype dtype;
  fvattn_order order;
  fvattn_layout layout;   /* layout of q, k, v, out, lse in pool_select / block_sparse_fwd */
  float scale;            /* softmax scale for coarse and fine logits; 0 => 1/sqrt(head_dim) */
} fvattn_shape;

/* Selected key tiles per (batch, head, query tile).  counts [B,H,nT] int32;
 * idx [B,H,nT,cap] int32 with row r's first counts[r] entries the selected
 * tile ids in ascending order; entries past counts[r] are not written and
 * not read.  cap >= nT. */
typedef struct { int32_t* counts; int32_t* idx; int32_t cap; } fvattn_blocks;

/* Block lists kept across diffusion steps ("DFSAttn" digest, section 3).
 * blocks are caller-owned device buffers; shape/top_p/k_min/valid are
 * written by fvattn_forward when it fills the cache. */
typedef struct {
  fvattn_blocks blocks;
  fvattn_shape shape;
  float top_p;
  int32_t k_min;
  int32_t valid;
} fvattn_mask_cache;

/* nT = N / 64 for a valid shape. */
int fvattn_num_tiles(const fvattn_shape* shape, int64_t* num_tiles);

/* Bytes of device workspace every entry point below needs for this shape
 * (the maximum over them, rope included when rope != NULL && rope->enabled). */
int fvattn_workspace_size(const fvattn_shape* shape, const fvattn_rope* rope, size_t* bytes);

/* Step 1 ("VSA" digest, section 3: (4,4,4) cubes; "DFSAttn" digest,
 * section 1: Hilbert reordering before blocking).  Permutes token rows of a
 * [B*H, N, row_bytes] tensor between natural and tiled layout:
 * inverse == 0: y[pi(n)] = x[n]; inverse != 0: y[n] = x[pi(n)], where pi(n)
 * is token n's tiled position in shape->order.  row_bytes is a multiple of 4
 * in [4, 1024] (d*sizeof(dtype) for q/k/v/out, 4 for lse).  x and y must not
 * overlap.  shape->layout is ignored. */
int fvattn_tile_reorder(const fvattn_shape* shape, const void* x, void* y, int32_t row_bytes,
                        int inverse, void* ws, size_t ws_bytes, fvattn_stream_t stream);

/* Steps 2-5 ("VSA" digest, section 3: pooled coarse stage predicting tile
 * importance; "FVAttn" digest, sections 00/02: top-p routing with a top-k
 * floor).  q, k in shape->layout.  Writes out->counts and out->idx.
 * count = min(nT, max(m, k_min)), m >= 1 the fewest tiles whose coarse
 * softmax mass reaches top_p (ties to the lower tile id); top_p >= 1 keeps
 * every tile; top_p <= 0 with k_min = k is fixed top-k.  rope may be NULL. */
int fvattn_pool_select(const fvattn_shape* shape, const void* q, const void* k,
                       const fvattn_rope* rope, float top_p, int32_t k_min,
                       const fvattn_blocks* out, void* ws, size_t ws_bytes,
                       fvattn_stream_t stream);

/* Steps 2-5 with hierarchical sub-block scoring ("DFSAttn" digest, section 2:
 * a block is split into smaller sub-blocks whose scores are summed into the
 * block's importance).  Each 4x4x4 tile splits into the eight 2x2x2
 * sub-cubes of its grid coordinates; Q and K are mean-pooled per sub-cube;
 * every query sub-block takes a softmax over all key sub-blocks of the
 * head; the importance of key tile j for query tile i is the mean over the
 * eight query sub-blocks of i of the probability mass they give to the
 * eight key sub-blocks of j.  Top-p and k_min act on these importances
 * exactly as in fvattn_pool_select (ranked by their logarithm, ties to the
 * lower tile id).  Arguments, layouts and results as fvattn_pool_select;
 * the workspace is fvattn_workspace_size_subblock bytes (it adds
 * 4 * B*H*nT*8*d + B*H*nT*8*nT floats).  The fine stage for these lists is
 * fvattn_block_sparse_fwd. */
int fvattn_workspace_size_subblock(const fvattn_shape* shape, const fvattn_rope* rope, size_t* bytes);
int fvattn_pool_select_subblock(const fvattn_shape* shape, const void* q, const void* k,
                                const fvattn_rope* rope, float top_p, int32_t k_min,
                                const fvattn_blocks* out, void* ws, size_t ws_bytes,
                                fvattn_stream_t stream);

/* Steps 2-5 without a caller workspace.  The pages have no counterpart:
 * this is for callers that cannot allocate device memory (a plugin whose
 * host application owns every device allocation and passes in only the
 * input and output tensors, or code on a latency-critical path where the
 * device-wide synchronisation of cudaMalloc is not allowed).  Arguments,
 * layout and results are those of fvattn_pool_select; the scratch memory
 * is a 32 MiB array inside the library that every GPU loading the library
 * holds until the process exits.  Shapes whose workspace
 * (fvattn_workspace_size) exceeds 32 MiB are rejected with
 * FVATTN_ERR_WORKSPACE before anything is enqueued.  No call allocates
 * memory.  The first call on each device looks up the array's device
 * address (cudaGetSymbolAddress, with that device current); make that first
 * call before any stream capture.  All calls share the one array and it
 * keeps the last call's contents (each call rewrites every part it reads),
 * so calls that overlap on the GPU (other streams, other host threads)
 * race: serialise them. */
int fvattn_pool_select_noalloc(const fvattn_shape* shape, const void* q, const void* k,
                               const fvattn_rope* rope, float top_p, int32_t k_min,
                               const fvattn_blocks* out, fvattn_stream_t stream);

/* Device status of fvattn_pool_select_noalloc (the pages have no
 * counterpart either).  A caller without a workspace cannot pass one to
 * fvattn_get_device_status, so this reads the status word that the
 * kernels of fvattn_pool_select_noalloc set on a device-detected error (0:
 * none; 1: an out-of-range block index; 2: a wait that hit its iteration
 * cap) from the library's own scratch array, clears it, and returns it in
 * *status (a HOST pointer).  It synchronises `stream` first, then copies
 * 4 bytes with cudaMemcpy; it allocates nothing.  Call it on the device
 * and stream of the noalloc calls it checks; calls that overlap race as
 * above. */
int fvattn_pool_select_noalloc_status(fvattn_stream_t stream, int32_t* status);

/* Schedule of the fine stage (single-GPU analogue of the "FVAttn" digest's
 * runtime head-level load balancing, section 02): a work item is two
 * adjacent query tiles 2q, 2q+1 of one (batch, head), encoded
 * ((b*H + h)*P + q) with P = ceil(nT/2); its cost is the size of the union
 * of the two tiles' lists (a tile past nT contributes nothing); items are
 * sorted by cost descending, ties by ascending item code
 * (longest-processing-time first).  worklist has B*H*P int32.  (The work
 * list fvattn_forward and fvattn_block_sparse_fwd build for their own fine
 * stage ranks union sizes in buckets of 16 entries, ties by item, so that
 * items of one head run together, runs it serpentine (CTA c takes slot c of
 * even rounds of G slots and slot G - 1 - c of odd ones), and applies that
 * order within groups of consecutive heads when one head's K and V take more
 * than a quarter of the L2: groups of about 40 MB of K/V, in head order, so
 * that the CTAs running together share those heads' K/V in the cache.) */
int fvattn_build_worklist(const fvattn_shape* shape, const fvattn_blocks* blocks,
                          int32_t* worklist, void* ws, size_t ws_bytes, fvattn_stream_t stream);

/* Step 6 ("VSA" digest, section 3: token-level attention inside the selected
 * tiles; "CalibAtt" digest: selected connections computed densely, the rest
 * skipped).  q, k, v, out, lse in shape->layout; out has the input dtype,
 * lse is the natural-log softmax normaliser.  With rope enabled q and k are
 * rotated first.  Block ids are checked on the device (bad ids set the
 * status word and the row's output is left unwritten). */
int fvattn_block_sparse_fwd(const fvattn_shape* shape, const void* q, const void* k,
                            const void* v, const fvattn_rope* rope, const fvattn_blocks* blocks,
                            void* out, float* lse, void* ws, size_t ws_bytes,
                            fvattn_stream_t stream);

/* The whole path on natural-layout tensors (shape->layout is ignored).
 * cache == NULL: select and attend.  cache != NULL, reuse_mask == 0: select,
 * store the lists into cache->blocks and stamp the cache.  reuse_mask != 0:
 * skip steps 2-5 and attend with cache->blocks ("DFSAttn" digest, section 3);
 * returns FVATTN_ERR_CACHE_MISMATCH if the cache is not valid for this shape. */
int fvattn_forward(const fvattn_shape* shape, const void* q, const void* k, const void* v,
                   const fvattn_rope* rope, float top_p, int32_t k_min, fvattn_mask_cache* cache,
                   int reuse_mask, void* out, float* lse, void* ws, size_t ws_bytes,
                   fvattn_stream_t stream);

/* Slack-aware augmentation on one GPU ("FVAttn" digest, section 02: ranks
 * off the critical path spend their spare time on extra, somewhat important
 * blocks).  The persistent fine stage's CTAs play the ranks.  From the lists
 * in `base` (selected by any means; shape->layout as in fvattn_pool_select),
 * builds the fine stage's work list (fvattn_build_worklist's order) into
 * `worklist` [B*H*P] and assumes CTA c of G = min(num_ctas, B*H*P) runs the
 * slots c, c + G, ...; an item costs its union size (at least 1).  Each CTA's
 * slack (the largest CTA load minus its own) is split evenly over its items,
 * the first in slot order taking the remainder; an item with at least one
 * non-empty row then adds up to that many key tiles outside its union, by
 * the largest coarse logit over its non-empty rows (ties to the lower tile
 * id; logits as fvattn_pool_select computes them, with rope), to each of
 * those rows.  Writes the augmented lists (ascending) to `out`, which may be
 * `base` itself.  Run the fine stage with fvattn_block_sparse_fwd_worklist
 * and the same worklist and num_ctas so that the critical path keeps its
 * length.  num_ctas in [0, 1024], 0 = the device's SM count (the fine
 * stage's grid).
 * cta_busy_ns: NULL (slack in union entries, as above), or a HOST array of
 *   G = min(num_ctas or the SM count, B*H*P, 1024) busy times in ns, one per
 *   CTA, each in [0, 2^40), measured on a run of the same work list and
 *   num_ctas on the unaugmented lists (fvattn_profile_cta_times: end minus
 *   start).  A CTA's slack is then its measured idle time in entries at that
 *   run's mean time per entry, scaled by fill_percent in [0, 100]:
 *   floor((max busy - busy_c) * total entries * fill / (100 * total busy)).
 *   The array is read during the call. */
int fvattn_augment_lists(const fvattn_shape* shape, const void* q, const void* k, const fvattn_rope* rope,
                         const fvattn_blocks* base, int32_t num_ctas, const int64_t* cta_busy_ns,
                         int32_t fill_percent, const fvattn_blocks* out, int32_t* worklist, void* ws,
                         size_t ws_bytes, fvattn_stream_t stream);

/* Step 6 with a caller's work list (B*H*P item codes, each once) and
 * persistent grid of num_ctas CTAs (0 = the SM count); otherwise as
 * fvattn_block_sparse_fwd.  fp32 workloads ignore the work list. */
int fvattn_block_sparse_fwd_worklist(const fvattn_shape* shape, const void* q, const void* k,
                                     const void* v, const fvattn_rope* rope,
                                     const fvattn_blocks* blocks, const int32_t* worklist,
                                     int32_t num_ctas, void* out, float* lse, void* ws,
                                     size_t ws_bytes, fvattn_stream_t stream);

/* Timestep schedule of the selection ("DFSAttn" digest, section 3: sparsity
 * is low while the frames are still noise and rises as the video sharpens).
 * Host-only arithmetic, no device call.  For diffusion step `step` of
 * `num_steps`: the first `dense_steps` steps keep every tile (*top_p = 1,
 * *k_min = k_start); over the remaining steps top_p and k_min move linearly
 * from (p_start, k_start) to (p_end, k_end), k_min rounded half up.  Feed
 * the result to fvattn_forward (a cache refilled when the lists should
 * follow the new sparsity). */
int fvattn_timestep_params(int32_t step, int32_t num_steps, float p_start, float p_end,
                           int32_t k_start, int32_t k_end, int32_t dense_steps, float* top_p,
                           int32_t* k_min);

/* Backward pass of step 6 ("VSA" digest, section 3: the fine block-sparse
 * attention is trained end to end).  For the lists in `blocks` (fixed: the
 * selection is piecewise constant in q and k and passes no gradient) and
 * the forward's out and lse, computes the gradients of
 * L = sum(out * dout): with s = scale q k^T and p = exp(s - lse) over each
 * row's selected keys,
 *   dv = p^T dout,  ds = p * (dout v^T - rowsum(dout * out)),
 *   dq = scale ds k,  dk = scale ds^T q,
 * summed over every query tile that selected a key's tile (keys no tile
 * selected get zero gradients; a query tile with an empty list gets dq = 0).
 * q, k, v, out, dout, dq, dk, dv are [B, H, N, 128] bf16 in the TILED layout
 * (shape->layout must be FVATTN_LAYOUT_TILED, else FVATTN_ERR_UNSUPPORTED);
 * lse [B, H, N] float32 as fvattn_block_sparse_fwd wrote it; q and k are the
 * tensors the fine stage consumed (rotated ones when RoPE was used).  bf16
 * only (FVATTN_ERR_DTYPE otherwise).  P and dS are rounded to bf16 for the
 * tensor cores, accumulation is fp32, the gradients are rounded once to bf16.
 * No atomics: the result is deterministic.  Workspace:
 * fvattn_workspace_size_bwd bytes.  Bad block ids set status 1 and are
 * dropped. */
int fvattn_workspace_size_bwd(const fvattn_shape* shape, size_t* bytes);
int fvattn_block_sparse_bwd(const fvattn_shape* shape, const void* q, const void* k, const void* v,
                            const void* out, const void* dout, const float* lse,
                            const fvattn_blocks* blocks, void* dq, void* dk, void* dv, void* ws,
                            size_t ws_bytes, fvattn_stream_t stream);

/* Attention prologue ("Causal-RoPE SP" digest, section 2.3: the QKV
 * projection and the rotary encoding fused into one kernel; section 2.2: a
 * block that starts at frame s encodes its local frame t at global frame
 * t + s, so a rank needs only s to rotate its own tokens).
 *   x     [B, N, C] bf16, natural token order (row n = token (t, h, w)).
 *   w     [3*H*d, C] bf16, a linear layer's weight (output rows first):
 *         rows 0..H*d-1 project Q (head h at rows h*d..h*d+d-1), then K,
 *         then V.
 *   bias  [3*H*d] float32, or NULL for none.
 *   For every token and output row o: y = sum_c x[n, c] * w[o, c] with fp32
 *   accumulation of the exact bf16 products, plus bias[o]; with rope
 *   enabled the Q and K head slices are rotated as in fvattn_rope at
 *   coordinates (t + t_offset, h, w) in fp32; every result is rounded once
 *   to bf16.  q, k, v [B, H, N, d] bf16 receive the three parts in
 *   shape->layout: natural, or tiled in shape->order (the layout
 *   fvattn_tile_reorder produces), ready for fvattn_pool_select and
 *   fvattn_block_sparse_fwd.
 * Requirements: shape->dtype FVATTN_BF16 and head_dim 128; channels a
 * multiple of 64 in [64, 65536]; 0 <= t_offset <= 2^20; x, w, bias, q, k, v
 * 16-byte aligned, q, k, v not overlapping x, w or each other.  The
 * workspace is fvattn_workspace_size_qkv bytes (tables only: N + 2 nT int32
 * and the (cos, sin) pairs). */
int fvattn_workspace_size_qkv(const fvattn_shape* shape, const fvattn_rope* rope, size_t* bytes);
int fvattn_qkv_rope(const fvattn_shape* shape, const void* x, int32_t channels, const void* w,
                    const float* bias, const fvattn_rope* rope, int32_t t_offset, void* q, void* k,
                    void* v, void* ws, size_t ws_bytes, fvattn_stream_t stream);

/* Synchronises the stream, reads and clears the workspace status word.
 * *status is 0 or a positive code: 1 bad block id, 2 wait cap reached. */
int fvattn_get_device_status(void* ws, fvattn_stream_t stream, int32_t* status);

/* Failure-detection self test: launches one block that waits, with the
 * library's bounded wait, on a barrier nothing ever completes, using the
 * given iteration cap.  The kernel gives up, sets status 2 in the workspace
 * status word and returns; read it with fvattn_get_device_status. */
int fvattn_selftest_wait_timeout(void* ws, size_t ws_bytes, int64_t cap_iterations,
                                 fvattn_stream_t stream);

/* Per-stage timing.  While enabled, every entry point records a pair of CUDA
 * events on its stream around each stage it runs (host-side event objects
 * only; no device memory).  fvattn_profile_read synchronises on the recorded
 * events, writes per stage the summed milliseconds and the number of this
 * library's kernels launched into ms[FVATTN_STAGE_COUNT] and
 * launches[FVATTN_STAGE_COUNT] (either may be NULL) and clears the record.  Not thread-safe against
 * concurrent calls from several host threads. */
typedef enum {
  FVATTN_STAGE_TABLES = 0,    /* tile / token / RoPE tables */
  FVATTN_STAGE_REORDER = 1,   /* fvattn_tile_reorder */
  FVATTN_STAGE_POOL = 2,      /* pooling (+ RoPE, rotated copies) */
  FVATTN_STAGE_SELECT = 3,    /* coarse scores, softmax, top-p selection */
  FVATTN_STAGE_SCHEDULE = 4,  /* union lists + work-list sort */
  FVATTN_STAGE_FINE = 5,      /* block-sparse fine attention */
  FVATTN_STAGE_PROLOGUE = 6,  /* fused QKV projection + RoPE */
  FVATTN_STAGE_BWD_PREP = 7,  /* backward: D = rowsum(dout * out), lse * log2(e) */
  FVATTN_STAGE_BWD_KV = 8,    /* backward: key-stationary dK, dV kernel */
  FVATTN_STAGE_BWD_Q = 9,     /* backward: query-stationary dQ kernel */
  FVATTN_STAGE_COUNT = 10
} fvattn_stage;
int fvattn_profile_enable(int enable);
int fvattn_profile_read(double* ms, int64_t* launches);

/* Per-CTA busy time of the persistent fine stage, the single-GPU analogue of
 * the per-rank load the "FVAttn" digest balances (section 02; section 03
 * reports the mean imbalance ratio).  While profiling is enabled, every
 * fine-stage launch of a call records, for each CTA, the global-timer
 * nanoseconds when its set-up was done and when its last item finished, in
 * the call's workspace.  This reads the record of the last such launch that
 * used workspace `ws` (a DEVICE pointer; shape and rope as in that call, to
 * locate the record): it synchronises `stream`, writes 2 * min(n, capacity)
 * int64 (start, end pairs) to the HOST array `ns` and n (the grid size) to
 * *num_ctas.  Returns FVATTN_ERR_DEVICE if the record is not valid. */
int fvattn_profile_cta_times(const fvattn_shape* shape, const fvattn_rope* rope, void* ws,
                             fvattn_stream_t stream, int64_t* ns, int32_t capacity, int32_t* num_ctas);

const char* fvattn_status_string(int status);

#ifdef __cplusplus
}
#endif
#endif /* FVATTN_H */
