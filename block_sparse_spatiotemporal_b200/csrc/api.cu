// C-ABI entry points of libfvattn.so (declared in include/fvattn.h): host-side
// validation, workspace carve-up, TMA descriptors and the launch sequence of
// each call.  No entry point allocates device memory.
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "fvattn_internal.cuh"

using namespace fvattn;

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

int map_cuda(cudaError_t e) { return e == cudaSuccess ? FVATTN_OK : FVATTN_ERR_CUDA; }

#define FV_TRY(expr)                          \
  do {                                        \
    const int _st = (expr);                   \
    if (_st != FVATTN_OK) return _st;         \
  } while (0)
#define FV_CUDA(expr) FV_TRY(map_cuda(expr))

int elem_size(int dtype) { return dtype == FVATTN_BF16 ? 2 : 4; }

int make_geom(const fvattn_shape* s, Geom* g) {
  if (!s) return FVATTN_ERR_INVALID_ARG;
  if (s->dtype != FVATTN_F32 && s->dtype != FVATTN_BF16) return FVATTN_ERR_DTYPE;
  if (s->order != FVATTN_ORDER_RASTER_CUBE && s->order != FVATTN_ORDER_HILBERT) return FVATTN_ERR_INVALID_ARG;
  if (s->layout != FVATTN_LAYOUT_NATURAL && s->layout != FVATTN_LAYOUT_TILED) return FVATTN_ERR_INVALID_ARG;
  if (s->batch < 1 || s->heads < 1) return FVATTN_ERR_SHAPE;
  if (s->tile.t != 4 || s->tile.h != 4 || s->tile.w != 4) return FVATTN_ERR_SHAPE;
  const int T = s->grid.T, Hg = s->grid.H, W = s->grid.W;
  if (T < 4 || Hg < 4 || W < 4 || T % 4 || Hg % 4 || W % 4 || T > 4096 || Hg > 4096 || W > 4096)
    return FVATTN_ERR_SHAPE;
  const int d = s->head_dim;
  if (s->dtype == FVATTN_BF16) {
    if (d == 32 || d == 64) return FVATTN_ERR_UNSUPPORTED;
    if (d != 128) return FVATTN_ERR_SHAPE;
  } else if (d != 32 && d != 64 && d != 128) {
    return FVATTN_ERR_SHAPE;
  }
  const long long N = (long long)T * Hg * W;
  const long long nT = N / 64;
  if (nT > 4096) return FVATTN_ERR_SHAPE;
  const long long BH = (long long)s->batch * s->heads;
  if (BH * N * d >= (1ll << 31)) return FVATTN_ERR_SHAPE;
  if (std::isnan(s->scale) || s->scale < 0.f || std::isinf(s->scale)) return FVATTN_ERR_INVALID_ARG;
  g->B = s->batch;
  g->H = s->heads;
  g->d = d;
  g->T = T;
  g->Hg = Hg;
  g->W = W;
  g->nt = T / 4;
  g->nh = Hg / 4;
  g->nw = W / 4;
  g->nT = (int)nT;
  g->N = (int)N;
  g->BH = (int)BH;
  g->P = (int)((nT + kItemTiles - 1) / kItemTiles);
  g->Qn = (int)((nT + 3) / 4);
  g->order = s->order;
  g->scale = s->scale > 0.f ? s->scale : (float)(1.0 / std::sqrt((double)d));
  return FVATTN_OK;
}

bool rope_on(const fvattn_rope* r) { return r && r->enabled; }

int check_rope(const fvattn_rope* r, const Geom& g) {
  if (!rope_on(r)) return FVATTN_OK;
  if (r->dt < 0 || r->dh < 0 || r->dw < 0 || (r->dt | r->dh | r->dw) & 1) return FVATTN_ERR_INVALID_ARG;
  if (r->dt + r->dh + r->dw != g.d) return FVATTN_ERR_INVALID_ARG;
  if (!(r->base > 0.f) || std::isinf(r->base)) return FVATTN_ERR_INVALID_ARG;
  return FVATTN_OK;
}

// sub: also the sub-block scoring buffers (pooled sub-blocks, key-tile masses).
WsLayout layout_for(const Geom& g, int dtype, const fvattn_rope* r, bool sub = false) {
  WsLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes);
    return at;
  };
  L.status = take(kAlign);
  L.tile_cube = take(sizeof(int) * g.nT);
  L.cube_rank = take(sizeof(int) * g.nT);
  L.tile_tok = take(sizeof(int) * (size_t)g.N);
  const size_t rope_pairs =
      rope_on(r) ? (size_t)g.T * (r->dt / 2) + (size_t)g.Hg * (r->dh / 2) + (size_t)g.W * (r->dw / 2) : 0;
  L.rope_tab = take(sizeof(float2) * rope_pairs);
  const size_t pooled = sizeof(float) * (size_t)g.BH * g.nT * g.d;
  L.qh = take(pooled);
  L.ql = take(pooled);
  L.kh = take(pooled);
  L.kl = take(pooled);
  L.scores = take(sizeof(float) * (size_t)g.BH * g.nT * g.nT);
  L.counts = take(sizeof(int) * (size_t)g.BH * g.nT);
  L.idx = take(sizeof(int) * (size_t)g.BH * g.nT * g.nT);
  L.uni = take(sizeof(int) * (size_t)g.BH * g.P * g.nT);
  L.ucount = take(sizeof(int) * (size_t)g.BH * g.P);
  L.worklist = take(sizeof(int) * (size_t)g.BH * g.P);
  L.rank = take(sizeof(int) * (size_t)g.BH * g.P);
  L.useg = take(sizeof(int) * (size_t)g.BH * g.Qn);
  L.qcost = take(sizeof(int) * (size_t)g.BH * g.Qn);
  L.cta_times = take(sizeof(unsigned long long) * (1 + 2 * (size_t)kMaxCtas));
  L.cta_busy = take(sizeof(long long) * (size_t)kMaxCtas);
  L.next_slot = take(sizeof(int));
  // RoPE: the rotated K (tiled); the rotated Q goes to the caller's output buffer
  L.krot = take(rope_on(r) ? (size_t)g.BH * g.N * g.d * elem_size(dtype) : 0);
  if (sub) {
    const size_t sb = sizeof(float) * (size_t)g.BH * g.nT * kSubBlocks * g.d;
    L.sqh = take(sb);
    L.sql = take(sb);
    L.skh = take(sb);
    L.skl = take(sb);
    L.tmass = take(sizeof(float) * (size_t)g.BH * g.nT * kSubBlocks * g.nT);
  }
  L.total = off;
  return L;
}

// Prologue workspace: tables only.
WsLayout layout_qkv(const Geom& g, const fvattn_rope* r) {
  WsLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes);
    return at;
  };
  L.status = take(kAlign);
  L.tile_cube = take(sizeof(int) * g.nT);
  L.cube_rank = take(sizeof(int) * g.nT);
  L.tok_pos = take(sizeof(int) * (size_t)g.N);
  const size_t rope_pairs =
      rope_on(r) ? (size_t)g.T * (r->dt / 2) + (size_t)g.Hg * (r->dh / 2) + (size_t)g.W * (r->dw / 2) : 0;
  L.rope_pairs = take(sizeof(float2) * rope_pairs);
  L.total = off;
  return L;
}

// Backward workspace: both schedules, the transposed selection bitmap, D and lse * log2(e).
WsLayout layout_bwd(const Geom& g) {
  WsLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes);
    return at;
  };
  const size_t items = (size_t)g.BH * g.P;
  L.status = take(kAlign);
  L.uni = take(sizeof(int) * items * g.nT);
  L.ucount = take(sizeof(int) * items);
  L.worklist = take(sizeof(int) * items);
  L.rank = take(sizeof(int) * items);
  L.bits = take(sizeof(uint32_t) * (size_t)g.BH * g.nT * ((g.nT + 31) / 32));
  L.uni_t = take(sizeof(int) * items * g.nT);
  L.ucount_t = take(sizeof(int) * items);
  L.worklist_t = take(sizeof(int) * items);
  L.rank_t = take(sizeof(int) * items);
  L.lse2 = take(sizeof(float) * (size_t)g.BH * g.N);
  L.dd = take(sizeof(float) * (size_t)g.BH * g.N);
  L.total = off;
  return L;
}

struct DeviceInfo {
  int sms = 0;
  int major = 0;
};

int device_info(DeviceInfo* out) {
  static std::mutex mu;
  static DeviceInfo cache[64];
  int dev = 0;
  FV_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return FVATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev].sms == 0) {
    FV_CUDA(cudaDeviceGetAttribute(&cache[dev].sms, cudaDevAttrMultiProcessorCount, dev));
    FV_CUDA(cudaDeviceGetAttribute(&cache[dev].major, cudaDevAttrComputeCapabilityMajor, dev));
  }
  *out = cache[dev];
  if (out->major != 10) return FVATTN_ERR_UNSUPPORTED;
  return FVATTN_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// TMA descriptor over a bf16 [BH, N, 128] tensor, box = one 64-token tile x
// 64 head dims, 128-byte swizzle.  natural: 5D (d, W, Hg, T, BH) with a
// 64 x 4 x 4 x 4 box (one aligned cube); tiled: 3D (d, N, BH), 64 x 64 box.
int make_tile_map(CUtensorMap* map, const void* base, const Geom& g, bool natural) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return FVATTN_ERR_CUDA;
  const cuuint64_t row = (cuuint64_t)g.d * 2;
  CUresult r;
  if (natural) {
    const cuuint64_t dims[5] = {(cuuint64_t)g.d, (cuuint64_t)g.W, (cuuint64_t)g.Hg, (cuuint64_t)g.T,
                                (cuuint64_t)g.BH};
    const cuuint64_t strides[4] = {row, row * g.W, row * g.W * g.Hg, row * (cuuint64_t)g.N};
    const cuuint32_t box[5] = {64, 4, 4, 4, 1};
    const cuuint32_t es[5] = {1, 1, 1, 1, 1};
    r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  } else {
    const cuuint64_t dims[3] = {(cuuint64_t)g.d, (cuuint64_t)g.N, (cuuint64_t)g.BH};
    const cuuint64_t strides[2] = {row, row * (cuuint64_t)g.N};
    const cuuint32_t box[3] = {64, 64, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  }
  return r == CUDA_SUCCESS ? FVATTN_OK : FVATTN_ERR_CUDA;
}

// TMA descriptor over a pooled fp32 [BH, rows, d] tensor (tf32 operand of the
// score kernel; rows = nT tiles, or nT * 8 sub-blocks): 3D (d, rows, BH),
// box = 32 dims (128 bytes) x 128 rows, 128-byte swizzle; rows past the end
// read as zero.
int make_pooled_map(CUtensorMap* map, const float* base, const Geom& g, int rows = 0) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return FVATTN_ERR_CUDA;
  if (rows <= 0) rows = g.nT;
  const cuuint64_t row = (cuuint64_t)g.d * 4;
  const cuuint64_t dims[3] = {(cuuint64_t)g.d, (cuuint64_t)rows, (cuuint64_t)g.BH};
  const cuuint64_t strides[2] = {row, row * (cuuint64_t)rows};
  const cuuint32_t box[3] = {32, 128, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FVATTN_OK : FVATTN_ERR_CUDA;
}

// TMA descriptor over a bf16 [rows, cols] row-major matrix (cols a multiple
// of 64): box = box_k columns (64 -> 128-byte swizzle, 32 -> 64-byte
// swizzle) x box_rows rows; rows past the end read as zero.
int make_rows_map(CUtensorMap* map, const void* base, long long rows, int cols, int box_rows, int box_k) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return FVATTN_ERR_CUDA;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)box_k, (cuuint32_t)box_rows};
  const cuuint32_t es[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE,
                         box_k == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FVATTN_OK : FVATTN_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Optional per-stage timing with CUDA events (host objects only).
// ---------------------------------------------------------------------------
struct Profiler {
  std::mutex mu;
  bool on = false;
  struct Rec { int stage; cudaEvent_t a, b; int kernels; };
  std::vector<Rec> recs;
  std::vector<cudaEvent_t> pool;

  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
  }
};
Profiler& prof() {
  static Profiler p;
  return p;
}

bool profiling() {
  Profiler& p = prof();
  std::lock_guard<std::mutex> lock(p.mu);
  return p.on;
}

// Records events around one launch when profiling is on.
struct StageTimer {
  int stage;
  int kernels = 0;       // kernels this stage launched (for the launch count)
  cudaStream_t s;
  cudaEvent_t a = nullptr, b = nullptr;
  StageTimer(int st, cudaStream_t stream) : stage(st), s(stream) {
    Profiler& p = prof();
    std::lock_guard<std::mutex> lock(p.mu);
    if (!p.on) return;
    a = p.get();
    b = p.get();
    if (a && b) cudaEventRecord(a, s);
  }
  ~StageTimer() {
    if (!a || !b) return;
    cudaEventRecord(b, s);
    Profiler& p = prof();
    std::lock_guard<std::mutex> lock(p.mu);
    p.recs.push_back({stage, a, b, kernels});
  }
};

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Common prologue: shape, workspace, device.
struct Call {
  Geom g{};
  WsLayout L{};
  DeviceInfo dev{};
  char* ws = nullptr;
  int* status = nullptr;
  cudaStream_t s = nullptr;

  template <typename T>
  T* at(size_t off) const {
    return reinterpret_cast<T*>(ws + off);
  }
};

int begin(Call* c, const fvattn_shape* shape, const fvattn_rope* rope, void* ws, size_t ws_bytes,
          fvattn_stream_t stream, bool sub = false) {
  FV_TRY(make_geom(shape, &c->g));
  FV_TRY(check_rope(rope, c->g));
  if (!ws || !aligned(ws, kAlign)) return FVATTN_ERR_INVALID_ARG;
  c->L = layout_for(c->g, shape->dtype, rope, sub);
  if (ws_bytes < c->L.total) return FVATTN_ERR_WORKSPACE;
  FV_TRY(device_info(&c->dev));
  c->ws = static_cast<char*>(ws);
  c->status = c->at<int>(c->L.status);
  c->s = reinterpret_cast<cudaStream_t>(stream);
  FV_CUDA(cudaMemsetAsync(c->status, 0, sizeof(int), c->s));
  return FVATTN_OK;
}

// As begin(), with the workspace carved by `layout`.
template <typename F>
int begin_custom(Call* c, const fvattn_shape* shape, const fvattn_rope* rope, void* ws, size_t ws_bytes,
                 fvattn_stream_t stream, F layout) {
  FV_TRY(make_geom(shape, &c->g));
  FV_TRY(check_rope(rope, c->g));
  if (!ws || !aligned(ws, kAlign)) return FVATTN_ERR_INVALID_ARG;
  c->L = layout(c->g);
  if (ws_bytes < c->L.total) return FVATTN_ERR_WORKSPACE;
  FV_TRY(device_info(&c->dev));
  c->ws = static_cast<char*>(ws);
  c->status = c->at<int>(c->L.status);
  c->s = reinterpret_cast<cudaStream_t>(stream);
  FV_CUDA(cudaMemsetAsync(c->status, 0, sizeof(int), c->s));
  return FVATTN_OK;
}

int tables(const Call& c, const fvattn_rope* rope, bool need_tok) {
  StageTimer t(FVATTN_STAGE_TABLES, c.s);
  FV_CUDA(launch_tile_table(c.g, c.at<int>(c.L.tile_cube), c.at<int>(c.L.cube_rank), c.s));
  t.kernels = 1 + (need_tok ? 1 : 0) + (rope_on(rope) ? 1 : 0);
  if (need_tok) FV_CUDA(launch_tile_token(c.g, c.at<int>(c.L.cube_rank), c.at<int>(c.L.tile_tok), c.s));
  if (rope_on(rope))
    FV_CUDA(launch_rope_table(c.g, rope->dt, rope->dh, rope->dw, rope->base, c.at<float2>(c.L.rope_tab), c.s));
  return FVATTN_OK;
}

int check_blocks(const fvattn_blocks* b, const Geom& g) {
  if (!b || !b->counts || !b->idx) return FVATTN_ERR_INVALID_ARG;
  if (!aligned(b->counts, 4) || !aligned(b->idx, 4)) return FVATTN_ERR_INVALID_ARG;
  if (b->cap < g.nT) return FVATTN_ERR_CAPACITY;
  return FVATTN_OK;
}

// Pool (+ RoPE) and select into `blocks`.  qrot (RoPE only): where the
// rotated Q goes, in the call's layout (the fine stage's output buffer); the
// rotated K goes to the workspace, tiled.
int run_coarse(const Call& c, const fvattn_shape* shape, const void* q, const void* k, const fvattn_rope* rope,
               bool natural, bool pooled, void* qrot, float top_p, int k_min, const fvattn_blocks* blocks) {
  const bool rot = qrot != nullptr;
  const bool r = rope_on(rope);
  PooledOut po{};
  if (pooled) {
    po.hi[0] = c.at<float>(c.L.qh);
    po.lo[0] = c.at<float>(c.L.ql);
    po.hi[1] = c.at<float>(c.L.kh);
    po.lo[1] = c.at<float>(c.L.kl);
  }
  {
  StageTimer t(FVATTN_STAGE_POOL, c.s);
  FV_CUDA(launch_pool(c.g, shape->dtype, q, k, natural ? 1 : 0, c.at<int>(c.L.tile_cube), c.at<int>(c.L.tile_tok),
                      r ? 1 : 0, r ? rope->dt : 0, r ? rope->dh : 0, r ? rope->dw : 0, c.at<float2>(c.L.rope_tab),
                      po, qrot, rot ? c.at<void>(c.L.krot) : nullptr, c.s));
  t.kernels = 1;
  }
  if (!pooled) return FVATTN_OK;
  StageTimer t(FVATTN_STAGE_SELECT, c.s);
  CUtensorMap mqh, mql, mkh, mkl;
  FV_TRY(make_pooled_map(&mqh, po.hi[0], c.g));
  FV_TRY(make_pooled_map(&mql, po.lo[0], c.g));
  FV_TRY(make_pooled_map(&mkh, po.hi[1], c.g));
  FV_TRY(make_pooled_map(&mkl, po.lo[1], c.g));
  ScoreArgs sa{c.g, c.at<float>(c.L.scores), c.status, kDefaultWaitCap};
  FV_CUDA(launch_scores(mqh, mql, mkh, mkl, sa, c.s));
  t.kernels = 1;
  if (!blocks) return FVATTN_OK;   // coarse logits only
  FV_CUDA(launch_select(c.g, sa.S, top_p, k_min, blocks->counts, blocks->idx, blocks->cap, c.s));
  t.kernels = 2;
  return FVATTN_OK;
}

// Heads per group of the fine stage's work list.  A head whose K and V take
// more than a quarter of the 126 MB L2 is evicted by the others when the
// longest-first order interleaves all heads, so such heads are grouped
// (groups of about 40 MB of K/V, at least one head: at 720p, 39 MB a head,
// 31.3 -> 29.2 ms); smaller heads keep one order over all of them, whose
// load balance is better (at 480p, 17 MB a head, 2.43 ms ungrouped, 2.48 in
// groups of two heads: the CTA busy-time ratio max/mean rises 1.06 -> 1.11).
// The forward's own work list ranks items by union size in buckets of 16
// entries (8 steps), ties by item code: within a bucket the items run head
// by head, so the CTAs running together share fewer heads' K/V in the L2
// (480p: DRAM reads of the fine stage 3.27 -> 2.30 GB a launch, same time),
// and a bucket's spread is small against the tail the light items fill.
constexpr int kLptShift = 4;
#ifndef FVATTN_FT_DYNAMIC
#define FVATTN_FT_DYNAMIC 1
#endif
constexpr bool kFineDynamic = FVATTN_FT_DYNAMIC != 0;
int heads_per_group(const Geom& g, int dtype) {
  const double per_head = 2.0 * (double)g.N * g.d * elem_size(dtype);
  if (per_head <= 126.0e6 / 4) return g.BH;
  const int h = (int)(40.0e6 / per_head);
  return h < 1 ? 1 : h;
}

// head_grouped: the fine stage's own work list, longest first (in buckets of
// 1 << kLptShift entries) within groups of heads_per_group heads (their K/V
// stay in L2 while the CTAs run them);
// otherwise one longest-first order over all items (fvattn_build_worklist,
// the augmentation's kept work list).
int run_schedule(const Call& c, const fvattn_blocks* blocks, int* worklist, int dtype = FVATTN_BF16,
                 bool head_grouped = false) {
  StageTimer t(FVATTN_STAGE_SCHEDULE, c.s);
  FV_CUDA(launch_union(c.g, blocks->counts, blocks->idx, blocks->cap, c.at<int>(c.L.uni), c.at<int>(c.L.ucount),
                       c.status, c.s));
  const int group = head_grouped ? heads_per_group(c.g, dtype) * c.g.P : 0;
  FV_CUDA(launch_rank(c.at<int>(c.L.ucount), c.g.BH * c.g.P, c.g.nT, group, head_grouped ? kLptShift : 0, worklist,
                      c.s));
  t.kernels = 2;      // union, counting sort
  return FVATTN_OK;
}

// Fine-stage kernel of the forward: 1 = quad items (fine_q_kernel, four
// query tiles sharing one K/V stream), 0 = two-tile items (fine_tc_kernel).
#ifndef FVATTN_FINE_QUAD
#define FVATTN_FINE_QUAD 0
#endif
constexpr bool kFineQuad = FVATTN_FINE_QUAD != 0;

// Schedule of the quad items of the forward's fine stage: union lists in
// the order both halves / A only / B only, and the longest-first work list.
int run_schedule_quad(const Call& c, const fvattn_blocks* blocks) {
  StageTimer t(FVATTN_STAGE_SCHEDULE, c.s);
  FV_CUDA(launch_quad_schedule(c.g, c.g.Qn, blocks->counts, blocks->idx, blocks->cap, c.at<int>(c.L.uni),
                               c.at<int>(c.L.ucount), c.at<int>(c.L.useg), c.at<int>(c.L.qcost),
                               c.at<int>(c.L.worklist), c.status, c.s));
  t.kernels = 2;      // quad unions, counting sort
  return FVATTN_OK;
}

// Fine stage.  Under RoPE, q is the rotated copy the coarse stage wrote into
// `out` (call layout) and k the rotated tiled copy in the workspace.
// worklist / grid: a caller's work list and persistent grid (default: the
// schedule's work list in the workspace and one CTA per SM).
int run_fine(const Call& c, const fvattn_shape* shape, const void* q, const void* k, const void* v,
             const fvattn_rope* rope, bool natural, const fvattn_blocks* blocks, void* out, float* lse,
             const int* worklist = nullptr, int grid = 0) {
  const bool r = rope_on(rope);
  const void* qs = r ? out : q;
  const void* ks = r ? c.at<void>(c.L.krot) : k;
  const bool k_nat = natural && !r;
  if (kFineQuad && shape->dtype == FVATTN_BF16 && !worklist) {
    // quad items over the schedule of run_schedule_quad
    CUtensorMap mq, mk, mv;
    FV_TRY(make_tile_map(&mq, qs, c.g, natural));
    FV_TRY(make_tile_map(&mk, ks, c.g, k_nat));
    FV_TRY(make_tile_map(&mv, v, c.g, natural));
    FineQArgs a{};
    a.g = c.g;
    a.cta_times = profiling() ? c.at<unsigned long long>(c.L.cta_times) : nullptr;
    a.uni = c.at<int>(c.L.uni);
    a.ucount = c.at<int>(c.L.ucount);
    a.useg = c.at<int>(c.L.useg);
    a.worklist = c.at<int>(c.L.worklist);
    a.n_items = c.g.BH * c.g.Qn;
    a.Qn = c.g.Qn;
    a.tile_cube = c.at<int>(c.L.tile_cube);
    a.q_nat = natural;
    a.k_nat = k_nat;
    a.v_nat = natural;
    a.out = static_cast<__nv_bfloat16*>(out);
    a.lse = lse;
    a.out_nat = natural;
    a.status = c.status;
    a.wait_cap = kDefaultWaitCap;
    StageTimer t(FVATTN_STAGE_FINE, c.s);
    FV_CUDA(launch_fine_q(mq, mk, mv, a, grid > 0 ? grid : c.dev.sms, c.s));
    t.kernels = a.n_items > 0 ? 1 : 0;
  } else if (shape->dtype == FVATTN_BF16) {
    // two-tile items over a caller's work list (augmented lists)
    CUtensorMap mq, mk, mv;
    FV_TRY(make_tile_map(&mq, qs, c.g, natural));
    FV_TRY(make_tile_map(&mk, ks, c.g, k_nat));
    FV_TRY(make_tile_map(&mv, v, c.g, natural));
    FineTcArgs a{};
    a.g = c.g;
    a.cta_times = profiling() ? c.at<unsigned long long>(c.L.cta_times) : nullptr;
    a.uni = c.at<int>(c.L.uni);
    a.ucount = c.at<int>(c.L.ucount);
    a.worklist = worklist ? worklist : c.at<int>(c.L.worklist);
    a.n_items = c.g.BH * c.g.P;
    // the schedule's own list is handed out greedily (each CTA takes the next
    // slot when it starts an item) or serpentine; a caller's list (the
    // augmentation's kept work list, whose per-CTA loads assume CTA c runs
    // c, c + G, ...) keeps that static order
    a.snake = worklist ? 0 : 1;
    if (!worklist && kFineDynamic) {
      a.next_slot = c.at<int>(c.L.next_slot);
      FV_CUDA(cudaMemsetAsync(a.next_slot, 0, sizeof(int), c.s));
    }
    a.tile_cube = c.at<int>(c.L.tile_cube);
    a.q_nat = natural;
    a.k_nat = k_nat;
    a.v_nat = natural;
    a.out = static_cast<__nv_bfloat16*>(out);
    a.lse = lse;
    a.out_nat = natural;
    a.status = c.status;
    a.wait_cap = kDefaultWaitCap;
    StageTimer t(FVATTN_STAGE_FINE, c.s);
    FV_CUDA(launch_fine_tc(mq, mk, mv, a, grid > 0 ? grid : c.dev.sms, c.s));
    t.kernels = a.n_items > 0 ? 1 : 0;
  } else {
    FineF32Args a{};
    a.g = c.g;
    a.q = static_cast<const float*>(qs);
    a.k = static_cast<const float*>(ks);
    a.v = static_cast<const float*>(v);
    a.q_nat = natural;
    a.k_nat = k_nat;
    a.v_nat = natural;
    a.counts = blocks->counts;
    a.idx = blocks->idx;
    a.cap = blocks->cap;
    a.tile_cube = c.at<int>(c.L.tile_cube);
    a.out = static_cast<float*>(out);
    a.lse = lse;
    a.out_nat = natural;
    a.status = c.status;
    StageTimer t(FVATTN_STAGE_FINE, c.s);
    FV_CUDA(launch_fine_f32(a, c.s));
    t.kernels = 1;
  }
  return FVATTN_OK;
}

bool same_shape(const fvattn_shape& a, const fvattn_shape& b) {
  return a.batch == b.batch && a.heads == b.heads && a.head_dim == b.head_dim && a.grid.T == b.grid.T &&
         a.grid.H == b.grid.H && a.grid.W == b.grid.W && a.tile.t == b.tile.t && a.tile.h == b.tile.h &&
         a.tile.w == b.tile.w && a.dtype == b.dtype && a.order == b.order;
}

bool tensor_ok(const void* p) { return p && aligned(p, 16); }

}  // namespace

extern "C" {

int fvattn_num_tiles(const fvattn_shape* shape, int64_t* num_tiles) {
  Geom g;
  if (!num_tiles) return FVATTN_ERR_INVALID_ARG;
  FV_TRY(make_geom(shape, &g));
  *num_tiles = g.nT;
  return FVATTN_OK;
}

int fvattn_workspace_size(const fvattn_shape* shape, const fvattn_rope* rope, size_t* bytes) {
  Geom g;
  if (!bytes) return FVATTN_ERR_INVALID_ARG;
  FV_TRY(make_geom(shape, &g));
  FV_TRY(check_rope(rope, g));
  *bytes = layout_for(g, shape->dtype, rope).total;
  return FVATTN_OK;
}

int fvattn_tile_reorder(const fvattn_shape* shape, const void* x, void* y, int32_t row_bytes, int inverse, void* ws,
                        size_t ws_bytes, fvattn_stream_t stream) {
  if (!tensor_ok(x) || !tensor_ok(y) || x == y) return FVATTN_ERR_INVALID_ARG;
  if (row_bytes < 4 || row_bytes > 1024 || row_bytes % 4) return FVATTN_ERR_INVALID_ARG;
  Call c;
  FV_TRY(begin(&c, shape, nullptr, ws, ws_bytes, stream));
  FV_TRY(tables(c, nullptr, false));
  StageTimer t(FVATTN_STAGE_REORDER, c.s);
  FV_CUDA(launch_reorder(c.g, c.at<int>(c.L.cube_rank), x, y, row_bytes, inverse ? 1 : 0, c.dev.sms, c.s));
  t.kernels = 1;
  return FVATTN_OK;
}

int fvattn_pool_select(const fvattn_shape* shape, const void* q, const void* k, const fvattn_rope* rope, float top_p,
                       int32_t k_min, const fvattn_blocks* out, void* ws, size_t ws_bytes, fvattn_stream_t stream) {
  if (!tensor_ok(q) || !tensor_ok(k)) return FVATTN_ERR_INVALID_ARG;
  if (std::isnan(top_p) || k_min < 0) return FVATTN_ERR_INVALID_ARG;
  Call c;
  FV_TRY(begin(&c, shape, rope, ws, ws_bytes, stream));
  FV_TRY(check_blocks(out, c.g));
  const bool natural = shape->layout == FVATTN_LAYOUT_NATURAL;
  FV_TRY(tables(c, rope, rope_on(rope) && !natural));
  FV_TRY(run_coarse(c, shape, q, k, rope, natural, true, nullptr, top_p, k_min, out));
  return FVATTN_OK;
}

int fvattn_workspace_size_subblock(const fvattn_shape* shape, const fvattn_rope* rope, size_t* bytes) {
  if (!bytes) return FVATTN_ERR_INVALID_ARG;
  Geom g{};
  FV_TRY(make_geom(shape, &g));
  FV_TRY(check_rope(rope, g));
  *bytes = layout_for(g, shape->dtype, rope, true).total;
  return FVATTN_OK;
}

int fvattn_pool_select_subblock(const fvattn_shape* shape, const void* q, const void* k, const fvattn_rope* rope,
                                float top_p, int32_t k_min, const fvattn_blocks* out, void* ws, size_t ws_bytes,
                                fvattn_stream_t stream) {
  if (!tensor_ok(q) || !tensor_ok(k)) return FVATTN_ERR_INVALID_ARG;
  if (std::isnan(top_p) || k_min < 0) return FVATTN_ERR_INVALID_ARG;
  Call c;
  FV_TRY(begin(&c, shape, rope, ws, ws_bytes, stream, true));
  FV_TRY(check_blocks(out, c.g));
  const bool natural = shape->layout == FVATTN_LAYOUT_NATURAL;
  FV_TRY(tables(c, rope, !natural));
  const bool r = rope_on(rope);
  PooledOut po{};
  po.hi[0] = c.at<float>(c.L.sqh);
  po.lo[0] = c.at<float>(c.L.sql);
  po.hi[1] = c.at<float>(c.L.skh);
  po.lo[1] = c.at<float>(c.L.skl);
  {
    StageTimer t(FVATTN_STAGE_POOL, c.s);
    FV_CUDA(launch_pool_sub(c.g, shape->dtype, q, k, natural ? 1 : 0, c.at<int>(c.L.tile_cube),
                            c.at<int>(c.L.tile_tok), r ? 1 : 0, r ? rope->dt : 0, r ? rope->dh : 0, r ? rope->dw : 0,
                            c.at<float2>(c.L.rope_tab), po, c.s));
    t.kernels = 1;
  }
  StageTimer t(FVATTN_STAGE_SELECT, c.s);
  const int rows = c.g.nT * kSubBlocks;
  CUtensorMap mqh, mql, mkh, mkl;
  FV_TRY(make_pooled_map(&mqh, po.hi[0], c.g, rows));
  FV_TRY(make_pooled_map(&mql, po.lo[0], c.g, rows));
  FV_TRY(make_pooled_map(&mkh, po.hi[1], c.g, rows));
  FV_TRY(make_pooled_map(&mkl, po.lo[1], c.g, rows));
  ScoreArgs sa{c.g, c.at<float>(c.L.tmass), c.status, kDefaultWaitCap};
  FV_CUDA(launch_scores_sub(mqh, mql, mkh, mkl, sa, c.s));
  FV_CUDA(launch_subblock_agg(c.g, sa.S, c.at<float>(c.L.scores), c.s));
  FV_CUDA(launch_select(c.g, c.at<float>(c.L.scores), top_p, k_min, out->counts, out->idx, out->cap, c.s));
  t.kernels = 3;
  return FVATTN_OK;
}

int fvattn_build_worklist(const fvattn_shape* shape, const fvattn_blocks* blocks, int32_t* worklist, void* ws,
                          size_t ws_bytes, fvattn_stream_t stream) {
  if (!worklist || !aligned(worklist, 4)) return FVATTN_ERR_INVALID_ARG;
  Call c;
  FV_TRY(begin(&c, shape, nullptr, ws, ws_bytes, stream));
  FV_TRY(check_blocks(blocks, c.g));
  FV_TRY(run_schedule(c, blocks, worklist));
  return FVATTN_OK;
}

int fvattn_block_sparse_fwd(const fvattn_shape* shape, const void* q, const void* k, const void* v,
                            const fvattn_rope* rope, const fvattn_blocks* blocks, void* out, float* lse, void* ws,
                            size_t ws_bytes, fvattn_stream_t stream) {
  if (!tensor_ok(q) || !tensor_ok(k) || !tensor_ok(v) || !tensor_ok(out) || !lse || !aligned(lse, 4))
    return FVATTN_ERR_INVALID_ARG;
  Call c;
  FV_TRY(begin(&c, shape, rope, ws, ws_bytes, stream));
  FV_TRY(check_blocks(blocks, c.g));
  const bool natural = shape->layout == FVATTN_LAYOUT_NATURAL;
  FV_TRY(tables(c, rope, rope_on(rope) && !natural));
  if (rope_on(rope)) FV_TRY(run_coarse(c, shape, q, k, rope, natural, false, out, 0.f, 0, blocks));
  if (shape->dtype == FVATTN_BF16) FV_TRY(kFineQuad ? run_schedule_quad(c, blocks)
                                                   : run_schedule(c, blocks, c.at<int>(c.L.worklist), shape->dtype,
                                                                  true));
  FV_TRY(run_fine(c, shape, q, k, v, rope, natural, blocks, out, lse));
  return FVATTN_OK;
}

int fvattn_augment_lists(const fvattn_shape* shape, const void* q, const void* k, const fvattn_rope* rope,
                         const fvattn_blocks* base, int32_t num_ctas, const int64_t* cta_busy_ns,
                         int32_t fill_percent, const fvattn_blocks* out, int32_t* worklist, void* ws, size_t ws_bytes,
                         fvattn_stream_t stream) {
  if (!tensor_ok(q) || !tensor_ok(k) || !worklist || !aligned(worklist, 4)) return FVATTN_ERR_INVALID_ARG;
  if (num_ctas < 0 || num_ctas > 1024) return FVATTN_ERR_INVALID_ARG;
  if (cta_busy_ns && (fill_percent < 0 || fill_percent > 100)) return FVATTN_ERR_INVALID_ARG;
  Call c;
  FV_TRY(begin(&c, shape, rope, ws, ws_bytes, stream));
  FV_TRY(check_blocks(base, c.g));
  FV_TRY(check_blocks(out, c.g));
  const int items = c.g.BH * c.g.P;
  int G = num_ctas > 0 ? num_ctas : c.dev.sms;
  if (G > items) G = items;
  if (G > 1024) G = 1024;
  if (cta_busy_ns)
    for (int i = 0; i < G; ++i)
      if (cta_busy_ns[i] < 0 || cta_busy_ns[i] >= (1ll << 40)) return FVATTN_ERR_INVALID_ARG;
  const bool natural = shape->layout == FVATTN_LAYOUT_NATURAL;
  FV_TRY(tables(c, rope, rope_on(rope) && !natural));
  FV_TRY(run_coarse(c, shape, q, k, rope, natural, true, nullptr, 0.f, 0, nullptr));
  FV_TRY(run_schedule(c, base, worklist));
  long long* busy = nullptr;
  if (cta_busy_ns) {
    busy = c.at<long long>(c.L.cta_busy);
    FV_CUDA(cudaMemcpyAsync(busy, cta_busy_ns, sizeof(long long) * (size_t)G, cudaMemcpyHostToDevice, c.s));
  }
  StageTimer t(FVATTN_STAGE_SCHEDULE, c.s);
  // the rank buffer is free once the work list is built: it holds the per-item extra tiles
  FV_CUDA(launch_augment(c.g, c.at<float>(c.L.scores), base->counts, base->idx, base->cap, c.at<int>(c.L.ucount),
                         worklist, G, busy, fill_percent, c.at<int>(c.L.rank), out->counts, out->idx, out->cap,
                         c.status, c.s));
  t.kernels = 2;
  return FVATTN_OK;
}

int fvattn_block_sparse_fwd_worklist(const fvattn_shape* shape, const void* q, const void* k, const void* v,
                                     const fvattn_rope* rope, const fvattn_blocks* blocks, const int32_t* worklist,
                                     int32_t num_ctas, void* out, float* lse, void* ws, size_t ws_bytes,
                                     fvattn_stream_t stream) {
  if (!tensor_ok(q) || !tensor_ok(k) || !tensor_ok(v) || !tensor_ok(out) || !lse || !aligned(lse, 4))
    return FVATTN_ERR_INVALID_ARG;
  if (!worklist || !aligned(worklist, 4) || num_ctas < 0) return FVATTN_ERR_INVALID_ARG;
  Call c;
  FV_TRY(begin(&c, shape, rope, ws, ws_bytes, stream));
  FV_TRY(check_blocks(blocks, c.g));
  const bool natural = shape->layout == FVATTN_LAYOUT_NATURAL;
  FV_TRY(tables(c, rope, rope_on(rope) && !natural));
  if (rope_on(rope)) FV_TRY(run_coarse(c, shape, q, k, rope, natural, false, out, 0.f, 0, blocks));
  {
    StageTimer t(FVATTN_STAGE_SCHEDULE, c.s);
    FV_CUDA(launch_union(c.g, blocks->counts, blocks->idx, blocks->cap, c.at<int>(c.L.uni), c.at<int>(c.L.ucount),
                         c.status, c.s));
    t.kernels = 1;
  }
  FV_TRY(run_fine(c, shape, q, k, v, rope, natural, blocks, out, lse, worklist, num_ctas));
  return FVATTN_OK;
}

int fvattn_timestep_params(int32_t step, int32_t num_steps, float p_start, float p_end, int32_t k_start,
                           int32_t k_end, int32_t dense_steps, float* top_p, int32_t* k_min) {
  if (!top_p || !k_min || num_steps < 1 || step < 0 || step >= num_steps || dense_steps < 0) return FVATTN_ERR_INVALID_ARG;
  if (std::isnan(p_start) || std::isnan(p_end) || k_start < 0 || k_end < 0) return FVATTN_ERR_INVALID_ARG;
  if (step < dense_steps) {
    *top_p = 1.f;
    *k_min = k_start;
    return FVATTN_OK;
  }
  const int span = num_steps - dense_steps - 1;
  double f = span <= 0 ? 0.0 : (double)(step - dense_steps) / span;
  f = f < 0.0 ? 0.0 : (f > 1.0 ? 1.0 : f);
  *top_p = (float)(p_start + (p_end - (double)p_start) * f);
  *k_min = (int32_t)std::floor(k_start + (k_end - (double)k_start) * f + 0.5);
  return FVATTN_OK;
}

int fvattn_forward(const fvattn_shape* shape, const void* q, const void* k, const void* v, const fvattn_rope* rope,
                   float top_p, int32_t k_min, fvattn_mask_cache* cache, int reuse_mask, void* out, float* lse,
                   void* ws, size_t ws_bytes, fvattn_stream_t stream) {
  if (!shape) return FVATTN_ERR_INVALID_ARG;
  if (!tensor_ok(q) || !tensor_ok(k) || !tensor_ok(v) || !tensor_ok(out) || !lse || !aligned(lse, 4))
    return FVATTN_ERR_INVALID_ARG;
  if (std::isnan(top_p) || k_min < 0) return FVATTN_ERR_INVALID_ARG;
  fvattn_shape sh = *shape;
  sh.layout = FVATTN_LAYOUT_NATURAL;
  Call c;
  FV_TRY(begin(&c, &sh, rope, ws, ws_bytes, stream));
  fvattn_blocks local{c.at<int>(c.L.counts), c.at<int>(c.L.idx), c.g.nT};
  const fvattn_blocks* blocks = &local;
  if (reuse_mask) {
    if (!cache || !cache->valid || !same_shape(cache->shape, sh)) return FVATTN_ERR_CACHE_MISMATCH;
    blocks = &cache->blocks;
    FV_TRY(check_blocks(blocks, c.g));
  } else if (cache) {
    blocks = &cache->blocks;
    FV_TRY(check_blocks(blocks, c.g));
  }
  FV_TRY(tables(c, rope, false));
  if (!reuse_mask) {
    FV_TRY(run_coarse(c, &sh, q, k, rope, true, true, rope_on(rope) ? out : nullptr, top_p, k_min, blocks));
  } else if (rope_on(rope)) {
    FV_TRY(run_coarse(c, &sh, q, k, rope, true, false, out, 0.f, 0, blocks));
  }
  if (sh.dtype == FVATTN_BF16) FV_TRY(kFineQuad ? run_schedule_quad(c, blocks)
                                               : run_schedule(c, blocks, c.at<int>(c.L.worklist), sh.dtype, true));
  FV_TRY(run_fine(c, &sh, q, k, v, rope, true, blocks, out, lse));
  if (cache && !reuse_mask) {
    cache->shape = sh;
    cache->top_p = top_p;
    cache->k_min = k_min;
    cache->valid = 1;
  }
  return FVATTN_OK;
}

int fvattn_workspace_size_bwd(const fvattn_shape* shape, size_t* bytes) {
  if (!bytes) return FVATTN_ERR_INVALID_ARG;
  Geom g{};
  FV_TRY(make_geom(shape, &g));
  *bytes = layout_bwd(g).total;
  return FVATTN_OK;
}

int fvattn_block_sparse_bwd(const fvattn_shape* shape, const void* q, const void* k, const void* v, const void* out,
                            const void* dout, const float* lse, const fvattn_blocks* blocks, void* dq, void* dk,
                            void* dv, void* ws, size_t ws_bytes, fvattn_stream_t stream) {
  if (!tensor_ok(q) || !tensor_ok(k) || !tensor_ok(v) || !tensor_ok(out) || !tensor_ok(dout) || !tensor_ok(lse) ||
      !tensor_ok(dq) || !tensor_ok(dk) || !tensor_ok(dv))
    return FVATTN_ERR_INVALID_ARG;
  if (!shape) return FVATTN_ERR_INVALID_ARG;
  if (shape->dtype != FVATTN_BF16) return FVATTN_ERR_DTYPE;
  if (shape->layout != FVATTN_LAYOUT_TILED) return FVATTN_ERR_UNSUPPORTED;
  Call c;
  FV_TRY(begin_custom(&c, shape, nullptr, ws, ws_bytes, stream, [](const Geom& g) { return layout_bwd(g); }));
  FV_TRY(check_blocks(blocks, c.g));
  const Geom& g = c.g;
  {
    StageTimer t(FVATTN_STAGE_SCHEDULE, c.s);
    FV_CUDA(launch_union(g, blocks->counts, blocks->idx, blocks->cap, c.at<int>(c.L.uni), c.at<int>(c.L.ucount),
                         c.status, c.s));
    const int group = heads_per_group(g, FVATTN_BF16) * g.P;   // longest first within L2-sized head groups
    FV_CUDA(launch_rank(c.at<int>(c.L.ucount), g.BH * g.P, g.nT, group, 0, c.at<int>(c.L.worklist), c.s));
    FV_CUDA(launch_key_union(g, blocks->counts, blocks->idx, blocks->cap, c.at<uint32_t>(c.L.bits),
                             c.at<int>(c.L.uni_t), c.at<int>(c.L.ucount_t), c.status, c.s));
    FV_CUDA(launch_rank(c.at<int>(c.L.ucount_t), g.BH * g.P, g.nT, group, 0, c.at<int>(c.L.worklist_t), c.s));
    t.kernels = 5;   // union, 2 x counting sort, transpose bits, key union
  }
  CUtensorMap mq, mk, mv, mdo;
  FV_TRY(make_tile_map(&mq, q, g, false));
  FV_TRY(make_tile_map(&mk, k, g, false));
  FV_TRY(make_tile_map(&mv, v, g, false));
  FV_TRY(make_tile_map(&mdo, dout, g, false));
  {
    StageTimer t(FVATTN_STAGE_BWD_PREP, c.s);
    FV_CUDA(launch_bwd_prep(out, dout, lse, c.at<float>(c.L.lse2), c.at<float>(c.L.dd), (long long)g.BH * g.N, c.s));
    t.kernels = 1;
  }
  BwdArgs a{};
  a.g = g;
  a.n_items = g.BH * g.P;
  a.lse2 = c.at<float>(c.L.lse2);
  a.dd = c.at<float>(c.L.dd);
  a.scale = g.scale;
  a.scale_log2 = g.scale * 1.4426950408889634f;
  a.status = c.status;
  a.wait_cap = kDefaultWaitCap;
  // key-stationary: X = (K, V), Y = (Q, dO) -> dK, dV
  a.uni = c.at<int>(c.L.uni_t);
  a.ucount = c.at<int>(c.L.ucount_t);
  a.worklist = c.at<int>(c.L.worklist_t);
  a.out0 = static_cast<__nv_bfloat16*>(dk);
  a.out1 = static_cast<__nv_bfloat16*>(dv);
  {
    StageTimer t(FVATTN_STAGE_BWD_KV, c.s);
    FV_CUDA(launch_bwd(mk, mv, mq, mdo, a, true, c.dev.sms, c.s));
    t.kernels = 1;
  }
  // query-stationary: X = (Q, dO), Y = (K, V) -> dQ
  a.uni = c.at<int>(c.L.uni);
  a.ucount = c.at<int>(c.L.ucount);
  a.worklist = c.at<int>(c.L.worklist);
  a.out0 = static_cast<__nv_bfloat16*>(dq);
  a.out1 = nullptr;
  StageTimer t(FVATTN_STAGE_BWD_Q, c.s);
  FV_CUDA(launch_bwd(mq, mdo, mk, mv, a, false, c.dev.sms, c.s));
  t.kernels = 1;
  return FVATTN_OK;
}

int fvattn_workspace_size_qkv(const fvattn_shape* shape, const fvattn_rope* rope, size_t* bytes) {
  if (!bytes) return FVATTN_ERR_INVALID_ARG;
  Geom g{};
  FV_TRY(make_geom(shape, &g));
  FV_TRY(check_rope(rope, g));
  *bytes = layout_qkv(g, rope).total;
  return FVATTN_OK;
}

#ifndef FVATTN_QKV_VARIANT
#define FVATTN_QKV_VARIANT 1   // 128 x 256 tiles, double-buffered accumulators
#endif
#ifndef FVATTN_QKV_GROUP_M
#define FVATTN_QKV_GROUP_M 16   // row tiles per band (16 beat 4, 8 and 32 at 720p)
#endif

int fvattn_qkv_rope(const fvattn_shape* shape, const void* x, int32_t channels, const void* w, const float* bias,
                    const fvattn_rope* rope, int32_t t_offset, void* q, void* k, void* v, void* ws, size_t ws_bytes,
                    fvattn_stream_t stream) {
  if (!tensor_ok(x) || !tensor_ok(w) || !tensor_ok(q) || !tensor_ok(k) || !tensor_ok(v))
    return FVATTN_ERR_INVALID_ARG;
  if (bias && !aligned(bias, 16)) return FVATTN_ERR_INVALID_ARG;
  if (t_offset < 0 || t_offset > (1 << 20)) return FVATTN_ERR_INVALID_ARG;
  if (!shape) return FVATTN_ERR_INVALID_ARG;
  if (shape->dtype != FVATTN_BF16) return FVATTN_ERR_DTYPE;
  if (channels < 64 || channels > 65536 || channels % 64) return FVATTN_ERR_SHAPE;
  Call c;
  FV_TRY(begin_custom(&c, shape, rope, ws, ws_bytes, stream, [&](const Geom& g) { return layout_qkv(g, rope); }));
  const Geom& g = c.g;
  const bool tiled = shape->layout == FVATTN_LAYOUT_TILED;
  const bool r = rope_on(rope);
  {
    StageTimer t(FVATTN_STAGE_TABLES, c.s);
    if (tiled) {
      FV_CUDA(launch_tile_table(g, c.at<int>(c.L.tile_cube), c.at<int>(c.L.cube_rank), c.s));
      FV_CUDA(launch_token_pos(g, c.at<int>(c.L.cube_rank), c.at<int>(c.L.tok_pos), c.s));
      t.kernels += 2;
    }
    if (r) {
      FV_CUDA(launch_rope_pairs(g, rope->dt, rope->dh, rope->dw, rope->base, t_offset, c.at<float2>(c.L.rope_pairs),
                                c.s));
      t.kernels += 1;
    }
  }
  const int variant = FVATTN_QKV_VARIANT;
  const long long M = (long long)g.B * g.N;
  const int Nout = 3 * g.H * g.d;
  const QkvTma tm = qkv_tma(variant);
  CUtensorMap mx, mw;
  FV_TRY(make_rows_map(&mx, x, M, channels, tm.box_rows, tm.box_k));
  FV_TRY(make_rows_map(&mw, w, Nout, channels, 256, tm.box_k));
  QkvArgs a{};
  a.bias = bias;
  a.out[0] = static_cast<__nv_bfloat16*>(q);
  a.out[1] = static_cast<__nv_bfloat16*>(k);
  a.out[2] = static_cast<__nv_bfloat16*>(v);
  a.pos = tiled ? c.at<int>(c.L.tok_pos) : nullptr;
  a.rope_tab = r ? c.at<float2>(c.L.rope_pairs) : nullptr;
  a.dt = r ? rope->dt : 0;
  a.dh = r ? rope->dh : 0;
  a.dw = r ? rope->dw : 0;
  a.M = (int)M;
  a.N = g.N;
  a.H = g.H;
  a.T = g.T;
  a.Hg = g.Hg;
  a.W = g.W;
  a.Nout = Nout;
  a.kblocks = channels / tm.box_k;
  a.group_m = FVATTN_QKV_GROUP_M;
  a.status = c.status;
  a.wait_cap = kDefaultWaitCap;
  StageTimer t(FVATTN_STAGE_PROLOGUE, c.s);
  FV_CUDA(launch_qkv(mx, mw, a, variant, c.dev.sms, c.s));
  t.kernels = 1;
  return FVATTN_OK;
}

int fvattn_get_device_status(void* ws, fvattn_stream_t stream, int32_t* status) {
  if (!ws || !status) return FVATTN_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  FV_CUDA(cudaStreamSynchronize(s));
  int v = 0;
  FV_CUDA(cudaMemcpy(&v, ws, sizeof(int), cudaMemcpyDeviceToHost));
  FV_CUDA(cudaMemset(ws, 0, sizeof(int)));
  *status = v;
  return FVATTN_OK;
}

int fvattn_selftest_wait_timeout(void* ws, size_t ws_bytes, int64_t cap_iterations, fvattn_stream_t stream) {
  if (!ws || !aligned(ws, kAlign) || ws_bytes < kAlign || cap_iterations < 1) return FVATTN_ERR_INVALID_ARG;
  DeviceInfo dev;
  FV_TRY(device_info(&dev));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  FV_CUDA(cudaMemsetAsync(ws, 0, sizeof(int), s));
  FV_CUDA(launch_wait_selftest(static_cast<int*>(ws), cap_iterations, s));
  return FVATTN_OK;
}

int fvattn_profile_enable(int enable) {
  Profiler& p = prof();
  std::lock_guard<std::mutex> lock(p.mu);
  p.on = enable != 0;
  return FVATTN_OK;
}

int fvattn_profile_read(double* ms, int64_t* launches) {
  Profiler& p = prof();
  std::lock_guard<std::mutex> lock(p.mu);
  double acc[FVATTN_STAGE_COUNT] = {0};
  int64_t cnt[FVATTN_STAGE_COUNT] = {0};
  int st = FVATTN_OK;
  for (auto& r : p.recs) {
    float t = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
      st = FVATTN_ERR_CUDA;
    acc[r.stage] += t;
    cnt[r.stage] += r.kernels;
    p.pool.push_back(r.a);
    p.pool.push_back(r.b);
  }
  p.recs.clear();
  for (int i = 0; i < FVATTN_STAGE_COUNT; ++i) {
    if (ms) ms[i] = acc[i];
    if (launches) launches[i] = cnt[i];
  }
  return st;
}

int fvattn_profile_cta_times(const fvattn_shape* shape, const fvattn_rope* rope, void* ws, fvattn_stream_t stream,
                             int64_t* ns, int32_t capacity, int32_t* num_ctas) {
  if (!ws || !ns || !num_ctas || capacity < 0) return FVATTN_ERR_INVALID_ARG;
  Geom g{};
  FV_TRY(make_geom(shape, &g));
  FV_TRY(check_rope(rope, g));
  const WsLayout L = layout_for(g, shape->dtype, rope);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  FV_CUDA(cudaStreamSynchronize(s));
  unsigned long long n = 0;
  const char* base = static_cast<const char*>(ws) + L.cta_times;
  FV_CUDA(cudaMemcpy(&n, base, sizeof(n), cudaMemcpyDeviceToHost));
  if (n > (unsigned long long)kMaxCtas) return FVATTN_ERR_DEVICE;
  const int32_t m = (int32_t)n < capacity ? (int32_t)n : capacity;
  if (m > 0) FV_CUDA(cudaMemcpy(ns, base + sizeof(unsigned long long), sizeof(int64_t) * 2 * (size_t)m,
                                cudaMemcpyDeviceToHost));
  *num_ctas = (int32_t)n;
  return FVATTN_OK;
}

const char* fvattn_status_string(int status) {
  switch (status) {
    case FVATTN_OK: return "ok";
    case FVATTN_ERR_INVALID_ARG: return "invalid argument";
    case FVATTN_ERR_SHAPE: return "unsupported or inconsistent shape";
    case FVATTN_ERR_DTYPE: return "unsupported dtype";
    case FVATTN_ERR_CAPACITY: return "block list capacity smaller than the number of tiles";
    case FVATTN_ERR_CUDA: return "CUDA call failed";
    case FVATTN_ERR_CACHE_MISMATCH: return "mask cache not valid for this shape";
    case FVATTN_ERR_DEVICE: return "a kernel reported an error";
    case FVATTN_ERR_WORKSPACE: return "workspace too small";
    case FVATTN_ERR_UNSUPPORTED: return "unsupported device or combination";
    default: return "unknown status";
  }
}

}  // extern "C"
