// Internal declarations shared by the fvattn CUDA sources (sm_100a only).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fvattn.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "fvattn kernels are written for sm_100a (B200) only"
#endif

namespace fvattn {

constexpr int kTileTokens = 64;
constexpr int kItemTiles = 2;   // query tiles per fine-stage work item (one 128-row tile)
constexpr int kSubBlocks = 8;   // 2x2x2 sub-cubes of a tile in sub-block scoring
constexpr int kMaxTiles = 8192;
constexpr int kMaxCtas = 1024;  // persistent grid bound (fine-stage CTA time record)

// Global nanosecond timer (the same clock on every SM).
__device__ inline unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Device status codes (workspace status word).
constexpr int kStatusBadBlock = 1;
constexpr int kStatusWaitCap = 2;

// Default iteration cap of a bounded wait: on the order of a second.
constexpr long long kDefaultWaitCap = 1ll << 24;

// ---------------------------------------------------------------------------
// Problem geometry passed to kernels by value.
// ---------------------------------------------------------------------------
struct Geom {
  int B, H, d;
  int T, Hg, W;          // latent grid
  int nt, nh, nw;        // tile grid
  int nT;                // tiles per head
  int N;                 // tokens per head
  int BH;
  int P;                 // two-tile work items per head = ceil(nT / kItemTiles)
  int Qn;                // quad work items per head = ceil(nT / 4)
  int order;             // fvattn_order
  float scale;           // softmax scale
};

// Workspace carve-up (byte offsets from the workspace base).
struct WsLayout {
  size_t status;         // int32 status word + padding
  size_t tile_cube;      // int32 [nT]: packed (ct<<20 | ch<<10 | cw) of tile rank j
  size_t cube_rank;      // int32 [nT]: tile rank of raster cube id
  size_t tile_tok;       // int32 [N]: natural token index of each tiled row
  size_t rope_tab;       // float2 [(T*dt + Hg*dh + W*dw)/2]: (cos, sin)
  size_t qh, ql;         // float [BH*nT*d] pooled Q as tf32 hi + lo
  size_t kh, kl;         // float [BH*nT*d] pooled K as tf32 hi + lo
  size_t scores;         // float [BH*nT*nT] scaled coarse logits
  size_t counts, idx;    // int32 [BH*nT], [BH*nT*nT] (forward without cache)
  size_t uni, ucount;    // int32 [BH*P*nT], [BH*P]
  size_t worklist;       // int32 [BH*P]
  size_t useg, qcost;    // int32 [BH*Qn] quad items: union segments and cost
  size_t cta_times;      // u64 [1 + 2 * kMaxCtas] fine-stage CTA start / end times (profiling)
  size_t cta_busy;       // i64 [kMaxCtas] measured CTA busy times for the augmentation's slack
  size_t next_slot;      // int32 work-list counter of the fine stage's greedy dispatch
  size_t rank;           // int32 [BH*P] scratch of the work-list sort
  size_t krot;           // dtype [BH*N*d] rotated K, tiled (rope only)
  size_t sqh, sql;       // sub-block scoring only: float [BH*nT*8*d] pooled sub-blocks of Q (tf32 hi + lo)
  size_t skh, skl;       //   ... of K
  size_t tmass;          //   float [BH*nT*8*nT] log2 key-tile masses per query sub-block
  size_t bits;           // backward only: u32 [BH*nT*ceil(nT/32)] transposed selection bitmap
  size_t uni_t, ucount_t;  //   union lists of key-tile pairs
  size_t worklist_t, rank_t;
  size_t lse2, dd;       //   float [BH*N] lse * log2(e) and rowsum(dout * out)
  size_t tok_pos;        // prologue only: int32 [N] tiled row of natural token n
  size_t rope_pairs;     //   float2 pair-major (cos, sin) table at the start-frame offset
  size_t total;
};

// Kernel arguments filled by the host entry points.
struct RopeArgs {
  int enabled, dt, dh, dw;
  const float2* tab;     // [T*dt/2 | Hg*dh/2 | W*dw/2]
};

// Pooled means split into tf32 hi/lo parts; [0] = Q, [1] = K.
struct PooledOut {
  float* hi[2];
  float* lo[2];
};

struct ScoreArgs {
  Geom g;
  float* S;              // [BH][nT][nT]
  int* status;
  long long wait_cap;
};

struct FineTcArgs {
  Geom g;
  unsigned long long* cta_times;   // optional: [0] = CTAs, then per CTA (start, end) in ns
  const int* uni;
  const int* ucount;
  const int* worklist;
  int n_items;
  int snake;             // 1: serpentine slots (the forward's own list); 0: CTA c runs c, c + G, ...
  int* next_slot;        // optional: zeroed counter; CTA c starts with slot c and then takes
                         // slot G + atomicAdd(next_slot, 1) when it starts an item (greedy)
  const int* tile_cube;
  int q_nat, k_nat, v_nat;
  __nv_bfloat16* out;
  float* lse;
  int out_nat;
  int* status;
  long long wait_cap;
};

// Fine stage over quad items (four query tiles in two 128-row halves).
struct FineQArgs {
  Geom g;
  unsigned long long* cta_times;   // optional: [0] = CTAs, then per CTA (start, end) in ns
  const int* uni;        // [items][nT] union entries (key tile | selection bits << 16)
  const int* ucount;     // [items] entries
  const int* useg;       // [items] entries of both halves | entries of half A only << 16
  const int* worklist;   // [items] longest first
  int n_items;
  int Qn;                // quad items per (batch, head) = ceil(nT / 4)
  const int* tile_cube;
  int q_nat, k_nat, v_nat;
  __nv_bfloat16* out;
  float* lse;
  int out_nat;
  int* status;
  long long wait_cap;
};

// Prologue: Q | K | V = X W^T (+ bias), RoPE on Q and K, bf16 out.
struct QkvArgs {
  const float* bias;       // [Nout] or null
  __nv_bfloat16* out[3];   // q, k, v: [B, H, N, 128]
  const int* pos;          // [N] output row of natural token n, or null (natural layout)
  const float2* rope_tab;  // pair-major: [dt/2][T] | [dh/2][Hg] | [dw/2][W] (cos, sin), or null
  int dt, dh, dw;
  int M;                   // B * N rows of X
  int N, H, T, Hg, W;
  int Nout;                // 3 * H * 128 rows of W
  int kblocks;             // C / 64
  int mt, nt, n_tiles, group_m;
  int* status;
  long long wait_cap;
};

// Backward of the fine stage (both kernels of the template).
struct BwdArgs {
  Geom g;
  const int* uni;          // union lists of the items (key-stationary: of key-tile pairs)
  const int* ucount;
  const int* worklist;
  int n_items;
  const float* lse2;       // [BH, N] lse * log2(e), tiled rows
  const float* dd;         // [BH, N] rowsum(dout * out)
  __nv_bfloat16* out0;     // dK (key-stationary) or dQ
  __nv_bfloat16* out1;     // dV (key-stationary)
  float scale, scale_log2;
  int* status;
  long long wait_cap;
};

struct FineF32Args {
  Geom g;
  const float* q;
  const float* k;
  const float* v;
  int q_nat, k_nat, v_nat;
  const int* counts;
  const int* idx;
  int cap;
  const int* tile_cube;
  float* out;
  float* lse;
  int out_nat;
  int* status;
};

__host__ __device__ inline int pack_cube(int ct, int ch, int cw) { return (ct << 20) | (ch << 10) | cw; }
__host__ __device__ inline int cube_t(int p) { return p >> 20; }
__host__ __device__ inline int cube_h(int p) { return (p >> 10) & 1023; }
__host__ __device__ inline int cube_w(int p) { return p & 1023; }

// Natural token index of row r (0..63, raster inside the cube) of a cube.
__device__ inline int cube_row_token(const Geom& g, int packed, int r) {
  int t = cube_t(packed) * 4 + (r >> 4);
  int h = cube_h(packed) * 4 + ((r >> 2) & 3);
  int w = cube_w(packed) * 4 + (r & 3);
  return (t * g.Hg + h) * g.W + w;
}

__device__ inline void set_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Vector load / store of DPL consecutive elements as fp32.
template <typename T, int DPL> struct Vec;
template <int DPL> struct Vec<float, DPL> {
  static __device__ inline void load(const float* p, float (&v)[DPL]) {
    if constexpr (DPL == 4) {
      const float4 t = *reinterpret_cast<const float4*>(p);
      v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    } else if constexpr (DPL == 2) {
      const float2 t = *reinterpret_cast<const float2*>(p);
      v[0] = t.x; v[1] = t.y;
    } else {
#pragma unroll
      for (int i = 0; i < DPL; ++i) v[i] = p[i];
    }
  }
  static __device__ inline void store(float* p, const float (&v)[DPL]) {
    if constexpr (DPL == 4) {
      *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    } else if constexpr (DPL == 2) {
      *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
    } else {
#pragma unroll
      for (int i = 0; i < DPL; ++i) p[i] = v[i];
    }
  }
};
template <int DPL> struct Vec<__nv_bfloat16, DPL> {
  static_assert(DPL % 2 == 0, "bf16 rows are read in pairs");
  static __device__ inline void load(const __nv_bfloat16* p, float (&v)[DPL]) {
    uint32_t w[DPL / 2];
    if constexpr (DPL == 8) {
      const uint4 t = *reinterpret_cast<const uint4*>(p);
      w[0] = t.x; w[1] = t.y; w[2] = t.z; w[3] = t.w;
    } else if constexpr (DPL == 4) {
      const uint2 t = *reinterpret_cast<const uint2*>(p);
      w[0] = t.x; w[1] = t.y;
    } else {
#pragma unroll
      for (int i = 0; i < DPL / 2; ++i) w[i] = reinterpret_cast<const uint32_t*>(p)[i];
    }
#pragma unroll
    for (int i = 0; i < DPL / 2; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
  static __device__ inline void store(__nv_bfloat16* p, const float (&v)[DPL]) {
    uint32_t w[DPL / 2];
#pragma unroll
    for (int i = 0; i < DPL / 2; ++i) {
      __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&b);
    }
    if constexpr (DPL == 8) {
      *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    } else if constexpr (DPL == 4) {
      *reinterpret_cast<uint2*>(p) = make_uint2(w[0], w[1]);
    } else {
#pragma unroll
      for (int i = 0; i < DPL / 2; ++i) reinterpret_cast<uint32_t*>(p)[i] = w[i];
    }
  }
};

// ---------------------------------------------------------------------------
// PTX wrappers: shared-memory addresses, mbarriers, TMA, tcgen05.
// ---------------------------------------------------------------------------
__device__ inline uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ inline void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (TMA, tcgen05.mma operands) before a release that hands them over.
__device__ inline void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ inline void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ inline void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// One arrival for a converged warp: __syncwarp orders every lane's earlier
// memory operations (and tcgen05 fences) before lane 0's arrive.
__device__ inline void mbar_arrive_warp(uint64_t* bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

__device__ inline void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ inline bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of the phase with the given parity (for polling loops;
// try_wait may suspend the thread for a while before it reports failure).
__device__ inline bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity.  Gives up after `cap`
// polls, or as soon as another thread of the block raised `abort`; on
// giving up it raises `abort`, records kStatusWaitCap and returns false.
__device__ inline bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int* status,
                                 long long cap) {
  for (long long i = 0;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255) == 255 && *abort) return false;
    if (i >= cap) {
      *abort = 1;
      set_status(status, kStatusWaitCap);
      return false;
    }
  }
}

// One lane of a converged warp returns true (elect.sync over the full mask).
// Issuing tcgen05 work from an elected lane inside warp-uniform control flow
// keeps descriptors and TMEM addresses warp-uniform.
__device__ inline bool elect_one() {
  uint32_t p = 0;
  asm volatile(
      "{\n\t.reg .pred P;\n\t.reg .b32 L;\n\telect.sync L|P, 0xffffffff;\n\tselp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(p));
  return p != 0;
}

// mbar_wait by every lane of a converged warp; the result is lane 0's, so
// the warp leaves the wait together.
__device__ inline bool mbar_wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort, int* status,
                                      long long cap) {
  const bool ok = mbar_wait(bar, parity, abort, status, cap);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// Wait that ignores `abort`: used on the way out to let copies or MMAs that
// were already issued land before the block exits or frees TMEM.
__device__ inline bool mbar_drain(uint64_t* bar, uint32_t parity, int* status, long long cap) {
  for (long long i = 0; i < cap; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  set_status(status, kStatusWaitCap);
  return false;
}

__device__ inline void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

__device__ inline void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                   int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ inline void tma_load_5d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                   int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
      : "memory");
}

__device__ inline void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// tcgen05 --------------------------------------------------------------------
__device__ inline void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ inline void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ inline void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ inline void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ inline void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]
__device__ inline void mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]
__device__ inline void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ inline void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// 32 consecutive 32-bit TMEM columns of this thread's lane.
__device__ inline void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ inline void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ inline void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ inline void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// UMMA shared-memory matrix descriptor, 128-byte swizzle, sm_100 version 1.
//   start: byte address in shared memory; lbo/sbo: byte offsets.
__device__ inline uint64_t umma_desc_sw128(uint32_t start, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((start >> 4) & 0x3FFF);
  d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;            // descriptor version for sm_100
  d |= (uint64_t)2 << 61;            // SWIZZLE_128B
  return d;
}

// The same with 64-byte swizzle (8-row atoms of 512 bytes).
__device__ inline uint64_t umma_desc_sw64(uint32_t start, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((start >> 4) & 0x3FFF);
  d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)4 << 61;            // SWIZZLE_64B
  return d;
}

// Instruction descriptor of kind::f16 with bf16 A/B and fp32 accumulation.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4)                       // D format: f32
         | (1u << 7)                     // A format: bf16
         | (1u << 10)                    // B format: bf16
         | ((a_mn_major ? 1u : 0u) << 15)
         | ((b_mn_major ? 1u : 0u) << 16)
         | ((uint32_t)(N >> 3) << 17)
         | ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------------------
// Launchers (one per kernel family); each returns the launch error.
// ---------------------------------------------------------------------------
cudaError_t launch_tile_table(const Geom& g, int* tile_cube, int* cube_rank, cudaStream_t s);
cudaError_t launch_tile_token(const Geom& g, const int* cube_rank, int* tile_tok, cudaStream_t s);
cudaError_t launch_reorder(const Geom& g, const int* cube_rank, const void* x, void* y, int row_bytes, int inverse,
                           int num_sms, cudaStream_t s);
cudaError_t launch_rope_table(const Geom& g, int dt, int dh, int dw, float base, float2* tab, cudaStream_t s);
cudaError_t launch_pool(const Geom& g, int dtype, const void* q, const void* k, int natural, const int* tile_cube,
                        const int* tile_tok, int rope_enabled, int dt, int dh, int dw, const float2* rope_tab,
                        const PooledOut& po, void* qrot, void* krot, cudaStream_t s);
cudaError_t launch_scores(const CUtensorMap& mqh, const CUtensorMap& mql, const CUtensorMap& mkh,
                          const CUtensorMap& mkl, const ScoreArgs& a, cudaStream_t s);
cudaError_t launch_select(const Geom& g, const float* S, float top_p, int k_min, int* counts, int* idx, int cap,
                          cudaStream_t s);
cudaError_t launch_pool_sub(const Geom& g, int dtype, const void* q, const void* k, int natural, const int* tile_cube,
                            const int* tile_tok, int rope_enabled, int dt, int dh, int dw, const float2* rope_tab,
                            const PooledOut& po, cudaStream_t s);
cudaError_t launch_scores_sub(const CUtensorMap& mqh, const CUtensorMap& mql, const CUtensorMap& mkh,
                              const CUtensorMap& mkl, const ScoreArgs& a, cudaStream_t s);
cudaError_t launch_subblock_agg(const Geom& g, const float* Tb, float* logp, cudaStream_t s);
cudaError_t launch_union(const Geom& g, const int* counts, const int* idx, int cap, int* uni, int* ucount, int* status,
                         cudaStream_t s);
// Longest-first order of n items by key >> shift (descending; ties by
// ascending item index), keys in [0, max_key], within each group of `group`
// consecutive items (group <= 0: one group).
cudaError_t launch_rank(const int* key, int n, int max_key, int group, int shift, int* worklist, cudaStream_t s);
cudaError_t launch_fine_tc(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const FineTcArgs& a,
                           int num_sms, cudaStream_t s);
cudaError_t launch_fine_f32(const FineF32Args& a, cudaStream_t s);
cudaError_t launch_quad_schedule(const Geom& g, int Qn, const int* counts, const int* idx, int cap, int* uni,
                                 int* ucount, int* useg, int* qcost, int* worklist, int* status, cudaStream_t s);
cudaError_t launch_fine_q(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const FineQArgs& a,
                          int num_sms, cudaStream_t s);
cudaError_t launch_token_pos(const Geom& g, const int* cube_rank, int* pos, cudaStream_t s);
cudaError_t launch_rope_pairs(const Geom& g, int dt, int dh, int dw, float base, int t_offset, float2* tab,
                              cudaStream_t s);
struct QkvTma {
  int box_rows;    // X rows per tile (the W box is 256 rows)
  int box_k;       // channels per stage: 64 (128-byte swizzle) or 32 (64-byte swizzle)
};
QkvTma qkv_tma(int variant);
cudaError_t launch_qkv(const CUtensorMap& mx, const CUtensorMap& mw, QkvArgs a, int variant, int num_sms,
                       cudaStream_t s);
cudaError_t launch_bwd_prep(const void* out, const void* dout, const float* lse, float* lse2, float* dd, long long rows,
                            cudaStream_t s);
cudaError_t launch_key_union(const Geom& g, const int* counts, const int* idx, int cap, uint32_t* bits, int* uni,
                             int* ucount, int* status, cudaStream_t s);
cudaError_t launch_bwd(const CUtensorMap& s0, const CUtensorMap& s1, const CUtensorMap& m0, const CUtensorMap& m1,
                       const BwdArgs& a, bool key_stationary, int num_sms, cudaStream_t s);
cudaError_t launch_augment(const Geom& g, const float* S, const int* counts, const int* idx, int cap,
                           const int* ucount, const int* worklist, int G, const long long* busy, int fill_percent,
                           int* extra, int* out_counts, int* out_idx, int out_cap, int* status, cudaStream_t s);
cudaError_t launch_wait_selftest(int* status, long long cap, cudaStream_t s);

}  // namespace fvattn
