// Fine stage on the 5th-generation tensor cores ("VSA" digest, section 3:
// token-level attention restricted to the selected tiles; "CalibAtt"
// digest: selected connections computed densely, the rest skipped).
//
// Persistent kernel, one CTA per SM, 384 threads.  A work item is two
// adjacent query tiles of one head: one 128-row tensor-core tile walking the
// union of the two tiles' key lists two entries (128 keys) per step.
//   warp 0       TMA producer: picks the CTA's next item (the next slot of
//                a work-list counter when it starts an item, or a static
//                slot sequence) and publishes its code in a shared ring;
//                loads the item's Q, K of every step's two key tiles into a
//                3-stage ring and V into a 3-stage ring; after the last item
//                it arrives on the next Q buffer without rows (code -1),
//                which every role passes on and stops at;
//   warp 1       S issuer (one thread): S = Q K^T (M=128, N=128, K=128) of
//                step c into TMEM S buffer c & 1 once the PV of step c - 2
//                (the buffer's previous P) is complete;
//   warp 2       PV issuer (one thread): O_t += P_t V_t (M=128, N=128,
//                K=64) for the step's key tiles t = 0, 1 once P is written;
//   warps 4-7    softmax of the first key tile of every step, warps 8-11 of
//                the second: thread r of a group owns row r (TMEM lane r).
// Each group keeps its own online-softmax state and its own O accumulator,
// so the groups never synchronise per step; the epilogue merges the two
// (m, l, O) triples.  A key tile selected by only one of the item's query
// tiles is masked for the other tile's rows: their P row is written as zeros
// and no exponential is evaluated for them, so every row sees exactly its
// own tile's selection.  An item with an odd number of entries pads its last
// step with a masked copy of its last key tile.
// Online softmax in base 2 with a lazy rescale: a row keeps its reference
// max m until a step's probabilities sum past 2^64, and only then is its O
// rescaled in TMEM, so the max is evaluated once per item and on those rare
// steps.  The normaliser sums the bf16 probabilities the PV MMA consumes.
// The elementwise math runs on packed f32x2 instructions; exponentials can
// be split between the MUFU unit and a polynomial on the FMA pipe (see
// exp2_poly2).
//
// TMEM (512 columns): S buffers 0, 1 at [128 b, 128 b + 128), key tile t in
// columns 64 t .. 64 t + 63 (its P, bf16, overwrites the first 32); O of
// key tile 0 at [256, 384), of key tile 1 at [384, 512), fp32.
// Shared memory (1024-aligned, 128-byte swizzle), default build:
//   Q    = 2 d-halves x 128 rows x 128 B                    32 KB
//   K[3] = 3 x (2 d-halves x 128 keys x 128 B)              96 KB
//   V[3] = 3 x (2 tiles x 2 d-halves x 64 keys x 128 B)     96 KB
#include "fvattn_internal.cuh"

namespace fvattn {
namespace ft {

#ifndef FVATTN_FT_KSTAGES
#define FVATTN_FT_KSTAGES 3
#endif
#ifndef FVATTN_FT_VSTAGES
#define FVATTN_FT_VSTAGES 3
#endif
#ifndef FVATTN_FT_QBUF
#define FVATTN_FT_QBUF 1
#endif

constexpr int D = 128;
constexpr int KST = FVATTN_FT_KSTAGES;     // K ring depth
constexpr int VST = FVATTN_FT_VSTAGES;     // V ring depth
constexpr int QBUF = FVATTN_FT_QBUF;       // Q buffers (items in flight)
constexpr int SBUF = 2;                    // TMEM S buffers
constexpr int THREADS = 384;
constexpr int SM_WARP0 = 4;                             // first softmax warp
constexpr uint32_t BOX = 64 * 128;                      // one 64-row x 128-byte box: 8 KB
constexpr uint32_t Q_BYTES = 4 * BOX;                   // 2 tiles x 2 d-halves: 32 KB
constexpr uint32_t Q_HALF = 2 * BOX;                    // one d-half of the 128 Q rows
constexpr uint32_t STAGE_BYTES = 4 * BOX;               // K or V of a step's two key tiles: 32 KB
constexpr uint32_t K_HALF = 2 * BOX;                    // one d-half of the step's 128 keys
constexpr uint32_t V_TILE = 2 * BOX;                    // one key tile of V (2 d-halves)
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_O = 256;                        // O of keys 0-31; keys 32-63 at +128
constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, false, false);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 128, false, true);
constexpr int STEP_LAST = 1 << 4;     // step word: sel of tile 0 (bits 0-1), tile 1 (bits 2-3), last
constexpr int STEP_END = 1 << 5;      // step word: the CTA has no further item
constexpr int kItemRing = 8;          // item codes in flight between the producer and the softmax

struct Ctl {
  uint64_t q_full[QBUF], q_empty[QBUF];
  uint64_t k_full[KST], k_empty[KST];
  uint64_t v_full[VST], v_empty[VST];
  uint64_t s_full[SBUF];   // S ready (MMA commit) + step info written (MMA thread arrive)
  uint64_t p_full[SBUF];   // both halves' P written (one arrival per softmax warp)
  uint64_t pv_done[SBUF];  // PV of step c complete: barrier c & 1, phase c >> 1 (the S of step
                           // c waits for PV(c - 2), and PV(c + 2) needs P(c + 2), so a waiter
                           // never sees two outstanding phases)
  uint64_t o_empty;        // epilogue read both O (8 warp arrivals per item)
  uint64_t xchg1;          // epilogue: group 1 published (m, l) (4 warp arrivals per item)
  uint64_t xchg2;          // epilogue: group 0 replaced them with the merge scales (4 per item)
  uint64_t drain;          // final commits of the two MMA threads
  int info[SBUF];          // per S buffer: the step word
  int meta[KST];
  int item_ring[kItemRing]; // item code of this CTA's k-th item at k % kItemRing (-1: no more items),
                            // written by the producer before the item's Q arrival
  float2 ex[128];                 // epilogue exchange per row: group 1's (m, l), then the scales
                                  // (s0, s1) group 0 computed from both groups' (m, l)
  uint32_t tmem_base;
  int abort;
};

// The 128-byte swizzle atoms of TMA and UMMA need 1024-byte alignment: the
// kernel rounds its dynamic shared-memory base up inside a 1 KB larger
// allocation.
constexpr uint32_t SMEM_BYTES = 1024 + QBUF * Q_BYTES + (KST + VST) * STAGE_BYTES;
// A step whose probabilities (relative to the half-row's reference max) sum
// past this bound triggers a rescale: P is bf16 (exponent range 2^+-127) and
// O, l are fp32, so probabilities up to 2^64 are exact enough, and the
// rescale (a wait on the in-flight PV plus a TMEM read-modify-write of O)
// almost never runs.
constexpr float RESCALE_SUM = 18446744073709551616.f;   // 2^64
// Pairs of a key tile (32 pairs) whose exponentials use the polynomial.
#ifndef FVATTN_FT_POLY_PAIRS
#define FVATTN_FT_POLY_PAIRS 0
#endif
constexpr int POLY_PAIRS = FVATTN_FT_POLY_PAIRS;
static_assert(POLY_PAIRS == 0 || POLY_PAIRS == 8 || POLY_PAIRS == 12 || POLY_PAIRS == 16, "poly split");
__host__ __device__ constexpr bool poly_pair(int i) {
  return POLY_PAIRS == 8 ? (i & 3) == 3
       : POLY_PAIRS == 12 ? ((i & 7) == 1 || (i & 7) == 3 || (i & 7) == 6)
       : POLY_PAIRS == 16 ? (i & 1) == 1 : false;
}
static_assert(SMEM_BYTES + sizeof(Ctl) <= 232448, "shared memory budget (dynamic + static)");

}  // namespace ft

// One 64-token tile of a [BH, N, 128] bf16 tensor: two 64-column boxes
// (d 0-63 and 64-127) written `stride` bytes apart.  `cube` is the tile's
// packed cube coordinates (natural layout) and is unused for the tiled one.
__device__ inline void tma_tile(const CUtensorMap* map, int natural, int cube, int bh, int tile, uint8_t* dst,
                                uint32_t stride, uint64_t* bar) {
  if (natural) {
    const int w0 = cube_w(cube) * 4, h0 = cube_h(cube) * 4, t0 = cube_t(cube) * 4;
    tma_load_5d(dst, map, bar, 0, w0, h0, t0, bh);
    tma_load_5d(dst + stride, map, bar, 64, w0, h0, t0, bh);
  } else {
    tma_load_3d(dst, map, bar, 0, tile * kTileTokens, bh);
    tma_load_3d(dst + stride, map, bar, 64, tile * kTileTokens, bh);
  }
}

__device__ inline float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ inline uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&b);
}

// Packed f32x2 helpers (sm_100 FFMA2 / FADD2).
__device__ inline uint64_t f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ inline void uf2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ inline uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ inline uint64_t add2_rm(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rm.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ inline uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ inline float max3f(float a, float b, float c) {
  float m;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(a), "f"(b), "f"(c));
  return m;
}
// bf16x2 of (lo, hi), round to nearest even.
__device__ inline uint32_t cvt_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// acc + the low / high bf16 half of w (exact widening, one fp32 rounding).
__device__ inline float add_bf16_lo(float acc, uint32_t w) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tadd.rn.f32.bf16 %0, l, %0;\n\t}" : "+f"(acc) : "r"(w));
  return acc;
}
__device__ inline float add_bf16_hi(float acc, uint32_t w) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tadd.rn.f32.bf16 %0, h, %0;\n\t}" : "+f"(acc) : "r"(w));
  return acc;
}

// 2^x for a pair on the FMA pipe (Cody-Waite style range reduction): x is
// clamped to [-126, 126]; i = floor(x) comes from a round-down add of
// 1.5 * 2^23 (the low mantissa bits of the sum hold i), f = x - i in [0, 1),
// 2^f by a degree-3 polynomial, and i is added to the exponent field.  The
// coefficients are a minimax fit of 2^f on [0, 1) in relative error, solved
// as a linear program over a dense grid: max relative error 7.5e-5, below
// half a bf16 ulp (2^-9), which is the precision P is stored in.
__device__ inline void exp2_poly2(float x0, float x1, float& y0, float& y1) {
  constexpr float C0 = 0.9999252557754517f, C1 = 0.6958333253860474f, C2 = 0.22606715559959412f,
                  C3 = 0.07802474498748779f, MAGIC = 12582912.f;
  x0 = fminf(fmaxf(x0, -126.f), 126.f);
  x1 = fminf(fmaxf(x1, -126.f), 126.f);
  const uint64_t X = f2(x0, x1), M = f2(MAGIC, MAGIC);
  const uint64_t Y = add2_rm(X, M);
  const uint64_t F = sub2(X, sub2(Y, M));
  uint64_t P = fma2(F, f2(C3, C3), f2(C2, C2));
  P = fma2(P, F, f2(C1, C1));
  P = fma2(P, F, f2(C0, C0));
  float p0, p1, q0, q1;
  uf2(P, p0, p1);
  uf2(Y, q0, q1);
  y0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(q0) << 23));
  y1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(q1) << 23));
}

// Largest logit of a row's 64-key step.
__device__ inline float row_max64(const uint32_t (&s0)[32], const uint32_t (&s1)[32]) {
  float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    m0 = max3f(m0, __uint_as_float(s0[i]), __uint_as_float(s0[i + 1]));
    m1 = max3f(m1, __uint_as_float(s1[i]), __uint_as_float(s1[i + 1]));
  }
  return fmaxf(m0, m1);
}

// P = 2^(s * sl2 - m) of a row's 64-key step as 32 bf16x2 words (word k =
// keys 2k, 2k+1); returns the sum of the bf16 values.
__device__ inline float exp_step(const uint32_t (&s0)[32], const uint32_t (&s1)[32], float sl2, float m,
                                 uint32_t (&pk)[32]) {
  const uint64_t SL = f2(sl2, sl2), NM = f2(-m, -m);
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const uint32_t* src = i < 16 ? s0 : s1;
    const int j = 2 * (i & 15);
    float x0, x1, p0, p1;
    uf2(fma2(f2(__uint_as_float(src[j]), __uint_as_float(src[j + 1])), SL, NM), x0, x1);
    if (ft::poly_pair(i)) {
      exp2_poly2(x0, x1, p0, p1);
    } else {
      p0 = ex2(x0);
      p1 = ex2(x1);
    }
    const uint32_t w = cvt_bf16x2(p0, p1);
    pk[i] = w;
    if (i & 1) {
      a2 = add_bf16_lo(a2, w);
      a3 = add_bf16_hi(a3, w);
    } else {
      a0 = add_bf16_lo(a0, w);
      a1 = add_bf16_hi(a1, w);
    }
  }
  return (a0 + a1) + (a2 + a3);
}

// 16 consecutive 32-bit TMEM columns of this thread's lane.
__device__ inline void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// S = Q K^T of one step (M=128 rows, N=128 keys, K=128 dims in 8 MMAs of
// K=16) into TMEM at tS; Q and K in 128-byte swizzled d-halves.
__device__ __forceinline__ void s_mmas(uint32_t tS, uint64_t qd, uint64_t kd) {
  using namespace ft;
  mma_ss(tS, qd, kd, IDESC_S, 0u);
#pragma unroll
  for (int kk = 1; kk < 8; ++kk)
    mma_ss(tS, qd + (((kk >> 2) * Q_HALF + (kk & 3) * 32) >> 4), kd + (((kk >> 2) * K_HALF + (kk & 3) * 32) >> 4),
           IDESC_S, 1u);
}

// O_t (+)= P_t V_t for the step's key tiles t = 0, 1: P_t (bf16) in TMEM at
// tP + 64 t, V_t MN-major in the stage; 16 keys = 16 V rows = 2048 bytes
// per K=16 MMA.
__device__ __forceinline__ void pv_mmas(uint32_t tbase, uint32_t tP, const uint8_t* vstage, bool first) {
  using namespace ft;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const uint64_t vd = umma_desc_sw128(smem_u32(vstage + t * V_TILE), BOX, 1024);
    const uint32_t tO = tbase + TMEM_O + 128 * t;
    mma_ts(tO, tP + 64 * t, vd, IDESC_PV, first ? 0u : 1u);
#pragma unroll
    for (int kk = 1; kk < 4; ++kk) mma_ts(tO, tP + 64 * t + 8 * kk, vd + ((kk * 2048) >> 4), IDESC_PV, 1u);
  }
}

// Work-list slot of this CTA's k-th item: round k of G consecutive slots,
// CTA c taking slot c of each round, or slot G - 1 - c of the odd rounds when
// `snake` (serpentine: on a longest-first list the CTA that took a round's
// longest item takes the next round's shortest).  Strictly increasing in k,
// so a CTA's items end at its first slot past the list.
__device__ __forceinline__ int cta_slot(int k, int snake) {
  const int c = (snake && (k & 1)) ? (int)gridDim.x - 1 - (int)blockIdx.x : (int)blockIdx.x;
  return k * (int)gridDim.x + c;
}

__global__ void __launch_bounds__(ft::THREADS, 1)
    fine_tc_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                   const __grid_constant__ CUtensorMap mv, const FineTcArgs a) {
  using namespace ft;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + QBUF * Q_BYTES;
  uint8_t* sV = sK + KST * STAGE_BYTES;
  __shared__ Ctl ctl_s;
  Ctl* ctl = &ctl_s;
  volatile int* abort_flag = &ctl->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Geom& g = a.g;
  const long long cap = a.wait_cap;

  if (threadIdx.x == 0) {
    for (int i = 0; i < QBUF; ++i) {
      mbar_init(&ctl->q_full[i], 1);
      mbar_init(&ctl->q_empty[i], 1);
    }
    for (int i = 0; i < KST; ++i) {
      mbar_init(&ctl->k_full[i], 1);
      mbar_init(&ctl->k_empty[i], 1);
    }
    for (int i = 0; i < VST; ++i) {
      mbar_init(&ctl->v_full[i], 1);
      mbar_init(&ctl->v_empty[i], 1);
    }
    for (int i = 0; i < SBUF; ++i) {
      mbar_init(&ctl->s_full[i], 2);
      mbar_init(&ctl->p_full[i], 8);      // one arrival per softmax warp
      mbar_init(&ctl->pv_done[i], 1);
    }
    mbar_init(&ctl->o_empty, 8);
    mbar_init(&ctl->xchg1, 4);
    mbar_init(&ctl->xchg2, 4);
    mbar_init(&ctl->drain, 2);   // one final commit per MMA issuer
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = ctl->tmem_base;
  const unsigned long long t_start = threadIdx.x == 0 && a.cta_times ? global_ns() : 0ull;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    // The whole warp fetches the next 32 union entries (16 steps) and their
    // cube coordinates with one pair of coalesced loads; lane 0 then issues
    // the waits and copies step by step, so no copy waits on a global load.
    const bool leader = lane == 0;
    const bool nat = a.q_nat || a.k_nat || a.v_nat;
    if (leader) {
      prefetch_tensormap(&mq);
      prefetch_tensormap(&mk);
      prefetch_tensormap(&mv);
    }
    long long gs = 0;                 // steps loaded
    int k = 0, q_issued = 0;
    bool ok = true;
    // This CTA's items: the work-list slots cta_slot(k), or (a.next_slot) slot
    // blockIdx.x first and then each slot taken from the shared counter when
    // the previous item starts (greedy list scheduling, one item ahead).
    int slot = a.next_slot ? (int)blockIdx.x : cta_slot(0, a.snake);
    int slot_next = 0;
    int item_next = slot < a.n_items ? a.worklist[slot] : 0;
    for (; slot < a.n_items && ok; ++k, slot = slot_next) {
      const int item = item_next;
      if (a.next_slot) {
        if (leader) slot_next = (int)gridDim.x + atomicAdd(a.next_slot, 1);
        slot_next = __shfl_sync(0xffffffffu, slot_next, 0);
      } else {
        slot_next = cta_slot(k + 1, a.snake);
      }
      if (slot_next < a.n_items) item_next = a.worklist[slot_next];
      const int bh = item / g.P, qd = item % g.P;
      const int qb = k % QBUF;
      // lanes 0, 1: the item's two query tiles (a missing second tile repeats the first; its rows
      // are never stored)
      int qtile = kItemTiles * qd + (lane & 1);
      if (qtile >= g.nT) qtile = kItemTiles * qd;
      const int qcube = nat && lane < kItemTiles ? a.tile_cube[qtile] : 0;
      const int n = a.ucount[item];
      const int* list = a.uni + (size_t)item * g.nT;
      if (leader && k >= QBUF) ok = mbar_wait(&ctl->q_empty[qb], ((k / QBUF) - 1) & 1, abort_flag, a.status, cap);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      const int qc0 = __shfl_sync(0xffffffffu, qcube, 0), qc1 = __shfl_sync(0xffffffffu, qcube, 1);
      const int qt0 = __shfl_sync(0xffffffffu, qtile, 0), qt1 = __shfl_sync(0xffffffffu, qtile, 1);
      if (leader) {
        ctl->item_ring[k % kItemRing] = item;     // released by the arrival below
        mbar_arrive_expect_tx(&ctl->q_full[qb], Q_BYTES);
        uint8_t* qd_smem = sQ + qb * Q_BYTES;
        tma_tile(&mq, a.q_nat, qc0, bh, qt0, qd_smem, Q_HALF, &ctl->q_full[qb]);
        tma_tile(&mq, a.q_nat, qc1, bh, qt1, qd_smem + BOX, Q_HALF, &ctl->q_full[qb]);
      }
      ++q_issued;
      const int steps = (n + 1) >> 1;
      for (int e0 = 0; e0 < n && ok; e0 += 32) {
        int ent = e0 + lane < n ? list[e0 + lane] : 0;
        int j = ent & 0xFFFF;
        if (j >= g.nT) {  // never produced by the schedule; keep the copy in bounds
          set_status(a.status, kStatusBadBlock);
          j = 0;
          ent &= ~0x30000;
        }
        const int cube = nat ? a.tile_cube[j] : 0;
        const int cnt = n - e0 < 32 ? n - e0 : 32;
        for (int i = 0; i < cnt; i += 2, ++gs) {
          // the step's key tiles: entries e0 + i and e0 + i + 1 (a masked copy of the first when
          // the item's entry count is odd)
          const bool two = i + 1 < cnt;
          const int ent0 = __shfl_sync(0xffffffffu, ent, i);
          const int cube0 = __shfl_sync(0xffffffffu, cube, i);
          const int ent1 = __shfl_sync(0xffffffffu, ent, two ? i + 1 : i);
          const int cube1 = __shfl_sync(0xffffffffu, cube, two ? i + 1 : i);
          if (leader) {
            const int j0 = ent0 & 0xFFFF, j1 = ent1 & 0xFFFF;
            const int ks = (int)(gs % KST), vs = (int)(gs % VST);
            const int step = (e0 + i) >> 1;
            if (gs >= KST)
              ok = mbar_wait(&ctl->k_empty[ks], (uint32_t)((gs / KST) - 1) & 1, abort_flag, a.status, cap);
            if (ok) {
              ctl->meta[ks] = ((ent0 >> 16) & 3) | (two ? ((ent1 >> 16) & 3) << 2 : 0) |
                              (step == steps - 1 ? STEP_LAST : 0);
              mbar_arrive_expect_tx(&ctl->k_full[ks], STAGE_BYTES);
              uint8_t* kd = sK + ks * STAGE_BYTES;
              tma_tile(&mk, a.k_nat, cube0, bh, j0, kd, K_HALF, &ctl->k_full[ks]);
              tma_tile(&mk, a.k_nat, cube1, bh, j1, kd + BOX, K_HALF, &ctl->k_full[ks]);
              if (gs >= VST)
                ok = mbar_wait(&ctl->v_empty[vs], (uint32_t)((gs / VST) - 1) & 1, abort_flag, a.status, cap);
            }
            if (ok) {
              mbar_arrive_expect_tx(&ctl->v_full[vs], STAGE_BYTES);
              uint8_t* vd = sV + vs * STAGE_BYTES;
              tma_tile(&mv, a.v_nat, cube0, bh, j0, vd, BOX, &ctl->v_full[vs]);
              tma_tile(&mv, a.v_nat, cube1, bh, j1, vd + V_TILE, BOX, &ctl->v_full[vs]);
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
        }
      }
    }
    // every copy issued has landed before the block exits
    if (leader) {
      for (int qb = 0; qb < QBUF && qb < q_issued; ++qb) {
        const int last = qb + ((q_issued - 1 - qb) / QBUF) * QBUF;
        mbar_drain(&ctl->q_full[qb], (uint32_t)(last / QBUF) & 1, a.status, cap);
      }
      for (int i = 0; i < KST && i < gs; ++i) {
        const long long last = i + ((gs - 1 - i) / KST) * KST;
        mbar_drain(&ctl->k_full[i], (uint32_t)(last / KST) & 1, a.status, cap);
      }
      for (int i = 0; i < VST && i < gs; ++i) {
        const long long last = i + ((gs - 1 - i) / VST) * VST;
        mbar_drain(&ctl->v_full[i], (uint32_t)(last / VST) & 1, a.status, cap);
      }
    }
    // then the end of this CTA's items: a Q buffer that carries no rows,
    // item code -1 (after the drain above, which waits for the last loaded
    // phase of each Q buffer)
    if (ok) {
      const int qb = k % QBUF;
      if (leader && k >= QBUF) ok = mbar_wait(&ctl->q_empty[qb], ((k / QBUF) - 1) & 1, abort_flag, a.status, cap);
      if (leader && ok) {
        ctl->item_ring[k % kItemRing] = -1;
        mbar_arrive(&ctl->q_full[qb]);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------- MMA: S
    // S(c) into buffer c & 1 once the PV of step c - 2, which read its P
    // from that buffer, is complete; a K stage is released when its S
    // completes, the Q buffer after the item's last S.  The producer ends
    // the CTA's items with a Q buffer that carries no rows (item code -1 in
    // the ring): passed on to the softmax as a step word with STEP_END.
    long long c = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int qb = k % QBUF;
      if (!mbar_wait(&ctl->q_full[qb], (uint32_t)(k / QBUF) & 1, abort_flag, a.status, cap)) break;
      if (ctl->item_ring[k % kItemRing] < 0) {
        const int b = (int)(c & 1);
        if (c >= SBUF && !mbar_wait(&ctl->pv_done[b], (uint32_t)((c - SBUF) >> 1) & 1, abort_flag, a.status, cap))
          break;
        ctl->info[b] = STEP_END;
        mbar_arrive(&ctl->s_full[b]);     // both arrivals of the buffer's phase, no MMA
        mbar_arrive(&ctl->s_full[b]);
        break;
      }
      const uint64_t qd = umma_desc_sw128(smem_u32(sQ + qb * Q_BYTES), 16, 1024);
      while (true) {
        const int ks = (int)(c % KST);
        const int b = (int)(c & 1);
        // K first: it is loaded well ahead, the PV wait is the one on the critical path
        if (!mbar_wait(&ctl->k_full[ks], (uint32_t)(c / KST) & 1, abort_flag, a.status, cap)) {
          ok = false;
          break;
        }
        if (c >= SBUF && !mbar_wait(&ctl->pv_done[b], (uint32_t)((c - SBUF) >> 1) & 1, abort_flag, a.status, cap)) {
          ok = false;
          break;
        }
        const int meta = ctl->meta[ks];
        ctl->info[b] = meta;
        tc_fence_after();
        s_mmas(tbase + 128 * b, qd, umma_desc_sw128(smem_u32(sK + ks * STAGE_BYTES), 16, 1024));
        mma_commit(&ctl->s_full[b]);
        mma_commit(&ctl->k_empty[ks]);
        mbar_arrive(&ctl->s_full[b]);
        ++c;
        if (meta & STEP_LAST) break;
      }
      if (!ok) break;
      mma_commit(&ctl->q_empty[qb]);
    }
    // every MMA this thread issued has completed before TMEM is freed
    mma_commit(&ctl->drain);
    mbar_drain(&ctl->drain, 0, a.status, cap);
  } else if (warp == 2 && lane == 0) {
    // ------------------------------------------------------------ MMA: PV
    // O_t += P_t V_t for the step's key tiles t = 0, 1 once both softmax
    // groups wrote P; the first step of an item overwrites O after the
    // previous item's epilogue read it.  A V stage is released when its PV
    // completes.  A step word with STEP_END (no V loaded for it) ends the loop.
    long long c = 0;
    bool ok = true;
    bool end = false;
    for (int k = 0; ok && !end; ++k) {
      bool first = true;
      while (true) {
        const int b = (int)(c & 1);
        const int vs = (int)(c % VST);
        // O free comes well before P, the wait on the critical path
        if (first && k >= 1 && !mbar_wait(&ctl->o_empty, (uint32_t)(k - 1) & 1, abort_flag, a.status, cap)) {
          ok = false;
          break;
        }
        if (!mbar_wait(&ctl->p_full[b], (uint32_t)(c >> 1) & 1, abort_flag, a.status, cap)) {
          ok = false;
          break;
        }
        const int info = ctl->info[b];
        if (info & STEP_END) {
          end = true;
          break;
        }
        if (!mbar_wait(&ctl->v_full[vs], (uint32_t)(c / VST) & 1, abort_flag, a.status, cap)) {
          ok = false;
          break;
        }
        tc_fence_after();
        pv_mmas(tbase, tbase + 128 * b, sV + vs * STAGE_BYTES, first);
        mma_commit(&ctl->pv_done[b]);
        mma_commit(&ctl->v_empty[vs]);
        first = false;
        ++c;
        if (info & STEP_LAST) break;
      }
    }
    mma_commit(&ctl->drain);
    mbar_drain(&ctl->drain, 0, a.status, cap);
  } else if (warp >= SM_WARP0) {
    // ------------------------------------------------------------ softmax
    const int h = (warp - SM_WARP0) >> 2;             // key tile of every step
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;                     // row of the item
    const int half = r >> 6, rr = r & 63;             // query tile of the row, row in it
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t tO = tbase + TMEM_O + 128 * h + lane_off;
    const float sl2 = g.scale * 1.4426950408889634f;
    long long c = 0;
    bool end = false;
    for (int k = 0; !end; ++k) {
      int bh = 0, qd = 0, tile = 0, cube = 0;         // the item's, read at its first step
      bool valid = false, first = true;
      float m_use = -INFINITY, l = 0.f;
      bool ok = true;
      while (true) {
        const int b = (int)(c & 1);
        if (!mbar_wait(&ctl->s_full[b], (uint32_t)(c >> 1) & 1, abort_flag, a.status, cap)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int info = ctl->info[b];
        if (info & STEP_END) {                        // no further item; the PV thread stops on it too
          mbar_arrive_warp(&ctl->p_full[b]);
          end = true;
          break;
        }
        if (first) {
          // the item's code, written by the producer before its Q arrival
          const int item = ctl->item_ring[k % kItemRing];
          bh = item / g.P;
          qd = item % g.P;
          tile = kItemTiles * qd + half;
          valid = tile < g.nT;
          cube = valid && a.out_nat ? a.tile_cube[tile] : 0;   // used by the epilogue
          first = false;
        }
        const bool sel = (info >> (2 * h + half)) & 1;
        const uint32_t tS = tbase + 128 * b + 64 * h + lane_off;
        uint32_t pk[32];
        float alpha = 1.f;
        bool rescale = false;
        {
          uint32_t s0[32], s1[32];
          tmem_ld32(tS, s0);
          tmem_ld32(tS + 32, s1);
          tmem_wait_ld();
          if (sel) {
            if (m_use == -INFINITY) m_use = row_max64(s0, s1) * sl2;   // first selected tile of the row
            float sum = exp_step(s0, s1, sl2, m_use, pk);
            if (!(sum <= RESCALE_SUM)) {      // too large (or inf): move the reference max up
              const float m_new = fmaxf(row_max64(s0, s1) * sl2, m_use);
              alpha = ex2(m_use - m_new);
              rescale = l > 0.f;
              l *= alpha;
              m_use = m_new;
              sum = exp_step(s0, s1, sl2, m_use, pk);
            }
            l += sum;
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) pk[i] = 0u;
          }
        }
        tmem_st32(tS, pk);
        if (__any_sync(0xffffffffu, rescale)) {
          // O must hold every PV before step c; PV(c) waits for this step's P
          if (!mbar_wait(&ctl->pv_done[(c - 1) & 1], (uint32_t)((c - 1) >> 1) & 1, abort_flag, a.status, cap)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int ch = 0; ch < 4; ++ch) {
            uint32_t o[32];
            tmem_ld32(tO + ch * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tO + ch * 32, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive_warp(&ctl->p_full[b]);
        ++c;
        if (info & STEP_LAST) break;
      }
      if (!ok || end) break;
      // ---- epilogue: merge the groups' (m, l, O); this group writes dims 64 h .. 64 h + 63
      if (!mbar_wait(&ctl->pv_done[(c - 1) & 1], (uint32_t)((c - 1) >> 1) & 1, abort_flag, a.status, cap)) break;
      tc_fence_after();
      // group 1 publishes (m, l); group 0 merges and writes back both scales into the same slot
      float s0 = 0.f, s1 = 0.f, M = -INFINITY, L = 0.f;
      if (h == 1) {
        ctl->ex[r] = make_float2(m_use, l);
        mbar_arrive_warp(&ctl->xchg1);
        if (!mbar_wait(&ctl->xchg2, (uint32_t)(k & 1), abort_flag, a.status, cap)) break;
        const float2 sc = ctl->ex[r];
        s0 = sc.x;
        s1 = sc.y;
      } else {
        if (!mbar_wait(&ctl->xchg1, (uint32_t)(k & 1), abort_flag, a.status, cap)) break;
        const float2 o1 = ctl->ex[r];
        M = fmaxf(m_use, o1.x);
        const float w0 = m_use == -INFINITY ? 0.f : ex2(m_use - M);
        const float w1 = o1.x == -INFINITY ? 0.f : ex2(o1.x - M);
        L = l * w0 + o1.y * w1;
        const float inv = L > 0.f ? 1.f / L : 0.f;
        s0 = w0 * inv;
        s1 = w1 * inv;
        ctl->ex[r] = make_float2(s0, s1);
        mbar_arrive_warp(&ctl->xchg2);
      }
      const int tok = !valid ? 0 : (a.out_nat ? cube_row_token(g, cube, rr) : tile * kTileTokens + rr);
      __nv_bfloat16* orow = a.out + ((size_t)bh * g.N + tok) * D + 64 * h;
      const uint32_t tO0 = tbase + TMEM_O + lane_off + 64 * h, tO1 = tO0 + 128;
#pragma unroll 1
      for (int ch = 0; ch < 2; ++ch) {
        uint32_t o0[32], o1[32];
        tmem_ld32(tO0 + ch * 32, o0);
        tmem_ld32(tO1 + ch * 32, o1);
        tmem_wait_ld();
        if (valid) {
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            w[i] = pack_bf16(__uint_as_float(o0[2 * i]) * s0 + __uint_as_float(o1[2 * i]) * s1,
                             __uint_as_float(o0[2 * i + 1]) * s0 + __uint_as_float(o1[2 * i + 1]) * s1);
          uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
      }
      if (valid && h == 0)
        a.lse[(size_t)bh * g.N + tok] = L > 0.f ? (M + __log2f(L)) * 0.6931471805599453f : -INFINITY;
      tc_fence_before();
      mbar_arrive_warp(&ctl->o_empty);
    }
  }

  __syncthreads();
  if (threadIdx.x == 0 && a.cta_times && blockIdx.x < kMaxCtas) {
    // busy time of this CTA: setup done to its last item finished
    a.cta_times[1 + 2 * blockIdx.x] = t_start;
    a.cta_times[2 + 2 * blockIdx.x] = global_ns();
    if (blockIdx.x == 0) a.cta_times[0] = gridDim.x;
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, ft::TMEM_COLS);
  }
}

cudaError_t launch_fine_tc(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const FineTcArgs& a,
                           int num_sms, cudaStream_t s) {
  cudaError_t e =
      cudaFuncSetAttribute(fine_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ft::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int grid = a.n_items < num_sms ? a.n_items : num_sms;
  if (grid <= 0) return cudaSuccess;
  fine_tc_kernel<<<grid, ft::THREADS, ft::SMEM_BYTES, s>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

}  // namespace fvattn
