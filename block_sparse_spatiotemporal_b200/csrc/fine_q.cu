// Fine stage on the 5th-generation tensor cores, quad items ("VSA" digest,
// section 3: token-level attention restricted to the selected tiles;
// "CalibAtt" digest: selected connections computed densely, the rest
// skipped).
//
// Persistent kernel, one CTA per SM, 384 threads.  A work item is four
// consecutive query tiles 4u .. 4u+3 of one head in two halves, A (tiles
// 4u, 4u+1) and B (4u+2, 4u+3); each half is one 128-row tensor-core tile.
// The item walks the union of the four tiles' key lists, two key tiles (128
// keys) per step, and both halves read the same K and V tiles from shared
// memory, so each K/V byte brought in from L2 feeds twice the rows of a
// two-tile item.  The union is ordered key tiles of both halves, then of A
// only, then of B only: a half issues no MMA and no softmax on the steps it
// does not need, so the extra rows cost no tensor work.
//   warp 0       TMA producer: the item's four Q tiles, then K of every
//                step into a 3-stage ring and V into a 2-stage ring;
//   warp 1       MMA issuer (one elected lane): per step slot c, in this
//                order, PV_A(c-1), S_A(c), PV_B(c-1), S_B(c) for the
//                halves active on those steps.  One thread's tcgen05.mma
//                execute in issue order, so S_h(c) may overwrite P_h(c-1)
//                in TMEM as soon as PV_h(c-1) has been issued, and the
//                softmax of one half runs while the tensor core works on
//                the other half's products (ping-pong);
//   warps 2-5    softmax and epilogue of half A, warps 6-9 of half B:
//                thread r owns row r of its half (TMEM lane r, the lane
//                quarter of warp w being w mod 4) and all 128 keys of a
//                step, loaded from TMEM at once.
// Online softmax in base 2 with a lazy rescale: a row keeps its reference
// max m (set by its first selected key tile) until a key tile's largest
// logit exceeds it by more than 64 (in log2 units); then m moves up by a
// whole power of two, so the rescale of l, of O in TMEM and of the step's
// P already written is exact.  The normaliser sums the bf16 probabilities
// the PV MMA consumes.
//
// TMEM (512 columns): S_A [0, 128), S_B [128, 256), fp32, key tile t of a
// step in columns 64 t .. 64 t + 63, its P (bf16 pairs) written over
// columns 32 t .. 32 t + 31; O_A [256, 384), O_B [384, 512), fp32.
// Shared memory (1024-aligned, 128-byte swizzle):
//   Q    = 2 halves x 2 d-halves x 128 rows x 128 B              64 KB
//   K[3] = 3 x (2 d-halves x 128 keys x 128 B)                    96 KB
//   V[2] = 2 x (2 key tiles x 2 d-halves x 64 keys x 128 B)       64 KB
#include "fvattn_internal.cuh"

namespace fvattn {
namespace fq {

constexpr int D = 128;
constexpr int KST = 3;                                  // K ring depth
constexpr int VST = 2;                                  // V ring depth
constexpr int THREADS = 320;
constexpr int SM_WARP0 = 2;                             // first softmax warp
constexpr uint32_t BOX = 64 * 128;                      // one 64-row x 128-byte box: 8 KB
constexpr uint32_t QH_BYTES = 4 * BOX;                  // one half: 2 tiles x 2 d-halves: 32 KB
constexpr uint32_t QH_DHALF = 2 * BOX;                  // one d-half of a half's 128 rows
constexpr uint32_t Q_BYTES = 2 * QH_BYTES;              // 64 KB
constexpr uint32_t STAGE_BYTES = 4 * BOX;               // K or V of a step's two key tiles: 32 KB
constexpr uint32_t K_DHALF = 2 * BOX;                   // one d-half of the step's 128 keys
constexpr uint32_t V_TILE = 2 * BOX;                    // one key tile of V (2 d-halves)
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_O = 256;
constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, false, false);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 128, false, true);
constexpr uint32_t SMEM_BYTES = 1024 + Q_BYTES + (KST + VST) * STAGE_BYTES;
constexpr float RESCALE_X = 64.f;   // log2 headroom above the reference max before a rescale

struct Ctl {
  uint64_t q_full, q_empty;
  uint64_t k_full[KST], k_empty[KST];
  uint64_t v_full[VST], v_empty[VST];
  uint64_t s_full[2];    // S_h ready (MMA commit) + the step's selection bits written (issuer arrive)
  uint64_t p_full[2];    // P_h written (128 softmax threads of half h)
  uint64_t pv_done[2];   // PV_h complete
  uint64_t drain;        // the issuer's final commit
  int info[2];           // per half: selection bits of the step whose S_h is in TMEM
  int meta[KST];         // per K stage: selection bits of the step's two entries
  uint32_t tmem_base;
  int abort;
};
static_assert(SMEM_BYTES + sizeof(Ctl) <= 232448, "shared memory budget (dynamic + static)");

}  // namespace fq

// One 64-token tile of a [BH, N, 128] bf16 tensor: two 64-column boxes
// (d 0-63 and 64-127) written `stride` bytes apart.  `cube` is the tile's
// packed cube coordinates (natural layout), unused for the tiled one.
__device__ inline void fq_tma_tile(const CUtensorMap* map, int natural, int cube, int bh, int tile, uint8_t* dst,
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

// L2 prefetch of the same tile (no shared memory, no barrier).
__device__ inline void fq_prefetch_tile(const CUtensorMap* map, int natural, int cube, int bh, int tile) {
  if (natural) {
    const int w0 = cube_w(cube) * 4, h0 = cube_h(cube) * 4, t0 = cube_t(cube) * 4;
#pragma unroll
    for (int c0 = 0; c0 < 128; c0 += 64)
      asm volatile("cp.async.bulk.prefetch.tensor.5d.L2.global.tile [%0, {%1, %2, %3, %4, %5}];" ::"l"(map),
                   "r"(c0), "r"(w0), "r"(h0), "r"(t0), "r"(bh)
                   : "memory");
  } else {
#pragma unroll
    for (int c0 = 0; c0 < 128; c0 += 64)
      asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(map), "r"(c0),
                   "r"(tile * kTileTokens), "r"(bh)
                   : "memory");
  }
}

__device__ inline float fq_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ inline uint64_t fq_f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ inline void fq_uf2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ inline uint64_t fq_fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ inline float fq_max3(float a, float b, float c) {
  float m;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(a), "f"(b), "f"(c));
  return m;
}
// bf16x2 of (lo, hi), round to nearest even.
__device__ inline uint32_t fq_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// acc + the low / high bf16 half of w (exact widening, one fp32 rounding).
__device__ inline float fq_add_lo(float acc, uint32_t w) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tadd.rn.f32.bf16 %0, l, %0;\n\t}" : "+f"(acc) : "r"(w));
  return acc;
}
__device__ inline float fq_add_hi(float acc, uint32_t w) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tadd.rn.f32.bf16 %0, h, %0;\n\t}" : "+f"(acc) : "r"(w));
  return acc;
}

// Largest logit of 64 keys (two 32-column loads).
__device__ inline float fq_max64(const uint32_t (&s0)[32], const uint32_t (&s1)[32]) {
  float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    m0 = fq_max3(m0, __uint_as_float(s0[i]), __uint_as_float(s0[i + 1]));
    m1 = fq_max3(m1, __uint_as_float(s1[i]), __uint_as_float(s1[i + 1]));
  }
  return fmaxf(m0, m1);
}

// P = 2^(s * sl2 - m) of 64 keys as 32 bf16x2 words (word k = keys 2k,
// 2k + 1); returns the sum of the bf16 values.
__device__ inline float fq_exp64(const uint32_t (&s0)[32], const uint32_t (&s1)[32], float sl2, float m,
                                 uint32_t (&pk)[32]) {
  const uint64_t SL = fq_f2(sl2, sl2), NM = fq_f2(-m, -m);
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const uint32_t* src = i < 16 ? s0 : s1;
    const int j = 2 * (i & 15);
    float x0, x1;
    fq_uf2(fq_fma2(fq_f2(__uint_as_float(src[j]), __uint_as_float(src[j + 1])), SL, NM), x0, x1);
    const uint32_t w = fq_bf16x2(fq_ex2(x0), fq_ex2(x1));
    pk[i] = w;
    if (i & 1) {
      a2 = fq_add_lo(a2, w);
      a3 = fq_add_hi(a3, w);
    } else {
      a0 = fq_add_lo(a0, w);
      a1 = fq_add_hi(a1, w);
    }
  }
  return (a0 + a1) + (a2 + a3);
}

// tcgen05.wait::ld that also names the destination registers of the loads it
// waits for, so the compiler cannot move their first use above the wait.
__device__ inline void fq_wait_ld(uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), "+r"(r[8]),
        "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]),
        "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]),
        "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
      :
      : "memory");
}

// 16 consecutive 32-bit TMEM columns of this thread's lane.
__device__ inline void fq_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ inline void fq_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// Largest logit of 32 keys.
__device__ inline float fq_max32(const uint32_t (&s)[32]) {
  float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
  for (int i = 0; i < 32; i += 4) {
    m0 = fq_max3(m0, __uint_as_float(s[i]), __uint_as_float(s[i + 1]));
    m1 = fq_max3(m1, __uint_as_float(s[i + 2]), __uint_as_float(s[i + 3]));
  }
  return fmaxf(m0, m1);
}

// Pairs of a 32-key chunk (16 pairs) whose exponentials run on the FMA
// pipe (exp2 by a polynomial) instead of the MUFU unit: 0, every 4th, or
// every 2nd pair.
#ifndef FVATTN_FQ_POLY
#define FVATTN_FQ_POLY 0
#endif
__host__ __device__ constexpr bool fq_poly_pair(int i) {
  return FVATTN_FQ_POLY == 4 ? (i & 3) == 3 : FVATTN_FQ_POLY == 2 ? (i & 1) == 1 : false;
}

// 2^x for a pair on the FMA pipe: x clamped to [-126, 126]; i = floor(x)
// from a round-down add of 1.5 * 2^23 (the low mantissa bits of the sum
// hold i), f = x - i in [0, 1), 2^f by a degree-3 polynomial, i added to the
// exponent field.  The coefficients are a minimax fit of 2^f on [0, 1) in
// relative error (a linear program over a dense grid): max relative error
// 7.5e-5, below half a bf16 ulp (2^-9), the precision P is stored in.
__device__ inline void fq_exp2_poly(float x0, float x1, float& y0, float& y1) {
  constexpr float C0 = 0.9999252557754517f, C1 = 0.6958333253860474f, C2 = 0.22606715559959412f,
                  C3 = 0.07802474498748779f, MAGIC = 12582912.f;
  x0 = fminf(fmaxf(x0, -126.f), 126.f);
  x1 = fminf(fmaxf(x1, -126.f), 126.f);
  uint64_t X = fq_f2(x0, x1), M = fq_f2(MAGIC, MAGIC), Y, F;
  asm("add.rm.f32x2 %0, %1, %2;" : "=l"(Y) : "l"(X), "l"(M));
  uint64_t YM;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(YM) : "l"(Y), "l"(M));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(F) : "l"(X), "l"(YM));
  uint64_t P = fq_fma2(F, fq_f2(C3, C3), fq_f2(C2, C2));
  P = fq_fma2(P, F, fq_f2(C1, C1));
  P = fq_fma2(P, F, fq_f2(C0, C0));
  float p0, p1, q0, q1;
  fq_uf2(P, p0, p1);
  fq_uf2(Y, q0, q1);
  y0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(q0) << 23));
  y1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(q1) << 23));
}

// P = 2^(s * sl2 - m) of 32 keys as 16 bf16x2 words; returns their sum.
__device__ inline float fq_exp32(const uint32_t (&s)[32], float sl2, float m, uint32_t (&pk)[16]) {
  const uint64_t SL = fq_f2(sl2, sl2), NM = fq_f2(-m, -m);
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float x0, x1, p0, p1;
    fq_uf2(fq_fma2(fq_f2(__uint_as_float(s[2 * i]), __uint_as_float(s[2 * i + 1])), SL, NM), x0, x1);
    if (fq_poly_pair(i)) {
      fq_exp2_poly(x0, x1, p0, p1);
    } else {
      p0 = fq_ex2(x0);
      p1 = fq_ex2(x1);
    }
    const uint32_t w = fq_bf16x2(p0, p1);
    pk[i] = w;
    if (i & 1) {
      a2 = fq_add_lo(a2, w);
      a3 = fq_add_hi(a3, w);
    } else {
      a0 = fq_add_lo(a0, w);
      a1 = fq_add_hi(a1, w);
    }
  }
  return (a0 + a1) + (a2 + a3);
}

// 2^k for an integer k in [-126, 127], exact.
__device__ inline float fq_pow2i(int k) { return __int_as_float((127 + k) << 23); }

// Scale each bf16 of 32 packed words by an exact power of two (exact unless
// the result leaves the normal range).
__device__ inline void fq_scale_bf16(uint32_t (&w)[32], float alpha) {
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float lo = __uint_as_float(w[i] << 16) * alpha, hi = __uint_as_float(w[i] & 0xFFFF0000u) * alpha;
    w[i] = fq_bf16x2(lo, hi);
  }
}

// S_h = Q_h K^T of one step (M=128, N=128 keys, K=128 dims in 8 MMAs of K=16).
__device__ __forceinline__ void fq_s_mmas(uint32_t tS, uint64_t qd, uint64_t kd) {
  using namespace fq;
  mma_ss(tS, qd, kd, IDESC_S, 0u);
#pragma unroll
  for (int kk = 1; kk < 8; ++kk)
    mma_ss(tS, qd + (((kk >> 2) * QH_DHALF + (kk & 3) * 32) >> 4), kd + (((kk >> 2) * K_DHALF + (kk & 3) * 32) >> 4),
           IDESC_S, 1u);
}

// O_h (+)= P_h V of one step: P_h of key tile t (bf16) at tS + 32 t, V_t
// MN-major in the stage; 16 keys = 16 V rows = 2048 bytes per K=16 MMA.
__device__ __forceinline__ void fq_pv_mmas(uint32_t tO, uint32_t tS, const uint8_t* vstage, bool first) {
  using namespace fq;
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const uint64_t vd = umma_desc_sw128(smem_u32(vstage + t * V_TILE), BOX, 1024);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_ts(tO, tS + 32 * t + 8 * kk, vd + ((kk * 2048) >> 4), IDESC_PV, (first && t == 0 && kk == 0) ? 0u : 1u);
  }
}

__global__ void __launch_bounds__(fq::THREADS, 1)
    fine_q_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                  const __grid_constant__ CUtensorMap mv, const FineQArgs a) {
  using namespace fq;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + Q_BYTES;
  uint8_t* sV = sK + KST * STAGE_BYTES;
  __shared__ Ctl ctl_s;
  Ctl* ctl = &ctl_s;
  volatile int* abort_flag = &ctl->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Geom& g = a.g;
  const long long cap = a.wait_cap;
  const bool nat = a.q_nat || a.k_nat || a.v_nat;

  if (threadIdx.x == 0) {
    mbar_init(&ctl->q_full, 1);
    mbar_init(&ctl->q_empty, 1);
    for (int i = 0; i < KST; ++i) {
      mbar_init(&ctl->k_full[i], 1);
      mbar_init(&ctl->k_empty[i], 1);
    }
    for (int i = 0; i < VST; ++i) {
      mbar_init(&ctl->v_full[i], 1);
      mbar_init(&ctl->v_empty[i], 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&ctl->s_full[h], 2);
      mbar_init(&ctl->p_full[h], 128);
      mbar_init(&ctl->pv_done[h], 1);
    }
    mbar_init(&ctl->drain, 1);
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
    // The warp fetches the next 32 union entries and their cube coordinates
    // with one pair of coalesced loads; lane 0 then issues the waits and
    // copies step by step.
    const bool leader = lane == 0;
    if (leader) {
      prefetch_tensormap(&mq);
      prefetch_tensormap(&mk);
      prefetch_tensormap(&mv);
    }
    long long gs = 0;   // steps loaded
    int kq = 0;         // items with steps loaded
    bool ok = true;
    for (int slot = blockIdx.x; slot < a.n_items && ok; slot += gridDim.x) {
      const int item = a.worklist[slot];
      const int n = a.ucount[item];
      if (n <= 0) continue;
      const int bh = item / a.Qn, u = item % a.Qn;
      // lanes 0-3: the item's four query tiles (a missing tile repeats the first; its rows are never stored)
      int qtile = 4 * u + (lane & 3);
      if (qtile >= g.nT) qtile = 4 * u;
      const int qcube = nat && lane < 4 ? a.tile_cube[qtile] : 0;
      if (leader && kq >= 1) ok = mbar_wait(&ctl->q_empty, (uint32_t)(kq - 1) & 1, abort_flag, a.status, cap);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      {
        const int qc0 = __shfl_sync(0xffffffffu, qcube, 0), qc1 = __shfl_sync(0xffffffffu, qcube, 1);
        const int qc2 = __shfl_sync(0xffffffffu, qcube, 2), qc3 = __shfl_sync(0xffffffffu, qcube, 3);
        const int qt0 = __shfl_sync(0xffffffffu, qtile, 0), qt1 = __shfl_sync(0xffffffffu, qtile, 1);
        const int qt2 = __shfl_sync(0xffffffffu, qtile, 2), qt3 = __shfl_sync(0xffffffffu, qtile, 3);
        if (leader) {
          // half h, tile i of the half: rows 64 i of the half, d-halves QH_DHALF apart
          mbar_arrive_expect_tx(&ctl->q_full, Q_BYTES);
          fq_tma_tile(&mq, a.q_nat, qc0, bh, qt0, sQ, QH_DHALF, &ctl->q_full);
          fq_tma_tile(&mq, a.q_nat, qc1, bh, qt1, sQ + BOX, QH_DHALF, &ctl->q_full);
          fq_tma_tile(&mq, a.q_nat, qc2, bh, qt2, sQ + QH_BYTES, QH_DHALF, &ctl->q_full);
          fq_tma_tile(&mq, a.q_nat, qc3, bh, qt3, sQ + QH_BYTES + BOX, QH_DHALF, &ctl->q_full);
        }
      }
      ++kq;
      // the next item's query tiles into L2 while this item runs
      {
        const int nslot = slot + (int)gridDim.x;
        if (nslot < a.n_items) {
          const int nitem = a.worklist[nslot];
          const int nbh = nitem / a.Qn, nu = nitem % a.Qn;
          int nt = 4 * nu + (lane & 3);
          if (nt >= g.nT) nt = 4 * nu;
          const int nc = nat && lane < 4 ? a.tile_cube[nt] : 0;
          if (lane < 4 && (lane == 0 || 4 * nu + lane < g.nT)) fq_prefetch_tile(&mq, a.q_nat, nc, nbh, nt);
        }
      }
      const int* list = a.uni + (size_t)item * g.nT;
      for (int e0 = 0; e0 < n && ok; e0 += 32) {
        int ent = e0 + lane < n ? list[e0 + lane] : 0;
        int j = ent & 0xFFFF;
        if (j >= g.nT) {  // never produced by the schedule; keep the copy in bounds
          set_status(a.status, kStatusBadBlock);
          j = 0;
          ent &= ~0xF0000;
        }
        const int cube = nat ? a.tile_cube[j] : 0;
        const int cnt = n - e0 < 32 ? n - e0 : 32;
        for (int i = 0; i < cnt; i += 2, ++gs) {
          // the step's key tiles: entries e0 + i and e0 + i + 1 (a copy of the first, selected by no
          // tile, when the item's entry count is odd)
          const bool two = i + 1 < cnt;
          const int ent0 = __shfl_sync(0xffffffffu, ent, i);
          const int cube0 = __shfl_sync(0xffffffffu, cube, i);
          const int ent1 = __shfl_sync(0xffffffffu, ent, two ? i + 1 : i);
          const int cube1 = __shfl_sync(0xffffffffu, cube, two ? i + 1 : i);
          if (leader) {
            const int j0 = ent0 & 0xFFFF, j1 = ent1 & 0xFFFF;
            const int ks = (int)(gs % KST), vs = (int)(gs % VST);
            if (gs >= KST)
              ok = mbar_wait(&ctl->k_empty[ks], (uint32_t)((gs / KST) - 1) & 1, abort_flag, a.status, cap);
            if (ok) {
              ctl->meta[ks] = ((ent0 >> 16) & 15) | (two ? ((ent1 >> 16) & 15) << 4 : 0);
              mbar_arrive_expect_tx(&ctl->k_full[ks], STAGE_BYTES);
              uint8_t* kd = sK + ks * STAGE_BYTES;
              fq_tma_tile(&mk, a.k_nat, cube0, bh, j0, kd, K_DHALF, &ctl->k_full[ks]);
              fq_tma_tile(&mk, a.k_nat, cube1, bh, j1, kd + BOX, K_DHALF, &ctl->k_full[ks]);
              if (gs >= VST)
                ok = mbar_wait(&ctl->v_empty[vs], (uint32_t)((gs / VST) - 1) & 1, abort_flag, a.status, cap);
            }
            if (ok) {
              mbar_arrive_expect_tx(&ctl->v_full[vs], STAGE_BYTES);
              uint8_t* vd = sV + vs * STAGE_BYTES;
              fq_tma_tile(&mv, a.v_nat, cube0, bh, j0, vd, BOX, &ctl->v_full[vs]);
              fq_tma_tile(&mv, a.v_nat, cube1, bh, j1, vd + V_TILE, BOX, &ctl->v_full[vs]);
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
        }
      }
    }
    // every copy issued has landed before the block exits
    if (leader) {
      if (kq > 0) mbar_drain(&ctl->q_full, (uint32_t)(kq - 1) & 1, a.status, cap);
      for (int i = 0; i < KST && i < gs; ++i) {
        const long long last = i + ((gs - 1 - i) / KST) * KST;
        mbar_drain(&ctl->k_full[i], (uint32_t)(last / KST) & 1, a.status, cap);
      }
      for (int i = 0; i < VST && i < gs; ++i) {
        const long long last = i + ((gs - 1 - i) / VST) * VST;
        mbar_drain(&ctl->v_full[i], (uint32_t)(last / VST) & 1, a.status, cap);
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    // Slot c: PV_A(c-1), S_A(c), PV_B(c-1), S_B(c), each only if its half
    // is active on that step.  A K stage is released after the step's last
    // S, a V stage after the step's last PV, the Q buffer after the item's
    // last step's S.
    long long c = 0;
    int kq = 0;
    int prev_act = 0, prev_vs = 0;     // halves active on the previous step, its V stage
    long long prev_c = -1;
    int chP[2] = {0, 0};               // PVs issued per half
    bool pv_first[2] = {false, false}; // the pending PV_h starts its item's O_h
    bool first_in_item[2] = {true, true};
    bool ok = true;
    // PV_h of the previous step; `last`: the previous step's last PV (releases its V stage)
    auto issue_pv = [&](int h) -> bool {
      if (!mbar_wait_warp(&ctl->p_full[h], (uint32_t)chP[h] & 1, abort_flag, a.status, cap)) return false;
      tc_fence_after();
      const bool last = h == 1 || !((prev_act >> 1) & 1);
      if (elect_one()) {
        fq_pv_mmas(tbase + TMEM_O + 128 * h, tbase + 128 * h, sV + prev_vs * STAGE_BYTES, pv_first[h]);
        mma_commit(&ctl->pv_done[h]);
        if (last) mma_commit(&ctl->v_empty[prev_vs]);
      }
      __syncwarp();
      ++chP[h];
      return true;
    };
    for (int slot = blockIdx.x; slot < a.n_items && ok; slot += gridDim.x) {
      const int item = a.worklist[slot];
      const int n = a.ucount[item];
      if (n <= 0) continue;
      const int steps = (n + 1) >> 1;
      first_in_item[0] = first_in_item[1] = true;
      for (int i = 0; i < steps; ++i, ++c) {
        const int ks = (int)(c % KST);
        // K(c) (and the item's Q) and V(c-1) first, so that PV_A(c-1) and S_A(c) go out back to back
        if (!mbar_wait_warp(&ctl->k_full[ks], (uint32_t)(c / KST) & 1, abort_flag, a.status, cap) ||
            (i == 0 && !mbar_wait_warp(&ctl->q_full, (uint32_t)kq & 1, abort_flag, a.status, cap)) ||
            (prev_act && !mbar_wait_warp(&ctl->v_full[prev_vs], (uint32_t)(prev_c / VST) & 1, abort_flag,
                                         a.status, cap))) {
          ok = false;
          break;
        }
        if ((prev_act & 1) && !issue_pv(0)) {
          ok = false;
          break;
        }
        const int meta = ctl->meta[ks];
        const int act = ((meta & 0x33) ? 1 : 0) | ((meta & 0xCC) ? 2 : 0);
        tc_fence_after();
        const uint64_t kd = umma_desc_sw128(smem_u32(sK + ks * STAGE_BYTES), 16, 1024);
        for (int h = 0; h < 2; ++h) {
          if (h == 1 && (prev_act & 2) && !issue_pv(1)) {
            ok = false;
            break;
          }
          if ((act >> h) & 1) {
            const bool last_s = h == 1 || !(act & 2);
            const uint64_t qd = umma_desc_sw128(smem_u32(sQ + h * QH_BYTES), 16, 1024);
            if (elect_one()) {
              ctl->info[h] = meta;
              fq_s_mmas(tbase + 128 * h, qd, kd);
              mma_commit(&ctl->s_full[h]);
              if (last_s) {
                mma_commit(&ctl->k_empty[ks]);
                if (i == steps - 1) mma_commit(&ctl->q_empty);
              }
              mbar_arrive(&ctl->s_full[h]);
            }
            __syncwarp();
            pv_first[h] = first_in_item[h];
            first_in_item[h] = false;
          }
        }
        if (!ok) break;
        prev_act = act;
        prev_vs = (int)(c % VST);
        prev_c = c;
      }
      ++kq;
    }
    // the last step's PVs
    if (ok && prev_act &&
        mbar_wait_warp(&ctl->v_full[prev_vs], (uint32_t)(prev_c / VST) & 1, abort_flag, a.status, cap)) {
      if (!(prev_act & 1) || issue_pv(0))
        if (prev_act & 2) issue_pv(1);
    }
    // every MMA this warp issued has completed before TMEM is freed
    if (elect_one()) mma_commit(&ctl->drain);
    __syncwarp();
    mbar_drain(&ctl->drain, 0, a.status, cap);
  } else if (warp >= SM_WARP0) {
    // ------------------------------------------------ softmax and epilogue
    const int h = (warp - SM_WARP0) >> 2;             // half
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;                     // row of the half
    const int qsel = 2 * h + (r >> 6);                // query tile of the row within the quad
    const int rr = r & 63;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t tS = tbase + 128 * h + lane_off;
    const uint32_t tO = tbase + TMEM_O + 128 * h + lane_off;
    const float sl2 = g.scale * 1.4426950408889634f;
    int ch = 0;   // active steps of this half so far (barrier phases)
    for (int slot = blockIdx.x; slot < a.n_items; slot += gridDim.x) {
      const int item = a.worklist[slot];
      const int n = a.ucount[item];
      const int seg = a.useg[item];
      int sa = 0, sb = 0;
      if (n > 0) {
        const int nb = seg & 0xFFFF, na = seg >> 16;
        const int steps = (n + 1) >> 1;
        sa = (nb + na + 1) >> 1;
        const int pre = (nb + 1) >> 1;
        sb = pre;
        if (n - nb - na > 0) {
          const int start = (nb + na) >> 1;
          sb += steps - start - (pre > start ? pre - start : 0);
        }
      }
      const int my_steps = h == 0 ? sa : sb;
      const int bh = item / a.Qn, u = item % a.Qn;
      const int tile = 4 * u + qsel;
      const bool valid = tile < g.nT;
      const int cube = valid && a.out_nat ? a.tile_cube[tile] : 0;   // used by the epilogue
      float m_use = -INFINITY, l = 0.f;
      bool ok = true;
      for (int st = 0; st < my_steps; ++st, ++ch) {
        if (!mbar_wait(&ctl->s_full[h], (uint32_t)ch & 1, abort_flag, a.status, cap)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int info = ctl->info[h];
        // four chunks of 32 keys (chunks 2t, 2t+1 = key tile t), all loaded at once; P of chunk j
        // (16 bf16x2 words) goes to columns 16 j .. 16 j + 15, over S values already read
        // chunks 0-2 are loaded at once; chunk 3 goes into chunk 0's registers once chunk 0 is done
        // and lands while chunks 1 and 2 are computed
        uint32_t sc[3][32];
#pragma unroll
        for (int j = 0; j < 3; ++j) tmem_ld32(tS + 32 * j, sc[j]);
#pragma unroll
        for (int j = 0; j < 3; ++j) fq_wait_ld(sc[j]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (j == 1) tmem_ld32(tS + 96, sc[0]);
          if (j == 3) fq_wait_ld(sc[0]);
          const bool sel = (info >> (4 * (j >> 1) + qsel)) & 1;
          uint32_t pk[16];
          float alpha = 1.f;
          bool rescale = false;
          if (sel) {
            const float mx = fq_max32(sc[j == 3 ? 0 : j]) * sl2;
            if (m_use == -INFINITY) {
              m_use = mx;                       // first selected chunk of the row
            } else if (mx > m_use + RESCALE_X) {
              // move the reference max up by a whole power of two
              const int k = (int)ceilf(mx - m_use);
              alpha = fq_pow2i(-(k < 126 ? k : 126));
              m_use += (float)k;
              rescale = true;
            }
            l = l * alpha + fq_exp32(sc[j == 3 ? 0 : j], sl2, m_use, pk);
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = 0u;
          }
          if (__any_sync(0xffffffffu, rescale)) {
            // P of the earlier chunks of this step is in TMEM, and O holds the PVs of the earlier
            // steps of this item: scale both by alpha (1 on the rows that keep their max)
            tmem_wait_st();
#pragma unroll 1
            for (int jj = 0; jj < j; ++jj) {
              uint32_t p0[16];
              fq_ld16(tS + 16 * jj, p0);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float lo = __uint_as_float(p0[i] << 16) * alpha, hi = __uint_as_float(p0[i] & 0xFFFF0000u) * alpha;
                p0[i] = fq_bf16x2(lo, hi);
              }
              fq_st16(tS + 16 * jj, p0);
            }
            if (st > 0) {
              if (!mbar_wait(&ctl->pv_done[h], (uint32_t)(ch - 1) & 1, abort_flag, a.status, cap)) {
                ok = false;
                break;
              }
              tc_fence_after();
#pragma unroll 1
              for (int cc = 0; cc < 4; ++cc) {
                uint32_t o[32];
                tmem_ld32(tO + cc * 32, o);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                tmem_st32(tO + cc * 32, o);
              }
            }
          }
          fq_st16(tS + 16 * j, pk);
        }

        if (!ok) break;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&ctl->p_full[h]);
      }
      if (!ok) break;
      // ---- epilogue: O / l and lse of this row, straight to its token's row
      if (my_steps > 0) {
        if (!mbar_wait(&ctl->pv_done[h], (uint32_t)(ch - 1) & 1, abort_flag, a.status, cap)) break;
        tc_fence_after();
      }
      const int tok = !valid ? 0 : (a.out_nat ? cube_row_token(g, cube, rr) : tile * kTileTokens + rr);
      __nv_bfloat16* orow = a.out + ((size_t)bh * g.N + tok) * D;
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t o[32];
        if (my_steps > 0) {
          tmem_ld32(tO + cc * 32, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
        if (valid) {
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            w[i] = fq_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
          uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
      }
      if (valid) a.lse[(size_t)bh * g.N + tok] = l > 0.f ? (m_use + __log2f(l)) * 0.6931471805599453f : -INFINITY;
      tc_fence_before();
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
    tmem_dealloc(tbase, fq::TMEM_COLS);
  }
}

cudaError_t launch_fine_q(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const FineQArgs& a,
                          int num_sms, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(fine_q_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fq::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int grid = a.n_items < num_sms ? a.n_items : num_sms;
  if (grid <= 0) return cudaSuccess;
  fine_q_kernel<<<grid, fq::THREADS, fq::SMEM_BYTES, s>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

}  // namespace fvattn
