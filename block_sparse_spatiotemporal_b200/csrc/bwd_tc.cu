// Backward pass of the block-sparse fine stage ("VSA" digest, section 3: the
// coarse predictor and the fine block-sparse attention are trained end to
// end; the fine stage is token-level softmax attention inside the selected
// tiles).  For fixed lists, with s = scale q k^T, p = exp(s - lse):
//   dv = p^T dout,  dp = dout v^T,  ds = p (dp - D),  D = rowsum(dout * out),
//   dq = scale ds k,  dk = scale ds^T q.
// The selection is piecewise constant in q and k and passes no gradient.
//
// Two persistent tcgen05 kernels share one template, so no gradient needs
// atomics:
//   * key-stationary (KV = true): a work item is two adjacent key tiles of one
//     head (128 TMEM lanes); it walks the union of the query tiles that
//     selected either key tile, one query tile (64 queries) per step, and
//     accumulates dV += P^T dO and dK += dS^T Q in TMEM;
//   * query-stationary (KV = false): a work item is two adjacent query tiles
//     (the forward's items and union lists); one selected key tile per step,
//     accumulating dQ += dS K.
// Per step two threads issue S = X0 Y0^T and dP = X1 Y1^T (X stationary:
// K, V or Q, dO; Y moving: Q, dO or K, V; M128 N64) into one of NB TMEM
// buffers (two in the key-stationary kernel, three in the query-stationary
// one, which has a single accumulator); eight warps (two per TMEM lane
// quarter, half the columns each) turn them into P and dS and write both
// back into the same TMEM columns as bf16, and a third thread's accumulating
// MMAs read them from TMEM as the A operand.  With several buffers the next
// steps' scores run on the tensor cores while the warps work on this step's.
// The moving tiles are used twice: K-major for the scores, MN-major for the
// accumulations.  Layout: tiled only.
#include "fvattn_internal.cuh"

namespace fvattn {
namespace bw {

constexpr int THREADS = 384;          // warp 0 TMA, warps 1-3 MMA, warps 4..11 compute + epilogue
constexpr int CW0 = 4;
constexpr int CTHREADS = 256;         // compute threads: two warps per TMEM lane quarter
constexpr uint32_t BOX = 64 * 128;    // 64 rows x 128 bytes
constexpr uint32_t HALF = 2 * BOX;    // one 64-dim half of the 128 stationary rows: 16 KB
constexpr uint32_t TENSOR = 4 * BOX;  // 128 rows x 128 dims bf16: 32 KB
constexpr uint32_t MTENSOR = 2 * BOX; // one moving tile, 64 rows x 128 dims: 16 KB (halves BOX apart)
constexpr int MST = 4;                // moving stages
constexpr uint32_t STAT_BYTES = 2 * TENSOR;
constexpr uint32_t MOV_BYTES = 2 * MTENSOR;
constexpr uint32_t SMEM_BYTES = 1024 + STAT_BYTES + MST * MOV_BYTES;
constexpr uint32_t TMEM_COLS = 512;
// NB score buffers: S buffer b at columns 64 b, dP buffer b at 64 (NB + b), then the
// accumulators (128 columns each).  The key-stationary kernel has two accumulators and
// room for two buffers, the query-stationary kernel one accumulator and three buffers.
template <bool KV> struct Tm {
  static constexpr int NB = KV ? 2 : 3;
  static constexpr uint32_t S = 0, DP = 64 * NB, ACC0 = 128 * NB, ACC1 = ACC0 + 128;
  static_assert(ACC0 + (KV ? 256 : 128) <= TMEM_COLS, "TMEM columns");
};
constexpr int MAXNB = 3;
constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 64, false, false);
constexpr uint32_t IDESC_ACC = idesc_bf16_f32(128, 128, false, true);
constexpr int STEP_LAST = 1 << 4;     // step word: sel of the moving tile (bits 0-1), last
static_assert(SMEM_BYTES + 3 * 1024 <= 227 * 1024, "shared memory");

struct Ctl {
  uint64_t stat_full, stat_empty;
  uint64_t mov_full[MST], mov_empty[MST];
  uint64_t s_full[MAXNB];   // S and dP of step c in buffer c % NB (two commits) + step word written
  uint64_t p_full[MAXNB];   // P / dS of step c written back (256 compute threads)
  uint64_t step_done[MAXNB];// the accumulating MMAs of step c, which read buffer c % NB, complete
  uint64_t acc_full;    // the item's accumulators complete
  uint64_t acc_empty;   // the epilogue read them (256 threads)
  uint64_t drain;
  int meta[MST];        // step word per moving stage
  int info[MAXNB];      // step word of the step in each buffer
  float lse2[MST][64];  // key-stationary only: lse * log2(e) of the step's queries
  float dd[MST][64];    //   and their D
  uint32_t tmem_base;
  int abort;
};

__device__ inline float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ inline uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&b);
}

__device__ inline void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Both 64-dim halves of one 64-row tile of a tiled [BH, N, 128] tensor, the
// second half `stride` bytes after the first.
__device__ inline void load_tile(const CUtensorMap* map, int bh, int tile, uint8_t* dst, uint32_t stride,
                                 uint64_t* bar) {
  tma_load_3d(dst, map, bar, 0, tile * kTileTokens, bh);
  tma_load_3d(dst + stride, map, bar, 64, tile * kTileTokens, bh);
}

// K-major operand whose two 64-dim halves are `stride` bytes apart.
__device__ inline uint64_t kdesc(uint32_t base, uint32_t stride, int kk) {
  return umma_desc_sw128(base + (kk >> 2) * stride + (kk & 3) * 32, 16, 1024);
}

template <bool KV>
__global__ void __launch_bounds__(THREADS, 1)
    bwd_tc_kernel(const __grid_constant__ CUtensorMap ms0, const __grid_constant__ CUtensorMap ms1,
                  const __grid_constant__ CUtensorMap mm0, const __grid_constant__ CUtensorMap mm1,
                  const BwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sStat = smem;                      // X0 (32 KB) then X1 (32 KB)
  uint8_t* sMov = smem + STAT_BYTES;          // per stage: Y0 then Y1
  __shared__ Ctl ctl_s;
  Ctl* ctl = &ctl_s;
  volatile int* abort_flag = &ctl->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Geom& g = a.g;
  const long long cap = a.wait_cap;

  if (threadIdx.x == 0) {
    mbar_init(&ctl->stat_full, 1);
    mbar_init(&ctl->stat_empty, 2);      // one commit per score thread
    for (int i = 0; i < MST; ++i) {
      mbar_init(&ctl->mov_full[i], KV ? 32 : 1);
      mbar_init(&ctl->mov_empty[i], 1);
    }
    for (int i = 0; i < MAXNB; ++i) {
      mbar_init(&ctl->s_full[i], 3);     // two commits + the step word
      mbar_init(&ctl->p_full[i], CTHREADS);
      mbar_init(&ctl->step_done[i], 1);
    }
    mbar_init(&ctl->acc_full, 1);
    mbar_init(&ctl->acc_empty, CTHREADS);
    mbar_init(&ctl->drain, 3);           // final commit of each MMA thread
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

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    const bool leader = lane == 0;
    if (leader) {
      prefetch_tensormap(&ms0);
      prefetch_tensormap(&ms1);
      prefetch_tensormap(&mm0);
      prefetch_tensormap(&mm1);
    }
    long long gs = 0;       // moving steps loaded
    int k = 0, stat_issued = 0;
    bool ok = true;
    for (int slot = blockIdx.x; slot < a.n_items && ok; slot += gridDim.x, ++k) {
      const int item = a.worklist[slot];
      const int bh = item / g.P, pd = item % g.P;
      const int t0 = kItemTiles * pd;
      const int t1 = t0 + 1 < g.nT ? t0 + 1 : t0;   // a missing second tile repeats the first (never stored)
      if (leader) {
        if (k >= 1) ok = mbar_wait(&ctl->stat_empty, (uint32_t)(k - 1) & 1, abort_flag, a.status, cap);
        if (ok) {
          mbar_arrive_expect_tx(&ctl->stat_full, STAT_BYTES);
          load_tile(&ms0, bh, t0, sStat, HALF, &ctl->stat_full);
          load_tile(&ms0, bh, t1, sStat + BOX, HALF, &ctl->stat_full);
          load_tile(&ms1, bh, t0, sStat + TENSOR, HALF, &ctl->stat_full);
          load_tile(&ms1, bh, t1, sStat + TENSOR + BOX, HALF, &ctl->stat_full);
          ++stat_issued;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      const int n = a.ucount[item];
      const int* list = a.uni + (size_t)item * g.nT;
      for (int e0 = 0; e0 < n && ok; e0 += 32) {
        int ent = e0 + lane < n ? list[e0 + lane] : 0;
        if ((ent & 0xFFFF) >= g.nT) {  // never produced by the schedule; keep the copy in bounds
          set_status(a.status, kStatusBadBlock);
          ent &= ~0x3FFFF;
        }
        const int cnt = n - e0 < 32 ? n - e0 : 32;
        for (int i = 0; i < cnt; ++i, ++gs) {
          const int e = __shfl_sync(0xffffffffu, ent, i);
          const int j = e & 0xFFFF;
          const int st = (int)(gs % MST);
          if (leader && gs >= MST)
            ok = mbar_wait(&ctl->mov_empty[st], (uint32_t)((gs / MST) - 1) & 1, abort_flag, a.status, cap);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          if (KV) {
            // the step's 64 queries: lse * log2(e) and D, 2 per lane
            const size_t row = (size_t)bh * g.N + (size_t)j * kTileTokens + 2 * lane;
            const float2 l2 = *reinterpret_cast<const float2*>(a.lse2 + row);
            const float2 d2 = *reinterpret_cast<const float2*>(a.dd + row);
            ctl->lse2[st][2 * lane] = l2.x;
            ctl->lse2[st][2 * lane + 1] = l2.y;
            ctl->dd[st][2 * lane] = d2.x;
            ctl->dd[st][2 * lane + 1] = d2.y;
          }
          if (leader) {
            ctl->meta[st] = ((e >> 16) & 3) | ((e0 + i == n - 1) ? STEP_LAST : 0);
            mbar_arrive_expect_tx(&ctl->mov_full[st], MOV_BYTES);
            uint8_t* dst = sMov + st * MOV_BYTES;
            load_tile(&mm0, bh, j, dst, BOX, &ctl->mov_full[st]);
            load_tile(&mm1, bh, j, dst + MTENSOR, BOX, &ctl->mov_full[st]);
          } else if (KV) {
            mbar_arrive(&ctl->mov_full[st]);
          }
        }
      }
    }
    // every copy issued has landed before the block exits
    if (leader) {
      if (stat_issued >= 1) mbar_drain(&ctl->stat_full, (uint32_t)(stat_issued - 1) & 1, a.status, cap);
      for (int i = 0; i < MST && i < gs; ++i) {
        const long long last = i + ((gs - 1 - i) / MST) * MST;
        mbar_drain(&ctl->mov_full[i], (uint32_t)(last / MST) & 1, a.status, cap);
      }
    }
  } else if ((warp == 1 || warp == 2) && lane == 0) {
    // ------------------------------------------------------- MMA: scores
    // Warp 1 issues S = X0 Y0^T, warp 2 dP = X1 Y1^T (one thread issues a
    // tcgen05.mma only every ~100 clk, about what an N=64 MMA takes to run,
    // so the step's MMAs are spread over three threads).  Step c goes to
    // buffer c % NB once the accumulations of step c - NB, which read it, are
    // complete; the stationary tiles are released after the item's last score.
    const bool is_s = warp == 1;
    long long c = 0;
    int k = 0;
    bool ok = true;
    const uint32_t x = smem_u32(sStat) + (is_s ? 0u : TENSOR);
    const uint32_t tdst = tbase + (is_s ? Tm<KV>::S : Tm<KV>::DP);
    for (int slot = blockIdx.x; slot < a.n_items && ok; slot += gridDim.x, ++k) {
      if (!mbar_wait(&ctl->stat_full, (uint32_t)k & 1, abort_flag, a.status, cap)) break;
      while (true) {
        const int st = (int)(c % MST);
        constexpr int NB = Tm<KV>::NB;
        const int b = (int)(c % NB);
        if (!mbar_wait(&ctl->mov_full[st], (uint32_t)(c / MST) & 1, abort_flag, a.status, cap) ||
            (c >= NB && !mbar_wait(&ctl->step_done[b], (uint32_t)((c - NB) / NB) & 1, abort_flag, a.status, cap))) {
          ok = false;
          break;
        }
        const int meta = ctl->meta[st];
        if (is_s) ctl->info[b] = meta;
        tc_fence_after();
        const uint32_t y = smem_u32(sMov + st * MOV_BYTES) + (is_s ? 0u : MTENSOR);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tdst + 64 * b, kdesc(x, HALF, kk), kdesc(y, BOX, kk), IDESC_S, kk ? 1u : 0u);
        mma_commit(&ctl->s_full[b]);
        if (is_s) mbar_arrive(&ctl->s_full[b]);
        ++c;
        if (meta & STEP_LAST) break;
      }
      if (!ok) break;
      mma_commit(&ctl->stat_empty);
    }
    // every MMA issued has completed before TMEM is freed
    mma_commit(&ctl->drain);
    mbar_drain(&ctl->drain, 0, a.status, cap);
  } else if (warp == 3 && lane == 0) {
    // ------------------------------------------------- MMA: accumulations
    long long c = 0;
    int k = 0;
    bool ok = true;
    for (int slot = blockIdx.x; slot < a.n_items && ok; slot += gridDim.x, ++k) {
      if (k >= 1 && !mbar_wait(&ctl->acc_empty, (uint32_t)(k - 1) & 1, abort_flag, a.status, cap)) break;
      bool first = true;
      while (true) {
        constexpr int NB = Tm<KV>::NB;
        const int b = (int)(c % NB);
        const int st = (int)(c % MST);
        if (!mbar_wait(&ctl->p_full[b], (uint32_t)(c / NB) & 1, abort_flag, a.status, cap)) {
          ok = false;
          break;
        }
        const int info = ctl->info[b];
        tc_fence_after();
        // 16 moving rows = 2048 bytes of the MN-major operand per K step; P / dS of moving rows
        // 16 kk .. 16 kk + 15 in TMEM columns 32 (kk / 2) + 8 (kk % 2) .. + 7 of the buffer
        // (bf16 pairs; each 32-row half packed at the start of its own 32 columns)
        const uint32_t y0 = smem_u32(sMov + st * MOV_BYTES), y1 = y0 + MTENSOR;
        const uint64_t b0 = umma_desc_sw128(y0, BOX, 1024), b1 = umma_desc_sw128(y1, BOX, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t acc = (first && kk == 0) ? 0u : 1u;
          const uint32_t col = 64 * b + 32 * (kk >> 1) + 8 * (kk & 1);
          if (KV) {
            mma_ts(tbase + Tm<KV>::ACC1, tbase + Tm<KV>::S + col, b1 + ((kk * 2048) >> 4), IDESC_ACC, acc);  // dV
            mma_ts(tbase + Tm<KV>::ACC0, tbase + Tm<KV>::DP + col, b0 + ((kk * 2048) >> 4), IDESC_ACC, acc); // dK
          } else {
            mma_ts(tbase + Tm<KV>::ACC0, tbase + Tm<KV>::DP + col, b0 + ((kk * 2048) >> 4), IDESC_ACC, acc); // dQ
          }
        }
        mma_commit(&ctl->mov_empty[st]);
        mma_commit(&ctl->step_done[b]);
        first = false;
        ++c;
        if (info & STEP_LAST) break;
      }
      if (!ok) break;
      mma_commit(&ctl->acc_full);
    }
    mma_commit(&ctl->drain);
    mbar_drain(&ctl->drain, 0, a.status, cap);
  } else if (warp >= CW0) {
    // ------------------------------------------------- P, dS and epilogue
    // warps 4..7 take moving columns 0..31 of every step and accumulator
    // columns 0..63, warps 8..11 the other half
    const int q4 = warp & 3;
    const int part = (warp - CW0) >> 2;
    const int r = q4 * 32 + lane;                 // TMEM lane = row of the item
    const int h = r >> 6;                         // stationary tile of the row
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const float sl2 = a.scale_log2;
    long long c = 0;
    int k = 0;
    for (int slot = blockIdx.x; slot < a.n_items; slot += gridDim.x, ++k) {
      const int item = a.worklist[slot];
      const int bh = item / g.P, pd = item % g.P;
      const int tile = kItemTiles * pd + h;
      const bool valid = tile < g.nT;
      const size_t row = (size_t)bh * g.N + (size_t)(valid ? tile : 0) * kTileTokens + (r & 63);
      float lr = 0.f, dr = 0.f;
      if (!KV) {
        lr = a.lse2[row];
        dr = a.dd[row];
      }
      bool ok = true;
      while (true) {
        constexpr int NB = Tm<KV>::NB;
        const int b = (int)(c % NB);
        if (!mbar_wait(&ctl->s_full[b], (uint32_t)(c / NB) & 1, abort_flag, a.status, cap)) {
          ok = false;
          break;
        }
        const int info = ctl->info[b];
        const int st = (int)(c % MST);
        tc_fence_after();
        const bool on = ((info & 3) >> h) & 1;       // uniform across the warp
        const uint32_t tS = tbase + Tm<KV>::S + 64 * b + lane_off, tD = tbase + Tm<KV>::DP + 64 * b + lane_off;
        {
          const int ch = part;
          uint32_t pk[16], dk[16];
          if (on) {
            uint32_t s[32], dp[32];
            tmem_ld32(tS + 32 * ch, s);
            tmem_ld32(tD + 32 * ch, dp);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float p[2], d[2];
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                const int col = 32 * ch + 2 * i + u;
                const float l2 = KV ? ctl->lse2[st][col] : lr;
                const float dv = KV ? ctl->dd[st][col] : dr;
                p[u] = ex2(fmaf(__uint_as_float(s[2 * i + u]), sl2, -l2));
                d[u] = p[u] * (__uint_as_float(dp[2 * i + u]) - dv);
              }
              pk[i] = pack_bf16(p[0], p[1]);
              dk[i] = pack_bf16(d[0], d[1]);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[i] = dk[i] = 0u;
          }
          // packed into the first 16 of the 32 columns this warp read (the other
          // warp of the lane quarter reads and writes only its own 32)
          if (KV) tmem_st16(tS + 32 * ch, pk);
          tmem_st16(tD + 32 * ch, dk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&ctl->p_full[b]);
        ++c;
        if (info & STEP_LAST) break;
      }
      if (!ok) break;
      // ---- epilogue: accumulators to bf16 rows of the stationary tiles
      if (!mbar_wait(&ctl->acc_full, (uint32_t)k & 1, abort_flag, a.status, cap)) break;
      tc_fence_after();
#pragma unroll 1
      for (int o = 0; o < (KV ? 2 : 1); ++o) {
        const uint32_t tacc = tbase + (o == 0 ? Tm<KV>::ACC0 : Tm<KV>::ACC1) + lane_off;
        const float mul = o == 0 ? a.scale : 1.f;      // dq, dk carry the softmax scale; dv does not
        __nv_bfloat16* dst = (o == 0 ? a.out0 : a.out1) + row * 128;
#pragma unroll 1
        for (int ch = 2 * part; ch < 2 * part + 2; ++ch) {
          uint32_t v[32];
          tmem_ld32(tacc + 32 * ch, v);
          tmem_wait_ld();
          if (valid) {
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              w[i] = pack_bf16(__uint_as_float(v[2 * i]) * mul, __uint_as_float(v[2 * i + 1]) * mul);
            uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * ch);
#pragma unroll
            for (int i = 0; i < 4; ++i) d4[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&ctl->acc_empty);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, TMEM_COLS);
  }
}

// D = rowsum(dout * out) in fp32 and lse * log2(e), one row per 16 threads.
__global__ void bwd_prep_kernel(const __nv_bfloat16* __restrict__ out, const __nv_bfloat16* __restrict__ dout,
                                const float* __restrict__ lse, float* __restrict__ lse2, float* __restrict__ dd,
                                long long rows) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long row = t >> 4;
  const int part = (int)(t & 15);
  float acc = 0.f;
  if (row < rows) {
    const uint4 o4 = reinterpret_cast<const uint4*>(out + row * 128)[part];
    const uint4 g4 = reinterpret_cast<const uint4*>(dout + row * 128)[part];
    const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&o4);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&g4);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 of = __bfloat1622float2(o2[i]), gf = __bfloat1622float2(g2[i]);
      acc = fmaf(of.x, gf.x, acc);
      acc = fmaf(of.y, gf.y, acc);
    }
  }
#pragma unroll
  for (int o = 8; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (row < rows && part == 0) {
    dd[row] = acc;
    lse2[row] = lse[row] * 1.4426950408889634f;
  }
}

// bit i of bitmap[bh][j] <=> query tile i of head bh selected key tile j.
__global__ void transpose_bits_kernel(Geom g, const int* __restrict__ counts, const int* __restrict__ idx, int cap,
                                      uint32_t* __restrict__ bits, int* status) {
  const int words = (g.nT + 31) / 32;
  const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= (long long)g.BH * g.nT) return;
  const int bh = (int)(warp / g.nT), i = (int)(warp % g.nT);
  int c = counts[warp];
  if (c < 0 || c > g.nT) {
    if (lane == 0) set_status(status, kStatusBadBlock);
    c = c < 0 ? 0 : g.nT;
  }
  const int* list = idx + (size_t)warp * cap;
  for (int e = lane; e < c; e += 32) {
    const int j = list[e];
    if (j < 0 || j >= g.nT || (e > 0 && list[e - 1] >= j)) {
      set_status(status, kStatusBadBlock);
      continue;
    }
    atomicOr(&bits[((size_t)bh * g.nT + j) * words + (i >> 5)], 1u << (i & 31));
  }
}

// Union lists of the key-stationary items (key tiles 2p, 2p+1 of a head):
// entry = query tile | (selected key tile 2p, 2p+1) << 16, last entry flagged
// with bit 22; an item no query tile attends gets one fully masked entry.
// One warp per item, entries in ascending query tile order.
__global__ void key_union_kernel(Geom g, const uint32_t* __restrict__ bits, int* __restrict__ uni,
                                 int* __restrict__ ucount) {
  const int words = (g.nT + 31) / 32;
  const long long item = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (item >= (long long)g.BH * g.P) return;
  const int bh = (int)(item / g.P), pd = (int)(item % g.P);
  const int j0 = kItemTiles * pd, j1 = j0 + 1;
  const uint32_t* b0 = bits + ((size_t)bh * g.nT + j0) * words;
  const uint32_t* b1 = j1 < g.nT ? bits + ((size_t)bh * g.nT + j1) * words : nullptr;
  int* out = uni + item * (long long)g.nT;
  int n = 0;
  for (int w = 0; w < words; ++w) {
    const int i = w * 32 + lane;
    const uint32_t w0 = b0[w], w1 = b1 ? b1[w] : 0u;
    const uint32_t sel = ((w0 >> lane) & 1u) | (((w1 >> lane) & 1u) << 1);
    const unsigned bal = __ballot_sync(0xffffffffu, sel != 0u);
    const int pos = n + __popc(bal & ((1u << lane) - 1u));
    if (sel) out[pos] = i | (int)(sel << 16);
    n += __popc(bal);
  }
  __syncwarp();
  if (lane == 0) {
    if (n == 0) {
      out[0] = 0;
      n = 1;
    }
    out[n - 1] |= 1 << 22;
    ucount[item] = n;
  }
}

template <bool KV>
cudaError_t launch_v(const CUtensorMap& s0, const CUtensorMap& s1, const CUtensorMap& m0, const CUtensorMap& m1,
                     const BwdArgs& a, int num_sms, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(bwd_tc_kernel<KV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int grid = a.n_items < num_sms ? a.n_items : num_sms;
  if (grid <= 0) return cudaSuccess;
  bwd_tc_kernel<KV><<<grid, THREADS, SMEM_BYTES, s>>>(s0, s1, m0, m1, a);
  return cudaGetLastError();
}

}  // namespace bw

cudaError_t launch_bwd_prep(const void* out, const void* dout, const float* lse, float* lse2, float* dd, long long rows,
                            cudaStream_t s) {
  const long long threads = rows * 16;
  bw::bwd_prep_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(out), static_cast<const __nv_bfloat16*>(dout), lse, lse2, dd, rows);
  return cudaGetLastError();
}

cudaError_t launch_key_union(const Geom& g, const int* counts, const int* idx, int cap, uint32_t* bits, int* uni,
                             int* ucount, int* status, cudaStream_t s) {
  const int words = (g.nT + 31) / 32;
  cudaError_t e = cudaMemsetAsync(bits, 0, sizeof(uint32_t) * (size_t)g.BH * g.nT * words, s);
  if (e != cudaSuccess) return e;
  const long long rows = (long long)g.BH * g.nT;
  bw::transpose_bits_kernel<<<(unsigned)((rows * 32 + 255) / 256), 256, 0, s>>>(g, counts, idx, cap, bits, status);
  const long long items = (long long)g.BH * g.P;
  bw::key_union_kernel<<<(unsigned)((items * 32 + 255) / 256), 256, 0, s>>>(g, bits, uni, ucount);
  return cudaGetLastError();
}

cudaError_t launch_bwd(const CUtensorMap& s0, const CUtensorMap& s1, const CUtensorMap& m0, const CUtensorMap& m1,
                       const BwdArgs& a, bool key_stationary, int num_sms, cudaStream_t s) {
  return key_stationary ? bw::launch_v<true>(s0, s1, m0, m1, a, num_sms, s)
                        : bw::launch_v<false>(s0, s1, m0, m1, a, num_sms, s);
}

}  // namespace fvattn
