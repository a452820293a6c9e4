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
//     selected either key tile, two query tiles (128 queries) per step, and
//     accumulates dV += P^T dO and dK += dS^T Q in TMEM;
//   * query-stationary (KV = false): a work item is two adjacent query tiles
//     (the forward's items and union lists); per step two selected key tiles,
//     accumulating dQ += dS K.
// Per step one thread issues S = X0 Y0^T and dP = X1 Y1^T (X stationary:
// K, V or Q, dO; Y moving: Q, dO or K, V) into TMEM; four warps (one TMEM lane
// per thread) turn them into P and dS, write both back into the same TMEM
// columns as bf16, and the accumulating MMAs read them from TMEM as the A
// operand.  The moving tiles are used twice: K-major for the scores,
// MN-major for the accumulations.  Layout: tiled only.
#include "fvattn_internal.cuh"

namespace fvattn {
namespace bw {

constexpr int THREADS = 256;          // warp 0 TMA, warp 1 MMA, warps 4..7 compute + epilogue
constexpr int CW0 = 4;
constexpr uint32_t BOX = 64 * 128;    // 64 rows x 128 bytes
constexpr uint32_t HALF = 2 * BOX;    // one 64-dim half of 128 rows: 16 KB
constexpr uint32_t TENSOR = 4 * BOX;  // 128 rows x 128 dims bf16: 32 KB
constexpr int MST = 2;                // moving stages
constexpr uint32_t STAT_BYTES = 2 * TENSOR;
constexpr uint32_t MOV_BYTES = 2 * TENSOR;
constexpr uint32_t SMEM_BYTES = 1024 + STAT_BYTES + MST * MOV_BYTES;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t T_S = 0, T_DP = 128, T_ACC0 = 256, T_ACC1 = 384;
constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, false, false);
constexpr uint32_t IDESC_ACC = idesc_bf16_f32(128, 128, false, true);
constexpr int STEP_LAST = 1 << 4;     // step word: sel of moving tile 0 (bits 0-1), tile 1 (2-3), last
static_assert(SMEM_BYTES + 3 * 1024 <= 227 * 1024, "shared memory");

struct Ctl {
  uint64_t stat_full, stat_empty;
  uint64_t mov_full[MST], mov_empty[MST];
  uint64_t s_full;      // S and dP of the step in TMEM (commit) + step word written (MMA thread)
  uint64_t p_full;      // P / dS written back (128 compute threads)
  uint64_t step_done;   // the step's accumulating MMAs complete (they read P / dS)
  uint64_t acc_full;    // the item's accumulators complete
  uint64_t acc_empty;   // the epilogue read them (128 threads)
  uint64_t drain;
  int meta[MST];        // step word per moving stage
  int info;             // step word of the step in TMEM
  float lse2[MST][128]; // key-stationary only: lse * log2(e) of the step's queries
  float dd[MST][128];   //   and their D
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

// Both 64-dim halves of one 64-row tile of a tiled [BH, N, 128] tensor into
// rows 0..63 (slot 0) or 64..127 (slot 1) of a 128-row operand.
__device__ inline void load_tile(const CUtensorMap* map, int bh, int tile, uint8_t* base, int slot, uint64_t* bar) {
  tma_load_3d(base + slot * BOX, map, bar, 0, tile * kTileTokens, bh);
  tma_load_3d(base + slot * BOX + HALF, map, bar, 64, tile * kTileTokens, bh);
}

// 128 rows x 128 bytes of a tensor in SMEM (two 16 KB halves), K-major.
__device__ inline uint64_t kdesc(uint32_t base, int kk) {
  return umma_desc_sw128(base + (kk >> 2) * HALF + (kk & 3) * 32, 16, 1024);
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
    mbar_init(&ctl->stat_empty, 1);
    for (int i = 0; i < MST; ++i) {
      mbar_init(&ctl->mov_full[i], KV ? 32 : 1);
      mbar_init(&ctl->mov_empty[i], 1);
    }
    mbar_init(&ctl->s_full, 2);
    mbar_init(&ctl->p_full, 128);
    mbar_init(&ctl->step_done, 1);
    mbar_init(&ctl->acc_full, 1);
    mbar_init(&ctl->acc_empty, 128);
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
          load_tile(&ms0, bh, t0, sStat, 0, &ctl->stat_full);
          load_tile(&ms0, bh, t1, sStat, 1, &ctl->stat_full);
          load_tile(&ms1, bh, t0, sStat + TENSOR, 0, &ctl->stat_full);
          load_tile(&ms1, bh, t1, sStat + TENSOR, 1, &ctl->stat_full);
          ++stat_issued;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      const int n = a.ucount[item];
      const int* list = a.uni + (size_t)item * g.nT;
      const int steps = (n + 1) >> 1;
      for (int e0 = 0; e0 < n && ok; e0 += 32) {
        int ent = e0 + lane < n ? list[e0 + lane] : 0;
        if ((ent & 0xFFFF) >= g.nT) {  // never produced by the schedule; keep the copy in bounds
          set_status(a.status, kStatusBadBlock);
          ent &= ~0x3FFFF;
        }
        const int cnt = n - e0 < 32 ? n - e0 : 32;
        for (int i = 0; i < cnt; i += 2, ++gs) {
          const bool two = i + 1 < cnt;
          const int ent0 = __shfl_sync(0xffffffffu, ent, i);
          const int ent1 = __shfl_sync(0xffffffffu, ent, two ? i + 1 : i);
          const int j0 = ent0 & 0xFFFF, j1 = ent1 & 0xFFFF;
          const int st = (int)(gs % MST);
          const int step = (e0 + i) >> 1;
          if (leader && gs >= MST)
            ok = mbar_wait(&ctl->mov_empty[st], (uint32_t)((gs / MST) - 1) & 1, abort_flag, a.status, cap);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          if (KV) {
            // the step's 128 queries: lse * log2(e) and D, 4 per lane
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int q = lane * 4 + u;
              const size_t row = (size_t)bh * g.N + (size_t)(q < 64 ? j0 : j1) * kTileTokens + (q & 63);
              ctl->lse2[st][q] = a.lse2[row];
              ctl->dd[st][q] = a.dd[row];
            }
          }
          if (leader) {
            ctl->meta[st] = ((ent0 >> 16) & 3) | (two ? ((ent1 >> 16) & 3) << 2 : 0) |
                            (step == steps - 1 ? STEP_LAST : 0);
            mbar_arrive_expect_tx(&ctl->mov_full[st], MOV_BYTES);
            uint8_t* dst = sMov + st * MOV_BYTES;
            load_tile(&mm0, bh, j0, dst, 0, &ctl->mov_full[st]);
            load_tile(&mm0, bh, j1, dst, 1, &ctl->mov_full[st]);
            load_tile(&mm1, bh, j0, dst + TENSOR, 0, &ctl->mov_full[st]);
            load_tile(&mm1, bh, j1, dst + TENSOR, 1, &ctl->mov_full[st]);
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
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA
    long long c = 0;
    int k = 0;
    bool ok = true;
    const uint32_t s0 = smem_u32(sStat), s1 = s0 + TENSOR;
    for (int slot = blockIdx.x; slot < a.n_items && ok; slot += gridDim.x, ++k) {
      if (!mbar_wait(&ctl->stat_full, (uint32_t)k & 1, abort_flag, a.status, cap)) break;
      if (k >= 1 && !mbar_wait(&ctl->acc_empty, (uint32_t)(k - 1) & 1, abort_flag, a.status, cap)) break;
      tc_fence_after();
      bool first = true;
      while (true) {
        const int st = (int)(c % MST);
        if (!mbar_wait(&ctl->mov_full[st], (uint32_t)(c / MST) & 1, abort_flag, a.status, cap)) {
          ok = false;
          break;
        }
        // S and dP overwrite the P / dS the previous step's accumulations read
        if (c >= 1 && !mbar_wait(&ctl->step_done, (uint32_t)(c - 1) & 1, abort_flag, a.status, cap)) {
          ok = false;
          break;
        }
        const int meta = ctl->meta[st];
        ctl->info = meta;
        tc_fence_after();
        const uint32_t y0 = smem_u32(sMov + st * MOV_BYTES), y1 = y0 + TENSOR;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_ss(tbase + T_S, kdesc(s0, kk), kdesc(y0, kk), IDESC_S, kk ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_ss(tbase + T_DP, kdesc(s1, kk), kdesc(y1, kk), IDESC_S, kk ? 1u : 0u);
        mma_commit(&ctl->s_full);
        mbar_arrive(&ctl->s_full);
        if (!mbar_wait(&ctl->p_full, (uint32_t)c & 1, abort_flag, a.status, cap)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // 16 moving rows = 16 operand rows of 128 bytes per K step; P / dS of moving row 16 kk in
        // TMEM columns 8 kk .. 8 kk + 7 (bf16 pairs)
        const uint64_t b0 = umma_desc_sw128(y0, HALF, 1024), b1 = umma_desc_sw128(y1, HALF, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t acc = (first && kk == 0) ? 0u : 1u;
          if (KV) {
            mma_ts(tbase + T_ACC1, tbase + T_S + 8 * kk, b1 + ((kk * 2048) >> 4), IDESC_ACC, acc);   // dV
            mma_ts(tbase + T_ACC0, tbase + T_DP + 8 * kk, b0 + ((kk * 2048) >> 4), IDESC_ACC, acc);  // dK
          } else {
            mma_ts(tbase + T_ACC0, tbase + T_DP + 8 * kk, b0 + ((kk * 2048) >> 4), IDESC_ACC, acc);  // dQ
          }
        }
        mma_commit(&ctl->mov_empty[st]);
        mma_commit(&ctl->step_done);
        first = false;
        ++c;
        if (meta & STEP_LAST) break;
      }
      if (!ok) break;
      mma_commit(&ctl->acc_full);
      mma_commit(&ctl->stat_empty);
    }
    // every MMA issued has completed before TMEM is freed
    mma_commit(&ctl->drain);
    mbar_drain(&ctl->drain, 0, a.status, cap);
  } else if (warp >= CW0) {
    // ------------------------------------------------- P, dS and epilogue
    const int q4 = warp & 3;
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
        if (!mbar_wait(&ctl->s_full, (uint32_t)c & 1, abort_flag, a.status, cap)) {
          ok = false;
          break;
        }
        const int info = ctl->info;
        const int st = (int)(c % MST);
        tc_fence_after();
#pragma unroll 1
        for (int ch = 0; ch < 4; ++ch) {
          const int t = ch >> 1;
          const bool on = (((info >> (2 * t)) & 3) >> h) & 1;     // uniform across the warp
          uint32_t pk[16], dk[16];
          if (on) {
            uint32_t s[32], dp[32];
            tmem_ld32(tbase + T_S + lane_off + 32 * ch, s);
            tmem_ld32(tbase + T_DP + lane_off + 32 * ch, dp);
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
          if (KV) tmem_st16(tbase + T_S + lane_off + 16 * ch, pk);
          tmem_st16(tbase + T_DP + lane_off + 16 * ch, dk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&ctl->p_full);
        ++c;
        if (info & STEP_LAST) break;
      }
      if (!ok) break;
      // ---- epilogue: accumulators to bf16 rows of the stationary tiles
      if (!mbar_wait(&ctl->acc_full, (uint32_t)k & 1, abort_flag, a.status, cap)) break;
      tc_fence_after();
#pragma unroll 1
      for (int o = 0; o < (KV ? 2 : 1); ++o) {
        const uint32_t tacc = tbase + (o == 0 ? T_ACC0 : T_ACC1) + lane_off;
        const float mul = o == 0 ? a.scale : 1.f;      // dq, dk carry the softmax scale; dv does not
        __nv_bfloat16* dst = (o == 0 ? a.out0 : a.out1) + row * 128;
#pragma unroll 1
        for (int ch = 0; ch < 4; ++ch) {
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
