// Coarse scores on the tensor cores ("VSA" digest, section 3: pooled coarse
// stage predicting per-tile importance): S = scale * Qp Kp^T for every
// (query tile, key tile) pair of a head, in fp32.
//
// The pooled means are fp32.  Each arrives split into two tf32 values,
// hi = rn_tf32(x) and lo = rn_tf32(x - hi), so |x - hi - lo| <= 2^-22 |x|
// and |lo| <= 2^-11 |x|.  The product is accumulated from the three tf32
// products hi.hi + hi.lo + lo.hi (kind::tf32, fp32 accumulation); the
// dropped lo.lo term is below 2^-22 |q||k| per dimension.  The result has
// about the accuracy of an fp32 FFMA dot product.
//
// Persistent, one CTA per SM, 192 threads.  A unit is one 128 x 128 block
// (head, query block, key block); CTA c takes the units [c U / G, (c+1) U / G)
// of the U in that order, so every CTA gets the same number of blocks within
// one and consecutive units share their query rows.  Warp 0 loads a unit's
// pooled query rows when they change (after the MMAs reading the previous
// ones completed) and streams pooled key rows in 32-dim slices of 128 rows
// (TMA, 3-stage ring); warp 1 issues the MMAs (M=128, N=128, K=8) into one of
// two TMEM accumulators; warps 2-5 drain a finished block (thread r = query
// row r) while the next is computed.
//
// Two epilogues.  Tile scores (rows = tiles): the scaled logits go to the
// fp32 score buffer.  Sub-block scores ("DFSAttn" digest, section 2; rows =
// 2x2x2 sub-blocks, 8 per tile, key sub-blocks of a tile adjacent): every
// group of 8 columns is one key tile, reduced to T = log2 sum 2^(s log2 e),
// the log of the unnormalised softmax mass the query sub-block gives that
// key tile.
#include "fvattn_internal.cuh"

namespace fvattn {
namespace sc {

constexpr int THREADS = 192;
constexpr uint32_t BOX = 128 * 128;      // 128 rows x 32 fp32 (128 B): 16 KB
constexpr int STAGES = 3;
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t IDESC = (1u << 4)          // D: f32
                           | (2u << 7)        // A: tf32
                           | (2u << 10)       // B: tf32
                           | ((128u >> 3) << 17) | ((128u >> 4) << 24);

struct Ctl {
  uint64_t a_full, a_empty;
  uint64_t b_full[STAGES], b_empty[STAGES];
  uint64_t s_full[2], s_empty[2];
  uint64_t drain;
  uint32_t tmem;
  int abort;
};

}  // namespace sc

__device__ inline void mma_tf32_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ inline float sc_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ inline float sc_lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <bool SUB>
__global__ void __launch_bounds__(sc::THREADS, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap mqh, const __grid_constant__ CUtensorMap mql,
                    const __grid_constant__ CUtensorMap mkh, const __grid_constant__ CUtensorMap mkl,
                    const ScoreArgs a) {
  using namespace sc;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Geom& g = a.g;
  const int DC = g.d / 32;                  // 32-dim slices
  uint8_t* sA = smem;                       // [hi, lo] x DC boxes
  uint8_t* sB = smem + 2 * DC * BOX;        // STAGES x [hi, lo]
  __shared__ Ctl ctl;
  volatile int* abort_flag = &ctl.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows = SUB ? g.nT * kSubBlocks : g.nT;   // pooled rows per head (query and key alike)
  const int nkc = (rows + 127) / 128;                 // 128-row blocks per head
  const long long units = (long long)g.BH * nkc * nkc;
  const long long u0 = units * blockIdx.x / gridDim.x, u1 = units * (blockIdx.x + 1) / gridDim.x;
  const long long cap = a.wait_cap;

  if (threadIdx.x == 0) {
    mbar_init(&ctl.a_full, 1);
    mbar_init(&ctl.a_empty, 1);
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&ctl.b_full[i], 1);
      mbar_init(&ctl.b_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl.s_full[i], 1);
      mbar_init(&ctl.s_empty[i], 128);
    }
    mbar_init(&ctl.drain, 1);
    ctl.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&ctl.tmem, TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = ctl.tmem;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA
    int step = 0, gq = 0;          // key slices issued, query-row groups loaded
    long long prev = -1;           // bh * nkc + query block of the loaded rows
    for (long long u = u0; u < u1; ++u) {
      const long long qg = u / nkc;
      const int j = (int)(u % nkc), bh = (int)(qg / nkc), rb = (int)(qg % nkc);
      if (qg != prev) {
        // the MMAs that read the previous query rows have completed
        if (gq >= 1 && !mbar_wait(&ctl.a_empty, (uint32_t)(gq - 1) & 1, abort_flag, a.status, cap))
          goto producer_done;
        mbar_arrive_expect_tx(&ctl.a_full, 2 * DC * BOX);
        for (int c = 0; c < DC; ++c) {
          tma_load_3d(sA + c * BOX, &mqh, &ctl.a_full, c * 32, rb * 128, bh);
          tma_load_3d(sA + (DC + c) * BOX, &mql, &ctl.a_full, c * 32, rb * 128, bh);
        }
        ++gq;
        prev = qg;
      }
      for (int c = 0; c < DC; ++c, ++step) {
        const int st = step % STAGES;
        if (step >= STAGES &&
            !mbar_wait(&ctl.b_empty[st], (uint32_t)((step / STAGES) - 1) & 1, abort_flag, a.status, cap))
          goto producer_done;
        mbar_arrive_expect_tx(&ctl.b_full[st], 2 * BOX);
        tma_load_3d(sB + (2 * st) * BOX, &mkh, &ctl.b_full[st], c * 32, j * 128, bh);
        tma_load_3d(sB + (2 * st + 1) * BOX, &mkl, &ctl.b_full[st], c * 32, j * 128, bh);
      }
    }
  producer_done:
    // every copy issued has landed before the block exits
    if (gq > 0) mbar_drain(&ctl.a_full, (uint32_t)(gq - 1) & 1, a.status, cap);
    for (int st = 0; st < STAGES && st < step; ++st) {
      const int last = st + ((step - 1 - st) / STAGES) * STAGES;
      mbar_drain(&ctl.b_full[st], (uint32_t)(last / STAGES) & 1, a.status, cap);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA
    {
      const uint64_t ad0 = umma_desc_sw128(smem_u32(sA), 16, 1024);
      const uint64_t bd0 = umma_desc_sw128(smem_u32(sB), 16, 1024);
      int step = 0, k = 0, gq = 0;
      long long prev = -1;
      bool ok = true;
      for (long long u = u0; u < u1 && ok; ++u, ++k) {
        const long long qg = u / nkc;
        if (qg != prev) {
          // the MMAs issued so far read the previous query rows: release them on completion
          if (gq >= 1) mma_commit(&ctl.a_empty);
          if (!mbar_wait(&ctl.a_full, (uint32_t)gq & 1, abort_flag, a.status, cap)) break;
          ++gq;
          prev = qg;
        }
        const int b = k & 1;
        if (k >= 2 && !mbar_wait(&ctl.s_empty[b], (uint32_t)((k >> 1) - 1) & 1, abort_flag, a.status, cap)) break;
        const uint32_t tS = tbase + 128 * b;
        for (int c = 0; c < DC; ++c, ++step) {
          const int st = step % STAGES;
          if (!mbar_wait(&ctl.b_full[st], (uint32_t)(step / STAGES) & 1, abort_flag, a.status, cap)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // hi.hi + hi.lo + lo.hi over the 4 k-steps (8 dims each) of this slice
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
            for (int p = 0; p < 3; ++p) {
              const int pa = p == 2 ? 1 : 0, pb = p == 1 ? 1 : 0;
              const uint64_t ad = ad0 + (uint64_t)((((pa * DC + c) * BOX) + kk * 32) >> 4);
              const uint64_t bd = bd0 + (uint64_t)((((2 * st + pb) * BOX) + kk * 32) >> 4);
              mma_tf32_ss(tS, ad, bd, IDESC, (c == 0 && kk == 0 && p == 0) ? 0u : 1u);
            }
          }
          mma_commit(&ctl.b_empty[st]);
        }
        if (ok) mma_commit(&ctl.s_full[b]);
      }
      // every MMA issued has completed before TMEM is freed
      mma_commit(&ctl.drain);
      mbar_drain(&ctl.drain, 0, a.status, cap);
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int q4 = warp & 3;
    const int row = 32 * q4 + lane;
    const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
    const float sl2 = g.scale * 1.4426950408889634f;
    int k = 0;
    for (long long u = u0; u < u1; ++u, ++k) {
      const long long qg = u / nkc;
      const int j = (int)(u % nkc), bh = (int)(qg / nkc), rb = (int)(qg % nkc);
      const int grow = rb * 128 + row;
      float* srow = a.S + ((size_t)bh * rows + (grow < rows ? grow : 0)) * g.nT;
      const int b = k & 1;
      if (!mbar_wait(&ctl.s_full[b], (uint32_t)(k >> 1) & 1, abort_flag, a.status, cap)) break;
      tc_fence_after();
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t v[32];
        tmem_ld32(tbase + 128 * b + 32 * ch + lane_off, v);
        tmem_wait_ld();
        const int col0 = j * 128 + 32 * ch;
        if (SUB) {
          // four key tiles of 8 sub-block columns each; tiles past nT are padding
          if (grow < rows) {
            float t4[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              float m = -INFINITY;
#pragma unroll
              for (int i = 0; i < 8; ++i) m = fmaxf(m, __uint_as_float(v[8 * t + i]) * sl2);
              float z = 0.f;
#pragma unroll
              for (int i = 0; i < 8; ++i) z += sc_ex2(fmaf(__uint_as_float(v[8 * t + i]), sl2, -m));
              t4[t] = m + sc_lg2(z);
            }
            const int key_tile0 = col0 / kSubBlocks;
            if (key_tile0 + 4 <= g.nT && (g.nT & 3) == 0) {
              *reinterpret_cast<float4*>(srow + key_tile0) = make_float4(t4[0], t4[1], t4[2], t4[3]);
            } else {
#pragma unroll
              for (int t = 0; t < 4; ++t)
                if (key_tile0 + t < g.nT) srow[key_tile0 + t] = t4[t];
            }
          }
        } else if (grow < g.nT) {
          if (col0 + 32 <= g.nT && (g.nT & 3) == 0) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              *reinterpret_cast<float4*>(srow + col0 + 4 * i) =
                  make_float4(__uint_as_float(v[4 * i]) * g.scale, __uint_as_float(v[4 * i + 1]) * g.scale,
                              __uint_as_float(v[4 * i + 2]) * g.scale, __uint_as_float(v[4 * i + 3]) * g.scale);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (col0 + i < g.nT) srow[col0 + i] = __uint_as_float(v[i]) * g.scale;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&ctl.s_empty[b]);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, sc::TMEM_COLS);
  }
}

template <bool SUB>
static cudaError_t launch_scores_t(const CUtensorMap& mqh, const CUtensorMap& mql, const CUtensorMap& mkh,
                                   const CUtensorMap& mkl, const ScoreArgs& a, cudaStream_t s) {
  const int DC = a.g.d / 32;
  const size_t smem = 1024 + (size_t)(2 * DC + 2 * sc::STAGES) * sc::BOX;
  cudaError_t e =
      cudaFuncSetAttribute(score_tc_kernel<SUB>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int rows = SUB ? a.g.nT * kSubBlocks : a.g.nT;
  const long long nkc = (rows + 127) / 128;
  const long long units = (long long)a.g.BH * nkc * nkc;
  if (units <= 0) return cudaSuccess;
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)(units < sms ? units : sms);   // one CTA per SM (shared memory)
  score_tc_kernel<SUB><<<grid, sc::THREADS, smem, s>>>(mqh, mql, mkh, mkl, a);
  return cudaGetLastError();
}

cudaError_t launch_scores(const CUtensorMap& mqh, const CUtensorMap& mql, const CUtensorMap& mkh,
                          const CUtensorMap& mkl, const ScoreArgs& a, cudaStream_t s) {
  return launch_scores_t<false>(mqh, mql, mkh, mkl, a, s);
}

cudaError_t launch_scores_sub(const CUtensorMap& mqh, const CUtensorMap& mql, const CUtensorMap& mkh,
                              const CUtensorMap& mkl, const ScoreArgs& a, cudaStream_t s) {
  return launch_scores_t<true>(mqh, mql, mkh, mkl, a, s);
}

}  // namespace fvattn
