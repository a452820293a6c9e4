// Attention prologue: the QKV projection with the 3D rotary encoding fused
// into its epilogue ("Causal-RoPE SP" digest, section 2.3: projection and
// rotary encoding as one kernel; section 2.2: a block that starts at frame s
// encodes local frame t at t + s).
//
// Y = X W^T is a dense bf16 contraction (M = B*N tokens, Nout = 3*H*128,
// K = C channels), so it runs on the tensor cores: a persistent kernel, one
// CTA per SM, TMA-fed tcgen05.mma accumulating in TMEM.  The epilogue reads
// the fp32 accumulators out of TMEM, adds the bias, rotates the Q and K pairs
// with a precomputed (cos, sin) table, rounds once to bf16 and stores each
// token's head slice straight to its row of q, k or v in the attention's
// [B, H, N, 128] layout (natural, or the tiled order of the block-sparse
// path), so no separate transpose, rotation or reorder pass follows.
//
// Tile shapes (variant):
//   0: 256 x 256 per CTA as two M=128 accumulators filling all 512 TMEM
//      columns; per 16-deep k step the CTA reads 8 KB of X and 8 KB of W
//      for 2 x 128 clk of MMA (64 B/clk from L2); the epilogue stalls the
//      MMA for its duration.
//   1: 128 x 256 per CTA, accumulators double-buffered (2 x 256 columns) so
//      the epilogue overlaps the next tile's MMAs; 96 B/clk from L2.
//   2, 3: the tiles of 0 and 1 with 32-channel stages (64-byte swizzle):
//      the same shared memory holds 7 or 9 stages instead of 3 or 4, so
//      more bytes are in flight while the MMAs drain the oldest stage.
//
// Roles (320 threads): warp 0 lane 0 issues the TMA loads, warp 1 lane 0 the
// MMAs, warps 2..9 run the epilogue (warp w reads TMEM lanes 32 (w % 4) ..).
#include "fvattn_internal.cuh"

namespace fvattn {
namespace qkv {

constexpr int BN = 256;                   // output columns per tile (two heads)
constexpr int THREADS = 320;
constexpr int EPI_THREADS = 256;
constexpr int TMEM_COLS = 512;
constexpr uint32_t IDESC = idesc_bf16_f32(128, BN, false, false);

// MA accumulators of 128 rows; BK channels per stage (one swizzle row of
// 2 * BK bytes); ACC_BUFS TMEM accumulator sets.
template <int V> struct Cfg;
template <> struct Cfg<0> {
  static constexpr int MA = 2, BK = 64, STAGES = 3, ACC_BUFS = 1;
};
template <> struct Cfg<1> {
  static constexpr int MA = 1, BK = 64, STAGES = 4, ACC_BUFS = 2;
};
template <> struct Cfg<2> {
  static constexpr int MA = 2, BK = 32, STAGES = 7, ACC_BUFS = 1;
};
template <> struct Cfg<3> {
  static constexpr int MA = 1, BK = 32, STAGES = 9, ACC_BUFS = 2;
};

template <int V> struct Sizes {
  static constexpr int MA = Cfg<V>::MA;
  static constexpr int BK = Cfg<V>::BK;
  static constexpr int BM = 128 * MA;
  static constexpr int ROW = BK * 2;                 // bytes per smem row = swizzle width
  static constexpr int A_BYTES = BM * ROW;
  static constexpr int B_BYTES = BN * ROW;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int SMEM = Cfg<V>::STAGES * STAGE + 1024;
  static_assert(SMEM + 512 <= 227 * 1024, "shared memory");
};

// K-major operand descriptor: 8-row atoms of 8 * ROW bytes.
template <int ROW>
__device__ inline uint64_t kmajor_desc(uint32_t start) {
  if constexpr (ROW == 128)
    return umma_desc_sw128(start, 16, 1024);
  else
    return umma_desc_sw64(start, 16, 512);
}

template <int STAGES>
struct Ctl {
  uint64_t full[STAGES], empty[STAGES];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

// Tiles are visited in bands of group_m row tiles, row tile fastest inside a
// band, so the CTAs resident at one time share their X rows and W rows in L2.
__device__ inline void tile_origin(const QkvArgs& a, int BM, int tile, int& m0, int& n0) {
  const int per = a.group_m * a.nt;
  const int g = tile / per, r = tile - g * per;
  const int mf = g * a.group_m;
  const int gm = min(a.group_m, a.mt - mf);
  m0 = (mf + r % gm) * BM;
  n0 = (r / gm) * BN;
}

__device__ inline uint32_t pack2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Rotate the 16 pairs of a 32-column chunk that starts at head dim j0.
__device__ inline void rope_chunk(float (&f)[32], const QkvArgs& a, int j0, int t, int h, int w) {
  const int offh = (a.dt >> 1) * a.T, offw = offh + (a.dh >> 1) * a.Hg;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int dim = j0 + 2 * i;
    int idx;
    if (dim < a.dt)
      idx = (dim >> 1) * a.T + t;
    else if (dim < a.dt + a.dh)
      idx = offh + ((dim - a.dt) >> 1) * a.Hg + h;
    else
      idx = offw + ((dim - a.dt - a.dh) >> 1) * a.W + w;
    const float2 cs = __ldg(a.rope_tab + idx);
    const float x0 = f[2 * i], x1 = f[2 * i + 1];
    f[2 * i] = fmaf(x0, cs.x, -x1 * cs.y);
    f[2 * i + 1] = fmaf(x0, cs.y, x1 * cs.x);
  }
}

template <int V>
__global__ void __launch_bounds__(THREADS, 1)
    qkv_rope_kernel(const __grid_constant__ CUtensorMap mx, const __grid_constant__ CUtensorMap mw,
                    const QkvArgs a) {
  using S = Sizes<V>;
  constexpr int MA = S::MA, BM = S::BM, BK = S::BK, STAGES = Cfg<V>::STAGES, ACC_BUFS = Cfg<V>::ACC_BUFS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ Ctl<STAGES> ctl_s;
  Ctl<STAGES>* ctl = &ctl_s;
  volatile int* abort_flag = &ctl->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long cap = a.wait_cap;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&ctl->full[i], 1);
      mbar_init(&ctl->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl->acc_full[i], 1);
      mbar_init(&ctl->acc_empty[i], EPI_THREADS);
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

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------------- TMA
    prefetch_tensormap(&mx);
    prefetch_tensormap(&mw);
    long long it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < a.n_tiles && ok; tile += gridDim.x) {
      int m0, n0;
      tile_origin(a, BM, tile, m0, n0);
      for (int kb = 0; kb < a.kblocks; ++kb, ++it) {
        const int s = (int)(it % STAGES);
        if (it >= STAGES &&
            !mbar_wait(&ctl->empty[s], (uint32_t)((it / STAGES) - 1) & 1, abort_flag, a.status, cap)) {
          ok = false;
          break;
        }
        uint8_t* st = smem + s * S::STAGE;
        mbar_arrive_expect_tx(&ctl->full[s], S::STAGE);
        tma_load_2d(st, &mx, &ctl->full[s], kb * BK, m0);
        tma_load_2d(st + S::A_BYTES, &mw, &ctl->full[s], kb * BK, n0);
      }
    }
    // every copy issued has landed before the block exits
    for (int i = 0; i < STAGES && i < it; ++i) {
      const long long last = i + ((it - 1 - i) / STAGES) * STAGES;
      mbar_drain(&ctl->full[i], (uint32_t)(last / STAGES) & 1, a.status, cap);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA
    long long it = 0;
    int tc = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < a.n_tiles && ok; tile += gridDim.x, ++tc) {
      const int ab = tc % ACC_BUFS, use = tc / ACC_BUFS;
      if (tc >= ACC_BUFS && !mbar_wait(&ctl->acc_empty[ab], (uint32_t)(use - 1) & 1, abort_flag, a.status, cap))
        break;
      tc_fence_after();
      const uint32_t tacc = tbase + (uint32_t)(ab * BN);
      for (int kb = 0; kb < a.kblocks; ++kb, ++it) {
        const int s = (int)(it % STAGES);
        if (!mbar_wait(&ctl->full[s], (uint32_t)(it / STAGES) & 1, abort_flag, a.status, cap)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + s * S::STAGE);
        const uint64_t bd = kmajor_desc<S::ROW>(sa + S::A_BYTES);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
#pragma unroll
          for (int m = 0; m < MA; ++m) {
            const uint64_t ad = kmajor_desc<S::ROW>(sa + m * (128 * S::ROW) + kk * 32);
            mma_ss(tacc + m * BN, ad, bd + ((kk * 32) >> 4), IDESC, (kb | kk) != 0 ? 1u : 0u);
          }
        }
        mma_commit(&ctl->empty[s]);
      }
      if (!ok) break;
      mma_commit(&ctl->acc_full[ab]);
    }
    // every MMA issued has completed before TMEM is freed
    mma_commit(&ctl->drain);
    mbar_drain(&ctl->drain, 0, a.status, cap);
  } else if (warp >= 2) {
    // ----------------------------------------------------------- epilogue
    const int e = warp - 2, q4 = warp & 3, half = e >> 2;
    const int lrow = q4 * 32 + lane;
    const int HD = a.H * 128, HgW = a.Hg * a.W;
    constexpr int CHUNKS = MA == 2 ? 8 : 4;
    int tc = 0;
    for (int tile = blockIdx.x; tile < a.n_tiles; tile += gridDim.x, ++tc) {
      const int ab = tc % ACC_BUFS, use = tc / ACC_BUFS;
      int m0, n0;
      tile_origin(a, BM, tile, m0, n0);
      const int row = (MA == 2 ? half * 128 : 0) + lrow;
      const int cbase = MA == 2 ? 0 : half * 128;    // first column of this thread's part
      const int m = m0 + row;
      const bool valid = m < a.M;
      int b = 0, p = 0, t = 0, hh = 0, ww = 0;
      if (valid) {
        b = m / a.N;
        const int n = m - b * a.N;
        t = n / HgW;
        hh = (n - t * HgW) / a.W;
        ww = n - t * HgW - hh * a.W;
        p = a.pos ? __ldg(a.pos + n) : n;
      }
      int nvalid = (a.Nout - (n0 + cbase) + 31) / 32;
      nvalid = nvalid < 0 ? 0 : (nvalid > CHUNKS ? CHUNKS : nvalid);
      if (!mbar_wait(&ctl->acc_full[ab], (uint32_t)use & 1, abort_flag, a.status, cap)) break;
      tc_fence_after();
      const uint32_t tcol =
          tbase + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(MA == 2 ? half * BN : ab * BN + half * 128);
      if (nvalid == 0) {
        tc_fence_before();
        mbar_arrive(&ctl->acc_empty[ab]);
        continue;
      }
#pragma unroll 1
      for (int c = 0; c < nvalid; ++c) {
        uint32_t r[32];
        tmem_ld32(tcol + c * 32, r);
        tmem_wait_ld();
        if (c == nvalid - 1) {
          // the accumulator is free once every thread holds its last chunk
          tc_fence_before();
          mbar_arrive(&ctl->acc_empty[ab]);
        }
        const int col = n0 + cbase + c * 32;
        const int which = col / HD;
        const int rem = col - which * HD;
        const int head = rem >> 7, j0 = rem & 127;
        float f[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(r[i]);
        if (a.bias) {
          const float4* bp = reinterpret_cast<const float4*>(a.bias + col);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 bv = __ldg(bp + i);
            f[4 * i] += bv.x;
            f[4 * i + 1] += bv.y;
            f[4 * i + 2] += bv.z;
            f[4 * i + 3] += bv.w;
          }
        }
        if (which < 2 && a.rope_tab) rope_chunk(f, a, j0, t, hh, ww);
        if (valid) {
          __nv_bfloat16* base = which == 0 ? a.out[0] : (which == 1 ? a.out[1] : a.out[2]);
          uint4* dst = reinterpret_cast<uint4*>(base + ((size_t)(b * a.H + head) * a.N + p) * 128 + j0);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(pack2(f[8 * i], f[8 * i + 1]), pack2(f[8 * i + 2], f[8 * i + 3]),
                                pack2(f[8 * i + 4], f[8 * i + 5]), pack2(f[8 * i + 6], f[8 * i + 7]));
        }
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, TMEM_COLS);
  }
}

// (cos, sin) of every rotation pair, pair-major so that the tokens of a warp
// (consecutive w) read consecutive entries: [dt/2][T] angles (t + t_offset)
// * theta_j, then [dh/2][Hg], then [dw/2][W]; theta_j = base^(-2j/d_axis).
__global__ void rope_pairs_kernel(Geom g, int dt, int dh, int dw, float base, int t_offset, float2* tab) {
  const int nt = (dt / 2) * g.T, nh = (dh / 2) * g.Hg, nw = (dw / 2) * g.W;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nt + nh + nw; i += gridDim.x * blockDim.x) {
    int pos, j, da;
    if (i < nt) {
      j = i / g.T;
      pos = i % g.T + t_offset;
      da = dt;
    } else if (i < nt + nh) {
      j = (i - nt) / g.Hg;
      pos = (i - nt) % g.Hg;
      da = dh;
    } else {
      j = (i - nt - nh) / g.W;
      pos = (i - nt - nh) % g.W;
      da = dw;
    }
    const double theta = pow((double)base, -2.0 * j / (double)da);
    double sn, cs;
    sincos((double)pos * theta, &sn, &cs);
    tab[i] = make_float2((float)cs, (float)sn);
  }
}

template <int V>
cudaError_t launch_v(const CUtensorMap& mx, const CUtensorMap& mw, QkvArgs a, int num_sms, cudaStream_t s) {
  using Sz = Sizes<V>;
  a.mt = (a.M + Sz::BM - 1) / Sz::BM;
  a.nt = (a.Nout + BN - 1) / BN;
  a.n_tiles = a.mt * a.nt;
  if (a.group_m < 1) a.group_m = 1;
  cudaError_t e = cudaFuncSetAttribute(qkv_rope_kernel<V>, cudaFuncAttributeMaxDynamicSharedMemorySize, Sz::SMEM);
  if (e != cudaSuccess) return e;
  const int grid = a.n_tiles < num_sms ? a.n_tiles : num_sms;
  if (grid <= 0) return cudaSuccess;
  qkv_rope_kernel<V><<<grid, THREADS, Sz::SMEM, s>>>(mx, mw, a);
  return cudaGetLastError();
}

}  // namespace qkv

QkvTma qkv_tma(int variant) {
  switch (variant) {
    case 1: return {qkv::Sizes<1>::BM, qkv::Sizes<1>::BK};
    case 2: return {qkv::Sizes<2>::BM, qkv::Sizes<2>::BK};
    case 3: return {qkv::Sizes<3>::BM, qkv::Sizes<3>::BK};
    default: return {qkv::Sizes<0>::BM, qkv::Sizes<0>::BK};
  }
}

cudaError_t launch_qkv(const CUtensorMap& mx, const CUtensorMap& mw, QkvArgs a, int variant, int num_sms,
                       cudaStream_t s) {
  switch (variant) {
    case 1: return qkv::launch_v<1>(mx, mw, a, num_sms, s);
    case 2: return qkv::launch_v<2>(mx, mw, a, num_sms, s);
    case 3: return qkv::launch_v<3>(mx, mw, a, num_sms, s);
    default: return qkv::launch_v<0>(mx, mw, a, num_sms, s);
  }
}

cudaError_t launch_rope_pairs(const Geom& g, int dt, int dh, int dw, float base, int t_offset, float2* tab,
                              cudaStream_t s) {
  const int total = (dt / 2) * g.T + (dh / 2) * g.Hg + (dw / 2) * g.W;
  qkv::rope_pairs_kernel<<<(total + 255) / 256, 256, 0, s>>>(g, dt, dh, dw, base, t_offset, tab);
  return cudaGetLastError();
}

}  // namespace fvattn
