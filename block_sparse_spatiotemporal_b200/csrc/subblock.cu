// Hierarchical (sub-block) scoring ("DFSAttn" digest, section 2: a block is
// split into smaller sub-blocks, each is scored, and the fine scores are
// summed into the block's importance).
//
// Each 4x4x4 tile splits into the eight 2x2x2 sub-cubes of its grid
// coordinates.  Q and K are pooled per sub-cube (pool_sub_kernel); the
// tensor-core score kernel reduces every (query sub-block, key tile) group of
// 8 logits to T = log2 of its unnormalised softmax mass; subblock_agg_kernel
// normalises each query sub-block's row and averages the 8 query sub-blocks
// of a tile in the log domain:
//   log P[i, j] = log( (1/8) sum_a 2^(T[(i,a), j] - Z[(i,a)]) ),
//   Z[(i,a)]    = log2 sum_j 2^T[(i,a), j],
// so each row of P sums to one and the top-p selection runs unchanged on
// log P in place of the tile logits.
#include "fvattn_internal.cuh"

namespace fvattn {

__device__ inline float sb_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ inline float sb_lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ inline float sb_round_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

// Sub-cube (0..7) of a token at grid coordinates (t, h, w): raster order of
// the 2x2x2 cube inside its 4x4x4 tile.
__device__ inline int sub_of(int t, int h, int w) {
  return (((t & 3) >> 1) << 2) | (((h & 3) >> 1) << 1) | ((w & 3) >> 1);
}

// One block per (tile, head, tensor), 128 threads.  Warp w reads rows w,
// w + 4, ... of the tile (lanes over head dims) and adds each row into the
// running sum of its sub-cube; the four warps' partial sums are added in warp
// order (a fixed order); mean = sum / 8; stored as tf32 hi + lo parts,
// [BH][nT * 8][d] with a tile's eight sub-blocks adjacent.
template <typename T, int D>
__global__ void __launch_bounds__(128) pool_sub_kernel(Geom g, const T* __restrict__ q, const T* __restrict__ k,
                                                       int natural, const int* __restrict__ tile_cube,
                                                       const int* __restrict__ tile_tok, RopeArgs rope,
                                                       PooledOut po) {
  constexpr int DPL = D / 32;
  __shared__ float part[4][kSubBlocks][D];
  const int j = blockIdx.x, bh = blockIdx.y, which = blockIdx.z;
  const T* x = which == 0 ? q : k;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cube = tile_cube[j];
  float acc[kSubBlocks][DPL];
#pragma unroll
  for (int s = 0; s < kSubBlocks; ++s)
#pragma unroll
    for (int i = 0; i < DPL; ++i) acc[s][i] = 0.f;
  for (int r = warp; r < kTileTokens; r += 4) {
    const int n = natural ? cube_row_token(g, cube, r) : j * kTileTokens + r;
    const int nn = natural ? n : tile_tok[j * kTileTokens + r];     // natural index: grid coordinates
    const int t = nn / (g.Hg * g.W), h = (nn / g.W) % g.Hg, w = nn % g.W;
    const int sb = sub_of(t, h, w);
    const T* row = x + ((size_t)bh * g.N + n) * D + lane * DPL;
    float v[DPL];
    Vec<T, DPL>::load(row, v);
    if (rope.enabled) {
#pragma unroll
      for (int i = 0; i < DPL; i += 2) {
        const int dim = lane * DPL + i;
        float2 cs;
        if (dim < rope.dt) cs = rope.tab[t * (rope.dt / 2) + dim / 2];
        else if (dim < rope.dt + rope.dh) cs = rope.tab[g.T * (rope.dt / 2) + h * (rope.dh / 2) + (dim - rope.dt) / 2];
        else cs = rope.tab[g.T * (rope.dt / 2) + g.Hg * (rope.dh / 2) + w * (rope.dw / 2) + (dim - rope.dt - rope.dh) / 2];
        const float x0 = v[i], x1 = v[i + 1];
        v[i] = x0 * cs.x - x1 * cs.y;
        v[i + 1] = x0 * cs.y + x1 * cs.x;
      }
    }
#pragma unroll
    for (int s = 0; s < kSubBlocks; ++s)
      if (s == sb) {
#pragma unroll
        for (int i = 0; i < DPL; ++i) acc[s][i] += v[i];
      }
  }
#pragma unroll
  for (int s = 0; s < kSubBlocks; ++s)
#pragma unroll
    for (int i = 0; i < DPL; ++i) part[warp][s][lane * DPL + i] = acc[s][i];
  __syncthreads();
  float* hi = po.hi[which];
  float* lo = po.lo[which];
  for (int e = threadIdx.x; e < kSubBlocks * D; e += blockDim.x) {
    const int s = e / D, c = e % D;
    const float mean = (((part[0][s][c] + part[1][s][c]) + part[2][s][c]) + part[3][s][c]) * 0.125f;
    const float hv = sb_round_tf32(mean);
    const size_t at = (((size_t)bh * g.nT + j) * kSubBlocks + s) * D + c;
    hi[at] = hv;
    lo[at] = sb_round_tf32(mean - hv);
  }
}

// One warp per (head, query tile): T rows [(i, a), :] for a = 0..7 (base-2
// logs of the unnormalised key-tile masses); writes the tile log-probability
// row (natural log) into logp [BH][nT][nT].  Sums and maxima are warp-tree
// reductions in a fixed order.
__global__ void __launch_bounds__(256) subblock_agg_kernel(Geom g, const float* __restrict__ Tb,
                                                           float* __restrict__ logp) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long gi = (long long)blockIdx.x * 8 + warp;            // bh * nT + query tile
  if (gi >= (long long)g.BH * g.nT) return;
  const float* trow = Tb + (size_t)gi * kSubBlocks * g.nT;           // rows (i, 0..7), nT columns each
  float Z[kSubBlocks];
#pragma unroll
  for (int a = 0; a < kSubBlocks; ++a) {
    const float* t = trow + (size_t)a * g.nT;
    float m = -INFINITY;
    for (int j = lane; j < g.nT; j += 32) m = fmaxf(m, t[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float z = 0.f;
    for (int j = lane; j < g.nT; j += 32) z += sb_ex2(t[j] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    Z[a] = m + sb_lg2(z);
  }
  float* out = logp + (size_t)gi * g.nT;
  for (int j = lane; j < g.nT; j += 32) {
    float u[kSubBlocks];
    float m = -INFINITY;
#pragma unroll
    for (int a = 0; a < kSubBlocks; ++a) {
      u[a] = trow[(size_t)a * g.nT + j] - Z[a];
      m = fmaxf(m, u[a]);
    }
    float z = 0.f;
#pragma unroll
    for (int a = 0; a < kSubBlocks; ++a) z += sb_ex2(u[a] - m);
    out[j] = (m + sb_lg2(z) - 3.0f) * 0.6931471805599453f;          // log2(1/8) = -3; to natural log
  }
}

template <typename T, int D>
static cudaError_t launch_pool_sub_t(const Geom& g, const void* q, const void* k, int natural, const int* tile_cube,
                                     const int* tile_tok, const RopeArgs& rope, const PooledOut& po, cudaStream_t s) {
  dim3 grid(g.nT, g.BH, 2);
  pool_sub_kernel<T, D><<<grid, 128, 0, s>>>(g, (const T*)q, (const T*)k, natural, tile_cube, tile_tok, rope, po);
  return cudaGetLastError();
}

cudaError_t launch_pool_sub(const Geom& g, int dtype, const void* q, const void* k, int natural, const int* tile_cube,
                            const int* tile_tok, int rope_enabled, int dt, int dh, int dw, const float2* rope_tab,
                            const PooledOut& po, cudaStream_t s) {
  RopeArgs r{rope_enabled, dt, dh, dw, rope_tab};
  if (dtype == FVATTN_BF16) {
    if (g.d == 128) return launch_pool_sub_t<__nv_bfloat16, 128>(g, q, k, natural, tile_cube, tile_tok, r, po, s);
  } else {
    if (g.d == 128) return launch_pool_sub_t<float, 128>(g, q, k, natural, tile_cube, tile_tok, r, po, s);
    if (g.d == 64) return launch_pool_sub_t<float, 64>(g, q, k, natural, tile_cube, tile_tok, r, po, s);
    if (g.d == 32) return launch_pool_sub_t<float, 32>(g, q, k, natural, tile_cube, tile_tok, r, po, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_subblock_agg(const Geom& g, const float* Tb, float* logp, cudaStream_t s) {
  const long long rows = (long long)g.BH * g.nT;
  subblock_agg_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(g, Tb, logp);
  return cudaGetLastError();
}

}  // namespace fvattn
