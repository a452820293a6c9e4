// Token orders and the tile reorder ("VSA" digest, section 3: (4,4,4) cubes;
// "DFSAttn" digest, section 1: 3D Hilbert reordering before blocking).
//
// A tile is always one aligned 4x4x4 cube of the latent grid.  The order
// decides (a) the rank of each cube, i.e. its tile id, and (b) the order of
// the 64 tokens inside a tiled-layout tile.  Raster-cube: cubes in raster
// order over the tile grid, tokens in raster order inside the cube.  Hilbert:
// cubes and tokens by their index on the 3D Hilbert curve of the enclosing
// 2^k cube (Skilling's transposed-axes construction, "Programming the
// Hilbert curve", 2004); an aligned 4-cube covers 64 consecutive curve
// indices, so the cube rank is the rank of (index >> 6) and the in-tile
// rank is (index & 63).
#include "fvattn_internal.cuh"

namespace fvattn {

// Hilbert index of (x0, x1, x2) with coordinates below 2^bits, bits <= 12.
__device__ uint64_t hilbert_index3(uint32_t x0, uint32_t x1, uint32_t x2, int bits) {
  uint32_t X[3] = {x0, x1, x2};
  const uint32_t top = 1u << (bits - 1);
  // Undo the excess rotations, top bit first.
  for (uint32_t q = top; q > 1; q >>= 1) {
    const uint32_t low = q - 1;
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      if (X[i] & q) {
        X[0] ^= low;
      } else {
        const uint32_t t = (X[0] ^ X[i]) & low;
        X[0] ^= t;
        X[i] ^= t;
      }
    }
  }
  // Gray encode.
  X[1] ^= X[0];
  X[2] ^= X[1];
  uint32_t flip = 0;
  for (uint32_t q = top; q > 1; q >>= 1)
    if (X[2] & q) flip ^= q - 1;
  X[0] ^= flip;
  X[1] ^= flip;
  X[2] ^= flip;
  // Interleave: one bit of each axis per level, most significant first.
  uint64_t idx = 0;
  for (int b = bits - 1; b >= 0; --b) {
#pragma unroll
    for (int i = 0; i < 3; ++i) idx = (idx << 1) | ((X[i] >> b) & 1u);
  }
  return idx;
}

__host__ __device__ inline int hilbert_bits_for(const Geom& g) {
  int m = g.T > g.Hg ? g.T : g.Hg;
  m = m > g.W ? m : g.W;
  int b = 1;
  while ((1 << b) < m) ++b;
  return b;
}

// One block builds tile_cube[rank] and cube_rank[raster cube id].
__global__ void __launch_bounds__(1024) tile_table_kernel(Geom g, int* tile_cube, int* cube_rank) {
  extern __shared__ unsigned long long keys[];  // [nT]
  const int nT = g.nT;
  if (g.order == FVATTN_ORDER_RASTER_CUBE) {
    for (int c = threadIdx.x; c < nT; c += blockDim.x) {
      const int ct = c / (g.nh * g.nw), ch = (c / g.nw) % g.nh, cw = c % g.nw;
      tile_cube[c] = pack_cube(ct, ch, cw);
      cube_rank[c] = c;
    }
    return;
  }
  const int bits = hilbert_bits_for(g);
  for (int c = threadIdx.x; c < nT; c += blockDim.x) {
    const int ct = c / (g.nh * g.nw), ch = (c / g.nw) % g.nh, cw = c % g.nw;
    keys[c] = hilbert_index3(ct * 4, ch * 4, cw * 4, bits) >> 6;
  }
  __syncthreads();
  for (int c = threadIdx.x; c < nT; c += blockDim.x) {
    const unsigned long long kc = keys[c];
    int rank = 0;
    for (int o = 0; o < nT; ++o) rank += keys[o] < kc ? 1 : 0;   // keys are distinct
    const int ct = c / (g.nh * g.nw), ch = (c / g.nw) % g.nh, cw = c % g.nw;
    tile_cube[rank] = pack_cube(ct, ch, cw);
    cube_rank[c] = rank;
  }
}

// Tiled position of natural token n.
__device__ inline int tiled_position(const Geom& g, const int* cube_rank, int n, int bits) {
  const int t = n / (g.Hg * g.W), h = (n / g.W) % g.Hg, w = n % g.W;
  const int c = ((t >> 2) * g.nh + (h >> 2)) * g.nw + (w >> 2);
  int intra;
  if (g.order == FVATTN_ORDER_HILBERT)
    intra = (int)(hilbert_index3(t, h, w, bits) & 63u);
  else
    intra = ((t & 3) * 4 + (h & 3)) * 4 + (w & 3);
  return cube_rank[c] * kTileTokens + intra;
}

// y[pi(n)] = x[n] (inverse == 0) or y[n] = x[pi(n)] (inverse != 0) for every
// row of every (batch, head).  Each thread moves one VEC-byte word.
template <typename VEC>
__global__ void reorder_kernel(Geom g, const int* cube_rank, const char* __restrict__ x, char* __restrict__ y,
                               int row_bytes, int inverse) {
  const int words = row_bytes / (int)sizeof(VEC);
  const long long total = (long long)g.BH * g.N * words;
  const int bits = hilbert_bits_for(g);
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int wd = (int)(i % words);
    const long long row = i / words;
    const int n = (int)(row % g.N);
    const long long bh = row / g.N;
    const int p = tiled_position(g, cube_rank, n, bits);
    const long long src = inverse ? bh * g.N + p : row;
    const long long dst = inverse ? row : bh * g.N + p;
    reinterpret_cast<VEC*>(y + dst * row_bytes)[wd] = reinterpret_cast<const VEC*>(x + src * row_bytes)[wd];
  }
}

// tile_tok[tiled row] = natural token index.
__global__ void tile_token_kernel(Geom g, const int* cube_rank, int* tile_tok) {
  const int bits = hilbert_bits_for(g);
  for (int n = blockIdx.x * blockDim.x + threadIdx.x; n < g.N; n += gridDim.x * blockDim.x)
    tile_tok[tiled_position(g, cube_rank, n, bits)] = n;
}

// pos[n] = tiled row of natural token n.
__global__ void token_pos_kernel(Geom g, const int* cube_rank, int* pos) {
  const int bits = hilbert_bits_for(g);
  for (int n = blockIdx.x * blockDim.x + threadIdx.x; n < g.N; n += gridDim.x * blockDim.x)
    pos[n] = tiled_position(g, cube_rank, n, bits);
}

cudaError_t launch_token_pos(const Geom& g, const int* cube_rank, int* pos, cudaStream_t s) {
  token_pos_kernel<<<(g.N + 255) / 256, 256, 0, s>>>(g, cube_rank, pos);
  return cudaGetLastError();
}

cudaError_t launch_tile_token(const Geom& g, const int* cube_rank, int* tile_tok, cudaStream_t s) {
  tile_token_kernel<<<(g.N + 255) / 256, 256, 0, s>>>(g, cube_rank, tile_tok);
  return cudaGetLastError();
}

cudaError_t launch_tile_table(const Geom& g, int* tile_cube, int* cube_rank, cudaStream_t s) {
  const size_t smem = (size_t)g.nT * sizeof(unsigned long long);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(tile_table_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  tile_table_kernel<<<1, 1024, smem, s>>>(g, tile_cube, cube_rank);
  return cudaGetLastError();
}

cudaError_t launch_reorder(const Geom& g, const int* cube_rank, const void* x, void* y, int row_bytes,
                           int inverse, int num_sms, cudaStream_t s) {
  const int threads = 256;
  const int blocks = num_sms * 8;
  if (row_bytes % 16 == 0)
    reorder_kernel<uint4><<<blocks, threads, 0, s>>>(g, cube_rank, (const char*)x, (char*)y, row_bytes, inverse);
  else if (row_bytes % 8 == 0)
    reorder_kernel<uint2><<<blocks, threads, 0, s>>>(g, cube_rank, (const char*)x, (char*)y, row_bytes, inverse);
  else
    reorder_kernel<uint32_t><<<blocks, threads, 0, s>>>(g, cube_rank, (const char*)x, (char*)y, row_bytes,
                                                        inverse);
  return cudaGetLastError();
}

}  // namespace fvattn
