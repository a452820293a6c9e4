// Fine stage for fp32 tensors ("VSA" digest, section 3: token-level attention
// inside the selected tiles).  fp32 operands would lose their precision on
// the tf32 tensor-core path, so this variant runs on the CUDA cores: one
// block per (batch*head, query tile), TPR = D/32 threads per query row each
// holding 32 dims of q and of the output accumulator, K/V tiles staged in
// shared memory, exact online softmax with expf.
#include "fvattn_internal.cuh"

namespace fvattn {

__device__ inline int row_token(const Geom& g, const int* tile_cube, int natural, int tile, int r) {
  return natural ? cube_row_token(g, tile_cube[tile], r) : tile * kTileTokens + r;
}

template <int D>
__global__ void __launch_bounds__(64 * (D / 32)) fine_f32_kernel(const FineF32Args a) {
  constexpr int TPR = D / 32;
  extern __shared__ float fsm[];
  float (*ks)[D] = reinterpret_cast<float (*)[D]>(fsm);
  float (*vs)[D] = reinterpret_cast<float (*)[D]>(fsm + kTileTokens * D);
  const Geom& g = a.g;
  const int i = blockIdx.x, bh = blockIdx.y;
  const int r = threadIdx.x / TPR, sub = threadIdx.x % TPR;
  const int tq = row_token(g, a.tile_cube, a.q_nat, i, r);
  float q[32], o[32];
  const float* qrow = a.q + ((size_t)bh * g.N + tq) * D + sub * 32;
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    q[c] = qrow[c];
    o[c] = 0.f;
  }
  const size_t row = (size_t)bh * g.nT + i;
  int cnt = a.counts[row];
  if (cnt < 0 || cnt > g.nT) {
    if (threadIdx.x == 0) set_status(a.status, kStatusBadBlock);
    cnt = cnt < 0 ? 0 : g.nT;
  }
  const int* list = a.idx + row * (size_t)a.cap;
  float m = -INFINITY, l = 0.f;
  for (int e = 0; e < cnt; ++e) {
    const int j = list[e];
    if (j < 0 || j >= g.nT) {
      if (threadIdx.x == 0) set_status(a.status, kStatusBadBlock);
      continue;
    }
    __syncthreads();
    for (int x = threadIdx.x; x < kTileTokens * D; x += blockDim.x) {
      const int rr = x / D, c = x % D;
      ks[rr][c] = a.k[((size_t)bh * g.N + row_token(g, a.tile_cube, a.k_nat, j, rr)) * D + c];
      vs[rr][c] = a.v[((size_t)bh * g.N + row_token(g, a.tile_cube, a.v_nat, j, rr)) * D + c];
    }
    __syncthreads();
    for (int c = 0; c < kTileTokens; ++c) {
      float s = 0.f;
#pragma unroll
      for (int x = 0; x < 32; ++x) s = fmaf(q[x], ks[c][sub * 32 + x], s);
#pragma unroll
      for (int off = 1; off < TPR; off <<= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
      s *= g.scale;
      const float m_new = fmaxf(m, s);
      const float corr = expf(m - m_new);
      const float p = expf(s - m_new);
      l = l * corr + p;
#pragma unroll
      for (int x = 0; x < 32; ++x) o[x] = fmaf(p, vs[c][sub * 32 + x], o[x] * corr);
      m = m_new;
    }
  }
  const int to = row_token(g, a.tile_cube, a.out_nat, i, r);
  float* orow = a.out + ((size_t)bh * g.N + to) * D + sub * 32;
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int x = 0; x < 32; ++x) orow[x] = o[x] * inv;
  if (sub == 0) a.lse[(size_t)bh * g.N + to] = l > 0.f ? m + logf(l) : -INFINITY;
}

cudaError_t launch_fine_f32(const FineF32Args& a, cudaStream_t s) {
  dim3 grid(a.g.nT, a.g.BH);
  const size_t smem = 2 * sizeof(float) * kTileTokens * (size_t)a.g.d;
  cudaError_t e = cudaSuccess;
  if (a.g.d == 64) {
    fine_f32_kernel<64><<<grid, 128, smem, s>>>(a);
  } else if (a.g.d == 128) {
    e = cudaFuncSetAttribute(fine_f32_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    fine_f32_kernel<128><<<grid, 256, smem, s>>>(a);
  } else if (a.g.d == 32) {
    fine_f32_kernel<32><<<grid, 64, smem, s>>>(a);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace fvattn
