// Fine-stage schedule: the single-GPU analogue of the "FVAttn" digest's
// runtime head-level load balancing (section 02), applied across the SMs of
// one GPU instead of across GPUs.
//
// A work item is two adjacent query tiles 2q, 2q+1 of one (batch, head): one
// 128-row tensor-core tile.  The item walks the union of the two tiles' key
// lists; each entry records which of the two tiles selected it (the other
// tile's rows are masked for it).  Items are ranked by union size, longest
// first (LPT), ties by item code, so the persistent fine kernel hands the
// heavy items out first and the light ones fill the tail.
#include "fvattn_internal.cuh"

namespace fvattn {

// Entry word of the union list.
//   bits  0-15  key tile id
//   bits 16-17  selected by tile 2q / 2q+1
//   bit     22  last entry of the item
// An item none of whose tiles selected anything gets one fully masked entry
// (its rows end with out = 0, lse = -inf).  One warp per item.  Validates
// the lists: counts in [0, nT], ids in [0, nT) and strictly ascending;
// violations set kStatusBadBlock and the offending entries are dropped.
__global__ void __launch_bounds__(128) union_kernel(Geom g, const int* __restrict__ counts,
                                                    const int* __restrict__ idx, int cap, int* __restrict__ uni,
                                                    int* __restrict__ ucount, int* status) {
  extern __shared__ uint32_t bm[];  // per warp: kItemTiles bitmaps of ceil(nT/32) words
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int words = (g.nT + 31) / 32;
  uint32_t* bmw = bm + warp * kItemTiles * words;
  const long long item = (long long)blockIdx.x * 4 + warp;
  if (item >= (long long)g.BH * g.P) return;
  const int bh = (int)(item / g.P), qd = (int)(item % g.P);
  for (int w = lane; w < kItemTiles * words; w += 32) bmw[w] = 0u;
  __syncwarp();
  for (int t = 0; t < kItemTiles; ++t) {
    const int tile = kItemTiles * qd + t;
    if (tile >= g.nT) break;
    const size_t row = (size_t)bh * g.nT + tile;
    int c = counts[row];
    if (c < 0 || c > g.nT) {
      if (lane == 0) set_status(status, kStatusBadBlock);
      c = c < 0 ? 0 : g.nT;
    }
    const int* list = idx + row * (size_t)cap;
    uint32_t* bmx = bmw + t * words;
    for (int e = lane; e < c; e += 32) {
      const int j = list[e];
      const bool ok = j >= 0 && j < g.nT && (e == 0 || list[e - 1] < j);
      if (!ok) {
        set_status(status, kStatusBadBlock);
        continue;
      }
      atomicOr(&bmx[j >> 5], 1u << (j & 31));
    }
  }
  __syncwarp();
  int* out = uni + item * (long long)g.nT;
  int n = 0;
  for (int w = 0; w < words; ++w) {
    const int j = w * 32 + lane;
    uint32_t sel = 0;
#pragma unroll
    for (int t = 0; t < kItemTiles; ++t) sel |= ((bmw[t * words + w] >> lane) & 1u) << t;
    const unsigned bal = __ballot_sync(0xffffffffu, sel != 0u);
    const int pos = n + __popc(bal & ((1u << lane) - 1u));
    if (sel) out[pos] = j | (int)(sel << 16);
    n += __popc(bal);
  }
  __syncwarp();
  if (lane == 0) {
    if (n == 0) {  // no tile selected anything: one fully masked step
      out[0] = 0;
      n = 1;
    }
    out[n - 1] |= 1 << 22;
    ucount[item] = n;
  }
}

// rank(e) = #{e' : key(e') > key(e)} + #{e' < e : key(e') == key(e)};
// worklist[rank(e)] = e.  The comparisons are split over segments of e'
// (grid y) whose partial counts are added into rank[] (integer adds, so the
// result does not depend on their order); a second kernel scatters.
constexpr int kRankSeg = 1024;

__global__ void __launch_bounds__(256) rank_partial_kernel(const int* __restrict__ key, int n, int* __restrict__ rank) {
  __shared__ int ks[kRankSeg];
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  const int s0 = blockIdx.y * kRankSeg;
  const int len = min(kRankSeg, n - s0);
  for (int i = threadIdx.x; i < len; i += blockDim.x) ks[i] = key[s0 + i];
  __syncthreads();
  if (e >= n) return;
  const int ke = key[e];
  int c = 0;
  for (int i = 0; i < len; ++i) {
    const int kk = ks[i];
    c += (kk > ke || (kk == ke && s0 + i < e)) ? 1 : 0;
  }
  if (c) atomicAdd(&rank[e], c);
}

__global__ void scatter_rank_kernel(const int* __restrict__ rank, int n, int* __restrict__ worklist) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e < n) worklist[rank[e]] = e;
}

cudaError_t launch_union(const Geom& g, const int* counts, const int* idx, int cap, int* uni, int* ucount, int* status,
                         cudaStream_t s) {
  const long long items = (long long)g.BH * g.P;
  const int words = (g.nT + 31) / 32;
  const size_t smem = (size_t)4 * kItemTiles * words * sizeof(uint32_t);
  union_kernel<<<(unsigned)((items + 3) / 4), 128, smem, s>>>(g, counts, idx, cap, uni, ucount, status);
  return cudaGetLastError();
}

cudaError_t launch_rank(const int* key, int n, int* rank, int* worklist, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(rank, 0, sizeof(int) * (size_t)n, s);
  if (e != cudaSuccess) return e;
  dim3 grid((n + 255) / 256, (n + kRankSeg - 1) / kRankSeg);
  rank_partial_kernel<<<grid, 256, 0, s>>>(key, n, rank);
  scatter_rank_kernel<<<(n + 255) / 256, 256, 0, s>>>(rank, n, worklist);
  return cudaGetLastError();
}

}  // namespace fvattn
