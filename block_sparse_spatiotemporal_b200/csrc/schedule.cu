// Fine-stage schedule: the single-GPU analogue of the "FVAttn" digest's
// runtime head-level load balancing (section 02), applied across the SMs of
// one GPU instead of across GPUs.
//
// A work item is four adjacent query tiles 4q .. 4q+3 of one (batch, head):
// two 128-row tensor-core streams, A = tiles (4q, 4q+1) and B = tiles
// (4q+2, 4q+3), that share every K/V tile the item loads.  The item walks
// the union of the four tiles' key lists; each entry records which of the
// four tiles selected it (the other tiles' rows are masked for it), which
// stream takes part in it, and each stream's last entry.  Items are ranked by
// union size, longest first (LPT), ties by item code, so the persistent fine
// kernel hands the heavy items out first and the light ones fill the tail.
#include "fvattn_internal.cuh"

namespace fvattn {

// Entry word of the union list.
//   bits  0-15  key tile id
//   bits 16-19  selected by tile 4q+0 .. 4q+3
//   bits 20-21  stream A / B takes part (a selecting tile, or the stream's
//               one forced step when none of its tiles selected anything)
//   bits 22-23  last entry of stream A / B in this item
// One warp per item.  Validates the lists: counts in [0, nT], ids in
// [0, nT) and strictly ascending; violations set kStatusBadBlock and the
// offending entries are dropped.
__global__ void __launch_bounds__(128) union_kernel(Geom g, const int* __restrict__ counts,
                                                    const int* __restrict__ idx, int cap, int* __restrict__ uni,
                                                    int* __restrict__ ucount, int* status) {
  extern __shared__ uint32_t bm[];  // per warp: 4 bitmaps of ceil(nT/32) words
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int words = (g.nT + 31) / 32;
  uint32_t* bmw = bm + warp * 4 * words;
  const long long item = (long long)blockIdx.x * 4 + warp;
  if (item >= (long long)g.BH * g.P) return;
  const int bh = (int)(item / g.P), qd = (int)(item % g.P);
  for (int w = lane; w < 4 * words; w += 32) bmw[w] = 0u;
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
  int n = 0, lastA = -1, lastB = -1;
  for (int w = 0; w < words; ++w) {
    const int j = w * 32 + lane;
    uint32_t sel = 0;
#pragma unroll
    for (int t = 0; t < kItemTiles; ++t) sel |= ((bmw[t * words + w] >> lane) & 1u) << t;
    const uint32_t part = ((sel & 3u) ? 1u : 0u) | ((sel & 12u) ? 2u : 0u);
    const unsigned bal = __ballot_sync(0xffffffffu, sel != 0u);
    const int pos = n + __popc(bal & ((1u << lane) - 1u));
    if (sel) out[pos] = j | (int)(sel << 16) | (int)(part << 20);
    const unsigned ba = __ballot_sync(0xffffffffu, (part & 1u) != 0u);
    const unsigned bb = __ballot_sync(0xffffffffu, (part & 2u) != 0u);
    if (ba) lastA = n + __popc(bal & ((2u << (31 - __clz(ba))) - 1u)) - 1;
    if (bb) lastB = n + __popc(bal & ((2u << (31 - __clz(bb))) - 1u)) - 1;
    n += __popc(bal);
  }
  __syncwarp();
  if (lane == 0) {
    if (n == 0) {  // no tile selected anything: one step, fully masked, for both streams
      out[0] = 0;
      n = 1;
    }
    if (lastA < 0) {  // stream A without a selection: it takes part in entry 0, masked
      out[0] |= 1 << 20;
      lastA = 0;
    }
    if (lastB < 0) {
      out[0] |= 1 << 21;
      lastB = 0;
    }
    out[lastA] |= 1 << 22;
    out[lastB] |= 1 << 23;
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
  const size_t smem = (size_t)4 * 4 * words * sizeof(uint32_t);
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
