// Fine-stage schedule: the single-GPU analogue of the "FVAttn" digest's
// runtime head-level load balancing (section 02), applied across the SMs of
// one GPU instead of across GPUs.
//
// A work item is two adjacent query tiles 2q, 2q+1 of one (batch, head): one
// 128-row tensor-core tile.  The item walks the union of the two tiles' key
// lists; each entry records which of the two tiles selected it (the other
// tile's rows are masked for it).  Items are ranked by union size, longest
// first (LPT), ties by item code, so the persistent fine kernel hands the
// heavy items out first and the light ones fill the tail; the ranking is a
// counting sort on the cost (lpt_sort_kernel).
#include "fvattn_internal.cuh"

namespace fvattn {

// Entry word of the union list.
//   bits  0-15  key tile id
//   bits 16-17  selected by tile 2q / 2q+1
//   bit     22  last entry of the item
// An item none of whose tiles selected anything gets one fully masked entry
// (its rows end with out = 0, lse = -inf).  One warp per item (a grid of
// one item per warp keeps more loads in flight than a grid-stride loop over
// a grid sized to the SMs, which measured slower).  Validates the lists:
// counts in [0, nT], ids in [0, nT) and strictly ascending; violations set
// kStatusBadBlock and the offending entries are dropped.
constexpr int kUnionWarps = 4;   // items (warps) per block
__global__ void __launch_bounds__(kUnionWarps * 32) union_kernel(Geom g, const int* __restrict__ counts,
                                                                 const int* __restrict__ idx, int cap,
                                                                 int* __restrict__ uni, int* __restrict__ ucount,
                                                                 int* status) {
  extern __shared__ uint32_t bm[];  // per warp: kItemTiles bitmaps of ceil(nT/32) words
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int words = (g.nT + 31) / 32;
  uint32_t* bmw = bm + warp * kItemTiles * words;
  const long long item = (long long)blockIdx.x * kUnionWarps + warp;
  if (item < (long long)g.BH * g.P) {
    const int bh = (int)(item / g.P), qd = (int)(item % g.P);
    // lanes 0, 1 read the two tiles' counts together (a missing second tile counts 0)
    int c = 0;
    if (lane < kItemTiles) {
      const int tile = kItemTiles * qd + lane;
      if (tile < g.nT) {
        c = counts[(size_t)bh * g.nT + tile];
        if (c < 0 || c > g.nT) {
          set_status(status, kStatusBadBlock);
          c = c < 0 ? 0 : g.nT;
        }
      }
    }
    for (int w = lane; w < kItemTiles * words; w += 32) bmw[w] = 0u;
    const int c0 = __shfl_sync(0xffffffffu, c, 0), c1 = __shfl_sync(0xffffffffu, c, 1);
    const int* list0 = idx + ((size_t)bh * g.nT + kItemTiles * qd) * (size_t)cap;
    const int* list1 = list0 + cap;
    __syncwarp();
    // both lists, 32 entries of each per pass, every load of a pass issued before the checks
    const int cmax = c0 > c1 ? c0 : c1;
    for (int e0 = 0; e0 < cmax; e0 += 32) {
      const int e = e0 + lane;
      const bool in0 = e < c0, in1 = e < c1;
      const int j0 = in0 ? list0[e] : 0, j1 = in1 ? list1[e] : 0;
      const int p0 = in0 && e > 0 ? list0[e - 1] : -1, p1 = in1 && e > 0 ? list1[e - 1] : -1;
      if (in0) {
        if (j0 >= 0 && j0 < g.nT && p0 < j0)
          atomicOr(&bmw[j0 >> 5], 1u << (j0 & 31));
        else
          set_status(status, kStatusBadBlock);
      }
      if (in1) {
        if (j1 >= 0 && j1 < g.nT && p1 < j1)
          atomicOr(&bmw[words + (j1 >> 5)], 1u << (j1 & 31));
        else
          set_status(status, kStatusBadBlock);
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
}

// ---------------------------------------------------------------------------
// Quad items of the fine stage: query tiles 4u .. 4u+3 of one (batch, head),
// two halves of two tiles (A = 4u, 4u+1; B = 4u+2, 4u+3), each half one
// 128-row tensor-core tile.  The item walks the union of the four tiles'
// lists once; both halves share its K/V tiles.  Entries are ordered: key
// tiles selected by both halves, then by half A only, then by half B only
// (ascending within each group), so that each half is active on a prefix
// and, for B, a suffix of the item's steps (two entries per step) and idle
// elsewhere.
//   entry: bits 0-15 key tile id, bits 16-19 selected by tile 4u + i.
//   ucount[item] = entries, useg[item] = n_both | n_a << 16,
//   qcost[item] = active steps of A + active steps of B.
// One warp per item; lists are validated as in union_kernel.
// ---------------------------------------------------------------------------
__host__ __device__ inline void quad_steps(int n, int nb, int na, int* sa, int* sb) {
  const int steps = (n + 1) >> 1;
  *sa = (nb + na + 1) >> 1;
  const int pre = (nb + 1) >> 1;
  int b = pre;
  if (n - nb - na > 0) {
    const int start = (nb + na) >> 1;
    const int overlap = pre > start ? pre - start : 0;
    b += steps - start - overlap;
  }
  *sb = b;
}

__global__ void __launch_bounds__(128) quad_union_kernel(Geom g, int Qn, const int* __restrict__ counts,
                                                         const int* __restrict__ idx, int cap, int* __restrict__ uni,
                                                         int* __restrict__ ucount, int* __restrict__ useg,
                                                         int* __restrict__ qcost, int* status) {
  extern __shared__ uint32_t bm[];  // per warp: 4 bitmaps of ceil(nT/32) words
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int words = (g.nT + 31) / 32;
  uint32_t* bmw = bm + warp * 4 * words;
  const long long item = (long long)blockIdx.x * 4 + warp;
  if (item >= (long long)g.BH * Qn) return;
  const int bh = (int)(item / Qn), u = (int)(item % Qn);
  for (int w = lane; w < 4 * words; w += 32) bmw[w] = 0u;
  __syncwarp();
  for (int t = 0; t < 4; ++t) {
    const int tile = 4 * u + t;
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
  int n = 0, seg[3] = {0, 0, 0};
  for (int pass = 0; pass < 3; ++pass) {
    const int n0 = n;
    for (int w = 0; w < words; ++w) {
      const int j = w * 32 + lane;
      uint32_t sel = 0;
#pragma unroll
      for (int t = 0; t < 4; ++t) sel |= ((bmw[t * words + w] >> lane) & 1u) << t;
      const bool a = (sel & 3u) != 0u, b = (sel & 12u) != 0u;
      const bool take = pass == 0 ? (a && b) : pass == 1 ? (a && !b) : (b && !a);
      const unsigned bal = __ballot_sync(0xffffffffu, take);
      if (take) out[n + __popc(bal & ((1u << lane) - 1u))] = j | (int)(sel << 16);
      n += __popc(bal);
    }
    seg[pass] = n - n0;
  }
  if (lane == 0) {
    ucount[item] = n;
    useg[item] = seg[0] | (seg[1] << 16);
    int sa, sb;
    quad_steps(n, seg[0], seg[1], &sa, &sb);
    qcost[item] = sa + sb;
  }
}

// Longest-first work list by a counting sort on the cost: bins of equal
// cost in descending order, items inside a bin in ascending code.  Items
// are taken in groups of consecutive codes (one block per group; a group of
// whole heads keeps the CTAs that run together on a few heads' K/V, which
// then stay in L2).  A block splits its group into `segs` consecutive
// segments, one warp each: per-segment histograms, per-bin offsets of every
// segment (bins in descending cost, segments in order), then each warp
// places its segment's items 32 at a time in code order (ranks among equal
// costs from __match_any_sync): stable and deterministic.
__global__ void __launch_bounds__(1024) lpt_sort_kernel(const int* __restrict__ cost_all, int n_all, int group, int maxc,
                                                        int shift, int segs, int* __restrict__ worklist_all) {
  extern __shared__ int sort_smem[];
  int* hist = sort_smem;                         // [segs][maxc + 1]: counts, then running offsets
  int* base = sort_smem + segs * (maxc + 1);     // [maxc + 1]: items of larger cost
  const int first = blockIdx.x * group;
  const int n = min(group, n_all - first);
  const int* cost = cost_all + first;
  int* worklist = worklist_all + first;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bins = maxc + 1;
  const int seg = (n + segs - 1) / segs;
  for (int i = tid; i < segs * bins; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  constexpr int U = 8;   // costs a lane loads ahead (the loads of a batch overlap)
  if (warp < segs) {
    const int lo = warp * seg, hi = min(n, lo + seg);
    for (int i0 = lo; i0 < hi; i0 += 32 * U) {
      int cv[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = i0 + u * 32 + lane;
        cv[u] = i < hi ? min(max(cost[i], 0), maxc) >> shift : -1;
      }
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (cv[u] >= 0) atomicAdd(&hist[warp * bins + cv[u]], 1);
    }
  }
  __syncthreads();
  for (int c = tid; c < bins; c += blockDim.x) {
    int t = 0;
    for (int w = 0; w < segs; ++w) t += hist[w * bins + c];
    base[c] = t;
  }
  __syncthreads();
  if (warp == 0) {   // descending exclusive scan of the bin totals
    int run = 0;
    for (int c0 = maxc; c0 >= 0; c0 -= 32) {
      const int c = c0 - lane;
      const int v = c >= 0 ? base[c] : 0;
      int x = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (c >= 0) base[c] = run + x - v;
      run += __shfl_sync(0xffffffffu, x, 31);
    }
  }
  __syncthreads();
  for (int c = tid; c < bins; c += blockDim.x) {   // each segment's first position in each bin
    int off = base[c];
    for (int w = 0; w < segs; ++w) {
      const int h = hist[w * bins + c];
      hist[w * bins + c] = off;
      off += h;
    }
  }
  __syncthreads();
  if (warp < segs) {
    int* offs = hist + warp * bins;
    const int lo = warp * seg, hi = min(n, lo + seg);
    for (int b0 = lo; b0 < hi; b0 += 32 * U) {
      int cv[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = b0 + u * 32 + lane;
        cv[u] = i < hi ? min(max(cost[i], 0), maxc) >> shift : -1;
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = b0 + u * 32 + lane;
        const bool valid = i < hi;
        const int c = cv[u];
        const unsigned peers = __match_any_sync(0xffffffffu, c);
        const int rank = __popc(peers & ((1u << lane) - 1u));
        const int pos0 = valid ? offs[c] : 0;
        __syncwarp();
        if (valid) {
          worklist[pos0 + rank] = first + i;
          if ((peers >> lane) == 1u) offs[c] = pos0 + __popc(peers);   // the group's highest lane advances the bin
        }
        __syncwarp();
      }
    }
  }
}

// Segments per block such that the histograms fit in 200 KB of shared memory.
static int sort_segments(int group, int maxc, size_t* smem) {
  int segs = (group + 31) / 32;
  if (segs > 32) segs = 32;
  while (segs > 1 && (size_t)(segs + 1) * (maxc + 1) * sizeof(int) > 200 * 1024) --segs;
  *smem = (size_t)(segs + 1) * (maxc + 1) * sizeof(int);
  return segs;
}

static cudaError_t launch_sort(const int* cost, int n, int group, int maxc, int shift, int* worklist,
                               cudaStream_t s) {
  size_t smem = 0;
  const int segs = sort_segments(group, maxc, &smem);
  cudaError_t e = cudaFuncSetAttribute(lpt_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  lpt_sort_kernel<<<(n + group - 1) / group, 1024, smem, s>>>(cost, n, group, maxc, shift, segs, worklist);
  return cudaGetLastError();
}

cudaError_t launch_quad_schedule(const Geom& g, int Qn, const int* counts, const int* idx, int cap, int* uni,
                                 int* ucount, int* useg, int* qcost, int* worklist, int* status, cudaStream_t s) {
  const long long items = (long long)g.BH * Qn;
  if (items <= 0) return cudaSuccess;
  const int words = (g.nT + 31) / 32;
  quad_union_kernel<<<(unsigned)((items + 3) / 4), 128, (size_t)4 * 4 * words * sizeof(uint32_t), s>>>(
      g, Qn, counts, idx, cap, uni, ucount, useg, qcost, status);
  const int maxc = 2 * ((g.nT + 1) / 2) + 2;
  return launch_sort(qcost, (int)items, (int)items, maxc, 0, worklist, s);
}

cudaError_t launch_union(const Geom& g, const int* counts, const int* idx, int cap, int* uni, int* ucount, int* status,
                         cudaStream_t s) {
  const long long items = (long long)g.BH * g.P;
  if (items <= 0) return cudaSuccess;
  const int words = (g.nT + 31) / 32;
  const size_t smem = (size_t)kUnionWarps * kItemTiles * words * sizeof(uint32_t);
  union_kernel<<<(unsigned)((items + kUnionWarps - 1) / kUnionWarps), kUnionWarps * 32, smem, s>>>(
      g, counts, idx, cap, uni, ucount, status);
  return cudaGetLastError();
}

cudaError_t launch_rank(const int* key, int n, int max_key, int group, int shift, int* worklist, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  if (group <= 0 || group > n) group = n;
  return launch_sort(key, n, group, max_key, shift, worklist, s);
}

}  // namespace fvattn
