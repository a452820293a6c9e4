// Slack-aware augmentation on one GPU ("FVAttn" digest, section 02: ranks off
// the critical path spend their spare time computing extra, somewhat
// important blocks that the selection cut).  Here the persistent fine
// stage's CTAs play the ranks: CTA c of G runs the work-list slots c, c + G,
// ..., so with the longest-first list its load (union entries) is known
// before the fine stage starts.  Every CTA below the largest load gets the
// difference spread over its items, and each item adds that many key tiles
// outside its union, best coarse logit first, to its rows with a list.  The
// fine stage then keeps the unaugmented work list, so the largest load, the
// critical path, does not grow.
#include "fvattn_internal.cuh"

namespace fvattn {

// One block: load of each CTA over its slots, the largest load, and each
// item's share of its CTA's slack (the first items in slot order take the
// remainder).  With measured busy times (ns, one per CTA, from a run of the
// same work list on the unaugmented lists) the slack is the CTA's idle time
// in entries at the run's mean time per entry, times fill_percent / 100:
// floor((max busy - busy) * total entries * fill / (100 * total busy)),
// exact in 128-bit integers.
__global__ void __launch_bounds__(1024) slack_kernel(const int* __restrict__ ucount, const int* __restrict__ worklist,
                                                     int n_items, int G, const long long* __restrict__ busy,
                                                     int fill_percent, int* __restrict__ extra) {
  __shared__ int top;
  __shared__ unsigned long long total_load, total_busy, top_busy;
  if (threadIdx.x == 0) {
    top = 0;
    total_load = total_busy = top_busy = 0ull;
  }
  __syncthreads();
  const int c = threadIdx.x;
  int load = 0, n = 0;
  long long b = 0;
  if (c < G) {
    for (int t = c; t < n_items; t += G, ++n) load += ucount[worklist[t]];
    atomicMax(&top, load);
    if (busy) {
      b = busy[c];
      atomicAdd(&total_load, (unsigned long long)load);
      atomicAdd(&total_busy, (unsigned long long)b);
      atomicMax(&top_busy, (unsigned long long)b);
    }
  }
  __syncthreads();
  if (c < G) {
    int slack = top - load;
    if (busy) {
      slack = 0;
      if (total_busy > 0) {
        const unsigned __int128 num =
            (unsigned __int128)(top_busy - (unsigned long long)b) * total_load * (unsigned)fill_percent;
        // at most the total entries: top_busy - b <= total_busy and fill <= 100
        slack = (int)(num / ((unsigned __int128)100 * total_busy));
      }
    }
    int u = 0;
    for (int t = c; t < n_items; t += G, ++u) extra[worklist[t]] = slack / n + (u < slack % n ? 1 : 0);
  }
}

constexpr int kAugWarps = 4;

// One warp per item: pick `extra` key tiles outside the item's union by the
// largest logit over its rows with a list (ties to the lower tile id), then
// write both rows' lists (base list plus the picks, ascending) to the output
// lists.  The base lists are read completely before anything is written, so
// the output may be the base lists themselves.
__global__ void __launch_bounds__(kAugWarps * 32)
    augment_kernel(Geom g, const float* __restrict__ S, const int* counts, const int* idx, int cap,
                   const int* __restrict__ extra, int* out_counts, int* out_idx, int out_cap, int* status) {
  extern __shared__ uint32_t bm[];   // per warp: union, picked, row 0, row 1 bitmaps
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int words = (g.nT + 31) / 32;
  uint32_t* uni = bm + warp * 4 * words;
  uint32_t* pick = uni + words;
  uint32_t* rowb = pick + words;     // [2][words]
  const long long item = (long long)blockIdx.x * kAugWarps + warp;
  if (item >= (long long)g.BH * g.P) return;
  const int bh = (int)(item / g.P), qd = (int)(item % g.P);
  for (int w = lane; w < 4 * words; w += 32) uni[w] = 0u;
  __syncwarp();
  bool live[2] = {false, false};
  for (int t = 0; t < 2; ++t) {
    const int r = 2 * qd + t;
    if (r >= g.nT) break;
    const size_t row = (size_t)bh * g.nT + r;
    int c = counts[row];
    if (c < 0 || c > g.nT) {
      if (lane == 0) set_status(status, kStatusBadBlock);
      c = c < 0 ? 0 : g.nT;
    }
    live[t] = c > 0;
    const int* list = idx + row * (size_t)cap;
    for (int e = lane; e < c; e += 32) {
      const int j = list[e];
      if (j < 0 || j >= g.nT) {
        set_status(status, kStatusBadBlock);
        continue;
      }
      atomicOr(&uni[j >> 5], 1u << (j & 31));
      atomicOr(&rowb[t * words + (j >> 5)], 1u << (j & 31));
    }
  }
  __syncwarp();
  int usize = 0;
  for (int w = lane; w < words; w += 32) usize += __popc(uni[w]);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) usize += __shfl_xor_sync(0xffffffffu, usize, o);
  int e = (live[0] || live[1]) ? extra[item] : 0;
  if (e > g.nT - usize) e = g.nT - usize;
  const float* S0 = S + ((size_t)bh * g.nT + 2 * qd) * g.nT;
  const float* S1 = S0 + g.nT;
  for (int round = 0; round < e; ++round) {
    float best = -INFINITY;
    int bj = g.nT;
    for (int j = lane; j < g.nT; j += 32) {
      const uint32_t bit = 1u << (j & 31);
      if ((uni[j >> 5] | pick[j >> 5]) & bit) continue;
      float sc = -INFINITY;
      if (live[0]) sc = S0[j];
      if (live[1]) sc = fmaxf(sc, S1[j]);
      if (sc > best || (sc == best && j < bj)) {
        best = sc;
        bj = j;
      }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
      if (ob > best || (ob == best && oj < bj)) {
        best = ob;
        bj = oj;
      }
    }
    if (lane == 0 && bj < g.nT) pick[bj >> 5] |= 1u << (bj & 31);
    __syncwarp();
  }
  for (int t = 0; t < 2; ++t) {
    const int r = 2 * qd + t;
    if (r >= g.nT) break;
    const size_t row = (size_t)bh * g.nT + r;
    int* out = out_idx + row * (size_t)out_cap;
    int n = 0;
    for (int w = 0; w < words; ++w) {
      const uint32_t bits = rowb[t * words + w] | (live[t] ? pick[w] : 0u);
      const int j = w * 32 + lane;
      const bool on = (bits >> lane) & 1u;
      const unsigned bal = __ballot_sync(0xffffffffu, on);
      if (on) out[n + __popc(bal & ((1u << lane) - 1u))] = j;
      n += __popc(bal);
    }
    if (lane == 0) out_counts[row] = n;   // a row without a list keeps none
  }
}

cudaError_t launch_augment(const Geom& g, const float* S, const int* counts, const int* idx, int cap,
                           const int* ucount, const int* worklist, int G, const long long* busy, int fill_percent,
                           int* extra, int* out_counts, int* out_idx, int out_cap, int* status, cudaStream_t s) {
  const int items = g.BH * g.P;
  slack_kernel<<<1, 1024, 0, s>>>(ucount, worklist, items, G, busy, fill_percent, extra);
  const int words = (g.nT + 31) / 32;
  const size_t smem = sizeof(uint32_t) * 4 * words * kAugWarps;
  augment_kernel<<<(items + kAugWarps - 1) / kAugWarps, kAugWarps * 32, smem, s>>>(g, S, counts, idx, cap, extra,
                                                                                    out_counts, out_idx, out_cap,
                                                                                    status);
  return cudaGetLastError();
}

}  // namespace fvattn
