// Coarse stage: 3D RoPE on load, tile mean-pooling, row softmax of the
// pooled scores and top-p selection with a k_min floor.  The pooled score
// GEMM itself runs on the tensor cores (scores_tc.cu).
//
//   "VSA" digest, section 3: the coarse stage pools each (4,4,4) cube and
//     predicts per-tile importance;
//   "FVAttn" digest, sections 00 and 02: top-p routing with a top-k floor;
//   "Causal-RoPE SP" digest, sections 2.2-2.3: 3D rotary encoding with a
//     precomputed frequency table, fused into the load.
//
// Selection rule (per query-tile row of the coarse softmax P): m is the
// fewest tiles, at least one, whose probabilities summed in descending order
// (ties to the lower tile id) reach top_p; count = min(nT, max(m, k_min));
// top_p >= 1 keeps every tile.  The kernel never sorts the row (see
// select_row), computes every mass as a deterministic warp-tree sum, and
// compares masses against top_p * Z instead of dividing.
#include "fvattn_internal.cuh"

namespace fvattn {

// --------------------------------------------------------------------------
// RoPE table: (cos, sin) of pos * base^(-2j/da) for every axis position and
// pair, computed in double and rounded to float once per call.
// --------------------------------------------------------------------------
__global__ void rope_table_kernel(Geom g, int dt, int dh, int dw, float base, float2* tab) {
  const int nt = g.T * (dt / 2), nh = g.Hg * (dh / 2), nw = g.W * (dw / 2);
  const int total = nt + nh + nw;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    int pos, j, da;
    if (i < nt) {
      pos = i / (dt / 2); j = i % (dt / 2); da = dt;
    } else if (i < nt + nh) {
      pos = (i - nt) / (dh / 2); j = (i - nt) % (dh / 2); da = dh;
    } else {
      pos = (i - nt - nh) / (dw / 2); j = (i - nt - nh) % (dw / 2); da = dw;
    }
    const double theta = pow((double)base, -2.0 * j / (double)da);
    double sn, cs;
    sincos((double)pos * theta, &sn, &cs);
    tab[i] = make_float2((float)cs, (float)sn);
  }
}

// Rotate the pair (a, b) = dims (dim, dim+1) of a token at (t, h, w).
__device__ inline void rope_pair(const RopeArgs& r, const Geom& g, int dim, int t, int h, int w, float& a,
                                 float& b) {
  float2 cs;
  if (dim < r.dt) {
    cs = r.tab[t * (r.dt / 2) + dim / 2];
  } else if (dim < r.dt + r.dh) {
    cs = r.tab[g.T * (r.dt / 2) + h * (r.dh / 2) + (dim - r.dt) / 2];
  } else {
    cs = r.tab[g.T * (r.dt / 2) + g.Hg * (r.dh / 2) + w * (r.dw / 2) + (dim - r.dt - r.dh) / 2];
  }
  // each product and the sum / difference rounded to float32 on its own (no
  // fused multiply-add), so the values rounded to the operand dtype are
  // reproducible: the oracle evaluates the same expression in float32
  const float x0 = a, x1 = b;
  a = __fsub_rn(__fmul_rn(x0, cs.x), __fmul_rn(x1, cs.y));
  b = __fadd_rn(__fmul_rn(x0, cs.y), __fmul_rn(x1, cs.x));
}

// --------------------------------------------------------------------------
// Pool: one block per (tile, head, tensor).  4 warps; every lane loads 16
// bytes (8 bf16 or 4 fp32 dims) of a token row per load, so a warp load
// covers one or more whole rows; a lane's loads for the whole tile are
// issued before any of them is summed.  Sums are fp32 in a fixed order:
// a lane's rows in sequence, then the lanes of a warp that hold the same
// dims (butterfly), then the 4 warp partials in warp order; mean = sum / 64.
// The mean is stored as two tf32 values, hi = rn_tf32(mean) and
// lo = rn_tf32(mean - hi) (the subtraction is exact), row-major [BH][nT][d],
// the operands of the tensor-core score kernel.  Optionally writes the
// rotated rows, rounded to T, at tiled positions.
// --------------------------------------------------------------------------
__device__ inline float round_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

template <typename T, int D>
__global__ void __launch_bounds__(128) pool_kernel(Geom g, const T* __restrict__ q, const T* __restrict__ k,
                                                   int natural, const int* __restrict__ tile_cube,
                                                   const int* __restrict__ tile_tok, RopeArgs rope, PooledOut po,
                                                   T* __restrict__ qrot, T* __restrict__ krot) {
  constexpr int DPL = 16 / sizeof(T);        // elements per 128-bit load
  constexpr int LPR = D / DPL;               // lanes per token row
  constexpr int RPL = 32 / LPR;              // rows per warp load
  constexpr int ITER = kTileTokens / (4 * RPL);
  __shared__ float part[4][D];
  const int j = blockIdx.x, bh = blockIdx.y, which = blockIdx.z;
  const T* x = which == 0 ? q : k;
  float* hi = po.hi[which];
  float* lo = po.lo[which];
  T* rot = which == 0 ? qrot : krot;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane / LPR, col = (lane % LPR) * DPL;
  const int cube = tile_cube[j];
  float acc[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) acc[i] = 0.f;
  // warp w, iteration it: rows (it * 4 + w) * RPL + sub; all ITER loads of a lane issued before the sums
  float v[ITER][DPL];
#pragma unroll
  for (int it = 0; it < ITER; ++it) {
    const int r = (it * 4 + warp) * RPL + sub;
    const int n = natural ? cube_row_token(g, cube, r) : j * kTileTokens + r;
    Vec<T, DPL>::load(x + ((size_t)bh * g.N + n) * D + col, v[it]);
  }
#pragma unroll
  for (int it = 0; it < ITER; ++it) {
    const int r = (it * 4 + warp) * RPL + sub;
    if (rope.enabled) {
      // grid coordinate of the token in this row (tiled rows follow the order)
      const int n = natural ? cube_row_token(g, cube, r) : j * kTileTokens + r;
      const int nn = natural ? n : tile_tok[j * kTileTokens + r];
      const int t = nn / (g.Hg * g.W), h = (nn / g.W) % g.Hg, w = nn % g.W;
#pragma unroll
      for (int i = 0; i < DPL; i += 2) rope_pair(rope, g, col + i, t, h, w, v[it][i], v[it][i + 1]);
    }
#pragma unroll
    for (int i = 0; i < DPL; ++i) acc[i] += v[it][i];
    if (rot) {
      // Q: at the position it was read from (the caller's output buffer, whose
      // rows of this tile the fine stage overwrites only after reading them);
      // K: tiled, the layout the fine stage streams key tiles in
      const int n = which == 0 && natural ? cube_row_token(g, cube, r) : j * kTileTokens + r;
      T* dst = rot + ((size_t)bh * g.N + n) * D + col;
      Vec<T, DPL>::store(dst, v[it]);
    }
  }
  if (!hi) return;
  // lanes holding the same dims (one per row of a warp load) combine in a fixed order
#pragma unroll
  for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
    for (int i = 0; i < DPL; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
  if (sub == 0) {
#pragma unroll
    for (int i = 0; i < DPL; ++i) part[warp][col + i] = acc[i];
  }
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    const float mean = (((part[0][c] + part[1][c]) + part[2][c]) + part[3][c]) * (1.0f / 64.0f);
    const float h = round_tf32(mean);
    const size_t at = ((size_t)bh * g.nT + j) * D + c;
    hi[at] = h;
    lo[at] = round_tf32(mean - h);
  }
}

// --------------------------------------------------------------------------
// Selection, one warp per query-tile row of S = scale * Qp Kp^T.
//
// Tiles are ranked by their logit (the probability order; exp(s - max)
// underflows to 0 for distant tiles, the logit does not), descending, ties
// to the lower tile id.  A row's logits sit in registers, lane-strided
// (element i of a lane is tile 32 i + lane).  Most rows are settled by a few
// argmax rounds that pick tiles in rank order and add their probabilities in
// that order until the cut and the k_min floor are both reached.  Rows whose
// cut lies deeper search the 32-bit order-preserving keys of the logits for
// the largest key u whose suffix mass sum_{key >= u} e reaches top_p * Z
// (warp-tree sums): a bisection of its 16 high bits, then the few keys that
// share them in descending order; ties at u are taken lowest id first.
// --------------------------------------------------------------------------
__device__ inline float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ inline float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ inline int warp_isum(int v) { return __reduce_add_sync(0xffffffffu, v); }

// Unsigned key with the order of the float (no NaNs expected).
__device__ inline uint32_t order_key(float v) {
  const uint32_t b = __float_as_uint(v);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

constexpr int kSelWarps = 8;     // rows (warps) per selection block
// Argmax rounds before falling back to bisection: a round costs about as
// much as four bisection steps, so rows whose cut (or k_min floor) lies
// deeper than this are cheaper to bisect.
#ifndef FVATTN_SEL_ROUNDS
#define FVATTN_SEL_ROUNDS 8
#endif
constexpr int kMaxRounds = FVATTN_SEL_ROUNDS;
constexpr int kCutRounds = 8;    // distinct keys below the bisected 16-bit prefix taken one by one

// Selection of one row: src holds the row's nT logits.  Each lane keeps its
// tiles' order keys in registers (a tile past nT has key 0, below every
// logit's key) and the numerators e_j = exp(s_j - max) in the warp's shared
// scratch row srow; up to 24 values a lane also keeps e_j in registers for
// the bisection (beyond that the registers would spill).
template <int MAXV>
__device__ void select_row(const float* __restrict__ src, float* srow, int nT, float top_p, int k_min,
                           int* count_out, int* list) {
  constexpr int NW = (MAXV + 31) / 32;
  constexpr bool kEReg = MAXV <= 24;
  const int lane = threadIdx.x & 31;
  uint32_t kv[MAXV];
  float e[kEReg ? MAXV : 1];
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int j = i * 32 + lane;
    const float x = j < nT ? __ldcs(src + j) : -INFINITY;
    kv[i] = __float_as_uint(x);
    mx = fmaxf(mx, x);
  }
  mx = warp_max(mx);
  float zp = 0.f;
  const float mx2 = mx * 1.4426950408889634f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int j = i * 32 + lane;
    const float s = __uint_as_float(kv[i]);
    kv[i] = j < nT ? order_key(s) : 0u;
    float x = 0.f;
    if (j < nT) {
      asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(x) : "f"(fmaf(s, 1.4426950408889634f, -mx2)));
      srow[j] = x;
      zp += x;
    }
    if constexpr (kEReg) e[i] = x;
  }
  // e_j of this lane's element i (only read for a tile below nT)
  auto ev = [&](int i) -> float {
    if constexpr (kEReg) return e[i];
    else return srow[i * 32 + lane];
  };
  const float Z = warp_sum(zp);
  __syncwarp();

  if (top_p >= 1.0f) {
    for (int j = lane; j < nT; j += 32) list[j] = j;
    if (lane == 0) *count_out = nT;
    return;
  }
  const float target = top_p * Z;
  const int floor_k = k_min > 1 ? k_min : 1;

  // ---- argmax rounds
  uint32_t tk[NW];
#pragma unroll
  for (int w = 0; w < NW; ++w) tk[w] = 0u;
  int m = top_p > 0.f ? 0 : 1;
  int count = m ? (floor_k < nT ? floor_k : nT) : -1;
  int picks = 0;
  float cum = 0.f;
  const int rounds = (floor_k > kMaxRounds) ? 0 : (nT < kMaxRounds ? nT : kMaxRounds);
  for (int r = 0; r < rounds; ++r) {
    if (count >= 0 && picks >= count) break;
    uint32_t bk = 0u;
    int bj = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const bool free_i = !((tk[i >> 5] >> (i & 31)) & 1u);
      if (free_i && kv[i] > bk) {
        bk = kv[i];
        bj = i * 32 + lane;
      }
    }
    // warp argmax in two single-instruction reductions: the largest key, then
    // the lowest id holding it (a lane's own ties already went to its lowest id)
    {
      const uint32_t kmx = __reduce_max_sync(0xffffffffu, bk);
      bj = (int)__reduce_min_sync(0xffffffffu, bk == kmx ? (uint32_t)bj : 0x7fffffffu);
    }
    if (bj == 0x7fffffff) break;
    if ((bj & 31) == lane) {
      const int i = bj >> 5;
#pragma unroll
      for (int w = 0; w < NW; ++w)
        if (w == (i >> 5)) tk[w] |= 1u << (i & 31);
    }
    cum += srow[bj];
    ++picks;
    if (m == 0 && cum >= target) m = picks;
    if (m > 0 && count < 0) {
      count = m > floor_k ? m : floor_k;
      if (count > nT) count = nT;
    }
  }

  int* out = list;
  if (count >= 0 && picks >= count) {
    int base = 0;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const bool sel = (tk[i >> 5] >> (i & 31)) & 1u;
      const unsigned b = __ballot_sync(0xffffffffu, sel);
      if (sel) out[base + __popc(b & ((1u << lane) - 1u))] = i * 32 + lane;
      base += __popc(b);
    }
    if (lane == 0) *count_out = count;
    return;
  }

  // ---- bisection over the keys
  uint32_t uT = 0;
  int take = 0;
  if (m == 0) {
    // the cut key u: the largest key whose suffix mass reaches the target.
    // Its 16 high bits (sign, exponent, 7 mantissa bits) by bisection over
    // every value ...
    uint32_t u = 0;
    for (int b = 31; b >= 16; --b) {
      const uint32_t cand = u | (1u << b);
      float part = 0.f;
#pragma unroll
      for (int i = 0; i < MAXV; ++i) part += kv[i] >= cand ? ev(i) : 0.f;
      if (warp_sum(part) >= target) u = cand;
    }
    // ... the rest from the few values sharing them: their distinct keys in
    // descending order, each adding its values' mass to the mass above the
    // prefix, until the target is reached (a bisection of the low bits over
    // every value if that takes more than kCutRounds keys)
    const uint32_t pre = u >> 16;
    float above = 0.f;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) above += (kv[i] >> 16) > pre ? ev(i) : 0.f;
    const float m_above = warp_sum(above);
    float acc = 0.f;
    uint32_t ub = 0xffffffffu;           // keys already added are >= ub
    bool found = false;
    for (int rr = 0; rr < kCutRounds && !found; ++rr) {
      uint32_t bk = 0u;
#pragma unroll
      for (int i = 0; i < MAXV; ++i)
        if ((kv[i] >> 16) == pre && kv[i] < ub && kv[i] > bk) bk = kv[i];
      const uint32_t kmx = __reduce_max_sync(0xffffffffu, bk);
      if (kmx == 0u) break;
      float grp = 0.f;
#pragma unroll
      for (int i = 0; i < MAXV; ++i) grp += kv[i] == kmx ? ev(i) : 0.f;
      acc += warp_sum(grp);
      if (m_above + acc >= target) {
        u = kmx;
        found = true;
      }
      ub = kmx;
    }
    if (!found) {
      for (int b = 15; b >= 0; --b) {
        const uint32_t cand = u | (1u << b);
        float part = 0.f;
#pragma unroll
        for (int i = 0; i < MAXV; ++i) part += kv[i] >= cand ? ev(i) : 0.f;
        if (warp_sum(part) >= target) u = cand;
      }
    }
    float gpart = 0.f;
    int cgt = 0, ceq = 0;
    float eu = 0.f;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      if (kv[i] > u) {
        gpart += ev(i);
        ++cgt;
      } else if (kv[i] == u) {
        ++ceq;
        eu = ev(i);
      }
    }
    const float mgt = warp_sum(gpart);
    cgt = warp_isum(cgt);
    ceq = warp_isum(ceq);
    eu = warp_max(eu);
    int r_ties = 0;
    if (ceq > 0) {
      float accm = mgt + eu;
      r_ties = 1;
      while (r_ties < ceq && accm < target) {
        accm += eu;
        ++r_ties;
      }
    }
    m = cgt + r_ties;
    if (m < 1) m = 1;
    count = m > floor_k ? m : floor_k;
    if (count > nT) count = nT;
    if (count == m) {
      uT = u;
      take = r_ties;
    }
  }
  if (take == 0 && !(count == m && m > 0 && uT != 0)) {
    // top-`count` set: largest key u2 with #{key >= u2} >= count
    uint32_t u2 = 0;
    for (int b = 31; b >= 0; --b) {
      const uint32_t cand = u2 | (1u << b);
      int c = 0;
#pragma unroll
      for (int i = 0; i < MAXV; ++i) c += kv[i] >= cand ? 1 : 0;
      if (warp_isum(c) >= count) u2 = cand;
    }
    int cgt = 0;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) cgt += kv[i] > u2 ? 1 : 0;
    cgt = warp_isum(cgt);
    uT = u2;
    take = count - cgt;
  }
  int base = 0, tie_base = 0;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int j = i * 32 + lane;
    const bool valid = j < nT;
    const bool tie = valid && kv[i] == uT;
    const unsigned tmask = __ballot_sync(0xffffffffu, tie);
    const int trank = tie_base + __popc(tmask & ((1u << lane) - 1u));
    const bool sel = valid && (kv[i] > uT || (tie && trank < take));
    const unsigned smask = __ballot_sync(0xffffffffu, sel);
    const int pos = base + __popc(smask & ((1u << lane) - 1u));
    if (sel && pos < count) out[pos] = j;
    base += __popc(smask);
    tie_base += __popc(tmask);
  }
  if (lane == 0) *count_out = count;
}

template <int MAXV>
__global__ void __launch_bounds__(kSelWarps * 32, MAXV <= 24 ? 3 : (MAXV <= 40 ? 2 : 1)) select_rows_kernel(Geom g, const float* __restrict__ S,
                                                                    float top_p, int k_min, int* __restrict__ counts,
                                                                    int* __restrict__ idx, int cap, int stride) {
  extern __shared__ __align__(16) float sm[];
  const int warp = threadIdx.x >> 5;
  const long long row = (long long)blockIdx.x * kSelWarps + warp;   // bh * nT + query tile
  if (row >= (long long)g.BH * g.nT) return;
  select_row<MAXV>(S + (size_t)row * g.nT, sm + (size_t)warp * stride, g.nT, top_p, k_min, counts + row,
                   idx + (size_t)row * (size_t)cap);
}

template <typename T, int D>
static cudaError_t launch_pool_t(const Geom& g, const void* q, const void* k, int natural, const int* tile_cube,
                                 const int* tile_tok, const RopeArgs& rope, const PooledOut& po, void* qrot,
                                 void* krot, cudaStream_t s) {
  dim3 grid(g.nT, g.BH, 2);
  pool_kernel<T, D><<<grid, 128, 0, s>>>(g, (const T*)q, (const T*)k, natural, tile_cube, tile_tok, rope, po,
                                         (T*)qrot, (T*)krot);
  return cudaGetLastError();
}

cudaError_t launch_pool(const Geom& g, int dtype, const void* q, const void* k, int natural, const int* tile_cube,
                        const int* tile_tok, int rope_enabled, int dt, int dh, int dw, const float2* rope_tab,
                        const PooledOut& po, void* qrot, void* krot, cudaStream_t s) {
  RopeArgs r{rope_enabled, dt, dh, dw, rope_tab};
  if (dtype == FVATTN_BF16) {
    if (g.d == 128) return launch_pool_t<__nv_bfloat16, 128>(g, q, k, natural, tile_cube, tile_tok, r, po, qrot, krot, s);
    if (g.d == 64) return launch_pool_t<__nv_bfloat16, 64>(g, q, k, natural, tile_cube, tile_tok, r, po, qrot, krot, s);
  } else {
    if (g.d == 128) return launch_pool_t<float, 128>(g, q, k, natural, tile_cube, tile_tok, r, po, qrot, krot, s);
    if (g.d == 64) return launch_pool_t<float, 64>(g, q, k, natural, tile_cube, tile_tok, r, po, qrot, krot, s);
    if (g.d == 32) return launch_pool_t<float, 32>(g, q, k, natural, tile_cube, tile_tok, r, po, qrot, krot, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_rope_table(const Geom& g, int dt, int dh, int dw, float base, float2* tab, cudaStream_t s) {
  const int total = g.T * (dt / 2) + g.Hg * (dh / 2) + g.W * (dw / 2);
  rope_table_kernel<<<(total + 255) / 256, 256, 0, s>>>(g, dt, dh, dw, base, tab);
  return cudaGetLastError();
}

// Shared scratch row stride: nT rounded up to 4 floats.
static int select_stride(int nT) { return (nT + 3) & ~3; }

template <int MAXV>
static cudaError_t launch_select_v(const Geom& g, const float* S, float top_p, int k_min, int* counts, int* idx,
                                   int cap, cudaStream_t s) {
  const int stride = select_stride(g.nT);
  const size_t smem = sizeof(float) * (size_t)kSelWarps * stride;
  auto kern = select_rows_kernel<MAXV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long rows = (long long)g.BH * g.nT;
  const unsigned blocks = (unsigned)((rows + kSelWarps - 1) / kSelWarps);
  kern<<<blocks, kSelWarps * 32, smem, s>>>(g, S, top_p, k_min, counts, idx, cap, stride);
  return cudaGetLastError();
}

// Values per lane: the smallest supported multiple covering nT / 32.
cudaError_t launch_select(const Geom& g, const float* S, float top_p, int k_min, int* counts, int* idx, int cap,
                          cudaStream_t s) {
  const int need = (g.nT + 31) / 32;
  if (need <= 2) return launch_select_v<2>(g, S, top_p, k_min, counts, idx, cap, s);
  if (need <= 4) return launch_select_v<4>(g, S, top_p, k_min, counts, idx, cap, s);
  if (need <= 8) return launch_select_v<8>(g, S, top_p, k_min, counts, idx, cap, s);
  if (need <= 16) return launch_select_v<16>(g, S, top_p, k_min, counts, idx, cap, s);
  if (need <= 24) return launch_select_v<24>(g, S, top_p, k_min, counts, idx, cap, s);
  if (need <= 40) return launch_select_v<40>(g, S, top_p, k_min, counts, idx, cap, s);
  if (need <= 64) return launch_select_v<64>(g, S, top_p, k_min, counts, idx, cap, s);
  return launch_select_v<128>(g, S, top_p, k_min, counts, idx, cap, s);
}

}  // namespace fvattn
