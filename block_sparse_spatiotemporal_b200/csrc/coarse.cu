// Coarse stage: 3D RoPE on load, tile mean-pooling, pooled scores, row
// softmax and top-p selection with a k_min floor.
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
// top_p >= 1 keeps every tile.  The kernel never sorts the row: it finds the
// cut by bisection over the bit patterns of e_j = exp(s_j - max) (a radix
// select; positive floats order like their bits), with every mass computed
// as a deterministic warp-tree sum, and compares masses against top_p * Z
// instead of dividing.
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

// Vector load / store of DPL consecutive elements as fp32.
template <typename T, int DPL> struct Vec;
template <int DPL> struct Vec<float, DPL> {
  static __device__ inline void load(const float* p, float (&v)[DPL]) {
    if constexpr (DPL == 4) {
      const float4 t = *reinterpret_cast<const float4*>(p);
      v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    } else if constexpr (DPL == 2) {
      const float2 t = *reinterpret_cast<const float2*>(p);
      v[0] = t.x; v[1] = t.y;
    } else {
#pragma unroll
      for (int i = 0; i < DPL; ++i) v[i] = p[i];
    }
  }
  static __device__ inline void store(float* p, const float (&v)[DPL]) {
    if constexpr (DPL == 4) {
      *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    } else if constexpr (DPL == 2) {
      *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
    } else {
#pragma unroll
      for (int i = 0; i < DPL; ++i) p[i] = v[i];
    }
  }
};
template <int DPL> struct Vec<__nv_bfloat16, DPL> {
  static_assert(DPL % 2 == 0, "bf16 rows are read in pairs");
  static __device__ inline void load(const __nv_bfloat16* p, float (&v)[DPL]) {
    uint32_t w[DPL / 2];
    if constexpr (DPL == 4) {
      const uint2 t = *reinterpret_cast<const uint2*>(p);
      w[0] = t.x; w[1] = t.y;
    } else {
#pragma unroll
      for (int i = 0; i < DPL / 2; ++i) w[i] = reinterpret_cast<const uint32_t*>(p)[i];
    }
#pragma unroll
    for (int i = 0; i < DPL / 2; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
  static __device__ inline void store(__nv_bfloat16* p, const float (&v)[DPL]) {
    uint32_t w[DPL / 2];
#pragma unroll
    for (int i = 0; i < DPL / 2; ++i) {
      __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&b);
    }
    if constexpr (DPL == 4) {
      *reinterpret_cast<uint2*>(p) = make_uint2(w[0], w[1]);
    } else {
#pragma unroll
      for (int i = 0; i < DPL / 2; ++i) reinterpret_cast<uint32_t*>(p)[i] = w[i];
    }
  }
};

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
  const float x0 = a, x1 = b;
  a = x0 * cs.x - x1 * cs.y;
  b = x0 * cs.y + x1 * cs.x;
}

// --------------------------------------------------------------------------
// Pool: one block per (tile, head, tensor).  4 warps; warp w reads rows
// w, w+4, ..., each lane DPL consecutive dims of the row (a warp reads one
// whole row per step).  Sums are fp32 in a fixed order: rows of a warp in
// sequence, then the 4 warp partials in warp order; mean = sum / 64.
// Optionally writes the rotated rows, rounded to T, at tiled positions.
// --------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(128) pool_kernel(Geom g, const T* __restrict__ q, const T* __restrict__ k,
                                                   int natural, const int* __restrict__ tile_cube,
                                                   const int* __restrict__ tile_tok, RopeArgs rope,
                                                   float* __restrict__ qp, float* __restrict__ kp,
                                                   T* __restrict__ qrot, T* __restrict__ krot) {
  constexpr int DPL = D / 32;
  __shared__ float part[4][D];
  const int j = blockIdx.x, bh = blockIdx.y, which = blockIdx.z;
  const T* x = which == 0 ? q : k;
  float* pooled = which == 0 ? qp : kp;
  T* rot = which == 0 ? qrot : krot;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cube = tile_cube[j];
  float acc[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) acc[i] = 0.f;
#pragma unroll 4
  for (int r = warp; r < kTileTokens; r += 4) {
    const int n = natural ? cube_row_token(g, cube, r) : j * kTileTokens + r;
    const T* row = x + ((size_t)bh * g.N + n) * D + lane * DPL;
    float v[DPL];
    Vec<T, DPL>::load(row, v);
    if (rope.enabled) {
      // grid coordinate of the token in this row (tiled rows follow the order)
      const int nn = natural ? n : tile_tok[j * kTileTokens + r];
      const int t = nn / (g.Hg * g.W), h = (nn / g.W) % g.Hg, w = nn % g.W;
#pragma unroll
      for (int i = 0; i < DPL; i += 2) rope_pair(rope, g, lane * DPL + i, t, h, w, v[i], v[i + 1]);
    }
#pragma unroll
    for (int i = 0; i < DPL; ++i) acc[i] += v[i];
    if (rot) {
      T* dst = rot + ((size_t)bh * g.N + (size_t)j * kTileTokens + r) * D + lane * DPL;
      Vec<T, DPL>::store(dst, v);
    }
  }
  if (!pooled) return;
#pragma unroll
  for (int i = 0; i < DPL; ++i) part[warp][lane * DPL + i] = acc[i];
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    const float s = ((part[0][c] + part[1][c]) + part[2][c]) + part[3][c];
    pooled[((size_t)bh * g.nT + j) * D + c] = s * (1.0f / 64.0f);
  }
}

// --------------------------------------------------------------------------
// Score + select.  Block = 8 warps handling R = 8*RPW consecutive query tiles
// of one head.  Phase 1 computes S[R][nT] = scale * Qp Kp^T in shared memory
// (fp32 FFMA, register-tiled: each thread RPW rows x 2 key tiles).  Phase 2:
// warp w selects rows w*RPW .. w*RPW+RPW-1.
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
__device__ inline int warp_isum(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

constexpr int kKC = 64;   // key tiles per phase-1 chunk
constexpr int kKCS = 66;  // padded chunk row stride (floats)

template <int RPW, int D>
__global__ void __launch_bounds__(256) select_kernel(Geom g, const float* __restrict__ qp,
                                                     const float* __restrict__ kp, float top_p, int k_min,
                                                     int* __restrict__ counts, int* __restrict__ idx, int cap) {
  constexpr int R = 8 * RPW;
  extern __shared__ __align__(16) float sm[];
  float* qs = sm;                       // [D][R]   transposed query rows
  float* ks = qs + D * R;               // [D][kKCS] transposed key chunk
  float* S = ks + D * kKCS;             // [R][nT]
  const int nT = g.nT;
  const int bh = blockIdx.y;
  const int row0 = blockIdx.x * R;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* qph = qp + (size_t)bh * nT * D;
  const float* kph = kp + (size_t)bh * nT * D;

  for (int i = threadIdx.x; i < D * R; i += blockDim.x) {
    const int r = i / D, c = i % D;
    qs[c * R + r] = (row0 + r < nT) ? qph[(size_t)(row0 + r) * D + c] : 0.f;
  }
  for (int kc = 0; kc < nT; kc += kKC) {
    __syncthreads();
    for (int i = threadIdx.x; i < D * kKC; i += blockDim.x) {
      const int kk = i / D, c = i % D;
      ks[c * kKCS + kk] = (kc + kk < nT) ? kph[(size_t)(kc + kk) * D + c] : 0.f;
    }
    __syncthreads();
    float acc[RPW][2];
#pragma unroll
    for (int r = 0; r < RPW; ++r) acc[r][0] = acc[r][1] = 0.f;
#pragma unroll 8
    for (int c = 0; c < D; ++c) {
      const float2 kv = *reinterpret_cast<const float2*>(&ks[c * kKCS + 2 * lane]);
      float qv[RPW];
      if constexpr (RPW == 4) {
        const float4 t = *reinterpret_cast<const float4*>(&qs[c * R + warp * 4]);
        qv[0] = t.x; qv[1] = t.y; qv[2] = t.z; qv[3] = t.w;
      } else {
#pragma unroll
        for (int r = 0; r < RPW; ++r) qv[r] = qs[c * R + warp * RPW + r];
      }
#pragma unroll
      for (int r = 0; r < RPW; ++r) {
        acc[r][0] = fmaf(qv[r], kv.x, acc[r][0]);
        acc[r][1] = fmaf(qv[r], kv.y, acc[r][1]);
      }
    }
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
      const int kk = kc + 2 * lane;
      if (kk < nT) S[(warp * RPW + r) * nT + kk] = acc[r][0] * g.scale;
      if (kk + 1 < nT) S[(warp * RPW + r) * nT + kk + 1] = acc[r][1] * g.scale;
    }
  }
  __syncthreads();

  for (int rr = 0; rr < RPW; ++rr) {
    const int lr = warp * RPW + rr;
    const int row = row0 + lr;
    if (row >= nT) break;
    float* s = S + lr * nT;
    uint32_t* bits = reinterpret_cast<uint32_t*>(s);
    float mx = -INFINITY;
    for (int j = lane; j < nT; j += 32) mx = fmaxf(mx, s[j]);
    mx = warp_max(mx);
    float zpart = 0.f;
    for (int j = lane; j < nT; j += 32) {
      const float e = expf(s[j] - mx);
      s[j] = e;
      zpart += e;
    }
    const float Z = warp_sum(zpart);
    __syncwarp();

    int count;
    uint32_t uT = 0;       // threshold bit pattern of the selected set
    int take = 0;          // tiles with bits == uT to take, lowest ids first
    if (top_p >= 1.0f) {
      count = nT;
    } else {
      int m = 1;
      uint32_t u = 0;
      int r_ties = 1;
      if (top_p > 0.f) {
        const float target = top_p * Z;
        for (int b = 29; b >= 0; --b) {
          const uint32_t cand = u | (1u << b);
          float part = 0.f;
          for (int j = lane; j < nT; j += 32) part += bits[j] >= cand ? s[j] : 0.f;
          if (warp_sum(part) >= target) u = cand;
        }
        float gpart = 0.f;
        int cgt = 0, ceq = 0;
        for (int j = lane; j < nT; j += 32) {
          gpart += bits[j] > u ? s[j] : 0.f;
          cgt += bits[j] > u ? 1 : 0;
          ceq += bits[j] == u ? 1 : 0;
        }
        const float mgt = warp_sum(gpart);
        cgt = warp_isum(cgt);
        ceq = warp_isum(ceq);
        const float eu = __uint_as_float(u);
        float accm = mgt + eu;
        r_ties = 1;
        while (r_ties < ceq && accm < target) {
          accm += eu;
          ++r_ties;
        }
        m = ceq > 0 ? cgt + r_ties : (cgt > 0 ? cgt : 1);
        if (ceq == 0) r_ties = 0;
      }
      count = m > k_min ? m : k_min;
      if (count > nT) count = nT;
      if (count == m && top_p > 0.f) {
        uT = u;
        take = r_ties;
      } else {
        // top-`count` set: largest u2 with #{bits >= u2} >= count
        uint32_t u2 = 0;
        for (int b = 30; b >= 0; --b) {
          const uint32_t cand = u2 | (1u << b);
          int c = 0;
          for (int j = lane; j < nT; j += 32) c += bits[j] >= cand ? 1 : 0;
          if (warp_isum(c) >= count) u2 = cand;
        }
        int cgt = 0;
        for (int j = lane; j < nT; j += 32) cgt += bits[j] > u2 ? 1 : 0;
        cgt = warp_isum(cgt);
        uT = u2;
        take = count - cgt;
      }
    }

    int* out = idx + ((size_t)bh * nT + row) * (size_t)cap;
    if (count == nT) {
      for (int j = lane; j < nT; j += 32) out[j] = j;
    } else {
      int base = 0, tie_base = 0;
      for (int j0 = 0; j0 < nT; j0 += 32) {
        const int j = j0 + lane;
        const uint32_t bj = j < nT ? bits[j] : 0u;
        const bool tie = j < nT && bj == uT;
        const unsigned tmask = __ballot_sync(0xffffffffu, tie);
        const int trank = tie_base + __popc(tmask & ((1u << lane) - 1u));
        const bool sel = j < nT && (bj > uT || (tie && trank < take));
        const unsigned smask = __ballot_sync(0xffffffffu, sel);
        const int pos = base + __popc(smask & ((1u << lane) - 1u));
        if (sel && pos < count) out[pos] = j;
        base += __popc(smask);
        tie_base += __popc(tmask);
      }
    }
    if (lane == 0) counts[(size_t)bh * nT + row] = count;
  }
}

template <typename T, int D>
static cudaError_t launch_pool_t(const Geom& g, const void* q, const void* k, int natural, const int* tile_cube,
                                 const int* tile_tok, const RopeArgs& rope, float* qp, float* kp, void* qrot,
                                 void* krot, cudaStream_t s) {
  dim3 grid(g.nT, g.BH, 2);
  pool_kernel<T, D><<<grid, 128, 0, s>>>(g, (const T*)q, (const T*)k, natural, tile_cube, tile_tok, rope, qp, kp,
                                         (T*)qrot, (T*)krot);
  return cudaGetLastError();
}

cudaError_t launch_pool(const Geom& g, int dtype, const void* q, const void* k, int natural, const int* tile_cube,
                        const int* tile_tok, int rope_enabled, int dt, int dh, int dw, const float2* rope_tab, float* qp, float* kp,
                        void* qrot, void* krot, cudaStream_t s) {
  RopeArgs r{rope_enabled, dt, dh, dw, rope_tab};
  if (dtype == FVATTN_BF16) {
    if (g.d == 128) return launch_pool_t<__nv_bfloat16, 128>(g, q, k, natural, tile_cube, tile_tok, r, qp, kp, qrot, krot, s);
    if (g.d == 64) return launch_pool_t<__nv_bfloat16, 64>(g, q, k, natural, tile_cube, tile_tok, r, qp, kp, qrot, krot, s);
  } else {
    if (g.d == 128) return launch_pool_t<float, 128>(g, q, k, natural, tile_cube, tile_tok, r, qp, kp, qrot, krot, s);
    if (g.d == 64) return launch_pool_t<float, 64>(g, q, k, natural, tile_cube, tile_tok, r, qp, kp, qrot, krot, s);
    if (g.d == 32) return launch_pool_t<float, 32>(g, q, k, natural, tile_cube, tile_tok, r, qp, kp, qrot, krot, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_rope_table(const Geom& g, int dt, int dh, int dw, float base, float2* tab, cudaStream_t s) {
  const int total = g.T * (dt / 2) + g.Hg * (dh / 2) + g.W * (dw / 2);
  rope_table_kernel<<<(total + 255) / 256, 256, 0, s>>>(g, dt, dh, dw, base, tab);
  return cudaGetLastError();
}

size_t select_smem_bytes(int nT, int d, int rpw) {
  const int R = 8 * rpw;
  return sizeof(float) * ((size_t)d * R + (size_t)d * kKCS + (size_t)R * nT);
}

template <int RPW, int D>
static cudaError_t launch_select_t(const Geom& g, const float* qp, const float* kp, float top_p, int k_min,
                                   int* counts, int* idx, int cap, cudaStream_t s) {
  const size_t smem = select_smem_bytes(g.nT, D, RPW);
  cudaError_t e = cudaFuncSetAttribute(select_kernel<RPW, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  constexpr int R = 8 * RPW;
  dim3 grid((g.nT + R - 1) / R, g.BH);
  select_kernel<RPW, D><<<grid, 256, smem, s>>>(g, qp, kp, top_p, k_min, counts, idx, cap);
  return cudaGetLastError();
}

// Rows per warp: 4 while the score block fits comfortably, else 1.
int select_rows_per_warp(int nT, int d) { return select_smem_bytes(nT, d, 4) <= 220 * 1024 ? 4 : 1; }

cudaError_t launch_select(const Geom& g, const float* qp, const float* kp, float top_p, int k_min, int* counts,
                          int* idx, int cap, cudaStream_t s) {
  const int rpw = select_rows_per_warp(g.nT, g.d);
  if (g.d == 128)
    return rpw == 4 ? launch_select_t<4, 128>(g, qp, kp, top_p, k_min, counts, idx, cap, s)
                    : launch_select_t<1, 128>(g, qp, kp, top_p, k_min, counts, idx, cap, s);
  if (g.d == 64)
    return rpw == 4 ? launch_select_t<4, 64>(g, qp, kp, top_p, k_min, counts, idx, cap, s)
                    : launch_select_t<1, 64>(g, qp, kp, top_p, k_min, counts, idx, cap, s);
  if (g.d == 32)
    return rpw == 4 ? launch_select_t<4, 32>(g, qp, kp, top_p, k_min, counts, idx, cap, s)
                    : launch_select_t<1, 32>(g, qp, kp, top_p, k_min, counts, idx, cap, s);
  return cudaErrorInvalidValue;
}

}  // namespace fvattn
