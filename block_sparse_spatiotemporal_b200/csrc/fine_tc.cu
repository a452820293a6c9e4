// Fine stage on the 5th-generation tensor cores ("VSA" digest, section 3:
// token-level attention restricted to the selected tiles; "CalibAtt"
// digest: selected connections computed densely, the rest skipped).
//
// Persistent kernel, one CTA per SM, 192 threads:
//   warp 0      TMA producer: Q of the item's two query tiles, then K/V of
//               every key tile of the item's union list into a 4-stage ring;
//   warp 1      MMA issuer (one thread): S = Q K^T (M=128, N=64, K=128, both
//               operands in shared memory) into one of two TMEM S buffers,
//               then O += P V (M=128, N=128, K=64) with P read from TMEM;
//   warps 2..5  softmax: thread r owns row r (TMEM lane r) of the 128-row
//               tile; rows 0-63 are query tile 2p, rows 64-127 tile 2p+1.
// A key tile that only one of the two query tiles selected is masked for the
// other tile's rows: their P row is written as zeros and no exponential is
// evaluated for them, so those rows see only their own selection.
// Online softmax in base 2 with a lazy rescale: O in TMEM is only rescaled
// when a row's running max grows by more than 8 (log2 units).
//
// TMEM (256 columns): S0 [0,64), S1 [64,128), O [128,256) fp32; P (bf16)
// overwrites the first 32 columns of its S buffer.
// Shared memory (1024-aligned, 128-byte swizzle everywhere):
//   Q[2]  = 2 x (2 d-halves x 128 rows x 128 B)      64 KB
//   KV[4] = 4 x (K: 2 x 64 x 128 B, V: 2 x 64 x 128 B) 128 KB
#include "fvattn_internal.cuh"

namespace fvattn {
namespace ft {

constexpr int D = 128;
constexpr int STAGES = 4;
constexpr int THREADS = 192;
constexpr uint32_t HALF_CHUNK = 64 * 128;               // one 64-row x 128-byte box: 8 KB
constexpr uint32_t Q_BYTES = 4 * HALF_CHUNK;            // 32 KB
constexpr uint32_t KV_TILE_BYTES = 2 * HALF_CHUNK;      // 16 KB
constexpr uint32_t STAGE_BYTES = 2 * KV_TILE_BYTES;     // 32 KB
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 64, false, false);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 128, false, true);
constexpr int LAST_FLAG = 1 << 20;

struct Ctl {
  uint64_t q_full[2], q_empty[2];
  uint64_t kv_full[STAGES], kv_empty[STAGES];
  uint64_t s_full[2], p_full[2];
  uint64_t pv_done, o_empty;
  int meta[STAGES];
  uint32_t tmem_base;
  int abort;
};

constexpr uint32_t SMEM_BYTES = 1024 + 2 * Q_BYTES + STAGES * STAGE_BYTES + sizeof(Ctl);

}  // namespace ft

// One 64-token tile of a [BH, N, 128] bf16 tensor: two 64-column boxes
// (d 0-63 and 64-127) written `stride` bytes apart.
__device__ inline void tma_tile(const CUtensorMap* map, int natural, const FineTcArgs& a, int bh, int tile,
                                uint8_t* dst, uint32_t stride, uint64_t* bar) {
  if (natural) {
    const int cube = a.tile_cube[tile];
    const int w0 = cube_w(cube) * 4, h0 = cube_h(cube) * 4, t0 = cube_t(cube) * 4;
    tma_load_5d(dst, map, bar, 0, w0, h0, t0, bh);
    tma_load_5d(dst + stride, map, bar, 64, w0, h0, t0, bh);
  } else {
    tma_load_3d(dst, map, bar, 0, tile * kTileTokens, bh);
    tma_load_3d(dst + stride, map, bar, 64, tile * kTileTokens, bh);
  }
}

__device__ inline float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ inline uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&b);
}

__global__ void __launch_bounds__(ft::THREADS, 1)
    fine_tc_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                   const __grid_constant__ CUtensorMap mv, const FineTcArgs a) {
  using namespace ft;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + 2 * Q_BYTES;
  Ctl* ctl = reinterpret_cast<Ctl*>(sKV + STAGES * STAGE_BYTES);
  volatile int* abort_flag = &ctl->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Geom& g = a.g;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl->q_full[i], 1);
      mbar_init(&ctl->q_empty[i], 1);
      mbar_init(&ctl->s_full[i], 1);
      mbar_init(&ctl->p_full[i], 128);
    }
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&ctl->kv_full[i], 1);
      mbar_init(&ctl->kv_empty[i], 1);
    }
    mbar_init(&ctl->pv_done, 1);
    mbar_init(&ctl->o_empty, 128);
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
    prefetch_tensormap(&mq);
    prefetch_tensormap(&mk);
    prefetch_tensormap(&mv);
    long long gs = 0;
    int k = 0;
    for (int slot = blockIdx.x; slot < a.n_items; slot += gridDim.x, ++k) {
      const int item = a.worklist[slot];
      const int bh = item / g.P, p = item % g.P;
      const int i0 = 2 * p, i1 = (2 * p + 1 < g.nT) ? 2 * p + 1 : 2 * p;
      const int qb = k & 1;
      if (k >= 2 && !mbar_wait(&ctl->q_empty[qb], ((k >> 1) - 1) & 1, abort_flag, a.status, a.wait_cap)) break;
      mbar_arrive_expect_tx(&ctl->q_full[qb], Q_BYTES);
      uint8_t* qd = sQ + qb * Q_BYTES;
      tma_tile(&mq, a.q_nat, a, bh, i0, qd, 2 * HALF_CHUNK, &ctl->q_full[qb]);
      tma_tile(&mq, a.q_nat, a, bh, i1, qd + HALF_CHUNK, 2 * HALF_CHUNK, &ctl->q_full[qb]);
      const int n = a.ucount[item];
      const int* list = a.uni + (size_t)item * g.nT;
      int next = list[0];
      bool ok = true;
      for (int e = 0; e < n; ++e, ++gs) {
        int ent = next;
        if (e + 1 < n) next = list[e + 1];
        const int st = (int)(gs % STAGES);
        if (gs >= STAGES &&
            !mbar_wait(&ctl->kv_empty[st], (uint32_t)((gs / STAGES) - 1) & 1, abort_flag, a.status, a.wait_cap)) {
          ok = false;
          break;
        }
        int j = ent & 0xFFFF;
        if (j >= g.nT) {  // never produced by the schedule; keep the copy in bounds
          set_status(a.status, kStatusBadBlock);
          j = 0;
          ent &= ~0x30000;
        }
        ctl->meta[st] = ent | (e == n - 1 ? LAST_FLAG : 0);
        mbar_arrive_expect_tx(&ctl->kv_full[st], STAGE_BYTES);
        uint8_t* kd = sKV + st * STAGE_BYTES;
        tma_tile(&mk, a.k_nat, a, bh, j, kd, HALF_CHUNK, &ctl->kv_full[st]);
        tma_tile(&mv, a.v_nat, a, bh, j, kd + KV_TILE_BYTES, HALF_CHUNK, &ctl->kv_full[st]);
      }
      if (!ok) break;
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------------- MMA
    const uint32_t tS[2] = {tbase, tbase + 64};
    const uint32_t tO = tbase + 128;
    long long gs = 0;
    int k = 0;
    bool have_pend = false, pend_first = false;
    long long pend_g = 0;
    int pend_k = 0;
    bool ok = true;
    auto issue_pv = [&](long long s, bool first, int kitem) -> bool {
      if (!mbar_wait(&ctl->p_full[s & 1], (uint32_t)(s >> 1) & 1, abort_flag, a.status, a.wait_cap)) return false;
      if (first && kitem >= 1 && !mbar_wait(&ctl->o_empty, (uint32_t)(kitem - 1) & 1, abort_flag, a.status, a.wait_cap))
        return false;
      tc_fence_after();
      const int st = (int)(s % STAGES);
      const uint32_t vaddr = smem_u32(sKV + st * STAGE_BYTES + KV_TILE_BYTES);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t bdesc = umma_desc_sw128(vaddr + kk * 2048, HALF_CHUNK, 1024);
        mma_ts(tO, tS[s & 1] + kk * 8, bdesc, IDESC_PV, (first && kk == 0) ? 0u : 1u);
      }
      mma_commit(&ctl->kv_empty[st]);
      mma_commit(&ctl->pv_done);
      return true;
    };
    for (int slot = blockIdx.x; slot < a.n_items && ok; slot += gridDim.x, ++k) {
      const int qb = k & 1;
      if (!mbar_wait(&ctl->q_full[qb], (uint32_t)(k >> 1) & 1, abort_flag, a.status, a.wait_cap)) {
        ok = false;
        break;
      }
      const uint32_t qaddr = smem_u32(sQ + qb * Q_BYTES);
      bool first = true;
      while (true) {
        const int st = (int)(gs % STAGES);
        if (!mbar_wait(&ctl->kv_full[st], (uint32_t)(gs / STAGES) & 1, abort_flag, a.status, a.wait_cap)) {
          ok = false;
          break;
        }
        const int meta = ctl->meta[st];
        tc_fence_after();
        const uint32_t kaddr = smem_u32(sKV + st * STAGE_BYTES);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t adesc = umma_desc_sw128(qaddr + (kk >> 2) * (2 * HALF_CHUNK) + (kk & 3) * 32, 16, 1024);
          const uint64_t bdesc = umma_desc_sw128(kaddr + (kk >> 2) * HALF_CHUNK + (kk & 3) * 32, 16, 1024);
          mma_ss(tS[gs & 1], adesc, bdesc, IDESC_S, kk > 0 ? 1u : 0u);
        }
        mma_commit(&ctl->s_full[gs & 1]);
        if (have_pend && !issue_pv(pend_g, pend_first, pend_k)) {
          ok = false;
          break;
        }
        have_pend = true;
        pend_g = gs;
        pend_first = first;
        pend_k = k;
        first = false;
        ++gs;
        if (meta & LAST_FLAG) break;
      }
      if (!ok) break;
      mma_commit(&ctl->q_empty[qb]);
    }
    if (ok && have_pend) issue_pv(pend_g, pend_first, pend_k);
  } else if (warp >= 2) {
    // ------------------------------------------------------------ softmax
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const int half = r >> 6, rr = r & 63;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t tO = tbase + 128 + lane_off;
    const float sl2 = g.scale * 1.4426950408889634f;
    long long gs = 0;
    int k = 0;
    for (int slot = blockIdx.x; slot < a.n_items; slot += gridDim.x, ++k) {
      const int item = a.worklist[slot];
      const int bh = item / g.P, p = item % g.P;
      const int tile = 2 * p + half;
      const bool valid = tile < g.nT;
      float m_use = -INFINITY, l = 0.f;
      bool ok = true;
      while (true) {
        const int sb = (int)(gs & 1);
        if (!mbar_wait(&ctl->s_full[sb], (uint32_t)(gs >> 1) & 1, abort_flag, a.status, a.wait_cap)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int meta = ctl->meta[gs % STAGES];
        const bool sel = (meta >> (16 + half)) & 1;
        const uint32_t tSrow = tbase + sb * 64 + lane_off;
        uint32_t pk[32];
        float alpha = 1.f;
        bool rescale = false;
        {
          uint32_t s0[32], s1[32];
          tmem_ld32(tSrow, s0);
          tmem_ld32(tSrow + 32, s1);
          tmem_wait_ld();
          if (sel) {
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 32; ++c) mx = fmaxf(mx, fmaxf(__uint_as_float(s0[c]), __uint_as_float(s1[c])));
            const float m_new = mx * sl2;
            if (m_new > m_use + 8.f) {
              alpha = ex2(m_use - m_new);
              rescale = l > 0.f;
              l *= alpha;
              m_use = m_new;
            }
            float sum = 0.f;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const float p0 = ex2(fmaf(__uint_as_float(s0[2 * c]), sl2, -m_use));
              const float p1 = ex2(fmaf(__uint_as_float(s0[2 * c + 1]), sl2, -m_use));
              const float p2 = ex2(fmaf(__uint_as_float(s1[2 * c]), sl2, -m_use));
              const float p3 = ex2(fmaf(__uint_as_float(s1[2 * c + 1]), sl2, -m_use));
              pk[c] = pack_bf16(p0, p1);
              pk[16 + c] = pack_bf16(p2, p3);
              // normalise with the probabilities as the MMA sees them (bf16)
              sum += (__uint_as_float(pk[c] << 16) + __uint_as_float(pk[c] & 0xFFFF0000u)) +
                     (__uint_as_float(pk[16 + c] << 16) + __uint_as_float(pk[16 + c] & 0xFFFF0000u));
            }
            l += sum;
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) pk[c] = 0u;
          }
        }
        tmem_st32(tSrow, pk);
        if (__any_sync(0xffffffffu, rescale)) {
          if (!mbar_wait(&ctl->pv_done, (uint32_t)(gs - 1) & 1, abort_flag, a.status, a.wait_cap)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int ch = 0; ch < 4; ++ch) {
            uint32_t o[32];
            tmem_ld32(tO + ch * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(tO + ch * 32, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&ctl->p_full[sb]);
        ++gs;
        if (meta & LAST_FLAG) break;
      }
      if (!ok) break;
      // ---- epilogue: O / l -> out, lse
      if (!mbar_wait(&ctl->pv_done, (uint32_t)(gs - 1) & 1, abort_flag, a.status, a.wait_cap)) break;
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const int tok = !valid ? 0 : (a.out_nat ? cube_row_token(g, a.tile_cube[tile], rr) : tile * kTileTokens + rr);
      __nv_bfloat16* orow = a.out + ((size_t)bh * g.N + tok) * D;
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t o[32];
        tmem_ld32(tO + ch * 32, o);
        tmem_wait_ld();
        if (valid) {
          uint32_t w[16];
#pragma unroll
          for (int c = 0; c < 16; ++c)
            w[c] = pack_bf16(__uint_as_float(o[2 * c]) * inv, __uint_as_float(o[2 * c + 1]) * inv);
          uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
          for (int c = 0; c < 4; ++c) dst[c] = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
        }
      }
      if (valid)
        a.lse[(size_t)bh * g.N + tok] = l > 0.f ? (m_use + __log2f(l)) * 0.6931471805599453f : -INFINITY;
      tc_fence_before();
      mbar_arrive(&ctl->o_empty);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, ft::TMEM_COLS);
  }
}

cudaError_t launch_fine_tc(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const FineTcArgs& a,
                           int num_sms, cudaStream_t s) {
  cudaError_t e =
      cudaFuncSetAttribute(fine_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ft::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int grid = a.n_items < num_sms ? a.n_items : num_sms;
  if (grid <= 0) return cudaSuccess;
  fine_tc_kernel<<<grid, ft::THREADS, ft::SMEM_BYTES, s>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

}  // namespace fvattn
