// Fine stage on the 5th-generation tensor cores ("VSA" digest, section 3:
// token-level attention restricted to the selected tiles; "CalibAtt"
// digest: selected connections computed densely, the rest skipped).
//
// Persistent kernel, one CTA per SM, 384 threads.  A work item is four
// adjacent query tiles of one head, run as two 128-row streams that share
// every K/V tile: stream A = tiles (4q, 4q+1), stream B = (4q+2, 4q+3).
//   warp 0       TMA producer: the item's four Q tiles, then K/V of every
//                entry of the item's union list into a 5-stage ring;
//   warps 1, 2   MMA issuers, one thread per stream: for each entry the
//                stream takes part in, S = Q K^T (M=128, N=64, K=128,
//                operands in shared memory) into one of its two TMEM S
//                buffers, then O += P V (M=128, N=128, K=64, P read from
//                TMEM) of its previous step;
//   warps 4-7    softmax of stream A, warps 8-11 softmax of stream B: thread
//                r of a group owns row r (TMEM lane r) of its stream.
// While one stream's softmax runs, the tensor core works on the other
// stream.  A key tile selected by only some of an item's tiles is masked for
// the others' rows: their P row is written as zeros and no exponential is
// evaluated for them, so every row sees exactly its own tile's selection.
// Online softmax in base 2 with a lazy rescale (O is rescaled in TMEM only
// when a row's running max grows by more than 2^64); the normaliser sums the
// bf16 probabilities the PV MMA consumes.
//
// TMEM (512 columns), per stream s at column 256 s: S0 [0,64), S1 [64,128),
// O [128,256), fp32; P (bf16) overwrites the first 32 columns of its S.
// Shared memory (1024-aligned, 128-byte swizzle), default build:
//   Q     = 2 d-halves x 256 rows x 128 B                   64 KB
//   KV[5] = 5 x (K: 2 x 64 x 128 B, V: 2 x 64 x 128 B)     160 KB
#include "fvattn_internal.cuh"

namespace fvattn {
namespace ft {

#ifndef FVATTN_FT_STAGES
#define FVATTN_FT_STAGES 5
#endif
#ifndef FVATTN_FT_QBUF
#define FVATTN_FT_QBUF 1
#endif
constexpr int D = 128;
constexpr int STAGES = FVATTN_FT_STAGES;   // K/V ring depth
constexpr int QBUF = FVATTN_FT_QBUF;       // Q buffers (items in flight)
constexpr int THREADS = 384;
constexpr int SM_WARP0 = 4;                             // first softmax warp
constexpr uint32_t BOX = 64 * 128;                      // one 64-row x 128-byte box: 8 KB
constexpr uint32_t Q_BYTES = 8 * BOX;                   // 4 tiles x 2 d-halves: 64 KB
constexpr uint32_t Q_HALF = 4 * BOX;                    // one d-half of the 256 Q rows
constexpr uint32_t KV_TILE_BYTES = 2 * BOX;             // 16 KB
constexpr uint32_t STAGE_BYTES = 2 * KV_TILE_BYTES;     // 32 KB
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 64, false, false);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, 128, false, true);
constexpr int ITEM_LAST = 1 << 24;

struct Stream {
  uint64_t s_full[2];     // S ready (MMA commit) + step info written (MMA thread arrive)
  uint64_t p_full[2];     // P written by the 128 softmax threads
  uint64_t pv_done[2];    // PV of step c completes pv_done[c & 1]; waiting on it by
                          // parity is exact because the thread has already seen the
                          // S commit that follows the PV of step c - 2
  uint64_t o_empty;       // epilogue read O (128 arrivals per item)
  int info[2];            // per S buffer: selection bits of this stream's two tiles | last << 2
};

struct Ctl {
  uint64_t q_full[QBUF], q_empty[QBUF];
  uint64_t kv_full[STAGES], kv_empty[STAGES];
  Stream st[2];
  int meta[STAGES];
  uint32_t tmem_base;
  int abort;
};

constexpr uint32_t SMEM_BYTES = 1024 + QBUF * Q_BYTES + STAGES * STAGE_BYTES;
// A row's running max may grow by this much (log2 units) before O is
// rescaled: P is bf16 (exponent range 2^+-127) and O, l are fp32, so
// probabilities up to 2^64 relative to the stale max are exact enough and
// the rescale (a wait on the in-flight PV plus a TMEM read-modify-write of
// O) almost never runs.
constexpr float RESCALE_LOG2 = 64.f;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

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
  uint8_t* sKV = smem + QBUF * Q_BYTES;
  __shared__ Ctl ctl_s;
  Ctl* ctl = &ctl_s;
  volatile int* abort_flag = &ctl->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Geom& g = a.g;
  const long long cap = a.wait_cap;

  if (threadIdx.x == 0) {
    for (int i = 0; i < QBUF; ++i) {
      mbar_init(&ctl->q_full[i], 1);
      mbar_init(&ctl->q_empty[i], 2);      // one release per stream
    }
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&ctl->kv_full[i], 1);
      mbar_init(&ctl->kv_empty[i], 2);     // one release per stream
    }
    for (int s = 0; s < 2; ++s) {
      for (int i = 0; i < 2; ++i) {
        mbar_init(&ctl->st[s].s_full[i], 2);
        mbar_init(&ctl->st[s].p_full[i], 128);
      }
      mbar_init(&ctl->st[s].pv_done[0], 1);
      mbar_init(&ctl->st[s].pv_done[1], 1);
      mbar_init(&ctl->st[s].o_empty, 128);
    }
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
    bool ok = true;
    for (int slot = blockIdx.x; slot < a.n_items && ok; slot += gridDim.x, ++k) {
      const int item = a.worklist[slot];
      const int bh = item / g.P, qd = item % g.P;
      const int qb = k % QBUF;
      if (k >= QBUF && !mbar_wait(&ctl->q_empty[qb], ((k / QBUF) - 1) & 1, abort_flag, a.status, cap)) break;
      mbar_arrive_expect_tx(&ctl->q_full[qb], Q_BYTES);
      uint8_t* qd_smem = sQ + qb * Q_BYTES;
#pragma unroll 1
      for (int t = 0; t < kItemTiles; ++t) {
        int tile = kItemTiles * qd + t;
        if (tile >= g.nT) tile = kItemTiles * qd;        // rows of a missing tile are never stored
        tma_tile(&mq, a.q_nat, a, bh, tile, qd_smem + t * BOX, Q_HALF, &ctl->q_full[qb]);
      }
      const int n = a.ucount[item];
      const int* list = a.uni + (size_t)item * g.nT;
      int next = list[0];
      for (int e = 0; e < n; ++e, ++gs) {
        int ent = next;
        if (e + 1 < n) next = list[e + 1];
        const int st = (int)(gs % STAGES);
        if (gs >= STAGES &&
            !mbar_wait(&ctl->kv_empty[st], (uint32_t)((gs / STAGES) - 1) & 1, abort_flag, a.status, cap)) {
          ok = false;
          break;
        }
        int j = ent & 0xFFFF;
        if (j >= g.nT) {  // never produced by the schedule; keep the copy in bounds
          set_status(a.status, kStatusBadBlock);
          j = 0;
          ent &= ~0xF0000;
        }
        ctl->meta[st] = ent | (e == n - 1 ? ITEM_LAST : 0);
        mbar_arrive_expect_tx(&ctl->kv_full[st], STAGE_BYTES);
        uint8_t* kd = sKV + st * STAGE_BYTES;
        tma_tile(&mk, a.k_nat, a, bh, j, kd, BOX, &ctl->kv_full[st]);
        tma_tile(&mv, a.v_nat, a, bh, j, kd + KV_TILE_BYTES, BOX, &ctl->kv_full[st]);
      }
    }
  } else if ((warp == 1 || warp == 2) && lane == 0) {
    // ------------------------------------------------- MMA (one per stream)
    // Stream x's issuer walks every entry in order.  Entries it takes part
    // in: S of step c into S buffer c & 1, then the PV of step c - 1 once its
    // P is written (so the softmax always has the next S ready).  Entries it
    // sits out: it settles any pending PV and releases its share of the
    // stage.  A stage is reloaded once both streams released it; a Q buffer
    // once both issuers passed the item's last entry.
    const int x = warp - 1;
    Stream& S = ctl->st[x];
    const uint64_t qdesc0 = umma_desc_sw128(smem_u32(sQ), 16, 1024) + (uint64_t)((x * 2 * BOX) >> 4);
    const uint64_t kdesc0 = umma_desc_sw128(smem_u32(sKV), 16, 1024);
    const uint64_t vdesc0 = umma_desc_sw128(smem_u32(sKV + KV_TILE_BYTES), BOX, 1024);
    const uint32_t tS0 = tbase + 256 * x, tO = tbase + 256 * x + 128;
    long long gs = 0, c = 0;
    int k = 0;
    bool pend = false, pend_first = false, ok = true;
    long long pend_c = 0;
    int pend_stage = 0, pend_item = 0;
    auto issue_pv = [&]() -> bool {
      const int b = (int)(pend_c & 1);
      if (!mbar_wait(&S.p_full[b], (uint32_t)(pend_c >> 1) & 1, abort_flag, a.status, cap)) return false;
      if (pend_first && pend_item >= 1 &&
          !mbar_wait(&S.o_empty, (uint32_t)(pend_item - 1) & 1, abort_flag, a.status, cap))
        return false;
      tc_fence_after();
      const uint64_t vd = vdesc0 + (uint64_t)((pend_stage * STAGE_BYTES) >> 4);
      const uint32_t tP = tS0 + 64 * b;
      mma_ts(tO, tP, vd, IDESC_PV, pend_first ? 0u : 1u);
#pragma unroll
      for (int kk = 1; kk < 4; ++kk) mma_ts(tO, tP + kk * 8, vd + kk * (2048 >> 4), IDESC_PV, 1u);
      mma_commit(&S.pv_done[b]);
      mma_commit(&ctl->kv_empty[pend_stage]);
      pend = false;
      return true;
    };
    for (int slot = blockIdx.x; slot < a.n_items && ok; slot += gridDim.x, ++k) {
      const int qb = k % QBUF;
      if (!mbar_wait(&ctl->q_full[qb], (uint32_t)(k / QBUF) & 1, abort_flag, a.status, cap)) break;
      const uint64_t qd = qdesc0 + (uint64_t)((qb * Q_BYTES) >> 4);
      bool first = true;
      while (true) {
        const int st = (int)(gs % STAGES);
        if (!mbar_wait(&ctl->kv_full[st], (uint32_t)(gs / STAGES) & 1, abort_flag, a.status, cap)) {
          ok = false;
          break;
        }
        const int meta = ctl->meta[st];
        if ((meta >> (20 + x)) & 1) {
          const int b = (int)(c & 1);
          S.info[b] = ((meta >> (16 + 2 * x)) & 3) | (((meta >> (22 + x)) & 1) << 2);
          tc_fence_after();
          const uint64_t kd = kdesc0 + (uint64_t)((st * STAGE_BYTES) >> 4);
          const uint32_t tS = tS0 + 64 * b;
          mma_ss(tS, qd, kd, IDESC_S, 0u);
#pragma unroll
          for (int kk = 1; kk < 8; ++kk)
            mma_ss(tS, qd + (((kk >> 2) * Q_HALF + (kk & 3) * 32) >> 4), kd + (((kk >> 2) * BOX + (kk & 3) * 32) >> 4),
                   IDESC_S, 1u);
          mma_commit(&S.s_full[b]);
          mbar_arrive(&S.s_full[b]);
          if (pend && !issue_pv()) {
            ok = false;
            break;
          }
          pend = true;
          pend_c = c;
          pend_stage = st;
          pend_first = first;
          pend_item = k;
          first = false;
          ++c;
        } else {
          if (pend && !issue_pv()) {
            ok = false;
            break;
          }
          mbar_arrive(&ctl->kv_empty[st]);
        }
        ++gs;
        if (meta & ITEM_LAST) break;
      }
      if (!ok) break;
      mma_commit(&ctl->q_empty[qb]);
    }
    if (ok && pend) issue_pv();
  } else if (warp >= SM_WARP0) {
    // ------------------------------------------------------------ softmax
    const int s = (warp - SM_WARP0) >> 2;             // stream
    Stream& S = ctl->st[s];
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;                     // row of the stream
    const int half = r >> 6, rr = r & 63;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t tcol = tbase + 256 * s;
    const uint32_t tO = tcol + 128 + lane_off;
    const float sl2 = g.scale * 1.4426950408889634f;
    long long c = 0;
    for (int slot = blockIdx.x; slot < a.n_items; slot += gridDim.x) {
      const int item = a.worklist[slot];
      const int bh = item / g.P, qd = item % g.P;
      const int tile = kItemTiles * qd + 2 * s + half;
      const bool valid = tile < g.nT;
      float m_use = -INFINITY, l = 0.f;
      bool ok = true;
      while (true) {
        const int sb = (int)(c & 1);
        if (!mbar_wait(&S.s_full[sb], (uint32_t)(c >> 1) & 1, abort_flag, a.status, cap)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int info = S.info[sb];
        const bool sel = (info >> half) & 1;
        const uint32_t tSrow = tcol + 64 * sb + lane_off;
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
            for (int i = 0; i < 32; ++i) mx = fmaxf(mx, fmaxf(__uint_as_float(s0[i]), __uint_as_float(s1[i])));
            const float m_new = mx * sl2;
            if (m_new > m_use + RESCALE_LOG2) {
              alpha = ex2(m_use - m_new);
              rescale = l > 0.f;
              l *= alpha;
              m_use = m_new;
            }
            float sum = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float p0 = ex2(fmaf(__uint_as_float(s0[2 * i]), sl2, -m_use));
              const float p1 = ex2(fmaf(__uint_as_float(s0[2 * i + 1]), sl2, -m_use));
              const float p2 = ex2(fmaf(__uint_as_float(s1[2 * i]), sl2, -m_use));
              const float p3 = ex2(fmaf(__uint_as_float(s1[2 * i + 1]), sl2, -m_use));
              pk[i] = pack_bf16(p0, p1);
              pk[16 + i] = pack_bf16(p2, p3);
              // normalise with the probabilities as the MMA sees them (bf16)
              sum += (__uint_as_float(pk[i] << 16) + __uint_as_float(pk[i] & 0xFFFF0000u)) +
                     (__uint_as_float(pk[16 + i] << 16) + __uint_as_float(pk[16 + i] & 0xFFFF0000u));
            }
            l += sum;
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) pk[i] = 0u;
          }
        }
        tmem_st32(tSrow, pk);
        if (__any_sync(0xffffffffu, rescale)) {
          if (!mbar_wait(&S.pv_done[(c - 1) & 1], (uint32_t)((c - 1) >> 1) & 1, abort_flag, a.status, cap)) {
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
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tO + ch * 32, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&S.p_full[sb]);
        ++c;
        if (info & 4) break;
      }
      if (!ok) break;
      // ---- epilogue: O / l -> out, lse
      if (!mbar_wait(&S.pv_done[(c - 1) & 1], (uint32_t)((c - 1) >> 1) & 1, abort_flag, a.status, cap)) break;
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
          for (int i = 0; i < 16; ++i)
            w[i] = pack_bf16(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
          uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
      }
      if (valid)
        a.lse[(size_t)bh * g.N + tok] = l > 0.f ? (m_use + __log2f(l)) * 0.6931471805599453f : -INFINITY;
      tc_fence_before();
      mbar_arrive(&S.o_empty);
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
