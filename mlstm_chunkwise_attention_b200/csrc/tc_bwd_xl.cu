// Intra-chunk backward kernels for large chunks (chunk >= 256, d_qk = d_hv =
// 128, bf16 I/O) on the organisation of the large-chunk forward kernel: dq,
// dk and dv each walk the 128-token partner tiles of a 128-row tile's chunk
// ("Tiled Flash Linear Attention: More Efficient Linear RNN and xLSTM
// Kernels", TFLA summary page, Approach: the second level of tiling inside a
// chunk, here applied to the backward as the same page's Key results time it).
//
// Mathematics (m held constant; dnum_t = dh_t / den_t, da_t the normaliser
// gradient, D_ts = exp(b_t - b_s + log i_s - m_t) for s <= t in the chunk):
//   dq_t = [alpha_t (C_{c-1} dnum_t + da_t n_{c-1}) + sum_s (dh_t.v_s/den_t + da_t) D_ts k_s] / sqrt(d_qk)
//   dk_s = w_s (dC_c v_s + dn_c) + sum_t (dh_t.v_s/den_t + da_t) D_ts q_t / sqrt(d_qk)
//   dv_s = w_s dC_c^T k_s + sum_t D_ts (q_t.k_s / sqrt(d_qk)) dh_t / den_t
// For a 128-row tile R (query rows for dq, key rows for dk and dv):
//   X_j = A_R B_j^T   (dq: dH V_j^T, dk: V dH_j^T, dv: K Q_j^T)
//   Y_j = gates, mask and normaliser terms applied to X_j (bf16, in TMEM)
//   Acc = rescale_rows(A_R G) + sum_j Y_j E_j   (E: dq K_j, dk Q_j, dv dH_j;
//         G the chunk state (dq) or its gradient (dk, dv), hi and lo planes)
//
// Organisation (one persistent CTA per SM; work items = (row tile, head,
// chunk), in balanced pairs of row tiles):
//  * warp 0 streams the row tile A (double-buffered, with its rows' gate
//    factors) and, through a ring, B_j and the two state planes; warp 18
//    streams E_j with its partners' gate factors through a second ring;
//  * warp 1 (lane 0 alone) issues tcgen05.mma from precomputed descriptors:
//    X_{j+1} before Y_j E_j, so the tensor core computes the next score tile
//    while the transform runs; the inter-chunk product lands in the item's
//    accumulator first and is rescaled per row in TMEM before the first
//    accumulate;
//  * warps 2-17 (a 32-row quarter of the tile and a 32-partner block each,
//    four warps per SM sub-partition) turn X into Y in TMEM in place, packed
//    into the first half of the block's own 32 columns, which the TS-form
//    accumulate reads;
//  * the accumulator is double-buffered in TMEM; the epilogue of an item
//    (scale, the per-token dot product q.dq or k.dk, the output through
//    swizzled staging and TMA stores) runs after the first step of the next.
// The gate factors come from a per-chunk table (layout in internal.h) that
// bwd_xl_table writes.  Off-diagonal 32 x 32 blocks use the separable form,
// split at the largest key exponent of the key block, so dq and dk round
// exactly the same bf16 values (same fp32 operations in the same order):
//   dq: ((x + QE_t) exp2(QX_t + KM)) KG_s,  dk: ((x + QE_t) exp2(QX_t + KM)) KG_s,
// and the forget-gate gradient (a reverse cumsum of q.dq - k.dk) keeps the
// cancellation it has in exact arithmetic.  The diagonal block of the
// diagonal tile takes each element's own exponent and the causal mask.
// Every wait is bounded; on a timeout the kernel raises its error flag and
// winds down.
#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace mlstm {

static __device__ unsigned int g_tc_bwd_xl_error;

namespace {

constexpr float kLog2e = 1.4426950408889634f;
enum { BX_DQ = 0, BX_DK = 1, BX_DV = 2 };

constexpr int kBxThreads = 608;    // A/B producer, MMA, 16 transform warps, E producer
constexpr int kBxTransform = 512;  // transform threads (warps 2..17)
constexpr int kBxEWarp = 18;       // E producer warp

struct BxCfg {
  static constexpr int TILE = 32768;        // 128 rows x 128 bf16: two 64-column SW128 blocks
  static constexpr int NA = 2, NB = 2, NE = 2;
  static constexpr int ROWAUX = 4 * 512 + 64;  // four row vectors of 128 floats; 4 block maxima
  static constexpr int COLAUX = 3 * 512 + 64;  // up to three partner vectors; 4 block maxima
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + NA * TILE;
  static constexpr int OFF_E = OFF_B + NB * TILE;
  static constexpr int OFF_ROW = OFF_E + NE * TILE;
  static constexpr int OFF_COL = OFF_ROW + NA * ROWAUX;
  static constexpr int OFF_FW = OFF_COL + NE * COLAUX;  // per transform warp: 32 partner factors
  // per transform warp: 16 rows of 32 bf16 output columns, 1024-byte aligned for the swizzle
  static constexpr int OFF_STG = (OFF_FW + 16 * 32 * 4 + 1023) & ~1023;
  static constexpr int STG_WARP = 1024;
  static constexpr int OFF_BAR = OFF_STG + 16 * STG_WARP;
  static constexpr int OFF_TMEM = OFF_BAR + 64 * 8;
  static constexpr int SMEM = OFF_TMEM + 16 + 1024;  // + alignment slack
  static constexpr uint32_t TMEM_COLS = 512;         // X0 [0,128) X1 [128,256) Acc0, Acc1 from 256
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

enum {
  Y_AF0 = 0,   // row tile (+ its gate factors) full, per A buffer
  Y_AE0 = 2,   // A buffer free: MMA commit + 512 transform threads
  Y_BF0 = 4,   // B stage full (B tile or one state plane)
  Y_BE0 = 6,   // B stage free (MMA commit)
  Y_EF0 = 8,   // E stage full (E tile + its partners' gate factors)
  Y_EE0 = 10,  // E stage free (MMA commit after the accumulate)
  Y_SF0 = 12,  // score written (MMA commit), per X buffer
  Y_PF0 = 14,  // Y written (512 threads), per X buffer
  Y_IF0 = 16,  // inter-chunk product written (MMA commit), per Acc buffer
  Y_IR0 = 18,  // inter-chunk product rescaled (512 threads), per Acc buffer
  Y_OF0 = 20,  // Acc complete (MMA commit), per Acc buffer
  Y_OE0 = 22,  // Acc read out (512 threads), per Acc buffer
  Y_DRAIN = 24,  // the MMA thread's last commit when it gives up
  Y_COUNT = 25
};

struct BxItem {
  int rt, bh, c, t0, len, np, p0;
  bool inter;  // a state product enters the accumulator
};

struct BxParams {
  const float* tab;     // per-chunk gate table (bwd_xl_table_stride(L) floats per chunk)
  const float* rowvec;  // dq: n_{c-1}, dk: dn_c [BH, NC, 128] (mLSTMexp); dv: unused
  const bf16* dot_src;  // dq: q, dk: k [BH, T, 128]
  float* pdot;          // dq: pq, dk: pk [4 planes][BH, T]: the share of 32 columns h in plane h
  size_t pdot_stride;   // elements per plane
  int T, L, NC, BH, ntq, total, tstride;
  bool init;  // the forward started from an initial state (dq: every chunk has a state)
  bool dfin;  // the final state has a gradient (dk, dv: every chunk has a state gradient)
  float scale;
  float log2_scale;
  unsigned int epoch;
};

// Items come in pairs of row tiles ntq-1-p and p of one (head, chunk), so a pair holds
// ntq + 1 partner tiles whatever the kind and a static split of pairs over the CTAs is
// balanced; the pair index varies fastest, so the CTAs running at one time cover few
// chunks and their partner tiles stay in L2.
template <int KIND>
__device__ __forceinline__ bool bx_item(int k, const BxParams& P, BxItem& it) {
  const int half_ntq = P.ntq >> 1;
  int r = k >> 1;
  const int pi = r % half_ntq;
  r /= half_ntq;
  it.c = r % P.NC;
  it.bh = r / P.NC;
  it.rt = (k & 1) ? pi : P.ntq - 1 - pi;
  it.t0 = it.rt * 128;
  it.len = min(P.L, P.T - it.c * P.L);
  if (it.t0 >= it.len) return false;
  if (KIND == BX_DQ) {
    it.np = it.rt + 1;
    it.p0 = 0;
    it.inter = it.c > 0 || P.init;
  } else {
    it.np = (it.len + 127) / 128 - it.rt;
    it.p0 = it.rt;
    it.inter = it.c < P.NC - 1 || P.dfin;
  }
  return true;
}

__device__ __forceinline__ int bx_first() { return 2 * blockIdx.x; }
__device__ __forceinline__ int bx_succ(int k) { return (k & 1) ? k + 2 * gridDim.x - 1 : k + 1; }

template <int KIND>
__device__ __forceinline__ int bx_next(int k, const BxParams& P, BxItem& it) {
  for (; k < P.total; k = bx_succ(k))
    if (bx_item<KIND>(k, P, it)) return k;
  return P.total;
}

// Epilogue of one item for the transform thread of row 32 qr + lane and columns
// [32 h, 32 h + 32): the accumulator leaves TMEM (freeing it for the next items'
// products), is scaled, dotted with the row's q (dq) or k (dk) for the gate
// gradients (this column block's share stored in plane h; the gate-gradient
// kernels add the four planes in block order), and stored through this warp's
// staging slot by 16-row TMA stores
// (rows past the sequence end are clipped by the TMA unit).  Inlined: an
// out-of-line call makes the caller save its live registers around it.
template <int KIND>
__device__ __forceinline__ bool bx_epilogue(int it, int y0, int bh, size_t tok, bool valid, int h,
                                         int qr, int lane, uint32_t tmem, uint8_t* smem,
                                         const CUtensorMap* tm_out, const BxParams& P,
                                         const tc::Abort& abort_flag) {
  const unsigned full = 0xffffffffu;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + BxCfg::OFF_BAR);
  const int warp = 2 + 4 * h + ((qr + 2) & 3);  // the warp of (h, qr): lane quarter = warp % 4
  const uint32_t lb = (uint32_t)(32 * qr) << 16;
  const int ob = it & 1, par = (it >> 1) & 1;
  // the row's 32 elements of q or k, in flight while the accumulator completes
  uint4 src[4] = {};
  if (KIND != BX_DV && valid) {
    const uint4* s = reinterpret_cast<const uint4*>(P.dot_src + tok * 128 + 32 * h);
#pragma unroll
    for (int i = 0; i < 4; ++i) src[i] = s[i];
  }
  if (!__all_sync(full, tc::mbar_wait(&bar[Y_OF0 + ob], par, abort_flag))) return false;
  tc::tc_fence_after();
  uint32_t o[32];
  tc::tmem_ld32_async(tmem + 256 + ob * 128 + lb + 32 * h, o);
  tc::tmem_wait_ld(o);
  tc::tc_fence_before();
  tc::mbar_arrive(&bar[Y_OE0 + ob]);
  const float fin = KIND == BX_DV ? 1.f : P.scale;
  // the output first (its stores need nothing else), while the q / k loads land
  uint8_t* stg = smem + BxCfg::OFF_STG + (warp - 2) * BxCfg::STG_WARP;
  const uint32_t astg = tc::smem_u32(stg);
#pragma unroll
  for (int rnd = 0; rnd < 2; ++rnd) {
    if (lane == 0) tc::bulk_wait_read_all();  // the slot's previous store has read it
    __syncwarp();
    if ((lane >> 4) == rnd) {
      // row r of the box (64 bytes), its 16-byte chunk c at chunk c ^ ((r >> 1) & 3): the
      // 64-byte swizzle of the output tensor map
      const int r = lane & 15;
      const uint32_t sw = (uint32_t)(r >> 1) & 3u;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t* v = &o[8 * c];
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(astg + r * 64 + ((c ^ sw) << 4)),
                     "r"(tc::pack_bf16(__uint_as_float(v[0]) * fin, __uint_as_float(v[1]) * fin)),
                     "r"(tc::pack_bf16(__uint_as_float(v[2]) * fin, __uint_as_float(v[3]) * fin)),
                     "r"(tc::pack_bf16(__uint_as_float(v[4]) * fin, __uint_as_float(v[5]) * fin)),
                     "r"(tc::pack_bf16(__uint_as_float(v[6]) * fin, __uint_as_float(v[7]) * fin))
                     : "memory");
      }
      tc::fence_proxy_async_smem();
    }
    __syncwarp();
    if (lane == 0) {
      tc::tma_store_3d(tm_out, stg, 32 * h, y0 + 16 * rnd, bh);
      tc::bulk_commit_group();
    }
  }
  if (KIND != BX_DV) {
    float dot = 0.f;
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {
      const uint32_t sw[4] = {src[c4].x, src[c4].y, src[c4].z, src[c4].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 s2 = *reinterpret_cast<const __nv_bfloat162*>(&sw[e]);
        dot = fmaf(__bfloat162float(s2.x), __uint_as_float(o[8 * c4 + 2 * e]) * fin, dot);
        dot = fmaf(__bfloat162float(s2.y), __uint_as_float(o[8 * c4 + 2 * e + 1]) * fin, dot);
      }
    }
    // this column block's share, in its own plane; the gate-gradient kernels add the four
    // planes in block order
    if (valid) P.pdot[(size_t)h * P.pdot_stride + tok] = dot;
  }
  return true;
}

template <int KIND, bool EXPV>
__global__ void __launch_bounds__(kBxThreads, 1) intra_bwd_xl_kernel(
    const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
    const __grid_constant__ CUtensorMap tm_e, const __grid_constant__ CUtensorMap tm_ghi,
    const __grid_constant__ CUtensorMap tm_glo, const __grid_constant__ CUtensorMap tm_out,
    const BxParams P) {
  using Cfg = BxCfg;
  constexpr int NA = Cfg::NA, NB = Cfg::NB, NE = Cfg::NE;
  const tc::Abort abort_flag{&g_tc_bwd_xl_error, P.epoch};
  // an earlier CTA gave up: the whole block leaves together
  if (__syncthreads_or(threadIdx.x == 0 && abort_flag.raised())) return;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_TMEM);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < Y_COUNT; ++i) {
      uint32_t cnt = 1;
      if (i == Y_AE0 || i == Y_AE0 + 1) cnt = kBxTransform + 1;
      if ((i >= Y_PF0 && i < Y_PF0 + 2) || (i >= Y_IR0 && i < Y_IR0 + 2) ||
          (i >= Y_OE0 && i < Y_OE0 + 2))
        cnt = kBxTransform;
      tc::mbar_init(&bar[i], cnt);
    }
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp == 0) {
    // ------------------------------------------------------------ A / B / state producer
    // B entries of an item, in the order the MMA thread consumes them: the first partner
    // tile, the two state planes (when a state product enters), the other partner tiles.
    const unsigned full = 0xffffffffu;
    const bool leader = lane == 0;
    if (leader) {
      tc::prefetch_tmap(&tm_a);
      tc::prefetch_tmap(&tm_b);
      tc::prefetch_tmap(&tm_ghi);
      tc::prefetch_tmap(&tm_glo);
    }
    int it = 0, gb = 0;
    uint32_t na = 0;  // row-tile fills issued
    for (int k = bx_first(); k < P.total && ok; k = bx_succ(k)) {
      BxItem I;
      if (!bx_item<KIND>(k, P, I)) continue;
      const int ia = it % NA;
      ok = __all_sync(full, tc::mbar_wait(&bar[Y_AE0 + ia], ((it / NA) & 1) ^ 1, abort_flag));
      if (!ok) break;
      const float* tb = P.tab + ((size_t)I.bh * P.NC + I.c) * P.tstride;
      if (leader) {
        uint64_t* af = &bar[Y_AF0 + ia];
        uint8_t* sa = smem + Cfg::OFF_A + ia * Cfg::TILE;
        uint8_t* rp = smem + Cfg::OFF_ROW + ia * Cfg::ROWAUX;
        const int L = P.L;
        if (KIND == BX_DQ) {
          tc::mbar_arrive_expect_tx(af, Cfg::TILE + 2048);
          tc::bulk_load(rp, tb + I.t0, 512, af);                 // QX
          tc::bulk_load(rp + 512, tb + L + I.t0, 512, af);       // QE
          tc::bulk_load(rp + 1024, tb + 4 * L + I.t0, 512, af);  // RQ
          tc::bulk_load(rp + 1536, tb + 5 * L + I.t0, 512, af);  // RV
        } else {
          tc::mbar_arrive_expect_tx(af, Cfg::TILE + 1552);
          tc::bulk_load(rp, tb + 2 * L + I.t0, 512, af);              // KX
          tc::bulk_load(rp + 512, tb + 3 * L + I.t0, 512, af);        // KG
          tc::bulk_load(rp + 1024, tb + 6 * L + I.t0, 512, af);       // RK
          tc::bulk_load(rp + 2048, tb + 7 * L + I.t0 / 32, 16, af);   // KM of the four row blocks
        }
        for (int kb = 0; kb < 2; ++kb)
          tc::tma_load_3d(sa + kb * 16384, &tm_a, af, kb * 64, I.c * P.L + I.t0, I.bh);
      }
      ++na;
      const int nent = I.np + (I.inter ? 2 : 0);
      for (int e = 0; e < nent && ok; ++e, ++gb) {
        const int st = gb % NB;
        ok = __all_sync(full, tc::mbar_wait(&bar[Y_BE0 + st], ((gb / NB) & 1) ^ 1, abort_flag));
        if (!ok) break;
        if (leader) {
          uint64_t* bf = &bar[Y_BF0 + st];
          uint8_t* sb = smem + Cfg::OFF_B + st * Cfg::TILE;
          tc::mbar_arrive_expect_tx(bf, Cfg::TILE);
          if (I.inter && (e == 1 || e == 2)) {
            const CUtensorMap* tg = e == 1 ? &tm_ghi : &tm_glo;
            for (int kb = 0; kb < 2; ++kb)
              tc::tma_load_3d(sb + kb * 16384, tg, bf, kb * 64, 0, I.bh * P.NC + I.c);
          } else {
            const int s = (I.inter && e > 2) ? e - 2 : e;  // partner step
            const int j = I.p0 + s;
            for (int kb = 0; kb < 2; ++kb)
              tc::tma_load_3d(sb + kb * 16384, &tm_b, bf, kb * 64, I.c * P.L + j * 128, I.bh);
          }
        }
      }
      ++it;
    }
    // gave up: the copies this warp issued land before the CTA exits
    if (!ok && leader) {
      tc::drain_ring(&bar[Y_AF0], NA, na);
      tc::drain_ring(&bar[Y_BF0], NB, (uint32_t)gb);
    }
  } else if (warp == kBxEWarp) {
    // ------------------------------------------------------------ E producer
    const unsigned full = 0xffffffffu;
    const bool leader = lane == 0;
    if (leader) tc::prefetch_tmap(&tm_e);
    int ge = 0;
    for (int k = bx_first(); k < P.total && ok; k = bx_succ(k)) {
      BxItem I;
      if (!bx_item<KIND>(k, P, I)) continue;
      const float* tb = P.tab + ((size_t)I.bh * P.NC + I.c) * P.tstride;
      for (int s = 0; s < I.np && ok; ++s, ++ge) {
        const int st = ge % NE;
        ok = __all_sync(full, tc::mbar_wait(&bar[Y_EE0 + st], ((ge / NE) & 1) ^ 1, abort_flag));
        if (!ok) break;
        if (leader) {
          const int j = I.p0 + s, L = P.L;
          uint64_t* ef = &bar[Y_EF0 + st];
          uint8_t* se = smem + Cfg::OFF_E + st * Cfg::TILE;
          uint8_t* cp = smem + Cfg::OFF_COL + st * Cfg::COLAUX;
          if (KIND == BX_DQ) {
            tc::mbar_arrive_expect_tx(ef, Cfg::TILE + 1040);
            tc::bulk_load(cp, tb + 2 * L + j * 128, 512, ef);        // KX
            tc::bulk_load(cp + 512, tb + 3 * L + j * 128, 512, ef);  // KG
            tc::bulk_load(cp + 1536, tb + 7 * L + j * 4, 16, ef);    // KM
          } else if (KIND == BX_DK) {
            tc::mbar_arrive_expect_tx(ef, Cfg::TILE + 1024);
            tc::bulk_load(cp, tb + j * 128, 512, ef);              // QX
            tc::bulk_load(cp + 512, tb + L + j * 128, 512, ef);    // QE
          } else {
            tc::mbar_arrive_expect_tx(ef, Cfg::TILE + 512);
            tc::bulk_load(cp, tb + j * 128, 512, ef);  // QX
          }
          for (int eb = 0; eb < 2; ++eb)
            tc::tma_load_3d(se + eb * 16384, &tm_e, ef, eb * 64, I.c * P.L + j * 128, I.bh);
        }
      }
    }
    if (!ok && leader) tc::drain_ring(&bar[Y_EF0], NE, (uint32_t)ge);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Lane 0 alone walks the schedule, waits and issues; the shared-memory descriptors
    // are built once and advanced by constant offsets (address / 16 in the low 14
    // bits, and no offset reaches past the 227 KB of shared memory).
    if (lane == 0) {
      constexpr uint32_t idS = tc::idesc_bf16(128, 128, false, false);
      constexpr uint32_t idAcc = tc::idesc_bf16(128, 128, false, true);
      constexpr uint32_t idG = tc::idesc_bf16(128, 128, false, KIND == BX_DV);
      const uint32_t aA0 = tc::smem_u32(smem + Cfg::OFF_A), aB0 = tc::smem_u32(smem + Cfg::OFF_B),
                     aE0 = tc::smem_u32(smem + Cfg::OFF_E);
      const uint64_t dA0 = tc::sdesc_sw128(aA0, 16, 1024), dB0 = tc::sdesc_sw128(aB0, 16, 1024),
                     dBmn0 = tc::sdesc_sw128(aB0, 16384, 1024), dE0 = tc::sdesc_sw128(aE0, 16384, 1024);
      // K-major k-step offset (16 contraction columns): within a 64-column block 32 bytes,
      // then the next block
      auto koff = [](int k) -> uint64_t { return (uint64_t)((((k >> 2) * 16384) + (k & 3) * 32) >> 4); };

      // score of partner step s (global step gs, B entry gb): X = A B^T, then the B stage is free
      auto issue_s = [&](int it, int s, int gs, int gb) -> bool {
        const int sb = gs & 1, ia = it % NA, st = gb % NB;
        if (s == 0 && !tc::mbar_wait(&bar[Y_AF0 + ia], (it / NA) & 1, abort_flag)) return false;
        if (!tc::mbar_wait(&bar[Y_BF0 + st], (gb / NB) & 1, abort_flag)) return false;
        tc::tc_fence_after();
        const uint64_t dA = dA0 + (uint64_t)((ia * Cfg::TILE) >> 4),
                       dB = dB0 + (uint64_t)((st * Cfg::TILE) >> 4);
#pragma unroll
        for (int k = 0; k < 8; ++k) tc::mma_bf16_ss(tmem + sb * 128, dA + koff(k), dB + koff(k), idS, k > 0);
        tc::tc_commit(&bar[Y_SF0 + sb]);
        tc::tc_commit(&bar[Y_BE0 + st]);
        return true;
      };
      // Items without a state product skip the inter handshake, so its barriers count
      // phases per accumulator buffer: nin[ob] = state products that buffer has had.
      int nin[2] = {0, 0};
      // the state product of item it into its accumulator (B entries gb, gb + 1: hi, lo)
      auto issue_inter = [&](int it, int gb) -> bool {
        const int ob = it & 1, ia = it % NA;
        const uint32_t tAcc = tmem + 256 + ob * 128;
        if (!tc::mbar_wait(&bar[Y_OE0 + ob], ((it >> 1) & 1) ^ 1, abort_flag)) return false;
        const uint64_t dA = dA0 + (uint64_t)((ia * Cfg::TILE) >> 4);
        for (int pl = 0; pl < 2; ++pl, ++gb) {
          const int st = gb % NB;
          if (!tc::mbar_wait(&bar[Y_BF0 + st], (gb / NB) & 1, abort_flag)) return false;
          tc::tc_fence_after();
          if (KIND == BX_DV) {  // G rows = contraction (d_qk), columns = output (d_hv)
            const uint64_t dG = dBmn0 + (uint64_t)((st * Cfg::TILE) >> 4);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              tc::mma_bf16_ss(tAcc, dA + koff(k), dG + (uint64_t)(k * 128), idG, pl > 0 || k > 0);
          } else {  // G rows = output (d_qk), columns = contraction (d_hv)
            const uint64_t dG = dB0 + (uint64_t)((st * Cfg::TILE) >> 4);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              tc::mma_bf16_ss(tAcc, dA + koff(k), dG + koff(k), idG, pl > 0 || k > 0);
          }
          tc::tc_commit(&bar[Y_BE0 + st]);
        }
        tc::tc_commit(&bar[Y_IF0 + ob]);
        ++nin[ob];
        return true;
      };
      // Acc += Y E of partner step s; Y is read from TMEM (packed bf16, partners 32 b ..
      // of block b at column 32 b); the transform threads saw E arrive before signalling Y
      auto issue_acc = [&](const BxItem& I, int it, int s, int gs) -> bool {
        const int sb = gs & 1, ob = it & 1, es = gs % NE;
        if (s == 0) {
          if (I.inter) {
            if (!tc::mbar_wait(&bar[Y_IR0 + ob], (nin[ob] - 1) & 1, abort_flag)) return false;
          } else {
            if (!tc::mbar_wait(&bar[Y_OE0 + ob], ((it >> 1) & 1) ^ 1, abort_flag)) return false;
          }
        }
        if (!tc::mbar_wait(&bar[Y_PF0 + sb], (gs >> 1) & 1, abort_flag)) return false;
        tc::tc_fence_after();
        const uint32_t tAcc = tmem + 256 + ob * 128, tY = tmem + sb * 128;
        const uint64_t dE = dE0 + (uint64_t)((es * Cfg::TILE) >> 4);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          tc::mma_bf16_ts(tAcc, tY + 32 * (k >> 1) + 8 * (k & 1), dE + (uint64_t)(k * 128), idAcc,
                          I.inter || s > 0 || k > 0);
        tc::tc_commit(&bar[Y_EE0 + es]);
        return true;
      };

      BxItem I, N;
      int k = bx_next<KIND>(bx_first(), P, I);
      int it = 0, gs = 0, gb = 0;
      if (k < P.total) ok = issue_s(0, 0, 0, gb++);
      while (k < P.total && ok) {
        const int kn = bx_next<KIND>(bx_succ(k), P, N);
        if (I.inter) {
          ok = issue_inter(it, gb);
          gb += 2;
        }
        for (int s = 0; s < I.np && ok; ++s, ++gs) {
          const bool last = s + 1 == I.np;
          // the next score goes before this step's accumulate
          if (!last) ok = issue_s(it, s + 1, gs + 1, gb++);
          else if (kn < P.total) ok = issue_s(it + 1, 0, gs + 1, gb++);
          if (!ok) break;
          ok = issue_acc(I, it, s, gs);
          if (!ok) break;
          if (last) {
            tc::tc_commit(&bar[Y_AE0 + it % NA]);
            tc::tc_commit(&bar[Y_OF0 + (it & 1)]);
          }
        }
        ++it;
        k = kn;
        I = N;
      }
      if (!ok) tc::drain_mma(&bar[Y_DRAIN]);  // no product still writes TMEM or reads smem
    }
  } else {
    // ------------------------------------------------------------ gate transform + epilogue
    const int h = (warp - 2) >> 2;  // this warpgroup's 32-partner block (and 32 output columns)
    const int qr = warp & 3;        // TMEM lane quarter = 32-row block of the tile
    const int row = 32 * qr + lane;
    const uint32_t lb = (uint32_t)(32 * qr) << 16;
    const unsigned full = 0xffffffffu;
    float* fwb = reinterpret_cast<float*>(smem + Cfg::OFF_FW) + (warp - 2) * 32;
    int it = 0, gs = 0;
    int nin[2] = {0, 0};  // state products per accumulator buffer so far (inter barrier phases)

    struct Pending {
      int it, y0, bh;
      size_t tok;
      bool valid;
    } pe{};
    bool pend = false;
    auto epilogue = [&](const Pending& e) -> bool {
      return bx_epilogue<KIND>(e.it, e.y0, e.bh, e.tok, e.valid, h, qr, lane, tmem, smem, &tm_out, P,
                               abort_flag);
    };

    for (int k = bx_first(); k < P.total && ok; k = bx_succ(k)) {
      BxItem I;
      if (!bx_item<KIND>(k, P, I)) continue;
      // the row's q (dq) or k (dk), read by this item's epilogue one item from now
      if (KIND != BX_DV && I.t0 + row < I.len)
        tc::prefetch_l2(P.dot_src + ((size_t)I.bh * P.T + (size_t)I.c * P.L + I.t0 + row) * 128 + 32 * h);
      const int ia = it % NA, ob = it & 1;
      ok = __all_sync(full, tc::mbar_wait(&bar[Y_AF0 + ia], (it / NA) & 1, abort_flag));
      if (!ok) break;
      const float* rp = reinterpret_cast<const float*>(smem + Cfg::OFF_ROW + ia * Cfg::ROWAUX);
      // row factors: dq (query rows) QX, QE; dk, dv (key rows) KX, KG and the row block's KM
      const float R = rp[row], F = rp[128 + row];
      const float Mrow = KIND == BX_DQ ? 0.f : rp[512 + qr];
      if (I.inter) {
        // Acc = rs_t (A G)_t + rvc_t rowvec, rescaled in TMEM before the first accumulate
        float rs = rp[256 + row], rvc = 0.f;
        if (KIND == BX_DQ) rvc = rp[384 + row];
        if (KIND == BX_DK) {
          rs /= P.scale;  // the epilogue multiplies the whole row by 1/sqrt(d_qk)
          rvc = rs;
        }
        ok = __all_sync(full, tc::mbar_wait(&bar[Y_IF0 + ob], nin[ob] & 1, abort_flag));
        if (!ok) break;
        ++nin[ob];
        tc::tc_fence_after();
        const uint32_t tAcc = tmem + 256 + ob * 128 + lb + 32 * h;
        uint32_t v[32];
        tc::tmem_ld32_async(tAcc, v);
        tc::tmem_wait_ld(v);
        if (KIND != BX_DV && EXPV) {
          const float4* rv = reinterpret_cast<const float4*>(
              P.rowvec + ((size_t)I.bh * P.NC + I.c) * 128 + 32 * h);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 r4 = rv[i];
            v[4 * i] = __float_as_uint(fmaf(rs, __uint_as_float(v[4 * i]), rvc * r4.x));
            v[4 * i + 1] = __float_as_uint(fmaf(rs, __uint_as_float(v[4 * i + 1]), rvc * r4.y));
            v[4 * i + 2] = __float_as_uint(fmaf(rs, __uint_as_float(v[4 * i + 2]), rvc * r4.z));
            v[4 * i + 3] = __float_as_uint(fmaf(rs, __uint_as_float(v[4 * i + 3]), rvc * r4.w));
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(rs * __uint_as_float(v[i]));
        }
        tc::tmem_st32_async(tAcc, v);
        tc::tmem_wait_st();
        tc::tc_fence_before();
        tc::mbar_arrive(&bar[Y_IR0 + ob]);
      }
      for (int s = 0; s < I.np && ok; ++s, ++gs) {
        const int sb = gs & 1, es = gs % NE;
        ok = __all_sync(full, tc::mbar_wait(&bar[Y_SF0 + sb], (gs >> 1) & 1, abort_flag));
        if (!ok) break;
        // the partner tile's gate factors; seeing them also tells the MMA thread
        // (through Y) that E has landed
        ok = __all_sync(full, tc::mbar_wait(&bar[Y_EF0 + es], (gs / NE) & 1, abort_flag));
        if (!ok) break;
        tc::tc_fence_after();
        const float* cp = reinterpret_cast<const float*>(smem + Cfg::OFF_COL + es * Cfg::COLAUX);
        const uint32_t tS = tmem + sb * 128 + lb + 32 * h;
        const bool diag = I.p0 + s == I.rt;
        // this block against the row block on the diagonal tile: dq keeps partners <= row
        // (blocks h < qr whole), dk and dv partners >= row (blocks h > qr whole)
        const bool whole = !diag || (KIND == BX_DQ ? h < qr : h > qr);
        const bool own = diag && h == qr;
        uint32_t sv[32];
        tc::tmem_ld32_async(tS, sv);
        if (KIND != BX_DQ && whole) {
          // partner factors 2^(QX_t + KM) of this block for the row block's KM, one per lane
          const float qx = cp[32 * h + lane];
          const float fw = tc::ex2(qx + Mrow + (KIND == BX_DV ? P.log2_scale : 0.f));
          __syncwarp();
          fwb[lane] = fw;
          __syncwarp();
        }
        tc::tmem_wait_ld(sv);
        uint32_t w[16];
        if (whole) {
          // separable: y = ((x + e_t) f) g in the same fp32 operations in dq and dk
          if (KIND == BX_DQ) {
            const float f = tc::ex2(R + cp[384 + h]);
            const uint64_t e2 = tc::f2_make(F, F), f2 = tc::f2_make(f, f);
            const float* kg = cp + 128 + 32 * h;
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              const float4 g4 = *reinterpret_cast<const float4*>(kg + e);
              const uint64_t y0 = tc::f2_mul(
                  tc::f2_mul(tc::f2_add(tc::f2_make(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), e2), f2),
                  tc::f2_make(g4.x, g4.y));
              const uint64_t y1 = tc::f2_mul(
                  tc::f2_mul(tc::f2_add(tc::f2_make(__uint_as_float(sv[e + 2]), __uint_as_float(sv[e + 3])), e2), f2),
                  tc::f2_make(g4.z, g4.w));
              const float2 a0 = tc::f2_split(y0), a1 = tc::f2_split(y1);
              w[e / 2] = tc::pack_bf16(a0.x, a0.y);
              w[e / 2 + 1] = tc::pack_bf16(a1.x, a1.y);
            }
          } else {
            const uint64_t g2 = tc::f2_make(F, F);
            const float* qe = cp + 128 + 32 * h;
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              const float4 f4 = *reinterpret_cast<const float4*>(fwb + e);
              uint64_t x0 = tc::f2_make(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1]));
              uint64_t x1 = tc::f2_make(__uint_as_float(sv[e + 2]), __uint_as_float(sv[e + 3]));
              if (KIND == BX_DK) {
                const float4 e4 = *reinterpret_cast<const float4*>(qe + e);
                x0 = tc::f2_add(x0, tc::f2_make(e4.x, e4.y));
                x1 = tc::f2_add(x1, tc::f2_make(e4.z, e4.w));
              }
              const uint64_t y0 = tc::f2_mul(tc::f2_mul(x0, tc::f2_make(f4.x, f4.y)), g2);
              const uint64_t y1 = tc::f2_mul(tc::f2_mul(x1, tc::f2_make(f4.z, f4.w)), g2);
              const float2 a0 = tc::f2_split(y0), a1 = tc::f2_split(y1);
              w[e / 2] = tc::pack_bf16(a0.x, a0.y);
              w[e / 2 + 1] = tc::pack_bf16(a1.x, a1.y);
            }
          }
        } else if (own) {
          // the block holding this row: each element's own exponent and the causal mask
          // (t-side term first, then the s-side term, in every kernel)
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float y[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int p = 32 * h + e + u;
              const float x = __uint_as_float(sv[e + u]);
              float val;
              bool keep;
              if (KIND == BX_DQ) {
                val = (x + F) * tc::ex2(R + cp[p]);
                keep = p <= row;
              } else if (KIND == BX_DK) {
                val = (x + cp[128 + p]) * tc::ex2(cp[p] + R);
                keep = p >= row;
              } else {
                val = x * tc::ex2(cp[p] + R + P.log2_scale);
                keep = p >= row;
              }
              y[u] = keep ? val : 0.f;
            }
            w[e / 2] = tc::pack_bf16(y[0], y[1]);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) w[e] = 0u;
        }
        // packed into the first 16 of this block's own 32 columns
        tc::tmem_st16_async(tS, w);
        tc::tmem_wait_st();
        tc::tc_fence_before();
        tc::mbar_arrive(&bar[Y_PF0 + sb]);
        if (s == 0) {
          tc::mbar_arrive(&bar[Y_AE0 + ia]);
          if (pend) {
            ok = epilogue(pe);
            pend = false;
          }
        }
      }
      if (!ok) break;
      pe.it = it;
      pe.y0 = I.c * P.L + I.t0 + 32 * qr;
      pe.bh = I.bh;
      pe.tok = (size_t)I.bh * P.T + (size_t)I.c * P.L + I.t0 + row;
      pe.valid = I.t0 + row < I.len;
      pend = true;
      ++it;
    }
    if (ok && pend) ok = epilogue(pe);
    if (lane == 0) tc::bulk_wait_all();  // the output stores have read the staging slot
  }

  if (!ok) abort_flag.raise();
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

// Per-chunk gate table of the large-chunk backward (layout in internal.h), from
// the forward's gate arrays and the backward's 1 / den_t and da_t.  One CTA per
// head; one warp per block of 32 tokens, so a block maximum is a warp maximum.
template <bool EXPV>
__global__ void __launch_bounds__(256) bwd_xl_table_kernel(
    const float* __restrict__ b, const float* __restrict__ li, const float* __restrict__ m,
    const float* __restrict__ inv_den, const float* __restrict__ da, float* __restrict__ tab, int T,
    int L, int NC, bool has_init, const float* __restrict__ m0) {
  const int bh = blockIdx.x;
  const size_t base = (size_t)bh * T;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  const int stride = bwd_xl_table_stride(L), bpc = L / 32;
  for (int blk = warp; blk < NC * bpc; blk += nwarps) {
    const int c = blk / bpc, r = (blk % bpc) * 32 + lane;
    const int t = c * L + r;
    const bool valid = t < T;
    float qx = -INFINITY, qe = 0.f, kx = -INFINITY, rq = 0.f, rv = 0.f, rk = 0.f;
    if (valid) {
      const float bt = b[base + t], lit = li[base + t];
      const float mt = EXPV ? m[base + t] : 0.f;
      const float invd = inv_den[base + t];
      const float dat = EXPV ? da[base + t] : 0.f;
      qx = (bt - mt) * kLog2e + log2f(invd);
      qe = dat / invd;
      kx = (lit - bt) * kLog2e;
      if (c > 0 || has_init) {
        const float mprev = EXPV ? chunk_mprev(m, base + (size_t)c * L, c, m0, bh) : 0.f;
        const float alpha = expf(bt + mprev - mt);
        rq = alpha * invd;
        rv = alpha * dat;
      }
      const size_t last = base + (size_t)c * L + (min(L, T - c * L) - 1);
      rk = expf(b[last] - bt + lit - (EXPV ? m[last] : 0.f));
    }
    float km = warp_max(kx);
    if (km == -INFINITY) km = 0.f;  // a block wholly past the sequence end
    float* tb = tab + ((size_t)bh * NC + c) * (size_t)stride;
    tb[r] = qx;
    tb[L + r] = qe;
    tb[2 * L + r] = kx;
    tb[3 * L + r] = valid ? exp2f(kx - km) : 0.f;
    tb[4 * L + r] = rq;
    tb[5 * L + r] = rv;
    tb[6 * L + r] = rk;
    if (lane == 0) tb[7 * L + r / 32] = km;
  }
}

}  // namespace

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

bool intra_bwd_xl_supported(const Problem& p) {
  return p.bf16() && p.L >= 256 && p.dqk == 128 && p.dhv == 128;
}

cudaError_t launch_bwd_xl_table(const Problem& p, const BwdArgs& a, cudaStream_t s) {
  if (a.btab == nullptr) return cudaErrorInvalidValue;
  const float* m0 = (a.init.on() && p.exp_variant()) ? a.init.m : nullptr;
  if (p.exp_variant())
    bwd_xl_table_kernel<true><<<p.BH, 256, 0, s>>>(a.b, a.li, a.m, a.inv_den, a.da, a.btab, p.T, p.L,
                                                   p.NC, a.init.on(), m0);
  else
    bwd_xl_table_kernel<false><<<p.BH, 256, 0, s>>>(a.b, a.li, a.m, a.inv_den, a.da, a.btab, p.T,
                                                    p.L, p.NC, a.init.on(), m0);
  return cudaGetLastError();
}

template <int KIND, bool EXPV>
static cudaError_t launch_xl_kind(const Problem& p, const BwdArgs& a, cudaStream_t s) {
  if (a.btab == nullptr) return cudaErrorInvalidValue;
  const size_t plane = (size_t)p.BH * p.NC * p.dqk * p.dhv;
  const bf16* G = (const bf16*)(KIND == BX_DQ ? a.C : a.dC);
  const uint64_t BHNC = (uint64_t)p.BH * p.NC;
  const void *A, *B, *E;
  void* out;
  if (KIND == BX_DQ) {
    A = a.dh; B = a.v; E = a.k; out = a.dq;
  } else if (KIND == BX_DK) {
    A = a.v; B = a.dh; E = a.q; out = a.dk;
  } else {
    A = a.k; B = a.q; E = a.dh; out = a.dv;
  }
  CUtensorMap tA, tB, tE, tGh, tGl, tO;
  if (!make_tmap_3d_bf16(&tA, A, 128, p.T, p.BH, 64, 128) ||
      !make_tmap_3d_bf16(&tB, B, 128, p.T, p.BH, 64, 128) ||
      !make_tmap_3d_bf16(&tE, E, 128, p.T, p.BH, 64, 128) ||
      !make_tmap_3d_bf16(&tGh, G, 128, 128, BHNC, 64, 128) ||
      !make_tmap_3d_bf16(&tGl, G + plane, 128, 128, BHNC, 64, 128) ||
      !make_tmap_3d_bf16_rows(&tO, out, 128, p.T, p.BH, 32, 16))
    return cudaErrorInvalidValue;
  BxParams P;
  P.tab = a.btab;
  P.rowvec = KIND == BX_DQ ? a.n : a.dn;
  P.dot_src = (const bf16*)(KIND == BX_DQ ? a.q : a.k);
  P.pdot = KIND == BX_DQ ? a.pq : a.pk;
  P.pdot_stride = a.pdot_stride;
  if (a.pdot_planes != 4) return cudaErrorInvalidValue;
  P.T = p.T;
  P.L = p.L;
  P.NC = p.NC;
  P.BH = p.BH;
  P.ntq = p.L / 128;  // even: L >= 256 is a power of two
  P.tstride = bwd_xl_table_stride(p.L);
  P.init = a.init.on();
  P.dfin = a.dCT != nullptr;
  P.scale = p.scale;
  P.log2_scale = log2f(p.scale);
  const long long total = (long long)P.ntq * p.BH * p.NC;
  if (total >= (1LL << 30)) return cudaErrorInvalidValue;
  P.total = (int)total;
  P.epoch = next_epoch();
  const int smem = BxCfg::SMEM;
  auto kern = intra_bwd_xl_kernel<KIND, EXPV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, nsm = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const long long pairs = total / 2;
  const int grid = (int)(pairs < nsm ? pairs : nsm);
  kern<<<grid, kBxThreads, smem, s>>>(tA, tB, tE, tGh, tGl, tO, P);
  return cudaGetLastError();
}

cudaError_t launch_dq_xl(const Problem& p, const BwdArgs& a, cudaStream_t s) {
  return p.exp_variant() ? launch_xl_kind<BX_DQ, true>(p, a, s) : launch_xl_kind<BX_DQ, false>(p, a, s);
}
cudaError_t launch_dk_xl(const Problem& p, const BwdArgs& a, cudaStream_t s) {
  return p.exp_variant() ? launch_xl_kind<BX_DK, true>(p, a, s) : launch_xl_kind<BX_DK, false>(p, a, s);
}
cudaError_t launch_dv_xl(const Problem& p, const BwdArgs& a, cudaStream_t s) {
  return p.exp_variant() ? launch_xl_kind<BX_DV, true>(p, a, s) : launch_xl_kind<BX_DV, false>(p, a, s);
}

cudaError_t fetch_tc_bwd_xl_error(unsigned int* flag) {
  return cudaMemcpyFromSymbol(flag, g_tc_bwd_xl_error, sizeof(unsigned int));
}

}  // namespace mlstm
