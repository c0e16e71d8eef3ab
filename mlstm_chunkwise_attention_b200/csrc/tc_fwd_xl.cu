// TFLA intra-chunk output kernel for large chunks (chunk >= 256): the second
// level of tiling walks 128-token key tiles inside the chunk ("Tiled Flash
// Linear Attention: More Efficient Linear RNN and xLSTM Kernels", TFLA summary
// page, Approach; arXiv abstract page, Abstract).  Same mathematics as the
// chunk-128 kernel (tc_fwd.cu):
//   S_j = Q K_j^T;  P_ts = S_ts D_ts / sqrt(d_qk),  D_ts = exp(b_t - b_s + log i_s - m_t) (s <= t)
//   O  = (alpha_t Q / sqrt(d_qk)) C_prev + sum_j P_j V_j;   h_t = O_t / den_t.
//
// Organisation (one persistent CTA per SM, work items = (query tile, head,
// chunk, value block), taken in balanced pairs of query tiles):
//  * warp 0 streams Q tiles (double-buffered) and, per step, K_j or the
//    chunk's entering state C_prev through a ring whose stages free as soon
//    as their score product is done; warp 18 streams V_j with the key
//    tile's gate factors through a second ring (TMA and bulk copies, no
//    multicast);
//  * warp 1 (lane 0 alone) issues tcgen05.mma: S_{g+1} before P_g V_g, so the tensor core
//    computes the next score tile while the gate transform runs;
//  * warps 2-17 (four warpgroups, one per 32-key block of a tile; four
//    warps per SM sub-partition, so the latency of one warp's TMEM traffic
//    and exp2 is hidden by the others) turn S into P in TMEM in place (bf16,
//    two per column, each block packed into the first half of its own 32
//    columns, which no other warp reads), and P V reads P straight from
//    TMEM.  The inter-chunk term is one more step of the same kind: the
//    transform writes alpha_t q_t / sqrt(d_qk) into the S buffer and the
//    tensor core multiplies it by C_prev, so it lands in the same
//    accumulator O;
//  * O is double-buffered in TMEM; the epilogue of an item (normalise,
//    store h) runs after the first step of the next item.
// Gate factors come from per-chunk tables written by gate_prep: off-diagonal
// 32-key blocks use the separable form exp2(R_t + MU) * KP_s (one exp per row
// and block), the diagonal block of the diagonal tile the per-element
// exp2(R_t + CC_s) with the causal mask, and blocks above the diagonal are 0.
#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace mlstm {

static __device__ unsigned int g_tc_fwd_xl_error;

namespace {

template <int DQK, int DV>
struct XlCfg {
  static constexpr int KB = DQK / 64, VB = DV / 64;
  static constexpr int NQ = DQK <= 128 ? 2 : 1;  // Q buffers
  // K ring (K tiles, and C_prev for the inter-chunk step); V ring (V tiles,
  // each with its key tile's gate factors)
  static constexpr int NK = DQK == 64 ? 4 : (DQK == 128 ? 2 : 1);
  static constexpr int NV = DQK == 64 ? (DV == 64 ? 4 : 3) : (DQK == 128 ? (DV == 64 ? 4 : 2) : 2);
  // the next S is issued before the current P V when the next Q and K can be resident
  static constexpr bool LOOK = NQ == 2 && NK >= 2;
  static constexpr int Q_BYTES = KB * 16384;
  static constexpr int K_BYTES = KB * 16384;
  static constexpr int V_BYTES = VB * 16384;
  static constexpr int C_BYTES = VB * DQK * 128;
  static constexpr int ROWAUX = 3 * 512 + DQK * 4;  // R, QF, FL of 128 rows; n_{c-1}
  static constexpr int COLAUX = 1040;               // CC, KP of 128 keys; 4 block maxima
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NQ * Q_BYTES;
  static constexpr int OFF_V = OFF_K + NK * K_BYTES;
  static constexpr int OFF_ROW = OFF_V + NV * V_BYTES;
  static constexpr int OFF_COL = OFF_ROW + NQ * ROWAUX;
  // normaliser shares [4 items][4 key blocks][128 rows] floats: an item's shares are written
  // when its last step ends and read by its epilogue one item later; four slots keep a slot
  // from being rewritten while any warp may still read it, however short the items
  static constexpr int OFF_XS = OFF_COL + NV * COLAUX;
  // per transform warp: 16 rows of h (DV / 4 bf16 each), 1024-byte aligned for the swizzle
  static constexpr int OFF_STG = (OFF_XS + 4 * 4 * 128 * 4 + 1023) & ~1023;
  static constexpr int STG_WARP = 8 * DV;
  static constexpr int OFF_BAR = OFF_STG + 16 * STG_WARP;
  static constexpr int OFF_TMEM = OFF_BAR + 64 * 8;
  static constexpr int SMEM = OFF_TMEM + 16 + 1024;  // + alignment slack
  static constexpr uint32_t TMEM_COLS = 512;         // S0 [0,128) S1 [128,256) O0, O1 from 256
  static_assert(C_BYTES <= K_BYTES, "C_prev must fit one K stage");
  static_assert(NK <= 4 && NV <= 8, "barrier slots");
  static_assert(256 + 2 * DV <= 512, "two O buffers must fit TMEM");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

enum {
  X_QF0 = 0,   // Q (+ row factors) full, per Q buffer
  X_QE0 = 2,   // Q buffer free: MMA commit + the 512 transform threads
  X_KF0 = 4,   // K stage full (K tile or C_prev)
  X_KE0 = 8,   // K stage free (MMA commit after the S or inter-chunk product)
  X_VF0 = 12,  // V stage full (V tile + its key tile's gate factors)
  X_VE0 = 20,  // V stage free (MMA commit after P V)
  X_SF0 = 28,  // S buffer written (MMA commit), per S buffer
  X_PF0 = 30,  // P written (512 threads, each having seen its step's V / C_prev), per S buffer
  X_OF0 = 34,  // O complete (MMA commit), per O buffer
  X_OE0 = 36,  // O read out (512 threads), per O buffer
  X_XS0 = 38,  // normaliser shares written (128 threads), per item slot (it % 4) and lane quarter
  X_DRAIN = 54,  // the MMA thread's last commit when it gives up
  X_COUNT = 55
};

constexpr int kXlThreads = 608;    // K producer, MMA, 16 transform warps, V producer
constexpr int kXlTransform = 512;  // transform threads (warps 2..17)
constexpr int kXlVWarp = 18;       // V producer warp

struct XlItem {
  int qt, bh, c, vb, t0, len, nkv;
  bool pseudo;  // a state enters the chunk: it has a C_prev step (c > 0, or an initial state)
};

// Work items come in pairs: query tiles ntq-1-p and p of one (head, chunk,
// value block), so every pair holds ntq + 1 key tiles and a static split of
// pairs over the CTAs is balanced.  Pair index fastest varies the pair inside
// a chunk, so the CTAs running at one time cover few chunks and their K / V
// tiles stay in L2 for every query tile that reads them.  Item k is half k & 1
// of pair k >> 1; a CTA walks pairs blockIdx.x, blockIdx.x + gridDim.x, ...
__device__ __forceinline__ bool xl_item(int k, int BH, int NC, int NVB, int ntq, int T, int L,
                                        bool init, XlItem& it) {
  const int half_ntq = ntq >> 1;
  int r = k >> 1;
  const int pi = r % half_ntq;
  r /= half_ntq;
  it.vb = r % NVB;
  r /= NVB;
  it.c = r % NC;
  it.bh = r / NC;
  it.qt = (k & 1) ? pi : ntq - 1 - pi;
  it.t0 = it.qt * 128;
  it.len = min(L, T - it.c * L);
  it.nkv = it.qt + 1;
  it.pseudo = it.c > 0 || init;
  return it.t0 < it.len;
}

__device__ __forceinline__ int xl_first() { return 2 * blockIdx.x; }
__device__ __forceinline__ int xl_succ(int k) { return (k & 1) ? k + 2 * gridDim.x - 1 : k + 1; }

__device__ __forceinline__ int xl_next(int k, int total, int BH, int NC, int NVB, int ntq, int T,
                                       int L, bool init, XlItem& it) {
  for (; k < total; k = xl_succ(k))
    if (xl_item(k, BH, NC, NVB, ntq, T, L, init, it)) return k;
  return total;
}

}  // namespace

// Epilogue of one work item for the transform thread of row 32 qr + lane and
// column quarter h (DV / 4 columns): for mLSTMexp the normaliser a_t (the
// four key blocks' shares, exchanged among the four warps of this TMEM lane
// quarter only) and 1 / den_t; then O is read out of TMEM, freeing it for the
// next items' products, and h leaves through this warp's staging slot, 16
// rows at a time, by TMA stores (the TMA unit clips rows past the sequence
// end), so the stores cost the load/store unit nothing.  Kept out of line so
// its registers do not count against the gate transform it is called from.
template <int DQK, int DV, bool EXPV>
__device__ __noinline__ bool xl_epilogue(int it, int vb, int y0, int bh, size_t tok, bool valid,
                                         float fl, int h, int qr, int lane, uint32_t tmem,
                                         uint8_t* smem, const CUtensorMap* tm_h,
                                         float* __restrict__ abar_out, const tc::Abort& abort_flag) {
  using Cfg = XlCfg<DQK, DV>;
  const unsigned full = 0xffffffffu;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  const int warp = 2 + 4 * h + ((qr + 2) & 3);  // the warp of (h, qr): lane quarter = warp % 4
  const int row = 32 * qr + lane;
  const uint32_t lb = (uint32_t)(32 * qr) << 16;
  const int ob = it & 1, par = (it >> 1) & 1;
  float inv = 1.f;
  if (EXPV) {
    // den_t = max(|a_t|, exp(-m_t)), a_t added in block order so the four threads of a row
    // agree; the four key blocks' shares were written when the item's last step ended
    const int xsl = it & 3;
    float* x = reinterpret_cast<float*>(smem + Cfg::OFF_XS) + xsl * 512;
    uint64_t* xb = &bar[X_XS0 + 4 * xsl + qr];
    if (!__all_sync(full, tc::mbar_wait(xb, (it >> 2) & 1, abort_flag))) return false;
    const float a = ((x[row] + x[128 + row]) + x[256 + row]) + x[384 + row];
    inv = 1.f / fmaxf(fabsf(a), fl);
    if (h == 0 && vb == 0 && valid) abar_out[tok] = a;
  }
  if (!__all_sync(full, tc::mbar_wait(&bar[X_OF0 + ob], par, abort_flag))) return false;
  tc::tc_fence_after();
  const uint32_t tO = tmem + 256 + ob * DV + lb + h * (DV / 4);
  constexpr int CPR = DV / 32;  // 16-byte chunks of this thread's DV / 4 columns
  uint4 w[CPR];
  {
    uint32_t o[32];
    if (DV >= 128) {
      tc::tmem_ld32_async(tO, o);
      tc::tmem_wait_ld(o);
    } else {
      tc::tmem_ld16(tO, o);
    }
    tc::tc_fence_before();
    tc::mbar_arrive(&bar[X_OE0 + ob]);
#pragma unroll
    for (int c4 = 0; c4 < CPR; ++c4) {
      const uint32_t* r = &o[8 * c4];
      uint4& d = w[c4];
      d.x = tc::pack_bf16(__uint_as_float(r[0]) * inv, __uint_as_float(r[1]) * inv);
      d.y = tc::pack_bf16(__uint_as_float(r[2]) * inv, __uint_as_float(r[3]) * inv);
      d.z = tc::pack_bf16(__uint_as_float(r[4]) * inv, __uint_as_float(r[5]) * inv);
      d.w = tc::pack_bf16(__uint_as_float(r[6]) * inv, __uint_as_float(r[7]) * inv);
    }
  }
  uint8_t* stg = smem + Cfg::OFF_STG + (warp - 2) * Cfg::STG_WARP;
  const uint32_t astg = tc::smem_u32(stg);
#pragma unroll
  for (int rnd = 0; rnd < 2; ++rnd) {
    if (lane == 0) tc::bulk_wait_read_all();  // the slot's previous store has read it
    __syncwarp();
    if ((lane >> 4) == rnd) {
      // row r of the box, its 16-byte chunk c at chunk c ^ (address bits 7.. of the row):
      // the swizzle of the h tensor map, whose span is one row (DV / 2 bytes)
      const int r = lane & 15;
      const uint32_t sw = ((uint32_t)(r * CPR * 16) >> 7) & (CPR - 1);
#pragma unroll
      for (int c = 0; c < CPR; ++c)
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(astg + r * (CPR * 16) + ((c ^ sw) << 4)),
                     "r"(w[c].x), "r"(w[c].y), "r"(w[c].z), "r"(w[c].w)
                     : "memory");
      tc::fence_proxy_async_smem();
    }
    __syncwarp();
    if (lane == 0) {
      tc::tma_store_3d(tm_h, stg, vb * DV + h * (DV / 4), y0 + 16 * rnd, bh);
      tc::bulk_commit_group();
    }
  }
  return true;
}

template <int DQK, int DV, bool EXPV>
__global__ void __launch_bounds__(kXlThreads, 1) output_fwd_xl_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_c,
    const __grid_constant__ CUtensorMap tm_h, const float* __restrict__ tab,
    const float* __restrict__ gn, bf16* __restrict__ hout,
    float* __restrict__ abar_out, int T, int L, int NC, int BH, int NVB, int ntq, int total,
    int tstride, int dhv, bool has_init, unsigned int epoch) {
  using Cfg = XlCfg<DQK, DV>;
  const tc::Abort abort_flag{&g_tc_fwd_xl_error, epoch};
  constexpr int NQ = Cfg::NQ, NK = Cfg::NK, NV = Cfg::NV;
  // an earlier CTA gave up: the whole block leaves together
  if (__syncthreads_or(threadIdx.x == 0 && abort_flag.raised())) return;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_TMEM);
  float* xs = reinterpret_cast<float*>(smem + Cfg::OFF_XS);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < X_COUNT; ++i) {
      uint32_t cnt = 1;
      if (i == X_QE0 || i == X_QE0 + 1) cnt = kXlTransform + 1;
      if (i >= X_PF0 && i < X_PF0 + 4) cnt = kXlTransform;
      if (i >= X_OE0 && i < X_OE0 + 2) cnt = kXlTransform;
      if (i >= X_XS0 && i < X_XS0 + 16) cnt = kXlTransform / 4;
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
    // ------------------------------------------------------------ Q / K / C_prev producer
    // The whole warp walks the schedule (warp-uniform values); lane 0 issues.
    {
      const unsigned full = 0xffffffffu;
      const bool leader = lane == 0;
      if (leader) {
        tc::prefetch_tmap(&tm_q);
        tc::prefetch_tmap(&tm_k);
        tc::prefetch_tmap(&tm_c);
      }
      int it = 0, g = 0;
      uint32_t nq = 0;  // Q fills issued
      for (int k = xl_first(); k < total && ok; k = xl_succ(k)) {
        XlItem I;
        if (!xl_item(k, BH, NC, NVB, ntq, T, L, has_init, I)) continue;
        const int qb = it % NQ;
        ok = __all_sync(full, tc::mbar_wait(&bar[X_QE0 + qb], ((it / NQ) & 1) ^ 1, abort_flag));
        if (!ok) break;
        const float* tb = tab + ((size_t)I.bh * NC + I.c) * tstride;
        const bool nv = EXPV && I.pseudo;
        if (leader) {
          uint64_t* qf = &bar[X_QF0 + qb];
          tc::mbar_arrive_expect_tx(qf, Cfg::Q_BYTES + 1536 + (nv ? DQK * 4 : 0));
          uint8_t* sq = smem + Cfg::OFF_Q + qb * Cfg::Q_BYTES;
          for (int kb = 0; kb < Cfg::KB; ++kb)
            tc::tma_load_3d(sq + kb * 16384, &tm_q, qf, kb * 64, I.c * L + I.t0, I.bh);
          uint8_t* rp = smem + Cfg::OFF_ROW + qb * Cfg::ROWAUX;
          tc::bulk_load(rp, tb + I.t0, 512, qf);
          tc::bulk_load(rp + 512, tb + L + I.t0, 512, qf);
          tc::bulk_load(rp + 1024, tb + 2 * L + I.t0, 512, qf);
          if (nv) tc::bulk_load(rp + 1536, gn + ((size_t)I.bh * NC + I.c) * DQK, DQK * 4, qf);
        }
        ++nq;
        const int nsteps = I.nkv + (I.pseudo ? 1 : 0);
        for (int s = 0; s < nsteps && ok; ++s, ++g) {
          const int kst = g % NK;
          ok = __all_sync(full, tc::mbar_wait(&bar[X_KE0 + kst], ((g / NK) & 1) ^ 1, abort_flag));
          if (!ok) break;
          uint64_t* kf = &bar[X_KF0 + kst];
          uint8_t* ks = smem + Cfg::OFF_K + kst * Cfg::K_BYTES;
          if (I.pseudo && s == 0) {
            if (leader) {
              tc::mbar_arrive_expect_tx(kf, Cfg::C_BYTES);
              for (int v = 0; v < Cfg::VB; ++v)
                tc::tma_load_3d(ks + v * DQK * 128, &tm_c, kf, I.vb * DV + v * 64, 0, I.bh * NC + I.c);
            }
          } else {
            const int j = s - (I.pseudo ? 1 : 0);
            if (leader) {
              tc::mbar_arrive_expect_tx(kf, Cfg::K_BYTES);
              for (int kb = 0; kb < Cfg::KB; ++kb)
                tc::tma_load_3d(ks + kb * 16384, &tm_k, kf, kb * 64, I.c * L + j * 128, I.bh);
            }
          }
        }
        ++it;
      }
      // gave up: the copies this warp issued land before the CTA exits
      if (!ok && leader) {
        tc::drain_ring(&bar[X_QF0], NQ, nq);
        tc::drain_ring(&bar[X_KF0], NK, (uint32_t)g);
      }
    }
  } else if (warp == kXlVWarp) {
    // ------------------------------------------------------------ V producer
    // Per key tile the V tile and the tile's gate factors (CC, KP of its 128
    // keys and the four 32-key block maxima).
    {
      const unsigned full = 0xffffffffu;
      const bool leader = lane == 0;
      if (leader) tc::prefetch_tmap(&tm_v);
      int gv = 0;
      for (int k = xl_first(); k < total && ok; k = xl_succ(k)) {
        XlItem I;
        if (!xl_item(k, BH, NC, NVB, ntq, T, L, has_init, I)) continue;
        const float* tb = tab + ((size_t)I.bh * NC + I.c) * tstride;
        for (int j = 0; j < I.nkv && ok; ++j, ++gv) {
          const int st = gv % NV;
          ok = __all_sync(full, tc::mbar_wait(&bar[X_VE0 + st], ((gv / NV) & 1) ^ 1, abort_flag));
          if (!ok) break;
          if (leader) {
            uint64_t* vf = &bar[X_VF0 + st];
            uint8_t* vs = smem + Cfg::OFF_V + st * Cfg::V_BYTES;
            uint8_t* cp = smem + Cfg::OFF_COL + st * Cfg::COLAUX;
            tc::mbar_arrive_expect_tx(vf, Cfg::V_BYTES + Cfg::COLAUX);
            for (int v = 0; v < Cfg::VB; ++v)
              tc::tma_load_3d(vs + v * 16384, &tm_v, vf, I.vb * DV + v * 64, I.c * L + j * 128, I.bh);
            tc::bulk_load(cp, tb + 3 * L + j * 128, 512, vf);
            tc::bulk_load(cp + 512, tb + 4 * L + j * 128, 512, vf);
            tc::bulk_load(cp + 1024, tb + 5 * L + j * 4, 16, vf);
          }
        }
      }
      if (!ok && leader) tc::drain_ring(&bar[X_VF0], NV, (uint32_t)gv);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Lane 0 alone walks the schedule, waits and issues.  tcgen05.mma issue
    // blocks behind a shallow queue, so every other instruction this thread
    // runs between two products (warp votes, descriptor arithmetic) is time
    // the tensor pipe stands idle: the shared-memory descriptors are built
    // once and advanced by constant offsets (the address field is the low
    // 14 bits of address / 16, and no offset reaches past the 227 KB of
    // shared memory, so adding to the descriptor is exact).
    if (lane == 0) {
      constexpr uint32_t idS = tc::idesc_bf16(128, 128, false, false);
      constexpr uint32_t idO = tc::idesc_bf16(128, DV, false, true);
      const uint32_t aQ0 = tc::smem_u32(smem + Cfg::OFF_Q), aK0 = tc::smem_u32(smem + Cfg::OFF_K),
                     aV0 = tc::smem_u32(smem + Cfg::OFF_V);
      const uint64_t dQ0 = tc::sdesc_sw128(aQ0, 16, 1024), dK0 = tc::sdesc_sw128(aK0, 16, 1024),
                     dV0 = tc::sdesc_sw128(aV0, 16384, 1024), dC0 = tc::sdesc_sw128(aK0, DQK * 128, 1024);

      // score step s of item I (its it-th item, global step g): S_j = Q K_j^T,
      // then the K stage is free; for the C_prev step only a commit, which
      // tells the transform the S buffer's last reader (P V of step g - 2) is done
      auto issue_s = [&](const XlItem& I, int it, int s, int g) -> bool {
        const int sb = g & 1;
        if (I.pseudo && s == 0) {
          tc::tc_commit(&bar[X_SF0 + sb]);
          return true;
        }
        const int qb = it % NQ, kst = g % NK;
        // the Q buffer is checked only before the item's first score product
        if (s == (I.pseudo ? 1 : 0) && !tc::mbar_wait(&bar[X_QF0 + qb], (it / NQ) & 1, abort_flag))
          return false;
        if (!tc::mbar_wait(&bar[X_KF0 + kst], (g / NK) & 1, abort_flag)) return false;
        const uint64_t dQ = dQ0 + (uint64_t)((qb * Cfg::Q_BYTES) >> 4),
                       dK = dK0 + (uint64_t)((kst * Cfg::K_BYTES) >> 4);
#pragma unroll
        for (int k = 0; k < DQK / 16; ++k) {
          const uint64_t off = (uint64_t)(((k >> 2) * 16384 + (k & 3) * 32) >> 4);
          tc::mma_bf16_ss(tmem + sb * 128, dQ + off, dK + off, idS, k > 0);
        }
        tc::tc_commit(&bar[X_SF0 + sb]);
        tc::tc_commit(&bar[X_KE0 + kst]);
        return true;
      };
      // accumulate step s into O: P_j V_j (V stage of real step gv),
      // or (alpha q / sqrt(d_qk)) C_prev (K stage of step g); A is read from
      // P in TMEM.  The transform threads see V / C_prev arrive before they
      // signal P, so one barrier check covers the whole product.
      auto issue_pv = [&](const XlItem& I, int it, int s, int g, int gv) -> bool {
        const int sb = g & 1, ob = it & 1;
        const uint32_t tO = tmem + 256 + ob * DV, tP = tmem + sb * 128;
        if (s == 0 && !tc::mbar_wait(&bar[X_OE0 + ob], ((it >> 1) & 1) ^ 1, abort_flag)) return false;
        if (!tc::mbar_wait(&bar[X_PF0 + sb], (g >> 1) & 1, abort_flag)) return false;
        tc::tc_fence_after();
        if (I.pseudo && s == 0) {
          const int kst = g % NK;
          const uint64_t dC = dC0 + (uint64_t)((kst * Cfg::K_BYTES) >> 4);
#pragma unroll
          for (int k = 0; k < DQK / 16; ++k) {  // 16 rows of C_prev
            // the q elements of block b = k / (DQK / 64) sit packed at column 32 b
            const int b = k / (DQK / 64), kk = k % (DQK / 64);
            tc::mma_bf16_ts(tO, tP + 32 * b + 8 * kk, dC + (uint64_t)(k * 128), idO, k > 0);
          }
          tc::tc_commit(&bar[X_KE0 + kst]);
          return true;
        }
        const uint64_t dV = dV0 + (uint64_t)(((gv % NV) * Cfg::V_BYTES) >> 4);
#pragma unroll
        for (int k = 0; k < 8; ++k)  // 16 keys per step; keys 32 b .. of P live at column 32 b
          tc::mma_bf16_ts(tO, tP + 32 * (k >> 1) + 8 * (k & 1), dV + (uint64_t)(k * 128), idO,
                          (s > 0 || k > 0));
        tc::tc_commit(&bar[X_VE0 + (gv % NV)]);
        return true;
      };

      XlItem I, N;
      int k = xl_next(xl_first(), total, BH, NC, NVB, ntq, T, L, has_init, I);
      int it = 0, g = 0, gv = 0;
      if (k < total) ok = issue_s(I, 0, 0, 0);
      while (k < total && ok) {
        const int kn = xl_next(xl_succ(k), total, BH, NC, NVB, ntq, T, L, has_init, N);
        const int nsteps = I.nkv + (I.pseudo ? 1 : 0);
        for (int s = 0; s < nsteps && ok; ++s, ++g) {
          const bool last = s + 1 == nsteps;
          // the look-ahead S goes before this step's P V when the next Q and K
          // stages can be resident at the same time; otherwise after it
          if (Cfg::LOOK) {
            if (!last) ok = issue_s(I, it, s + 1, g + 1);
            else if (kn < total) ok = issue_s(N, it + 1, 0, g + 1);
            if (!ok) break;
          }
          const bool real = !(I.pseudo && s == 0);
          ok = issue_pv(I, it, s, g, gv);
          if (!ok) break;
          if (real) ++gv;
          if (last) {
            tc::tc_commit(&bar[X_QE0 + it % NQ]);
            tc::tc_commit(&bar[X_OF0 + (it & 1)]);
          }
          if (!Cfg::LOOK) {
            if (!last) ok = issue_s(I, it, s + 1, g + 1);
            else if (kn < total) ok = issue_s(N, it + 1, 0, g + 1);
          }
        }
        ++it;
        k = kn;
        I = N;
      }
      if (!ok) tc::drain_mma(&bar[X_DRAIN]);  // no product still writes TMEM or reads smem
    }
  } else {
    // ------------------------------------------------------------ gate transform + epilogue
    const int h = (warp - 2) >> 2;  // this warpgroup's 32-key block of each tile (and DV / 4 h columns)
    const int qr = warp & 3;        // TMEM lane quarter = 32-row block of the tile
    const int row = 32 * qr + lane;
    const uint32_t lb = (uint32_t)(32 * qr) << 16;
    const unsigned full = 0xffffffffu;
    int it = 0, g = 0, gv = 0;

    // what the deferred epilogue of an item needs (kept small: it is live
    // through the next item's first step)
    struct Pending {
      int it, vb, y0, bh;  // item counter; value block; token of this warp's first row; head
      size_t tok;          // token of this thread's row ([BH, T] index)
      bool valid;          // this thread's row is in the sequence
      float fl;
    } pe{};
    bool pend = false;
    auto epilogue = [&](const Pending& e) -> bool {
      return xl_epilogue<DQK, DV, EXPV>(e.it, e.vb, e.y0, e.bh, e.tok, e.valid, e.fl, h, qr,
                                        lane, tmem, smem, &tm_h, abar_out, abort_flag);
    };

    for (int k = xl_first(); k < total && ok; k = xl_succ(k)) {
      XlItem I;
      if (!xl_item(k, BH, NC, NVB, ntq, T, L, has_init, I)) continue;
      const int qb = it % NQ;
      ok = __all_sync(full, tc::mbar_wait(&bar[X_QF0 + qb], (it / NQ) & 1, abort_flag));
      if (!ok) break;
      const float* rp = reinterpret_cast<const float*>(smem + Cfg::OFF_ROW + qb * Cfg::ROWAUX);
      const float R = rp[row], QFt = rp[128 + row], FLt = rp[256 + row];
      uint64_t part2 = tc::f2_make(0.f, 0.f);  // EXP: this block's share of the normaliser
      const int nsteps = I.nkv + (I.pseudo ? 1 : 0);
      for (int s = 0; s < nsteps && ok; ++s, ++g) {
        const int sb = g & 1;
        ok = __all_sync(full, tc::mbar_wait(&bar[X_SF0 + sb], (g >> 1) & 1, abort_flag));
        if (!ok) break;
        tc::tc_fence_after();
        const uint32_t tS = tmem + sb * 128 + lb + 32 * h;
        if (I.pseudo && s == 0) {
          // alpha_t q_t / sqrt(d_qk) over this block's d_qk / 4 elements, packed into the S buffer
          const uint8_t* sq = smem + Cfg::OFF_Q + qb * Cfg::Q_BYTES;
          const float* nvec = rp + 384;
          constexpr int NCH = DQK / 32;  // 16-byte chunks of the block's q elements
          uint32_t w[16];
#pragma unroll
          for (int ci = 0; ci < NCH; ++ci) {
            const int gc = h * NCH + ci, kb = gc >> 3, lc = gc & 7;
            const uint32_t addr = tc::smem_u32(sq) + kb * 16384 + row * 128 + ((lc ^ (row & 7)) << 4);
            uint32_t q4[4];
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(q4[0]), "=r"(q4[1]), "=r"(q4[2]), "=r"(q4[3])
                         : "r"(addr));
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 v2 = *reinterpret_cast<__nv_bfloat162*>(&q4[e]);
              const float x0 = __bfloat162float(v2.x) * QFt, x1 = __bfloat162float(v2.y) * QFt;
              if (EXPV) {
                const float2 n2 = *reinterpret_cast<const float2*>(nvec + gc * 8 + 2 * e);
                part2 = tc::f2_add(part2, tc::f2_mul(tc::f2_make(x0, x1), tc::f2_make(n2.x, n2.y)));
              }
              w[(ci & 3) * 4 + e] = tc::pack_bf16(x0, x1);
            }
            if (NCH == 2 && ci == 1) tc::tmem_st8_async(tS, w);
            if (NCH >= 4 && (ci & 3) == 3) tc::tmem_st16_async(tS + 16 * (ci >> 2), w);
          }
          // P signals the MMA thread that C_prev has landed as well
          ok = __all_sync(full, tc::mbar_wait(&bar[X_KF0 + g % NK], (g / NK) & 1, abort_flag));
          if (!ok) break;
        } else {
          const int j = s - (I.pseudo ? 1 : 0);
          const bool diag = j == I.qt;
          const int vst = gv % NV, vpar = (gv / NV) & 1;
          ++gv;
          // the key tile's gate factors, which arrive with its V tile; seeing
          // them also tells the MMA thread (through P) that V has landed
          ok = __all_sync(full, tc::mbar_wait(&bar[X_VF0 + vst], vpar, abort_flag));
          if (!ok) break;
          const float* cp = reinterpret_cast<const float*>(smem + Cfg::OFF_COL + vst * Cfg::COLAUX);
          uint32_t sv[32];
          tc::tmem_ld32_async(tS, sv);
          tc::tmem_wait_ld(sv);
          const int cc = h;  // this warp's 32-key block of the tile
          uint32_t w[16];
          if (!diag || cc < qr) {
            // the whole block lies before this row: separable factors
            const float rho = tc::ex2(R + cp[256 + cc]);
            const uint64_t rho2 = tc::f2_make(rho, rho);
            const float* kp = cp + 128 + 32 * cc;
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              const float4 k4 = *reinterpret_cast<const float4*>(kp + e);
              const uint64_t p0 = tc::f2_mul(
                  tc::f2_mul(tc::f2_make(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])),
                             tc::f2_make(k4.x, k4.y)), rho2);
              const uint64_t p1 = tc::f2_mul(
                  tc::f2_mul(tc::f2_make(__uint_as_float(sv[e + 2]), __uint_as_float(sv[e + 3])),
                             tc::f2_make(k4.z, k4.w)), rho2);
              if (EXPV) part2 = tc::f2_add(part2, tc::f2_add(p0, p1));
              const float2 a0 = tc::f2_split(p0), a1 = tc::f2_split(p1);
              w[e / 2] = tc::pack_bf16(a0.x, a0.y);
              w[e / 2 + 1] = tc::pack_bf16(a1.x, a1.y);
            }
          } else if (cc == qr) {
            // the block holding this row: per-element decay and causal mask
            const float* ccv = cp + 32 * cc;
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              float p[2];
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                const int key = 32 * cc + e + u;
                p[u] = key <= row ? __uint_as_float(sv[e + u]) * tc::ex2(R + ccv[e + u]) : 0.f;
              }
              if (EXPV) part2 = tc::f2_add(part2, tc::f2_make(p[0], p[1]));
              w[e / 2] = tc::pack_bf16(p[0], p[1]);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) w[e] = 0u;
          }
          // packed into the first 16 of this block's own 32 columns
          tc::tmem_st16_async(tS, w);
        }
        tc::tmem_wait_st();
        tc::tc_fence_before();
        tc::mbar_arrive(&bar[X_PF0 + sb]);
        if (s == 0) {
          tc::mbar_arrive(&bar[X_QE0 + qb]);
          if (pend) {
            ok = epilogue(pe);
            pend = false;
          }
        }
      }
      if (!ok) break;
      if (EXPV) {
        // this block's share of the normaliser, for the item's epilogue (one item from now)
        const float2 pf = tc::f2_split(part2);
        const int xsl = it & 3;
        xs[xsl * 512 + h * 128 + row] = pf.x + pf.y;
        tc::mbar_arrive(&bar[X_XS0 + 4 * xsl + qr]);
      }
      pe.it = it;
      pe.vb = I.vb;
      pe.y0 = I.c * L + I.t0 + 32 * qr;
      pe.bh = I.bh;
      pe.tok = (size_t)I.bh * T + (size_t)I.c * L + I.t0 + row;
      pe.valid = I.t0 + row < I.len;
      pe.fl = FLt;
      pend = true;
      ++it;
    }
    if (ok && pend) ok = epilogue(pe);
    if (lane == 0) tc::bulk_wait_all();  // the h stores have read the staging slot
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

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

template <int DQK, int DV, bool EXPV>
static cudaError_t launch_out_xl(const Problem& p, const FwdArgs& a, cudaStream_t s) {
  using Cfg = XlCfg<DQK, DV>;
  if (a.xt == nullptr) return cudaErrorInvalidValue;
  CUtensorMap tq, tk, tv, tcm, th;
  if (!make_tmap_3d_bf16_rows(&th, a.h, p.dhv, p.T, p.BH, DV / 4, 16) ||
      !make_tmap_3d_bf16(&tq, a.q, p.dqk, p.T, p.BH, 64, 128) ||
      !make_tmap_3d_bf16(&tk, a.k, p.dqk, p.T, p.BH, 64, 128) ||
      !make_tmap_3d_bf16(&tv, a.v, p.dhv, p.T, p.BH, 64, 128) ||
      !make_tmap_3d_bf16(&tcm, a.C, p.dhv, p.dqk, (uint64_t)p.BH * p.NC, 64, DQK))
    return cudaErrorInvalidValue;
  // at least 120 KB, so no second CTA shares the SM (each holds all 512 TMEM columns)
  const int smem = Cfg::SMEM > 120 * 1024 ? Cfg::SMEM : 120 * 1024;
  auto kern = output_fwd_xl_kernel<DQK, DV, EXPV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, nsm = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int ntq = p.L / 128, nvb = p.dhv / DV;  // ntq is even: L >= 256 is a power of two
  const long long total = (long long)ntq * p.BH * p.NC * nvb;
  if (total >= (1LL << 30)) return cudaErrorInvalidValue;
  const long long pairs = total / 2;
  const int grid = (int)(pairs < nsm ? pairs : nsm);
  kern<<<grid, kXlThreads, smem, s>>>(tq, tk, tv, tcm, th, a.xt, a.n, (bf16*)a.h, a.abar, p.T, p.L,
                                      p.NC, p.BH, nvb, ntq, (int)total, xl_table_stride(p.L),
                                      p.dhv, a.init.on(), next_epoch());
  return cudaGetLastError();
}

bool output_fwd_xl_supported(const Problem& p) {
  return p.bf16() && p.L >= 256 && (p.dqk == 64 || p.dqk == 128 || p.dqk == 256) &&
         (p.dhv == 64 || p.dhv % 128 == 0);
}

cudaError_t launch_output_fwd_xl(const Problem& p, const FwdArgs& a, cudaStream_t s) {
  const bool e = p.exp_variant();
#define MLSTM_XL(DQK)                                                                       \
  if (p.dqk == DQK) {                                                                       \
    if (p.dhv == 64) return e ? launch_out_xl<DQK, 64, true>(p, a, s) : launch_out_xl<DQK, 64, false>(p, a, s); \
    return e ? launch_out_xl<DQK, 128, true>(p, a, s) : launch_out_xl<DQK, 128, false>(p, a, s); \
  }
  MLSTM_XL(64)
  MLSTM_XL(128)
  MLSTM_XL(256)
#undef MLSTM_XL
  return cudaErrorInvalidValue;
}

cudaError_t fetch_tc_fwd_xl_error(unsigned int* flag) {
  return cudaMemcpyFromSymbol(flag, g_tc_fwd_xl_error, sizeof(unsigned int));
}

}  // namespace mlstm
