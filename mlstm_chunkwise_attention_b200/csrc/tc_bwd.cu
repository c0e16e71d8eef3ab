// Intra-chunk backward kernels (K-d2) on the fifth-generation tensor cores:
// dq, dk and dv, each a "score, gated transform, accumulate" walk over the
// 128-token tiles of one chunk, plus the inter-chunk term through the chunk
// states.  Timed as the training kernels of "Tiled Flash Linear Attention:
// More Efficient Linear RNN and xLSTM Kernels" (TFLA summary page, Key
// results); the second-level tiling along the sequence inside a chunk is the
// one the same page (Approach) describes for the forward pass.
//
// With m held constant, dnum_t = dh_t / den_t, da_t the normaliser gradient,
// D_ts = exp(b_t - b_s + log i_s - m_t) for s <= t inside the chunk:
//   dq'_t = alpha_t (C_{c-1} dnum_t + da_t n_{c-1}) + sum_s (dh_t.v_s/den_t + da_t) D_ts k_s
//   dk_s  = w_s (dC_c v_s + dn_c)                  + sum_t (dh_t.v_s/den_t + da_t) D_ts q'_t
//   dv_s  = w_s dC_c^T k_s                         + sum_t D_ts (q'_t.k_s) dh_t / den_t
// One CTA owns a 128-token row tile R (query rows for dq, key rows for dk and
// dv) and a slice of up to 128 output columns:
//   X  = A_R B_j^T      score tile (dq: dH V^T, dk: V dH^T, dv: K Q^T)
//   Y  = transform(X)   gates, mask and normaliser terms, bf16 to smem
//   Acc += Y E_j        (dq: E = K, dk: E = Q, dv: E = dH)
// The inter-chunk term Acc = A_R G (G the chunk state or its gradient, split
// into hi and lo bf16 planes so the product keeps about 16 mantissa bits) is
// computed first and rescaled per row in TMEM.  A 64-token chunk is one
// half-filled 128-row tile with one partner: its score product has N = 64,
// the accumulate contracts over 64 partners, and the result leaves through a
// 64-row store.  Warp roles: warp 0 TMA, warp 1 MMA (one thread), warps 2..5
// one tile row per thread.  Every wait is bounded; on a timeout the kernel
// raises an error flag and winds down.
#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace mlstm {

static __device__ unsigned int g_tc_bwd_error;

namespace {

constexpr float kLog2e = 1.4426950408889634f;
enum { KDQ = 0, KDK = 1, KDV = 2 };

// NXBUF score buffers in TMEM: 1 up to chunk 1024, so the CTA fits in 256 TMEM
// columns and ~100-108 KB of shared memory and two CTAs share an SM (one CTA's
// serial phases overlap the other's tiles); 2 for longer chunks, where only one
// CTA fits and the next score overlaps the transform instead.  The transformed
// tile Y is written back over its score as packed bf16 and read from TMEM by the
// accumulate product, so shared memory holds only the operand ring.
template <int D1, int D2S, bool G_MN, int NXBUF>
struct BwdTcCfg {
  static constexpr int STAGES = NXBUF == 1 ? 3 : 4;
  static constexpr int SLOT = 16384;  // one 128 x 64 bf16 block
  static constexpr int STAGE_BYTES = 2 * SLOT;
  static constexpr int NKB = D1 / 64;  // K-blocks of the score GEMM and the inter GEMM
  static constexpr int EB = D2S / 64;  // 64-column blocks of E and of the output slice
  static constexpr int OFF_RING = 0;   // ring stage 0 also stages the result tile at the end
  static constexpr int OFF_BAR = STAGES * STAGE_BYTES;
  static constexpr int NBAR = 16;
  static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
  static constexpr int OFF_RV = OFF_TMEM + 16;
  static constexpr int OFF_PW = OFF_RV + D2S * 4;   // per-warp partner factors, 4 x 128 floats
  static constexpr int OFF_PF = OFF_PW + 4 * 128 * 4;  // partner factors: 2 x PL, then PL / 32 (>= 4)
  static constexpr uint32_t TMEM_COLS = NXBUF == 1 ? 256 : 512;  // X buffers, then Acc
  static constexpr uint32_t ACC_COL = NXBUF * 128;
  static constexpr uint32_t G_BYTES = G_MN ? (uint32_t)EB * 8192u : (uint32_t)D2S * 128u;
  static constexpr uint32_t E_BYTES = (uint32_t)EB * SLOT;
  // PL = max(L, 128): a 64-token chunk still loads one whole 128-row partner tile
  static size_t smem_bytes(int L) {
    const size_t PL = L < 128 ? 128 : (size_t)L;
    return 1024 + OFF_PF + (2 * PL + (PL / 32 > 4 ? PL / 32 : 4)) * 4;
  }
};

enum {
  BB_FULL0 = 0, BB_EMPTY0 = 4, BB_X0 = 8, BB_Y = 10, BB_INTER, BB_ACC, BB_DONE, BB_STG,
  BB_DRAIN,  // the MMA thread's last commit when it gives up
  BB_COUNT
};
static_assert(BB_COUNT <= 16, "barrier slots");

}  // namespace

struct BwdTcParams {
  const float *b, *li, *m, *inv_den, *da;
  const float* rowvec;  // dq: n_{c-1} [BH, NC, dqk]; dk: dn_c [BH, NC, dqk]; dv: unused
  const bf16* dot_src;  // dq: q; dk: k (the per-token dot product with the result)
  bf16* out;            // dq, dk or dv [BH, T, d_out]
  float* pdot;          // dq: pq; dk: pk (atomically accumulated)
  int T, L, NC, BH, ntq, nsl, d_out, dqk;  // nsl: output column slices of D2S
  bool m0set;                              // the forward started from an initial state
  bool dfin;                               // the final state has a gradient (dk, dv)
  const float* m0;                         // its max state (mLSTMexp), else null
  float scale, log2_scale;
  unsigned int epoch;  // this launch's abort epoch
};

template <int KIND, int D1, int D2S, bool G_MN, bool EXPV, int NXBUF>
__global__ void __launch_bounds__(192, NXBUF == 1 ? 2 : 1) intra_bwd_tc_kernel(
    const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
    const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmGhi,
    const __grid_constant__ CUtensorMap tmGlo, const __grid_constant__ CUtensorMap tmOut,
    const BwdTcParams P) {
  using Cfg = BwdTcCfg<D1, D2S, G_MN, NXBUF>;
  const tc::Abort abort_flag{&g_tc_bwd_error, P.epoch};
  constexpr bool R_IS_QUERY = (KIND == KDQ);
  constexpr int ST = Cfg::STAGES;

  // The row tiles (and output column slices) of one chunk are consecutive CTAs, so
  // the partner tiles they all stream stay in L2 between them; inside a chunk the
  // heaviest tiles go first (dq tiles near the chunk end, dk/dv tiles near its start).
  const int slice = (int)(blockIdx.x % P.nsl);
  const int order = (int)((blockIdx.x / P.nsl) % P.ntq);
  const int it_tile = R_IS_QUERY ? P.ntq - 1 - order : order;
  const int rest = (int)(blockIdx.x / P.nsl / P.ntq);
  const int bh = rest / P.NC, c = rest % P.NC;
  const int c0 = c * P.L;
  const int len = min(P.L, P.T - c0);
  const int nt_len = (len + 127) / 128;  // tiles holding rows of this chunk
  const int NP = P.L < 128 ? P.L : 128;  // partners per partner tile (64 for a 64-token chunk)
  const int r0 = it_tile * 128;
  if (r0 >= len) return;
  // an earlier CTA gave up: the whole block leaves together
  if (__syncthreads_or(threadIdx.x == 0 && abort_flag.raised())) return;
  const int col0 = slice * D2S;
  const size_t tok0 = (size_t)bh * P.T + c0;
  // partner tiles: dq: 0..it_tile; dk, dv: it_tile..nt_len-1
  const int pj0 = R_IS_QUERY ? 0 : it_tile;
  const int np = R_IS_QUERY ? it_tile + 1 : nt_len - it_tile;
  // a state enters the chunk (dq: c > 0 or an initial state), one leaves it (dk, dv)
  const bool has_inter = R_IS_QUERY ? (c > 0 || P.m0set) : (c < P.NC - 1 || P.dfin);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* ring = smem + Cfg::OFF_RING;
  uint8_t* sOut = ring;  // result staging tile, once every product is done
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_TMEM);
  float* rowvec = reinterpret_cast<float*>(smem + Cfg::OFF_RV);
  float* pfC = reinterpret_cast<float*>(smem + Cfg::OFF_PF);  // partner exponent term
  const int PL = P.L < 128 ? 128 : P.L;  // partner slots: whole 128-row partner tiles
  float* pfE = pfC + PL;  // partner additive term (dk) or separable key factor (dq)
  float* pfM = pfE + PL;  // dq: stabiliser of every 32-key partner block
  float* pfW = reinterpret_cast<float*>(smem + Cfg::OFF_PW);  // dk, dv: this warp's partner factors

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < BB_COUNT; ++i) {
      const uint32_t cnt = (i == BB_Y || i == BB_ACC || i == BB_STG) ? 128u : 1u;
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
  const uint32_t tX0 = tmem, tAcc = tmem + Cfg::ACC_COL;
  bool ok = true;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Every operand goes through one ring, in the order the MMA thread consumes it:
    // inter (A, G_hi), (A, G_lo) per K-block; score(0); then per partner jj:
    // E(jj), score(jj + 1) with one score buffer, score(jj + 1), E(jj) with two.
    if (lane == 0) {
      tc::prefetch_tmap(&tmA);
      tc::prefetch_tmap(&tmB);
      tc::prefetch_tmap(&tmE);
      uint32_t it = 0;
      auto acquire = [&](uint32_t bytes, uint64_t*& fb) -> uint8_t* {
        const uint32_t st = it % ST, ph = (it / ST) & 1;
        if (!tc::mbar_wait(&bar[BB_EMPTY0 + st], ph ^ 1, abort_flag)) return nullptr;
        fb = &bar[BB_FULL0 + st];
        tc::mbar_arrive_expect_tx(fb, bytes);
        ++it;
        return ring + st * Cfg::STAGE_BYTES;
      };
      auto load_score = [&](int jj) -> bool {
        const int prow = c0 + (pj0 + jj) * 128;
        for (int kb = 0; kb < Cfg::NKB; ++kb) {
          uint64_t* fb;
          uint8_t* stg = acquire(2 * Cfg::SLOT, fb);
          if (!stg) return false;
          tc::tma_load_3d(stg, &tmA, fb, kb * 64, c0 + r0, bh);
          tc::tma_load_3d(stg + Cfg::SLOT, &tmB, fb, kb * 64, prow, bh);
        }
        return true;
      };
      if (has_inter) {
        const int gz = bh * P.NC + c;
        for (int kb = 0; kb < Cfg::NKB && ok; ++kb) {
          for (int half = 0; half < 2 && ok; ++half) {
            const CUtensorMap* tg = half == 0 ? &tmGhi : &tmGlo;
            uint64_t* fb;
            uint8_t* stg = acquire(Cfg::SLOT + Cfg::G_BYTES, fb);
            if (!stg) { ok = false; break; }
            tc::tma_load_3d(stg, &tmA, fb, kb * 64, c0 + r0, bh);
            if (G_MN) {  // G rows = contraction (d_qk block kb), columns = output slice
              for (int eb = 0; eb < Cfg::EB; ++eb)
                tc::tma_load_3d(stg + Cfg::SLOT + eb * 8192, tg, fb, col0 + eb * 64, kb * 64, gz);
            } else {  // G rows = output slice, columns = contraction (d_hv block kb)
              tc::tma_load_3d(stg + Cfg::SLOT, tg, fb, kb * 64, col0, gz);
            }
          }
        }
      }
      auto load_e = [&](int jj) -> bool {
        uint64_t* fb;
        uint8_t* stg = acquire(Cfg::E_BYTES, fb);
        if (!stg) return false;
        const int prow = c0 + (pj0 + jj) * 128;
        for (int eb = 0; eb < Cfg::EB; ++eb)
          tc::tma_load_3d(stg + eb * Cfg::SLOT, &tmE, fb, col0 + eb * 64, prow, bh);
        return true;
      };
      if (ok) ok = load_score(0);
      for (int jj = 0; jj < np && ok; ++jj) {
        if (NXBUF == 1) {
          ok = load_e(jj);
          if (ok && jj + 1 < np) ok = load_score(jj + 1);
        } else {
          if (jj + 1 < np) ok = load_score(jj + 1);
          if (ok) ok = load_e(jj);
        }
      }
      // stay until the last copies this thread issued have landed
      if (ok && it > 0)
        ok = tc::mbar_wait(&bar[BB_FULL0 + (it - 1) % ST], ((it - 1) / ST) & 1, abort_flag);
      // gave up: every copy still in flight lands before the CTA exits
      if (!ok) tc::drain_ring(&bar[BB_FULL0], ST, it);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idX = tc::idesc_bf16(128, NP, false, false);
      constexpr uint32_t idAcc = tc::idesc_bf16(128, D2S, false, true);
      constexpr uint32_t idG = tc::idesc_bf16(128, D2S, false, G_MN);
      const uint32_t aRing = tc::smem_u32(ring);
      uint32_t it = 0;
      // wait for the next ring entry; returns its shared address (0 on timeout)
      auto next_stage = [&]() -> uint32_t {
        const uint32_t st = it % ST;
        if (!tc::mbar_wait(&bar[BB_FULL0 + st], (it / ST) & 1, abort_flag)) return 0u;
        tc::tc_fence_after();
        return aRing + st * Cfg::STAGE_BYTES;
      };
      auto release = [&]() {
        tc::tc_commit(&bar[BB_EMPTY0 + (it % ST)]);
        ++it;
      };
      if (has_inter) {
        for (int kb = 0; kb < Cfg::NKB && ok; ++kb) {
          for (int half = 0; half < 2; ++half) {
            const uint32_t st = next_stage();
            if (!st) { ok = false; break; }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint64_t a = tc::sdesc_sw128(st + k * 32, 16, 1024);
              const uint64_t g = G_MN ? tc::sdesc_sw128(st + Cfg::SLOT + k * 2048, 8192, 1024)
                                      : tc::sdesc_sw128(st + Cfg::SLOT + k * 32, 16, 1024);
              tc::mma_bf16_ss(tAcc, a, g, idG, (kb > 0 || half > 0 || k > 0));
            }
            release();
          }
        }
        tc::tc_commit(&bar[BB_INTER]);
      }
      auto issue_score = [&](int jj) -> bool {
        const uint32_t tX = tX0 + (jj % NXBUF) * 128;
        for (int kb = 0; kb < Cfg::NKB; ++kb) {
          const uint32_t st = next_stage();
          if (!st) return false;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc::mma_bf16_ss(tX, tc::sdesc_sw128(st + k * 32, 16, 1024),
                            tc::sdesc_sw128(st + Cfg::SLOT + k * 32, 16, 1024), idX, (kb > 0 || k > 0));
          release();
        }
        tc::tc_commit(&bar[BB_X0 + (jj % NXBUF)]);
        return true;
      };
      // Acc += Y E_jj, Y read from TMEM (packed bf16 over its score, 16 partners per
      // 8 columns).  MMAs of this thread run in issue order, so a later score may
      // overwrite the columns this product reads.
      auto issue_acc = [&](int jj) -> bool {
        const uint32_t st = next_stage();  // E(jj)
        if (!st) return false;
        const uint32_t tY = tX0 + (jj % NXBUF) * 128;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (16 * k < NP)
            tc::mma_bf16_ts(tAcc, tY + 8 * k, tc::sdesc_sw128(st + k * 2048, Cfg::SLOT, 1024), idAcc,
                            (has_inter || jj > 0 || k > 0));
        release();
        return true;
      };
      if (ok) ok = issue_score(0);
      for (int jj = 0; jj < np && ok; ++jj) {
        // one X buffer: the next score follows this accumulate (it overwrites Y);
        // two buffers: the next score goes to the buffer the accumulate of jj - 1 read
        if (NXBUF != 1 && jj + 1 < np) ok = issue_score(jj + 1);
        if (ok) ok = tc::mbar_wait(&bar[BB_Y], jj & 1, abort_flag);
        if (ok && jj == 0 && has_inter) ok = tc::mbar_wait(&bar[BB_ACC], 0, abort_flag);
        if (ok) tc::tc_fence_after();
        if (ok) ok = issue_acc(jj);
        if (ok && NXBUF == 1 && jj + 1 < np) ok = issue_score(jj + 1);
      }
      tc::tc_commit(&bar[BB_DONE]);
      if (!ok) tc::drain_mma(&bar[BB_DRAIN]);  // no product still writes TMEM or reads smem
    }
  } else {
    // ------------------------------------------------------------ tile rows
    // Partner factors of every partner row this tile meets, and the inter row vector,
    // loaded by the four transform warps while the producer already streams operands.
    {
      // eight partners per thread at a time: all their loads issue before any store
      const int pbase = pj0 * 128, npart = np * 128;
      for (int pi0 = threadIdx.x - 64; pi0 < npart; pi0 += 8 * 128) {
        float g0[8], g1[8], g2[8], g3[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int pi = pi0 + u * 128, p = pbase + pi;
          const bool in = pi < npart && p < len;
          const size_t t = tok0 + (in ? p : 0);
          g0[u] = in ? P.b[t] : 0.f;
          g1[u] = in ? (R_IS_QUERY ? P.li[t] : (EXPV ? P.m[t] : 0.f)) : 0.f;
          g2[u] = (in && !R_IS_QUERY && EXPV) ? P.inv_den[t] : 1.f;
          g3[u] = (in && KIND == KDK && EXPV) ? P.da[t] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int pi = pi0 + u * 128, p = pbase + pi;
          if (pi >= npart) break;
          float cexp = -INFINITY, eadd = 0.f;
          if (p < len) {
            if (R_IS_QUERY) {
              cexp = (g1[u] - g0[u]) * kLog2e;
            } else {
              cexp = (g0[u] - g1[u]) * kLog2e + log2f(g2[u]);
              if (KIND == KDK && EXPV) eadd = g3[u] / g2[u];
            }
          }
          pfC[pi] = cexp;
          pfE[pi] = eadd;
        }
      }
      if (KIND != KDV && EXPV && has_inter)
        for (int i = threadIdx.x - 64; i < D2S; i += 128)
          rowvec[i] = P.rowvec[((size_t)bh * P.NC + c) * P.dqk + col0 + i];
      tc::named_bar_sync(1, 128);
      if (R_IS_QUERY) {
        // Off-diagonal tiles split the decay: 2^(A_t + B_s) = 2^(A_t + M) 2^(B_s - M), with
        // M the largest key term B_s of the key's 32-block (so the key factor is <= 1 and
        // the row factor is at most the row's 1 / den).  One warp per block.
        for (int blk = warp - 2; blk < np * 4; blk += 4) {
          const float v = pfC[blk * 32 + lane];
          float mx = v;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          if (mx == -INFINITY) mx = 0.f;  // a block wholly past the sequence end
          if (lane == 0) pfM[blk] = mx;
          pfE[blk * 32 + lane] = tc::ex2(v - mx);
        }
        tc::named_bar_sync(1, 128);
      }
    }
    const int row = 32 * (warp & 3) + lane;
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const int rl = r0 + row;
    const bool valid = rl < len;
    const int nch = NP / 32;  // 32-column chunks of a score tile
    const size_t tok = tok0 + rl;
    const unsigned full = 0xffffffffu;
    // row-side factors
    float Rexp = -INFINITY, eRow = 0.f, rs = 0.f, rvc = 0.f;
    if (valid) {
      const float bt = P.b[tok];
      if (R_IS_QUERY) {
        const float mt = EXPV ? P.m[tok] : 0.f;
        const float invd = EXPV ? P.inv_den[tok] : 1.f;
        const float dat = EXPV ? P.da[tok] : 0.f;
        Rexp = (bt - mt) * kLog2e + log2f(invd);
        eRow = dat / invd;
        const float mprev = EXPV ? chunk_mprev(P.m, tok0, c, P.m0, bh) : 0.f;
        const float alpha = has_inter ? expf(bt + mprev - mt) : 0.f;
        rs = alpha * invd;
        rvc = alpha * dat;
      } else {
        const float lis = P.li[tok];
        // dk rounds exactly the bf16 values the dq kernel rounds (same terms in the same
        // order); 1/sqrt(d_qk) is applied in its epilogue instead.  Then the row sums of
        // the rounded dS tile (q.dq) and its column sums (k.dk) cancel over the sequence
        // as they do in exact arithmetic, which the forget-gate gradient (a reverse cumsum
        // of q.dq - k.dk) needs.
        Rexp = (lis - bt) * kLog2e + (KIND == KDV ? P.log2_scale : 0.f);
        const int last = len - 1;
        const float g = P.b[tok0 + last];
        const float mc = EXPV ? P.m[tok0 + last] : 0.f;
        rs = expf(g - bt + lis - mc);
        if (KIND == KDK) rs /= P.scale;
        rvc = rs;
      }
    }
    // dk, dv: this warp's 32 rows are one key block; its stabiliser M (the same value the
    // dq kernel takes for the block) and the row's separable factor 2^(B_s - M)
    float Mrow = 0.f, grow = 0.f;
    if (!R_IS_QUERY) {
      float mx = Rexp;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(full, mx, o));
      Mrow = mx == -INFINITY ? 0.f : mx;
      grow = tc::ex2(Rexp - Mrow);
    }
    const uint32_t aOut = tc::smem_u32(sOut);

    if (has_inter) {
      ok = __all_sync(full, tc::mbar_wait(&bar[BB_INTER], 0, abort_flag));
      if (ok) {
        tc::tc_fence_after();
#pragma unroll 1
        for (int ch = 0; ch < D2S / 32; ++ch) {
          float v[32];
          tc::tmem_ld32(tAcc + lane_base + ch * 32, v);
          uint32_t w[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            float x = rs * v[i];
            if (KIND != KDV && EXPV) x += rvc * rowvec[ch * 32 + i];
            w[i] = __float_as_uint(x);
          }
          tc::tmem_st32(tAcc + lane_base + ch * 32, w);
        }
        tc::tc_fence_before();
        tc::mbar_arrive(&bar[BB_ACC]);
      }
    }

    for (int jj = 0; jj < np && ok; ++jj) {
      ok = __all_sync(full, tc::mbar_wait(&bar[BB_X0 + (jj % NXBUF)], (jj / NXBUF) & 1, abort_flag));
      if (!ok) break;
      tc::tc_fence_after();
      const bool diag = (pj0 + jj) == it_tile;
      const float* pc = pfC + jj * 128;
      const float* pe = pfE + jj * 128;
      const uint32_t tX = tX0 + (jj % NXBUF) * 128;
      float* fw = pfW + (warp & 3) * 128;
      if (!R_IS_QUERY) {
        // partner factors 2^(A_t + M) of this warp's key block (t-side term first, as in dq)
        __syncwarp();
#pragma unroll
        for (int u = 0; u < 4; ++u) fw[lane + 32 * u] = tc::ex2(pc[lane + 32 * u] + Mrow);
        __syncwarp();
      }
      // one 32-column chunk: gates, mask and normaliser terms, packed bf16 into TMEM
      // columns [16 ch, 16 ch + 16) of the score buffer (columns already read)
      auto transform_chunk = [&](const uint32_t (&xr)[32], int ch) {
        // 32 x 32 sub-blocks: the warp's row block against column block ch.  On the
        // diagonal tile, the diagonal sub-block takes every element's own exponent and
        // the causal mask, the sub-blocks on the far side of it are zero, and the rest
        // use the separable form like every other tile (dq and dk classify each
        // (query block, key block) pair alike).
        const int wb = warp & 3;
        const bool own = diag && ch == wb;
        const bool zero = diag && (R_IS_QUERY ? ch > wb : ch < wb);
        uint32_t pk[16];
        if (zero) {
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = 0u;
        } else if (own) {
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            float y[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int p = ch * 32 + i + u;
              float add = 0.f;
              if (KIND == KDQ) add = eRow;
              if (KIND == KDK) add = pe[p];
              // t-side term first, then the s-side term, in every kernel
              const float ex = R_IS_QUERY ? (Rexp + pc[p]) : (pc[p] + Rexp);
              const float val = (__uint_as_float(xr[i + u]) + add) * tc::ex2(ex);
              const bool masked = R_IS_QUERY ? (p > row) : (p < row);
              y[u] = masked ? 0.f : val;
            }
            pk[i >> 1] = tc::pack_bf16(y[0], y[1]);
          }
        } else {
          // y = ((x + e) f) g with f the t-side and g the s-side factor: the same fp32
          // operations (two lanes at a time, each rounded as alone), so the same bf16
          // values, in the dq and dk kernels
          const float fq = R_IS_QUERY ? tc::ex2(Rexp + pfM[jj * 4 + ch]) : 0.f;
          const uint64_t e2 = tc::f2_make(eRow, eRow), fq2 = tc::f2_make(fq, fq),
                         g2r = tc::f2_make(grow, grow);
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const int p = ch * 32 + i;
            const float4 g4 = *reinterpret_cast<const float4*>((R_IS_QUERY ? pe : fw) + p);
            float4 e4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (KIND == KDK) e4 = *reinterpret_cast<const float4*>(pe + p);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint64_t x2 = tc::f2_make(__uint_as_float(xr[i + 2 * h]), __uint_as_float(xr[i + 2 * h + 1]));
              const uint64_t gv = h ? tc::f2_make(g4.z, g4.w) : tc::f2_make(g4.x, g4.y);
              uint64_t y2;
              if (KIND == KDQ) {
                y2 = tc::f2_mul(tc::f2_mul(tc::f2_add(x2, e2), fq2), gv);
              } else if (KIND == KDK) {
                const uint64_t ev = h ? tc::f2_make(e4.z, e4.w) : tc::f2_make(e4.x, e4.y);
                y2 = tc::f2_mul(tc::f2_mul(tc::f2_add(x2, ev), gv), g2r);
              } else {
                y2 = tc::f2_mul(tc::f2_mul(x2, gv), g2r);
              }
              const float2 yy = tc::f2_split(y2);
              pk[(i >> 1) + h] = tc::pack_bf16(yy.x, yy.y);
            }
          }
        }
        tc::tmem_st16_async(tX + lane_base + 16 * ch, pk);
      };
      // the next chunk's TMEM load is in flight while this one is transformed
      uint32_t xa[32], xb[32];
      tc::tmem_ld32_async(tX + lane_base, xa);
      tc::tmem_wait_ld(xa);
      tc::tmem_ld32_async(tX + lane_base + 32, xb);
      transform_chunk(xa, 0);
      tc::tmem_wait_ld(xb);
      if (nch > 2) {
        tc::tmem_ld32_async(tX + lane_base + 64, xa);
        transform_chunk(xb, 1);
        tc::tmem_wait_ld(xa);
        tc::tmem_ld32_async(tX + lane_base + 96, xb);
        transform_chunk(xa, 2);
        tc::tmem_wait_ld(xb);
        transform_chunk(xb, 3);
      } else {
        transform_chunk(xb, 1);
      }
      tc::tmem_wait_st();
      tc::tc_fence_before();
      tc::mbar_arrive(&bar[BB_Y]);
    }

    if (ok) ok = __all_sync(full, tc::mbar_wait(&bar[BB_DONE], 0, abort_flag));
    if (ok) {
      // the result tile goes through the (now idle) first ring stage and one TMA store
      // per 64-column block; rows past the sequence end are clipped by the TMA unit
      tc::tc_fence_after();
      tc::fence_proxy_async_smem();
      const float fin = (KIND == KDV) ? 1.f : P.scale;
      const bf16* drow = (KIND != KDV) ? P.dot_src + tok * P.dqk + col0 : nullptr;
      float dot = 0.f;
#pragma unroll 1
      for (int ch = 0; ch < D2S / 32; ++ch) {
        float v[32];
        tc::tmem_ld32(tAcc + lane_base + ch * 32, v);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          float g[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) g[e] = v[8 * q4 + e] * fin;
          if (KIND != KDV && valid) {
            const uint4 src = *reinterpret_cast<const uint4*>(drow + ch * 32 + q4 * 8);
            const uint32_t sw[4] = {src.x, src.y, src.z, src.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 s2 = *reinterpret_cast<const __nv_bfloat162*>(&sw[e]);
              dot = fmaf(__bfloat162float(s2.x), g[2 * e], dot);
              dot = fmaf(__bfloat162float(s2.y), g[2 * e + 1], dot);
            }
          }
          const int col = ch * 32 + q4 * 8, blk = col >> 6, lc = (col & 63) >> 3;
          const uint32_t addr = aOut + blk * Cfg::SLOT + row * 128 + ((lc ^ (row & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                       "r"(tc::pack_bf16(g[0], g[1])), "r"(tc::pack_bf16(g[2], g[3])),
                       "r"(tc::pack_bf16(g[4], g[5])), "r"(tc::pack_bf16(g[6], g[7]))
                       : "memory");
        }
      }
      if (KIND != KDV && valid) atomicAdd(&P.pdot[tok], dot);
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bar[BB_STG]);
      if (row == 0) {
        ok = tc::mbar_wait(&bar[BB_STG], 0, abort_flag);
        if (ok) {
          for (int blk = 0; blk < Cfg::EB; ++blk)
            tc::tma_store_3d(&tmOut, sOut + blk * Cfg::SLOT, col0 + blk * 64, c0 + r0, bh);
          tc::bulk_commit_group();
          tc::bulk_wait_all();
        }
      }
    }
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

bool intra_bwd_tc_supported(const Problem& p) {
  return p.bf16() && p.L >= 64 && (p.dqk == 64 || p.dqk == 128 || p.dqk == 256) &&
         (p.dhv == 64 || p.dhv == 128 || p.dhv == 256 || p.dhv == 512);
}

template <int KIND, int D1, int D2S, bool G_MN, bool EXPV, int NXBUF>
static cudaError_t launch_kind(const Problem& p, const BwdArgs& a, cudaStream_t s) {
  using Cfg = BwdTcCfg<D1, D2S, G_MN, NXBUF>;
  const size_t plane = (size_t)p.BH * p.NC * p.dqk * p.dhv;
  const bf16* C = (const bf16*)a.C;
  const bf16* dC = (const bf16*)a.dC;
  CUtensorMap tA, tB, tE, tGh, tGl, tO;
  bool okm = true;
  const uint64_t BHNC = (uint64_t)p.BH * p.NC;
  if (KIND == KDQ) {
    okm &= make_tmap_3d_bf16(&tA, a.dh, p.dhv, p.T, p.BH, 64, 128);
    okm &= make_tmap_3d_bf16(&tB, a.v, p.dhv, p.T, p.BH, 64, 128);
    okm &= make_tmap_3d_bf16(&tE, a.k, p.dqk, p.T, p.BH, 64, 128);
    okm &= make_tmap_3d_bf16(&tGh, C, p.dhv, p.dqk, BHNC, 64, D2S);
    okm &= make_tmap_3d_bf16(&tGl, C + plane, p.dhv, p.dqk, BHNC, 64, D2S);
  } else if (KIND == KDK) {
    okm &= make_tmap_3d_bf16(&tA, a.v, p.dhv, p.T, p.BH, 64, 128);
    okm &= make_tmap_3d_bf16(&tB, a.dh, p.dhv, p.T, p.BH, 64, 128);
    okm &= make_tmap_3d_bf16(&tE, a.q, p.dqk, p.T, p.BH, 64, 128);
    okm &= make_tmap_3d_bf16(&tGh, dC, p.dhv, p.dqk, BHNC, 64, D2S);
    okm &= make_tmap_3d_bf16(&tGl, dC + plane, p.dhv, p.dqk, BHNC, 64, D2S);
  } else {
    okm &= make_tmap_3d_bf16(&tA, a.k, p.dqk, p.T, p.BH, 64, 128);
    okm &= make_tmap_3d_bf16(&tB, a.q, p.dqk, p.T, p.BH, 64, 128);
    okm &= make_tmap_3d_bf16(&tE, a.dh, p.dhv, p.T, p.BH, 64, 128);
    okm &= make_tmap_3d_bf16(&tGh, dC, p.dhv, p.dqk, BHNC, 64, 64);
    okm &= make_tmap_3d_bf16(&tGl, dC + plane, p.dhv, p.dqk, BHNC, 64, 64);
  }
  {
    void* outp = (KIND == KDQ) ? a.dq : (KIND == KDK) ? a.dk : a.dv;
    const int dout = (KIND == KDV) ? p.dhv : p.dqk;
    // one 64-row store per block for a 64-token chunk, so the next chunk's rows stay untouched
    okm &= make_tmap_3d_bf16(&tO, outp, dout, p.T, p.BH, 64, p.L < 128 ? (uint32_t)p.L : 128u);
  }
  if (!okm) return cudaErrorInvalidValue;
  BwdTcParams P;
  P.b = a.b; P.li = a.li; P.m = a.m; P.inv_den = a.inv_den; P.da = a.da;
  P.rowvec = (KIND == KDQ) ? a.n : a.dn;
  P.dot_src = (const bf16*)((KIND == KDQ) ? a.q : a.k);
  P.m0set = a.init.on();
  P.dfin = a.dCT != nullptr;
  P.m0 = (a.init.on() && p.exp_variant()) ? a.init.m : nullptr;
  P.out = (bf16*)((KIND == KDQ) ? a.dq : (KIND == KDK) ? a.dk : a.dv);
  P.pdot = (KIND == KDQ) ? a.pq : a.pk;
  P.T = p.T; P.L = p.L; P.NC = p.NC; P.BH = p.BH; P.ntq = p.L < 128 ? 1 : p.L / 128;
  P.d_out = (KIND == KDV) ? p.dhv : p.dqk;
  P.dqk = p.dqk;
  P.scale = p.scale;
  P.log2_scale = log2f(p.scale);
  P.epoch = next_epoch();
  const size_t smem = Cfg::smem_bytes(p.L);
  auto kern = intra_bwd_tc_kernel<KIND, D1, D2S, G_MN, EXPV, NXBUF>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  P.nsl = P.d_out / D2S;
  dim3 grid((unsigned)(p.BH * p.NC * P.ntq * P.nsl)), block(192);
  kern<<<grid, block, smem, s>>>(tA, tB, tE, tGh, tGl, tO, P);
  return cudaGetLastError();
}

template <int KIND, bool EXPV>
static cudaError_t dispatch_kind(const Problem& p, const BwdArgs& a, cudaStream_t s) {
  constexpr bool GMN = (KIND == KDV);
  const int d1 = (KIND == KDV) ? p.dqk : p.dhv;
  const int dout = (KIND == KDV) ? p.dhv : p.dqk;
  const bool wide = dout >= 128;
  // One score buffer (256 TMEM columns) lets two CTAs share an SM, so one CTA's
  // prologue, inter term and epilogue overlap the other's tiles; that needs both
  // CTAs' shared memory (about 100 KB plus 8 bytes per chunk token) to fit.
#define MLSTM_BWD_TC_D1(D1)                                                                  \
  if (d1 == D1) {                                                                            \
    if (p.L <= 1024)                                                                         \
      return wide ? launch_kind<KIND, D1, 128, GMN, EXPV, 1>(p, a, s)                        \
                  : launch_kind<KIND, D1, 64, GMN, EXPV, 1>(p, a, s);                        \
    return wide ? launch_kind<KIND, D1, 128, GMN, EXPV, 2>(p, a, s)                          \
                : launch_kind<KIND, D1, 64, GMN, EXPV, 2>(p, a, s);                          \
  }
  MLSTM_BWD_TC_D1(64)
  MLSTM_BWD_TC_D1(128)
  MLSTM_BWD_TC_D1(256)
  MLSTM_BWD_TC_D1(512)
#undef MLSTM_BWD_TC_D1
  return cudaErrorInvalidValue;
}

cudaError_t launch_dq_tc(const Problem& p, const BwdArgs& a, cudaStream_t s) {
  return p.exp_variant() ? dispatch_kind<KDQ, true>(p, a, s) : dispatch_kind<KDQ, false>(p, a, s);
}
cudaError_t launch_dk_tc(const Problem& p, const BwdArgs& a, cudaStream_t s) {
  return p.exp_variant() ? dispatch_kind<KDK, true>(p, a, s) : dispatch_kind<KDK, false>(p, a, s);
}
cudaError_t launch_dv_tc(const Problem& p, const BwdArgs& a, cudaStream_t s) {
  return p.exp_variant() ? dispatch_kind<KDV, true>(p, a, s) : dispatch_kind<KDV, false>(p, a, s);
}

cudaError_t fetch_tc_bwd_error(unsigned int* flag) {
  return cudaMemcpyFromSymbol(flag, g_tc_bwd_error, sizeof(unsigned int));
}

}  // namespace mlstm
