// Chunk-state recurrences on the fifth-generation tensor cores: the forward
// inter-chunk states (K-b) and the backward state gradients (K-d1).
//
// "Tiled Flash Linear Attention: More Efficient Linear RNN and xLSTM Kernels"
// (TFLA summary page, Problem; arXiv abstract page, Abstract): the chunkwise
// form materialises the state at every chunk boundary.
//   forward:  C_{c+1} = beta_c C_c + K_c^T diag(w) V_c,   w_s = exp(g_c - b_s + log i_s - m_c)
//             n_{c+1} = beta_c n_c + K_c^T w                               (mLSTMexp)
//   backward: G_{c-1} = beta_c G_c + Q_c^T diag(u) dH_c,  u_t = alpha_t / (sqrt(d_qk) den_t)
//             gn_{c-1} = beta_c gn_c + Q_c^T (alpha_t da_t / sqrt(d_qk))    (mLSTMexp)
// with beta_c = exp(g_c + m_{c-1} - m_c).  The forward stores the state
// entering every chunk, the backward the gradient of the state leaving it,
// both as hi/lo bf16 planes (hi + lo keeps about 16 mantissa bits).
//
// One CTA owns a 128-row (d_qk) by 64-column (d_hv) tile of the state and
// walks the chunks in order; the fp32 running state lives in registers of the
// four epilogue warps (one state row per thread).  When too few CTAs would
// walk too many chunks (few heads, long sequences), each head's chunk range is
// split into segments walked in parallel, every segment but the first from the
// zero state; state_fix then adds to each segment's states the true state
// entering it, carried through the segment's decay (the recurrence is linear).  Each chunk is streamed in
// 64-token sub-tiles through a TMA ring; two warps scale the value-side
// operand by the per-token weight and split it into hi and lo bf16 tiles, so
// the contraction K^T (w V) keeps fp32-level accuracy (two MMAs per step).
// Warp roles: 0 TMA, 1 MMA + TMEM, 2..3 scaling, 4..7 epilogue.
#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace mlstm {

static __device__ unsigned int g_tc_state_error;

namespace {

template <int NV>
struct StateTcCfg {
  static constexpr int STAGES = 2;
  static constexpr int SUB = 64;                 // tokens per sub-tile (the MMA K extent)
  static constexpr int A_BYTES = 2 * 8192;       // 64 tokens x 128 state rows, two 64-row blocks
  static constexpr int B_BYTES = (NV / 64) * 8192;
  static constexpr int BN_BYTES = 2048;          // 16 x 64 K-major tile of the normaliser column
  static constexpr int OFF_A = 0;
  static constexpr int OFF_BHI = OFF_A + A_BYTES;
  static constexpr int OFF_BLO = OFF_BHI + B_BYTES;
  static constexpr int OFF_NHI = OFF_BLO + B_BYTES;
  static constexpr int OFF_NLO = OFF_NHI + BN_BYTES;
  static constexpr int STAGE_BYTES = OFF_NLO + BN_BYTES;
  // staging tile of one chunk boundary for the TMA stores: hi then lo plane,
  // each 128 rows x NV columns in the 128-byte-swizzled layout
  static constexpr int OFF_STG = STAGES * STAGE_BYTES;
  static constexpr int STG_PLANE = (NV / 64) * 16384;
  static constexpr int OFF_BAR = OFF_STG + 2 * STG_PLANE;
  static constexpr int NBAR = 16;
  static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
  static constexpr size_t SMEM = 1024 + OFF_TMEM + 16;
  // two U buffers: U_b in [128 b, 128 b + NV), its normaliser column block at
  // [128 b + NV, 128 b + NV + 16); the MMA of chunk c+1 overlaps the epilogue of c
  static constexpr uint32_t TMEM_COLS = 256;
};

enum {
  SB_FULL0 = 0, SB_SCALED0 = 3, SB_EMPTY0 = 6, SB_U0 = 9, SB_UFREE0 = 11, SB_STG_FULL = 13,
  SB_STG_FREE = 14,
  SB_DRAIN = 15,  // the MMA thread's last commit when it gives up
  SB_COUNT = 16
};
static_assert(SB_COUNT <= 16, "barrier slots");

}  // namespace

struct StateTcParams {
  const float *b, *li, *m, *inv_den, *da;
  bf16* out;      // hi plane; the lo plane follows after `plane` elements
  float* nout;    // [BH, NC, dqk] normaliser state (forward) or its gradient (backward)
  size_t plane;
  int T, L, NC, dqk, dhv, BH;
  int seg_len, nseg;  // chunks (walk steps) per segment; segments per head (1: no split)
  float scale;
  InitState init;   // forward: the state entering chunk 0; both: its max state m0
  float *d0, *dn0;  // backward: gradient of the initial state (C, n), fp32, or null
  const float *dT, *dnT;  // backward: gradient of the final state (C, n), fp32, or null
  unsigned int epoch;     // this launch's abort epoch
};

template <bool BWD, bool EXPV, int NV>
__global__ void __launch_bounds__(256, 2) state_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                                                          const __grid_constant__ CUtensorMap tmB,
                                                          const __grid_constant__ CUtensorMap tmOhi,
                                                          const __grid_constant__ CUtensorMap tmOlo,
                                                          const StateTcParams P) {
  using Cfg = StateTcCfg<NV>;
  const tc::Abort abort_flag{&g_tc_state_error, P.epoch};
  constexpr int SUB = Cfg::SUB;
  // an earlier CTA gave up: the whole block leaves together
  if (__syncthreads_or(threadIdx.x == 0 && abort_flag.raised())) return;
  // value-column tiles vary fastest so the CTAs sharing one head's key rows run together
  const int dv0 = blockIdx.x * NV, dk0 = blockIdx.y * 128;
  const int bh = (int)(blockIdx.z % P.BH), seg = (int)(blockIdx.z / P.BH);
  const bool with_n = EXPV && blockIdx.x == 0;
  const size_t tokh = (size_t)bh * P.T;
  const int NC = P.NC;
  // this segment's walk steps [us, us + nlocal): chunks in order (forward) or in reverse
  // (backward).  Contributions needed: every step's but the walk's last (no state leaves
  // it), and that one too in the backward when the initial state's gradient is wanted.
  // Slots stored: the state entering each step of the segment (the first segment's first
  // one included, the others' first one being the previous segment's last) and, unless the
  // segment ends the walk, the state after its last step.
  const int us = seg * P.seg_len, nlocal = min(P.seg_len, NC - us);
  const bool last_seg = us + nlocal == NC;
  const int nsteps = last_seg ? nlocal - 1 + ((BWD && P.d0 != nullptr) ? 1 : 0) : nlocal;
  const int nslots = last_seg ? nlocal : nlocal + 1;
  const float* m0 = P.init.on() ? P.init.m : nullptr;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_TMEM);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < SB_COUNT; ++i) {
      uint32_t cnt = 1;
      if (i >= SB_SCALED0 && i < SB_SCALED0 + Cfg::STAGES) cnt = 64;
      if (i == SB_UFREE0 || i == SB_UFREE0 + 1 || i == SB_STG_FULL) cnt = 128;
      tc::mbar_init(&bar[i], cnt);
    }
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tc::tmem_relinquish();
  }
  // rows 1..15 of the normaliser-column tiles stay zero
  for (int i = threadIdx.x; i < Cfg::STAGES * 2 * Cfg::BN_BYTES / 4; i += blockDim.x) {
    const int st = i / (2 * Cfg::BN_BYTES / 4), r = i % (2 * Cfg::BN_BYTES / 4);
    reinterpret_cast<uint32_t*>(smem + st * Cfg::STAGE_BYTES + Cfg::OFF_NHI)[r] = 0u;
  }
  tc::fence_proxy_async_smem();
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tU0 = tmem;
  bool ok = true;

  auto chunk_of = [&](int u) { return BWD ? NC - 1 - (us + u) : us + u; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0;
      for (int u = 0; u < nsteps && ok; ++u) {
        const int c = chunk_of(u), c0 = c * P.L, len = min(P.L, P.T - c0);
        for (int q = 0; q * SUB < len; ++q, ++it) {
          const uint32_t st = it % Cfg::STAGES, ph = (it / Cfg::STAGES) & 1;
          ok = tc::mbar_wait(&bar[SB_EMPTY0 + st], ph ^ 1, abort_flag);
          if (!ok) break;
          uint8_t* stg = smem + st * Cfg::STAGE_BYTES;
          tc::mbar_arrive_expect_tx(&bar[SB_FULL0 + st], Cfg::A_BYTES + Cfg::B_BYTES);
          for (int h = 0; h < 2; ++h)
            tc::tma_load_3d(stg + Cfg::OFF_A + h * 8192, &tmA, &bar[SB_FULL0 + st], dk0 + h * 64,
                            c0 + q * SUB, bh);
          for (int h = 0; h < NV / 64; ++h)
            tc::tma_load_3d(stg + Cfg::OFF_BHI + h * 8192, &tmB, &bar[SB_FULL0 + st], dv0 + h * 64,
                            c0 + q * SUB, bh);
        }
      }
      // wait for the last loads this thread issued
      if (ok && it > 0) {
        const uint32_t last = it - 1;
        ok = tc::mbar_wait(&bar[SB_FULL0 + last % Cfg::STAGES], (last / Cfg::STAGES) & 1, abort_flag);
      }
      // gave up: every copy still in flight lands before the CTA exits
      if (!ok) tc::drain_ring(&bar[SB_FULL0], Cfg::STAGES, it);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idU = tc::idesc_bf16(128, NV, true, true);
      constexpr uint32_t idN = tc::idesc_bf16(128, 16, true, false);
      const uint32_t base = tc::smem_u32(smem);
      uint32_t it = 0;
      for (int u = 0; u < nsteps && ok; ++u) {
        const int c = chunk_of(u), c0 = c * P.L, len = min(P.L, P.T - c0);
        const int ub = u & 1;
        const uint32_t tU = tU0 + ub * 128, tN = tU + NV;
        // buffer ub was last read by the epilogue of step u - 2
        ok = tc::mbar_wait(&bar[SB_UFREE0 + ub], ((u >> 1) & 1) ^ 1, abort_flag);
        if (!ok) break;
        for (int q = 0; q * SUB < len; ++q, ++it) {
          const uint32_t st = it % Cfg::STAGES, ph = (it / Cfg::STAGES) & 1;
          ok = tc::mbar_wait(&bar[SB_FULL0 + st], ph, abort_flag) &&
               tc::mbar_wait(&bar[SB_SCALED0 + st], ph, abort_flag);
          if (!ok) break;
          tc::tc_fence_after();
          const uint32_t sa = base + st * Cfg::STAGE_BYTES;
#pragma unroll
          for (int k = 0; k < SUB / 16; ++k) {
            const uint64_t a = tc::sdesc_sw128(sa + Cfg::OFF_A + k * 2048, 8192, 1024);
            const uint64_t bhi = tc::sdesc_sw128(sa + Cfg::OFF_BHI + k * 2048, 8192, 1024);
            const uint64_t blo = tc::sdesc_sw128(sa + Cfg::OFF_BLO + k * 2048, 8192, 1024);
            tc::mma_bf16_ss(tU, a, bhi, idU, (q > 0 || k > 0));
            tc::mma_bf16_ss(tU, a, blo, idU, 1);
            if (with_n) {
              const uint64_t nhi = tc::sdesc_sw128(sa + Cfg::OFF_NHI + k * 32, 16, 1024);
              const uint64_t nlo = tc::sdesc_sw128(sa + Cfg::OFF_NLO + k * 32, 16, 1024);
              tc::mma_bf16_ss(tN, a, nhi, idN, (q > 0 || k > 0));
              tc::mma_bf16_ss(tN, a, nlo, idN, 1);
            }
          }
          tc::tc_commit(&bar[SB_EMPTY0 + st]);
        }
        if (!ok) break;
        tc::tc_commit(&bar[SB_U0 + ub]);
      }
      if (!ok) tc::drain_mma(&bar[SB_DRAIN]);  // no product still writes TMEM or reads smem
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ scaling (one token row per thread)
    // The weights of the next sub-tile are computed before this one is waited
    // for, so their global loads overlap the TMA wait and the scaling work.
    const int r = threadIdx.x - 64;  // 0..63
    auto weights = [&](int u, int q, float& wv, float& wn) {
      wv = 0.f;
      wn = 0.f;
      if (u >= nsteps) return;
      const int c = chunk_of(u), c0 = c * P.L, len = min(P.L, P.T - c0);
      const int s = q * SUB + r;
      if (s >= len) return;
      const size_t ct = tokh + c0, t = ct + s;
      if (!BWD) {
        const float g = P.b[ct + len - 1];
        const float mc = EXPV ? P.m[ct + len - 1] : 0.f;
        wv = expf(g - P.b[t] + P.li[t] - mc);
        wn = wv;
      } else {
        const float mprev = EXPV ? chunk_mprev(P.m, ct, c, m0, bh) : 0.f;
        const float mt = EXPV ? P.m[t] : 0.f;
        const float alpha = expf(P.b[t] + mprev - mt) * P.scale;
        wv = alpha * (EXPV ? P.inv_den[t] : 1.f);
        wn = EXPV ? alpha * P.da[t] : 0.f;
      }
    };
    auto nsub = [&](int u) {
      const int c = chunk_of(u), len = min(P.L, P.T - c * P.L);
      return (len + SUB - 1) / SUB;
    };
    uint32_t it = 0;
    float wv_next, wn_next;
    weights(0, 0, wv_next, wn_next);
    for (int u = 0; u < nsteps && ok; ++u) {
      const int ns = nsub(u);
      for (int q = 0; q < ns; ++q, ++it) {
        const uint32_t st = it % Cfg::STAGES, ph = (it / Cfg::STAGES) & 1;
        const float wv = wv_next, wn = wn_next;
        if (q + 1 < ns) weights(u, q + 1, wv_next, wn_next);
        else weights(u + 1, 0, wv_next, wn_next);
        ok = __all_sync(0xffffffffu, tc::mbar_wait(&bar[SB_FULL0 + st], ph, abort_flag));
        if (!ok) break;
        uint8_t* stg = smem + st * Cfg::STAGE_BYTES;
        // y = w v in packed f32x2 products; hi = bf16(y) in one packed conversion per pair,
        // lo = bf16(y - hi) likewise (a bf16 value is the upper half of its f32 bits)
        const uint64_t wv2 = tc::f2_make(wv, wv);
#pragma unroll
        for (int h = 0; h < NV / 64; ++h) {
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const int pch = (jj + r) & 7;
            const uint32_t off = h * 8192 + r * 128 + pch * 16;
            uint4 raw = *reinterpret_cast<const uint4*>(stg + Cfg::OFF_BHI + off);
            uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w}, hi[4], lo[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float x0 = __uint_as_float(w[e] << 16), x1 = __uint_as_float(w[e] & 0xffff0000u);
              const float2 y = tc::f2_split(tc::f2_mul(tc::f2_make(x0, x1), wv2));
              hi[e] = tc::pack_bf16(y.x, y.y);
              lo[e] = tc::pack_bf16(y.x - __uint_as_float(hi[e] << 16),
                                    y.y - __uint_as_float(hi[e] & 0xffff0000u));
            }
            *reinterpret_cast<uint4*>(stg + Cfg::OFF_BHI + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4*>(stg + Cfg::OFF_BLO + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
          }
        }
        if (with_n) {  // row 0 of the K-major normaliser tile: element s at byte 2 s
          const bf16 nh = __float2bfloat16_rn(wn);
          const bf16 nl = __float2bfloat16_rn(wn - __bfloat162float(nh));
          reinterpret_cast<bf16*>(stg + Cfg::OFF_NHI)[r] = nh;
          reinterpret_cast<bf16*>(stg + Cfg::OFF_NLO)[r] = nl;
        }
        tc::fence_proxy_async_smem();
        tc::mbar_arrive(&bar[SB_SCALED0 + st]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue: running state rows
    const int i = 32 * (warp & 3) + lane;  // state row within the tile (TMEM lane)
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const bool valid = dk0 + i < P.dqk;
    // the running state: the forward starts from the initial state (zero without one)
    // (the backward from the final state's gradient, if one is given)
    float S[NV];
    const float* S0 = BWD ? P.dT : P.init.C;
    const float* n0 = BWD ? P.dnT : P.init.n;
    const bool from_init = S0 != nullptr && valid && seg == 0;
#pragma unroll
    for (int j = 0; j < NV; ++j)
      S[j] = from_init ? S0[((size_t)bh * P.dqk + dk0 + i) * P.dhv + dv0 + j] : 0.f;
    float sn = (from_init && with_n) ? n0[(size_t)bh * P.dqk + dk0 + i] : 0.f;
    int nstored = 0;
    for (int u = 0; u < nslots; ++u) {
      const int c = chunk_of(u);
      // store the state at this chunk boundary: rows into the swizzled staging
      // tile, then one TMA store per plane issued by thread 0 of the epilogue
      if (u > 0 || seg == 0) {
      if (nstored > 0)
        ok = __all_sync(0xffffffffu, tc::mbar_wait(&bar[SB_STG_FREE], (nstored - 1) & 1, abort_flag));
      if (!ok) break;
      {
        uint8_t* stg_hi = smem + Cfg::OFF_STG;
        uint8_t* stg_lo = stg_hi + Cfg::STG_PLANE;
#pragma unroll
        for (int j = 0; j < NV; j += 8) {
          uint4 vh, vl;
          uint32_t* ph = reinterpret_cast<uint32_t*>(&vh);
          uint32_t* pl = reinterpret_cast<uint32_t*>(&vl);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float x0 = S[j + 2 * e], x1 = S[j + 2 * e + 1];
            const bf16 h0 = __float2bfloat16_rn(x0), h1 = __float2bfloat16_rn(x1);
            ph[e] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
            pl[e] = tc::pack_bf16(x0 - __bfloat162float(h0), x1 - __bfloat162float(h1));
          }
          const int blk = j >> 6, lc = (j & 63) >> 3;
          const uint32_t off = blk * 16384 + i * 128 + ((lc ^ (i & 7)) << 4);
          *reinterpret_cast<uint4*>(stg_hi + off) = vh;
          *reinterpret_cast<uint4*>(stg_lo + off) = vl;
        }
        if (valid && with_n) P.nout[((size_t)bh * NC + c) * P.dqk + dk0 + i] = sn;
        tc::fence_proxy_async_smem();
        tc::mbar_arrive(&bar[SB_STG_FULL]);
        if (i == 0) {
          ok = tc::mbar_wait(&bar[SB_STG_FULL], nstored & 1, abort_flag);
          if (ok) {
            const int z = bh * NC + c;
            for (int blk = 0; blk < NV / 64; ++blk) {
              tc::tma_store_3d(&tmOhi, stg_hi + blk * 16384, dv0 + blk * 64, dk0, z);
              tc::tma_store_3d(&tmOlo, stg_lo + blk * 16384, dv0 + blk * 64, dk0, z);
            }
            tc::bulk_commit_group();
            tc::bulk_wait_read_all();
            tc::mbar_arrive(&bar[SB_STG_FREE]);
          }
        }
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
      }
      ++nstored;
      }
      if (u == nsteps) break;  // the state leaving this chunk is not needed
      const int c0 = c * P.L, len = min(P.L, P.T - c0);
      const size_t ct = tokh + c0;
      const float g = P.b[ct + len - 1];
      float beta;
      if (EXPV) {
        const float mc = P.m[ct + len - 1];
        const float mp = chunk_mprev(P.m, ct, c, m0, bh);
        beta = (c > 0 || m0 != nullptr) ? expf(g + mp - mc) : 0.f;
      } else {
        beta = expf(g);
      }
      const int ub = u & 1;
      const uint32_t tU = tU0 + ub * 128, tN = tU + NV;
      ok = __all_sync(0xffffffffu, tc::mbar_wait(&bar[SB_U0 + ub], (u >> 1) & 1, abort_flag));
      if (!ok) break;
      tc::tc_fence_after();
#pragma unroll
      for (int ch = 0; ch < NV / 32; ++ch) {
        float v[32];
        tc::tmem_ld32(tU + lane_base + ch * 32, v);
#pragma unroll
        for (int e = 0; e < 32; ++e) S[ch * 32 + e] = fmaf(beta, S[ch * 32 + e], v[e]);
      }
      if (with_n) {
        float v[32];
        tc::tmem_ld32(tN + lane_base, v);  // reads the 16-column block and 16 unused columns
        sn = fmaf(beta, sn, v[0]);
      }
      tc::tc_fence_before();
      tc::mbar_arrive(&bar[SB_UFREE0 + ub]);
    }
    // backward with the initial state's gradient: after the first chunk's contribution
    // the running state is the gradient of the state entering it (this segment's share of
    // it when the walk is split; state_fix adds the rest)
    if (BWD && P.d0 != nullptr && last_seg && ok && valid) {
      float4* dst = reinterpret_cast<float4*>(P.d0 + ((size_t)bh * P.dqk + dk0 + i) * P.dhv + dv0);
#pragma unroll
      for (int j = 0; j < NV; j += 4) dst[j / 4] = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
      if (with_n) P.dn0[(size_t)bh * P.dqk + dk0 + i] = sn;
    }
  }

  if (warp >= 4 && threadIdx.x == 128) tc::bulk_wait_all();  // this thread's TMA stores are done
  if (!ok) abort_flag.raise();
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

// Completion of a split walk: segment k > 0 started from the zero state, so each
// of its stored states lacks the true state E entering the segment carried
// through the segment's decay: the state after j more walk steps is
// local_j + (beta_1 ... beta_j) E (the recurrence S <- beta S + U is linear, and
// with the max state the stabilisers of the betas telescope, so the same factors
// hold for the stored stabilised states).  Segments are completed in order; the
// state entering segment k + 1 is the completed last slot of segment k, and the
// first segment's slots are already complete.  The backward's initial-state
// gradient, written by the last segment, is completed the same way.  One thread
// per eight state elements (and one n element); CUDA cores, HBM-bound.
template <bool BWD, bool EXPV>
__global__ void __launch_bounds__(256) state_fix_kernel(
    bf16* __restrict__ out, float* __restrict__ nout, size_t plane, const float* __restrict__ b,
    const float* __restrict__ m, const float* __restrict__ m0, float* __restrict__ d0,
    float* __restrict__ dn0, int T, int L, int NC, int dqk, int dhv, int seg_len, int nseg) {
  const int bh = blockIdx.y;
  const size_t nel = (size_t)dqk * dhv;
  const int tid = blockIdx.x * blockDim.x + threadIdx.x;
  const size_t e0 = (size_t)tid * 8;
  const bool has_el = e0 < nel;
  const bool has_n = EXPV && nout != nullptr && tid < dqk;
  auto chunk_of = [&](int u) { return BWD ? NC - 1 - u : u; };
  auto beta_of = [&](int c) -> float {
    const size_t ct = (size_t)bh * T + (size_t)c * L;
    const int len = min(L, T - c * L);
    const float g = b[ct + len - 1];
    if (!EXPV) return expf(g);
    const float mc = m[ct + len - 1];
    const float mp = chunk_mprev(m, ct, c, m0, bh);
    return (c > 0 || m0 != nullptr) ? expf(g + mp - mc) : 0.f;
  };
  auto load8 = [&](int u, float (&x)[8]) {
    const size_t o = ((size_t)bh * NC + chunk_of(u)) * nel + e0;
    const uint4 h4 = *reinterpret_cast<const uint4*>(out + o);
    const uint4 l4 = *reinterpret_cast<const uint4*>(out + plane + o);
    const uint32_t hw[4] = {h4.x, h4.y, h4.z, h4.w}, lw[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 h2 = *reinterpret_cast<const __nv_bfloat162*>(&hw[e]);
      const __nv_bfloat162 l2 = *reinterpret_cast<const __nv_bfloat162*>(&lw[e]);
      x[2 * e] = __bfloat162float(h2.x) + __bfloat162float(l2.x);
      x[2 * e + 1] = __bfloat162float(h2.y) + __bfloat162float(l2.y);
    }
  };
  auto store8 = [&](int u, const float (&x)[8]) {
    const size_t o = ((size_t)bh * NC + chunk_of(u)) * nel + e0;
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const bf16 h0 = __float2bfloat16_rn(x[2 * e]), h1 = __float2bfloat16_rn(x[2 * e + 1]);
      hw[e] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
      const __nv_bfloat162 l2 = __floats2bfloat162_rn(x[2 * e] - __bfloat162float(h0),
                                                      x[2 * e + 1] - __bfloat162float(h1));
      lw[e] = *reinterpret_cast<const uint32_t*>(&l2);
    }
    *reinterpret_cast<uint4*>(out + o) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4*>(out + plane + o) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  };
  auto nslot = [&](int u) -> float* { return nout + ((size_t)bh * NC + chunk_of(u)) * dqk + tid; };
  // the state entering the second segment: stored by the first, which is complete
  float E[8] = {}, En = 0.f;
  if (has_el) load8(seg_len, E);
  if (has_n) En = *nslot(seg_len);
  for (int sg = 1; sg < nseg; ++sg) {
    const int us = sg * seg_len, nlocal = min(seg_len, NC - us);
    const bool last = us + nlocal == NC;
    const int nslots = last ? nlocal : nlocal + 1;  // slot us is complete already
    float D = 1.f;
    for (int k = 1; k < nslots; ++k) {
      D *= beta_of(chunk_of(us + k - 1));
      if (has_el) {
        float x[8];
        load8(us + k, x);
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = fmaf(D, E[e], x[e]);
        store8(us + k, x);
        if (k == nslots - 1 && !last) {
#pragma unroll
          for (int e = 0; e < 8; ++e) E[e] = x[e];
        }
      }
      if (has_n) {
        float* pn = nslot(us + k);
        const float nv = fmaf(D, En, *pn);
        *pn = nv;
        if (k == nslots - 1 && !last) En = nv;
      }
    }
    if (last && BWD && d0 != nullptr) {
      // the initial state's gradient: one step more, through the first chunk
      D *= beta_of(chunk_of(NC - 1));
      if (has_el) {
        float* pd = d0 + (size_t)bh * nel + e0;
#pragma unroll
        for (int e = 0; e < 8; ++e) pd[e] = fmaf(D, E[e], pd[e]);
      }
      if (has_n && dn0 != nullptr) dn0[(size_t)bh * dqk + tid] = fmaf(D, En, dn0[(size_t)bh * dqk + tid]);
    }
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

// Segments of a split state walk: enough for the CTAs of all heads to fill the two
// slots per SM of the 148 SMs, with at least four chunks per segment (1: no split).
// A function of the problem alone, so the launch plan knows it without a device.
static void state_split(const Problem& p, int& seg_len, int& nseg) {
  const int ctas = (p.dhv / 64) * ((p.dqk + 127) / 128) * p.BH;
  constexpr int kSlots = 2 * 148;
  int want = kSlots / (ctas > 0 ? ctas : 1);
  if (want > p.NC / 4) want = p.NC / 4;
  if (want < 1) want = 1;
  seg_len = (p.NC + want - 1) / want;
  nseg = (p.NC + seg_len - 1) / seg_len;
}

bool state_split_needed(const Problem& p) {
  int seg_len = 0, nseg = 0;
  state_split(p, seg_len, nseg);
  return nseg > 1;
}

bool state_tc_supported(const Problem& p) {
  return p.bf16() && (p.dqk == 64 || p.dqk == 128 || p.dqk == 256) && (p.dhv % 64 == 0);
}

template <bool BWD, bool EXPV, int NV>
static cudaError_t launch_state_tc(const Problem& p, const void* A, const void* B, bf16* out,
                                   float* nout, const float* b, const float* li, const float* m,
                                   const float* inv_den, const float* da, const InitState& init,
                                   float* d0, float* dn0, const float* dT, const float* dnT,
                                   cudaStream_t s) {
  using Cfg = StateTcCfg<NV>;
  CUtensorMap tA, tB, tOh, tOl;
  const uint64_t plane = (uint64_t)p.BH * p.NC * p.dqk * p.dhv;
  const uint64_t BHNC = (uint64_t)p.BH * p.NC;
  if (!make_tmap_3d_bf16(&tA, A, p.dqk, p.T, p.BH, 64, 64) ||
      !make_tmap_3d_bf16(&tB, B, p.dhv, p.T, p.BH, 64, 64) ||
      !make_tmap_3d_bf16(&tOh, out, p.dhv, p.dqk, BHNC, 64, 128) ||
      !make_tmap_3d_bf16(&tOl, out + plane, p.dhv, p.dqk, BHNC, 64, 128))
    return cudaErrorInvalidValue;
  StateTcParams P;
  P.b = b; P.li = li; P.m = m; P.inv_den = inv_den; P.da = da;
  P.out = out; P.nout = nout;
  P.plane = (size_t)p.BH * p.NC * p.dqk * p.dhv;
  P.T = p.T; P.L = p.L; P.NC = p.NC; P.dqk = p.dqk; P.dhv = p.dhv; P.BH = p.BH;
  state_split(p, P.seg_len, P.nseg);
  P.scale = p.scale;
  P.init = init;
  P.d0 = d0;
  P.dn0 = dn0;
  P.dT = dT;
  P.dnT = dnT;
  P.epoch = next_epoch();
  auto kern = state_tc_kernel<BWD, EXPV, NV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)(p.dhv / NV), (unsigned)((p.dqk + 127) / 128), (unsigned)(p.BH * P.nseg)),
      block(256);
  kern<<<grid, block, Cfg::SMEM, s>>>(tA, tB, tOh, tOl, P);
  return cudaGetLastError();
}

// 64 value columns per CTA keep the fp32 running state (64 registers per
// thread) inside the 128-register budget of two CTAs per SM.
template <bool BWD, bool EXPV>
static cudaError_t launch_state_tc_nv(const Problem& p, const void* A, const void* B, bf16* out,
                                      float* nout, const float* b, const float* li, const float* m,
                                      const float* inv_den, const float* da, const InitState& init,
                                      float* d0, float* dn0, const float* dT, const float* dnT,
                                      cudaStream_t s) {
  return launch_state_tc<BWD, EXPV, 64>(p, A, B, out, nout, b, li, m, inv_den, da, init, d0, dn0,
                                        dT, dnT, s);
}

cudaError_t launch_state_fwd_tc(const Problem& p, const FwdArgs& a, cudaStream_t s) {
  if (p.exp_variant())
    return launch_state_tc_nv<false, true>(p, a.k, a.v, (bf16*)a.C, a.n, a.b, a.li, a.m, nullptr,
                                           nullptr, a.init, nullptr, nullptr, nullptr, nullptr, s);
  return launch_state_tc_nv<false, false>(p, a.k, a.v, (bf16*)a.C, a.n, a.b, a.li, a.m, nullptr,
                                          nullptr, a.init, nullptr, nullptr, nullptr, nullptr, s);
}

cudaError_t launch_state_bwd_tc(const Problem& p, const BwdArgs& a, cudaStream_t s) {
  if (p.exp_variant())
    return launch_state_tc_nv<true, true>(p, a.q, a.dh, (bf16*)a.dC, a.dn, a.b, a.li, a.m,
                                          a.inv_den, a.da, a.init, a.dC0, a.dn0, a.dCT, a.dnT, s);
  return launch_state_tc_nv<true, false>(p, a.q, a.dh, (bf16*)a.dC, a.dn, a.b, a.li, a.m,
                                         a.inv_den, a.da, a.init, a.dC0, a.dn0, a.dCT, a.dnT, s);
}

template <bool BWD, bool EXPV>
static cudaError_t launch_fix(const Problem& p, bf16* out, float* nout, const float* b,
                              const float* m, const InitState& init, float* d0, float* dn0,
                              cudaStream_t s) {
  int seg_len = 0, nseg = 0;
  state_split(p, seg_len, nseg);
  if (nseg < 2) return cudaErrorInvalidValue;  // the plan launches this only for a split walk
  const size_t plane = (size_t)p.BH * p.NC * p.dqk * p.dhv;
  const size_t nel = (size_t)p.dqk * p.dhv;
  const float* m0 = (init.on() && EXPV) ? init.m : nullptr;
  dim3 grid((unsigned)((nel / 8 + 255) / 256), (unsigned)p.BH), block(256);
  state_fix_kernel<BWD, EXPV><<<grid, block, 0, s>>>(out, nout, plane, b, m, m0, d0, dn0, p.T, p.L,
                                                     p.NC, p.dqk, p.dhv, seg_len, nseg);
  return cudaGetLastError();
}

cudaError_t launch_state_fwd_fix(const Problem& p, const FwdArgs& a, cudaStream_t s) {
  if (p.exp_variant())
    return launch_fix<false, true>(p, (bf16*)a.C, a.n, a.b, a.m, a.init, nullptr, nullptr, s);
  return launch_fix<false, false>(p, (bf16*)a.C, nullptr, a.b, a.m, a.init, nullptr, nullptr, s);
}

cudaError_t launch_state_bwd_fix(const Problem& p, const BwdArgs& a, cudaStream_t s) {
  if (p.exp_variant())
    return launch_fix<true, true>(p, (bf16*)a.dC, a.dn, a.b, a.m, a.init, a.dC0, a.dn0, s);
  return launch_fix<true, false>(p, (bf16*)a.dC, nullptr, a.b, a.m, a.init, a.dC0, nullptr, s);
}

cudaError_t fetch_tc_state_error(unsigned int* flag) {
  return cudaMemcpyFromSymbol(flag, g_tc_state_error, sizeof(unsigned int));
}

}  // namespace mlstm
