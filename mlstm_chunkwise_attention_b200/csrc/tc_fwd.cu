// TFLA intra-chunk output kernel (K-c) on the fifth-generation tensor cores,
// for chunks that fit one 128-row tile (chunk 64 and 128): the single-level
// ("limit_chunk") form, where one tile holds a whole chunk's queries and keys.
// "Tiled Flash Linear Attention: More Efficient Linear RNN and xLSTM Kernels"
// (TFLA summary page, Approach and Measured effects; arXiv abstract page,
// Abstract).  One CTA owns one chunk and a slice of up to 128 value columns:
//
//   S    = Q K^T                          (tcgen05, bf16 in smem -> fp32 TMEM)
//   P    = S * exp(b_t - b_s + log i_s - m_t) / sqrt(d_qk), causal (registers)
//   O    = P V                            (tcgen05, P staged to smem in bf16)
//   O   += (alpha_t Q / sqrt(d_qk)) C_prev (inter-chunk term, hi and lo planes)
//   h_t  = O_t / max(|alpha_t q'_t.n_prev + sum_s P_ts|, exp(-m_t))   (mLSTMexp)
//
// A 64-token chunk occupies the first 64 rows of the tile: the score product
// has N = 64 keys, P V contracts over 64 keys, rows 64..127 compute nothing
// that is kept, and h leaves through a 64-row store.  The state entering the
// chunk is multiplied in both of its bf16 planes (hi + lo keeps about 16
// mantissa bits): where the normaliser nearly cancels, h = O / den amplifies
// the rounding of the inter-chunk term.
//
// Warp roles: warp 0 issues TMA loads, warp 1 allocates TMEM and issues the
// MMAs (one thread), warps 2..5 own one query row per thread (TMEM lane),
// turn S into P, and run the epilogue.  Every mbarrier wait is bounded; on a
// timeout the kernel sets an error flag and winds down.
#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace mlstm {

static __device__ unsigned int g_tc_fwd_error;

namespace {

constexpr float kLog2e = 1.4426950408889634f;

// Shared memory, 96 KB at d 128 so two CTAs fit on an SM: the K region takes
// K, then P once S is done, then the lo plane of C_prev once P V is done; the
// V region takes V, then the hi plane of C_prev, then the h staging tile.
template <int DQK, int DV>
struct OutTcCfg {
  static constexpr int KB = DQK / 64;  // 64-column blocks of Q and K
  static constexpr int VB = DV / 64;   // 64-column blocks of the V / C slice
  static constexpr int Q_BYTES = KB * 16384;
  static constexpr int K_BYTES = KB * 16384;
  static constexpr int C_BYTES = VB * DQK * 128;
  static constexpr int P_TILE = 2 * 16384;
  static constexpr int KC_BYTES = K_BYTES > P_TILE ? K_BYTES : P_TILE;
  static constexpr int V_BYTES = VB * 16384;  // one V tile: the bytes its TMA loads deliver
  static constexpr int V_REGION = V_BYTES > C_BYTES ? V_BYTES : C_BYTES;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KC = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_KC + KC_BYTES;
  static constexpr int OFF_BAR = OFF_V + V_REGION;  // 16 mbarriers
  static constexpr int OFF_TMEM = OFF_BAR + 16 * 8;
  static constexpr int OFF_NVEC = OFF_TMEM + 16;
  static constexpr int OFF_COLF = OFF_NVEC + DQK * 4;
  static constexpr size_t SMEM = 1024 + OFF_COLF + 128 * 4;
  static constexpr uint32_t TMEM_COLS = 256;  // S in [0, 128), O in [128, 128 + DV)
  static_assert(C_BYTES <= KC_BYTES, "the lo plane of C_prev must fit the K region");
};

enum { B_Q = 0, B_K, B_V, B_C, B_S, B_P, B_PV, B_QS, B_O, B_STG, B_DRAIN, B_COUNT };
static_assert(B_COUNT <= 16, "barrier slots");

}  // namespace

template <int DQK, int DV, bool EXPV>
__global__ void __launch_bounds__(192, 2) output_fwd_tc_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_chi,
    const __grid_constant__ CUtensorMap tm_clo, const __grid_constant__ CUtensorMap tm_h,
    const float* __restrict__ gb, const float* __restrict__ gli, const float* __restrict__ gm,
    const float* __restrict__ gn, float* __restrict__ abar_out, int T, int L, int NC, float scale,
    float log2_scale, bool has_init, const float* __restrict__ m0, unsigned int epoch) {
  using Cfg = OutTcCfg<DQK, DV>;
  const tc::Abort abort_flag{&g_tc_fwd_error, epoch};
  // NKEY keys per chunk (64 or 128): the score's N, P V's contraction extent
  const int NKEY = L < 128 ? L : 128;

  const int bh = (int)(blockIdx.x / NC), c = (int)(blockIdx.x % NC);
  const int c0 = c * L;
  const int len = min(L, T - c0);
  // an earlier CTA of this launch gave up: the whole block leaves together
  if (__syncthreads_or(threadIdx.x == 0 && abort_flag.raised())) return;
  const int dv0 = blockIdx.y * DV;
  const size_t tok0 = (size_t)bh * T + c0;
  const bool has_prev = c > 0 || has_init;  // a state enters this chunk

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + Cfg::OFF_Q;
  uint8_t* sKC = smem + Cfg::OFF_KC;  // K, then P, then the lo plane of C_prev (or h)
  uint8_t* sV = smem + Cfg::OFF_V;    // V, then the hi plane of C_prev (then h)
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_TMEM);
  float* nvec = reinterpret_cast<float*>(smem + Cfg::OFF_NVEC);
  float* colf = reinterpret_cast<float*>(smem + Cfg::OFF_COLF);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < B_COUNT; ++i) {
      const uint32_t cnt = (i == B_P || i == B_QS || i == B_STG) ? 128u : 1u;
      tc::mbar_init(&bar[i], cnt);
    }
    tc::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tc::tmem_relinquish();
  }
  // column factors (log i_s - b_s) log2(e) of the chunk's keys
  if (warp >= 2) {
    const int gt = threadIdx.x - 64;
    colf[gt] = gt < len ? (gli[tok0 + gt] - gb[tok0 + gt]) * kLog2e : -INFINITY;
    if (EXPV && has_prev)
      for (int i = gt; i < DQK; i += 128) nvec[i] = gn[((size_t)bh * NC + c) * DQK + i];
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tO = tmem + 128;
  bool ok = true;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tc::prefetch_tmap(&tm_q);
      tc::prefetch_tmap(&tm_k);
      tc::prefetch_tmap(&tm_v);
      tc::mbar_arrive_expect_tx(&bar[B_Q], Cfg::Q_BYTES);
      for (int kb = 0; kb < Cfg::KB; ++kb) tc::tma_load_3d(sQ + kb * 16384, &tm_q, &bar[B_Q], kb * 64, c0, bh);
      tc::mbar_arrive_expect_tx(&bar[B_K], Cfg::K_BYTES);
      for (int kb = 0; kb < Cfg::KB; ++kb) tc::tma_load_3d(sKC + kb * 16384, &tm_k, &bar[B_K], kb * 64, c0, bh);
      tc::mbar_arrive_expect_tx(&bar[B_V], Cfg::V_BYTES);
      for (int vb = 0; vb < Cfg::VB; ++vb)
        tc::tma_load_3d(sV + vb * 16384, &tm_v, &bar[B_V], dv0 + vb * 64, c0, bh);
      bool c_issued = false;
      if (has_prev) {
        // both planes of C_prev once P V is done: hi where V was, lo where P was
        ok = tc::mbar_wait(&bar[B_PV], 0, abort_flag);
        if (ok) {
          c_issued = true;
          tc::mbar_arrive_expect_tx(&bar[B_C], 2 * Cfg::C_BYTES);
          for (int vb = 0; vb < Cfg::VB; ++vb) {
            tc::tma_load_3d(sV + vb * DQK * 128, &tm_chi, &bar[B_C], dv0 + vb * 64, 0, bh * NC + c);
            tc::tma_load_3d(sKC + vb * DQK * 128, &tm_clo, &bar[B_C], dv0 + vb * 64, 0, bh * NC + c);
          }
        }
      }
      // do not leave while a copy this thread issued may still be landing
      if (ok) ok = tc::mbar_wait(&bar[B_V], 0, abort_flag);
      if (ok && has_prev) ok = tc::mbar_wait(&bar[B_C], 0, abort_flag);
      if (!ok) {  // gave up: the copies still in flight land before the CTA exits
        tc::drain_last(&bar[B_Q], 1);
        tc::drain_last(&bar[B_K], 1);
        tc::drain_last(&bar[B_V], 1);
        tc::drain_last(&bar[B_C], c_issued ? 1u : 0u);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idS = tc::idesc_bf16(128, NKEY, false, false);
      constexpr uint32_t idO = tc::idesc_bf16(128, DV, false, true);
      const uint32_t aQ = tc::smem_u32(sQ), aKC = tc::smem_u32(sKC), aV = tc::smem_u32(sV);
      ok = tc::mbar_wait(&bar[B_Q], 0, abort_flag) && tc::mbar_wait(&bar[B_K], 0, abort_flag);
      if (ok) {
        tc::tc_fence_after();
#pragma unroll
        for (int k = 0; k < DQK / 16; ++k) {
          const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
          tc::mma_bf16_ss(tS, tc::sdesc_sw128(aQ + off, 16, 1024), tc::sdesc_sw128(aKC + off, 16, 1024),
                          idS, k > 0);
        }
        tc::tc_commit(&bar[B_S]);
        ok = tc::mbar_wait(&bar[B_P], 0, abort_flag) && tc::mbar_wait(&bar[B_V], 0, abort_flag);
      }
      if (ok) {
        tc::tc_fence_after();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          if (16 * k < NKEY) {
            const uint32_t offp = (k >> 2) * 16384 + (k & 3) * 32;
            tc::mma_bf16_ss(tO, tc::sdesc_sw128(aKC + offp, 16, 1024),
                            tc::sdesc_sw128(aV + k * 2048, 16384, 1024), idO, k > 0);
          }
        }
        tc::tc_commit(&bar[B_PV]);
      }
      if (ok && has_prev) {
        ok = tc::mbar_wait(&bar[B_QS], 0, abort_flag) && tc::mbar_wait(&bar[B_C], 0, abort_flag);
        if (ok) {
          tc::tc_fence_after();
#pragma unroll
          for (int k = 0; k < DQK / 16; ++k) {
            const uint64_t a = tc::sdesc_sw128(aQ + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
            tc::mma_bf16_ss(tO, a, tc::sdesc_sw128(aV + k * 2048, DQK * 128, 1024), idO, 1);
            tc::mma_bf16_ss(tO, a, tc::sdesc_sw128(aKC + k * 2048, DQK * 128, 1024), idO, 1);
          }
        }
      }
      tc::tc_commit(&bar[B_O]);
      if (!ok) tc::drain_mma(&bar[B_DRAIN]);  // no product still writes TMEM or reads smem
    }
  } else {
    // ------------------------------------------------------------ gate rows + epilogue
    const int row = 32 * (warp & 3) + lane;  // TMEM lane == query row of the tile
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const bool valid = row < len;
    const size_t tok = tok0 + row;
    const float bt = valid ? gb[tok] : 0.f;
    const float mt = (EXPV && valid) ? gm[tok] : 0.f;
    const float mprev = EXPV ? chunk_mprev(gm, tok0, c, m0, bh) : 0.f;
    const float r2 = valid ? (bt - mt) * kLog2e + log2_scale : -INFINITY;
    const float qfac = (valid && has_prev) ? expf(bt + mprev - mt) * scale : 0.f;
    const uint32_t aP = tc::smem_u32(sKC), aQ = tc::smem_u32(sQ);
    float rowsum = 0.f;

    ok = __all_sync(0xffffffffu, tc::mbar_wait(&bar[B_S], 0, abort_flag));
    if (ok) {
      tc::tc_fence_after();
#pragma unroll 1
      for (int ch = 0; ch < NKEY / 32; ++ch) {
        float sv[32];
        tc::tmem_ld32(tS + lane_base + ch * 32, sv);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const int s0 = ch * 32 + i;
          float p0 = sv[i] * tc::ex2(r2 + colf[s0]);
          float p1 = sv[i + 1] * tc::ex2(r2 + colf[s0 + 1]);
          if (s0 > row) p0 = 0.f;
          if (s0 + 1 > row) p1 = 0.f;
          if (EXPV) rowsum += p0 + p1;
          pk[i >> 1] = tc::pack_bf16(p0, p1);
        }
        const int kb = ch >> 1;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int lc = (ch & 1) * 4 + q4;
          const uint32_t addr = aP + kb * 16384 + row * 128 + ((lc ^ (row & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[4 * q4]),
                       "r"(pk[4 * q4 + 1]), "r"(pk[4 * q4 + 2]), "r"(pk[4 * q4 + 3])
                       : "memory");
        }
      }
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      tc::mbar_arrive(&bar[B_P]);
    }

    // inter-chunk operand: scale the query rows by alpha_t / sqrt(d_qk) in place (the
    // score product that read Q is done)
    float inter_norm = 0.f;
    if (ok && has_prev) {
#pragma unroll 1
      for (int kb = 0; kb < Cfg::KB; ++kb) {
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int pch = (jj + row) & 7;
          const uint32_t addr = aQ + kb * 16384 + row * 128 + pch * 16;
          uint32_t w[4];
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                       : "r"(addr));
          const int col0 = kb * 64 + ((pch ^ (row & 7)) << 3);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            __nv_bfloat162 v2 = *reinterpret_cast<__nv_bfloat162*>(&w[e]);
            const float x0 = __bfloat162float(v2.x) * qfac;
            const float x1 = __bfloat162float(v2.y) * qfac;
            if (EXPV) inter_norm += x0 * nvec[col0 + 2 * e] + x1 * nvec[col0 + 2 * e + 1];
            w[e] = tc::pack_bf16(x0, x1);
          }
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w[0]),
                       "r"(w[1]), "r"(w[2]), "r"(w[3])
                       : "memory");
        }
      }
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bar[B_QS]);
    }

    if (ok) ok = __all_sync(0xffffffffu, tc::mbar_wait(&bar[B_O], 0, abort_flag));
    if (ok) {
      tc::tc_fence_after();
      float inv = 1.f;
      if (EXPV) {
        const float a = inter_norm + rowsum;
        inv = 1.f / fmaxf(fabsf(a), expf(-mt));
        if (blockIdx.y == 0 && valid) abar_out[tok] = a;
      }
      // h goes through an idle region and one TMA store per 64-column block (NKEY rows: a
      // 64-token chunk leaves the next chunk's rows alone): the V region once the inter
      // product has read C_prev's hi plane from it, else the K / P region.  (Staged over
      // V right after P V, the first 16 rows of h were measured to come out zero.)
      uint8_t* sH = has_prev ? sV : sKC;
      const uint32_t aH = tc::smem_u32(sH);
#pragma unroll 1
      for (int ch = 0; ch < DV / 32; ++ch) {
        float ov[32];
        tc::tmem_ld32(tO + lane_base + ch * 32, ov);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int col = ch * 32 + q4 * 8, blk = col >> 6, lc = (col & 63) >> 3;
          const uint32_t addr = aH + blk * 16384 + row * 128 + ((lc ^ (row & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                       "r"(tc::pack_bf16(ov[8 * q4 + 0] * inv, ov[8 * q4 + 1] * inv)),
                       "r"(tc::pack_bf16(ov[8 * q4 + 2] * inv, ov[8 * q4 + 3] * inv)),
                       "r"(tc::pack_bf16(ov[8 * q4 + 4] * inv, ov[8 * q4 + 5] * inv)),
                       "r"(tc::pack_bf16(ov[8 * q4 + 6] * inv, ov[8 * q4 + 7] * inv))
                       : "memory");
        }
      }
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bar[B_STG]);
      if (row == 0) {
        ok = tc::mbar_wait(&bar[B_STG], 0, abort_flag);
        if (ok) {
          for (int blk = 0; blk < DV / 64; ++blk)
            tc::tma_store_3d(&tm_h, sH + blk * 16384, dv0 + blk * 64, c0, bh);
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

bool output_fwd_tc_supported(const Problem& p) {
  return p.bf16() && (p.L == 64 || p.L == 128) && (p.dqk == 64 || p.dqk == 128 || p.dqk == 256) &&
         (p.dhv % 64 == 0);
}

template <int DQK, int DV, bool EXPV>
static cudaError_t launch_out_tc(const Problem& p, const FwdArgs& a, cudaStream_t s) {
  using Cfg = OutTcCfg<DQK, DV>;
  const bf16* C = (const bf16*)a.C;
  const size_t plane = (size_t)p.BH * p.NC * p.dqk * p.dhv;
  CUtensorMap tq, tk, tv, tch, tcl, th;
  const uint32_t rows = p.L < 128 ? (uint32_t)p.L : 128u;  // one chunk per tile
  if (!make_tmap_3d_bf16(&th, a.h, p.dhv, p.T, p.BH, 64, rows) ||
      !make_tmap_3d_bf16(&tq, a.q, p.dqk, p.T, p.BH, 64, 128) ||
      !make_tmap_3d_bf16(&tk, a.k, p.dqk, p.T, p.BH, 64, 128) ||
      !make_tmap_3d_bf16(&tv, a.v, p.dhv, p.T, p.BH, 64, 128) ||
      !make_tmap_3d_bf16(&tch, C, p.dhv, p.dqk, (uint64_t)p.BH * p.NC, 64, DQK) ||
      !make_tmap_3d_bf16(&tcl, C + plane, p.dhv, p.dqk, (uint64_t)p.BH * p.NC, 64, DQK))
    return cudaErrorInvalidValue;
  auto kern = output_fwd_tc_kernel<DQK, DV, EXPV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)(p.BH * p.NC), (unsigned)(p.dhv / DV)), block(192);
  kern<<<grid, block, Cfg::SMEM, s>>>(tq, tk, tv, tch, tcl, th, a.b, a.li, a.m, a.n, a.abar, p.T, p.L,
                                      p.NC, p.scale, log2f(p.scale), a.init.on(),
                                      a.init.on() ? a.init.m : nullptr, next_epoch());
  return cudaGetLastError();
}

template <int DQK, bool EXPV>
static cudaError_t launch_out_tc_dv(const Problem& p, const FwdArgs& a, cudaStream_t s) {
  if (p.dhv == 64) return launch_out_tc<DQK, 64, EXPV>(p, a, s);
  return launch_out_tc<DQK, 128, EXPV>(p, a, s);
}

cudaError_t launch_output_fwd_tc(const Problem& p, const FwdArgs& a, cudaStream_t s) {
  const bool e = p.exp_variant();
  switch (p.dqk) {
    case 64: return e ? launch_out_tc_dv<64, true>(p, a, s) : launch_out_tc_dv<64, false>(p, a, s);
    case 128: return e ? launch_out_tc_dv<128, true>(p, a, s) : launch_out_tc_dv<128, false>(p, a, s);
    case 256: return e ? launch_out_tc_dv<256, true>(p, a, s) : launch_out_tc_dv<256, false>(p, a, s);
    default: return cudaErrorInvalidValue;
  }
}

// Self-test of the failure report: one thread waits on an mbarrier that nothing
// completes, its bounded wait runs out, and it raises its launch's flag in this
// kernel family, as a chunk-128 output CTA whose hand-over never came would.
__global__ void selftest_timeout_kernel(unsigned int epoch) {
  __shared__ uint64_t bar;
  const tc::Abort abort_flag{&g_tc_fwd_error, epoch};
  tc::mbar_init(&bar, 1);
  tc::fence_mbar_init();
  if (!tc::mbar_wait(&bar, 0, abort_flag)) abort_flag.raise();
}

cudaError_t launch_selftest_timeout(cudaStream_t s) {
  selftest_timeout_kernel<<<1, 1, 0, s>>>(next_epoch());
  return cudaGetLastError();
}

cudaError_t fetch_tc_fwd_error(unsigned int* flag) {
  return cudaMemcpyFromSymbol(flag, g_tc_fwd_error, sizeof(unsigned int));
}

}  // namespace mlstm
