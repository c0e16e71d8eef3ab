// Forward walker for chunk 128 (d_qk = d_hv = 128, bf16): the inter-chunk state
// recurrence (K-b) and the TFLA output (K-c) of every chunk in one pass.
//
// One CTA per head walks the chunks in order, holding the state entering the
// current chunk, C_c (fp32, d_qk x d_hv), in TMEM and n_c (mLSTMexp) in
// registers.  At chunk c it stages C_c as hi and lo bf16 planes (stored as the
// saved state the backward reads, and the hi plane is the inter-chunk operand),
// computes the chunk's outputs
//   S = Q K^T, P = S * exp(b_t - b_s + log i_s - m_t) / sqrt(d_qk) (causal),
//   O = alpha_t / sqrt(d_qk) Q C_c + P V,
//   h_t = O_t / max(|alpha_t q_t.n_c / sqrt(d_qk) + sum_s P_ts|, exp(-m_t))  (mLSTMexp)
// as the chunk-128 output kernel of tc_fwd.cu does, then updates
//   C_{c+1} = beta_c C_c + K^T diag(w) V,  n_{c+1} = beta_c n_c + K^T w
// on the tensor core, w_s = exp(g_c - b_s + log i_s - m_c), as (diag(w) K)^T V so
// that the update does not wait for P V to finish reading V.  The states never
// make a round trip through HBM between the two halves of the forward, and q,
// k, v are read once.  "Tiled Flash Linear Attention" (TFLA summary page,
// Problem: materialised chunk states cost IO; Approach).
//
// Roles: one thread (warp 0) issues the MMAs; eight row warps, two per TMEM lane
// quarter, each own one token or state row (the TMEM lane) and half of its
// columns; one row thread issues the TMA loads and stores.  Hand-overs:
//   rows: stage C_c -> A, next gate factors | P transform, inter rescale -> B |
//         w K -> D | h out
//   MMA:  Q K^T, K^T w (hi, lo) | A: Q C_c (hi), Q n_c (hi, lo) | B: P V |
//         D: C += (w K)^T V (hi, lo)
// The next chunk's gate factors (and w as the n-update operand) are written while the
// first products run, before the hand-over D, so the next chunk's n update can start as
// soon as its tiles land.
// Two K/V buffer sets alternate between chunks; the set a chunk does not use
// holds its C staging, and takes the next chunk's K and V as soon as the inter
// product and the saved-state store have read it.  Every wait is bounded; on a
// timeout the kernel raises its error flag and winds down.
#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"
#include "walk_common.cuh"

namespace mlstm {

static __device__ unsigned int g_tc_fwalk_error;

namespace {

constexpr float kLog2e = 1.4426950408889634f;
using walk::sw_off;
using walk::TILE;

// Shared memory: Q tile; two K/V sets (K at +0, V at +TILE); the w K lo plane;
// per-token factors; the N = 16 operand tiles of n (one) and w (two, by chunk parity).
struct FwalkCfg {
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_SET0 = TILE, OFF_SET1 = 3 * TILE;
  static constexpr int OFF_WL = 5 * TILE;
  static constexpr int OFF_F = 6 * TILE;                // NF arrays of 128 floats
  static constexpr int NF = 8;
  static constexpr int OFF_NT = OFF_F + NF * 128 * 4;   // 1024-aligned: 16 x 128 bf16 K-major
  static constexpr int N16_BYTES = 4096;
  static constexpr int OFF_WT = OFF_NT + N16_BYTES;     // two buffers
  static constexpr int OFF_BAR = OFF_WT + 2 * N16_BYTES;
  static constexpr int OFF_TMEM = OFF_BAR + 8 * 8;
  static constexpr size_t SMEM = 1024 + OFF_TMEM + 16;
  static constexpr uint32_t TMEM_COLS = 512;  // C, S / P, O, q.n (16), K^T w (2 x 16)
};

// Per chunk (buffer c & 1, written a chunk ahead): the key factors cf_s = (log i_s - b_s)
// log2 e, their maxima M over each 32-key block (F_MB, 4 per buffer) and 2^(cf_s - M);
// the two halves' row-sum shares.
enum { F_CF0 = 0, F_CF1, F_KP0, F_KP1, F_RS0, F_RS1, F_MB };
// mbarriers: Q tile, K/V sets, rows -> MMA (A, B), rows -> MMA (D), MMA -> rows
// (after A, B), state update done.  Each barrier's phases alternate with its waiter.
// BF_DRAIN: the MMA thread's last commit when it gives up.
enum { BF_Q = 0, BF_KV0, BF_KV1, BF_R, BF_D, BF_M, BF_S, BF_DRAIN, BF_COUNT };
static_assert(BF_COUNT <= 8, "barrier slots");

}  // namespace

struct FwalkParams {
  const float *b, *li, *m;  // per token [BH, T] (gate_prep)
  float* abar;              // [BH, T] alpha q.n + sum P (mLSTMexp)
  float* n;                 // [BH, NC, dqk] n entering each chunk (mLSTMexp)
  InitState init;           // the state entering the first chunk (C null: zero)
  int T, NC;
  float scale, log2_scale;
  unsigned int epoch;  // this launch's abort epoch
};

template <bool EXPV>
__global__ void __launch_bounds__(288, 1) fwd_walk_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmH,
    const __grid_constant__ CUtensorMap tmChi, const __grid_constant__ CUtensorMap tmClo,
    const FwalkParams P) {
  using Cfg = FwalkCfg;
  const tc::Abort abort_flag{&g_tc_fwalk_error, P.epoch};
  if (__syncthreads_or(threadIdx.x == 0 && abort_flag.raised())) return;
  const int bh = blockIdx.x;
  const int NC = P.NC;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + Cfg::OFF_Q;
  uint8_t* sWL = smem + Cfg::OFF_WL;
  float* F = reinterpret_cast<float*>(smem + Cfg::OFF_F);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_TMEM);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the K/V set of chunk c, and the set holding its C staging (hi plane, lo plane at +TILE)
  auto set_of = [&](int c) { return smem + ((c & 1) ? Cfg::OFF_SET1 : Cfg::OFF_SET0); };
  auto stg_of = [&](int c) { return smem + ((c & 1) ? Cfg::OFF_SET0 : Cfg::OFF_SET1); };

  if (threadIdx.x == 0) {
    for (int i = 0; i < BF_COUNT; ++i) tc::mbar_init(&bar[i], (i == BF_R || i == BF_D) ? 256u : 1u);
    tc::fence_mbar_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // K^T w of chunk c goes to tNU + 16 (c & 1): the rows read the previous chunk's after its
  // state update, which may come after this chunk's first products
  const uint32_t tC = tmem, tS = tmem + 128, tO = tmem + 256, tN = tmem + 384, tNU = tmem + 400;
  bool ok = true;

  if (warp == 0) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idKK = tc::idesc_bf16(128, 128, false, false);  // A, B K-major
      constexpr uint32_t idKM = tc::idesc_bf16(128, 128, false, true);   // B MN-major
      constexpr uint32_t idMM = tc::idesc_bf16(128, 128, true, true);    // A, B MN-major
      constexpr uint32_t idNK = tc::idesc_bf16(128, 16, false, false);   // N = 16, A K-major
      constexpr uint32_t idNM = tc::idesc_bf16(128, 16, true, false);    // N = 16, A MN-major
      const uint32_t aQ = tc::smem_u32(sQ), aWL = tc::smem_u32(sWL),
                     aNT = tc::smem_u32(smem + Cfg::OFF_NT), aWT = tc::smem_u32(smem + Cfg::OFF_WT);
      auto kmaj = [](uint32_t base, int k) {
        return tc::sdesc_sw128(base + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
      };
      auto mnmaj = [](uint32_t base, int k) { return tc::sdesc_sw128(base + k * 2048, 16384, 1024); };
      auto n16 = [](uint32_t base, int k) {
        return tc::sdesc_sw128(base + (k >> 2) * 2048 + (k & 3) * 32, 16, 1024);
      };
      uint32_t nr = 0;  // row hand-overs A, B consumed
      auto wait_rows = [&]() -> bool {
        const bool w = tc::mbar_wait(&bar[BF_R], nr & 1, abort_flag);
        ++nr;
        tc::tc_fence_after();
        return w;
      };
      auto wait_bar = [&](int b, uint32_t parity) -> bool {
        const bool w = tc::mbar_wait(&bar[b], parity, abort_flag);
        tc::tc_fence_after();
        return w;
      };
      for (int c = 0; c < NC && ok; ++c) {
        const uint32_t aK = tc::smem_u32(set_of(c)), aV = aK + TILE, aG = tc::smem_u32(stg_of(c));
        // S = Q K^T
        ok = wait_bar(BF_Q, c & 1) && wait_bar((c & 1) ? BF_KV1 : BF_KV0, (c >> 1) & 1);
        if (!ok) break;
#pragma unroll
        for (int k = 0; k < 8; ++k) tc::mma_bf16_ss(tS, kmaj(aQ, k), kmaj(aK, k), idKK, k > 0);
        // the n increment K^T w (hi, lo): w of chunk c was written before the previous
        // chunk's hand-over D (in the prologue for the first chunk, so after A there)
        auto n_update = [&]() {
          const uint32_t wt = aWT + (c & 1) * Cfg::N16_BYTES;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            tc::mma_bf16_ss(tNU + 16 * (c & 1), mnmaj(aK, k), n16(wt, k), idNM, k > 0);
        };
        if (EXPV && c > 0 && c + 1 < NC) n_update();
        // A (C_c staged): O = Q C_c (hi and lo planes: where the normaliser nearly cancels,
        // h = O / den amplifies the rounding of the state); Q n_c (hi, lo) into the two q.n
        // columns
        ok = wait_rows();
        if (!ok) break;
        if (EXPV && c == 0 && c + 1 < NC) n_update();
#pragma unroll
        for (int k = 0; k < 8; ++k) tc::mma_bf16_ss(tO, kmaj(aQ, k), mnmaj(aG, k), idKM, k > 0);
#pragma unroll
        for (int k = 0; k < 8; ++k) tc::mma_bf16_ss(tO, kmaj(aQ, k), mnmaj(aG + TILE, k), idKM, 1);
        if (EXPV) {
#pragma unroll
          for (int k = 0; k < 8; ++k) tc::mma_bf16_ss(tN, kmaj(aQ, k), n16(aNT, k), idNK, k > 0);
        }
        tc::tc_commit(&bar[BF_M]);
        // B (P in TMEM, O rows rescaled): O += P V
        ok = wait_rows();
        if (!ok) break;
#pragma unroll
        for (int k = 0; k < 8; ++k)  // keys 64 h .. 64 h + 63 of P live at column 64 h
          tc::mma_bf16_ts(tO, tS + 64 * (k >> 2) + 8 * (k & 3), mnmaj(aV, k), idKM, 1);
        tc::tc_commit(&bar[BF_M]);
        // D (w K staged: hi plane over K, lo plane apart): C_{c+1} = beta_c C_c (the rows
        // scaled it) + (w K)^T V, while P V runs
        ok = wait_bar(BF_D, c & 1);
        if (!ok) break;
        if (c + 1 < NC) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            tc::mma_bf16_ss(tC, mnmaj(aK, k), mnmaj(aV, k), idMM, 1);
            tc::mma_bf16_ss(tC, mnmaj(aWL, k), mnmaj(aV, k), idMM, 1);
          }
        }
        tc::tc_commit(&bar[BF_S]);
      }
      if (!ok) {
        abort_flag.raise();
        tc::drain_mma(&bar[BF_DRAIN]);  // no product still writes TMEM or reads smem
      }
    }
  } else {
    // ------------------------------------------------------------ rows
    const int row = 32 * (warp & 3) + lane;  // TMEM lane: token row t or state row j
    const int half = (warp - 1) >> 2;        // columns [64 half, 64 half + 64)
    const int cb0 = 2 * half;                // its two 32-column chunks
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const unsigned full = 0xffffffffu;
    const bool lead = half == 0;             // writes the per-row factors
    const bool issuer = row == 0 && lead;    // issues the TMA loads and stores
    constexpr auto rows_and = walk::rows_and<256>;
    const float* m0 = (EXPV && P.init.on()) ? P.init.m : nullptr;
    uint8_t* sNT = smem + Cfg::OFF_NT;
    uint32_t nm = 0, ns = 0;  // product hand-overs (A, B) and state updates consumed
    auto wait_mma = [&]() -> bool {
      const bool w = __all_sync(full, tc::mbar_wait(&bar[BF_M], nm & 1, abort_flag));
      ++nm;
      if (!w && lane == 0) abort_flag.raise();
      tc::tc_fence_after();
      return w;
    };
    auto wait_state = [&]() -> bool {
      const bool w = __all_sync(full, tc::mbar_wait(&bar[BF_S], ns & 1, abort_flag));
      ++ns;
      if (!w && lane == 0) abort_flag.raise();
      tc::tc_fence_after();
      return w;
    };
    // this thread's TMEM stores and shared-memory writes, then a hand-over to the MMA thread
    auto signal = [&](int b) {
      tc::tmem_wait_st();
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      tc::mbar_arrive(&bar[b]);
    };
    uint32_t nq_fills = 0, nkv_fills[2] = {0, 0};  // copies the issuer started, per barrier
    auto load_q = [&](int c) {
      ++nq_fills;
      tc::mbar_arrive_expect_tx(&bar[BF_Q], TILE);
      tc::tma_load_3d(sQ, &tmQ, &bar[BF_Q], 0, c * 128, bh);
      tc::tma_load_3d(sQ + 16384, &tmQ, &bar[BF_Q], 64, c * 128, bh);
    };
    // the next chunk's tiles into L2 while this chunk runs (their loads wait for this
    // chunk's products and stores to free the buffers)
    auto prefetch_next = [&](int c) {
      tc::tma_prefetch_l2_3d(&tmQ, 0, c * 128, bh);
      tc::tma_prefetch_l2_3d(&tmQ, 64, c * 128, bh);
      tc::tma_prefetch_l2_3d(&tmK, 0, c * 128, bh);
      tc::tma_prefetch_l2_3d(&tmK, 64, c * 128, bh);
      tc::tma_prefetch_l2_3d(&tmV, 0, c * 128, bh);
      tc::tma_prefetch_l2_3d(&tmV, 64, c * 128, bh);
    };
    auto load_kv = [&](int c) {
      uint8_t* st = set_of(c);
      uint64_t* b = &bar[(c & 1) ? BF_KV1 : BF_KV0];
      ++nkv_fills[c & 1];
      tc::mbar_arrive_expect_tx(b, 2 * TILE);
      tc::tma_load_3d(st, &tmK, b, 0, c * 128, bh);
      tc::tma_load_3d(st + 16384, &tmK, b, 64, c * 128, bh);
      tc::tma_load_3d(st + TILE, &tmV, b, 0, c * 128, bh);
      tc::tma_load_3d(st + TILE + 16384, &tmV, b, 64, c * 128, bh);
    };

    // Gate values of chunk c (this row's token, the chunk's last token, the previous
    // chunk's max state), loaded a chunk ahead of their use.
    struct GateIn { float g, mc, mprev, bt, lit, mt; };
    auto gate_load = [&](int c) -> GateIn {
      GateIn I;
      const int c0 = c * 128, len = min(128, P.T - c0);
      const size_t tok0 = (size_t)bh * P.T + c0;
      const bool in = row < len;
      const size_t t = tok0 + (in ? row : 0);
      I.g = P.b[tok0 + len - 1];
      I.mc = EXPV ? P.m[tok0 + len - 1] : 0.f;
      I.mprev = EXPV ? chunk_mprev(P.m, tok0, c, m0, bh) : 0.f;
      I.bt = in ? P.b[t] : 0.f;
      I.lit = in ? P.li[t] : 0.f;
      I.mt = (in && EXPV) ? P.m[t] : 0.f;
      return I;
    };
    // Gate factors of chunk c: this row's factors as a query (r2: the exponent's t-side term
    // with 1/sqrt(d_qk); qfac: alpha_t / sqrt(d_qk)) and as a key (w: the state-update
    // weight; the key factor (log i_s - b_s) log2 e in shared memory, w as the rows of the
    // n-update operand), and the chunk's decay beta_c.
    struct Gates { float beta, r2, qfac, w, mt; int len; };
    auto gate_factors = [&](int c, const GateIn& I) -> Gates {
      Gates G;
      G.len = min(128, P.T - c * 128);
      const bool in = row < G.len;
      const bool has_prev = c > 0 || P.init.on();
      if (EXPV) G.beta = (c > 0 || m0 != nullptr) ? expf(I.g + I.mprev - I.mc) : 0.f;
      else G.beta = expf(I.g);
      G.r2 = in ? (I.bt - I.mt) * kLog2e + P.log2_scale : -INFINITY;
      G.qfac = (in && has_prev) ? expf(I.bt + I.mprev - I.mt) * P.scale : 0.f;
      G.w = in ? expf(I.g - I.bt + I.lit - I.mc) : 0.f;
      G.mt = I.mt;
      if (lead) {
        // this warp's 32 rows are one key block: its largest key factor (0 for a block wholly
        // past the end) and the separable key factor 2^(cf_s - M) <= 1
        const float cf = in ? (I.lit - I.bt) * kLog2e : -INFINITY;
        float mx = cf;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(full, mx, o));
        if (mx == -INFINITY) mx = 0.f;
        F[(F_CF0 + (c & 1)) * 128 + row] = cf;
        F[(F_KP0 + (c & 1)) * 128 + row] = tc::ex2(cf - mx);
        if (lane == 0) F[F_MB * 128 + 4 * (c & 1) + (warp & 3)] = mx;
        if (EXPV) {
          uint8_t* wt = smem + Cfg::OFF_WT + (c & 1) * Cfg::N16_BYTES;
          const bf16 hi = __float2bfloat16_rn(G.w);
          *reinterpret_cast<bf16*>(wt + walk::n16_off(0, row)) = hi;
          *reinterpret_cast<bf16*>(wt + walk::n16_off(1, row)) =
              __float2bfloat16_rn(G.w - __bfloat162float(hi));
        }
      }
      return G;
    };

    // Two 32-column chunks of this thread's lane, the next one's TMEM load in flight while
    // the first is processed.
#define MLSTM_WALK_PIPE(TA, ONE)                         \
  {                                                      \
    uint32_t xa[32], xb[32];                             \
    tc::tmem_ld32_async((TA) + lane_base + 32 * cb0, xa); \
    tc::tmem_wait_ld(xa);                                \
    tc::tmem_ld32_async((TA) + lane_base + 32 * cb0 + 32, xb); \
    ONE(xa, cb0);                                        \
    tc::tmem_wait_ld(xb);                                \
    ONE(xb, cb0 + 1);                                    \
  }

    // Stage C_c (row j) as hi and lo bf16 planes and scale it by beta_c in TMEM.
    auto stage_c = [&](uint8_t* stg, float beta) {
      auto one = [&](const uint32_t (&x)[32], int cb) {
        uint32_t w[32];
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int u = 0; u < 4; ++u)
            walk::split_hi_lo(__uint_as_float(x[e + 2 * u]), __uint_as_float(x[e + 2 * u + 1]), hi[u],
                              lo[u]);
          const uint32_t off = sw_off(row, 32 * cb + e);
          *reinterpret_cast<uint4*>(stg + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4*>(stg + TILE + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
        walk::scale32(x, beta, w);
        tc::tmem_st32_async(tC + lane_base + 32 * cb, w);
      };
      MLSTM_WALK_PIPE(tC, one)
    };
    // P of this query row over this half's keys, written over S in TMEM as packed bf16:
    // p = s 2^(r2 + cf_s), zero past the diagonal.  The 32-key blocks left of the diagonal
    // take the separable form s 2^(cf_s - M) 2^(r2 + M) (M: the block's largest cf, so
    // both factors are at most 1: every key there precedes the query); the diagonal block
    // takes each element's own exponent and the causal mask.  Returns the half's share of
    // the row sum.
    auto transform = [&](float r2, int c) -> float {
      float rs = 0.f;
      const int qd = warp & 3;
      const float* cf = F + (F_CF0 + (c & 1)) * 128;
      const float* kp = F + (F_KP0 + (c & 1)) * 128;
      const float* mb = F + F_MB * 128 + 4 * (c & 1);
      auto one = [&](const uint32_t (&xr)[32], int ch) {
        uint32_t pk[16];
        if (ch > qd) {
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = 0u;
        } else if (ch == qd) {
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const int s0 = ch * 32 + i;
            float p0 = __uint_as_float(xr[i]) * tc::ex2(r2 + cf[s0]);
            float p1 = __uint_as_float(xr[i + 1]) * tc::ex2(r2 + cf[s0 + 1]);
            if (s0 > row) p0 = 0.f;
            if (s0 + 1 > row) p1 = 0.f;
            if (EXPV) rs += p0 + p1;
            pk[i >> 1] = tc::pack_bf16(p0, p1);
          }
        } else {
          const float f = tc::ex2(r2 + mb[ch]);
          const uint64_t f2 = tc::f2_make(f, f);
          uint64_t acc = tc::f2_make(0.f, 0.f);
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const float4 g4 = *reinterpret_cast<const float4*>(kp + ch * 32 + i);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint64_t x2 =
                  tc::f2_make(__uint_as_float(xr[i + 2 * h]), __uint_as_float(xr[i + 2 * h + 1]));
              const uint64_t g2 = h ? tc::f2_make(g4.z, g4.w) : tc::f2_make(g4.x, g4.y);
              const uint64_t p2 = tc::f2_mul(tc::f2_mul(x2, g2), f2);
              if (EXPV) acc = tc::f2_add(acc, p2);
              const float2 pp = tc::f2_split(p2);
              pk[(i >> 1) + h] = tc::pack_bf16(pp.x, pp.y);
            }
          }
          if (EXPV) {
            const float2 a = tc::f2_split(acc);
            rs += a.x + a.y;
          }
        }
        // packed into this half's own columns [64 half, 64 half + 32): the other warp of the
        // lane quarter may still be reading its fp32 scores in [64 (1 - half), ...)
        tc::tmem_st16_async(tS + lane_base + 32 * cb0 + 16 * (ch - cb0), pk);
      };
      MLSTM_WALK_PIPE(tS, one)
      return rs;
    };
    // Scale this row of O (the inter term) by f.
    auto rescale = [&](float f) {
      auto one = [&](const uint32_t (&x)[32], int cb) {
        uint32_t w[32];
        walk::scale32(x, f, w);
        tc::tmem_st32_async(tO + lane_base + 32 * cb, w);
      };
      MLSTM_WALK_PIPE(tO, one)
    };
    // h = O / den of this row, packed to bf16 into the staging tile.
    auto epilogue = [&](float inv, uint8_t* stg) {
      auto one = [&](const uint32_t (&x)[32], int cb) {
        uint32_t g[32];
        walk::scale32(x, inv, g);
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          auto f = [&](int u) { return __uint_as_float(g[e + u]); };
          *reinterpret_cast<uint4*>(stg + sw_off(row, 32 * cb + e)) =
              make_uint4(tc::pack_bf16(f(0), f(1)), tc::pack_bf16(f(2), f(3)),
                         tc::pack_bf16(f(4), f(5)), tc::pack_bf16(f(6), f(7)));
        }
      };
      MLSTM_WALK_PIPE(tO, one)
    };
#undef MLSTM_WALK_PIPE

    // ---- prologue: chunk 0's tiles; the state entering it (the initial state or zero)
    if (issuer) {
      load_q(0);
      load_kv(0);
      if (NC > 1) prefetch_next(1);
    }
    float n = 0.f;  // n_c (mLSTMexp), state row j
    {
      uint32_t w[32];
      for (int cb = cb0; cb < cb0 + 2; ++cb) {
#pragma unroll
        for (int e = 0; e < 32; ++e)
          w[e] = __float_as_uint(P.init.on() ? P.init.C[((size_t)bh * 128 + row) * 128 + 32 * cb + e] : 0.f);
        tc::tmem_st32(tC + lane_base + 32 * cb, w);
      }
      if (EXPV && P.init.on()) n = P.init.n[(size_t)bh * 128 + row];
    }
    if (EXPV)  // rows 2..15 of the N = 16 operand tiles stay zero
      for (int i = row + 128 * half; i < 3 * Cfg::N16_BYTES / 16; i += 256)
        reinterpret_cast<uint4*>(sNT)[i] = make_uint4(0u, 0u, 0u, 0u);
    ok = rows_and(ok);  // the zeroing is done before any row writes its weights
    Gates cur = gate_factors(0, gate_load(0));
    ok = rows_and(ok);

    for (int c = 0; c < NC && ok; ++c) {
      if (c > 0) {
        // the Q tile is free once the previous h store has read it (the products that read
        // Q were waited for before that store): its load need not wait for the state update
        if (issuer) {
          tc::bulk_wait_read_all();
          load_q(c);
          if (c + 1 < NC) prefetch_next(c + 1);
        }
        // the previous chunk's state update is done: C_c is in TMEM
        ok = wait_state();
        if (EXPV) {
          float a, b;
          walk::tmem_ld2(tNU + 16 * ((c - 1) & 1) + lane_base, a, b);
          n += a + b;  // n_c = beta_{c-1} n_{c-1} (scaled below, a chunk ago) + K^T w
        }
        ok = rows_and(ok);
        if (!ok) break;
      }
      // the next chunk's gate values, in flight while this chunk runs
      GateIn nxt;
      if (c + 1 < NC) nxt = gate_load(c + 1);
      const bool valid = row < cur.len;
      // ---- A: stage C_c (hi, lo) in the other K/V set, scale it by beta_c; n_c as the q.n
      // operand and as the saved state
      uint8_t* stg = stg_of(c);
      stage_c(stg, cur.beta);
      if (EXPV) {
        if (lead) {
          const bf16 hi = __float2bfloat16_rn(n);
          *reinterpret_cast<bf16*>(sNT + walk::n16_off(0, row)) = hi;
          *reinterpret_cast<bf16*>(sNT + walk::n16_off(1, row)) =
              __float2bfloat16_rn(n - __bfloat162float(hi));
          P.n[((size_t)bh * NC + c) * 128 + row] = n;
        }
        n *= cur.beta;
      }
      signal(BF_R);
      ok = rows_and(ok);  // the staging is complete: store it as the saved state of chunk c
      if (!ok) break;
      if (issuer) {
        const int z = bh * NC + c;
        tc::tma_store_3d(&tmChi, stg, 0, 0, z);
        tc::tma_store_3d(&tmChi, stg + 16384, 64, 0, z);
        tc::tma_store_3d(&tmClo, stg + TILE, 0, 0, z);
        tc::tma_store_3d(&tmClo, stg + TILE + 16384, 64, 0, z);
        tc::bulk_commit_group();
      }
      // ---- the next chunk's gate factors (its key factors in the other buffer, its w as the
      // n-update operand), while the first products run; written before the hand-over D that
      // the next n update follows
      Gates nxtG = cur;
      if (c + 1 < NC) nxtG = gate_factors(c + 1, nxt);
      // ---- B: P over this half's keys and its row-sum share, the inter term scaled by qfac,
      // q.n
      ok = wait_mma();
      const float rs = transform(cur.r2, c);
      rescale(cur.qfac);
      float inter_norm = 0.f;
      if (EXPV) {
        float a, b;
        walk::tmem_ld2(tN + lane_base, a, b);
        inter_norm = cur.qfac * (a + b);
        F[(half ? F_RS1 : F_RS0) * 128 + row] = rs;
      }
      signal(BF_R);
      // the next chunk's K and V into the staging set, once the inter product (waited for
      // above) and the saved-state store have read it
      if (issuer && ok && c + 1 < NC) {
        tc::bulk_wait_read_all();
        load_kv(c + 1);
      }
      // ---- D: w K (hi plane over K, lo plane apart): the score, inter and n-update products
      // that read K are done (waited for above)
      if (c + 1 < NC) {
        uint8_t* sK = set_of(c);
#pragma unroll 4
        for (int col = 64 * half; col < 64 * half + 64; col += 8) {
          const uint32_t off = sw_off(row, col);
          const uint4 raw = *reinterpret_cast<const uint4*>(sK + off);
          const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            walk::split_hi_lo(walk::bf16_lo(w[e]) * cur.w, walk::bf16_hi(w[e]) * cur.w, hi[e], lo[e]);
          *reinterpret_cast<uint4*>(sK + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4*>(sWL + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
      signal(BF_D);
      // ---- h = O / den once P V is done, staged over Q (its products are done)
      ok = wait_mma() && ok;
      ok = rows_and(ok);  // and both halves' row sums are in shared memory
      if (!ok) break;
      float inv = 1.f;
      if (EXPV) {
        const float a = inter_norm + (F[F_RS0 * 128 + row] + F[F_RS1 * 128 + row]);
        inv = 1.f / fmaxf(fabsf(a), expf(-cur.mt));
        if (lead && valid) P.abar[(size_t)bh * P.T + (size_t)c * 128 + row] = a;
      }
      epilogue(inv, sQ);
      tc::fence_proxy_async_smem();
      ok = rows_and(ok);
      if (!ok) break;
      if (issuer) {
        tc::tma_store_3d(&tmH, sQ, 0, c * 128, bh);
        tc::tma_store_3d(&tmH, sQ + 16384, 64, c * 128, bh);
        tc::bulk_commit_group();
      }
      cur = nxtG;
    }
    // the last chunk's hand-over: every product has completed
    if (ok) ok = wait_state();
    if (issuer && !ok) {  // gave up: the copies still in flight land before the CTA exits
      tc::drain_last(&bar[BF_Q], nq_fills);
      tc::drain_last(&bar[BF_KV0], nkv_fills[0]);
      tc::drain_last(&bar[BF_KV1], nkv_fills[1]);
    }
    if (issuer) tc::bulk_wait_all();
    if (!ok) abort_flag.raise();
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

bool fwd_walk_supported(const Problem& p) {
  return p.bf16() && p.L == 128 && p.dqk == 128 && p.dhv == 128;
}

template <bool EXPV>
static cudaError_t launch_fwalk(const Problem& p, const FwdArgs& a, cudaStream_t s) {
  const bf16* C = (const bf16*)a.C;
  const size_t plane = (size_t)p.BH * p.NC * p.dqk * p.dhv;
  const uint64_t BHNC = (uint64_t)p.BH * p.NC;
  CUtensorMap tQ, tK, tV, tH, tCh, tCl;
  if (!make_tmap_3d_bf16(&tQ, a.q, 128, p.T, p.BH, 64, 128) ||
      !make_tmap_3d_bf16(&tK, a.k, 128, p.T, p.BH, 64, 128) ||
      !make_tmap_3d_bf16(&tV, a.v, 128, p.T, p.BH, 64, 128) ||
      !make_tmap_3d_bf16(&tH, a.h, 128, p.T, p.BH, 64, 128) ||
      !make_tmap_3d_bf16(&tCh, C, 128, 128, BHNC, 64, 128) ||
      !make_tmap_3d_bf16(&tCl, C + plane, 128, 128, BHNC, 64, 128))
    return cudaErrorInvalidValue;
  FwalkParams P;
  P.b = a.b; P.li = a.li; P.m = a.m;
  P.abar = a.abar;
  P.n = a.n;
  P.init = a.init;
  P.T = p.T; P.NC = p.NC;
  P.scale = p.scale;
  P.log2_scale = log2f(p.scale);
  P.epoch = next_epoch();
  auto kern = fwd_walk_kernel<EXPV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)FwalkCfg::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)p.BH, 288, FwalkCfg::SMEM, s>>>(tQ, tK, tV, tH, tCh, tCl, P);
  return cudaGetLastError();
}

cudaError_t launch_fwd_walk(const Problem& p, const FwdArgs& a, cudaStream_t s) {
  return p.exp_variant() ? launch_fwalk<true>(p, a, s) : launch_fwalk<false>(p, a, s);
}

cudaError_t fetch_tc_fwalk_error(unsigned int* flag) {
  return cudaMemcpyFromSymbol(flag, g_tc_fwalk_error, sizeof(unsigned int));
}

}  // namespace mlstm
