// Backward walker for chunk 128 (d_qk = d_hv = 128, bf16): the state-gradient
// recurrence (K-d1) and the dk, dv products (K-d2) of every chunk in one pass.
//
// One CTA per head walks the chunks from the last to the first, holding the
// gradient of the state leaving the current chunk, dC_c (fp32, d_qk x d_hv), in
// TMEM.  At chunk c it stages dC_c as hi and lo bf16 planes in shared memory,
// computes the chunk's dv and dk (intra-chunk products and the inter-chunk terms
// through dC_c, as the dk and dv kernels of tc_bwd.cu do, so dk rounds the same
// transform tile as dq), then updates dC_{c-1} = beta_c dC_c + Q_c^T diag(u) dH_c
// on the tensor core.  dC never goes to HBM, and each chunk's q, k, v, dh tiles
// are read once for all three products.  "Tiled Flash Linear Attention" (TFLA
// summary page, Problem: materialised chunk states cost IO; Approach).
//
// Roles: one thread (warp 0) issues the MMAs; eight row warps transform, rescale
// and store, two per TMEM lane quarter: a thread owns one key row, token row or
// state row (its TMEM lane) and one half of the columns.  One row thread issues
// the TMA loads and stores.  Rows and MMA thread hand over through mbarriers
// (four hand-overs each way per chunk), so work that does not feed the next product
// (the next chunk's gate factors, the dv and dk epilogues) runs while the tensor
// core works:
//   rows: stage dC -> A, next gates | rescale dv inter, dv transform -> B | rescale
//         dk inter, dk transform -> C | u dH, dn increment -> D | dv out | dk out
//   MMA:  K Q^T (dv score) | A: K dC (dv inter) | V dC^T (dk inter) | B: Y dH (dv),
//         V dH^T (dk score) | C: Y Q (dk), Q^T wn (dn increment) | D: dC += Q^T (u dH)
// The next chunk's K and V tiles load as soon as their buffers are free, Q and
// dH once the state update has read them.  Every wait is bounded; on a timeout
// the kernel raises its error flag and winds down.
#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"
#include "walk_common.cuh"

namespace mlstm {

static __device__ unsigned int g_tc_walk_error;

namespace {

constexpr float kLog2e = 1.4426950408889634f;

// Shared memory: six 32 KB tiles (128 rows x 128 bf16 as two 128-byte-swizzled
// 64-column blocks) and the per-token factors.  Reuse over one chunk:
//   Q: q (until the state update);  K: k (until the k.dk dot products);
//   V: v, then the dv staging tile;  H: dh, then u dH (hi plane);
//   G: dC hi plane, then the dk staging tile;  G + TILE: dC lo plane, then u dH lo.
struct WalkCfg {
  static constexpr int TILE = walk::TILE;
  static constexpr int OFF_Q = 0, OFF_K = TILE, OFF_V = 2 * TILE, OFF_H = 3 * TILE;
  static constexpr int OFF_G = 4 * TILE;
  static constexpr int OFF_F = 6 * TILE;              // per-token factors, NF arrays of 128 floats
  static constexpr int NF = 8;
  static constexpr int OFF_W = OFF_F + NF * 128 * 4;  // per-warp partner factors, 8 x 128
  // the normaliser weights as the B operand of the dn product: 16 x 128 K-major bf16 (row 0
  // the hi, row 1 the lo plane, rows 2..15 zero), two buffers (chunk parity)
  static constexpr int OFF_WN = OFF_W + 8 * 128 * 4;
  static constexpr int WN_BYTES = 4096;
  static constexpr int OFF_BAR = OFF_WN + 2 * WN_BYTES;
  static constexpr int OFF_TMEM = OFF_BAR + 9 * 8;
  static constexpr size_t SMEM = 1024 + OFF_TMEM + 16;
  static constexpr uint32_t TMEM_COLS = 512;  // dC, score / transformed tile, dv, dk
};

// per-token factor arrays in the OFF_F region (token t of the chunk, or state row j)
// (the partner factors and state-update weights of the chunk with walk index it are in
// buffer it & 1: the next chunk's are written while this chunk's are still read)
enum { F_PC0 = 0, F_PC1, F_PE0, F_PE1, F_WV0, F_WV1, F_DN, F_DOT };
// mbarriers: tile loads (one per tile); rows -> MMA thread (hand-overs A, B, C; and D on
// its own barrier, since the rows signal C and D back to back); MMA thread -> rows (the
// products after A, B, C; and the state update on its own barrier, which can complete
// before the rows wait for C's products).  Each barrier's phases strictly alternate
// with its waiter, so parity waits cannot alias.
// BW_DRAIN: the MMA thread's last commit when it gives up.
enum { BW_Q = 0, BW_K, BW_V, BW_H, BW_R, BW_D, BW_M, BW_S, BW_DRAIN, BW_COUNT };
static_assert(BW_COUNT <= 9, "barrier slots");

using walk::sw_off;
constexpr auto rows_and = walk::rows_and<256>;
using walk::bulk_wait_read_but_one;

}  // namespace

struct WalkParams {
  const float *b, *li, *m, *inv_den, *da;
  float* pk;               // [BH, T] k . dk
  const float* m0;         // the initial state's max state (mLSTMexp), or null
  const float *dCT, *dnT;  // gradient of the final state, or null
  float *d0, *dn0;         // gradient of the initial state, or null
  int T, NC;
  float scale, log2_scale;
  unsigned int epoch;  // this launch's abort epoch
};

template <bool EXPV>
__global__ void __launch_bounds__(288, 1) bwd_walk_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmH,
    const __grid_constant__ CUtensorMap tmDK, const __grid_constant__ CUtensorMap tmDV,
    const WalkParams P) {
  using Cfg = WalkCfg;
  const tc::Abort abort_flag{&g_tc_walk_error, P.epoch};
  if (__syncthreads_or(threadIdx.x == 0 && abort_flag.raised())) return;
  const int bh = blockIdx.x;
  const int NC = P.NC;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sQ = smem + Cfg::OFF_Q, *sK = smem + Cfg::OFF_K, *sV = smem + Cfg::OFF_V,
          *sH = smem + Cfg::OFF_H, *sG = smem + Cfg::OFF_G;
  float* F = reinterpret_cast<float*>(smem + Cfg::OFF_F);
  float* fwv = reinterpret_cast<float*>(smem + Cfg::OFF_W);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + Cfg::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_TMEM);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < BW_COUNT; ++i) tc::mbar_init(&bar[i], (i == BW_R || i == BW_D) ? 256u : 1u);
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
  const uint32_t tDC = tmem, tX = tmem + 128, tAV = tmem + 256, tAK = tmem + 384;
  bool ok = true;

  if (warp == 0) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idKK = tc::idesc_bf16(128, 128, false, false);  // A, B K-major
      constexpr uint32_t idKM = tc::idesc_bf16(128, 128, false, true);   // B MN-major
      constexpr uint32_t idMM = tc::idesc_bf16(128, 128, true, true);    // A, B MN-major
      constexpr uint32_t idN = tc::idesc_bf16(128, 16, true, false);     // A MN-major, N = 16
      const uint32_t aQ = tc::smem_u32(sQ), aK = tc::smem_u32(sK), aV = tc::smem_u32(sV),
                     aH = tc::smem_u32(sH), aG = tc::smem_u32(sG), aGl = aG + Cfg::TILE,
                     aWN = tc::smem_u32(smem + Cfg::OFF_WN);
      // K-step k (16 elements) of a K-major tile, or of an MN-major tile (rows = K)
      auto kmaj = [](uint32_t base, int k) {
        return tc::sdesc_sw128(base + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
      };
      auto mnmaj = [](uint32_t base, int k) { return tc::sdesc_sw128(base + k * 2048, 16384, 1024); };
      uint32_t nr = 0;  // row hand-overs A, B, C consumed
      auto wait_rows = [&]() -> bool {
        const bool w = tc::mbar_wait(&bar[BW_R], nr & 1, abort_flag);
        ++nr;
        tc::tc_fence_after();
        return w;
      };
      auto wait_tile = [&](int b, int it) -> bool {
        const bool w = tc::mbar_wait(&bar[b], it & 1, abort_flag);
        tc::tc_fence_after();
        return w;
      };
      for (int it = 0; it < NC && ok; ++it) {
        const int c = NC - 1 - it;
        // the dv score K Q^T (the score buffer is free: the rows read the previous chunk's
        // dn increment before they handed over its state update)
        ok = wait_tile(BW_K, it) && wait_tile(BW_Q, it);
        if (!ok) break;
#pragma unroll
        for (int k = 0; k < 8; ++k) tc::mma_bf16_ss(tX, kmaj(aK, k), kmaj(aQ, k), idKK, k > 0);
        // A (dC staged): dv inter K dC (hi + lo planes)
        ok = wait_rows();
        if (!ok) break;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          tc::mma_bf16_ss(tAV, kmaj(aK, k), mnmaj(aG, k), idKM, k > 0);
          tc::mma_bf16_ss(tAV, kmaj(aK, k), mnmaj(aGl, k), idKM, 1);
        }
        tc::tc_commit(&bar[BW_M]);
        // the dk inter V dC^T (hi + lo) while the rows transform the dv score
        ok = wait_tile(BW_V, it);
        if (!ok) break;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          tc::mma_bf16_ss(tAK, kmaj(aV, k), kmaj(aG, k), idKK, k > 0);
          tc::mma_bf16_ss(tAK, kmaj(aV, k), kmaj(aGl, k), idKK, 1);
        }
        // B (dv transform in TMEM): dv += Y dH, then the dk score V dH^T over Y
        ok = wait_rows() && wait_tile(BW_H, it);
        if (!ok) break;
#pragma unroll
        for (int k = 0; k < 8; ++k)  // keys 64 h .. 64 h + 63 of Y live at column 64 h
          tc::mma_bf16_ts(tAV, tX + 64 * (k >> 2) + 8 * (k & 3), mnmaj(aH, k), idKM, 1);
#pragma unroll
        for (int k = 0; k < 8; ++k) tc::mma_bf16_ss(tX, kmaj(aV, k), kmaj(aH, k), idKK, k > 0);
        tc::tc_commit(&bar[BW_M]);
        // C (dk transform in TMEM): dk += Y Q; then the normaliser's increment Q^T wn (hi, lo)
        // into columns 32 and 33 of the score buffer (Y lives in columns 0..31 and 64..95)
        ok = wait_rows();
        if (!ok) break;
        const bool update = c > 0 || P.d0 != nullptr;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          tc::mma_bf16_ts(tAK, tX + 64 * (k >> 2) + 8 * (k & 3), mnmaj(aQ, k), idKM, 1);
        if (EXPV && update) {
          const uint32_t wn = aWN + (it & 1) * Cfg::WN_BYTES;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            tc::mma_bf16_ss(tX + 32, mnmaj(aQ, k),
                            tc::sdesc_sw128(wn + (k >> 2) * 2048 + (k & 3) * 32, 16, 1024), idN,
                            k > 0);
        }
        tc::tc_commit(&bar[BW_M]);
        // D (u dH staged, hi plane over dH, lo plane over dC's): dC_{c-1} = beta_c dC_c (the
        // rows scaled it) + Q^T (u dH)
        ok = tc::mbar_wait(&bar[BW_D], it & 1, abort_flag);
        tc::tc_fence_after();
        if (!ok) break;
        if (update) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            tc::mma_bf16_ss(tDC, mnmaj(aQ, k), mnmaj(aH, k), idMM, 1);
            tc::mma_bf16_ss(tDC, mnmaj(aQ, k), mnmaj(aGl, k), idMM, 1);
          }
        }
        tc::tc_commit(&bar[BW_S]);
      }
      if (!ok) {
        abort_flag.raise();
        tc::drain_mma(&bar[BW_DRAIN]);  // no product still writes TMEM or reads smem
      }
    }
  } else {
    // ------------------------------------------------------------ rows
    const int row = 32 * (warp & 3) + lane;  // TMEM lane: key row s, token t or state row j
    const int half = (warp - 1) >> 2;        // columns [64 half, 64 half + 64)
    const int cb0 = 2 * half;                // its two 32-column chunks
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const unsigned full = 0xffffffffu;
    const bool lead = half == 0;             // writes the per-row factors
    const bool issuer = row == 0 && lead;    // issues the TMA loads and stores
    uint32_t nm = 0, ns = 0;       // product hand-overs (A, B, C) and state updates consumed
    auto wait_mma = [&]() -> bool {
      const bool w = __all_sync(full, tc::mbar_wait(&bar[BW_M], nm & 1, abort_flag));
      ++nm;
      if (!w && lane == 0) abort_flag.raise();
      tc::tc_fence_after();
      return w;
    };
    auto wait_state = [&]() -> bool {
      const bool w = __all_sync(full, tc::mbar_wait(&bar[BW_S], ns & 1, abort_flag));
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
    uint32_t fills[4] = {0, 0, 0, 0};  // copies the issuer started on BW_Q, BW_K, BW_V, BW_H
    auto load_tile = [&](int b, uint8_t* dst, const CUtensorMap* tm, int c) {
      ++fills[b - BW_Q];
      tc::mbar_arrive_expect_tx(&bar[b], Cfg::TILE);
      tc::tma_load_3d(dst, tm, &bar[b], 0, c * 128, bh);
      tc::tma_load_3d(dst + 16384, tm, &bar[b], 64, c * 128, bh);
    };
    auto store_tile = [&](const CUtensorMap* tm, const uint8_t* src, int c) {
      tc::tma_store_3d(tm, src, 0, c * 128, bh);
      tc::tma_store_3d(tm, src + 16384, 64, c * 128, bh);
      tc::bulk_commit_group();
    };

    // Gate values of chunk c (this row's token, the chunk's last token, the previous
    // chunk's max state), loaded a chunk ahead of their use.
    struct GateIn { float g, mc, mprev, bt, lis, mt, invd, dat; };
    auto gate_load = [&](int c) -> GateIn {
      GateIn I;
      const int c0 = c * 128, len = min(128, P.T - c0);
      const size_t tok0 = (size_t)bh * P.T + c0;
      const bool in = row < len;
      const size_t t = tok0 + (in ? row : 0);
      I.g = P.b[tok0 + len - 1];
      I.mc = EXPV ? P.m[tok0 + len - 1] : 0.f;
      I.mprev = EXPV ? chunk_mprev(P.m, tok0, c, P.m0, bh) : 0.f;
      I.bt = in ? P.b[t] : 0.f;
      I.lis = in ? P.li[t] : 0.f;
      I.mt = (in && EXPV) ? P.m[t] : 0.f;
      I.invd = (in && EXPV) ? P.inv_den[t] : 1.f;
      I.dat = (in && EXPV) ? P.da[t] : 0.f;
      return I;
    };
    // Gate factors of chunk c: partner factors of this row as a query (the dk and dv
    // transforms), its state-update weights (u in shared memory, wn as the hi and lo rows of
    // the dn product's operand), and the chunk's scalars.
    struct Gates { float g, mc, beta, bt, lis; int len; };
    auto gate_factors = [&](int c, const GateIn& I) -> Gates {
      Gates G;
      G.len = min(128, P.T - c * 128);
      const bool in = row < G.len;
      G.g = I.g;
      G.mc = I.mc;
      G.bt = I.bt;
      G.lis = I.lis;
      if (EXPV) G.beta = (c > 0 || P.m0 != nullptr) ? expf(I.g + I.mprev - I.mc) : 0.f;
      else G.beta = expf(I.g);
      if (!lead) return G;
      const int fb = (NC - 1 - c) & 1;
      F[(F_PC0 + fb) * 128 + row] = in ? (I.bt - I.mt) * kLog2e + log2f(I.invd) : -INFINITY;
      F[(F_PE0 + fb) * 128 + row] = (EXPV && in) ? I.dat / I.invd : 0.f;
      // exp(-inf) = 0 in the first chunk of an mLSTMexp sequence without an initial state
      const float alpha = in ? expf(I.bt + I.mprev - I.mt) * P.scale : 0.f;
      F[(F_WV0 + fb) * 128 + row] = alpha * I.invd;
      if (EXPV) {
        const float wn = alpha * I.dat;
        const bf16 hi = __float2bfloat16_rn(wn);
        const bf16 lo = __float2bfloat16_rn(wn - __bfloat162float(hi));
        uint8_t* wt = smem + Cfg::OFF_WN + ((NC - 1 - c) & 1) * Cfg::WN_BYTES;
        *reinterpret_cast<bf16*>(wt + walk::n16_off(0, row)) = hi;
        *reinterpret_cast<bf16*>(wt + walk::n16_off(1, row)) = lo;
      }
      return G;
    };
    // columns 32 and 33 of the score buffer after the dk accumulate: the normaliser's increment
    auto dn_increment = [&]() -> float {
      float a, b;
      walk::tmem_ld2(tX + 32 + lane_base, a, b);
      return a + b;
    };
    // Rescale an inter-term accumulator row in TMEM: x = rs x (+ rs dn[col] for dk, mLSTMexp).
    auto rescale = [&](uint32_t tA, float rs, bool with_dn) {
      auto one = [&](const uint32_t (&x)[32], int cb) {
        uint32_t w[32];
        if (EXPV && with_dn) {  // rs (x + dn[col]), two lanes per f32x2 operation
          const uint64_t r2 = tc::f2_make(rs, rs);
          const float4* dn4 = reinterpret_cast<const float4*>(F + F_DN * 128 + 32 * cb);
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 d = dn4[e / 4];
            const float2 y0 = tc::f2_split(tc::f2_mul(
                tc::f2_add(tc::f2_make(__uint_as_float(x[e]), __uint_as_float(x[e + 1])),
                           tc::f2_make(d.x, d.y)), r2));
            const float2 y1 = tc::f2_split(tc::f2_mul(
                tc::f2_add(tc::f2_make(__uint_as_float(x[e + 2]), __uint_as_float(x[e + 3])),
                           tc::f2_make(d.z, d.w)), r2));
            w[e] = __float_as_uint(y0.x);
            w[e + 1] = __float_as_uint(y0.y);
            w[e + 2] = __float_as_uint(y1.x);
            w[e + 3] = __float_as_uint(y1.y);
          }
        } else {
          walk::scale32(x, rs, w);
        }
        tc::tmem_st32_async(tA + lane_base + 32 * cb, w);
      };
      uint32_t xa[32], xb[32];
      tc::tmem_ld32_async(tA + lane_base + 32 * cb0, xa);
      tc::tmem_wait_ld(xa);
      tc::tmem_ld32_async(tA + lane_base + 32 * cb0 + 32, xb);
      one(xa, cb0);
      tc::tmem_wait_ld(xb);
      one(xb, cb0 + 1);
    };

    // The dk or dv transform of this key row (R: its row factor), written over the score
    // in TMEM as packed bf16.  The same 32 x 32 classes, factors and fp32 operations as
    // the dk and dv kernels of tc_bwd.cu on a diagonal tile: sub-blocks left of the
    // diagonal are zero, the diagonal one takes every element's own exponent and the
    // causal mask, the others the separable form ((x + e) f_t) g_s.
    auto transform = [&](bool is_dk, float R, int fb) {
      const float* pc = F + (F_PC0 + fb) * 128;
      float mx = R;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(full, mx, o));
      const float Mrow = mx == -INFINITY ? 0.f : mx;
      const float grow = tc::ex2(R - Mrow);
      float* fw = fwv + (warp - 1) * 128;
      __syncwarp();
#pragma unroll
      for (int u = cb0; u < cb0 + 2; ++u) fw[lane + 32 * u] = tc::ex2(pc[lane + 32 * u] + Mrow);
      __syncwarp();
      const float* pe = F + (F_PE0 + fb) * 128;
      const int wb = warp & 3;
      auto one = [&](const uint32_t (&xr)[32], int ch) {
        uint32_t pk[16];
        if (ch < wb) {
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = 0u;
        } else if (ch == wb) {
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            float y[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int p = ch * 32 + i + u;
              const float add = is_dk ? pe[p] : 0.f;
              const float val = (__uint_as_float(xr[i + u]) + add) * tc::ex2(pc[p] + R);
              y[u] = p < row ? 0.f : val;
            }
            pk[i >> 1] = tc::pack_bf16(y[0], y[1]);
          }
        } else {
          const uint64_t g2r = tc::f2_make(grow, grow);
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const int p = ch * 32 + i;
            const float4 g4 = *reinterpret_cast<const float4*>(fw + p);
            float4 e4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (is_dk) e4 = *reinterpret_cast<const float4*>(pe + p);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint64_t x2 =
                  tc::f2_make(__uint_as_float(xr[i + 2 * h]), __uint_as_float(xr[i + 2 * h + 1]));
              const uint64_t gv = h ? tc::f2_make(g4.z, g4.w) : tc::f2_make(g4.x, g4.y);
              uint64_t y2;
              if (is_dk) {
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
        // packed into this half's own columns [64 half, 64 half + 32): the other warp of the
        // lane quarter may still be reading its fp32 scores in [64 (1 - half), ...)
        tc::tmem_st16_async(tX + lane_base + 32 * cb0 + 16 * (ch - cb0), pk);
      };
      uint32_t xa[32], xb[32];
      tc::tmem_ld32_async(tX + lane_base + 32 * cb0, xa);
      tc::tmem_wait_ld(xa);
      tc::tmem_ld32_async(tX + lane_base + 32 * cb0 + 32, xb);
      one(xa, cb0);
      tc::tmem_wait_ld(xb);
      one(xb, cb0 + 1);
    };

    // An output row: TMEM x fin, packed to bf16 into a staging tile (swizzled as the TMA
    // store reads it); with dot, also k . (x fin), k read from the K tile, in the order of
    // the dk kernel's epilogue.
    auto epilogue = [&](uint32_t tA, float fin, uint8_t* stg, bool dot) -> float {
      float dsum = 0.f;
      auto one = [&](const uint32_t (&x)[32], int cb) {
        uint32_t g[32];
        walk::scale32(x, fin, g);
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          float gq[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) gq[u] = __uint_as_float(g[e + u]);
          const uint32_t off = sw_off(row, 32 * cb + e);
          if (dot) {
            const uint4 src = *reinterpret_cast<const uint4*>(sK + off);
            const uint32_t sw[4] = {src.x, src.y, src.z, src.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const __nv_bfloat162 s2 = *reinterpret_cast<const __nv_bfloat162*>(&sw[u]);
              dsum = fmaf(__bfloat162float(s2.x), gq[2 * u], dsum);
              dsum = fmaf(__bfloat162float(s2.y), gq[2 * u + 1], dsum);
            }
          }
          *reinterpret_cast<uint4*>(stg + off) =
              make_uint4(tc::pack_bf16(gq[0], gq[1]), tc::pack_bf16(gq[2], gq[3]),
                         tc::pack_bf16(gq[4], gq[5]), tc::pack_bf16(gq[6], gq[7]));
        }
      };
      uint32_t xa[32], xb[32];
      tc::tmem_ld32_async(tA + lane_base + 32 * cb0, xa);
      tc::tmem_wait_ld(xa);
      tc::tmem_ld32_async(tA + lane_base + 32 * cb0 + 32, xb);
      one(xa, cb0);
      tc::tmem_wait_ld(xb);
      one(xb, cb0 + 1);
      return dsum;
    };

    // Stage dC_c as hi and lo bf16 planes (row j of the state) and scale it by beta_c in
    // TMEM, ready for the update's accumulate.
    auto stage_dc = [&](float beta) {
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
          *reinterpret_cast<uint4*>(sG + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4*>(sG + Cfg::TILE + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
        walk::scale32(x, beta, w);
        tc::tmem_st32_async(tDC + lane_base + 32 * cb, w);
      };
      uint32_t xa[32], xb[32];
      tc::tmem_ld32_async(tDC + lane_base + 32 * cb0, xa);
      tc::tmem_wait_ld(xa);
      tc::tmem_ld32_async(tDC + lane_base + 32 * cb0 + 32, xb);
      one(xa, cb0);
      tc::tmem_wait_ld(xb);
      one(xb, cb0 + 1);
    };
    // ---- prologue: the last chunk's tiles, the final state's gradient (or zero), gates
    if (issuer) {
      load_tile(BW_Q, sQ, &tmQ, NC - 1);
      load_tile(BW_K, sK, &tmK, NC - 1);
      load_tile(BW_V, sV, &tmV, NC - 1);
      load_tile(BW_H, sH, &tmH, NC - 1);
    }
    float dn = 0.f;  // dn_c, the normaliser part of the state gradient (mLSTMexp), row j
    {
      uint32_t w[32];
      for (int cb = cb0; cb < cb0 + 2; ++cb) {
#pragma unroll
        for (int e = 0; e < 32; ++e)
          w[e] = __float_as_uint(P.dCT ? P.dCT[((size_t)bh * 128 + row) * 128 + 32 * cb + e] : 0.f);
        tc::tmem_st32(tDC + lane_base + 32 * cb, w);
      }
      if (EXPV && P.dnT) dn = P.dnT[(size_t)bh * 128 + row];
      if (EXPV && lead) F[F_DN * 128 + row] = dn;
    }
    if (EXPV)
      for (int i = row + 128 * half; i < 2 * Cfg::WN_BYTES / 16; i += 256)
        reinterpret_cast<uint4*>(smem + Cfg::OFF_WN)[i] = make_uint4(0u, 0u, 0u, 0u);
    ok = rows_and(ok);  // the zeroing is done before any row writes its weights
    Gates cur = gate_factors(NC - 1, gate_load(NC - 1));
    ok = rows_and(ok);

    for (int it = 0; it < NC && ok; ++it) {
      const int c = NC - 1 - it;
      if (it > 0) {
        // the previous chunk's state update is done: Q and dH are free for this chunk's
        // tiles, and the staging planes once the dk store has read its tile
        ok = wait_state();
        if (issuer && ok) {
          load_tile(BW_Q, sQ, &tmQ, c);
          load_tile(BW_H, sH, &tmH, c);
          tc::bulk_wait_read_all();
        }
        ok = rows_and(ok);
        if (!ok) break;
      }
      // the next chunk's gate values, in flight while this chunk runs
      GateIn nxt;
      if (c > 0) nxt = gate_load(c - 1);
      const bool valid = row < cur.len;
      // ---- A: stage dC_c (hi, lo), scale it by beta_c in TMEM
      stage_dc(cur.beta);
      if (EXPV) dn *= cur.beta;
      signal(BW_R);
      // the next chunk's gate factors (the other factor buffer) while the first products run
      Gates nxtG = cur;
      if (c > 0) nxtG = gate_factors(c - 1, nxt);
      // row-side factors of this key row (the dk and dv kernels' conventions)
      float rs_v = 0.f, rs_k = 0.f, Rk = -INFINITY, Rv = -INFINITY;
      if (valid) {
        rs_v = expf(cur.g - cur.bt + cur.lis - cur.mc);
        rs_k = rs_v / P.scale;
        Rk = (cur.lis - cur.bt) * kLog2e;
        Rv = Rk + P.log2_scale;
      }
      // ---- B: dv inter rescaled, dv transform
      ok = wait_mma();
      rescale(tAV, rs_v, false);
      transform(false, Rv, it & 1);
      signal(BW_R);
      // ---- C: dk inter rescaled (+ dn_c), dk transform
      ok = wait_mma() && ok;
      rescale(tAK, rs_k, true);
      transform(true, Rk, it & 1);
      signal(BW_R);
      // ---- D: u dH, hi plane over dH and lo plane over dC's lo plane (their products are
      // done), so the state update runs while the outputs are written
      const bool update = c > 0 || P.d0 != nullptr;
      if (update) {
        const float wv = F[(F_WV0 + (it & 1)) * 128 + row];
#pragma unroll 4
        for (int col = 64 * half; col < 64 * half + 64; col += 8) {
          const uint32_t off = sw_off(row, col);
          const uint4 raw = *reinterpret_cast<const uint4*>(sH + off);
          const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            walk::split_hi_lo(walk::bf16_lo(w[e]) * wv, walk::bf16_hi(w[e]) * wv, hi[e], lo[e]);
          *reinterpret_cast<uint4*>(sH + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4*>(sG + Cfg::TILE + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
      // dk accumulated and the normaliser's increment in the score buffer, which the next
      // chunk's dv score overwrites once the state update has been handed over
      ok = wait_mma() && ok;
      if (EXPV && update) {
        dn += dn_increment();  // dn_{c-1}
        // read by the next chunk's dk rescale (every row's dk rescale of this chunk is
        // done: the products waited for it)
        if (lead) F[F_DN * 128 + row] = dn;
      }
      signal(BW_D);
      // ---- dv out, staged over V (its products are done)
      epilogue(tAV, 1.f, sV, false);
      tc::fence_proxy_async_smem();
      ok = rows_and(ok);
      if (!ok) break;
      if (issuer) store_tile(&tmDV, sV, c);
      // ---- dk out, staged over dC's hi plane, with k . dk from the K tile
      const float dot = epilogue(tAK, P.scale, sG, true);
      if (!lead) F[F_DOT * 128 + row] = dot;  // this half's share of k . dk
      tc::fence_proxy_async_smem();
      ok = rows_and(ok);
      if (!ok) break;
      if (lead && valid) P.pk[(size_t)bh * P.T + (size_t)c * 128 + row] = dot + F[F_DOT * 128 + row];
      if (issuer) {
        store_tile(&tmDK, sG, c);
        if (c > 0) {
          load_tile(BW_K, sK, &tmK, c - 1);  // the k . dk reads are done
          bulk_wait_read_but_one();          // the dv store has read its tile
          load_tile(BW_V, sV, &tmV, c - 1);
        }
      }
      cur = nxtG;
    }
    // the last state update
    if (ok) ok = wait_state();
    if (ok && P.d0 != nullptr) {
      for (int cb = cb0; cb < cb0 + 2; ++cb) {
        float x[32];
        tc::tmem_ld32(tDC + lane_base + 32 * cb, x);
        float4* dst = reinterpret_cast<float4*>(P.d0 + ((size_t)bh * 128 + row) * 128 + 32 * cb);
#pragma unroll
        for (int e = 0; e < 32; e += 4) dst[e / 4] = make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
      }
      if (EXPV && lead) P.dn0[(size_t)bh * 128 + row] = dn;
    }
    if (issuer && !ok) {  // gave up: the copies still in flight land before the CTA exits
      for (int i = 0; i < 4; ++i) tc::drain_last(&bar[BW_Q + i], fills[i]);
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

bool bwd_walk_supported(const Problem& p) {
  return p.bf16() && p.L == 128 && p.dqk == 128 && p.dhv == 128;
}

template <bool EXPV>
static cudaError_t launch_walk(const Problem& p, const BwdArgs& a, cudaStream_t s) {
  CUtensorMap tQ, tK, tV, tH, tDK, tDV;
  if (!make_tmap_3d_bf16(&tQ, a.q, 128, p.T, p.BH, 64, 128) ||
      !make_tmap_3d_bf16(&tK, a.k, 128, p.T, p.BH, 64, 128) ||
      !make_tmap_3d_bf16(&tV, a.v, 128, p.T, p.BH, 64, 128) ||
      !make_tmap_3d_bf16(&tH, a.dh, 128, p.T, p.BH, 64, 128) ||
      !make_tmap_3d_bf16(&tDK, a.dk, 128, p.T, p.BH, 64, 128) ||
      !make_tmap_3d_bf16(&tDV, a.dv, 128, p.T, p.BH, 64, 128))
    return cudaErrorInvalidValue;
  WalkParams P;
  P.b = a.b; P.li = a.li; P.m = a.m; P.inv_den = a.inv_den; P.da = a.da;
  P.pk = a.pk;
  P.m0 = (a.init.on() && EXPV) ? a.init.m : nullptr;
  P.dCT = a.dCT; P.dnT = a.dnT;
  P.d0 = a.dC0; P.dn0 = a.dn0;
  P.T = p.T; P.NC = p.NC;
  P.scale = p.scale;
  P.log2_scale = log2f(p.scale);
  P.epoch = next_epoch();
  auto kern = bwd_walk_kernel<EXPV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)WalkCfg::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)p.BH, 288, WalkCfg::SMEM, s>>>(tQ, tK, tV, tH, tDK, tDV, P);
  return cudaGetLastError();
}

cudaError_t launch_bwd_walk(const Problem& p, const BwdArgs& a, cudaStream_t s) {
  return p.exp_variant() ? launch_walk<true>(p, a, s) : launch_walk<false>(p, a, s);
}

cudaError_t fetch_tc_walk_error(unsigned int* flag) {
  return cudaMemcpyFromSymbol(flag, g_tc_walk_error, sizeof(unsigned int));
}

}  // namespace mlstm
