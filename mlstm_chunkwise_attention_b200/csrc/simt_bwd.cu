// Backward kernels on CUDA cores in fp32 (the fp32-I/O path): the reverse
// state-gradient recurrence (K-d1) and the intra-chunk gradients dq, dk, dv
// (K-d2).
//
// With the max state m treated as a constant (the output does not depend on
// it), dnum_t = dh_t / den_t, da_t the normaliser gradient, and for s <= t in
// chunk c:  D_ts = exp(b_t - b_s + log i_s - m_t), A_ts = D_ts (q'_t . k_s),
// dA_ts = dnum_t . v_s + da_t:
//   dq'_t = alpha_t (C_{c-1} dnum_t + da_t n_{c-1}) + sum_s dA_ts D_ts k_s
//   dk_s  = w_s (dC_c v_s + dn_c)                    + sum_t dA_ts D_ts q'_t
//   dv_s  = w_s dC_c^T k_s                           + sum_t A_ts dnum_t
// where dC_c is the gradient of the state leaving chunk c:
//   dC_{c-1} = beta_c dC_c + sum_{t in c} alpha_t q'_t dnum_t^T,
//   dn_{c-1} = beta_c dn_c + sum_{t in c} alpha_t da_t q'_t,
// alpha_t = exp(b_t + m_{c-1} - m_t), w_s = exp(g_c - b_s + log i_s - m_c),
// beta_c = exp(g_c + m_{c-1} - m_c).  Timed as the training kernels of "Tiled
// Flash Linear Attention: More Efficient Linear RNN and xLSTM Kernels" (TFLA
// summary page, Key results).
#include "common.cuh"
#include "internal.h"

namespace mlstm {

// ---------------------------------------------------------------------------
// K-d1: reverse walk over the chunks; stores dC_c for every chunk.
// ---------------------------------------------------------------------------
template <typename TIO, typename TS, bool EXPV>
__global__ void __launch_bounds__(256) state_bwd_simt_kernel(
    const TIO* __restrict__ q, const TIO* __restrict__ dh, const float* __restrict__ b,
    const float* __restrict__ m, const float* __restrict__ inv_den, const float* __restrict__ da,
    TS* __restrict__ dC, float* __restrict__ dn, int T, int L, int NC, int dqk, int dhv,
    float scale, size_t plane, const float* __restrict__ m0, float* __restrict__ d0,
    float* __restrict__ dn0, const float* __restrict__ dT, const float* __restrict__ dnT) {
  __shared__ float sQ[32][64];
  __shared__ float sD[32][64];
  __shared__ float fq[32], fn[32];
  const int bh = blockIdx.x, i0 = blockIdx.y * 64, j0 = blockIdx.z * 64;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const size_t tokh = (size_t)bh * T;
  const bool own_n = EXPV && blockIdx.z == 0 && tid < 64;
  // the gradient of the state leaving the last chunk: the final state's, or zero
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
      acc[i][j] = dT ? dT[((size_t)bh * dqk + i0 + ty * 4 + i) * dhv + j0 + tx * 4 + j] : 0.f;
  float nacc = (own_n && dT) ? dnT[(size_t)bh * dqk + i0 + tid] : 0.f;

  for (int c = NC - 1; c >= 0; --c) {
    const size_t gbase = ((size_t)bh * NC + c) * dqk * dhv;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        StatePlanes<TS>::store(dC, plane, gbase + (size_t)(i0 + ty * 4 + i) * dhv + j0 + tx * 4 + j,
                               acc[i][j], true);
    if (own_n) dn[((size_t)bh * NC + c) * dqk + i0 + tid] = nacc;
    if (c == 0 && d0 == nullptr) break;  // the first chunk's contribution: the initial state's gradient

    const int c0 = c * L, len = min(L, T - c0), last = c0 + len - 1;
    const float g = b[tokh + last];
    const float mc = EXPV ? m[tokh + last] : 0.f;
    const float mprev = EXPV ? chunk_mprev(m, tokh + c0, c, m0, bh) : 0.f;
    const float beta = expf(g + mprev - mc);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] *= beta;
    nacc *= beta;

    for (int r0 = 0; r0 < len; r0 += 32) {
      __syncthreads();
      if (tid < 32) {
        const int t = r0 + tid;
        float f = 0.f, idn = 0.f, dat = 0.f;
        if (t < len) {
          const size_t ti = tokh + c0 + t;
          f = expf(b[ti] + mprev - (EXPV ? m[ti] : 0.f)) * scale;
          idn = EXPV ? inv_den[ti] : 1.f;
          dat = EXPV ? da[ti] : 0.f;
        }
        fq[tid] = f * idn;
        fn[tid] = f * dat;
      }
      __syncthreads();
      for (int e = tid; e < 32 * 64; e += 256) {
        const int r = e >> 6, col = e & 63, t = r0 + r;
        const bool ok = t < len;
        sQ[r][col] = ok ? to_f32(q[(tokh + c0 + t) * dqk + i0 + col]) : 0.f;
        sD[r][col] = ok ? to_f32(dh[(tokh + c0 + t) * dhv + j0 + col]) * fq[r] : 0.f;
      }
      __syncthreads();
#pragma unroll 4
      for (int r = 0; r < 32; ++r) {
        float qa[4], db[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) qa[i] = sQ[r][ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) db[j] = sD[r][tx * 4 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(qa[i], db[j], acc[i][j]);
      }
      if (own_n)
        for (int r = 0; r < 32; ++r) nacc = fmaf(sQ[r][tid], fn[r], nacc);
    }
  }
  if (d0 != nullptr) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) d0[((size_t)bh * dqk + i0 + ty * 4 + i) * dhv + j0 + tx * 4 + j] = acc[i][j];
    if (own_n) dn0[(size_t)bh * dqk + i0 + tid] = nacc;
  }
}

cudaError_t launch_state_bwd_simt(const Problem& p, const BwdArgs& a, cudaStream_t s) {
  dim3 grid(p.BH, p.dqk / 64, p.dhv / 64), block(256);
#define MLSTM_STATE_BWD(TIO, TS, E)                                                             \
  state_bwd_simt_kernel<TIO, TS, E><<<grid, block, 0, s>>>(                                     \
      (const TIO*)a.q, (const TIO*)a.dh, a.b, a.m, a.inv_den, a.da, (TS*)a.dC, a.dn, p.T, p.L,  \
      p.NC, p.dqk, p.dhv, p.scale, (size_t)p.BH * p.NC * p.dqk * p.dhv,                     \
      a.init.on() ? a.init.m : nullptr, a.dC0, a.dn0, a.dCT, a.dnT)
  if (p.bf16()) {
    if (p.exp_variant()) MLSTM_STATE_BWD(bf16, bf16, true);
    else MLSTM_STATE_BWD(bf16, bf16, false);
  } else {
    if (p.exp_variant()) MLSTM_STATE_BWD(float, float, true);
    else MLSTM_STATE_BWD(float, float, false);
  }
#undef MLSTM_STATE_BWD
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// K-d2 building blocks.  Each CTA owns a 64 x 64 output tile; thread (ty, tx)
// owns rows ty*4.., columns tx*4...  Tiles are staged through shared memory
// transposed ([contraction][row]) with one column of padding.
// ---------------------------------------------------------------------------
namespace {
constexpr int kP = 65;
struct BwdSmem {
  float a[32 * kP];  // contraction block of the "row" operand, [x][row]
  float bt[32 * kP]; // contraction block of the "column" operand, [x][col]
  float p[64 * kP];  // dS or A tile
  float w[64 * 64];  // right operand of the second product [k][col]
  // per-row (t) and per-column (s) gate factors of the current tiles
  float tb[64], tm[64], tinv[64], tda[64], talpha[64];
  float sb[64], sli[64], sw[64];
};

__device__ __forceinline__ void zero44(float (&x)[4][4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) x[i][j] = 0.f;
}

// x[i][j] += sum_k A[k][ty*4+i] * B[k][tx*4+j] over k < K (A, B with row stride ld)
__device__ __forceinline__ void mac44(float (&x)[4][4], const float* A, int lda, const float* B,
                                      int ldb, int K, int ty, int tx) {
#pragma unroll 4
  for (int kk = 0; kk < K; ++kk) {
    float ra[4], rb[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) ra[i] = A[kk * lda + ty * 4 + i];
#pragma unroll
    for (int j = 0; j < 4; ++j) rb[j] = B[kk * ldb + tx * 4 + j];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) x[i][j] = fmaf(ra[i], rb[j], x[i][j]);
  }
}

// Per-row (query side) gate factors for the rows t0.. of chunk c.
template <bool EXPV>
__device__ __forceinline__ void load_row_factors(BwdSmem& S, const float* b, const float* m,
                                                 const float* inv_den, const float* da,
                                                 size_t tok0, int t0, int len, float mprev,
                                                 bool has_prev) {
  const int tid = threadIdx.x;
  if (tid < 64) {
    const int t = t0 + tid;
    const bool ok = t < len;
    const float bt = ok ? b[tok0 + t] : 0.f;
    const float mt = (EXPV && ok) ? m[tok0 + t] : 0.f;
    S.tb[tid] = bt;
    S.tm[tid] = mt;
    S.tinv[tid] = ok ? (EXPV ? inv_den[tok0 + t] : 1.f) : 0.f;
    S.tda[tid] = (EXPV && ok) ? da[tok0 + t] : 0.f;
    S.talpha[tid] = (ok && has_prev) ? expf(bt + mprev - mt) : 0.f;
  }
}

// Per-column (key side) gate factors for the rows s0.. of chunk c.
__device__ __forceinline__ void load_col_factors(BwdSmem& S, const float* b, const float* li,
                                                 size_t tok0, int s0, int len, float g, float mc) {
  const int tid = threadIdx.x;
  if (tid < 64) {
    const int s = s0 + tid;
    const bool ok = s < len;
    const float bs = ok ? b[tok0 + s] : 0.f;
    const float ls = ok ? li[tok0 + s] : -INFINITY;
    S.sb[tid] = bs;
    S.sli[tid] = ls;
    S.sw[tid] = ok ? expf(g - bs + ls - mc) : 0.f;
  }
}
}  // namespace

// dq for a 64-row query tile and 64 columns of d_qk.
template <typename TIO, typename TS, bool EXPV>
__global__ void __launch_bounds__(256) dq_simt_kernel(
    const TIO* __restrict__ q, const TIO* __restrict__ k, const TIO* __restrict__ v,
    const TIO* __restrict__ dh, const float* __restrict__ b, const float* __restrict__ li,
    const float* __restrict__ m, const float* __restrict__ inv_den, const float* __restrict__ da,
    const TS* __restrict__ C, const float* __restrict__ n, TIO* __restrict__ dq,
    float* __restrict__ pq, int T, int L, int NC, int dqk, int dhv, float scale, size_t plane,
    bool has_init, const float* __restrict__ m0) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  BwdSmem& S = *reinterpret_cast<BwdSmem*>(smem_raw);
  const int bh = blockIdx.x / NC, c = blockIdx.x % NC;
  const int c0 = c * L, len = min(L, T - c0);
  const int t0 = blockIdx.y * 64;
  if (t0 >= len) return;
  const int i0 = blockIdx.z * 64;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const size_t tok0 = (size_t)bh * T + c0;
  const float mprev = EXPV ? chunk_mprev(m, (size_t)bh * T + c0, c, m0, bh) : 0.f;
  const bool has_prev = c > 0 || has_init;  // a state enters this chunk
  load_row_factors<EXPV>(S, b, m, inv_den, da, tok0, t0, len, mprev, has_prev);
  float acc[4][4];
  zero44(acc);

  if (has_prev) {  // alpha_t (C_{c-1} dnum_t + da_t n_{c-1})
    const size_t cbase = ((size_t)bh * NC + c) * dqk * dhv;
    for (int x0 = 0; x0 < dhv; x0 += 32) {
      __syncthreads();
      for (int e = tid; e < 64 * 32; e += 256) {
        const int r = e >> 5, x = e & 31, t = t0 + r;
        S.a[x * kP + r] = t < len ? to_f32(dh[(tok0 + t) * dhv + x0 + x]) * S.tinv[r] : 0.f;
        S.bt[x * kP + r] = StatePlanes<TS>::load(C, plane, cbase + (size_t)(i0 + r) * dhv + x0 + x);
      }
      __syncthreads();
      mac44(acc, S.a, kP, S.bt, kP, 32, ty, tx);
    }
    const float* nc = n + ((size_t)bh * NC + c) * dqk;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = ty * 4 + i;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        acc[i][j] = S.talpha[r] * (acc[i][j] + (EXPV ? S.tda[r] * nc[i0 + tx * 4 + j] : 0.f));
    }
  }

  for (int s0 = 0; s0 <= t0; s0 += 64) {
    __syncthreads();
    load_col_factors(S, b, li, tok0, s0, len, 0.f, 0.f);
    float pacc[4][4];
    zero44(pacc);
    for (int x0 = 0; x0 < dhv; x0 += 32) {  // dP_ts = dnum_t . v_s
      __syncthreads();
      for (int e = tid; e < 64 * 32; e += 256) {
        const int r = e >> 5, x = e & 31, t = t0 + r, s = s0 + r;
        S.a[x * kP + r] = t < len ? to_f32(dh[(tok0 + t) * dhv + x0 + x]) * S.tinv[r] : 0.f;
        S.bt[x * kP + r] = s < len ? to_f32(v[(tok0 + s) * dhv + x0 + x]) : 0.f;
      }
      __syncthreads();
      mac44(pacc, S.a, kP, S.bt, kP, 32, ty, tx);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = ty * 4 + i, t = t0 + r;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int cc = tx * 4 + j, s = s0 + cc;
        float d = 0.f;
        if (s <= t && t < len && s < len)
          d = (pacc[i][j] + S.tda[r]) * expf(S.tb[r] - S.sb[cc] + S.sli[cc] - S.tm[r]);
        S.p[cc * kP + r] = d;  // stored [s][t] as the contraction-major row operand
      }
    }
    for (int e = tid; e < 64 * 64; e += 256) {
      const int r = e >> 6, col = e & 63, s = s0 + r;
      S.w[r * 64 + col] = s < len ? to_f32(k[(tok0 + s) * dqk + i0 + col]) : 0.f;
    }
    __syncthreads();
    mac44(acc, S.p, kP, S.w, 64, 64, ty, tx);
  }

  // dq = dq' / sqrt(d_qk) ... = scale * dq'; and the partial q . dq of this column tile
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty * 4 + i, t = t0 + r;
    float part = 0.f;
    if (t < len) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float g = acc[i][j] * scale;
        const size_t idx = (tok0 + t) * dqk + i0 + tx * 4 + j;
        dq[idx] = from_f32<TIO>(g);
        part = fmaf(to_f32(q[idx]), g, part);
      }
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (tx == 0 && t < len) atomicAdd(&pq[tok0 + t], part);
  }
}

// dk for a 64-row key tile and 64 columns of d_qk.
template <typename TIO, typename TS, bool EXPV>
__global__ void __launch_bounds__(256) dk_simt_kernel(
    const TIO* __restrict__ q, const TIO* __restrict__ k, const TIO* __restrict__ v,
    const TIO* __restrict__ dh, const float* __restrict__ b, const float* __restrict__ li,
    const float* __restrict__ m, const float* __restrict__ inv_den, const float* __restrict__ da,
    const TS* __restrict__ dC, const float* __restrict__ dn, TIO* __restrict__ dk,
    float* __restrict__ pk, int T, int L, int NC, int dqk, int dhv, float scale, size_t plane,
    bool dfin) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  BwdSmem& S = *reinterpret_cast<BwdSmem*>(smem_raw);
  const int bh = blockIdx.x / NC, c = blockIdx.x % NC;
  const int c0 = c * L, len = min(L, T - c0);
  const int s0 = blockIdx.y * 64;
  if (s0 >= len) return;
  const int i0 = blockIdx.z * 64;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const size_t tok0 = (size_t)bh * T + c0;
  const float g = b[tok0 + len - 1];
  const float mc = EXPV ? m[tok0 + len - 1] : 0.f;
  load_col_factors(S, b, li, tok0, s0, len, g, mc);
  float acc[4][4];
  zero44(acc);

  if (c < NC - 1 || dfin) {  // w_s (dC_c v_s + dn_c)
    const size_t gbase = ((size_t)bh * NC + c) * dqk * dhv;
    for (int x0 = 0; x0 < dhv; x0 += 32) {
      __syncthreads();
      for (int e = tid; e < 64 * 32; e += 256) {
        const int r = e >> 5, x = e & 31, s = s0 + r;
        S.a[x * kP + r] = s < len ? to_f32(v[(tok0 + s) * dhv + x0 + x]) : 0.f;
        S.bt[x * kP + r] = StatePlanes<TS>::load(dC, plane, gbase + (size_t)(i0 + r) * dhv + x0 + x);
      }
      __syncthreads();
      mac44(acc, S.a, kP, S.bt, kP, 32, ty, tx);
    }
    const float* gn = dn + ((size_t)bh * NC + c) * dqk;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = ty * 4 + i;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        acc[i][j] = S.sw[r] * (acc[i][j] + (EXPV ? gn[i0 + tx * 4 + j] : 0.f));
    }
  }

  for (int t0 = s0; t0 < len; t0 += 64) {
    __syncthreads();
    load_row_factors<EXPV>(S, b, m, inv_den, da, tok0, t0, len, 0.f, false);
    float pacc[4][4];  // [s][t] = v_s . dnum_t
    zero44(pacc);
    for (int x0 = 0; x0 < dhv; x0 += 32) {
      __syncthreads();
      for (int e = tid; e < 64 * 32; e += 256) {
        const int r = e >> 5, x = e & 31, t = t0 + r, s = s0 + r;
        S.a[x * kP + r] = s < len ? to_f32(v[(tok0 + s) * dhv + x0 + x]) : 0.f;
        S.bt[x * kP + r] = t < len ? to_f32(dh[(tok0 + t) * dhv + x0 + x]) * S.tinv[r] : 0.f;
      }
      __syncthreads();
      mac44(pacc, S.a, kP, S.bt, kP, 32, ty, tx);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = ty * 4 + i, s = s0 + r;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int cc = tx * 4 + j, t = t0 + cc;
        float d = 0.f;
        if (s <= t && t < len && s < len)
          d = (pacc[i][j] + S.tda[cc]) * expf(S.tb[cc] - S.sb[r] + S.sli[r] - S.tm[cc]);
        S.p[cc * kP + r] = d;  // [t][s]
      }
    }
    for (int e = tid; e < 64 * 64; e += 256) {
      const int r = e >> 6, col = e & 63, t = t0 + r;
      S.w[r * 64 + col] = t < len ? to_f32(q[(tok0 + t) * dqk + i0 + col]) * scale : 0.f;
    }
    __syncthreads();
    mac44(acc, S.p, kP, S.w, 64, 64, ty, tx);
  }

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty * 4 + i, s = s0 + r;
    float part = 0.f;
    if (s < len) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const size_t idx = (tok0 + s) * dqk + i0 + tx * 4 + j;
        dk[idx] = from_f32<TIO>(acc[i][j]);
        part = fmaf(to_f32(k[idx]), acc[i][j], part);
      }
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (tx == 0 && s < len) atomicAdd(&pk[tok0 + s], part);
  }
}

// dv for a 64-row key tile and 64 columns of d_hv.
template <typename TIO, typename TS, bool EXPV>
__global__ void __launch_bounds__(256) dv_simt_kernel(
    const TIO* __restrict__ q, const TIO* __restrict__ k, const TIO* __restrict__ dh,
    const float* __restrict__ b, const float* __restrict__ li, const float* __restrict__ m,
    const float* __restrict__ inv_den, const TS* __restrict__ dC, TIO* __restrict__ dv, int T,
    int L, int NC, int dqk, int dhv, float scale, size_t plane, bool dfin) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  BwdSmem& S = *reinterpret_cast<BwdSmem*>(smem_raw);
  const int bh = blockIdx.x / NC, c = blockIdx.x % NC;
  const int c0 = c * L, len = min(L, T - c0);
  const int s0 = blockIdx.y * 64;
  if (s0 >= len) return;
  const int j0 = blockIdx.z * 64;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const size_t tok0 = (size_t)bh * T + c0;
  const float g = b[tok0 + len - 1];
  const float mc = EXPV ? m[tok0 + len - 1] : 0.f;
  load_col_factors(S, b, li, tok0, s0, len, g, mc);
  float acc[4][4];
  zero44(acc);

  if (c < NC - 1 || dfin) {  // w_s dC_c^T k_s
    const size_t gbase = ((size_t)bh * NC + c) * dqk * dhv;
    for (int x0 = 0; x0 < dqk; x0 += 32) {
      __syncthreads();
      for (int e = tid; e < 64 * 32; e += 256) {
        const int r = e >> 5, x = e & 31, s = s0 + r;
        S.a[x * kP + r] = s < len ? to_f32(k[(tok0 + s) * dqk + x0 + x]) : 0.f;
      }
      for (int e = tid; e < 32 * 64; e += 256) {
        const int x = e >> 6, col = e & 63;
        S.w[x * 64 + col] = StatePlanes<TS>::load(dC, plane, gbase + (size_t)(x0 + x) * dhv + j0 + col);
      }
      __syncthreads();
      mac44(acc, S.a, kP, S.w, 64, 32, ty, tx);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] *= S.sw[ty * 4 + i];
  }

  for (int t0 = s0; t0 < len; t0 += 64) {
    __syncthreads();
    load_row_factors<EXPV>(S, b, m, inv_den, inv_den, tok0, t0, len, 0.f, false);
    float sacc[4][4];  // [s][t] = k_s . q'_t
    zero44(sacc);
    for (int x0 = 0; x0 < dqk; x0 += 32) {
      __syncthreads();
      for (int e = tid; e < 64 * 32; e += 256) {
        const int r = e >> 5, x = e & 31, t = t0 + r, s = s0 + r;
        S.a[x * kP + r] = s < len ? to_f32(k[(tok0 + s) * dqk + x0 + x]) : 0.f;
        S.bt[x * kP + r] = t < len ? to_f32(q[(tok0 + t) * dqk + x0 + x]) * scale : 0.f;
      }
      __syncthreads();
      mac44(sacc, S.a, kP, S.bt, kP, 32, ty, tx);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = ty * 4 + i, s = s0 + r;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int cc = tx * 4 + j, t = t0 + cc;
        float a = 0.f;
        if (s <= t && t < len && s < len)
          a = sacc[i][j] * expf(S.tb[cc] - S.sb[r] + S.sli[r] - S.tm[cc]);
        S.p[cc * kP + r] = a;  // [t][s]
      }
    }
    for (int e = tid; e < 64 * 64; e += 256) {
      const int r = e >> 6, col = e & 63, t = t0 + r;
      S.w[r * 64 + col] = t < len ? to_f32(dh[(tok0 + t) * dhv + j0 + col]) * S.tinv[r] : 0.f;
    }
    __syncthreads();
    mac44(acc, S.p, kP, S.w, 64, 64, ty, tx);
  }

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int s = s0 + ty * 4 + i;
    if (s >= len) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) dv[(tok0 + s) * dhv + j0 + tx * 4 + j] = from_f32<TIO>(acc[i][j]);
  }
}

template <typename TIO, typename TS, bool E>
static cudaError_t dq_launch(const Problem& p, const BwdArgs& a, cudaStream_t s) {
  const int smem = (int)sizeof(BwdSmem);
  cudaError_t e = cudaFuncSetAttribute(dq_simt_kernel<TIO, TS, E>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.BH * p.NC, (p.L + 63) / 64, p.dqk / 64);
  dq_simt_kernel<TIO, TS, E><<<grid, 256, smem, s>>>(
      (const TIO*)a.q, (const TIO*)a.k, (const TIO*)a.v, (const TIO*)a.dh, a.b, a.li, a.m,
      a.inv_den, a.da, (const TS*)a.C, a.n, (TIO*)a.dq, a.pq, p.T, p.L, p.NC, p.dqk, p.dhv,
      p.scale, (size_t)p.BH * p.NC * p.dqk * p.dhv, a.init.on(), a.init.on() ? a.init.m : nullptr);
  return cudaGetLastError();
}

template <typename TIO, typename TS, bool E>
static cudaError_t dk_launch(const Problem& p, const BwdArgs& a, cudaStream_t s) {
  const int smem = (int)sizeof(BwdSmem);
  cudaError_t e = cudaFuncSetAttribute(dk_simt_kernel<TIO, TS, E>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.BH * p.NC, (p.L + 63) / 64, p.dqk / 64);
  dk_simt_kernel<TIO, TS, E><<<grid, 256, smem, s>>>(
      (const TIO*)a.q, (const TIO*)a.k, (const TIO*)a.v, (const TIO*)a.dh, a.b, a.li, a.m,
      a.inv_den, a.da, (const TS*)a.dC, a.dn, (TIO*)a.dk, a.pk, p.T, p.L, p.NC, p.dqk, p.dhv,
      p.scale, (size_t)p.BH * p.NC * p.dqk * p.dhv, a.dCT != nullptr);
  return cudaGetLastError();
}

template <typename TIO, typename TS, bool E>
static cudaError_t dv_launch(const Problem& p, const BwdArgs& a, cudaStream_t s) {
  const int smem = (int)sizeof(BwdSmem);
  cudaError_t e = cudaFuncSetAttribute(dv_simt_kernel<TIO, TS, E>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.BH * p.NC, (p.L + 63) / 64, p.dhv / 64);
  dv_simt_kernel<TIO, TS, E><<<grid, 256, smem, s>>>(
      (const TIO*)a.q, (const TIO*)a.k, (const TIO*)a.dh, a.b, a.li, a.m, a.inv_den,
      (const TS*)a.dC, (TIO*)a.dv, p.T, p.L, p.NC, p.dqk, p.dhv, p.scale,
      (size_t)p.BH * p.NC * p.dqk * p.dhv, a.dCT != nullptr);
  return cudaGetLastError();
}

#define MLSTM_BWD_DISPATCH(FN)                                                        \
  if (p.bf16())                                                                      \
    return p.exp_variant() ? FN<bf16, bf16, true>(p, a, s) : FN<bf16, bf16, false>(p, a, s); \
  return p.exp_variant() ? FN<float, float, true>(p, a, s) : FN<float, float, false>(p, a, s)

cudaError_t launch_dq_simt(const Problem& p, const BwdArgs& a, cudaStream_t s) {
  MLSTM_BWD_DISPATCH(dq_launch);
}
cudaError_t launch_dk_simt(const Problem& p, const BwdArgs& a, cudaStream_t s) {
  MLSTM_BWD_DISPATCH(dk_launch);
}
cudaError_t launch_dv_simt(const Problem& p, const BwdArgs& a, cudaStream_t s) {
  MLSTM_BWD_DISPATCH(dv_launch);
}
#undef MLSTM_BWD_DISPATCH

}  // namespace mlstm
