// Forward inter-chunk state (K-b) and intra-chunk output (K-c) kernels on CUDA
// cores in fp32: the path for fp32 I/O, where bf16 tensor-core operands cannot
// meet a 1e-4 relative error.
//
// Chunkwise form ("Tiled Flash Linear Attention: More Efficient Linear RNN and
// xLSTM Kernels", TFLA summary page, Problem and Approach; arXiv abstract):
// for chunk c with rows t, s and b_t the in-chunk cumsum of log f,
//   C_c = exp(g_c + m_{c-1} - m_c) C_{c-1} + K^T diag(exp(g_c - b_s + log i_s - m_c)) V
//   h_t = [alpha_t q'_t C_{c-1} + sum_{s<=t} exp(b_t - b_s + log i_s - m_t)(q'_t.k_s) v_s] / den_t
// with alpha_t = exp(b_t + m_{c-1} - m_t), m == 0 and den == 1 for mLSTMsig.
#include "common.cuh"
#include "internal.h"

namespace mlstm {

// ---------------------------------------------------------------------------
// K-b: one CTA per (b,h) x 64-row d_qk tile x 64-column d_hv tile walks the
// chunks in order, keeping its state tile in registers (4x4 per thread), and
// stores the state entering every chunk.
// ---------------------------------------------------------------------------
template <typename TIO, typename TS, bool EXPV>
__global__ void __launch_bounds__(256) state_fwd_simt_kernel(
    const TIO* __restrict__ k, const TIO* __restrict__ v, const float* __restrict__ b,
    const float* __restrict__ li, const float* __restrict__ m, TS* __restrict__ C,
    float* __restrict__ n, int T, int L, int NC, int dqk, int dhv, size_t plane, bool keep_lo,
    InitState init) {
  __shared__ float sK[32][64];
  __shared__ float sV[32][64];
  __shared__ float sw[32];
  const int bh = blockIdx.x, i0 = blockIdx.y * 64, j0 = blockIdx.z * 64;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const size_t tok0 = (size_t)bh * T;
  const bool own_n = EXPV && blockIdx.z == 0 && tid < 64;
  // the state entering the first chunk: the initial state, or zero
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
      acc[i][j] = init.on() ? init.C[((size_t)bh * dqk + i0 + ty * 4 + i) * dhv + j0 + tx * 4 + j] : 0.f;
  float nacc = (own_n && init.on()) ? init.n[(size_t)bh * dqk + i0 + tid] : 0.f;
  const float* m0 = init.on() ? init.m : nullptr;

  for (int c = 0; c < NC; ++c) {
    const size_t cbase = ((size_t)bh * NC + c) * dqk * dhv;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        StatePlanes<TS>::store(C, plane, cbase + (size_t)(i0 + ty * 4 + i) * dhv + j0 + tx * 4 + j,
                               acc[i][j], keep_lo);
    if (own_n) n[((size_t)bh * NC + c) * dqk + i0 + tid] = nacc;
    if (c == NC - 1) break;  // no state leaves the last chunk

    const int c0 = c * L, len = min(L, T - c0), last = c0 + len - 1;
    const float g = b[tok0 + last];
    const float mc = EXPV ? m[tok0 + last] : 0.f;
    const float mprev = EXPV ? chunk_mprev(m, tok0 + c0, c, m0, bh) : 0.f;
    const float beta = (c == 0 && !init.on()) ? 0.f : expf(g + mprev - mc);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] *= beta;
    nacc *= beta;

    for (int s0 = 0; s0 < len; s0 += 32) {
      __syncthreads();
      if (tid < 32) {
        const int s = s0 + tid;
        sw[tid] = s < len ? expf(g - b[tok0 + c0 + s] + li[tok0 + c0 + s] - mc) : 0.f;
      }
      __syncthreads();
      for (int e = tid; e < 32 * 64; e += 256) {
        const int r = e >> 6, col = e & 63, s = s0 + r;
        const bool ok = s < len;
        sK[r][col] = ok ? to_f32(k[(tok0 + c0 + s) * dqk + i0 + col]) * sw[r] : 0.f;
        sV[r][col] = ok ? to_f32(v[(tok0 + c0 + s) * dhv + j0 + col]) : 0.f;
      }
      __syncthreads();
#pragma unroll 4
      for (int r = 0; r < 32; ++r) {
        float kr[4], vr[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) kr[i] = sK[r][ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) vr[j] = sV[r][tx * 4 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(kr[i], vr[j], acc[i][j]);
      }
      if (own_n)
        for (int r = 0; r < 32; ++r) nacc += sK[r][tid];
    }
  }
}

cudaError_t launch_state_fwd_simt(const Problem& p, const FwdArgs& a, cudaStream_t s) {
  dim3 grid(p.BH, p.dqk / 64, p.dhv / 64), block(256);
  const size_t plane = (size_t)p.BH * p.NC * p.dqk * p.dhv;
#define MLSTM_STATE_FWD(TIO, TS, E)                                                              \
  state_fwd_simt_kernel<TIO, TS, E><<<grid, block, 0, s>>>((const TIO*)a.k, (const TIO*)a.v, a.b, \
                                                           a.li, a.m, (TS*)a.C, a.n, p.T, p.L,  \
                                                           p.NC, p.dqk, p.dhv, plane, a.keep_lo, a.init)
  if (p.bf16()) {
    if (p.exp_variant()) MLSTM_STATE_FWD(bf16, bf16, true);
    else MLSTM_STATE_FWD(bf16, bf16, false);
  } else {
    if (p.exp_variant()) MLSTM_STATE_FWD(float, float, true);
    else MLSTM_STATE_FWD(float, float, false);
  }
#undef MLSTM_STATE_FWD
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// K-c: one CTA per (b,h,chunk) x 64-row query tile x 64-column d_hv tile.
// Inter-chunk term alpha_t q'_t C_{c-1}, then the kv tiles of the chunk up to
// the diagonal (second-level tiling): S = Q K^T, P = S * D (causal), O += P V,
// and for mLSTMexp the normaliser alpha_t q'_t.n_{c-1} + sum_s P_ts.
// ---------------------------------------------------------------------------
namespace {
constexpr int kPad = 65;
struct OutSmem {
  float qt[32 * kPad];  // Q block, transposed: [kk][row]
  float kt[32 * kPad];  // K block, transposed: [kk][col]
  float p[64 * kPad];   // P tile [row][col]
  float v[64 * 64];     // V tile [s][col], or a [32][64] block of C
  float bt[64], mt[64], alpha[64], rowsum[64], ainter[64], inv[64], bs[64], lis[64];
};
}  // namespace

template <typename TIO, typename TS, bool EXPV>
__global__ void __launch_bounds__(256) output_fwd_simt_kernel(
    const TIO* __restrict__ q, const TIO* __restrict__ k, const TIO* __restrict__ v,
    const float* __restrict__ b, const float* __restrict__ li, const float* __restrict__ m,
    const TS* __restrict__ C, const float* __restrict__ n, TIO* __restrict__ h,
    float* __restrict__ abar_out, int T, int L, int NC, int dqk, int dhv, float scale,
    size_t plane, bool use_lo, bool has_init, const float* __restrict__ m0) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  OutSmem& S = *reinterpret_cast<OutSmem*>(smem_raw);
  const int bh = blockIdx.x / NC, c = blockIdx.x % NC;
  const int c0 = c * L, len = min(L, T - c0);
  const int t0 = blockIdx.y * 64;
  if (t0 >= len) return;
  const int j0 = blockIdx.z * 64;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const size_t tok0 = (size_t)bh * T + c0;  // first token of the chunk
  const float mprev = EXPV ? chunk_mprev(m, (size_t)bh * T + c0, c, m0, bh) : 0.f;
  const bool has_prev = c > 0 || has_init;  // a state enters this chunk

  if (tid < 64) {
    const int t = t0 + tid;
    const bool ok = t < len;
    const float bt = ok ? b[tok0 + t] : 0.f;
    const float mt = (EXPV && ok) ? m[tok0 + t] : 0.f;
    S.bt[tid] = bt;
    S.mt[tid] = mt;
    S.alpha[tid] = (ok && has_prev) ? expf(bt + mprev - mt) : 0.f;
    S.rowsum[tid] = 0.f;
    S.ainter[tid] = 0.f;
  }
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  // inter-chunk term
  if (has_prev) {
    const size_t cbase = ((size_t)bh * NC + c) * dqk * dhv;
    for (int kk0 = 0; kk0 < dqk; kk0 += 32) {
      __syncthreads();
      for (int e = tid; e < 64 * 32; e += 256) {
        const int r = e >> 5, x = e & 31, t = t0 + r;
        S.qt[x * kPad + r] = t < len ? to_f32(q[(tok0 + t) * dqk + kk0 + x]) : 0.f;
      }
      for (int e = tid; e < 32 * 64; e += 256) {
        const int x = e >> 6, col = e & 63;
        S.v[x * 64 + col] = StatePlanes<TS>::load(C, plane, cbase + (size_t)(kk0 + x) * dhv + j0 + col, use_lo);
      }
      __syncthreads();
#pragma unroll 4
      for (int x = 0; x < 32; ++x) {
        float qa[4], cb[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) qa[i] = S.qt[x * kPad + ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) cb[j] = S.v[x * 64 + tx * 4 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(qa[i], cb[j], acc[i][j]);
      }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float f = S.alpha[ty * 4 + i] * scale;
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] *= f;
    }
    if (EXPV && tid < 64 && t0 + tid < len) {
      const float* nc = n + ((size_t)bh * NC + c) * dqk;
      const size_t row = (tok0 + t0 + tid) * dqk;
      float dot = 0.f;
      for (int x = 0; x < dqk; ++x) dot = fmaf(to_f32(q[row + x]), nc[x], dot);
      S.ainter[tid] = dot * S.alpha[tid] * scale;
    }
  }

  // intra-chunk kv tiles up to the diagonal
  for (int s0 = 0; s0 <= t0; s0 += 64) {
    __syncthreads();
    if (tid < 64) {
      const int s = s0 + tid;
      S.bs[tid] = s < len ? b[tok0 + s] : 0.f;
      S.lis[tid] = s < len ? li[tok0 + s] : -INFINITY;
    }
    float sacc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) sacc[i][j] = 0.f;
    for (int kk0 = 0; kk0 < dqk; kk0 += 32) {
      __syncthreads();
      for (int e = tid; e < 64 * 32; e += 256) {
        const int r = e >> 5, x = e & 31;
        const int t = t0 + r, s = s0 + r;
        S.qt[x * kPad + r] = t < len ? to_f32(q[(tok0 + t) * dqk + kk0 + x]) : 0.f;
        S.kt[x * kPad + r] = s < len ? to_f32(k[(tok0 + s) * dqk + kk0 + x]) : 0.f;
      }
      __syncthreads();
#pragma unroll 4
      for (int x = 0; x < 32; ++x) {
        float qa[4], kb[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) qa[i] = S.qt[x * kPad + ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) kb[j] = S.kt[x * kPad + tx * 4 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) sacc[i][j] = fmaf(qa[i], kb[j], sacc[i][j]);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = ty * 4 + i, t = t0 + r;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int cc = tx * 4 + j, s = s0 + cc;
        float pv = 0.f;
        if (s <= t && t < len && s < len)
          pv = sacc[i][j] * scale * expf(S.bt[r] - S.bs[cc] + S.lis[cc] - S.mt[r]);
        S.p[r * kPad + cc] = pv;
      }
    }
    for (int e = tid; e < 64 * 64; e += 256) {
      const int r = e >> 6, col = e & 63, s = s0 + r;
      S.v[r * 64 + col] = s < len ? to_f32(v[(tok0 + s) * dhv + j0 + col]) : 0.f;
    }
    __syncthreads();
    if (EXPV && tid < 64) {
      float rs = 0.f;
      for (int x = 0; x < 64; ++x) rs += S.p[tid * kPad + x];
      S.rowsum[tid] += rs;
    }
#pragma unroll 4
    for (int x = 0; x < 64; ++x) {
      float pa[4], vb[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) pa[i] = S.p[(ty * 4 + i) * kPad + x];
#pragma unroll
      for (int j = 0; j < 4; ++j) vb[j] = S.v[x * 64 + tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(pa[i], vb[j], acc[i][j]);
    }
  }

  __syncthreads();
  if (tid < 64) {
    float inv = 1.f;
    if (EXPV) {
      const float a = S.ainter[tid] + S.rowsum[tid];
      inv = 1.f / fmaxf(fabsf(a), expf(-S.mt[tid]));
      if (blockIdx.z == 0 && t0 + tid < len) abar_out[tok0 + t0 + tid] = a;
    }
    S.inv[tid] = inv;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty * 4 + i, t = t0 + r;
    if (t >= len) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      h[(tok0 + t) * dhv + j0 + tx * 4 + j] = from_f32<TIO>(acc[i][j] * S.inv[r]);
  }
}

cudaError_t launch_output_fwd_simt(const Problem& p, const FwdArgs& a, cudaStream_t s) {
  dim3 grid(p.BH * p.NC, (p.L + 63) / 64, p.dhv / 64), block(256);
  const size_t smem = sizeof(OutSmem);
  const size_t plane = (size_t)p.BH * p.NC * p.dqk * p.dhv;
  cudaError_t e = cudaSuccess;
#define MLSTM_OUT_FWD(TIO, TS, E)                                                                \
  do {                                                                                           \
    e = cudaFuncSetAttribute(output_fwd_simt_kernel<TIO, TS, E>,                                 \
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);            \
    if (e != cudaSuccess) return e;                                                              \
    output_fwd_simt_kernel<TIO, TS, E><<<grid, block, smem, s>>>(                                \
        (const TIO*)a.q, (const TIO*)a.k, (const TIO*)a.v, a.b, a.li, a.m, (const TS*)a.C, a.n, \
        (TIO*)a.h, a.abar, p.T, p.L, p.NC, p.dqk, p.dhv, p.scale, plane, a.keep_lo,             \
        a.init.on(), a.init.on() ? a.init.m : nullptr);                                          \
  } while (0)
  if (p.bf16()) {
    if (p.exp_variant()) MLSTM_OUT_FWD(bf16, bf16, true);
    else MLSTM_OUT_FWD(bf16, bf16, false);
  } else {
    if (p.exp_variant()) MLSTM_OUT_FWD(float, float, true);
    else MLSTM_OUT_FWD(float, float, false);
  }
#undef MLSTM_OUT_FWD
  return cudaGetLastError();
}

}  // namespace mlstm
