// Recurrent-form kernels: the state after the last token of a chunkwise
// forward (so a prefill can hand its state to step-by-step generation) and one
// token of the recurrence (the FusedRecurrent form of the flash-linear-attention
// README; the mLSTM recurrence of "Tiled Flash Linear Attention", TFLA summary
// page, Approach).  State layout (fp32, per head): C [d_qk, d_hv], n [d_qk],
// m; for EXP C and n are stabilised, i.e. scaled by exp(-m).
//
// Both kernels are HBM-bound: the step reads and writes the whole state once
// per token; the final state reads the state entering the last chunk and that
// chunk's keys and values once.  They run on CUDA cores with fp32 arithmetic.
#include "common.cuh"
#include "internal.h"

namespace mlstm {

namespace {

constexpr float kNegInf = -INFINITY;
constexpr int kTok = 32;  // tokens per shared-memory tile of the final-state kernel

// One CTA per (64 columns of C, head).  C_final = beta C_enter + sum_s w_s k_s v_s^T over
// the last chunk's tokens, with beta = exp(g + m_enter - m_T), w_s = exp(g - b_s + log i_s - m_T)
// (m == 0 for SIG), g = b at the last token; n likewise (CTA of the first column block).
template <typename TIO, typename TS, bool EXPV, int DQK>
__global__ void __launch_bounds__(256) final_state_kernel(
    const TIO* __restrict__ k, const TIO* __restrict__ v, const float* __restrict__ b,
    const float* __restrict__ li, const float* __restrict__ m, const TS* __restrict__ C,
    const float* __restrict__ n, size_t plane, float* __restrict__ Cout,
    float* __restrict__ nout, float* __restrict__ mout, int T, int L, int NC, int dhv,
    bool has_init, const float* __restrict__ m0) {
  __shared__ float ks[kTok][DQK];
  __shared__ float vs[kTok][64];
  __shared__ float ws[kTok];
  const int bh = blockIdx.y, j0 = blockIdx.x * 64, tid = threadIdx.x;
  const int jj = tid & 63, rg = tid >> 6;  // column, row group (rows rg, rg + 4, ...)
  const int c = NC - 1, lo = c * L;
  const size_t tok0 = (size_t)bh * T;
  const float g = b[tok0 + T - 1];
  const float mT = EXPV ? m[tok0 + T - 1] : 0.f;
  // a state enters the last chunk: an earlier chunk's, or the initial state
  const bool has_prev = c > 0 || has_init;
  const float menter = EXPV ? chunk_mprev(m, tok0 + lo, c, m0, bh) : 0.f;
  const float beta = has_prev ? expf(g + menter - mT) : 0.f;
  constexpr int R = DQK / 4;
  float acc[R];
#pragma unroll
  for (int r = 0; r < R; ++r) acc[r] = 0.f;
  float nacc = 0.f;  // thread tid < DQK of column block 0: n_final[tid]
  for (int s0 = lo; s0 < T; s0 += kTok) {
    const int cnt = min(kTok, T - s0);
    __syncthreads();
    for (int e = tid; e < kTok * DQK; e += 256) {
      const int s = e / DQK, i = e % DQK;
      ks[s][i] = s < cnt ? to_f32(k[(tok0 + s0 + s) * DQK + i]) : 0.f;
    }
    for (int e = tid; e < kTok * 64; e += 256) {
      const int s = e >> 6, j = e & 63;
      vs[s][j] = (s < cnt && j0 + j < dhv) ? to_f32(v[(tok0 + s0 + s) * dhv + j0 + j]) : 0.f;
    }
    if (tid < kTok)
      ws[tid] = tid < cnt ? expf(g - b[tok0 + s0 + tid] + li[tok0 + s0 + tid] - mT) : 0.f;
    __syncthreads();
    for (int s = 0; s < cnt; ++s) {
      const float wv = ws[s] * vs[s][jj];
#pragma unroll
      for (int r = 0; r < R; ++r) acc[r] = fmaf(ks[s][rg + 4 * r], wv, acc[r]);
      if (EXPV && blockIdx.x == 0 && tid < DQK) nacc = fmaf(ws[s], ks[s][tid], nacc);
    }
  }
  const size_t cbase = ((size_t)bh * NC + c) * DQK * dhv;
  const int j = j0 + jj;
  if (j < dhv) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int i = rg + 4 * r;
      const float prev = has_prev ? StatePlanes<TS>::load(C, plane, cbase + (size_t)i * dhv + j) : 0.f;
      Cout[((size_t)bh * DQK + i) * dhv + j] = beta * prev + acc[r];
    }
  }
  if (EXPV && blockIdx.x == 0) {
    if (tid < DQK) {
      const float prev = has_prev ? n[((size_t)bh * NC + c) * DQK + tid] : 0.f;
      nout[(size_t)bh * DQK + tid] = beta * prev + nacc;
    }
    if (tid == 0) mout[bh] = mT;
  }
}

// One CTA per (64 columns, head): one token of the recurrence from state_in to
// state_out (distinct buffers: every column block reads the old n and m).
// Each thread moves 16-byte pieces of 4 columns in 16 row groups, so many
// loads are in flight per thread.
template <typename TIO, bool EXPV>
__global__ void __launch_bounds__(256) step_kernel(
    const TIO* __restrict__ q, const TIO* __restrict__ k, const TIO* __restrict__ v,
    const TIO* __restrict__ ig, const TIO* __restrict__ fg, TIO* __restrict__ h,
    const float* __restrict__ Cin, const float* __restrict__ nin, const float* __restrict__ min_,
    float* __restrict__ Cout, float* __restrict__ nout, float* __restrict__ mout, int dqk, int dhv,
    float scale) {
  extern __shared__ float sm[];
  float* qs = sm;            // [dqk] q / sqrt(d_qk)
  float* kk = sm + dqk;      // [dqk]
  float* red = kk + dqk;     // [16][64] partial column sums
  float* nred = red + 1024;  // [8] normaliser partials (one per warp)
  const int bh = blockIdx.y, j0 = blockIdx.x * 64, tid = threadIdx.x;
  const int cg = tid & 15, rg = tid >> 4;  // 4 columns 4 cg.., rows rg, rg + 16, ...
  for (int i = tid; i < dqk; i += 256) {
    qs[i] = to_f32(q[(size_t)bh * dqk + i]) * scale;
    kk[i] = to_f32(k[(size_t)bh * dqk + i]);
  }
  const float log_f = log_sigmoid(to_f32(fg[bh]));
  const float ipre = to_f32(ig[bh]);
  const float log_i = EXPV ? ipre : log_sigmoid(ipre);
  float decay, inp, m_new = 0.f;
  if (EXPV) {
    const float m_old = min_[bh];
    m_new = fmaxf(log_f + m_old, log_i);
    decay = expf(log_f + m_old - m_new);  // 0 from the zero state (m_old = -inf)
    inp = expf(log_i - m_new);
  } else {
    decay = expf(log_f);
    inp = expf(log_i);
  }
  __syncthreads();
  // d_hv is a multiple of 64, so the 4 columns are in range together
  const int j = j0 + 4 * cg;
  float vj[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) vj[e] = to_f32(v[(size_t)bh * dhv + j + e]);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  {
    const float4* cin = reinterpret_cast<const float4*>(Cin + (size_t)bh * dqk * dhv + j);
    float4* cout = reinterpret_cast<float4*>(Cout + (size_t)bh * dqk * dhv + j);
    const int stride4 = dhv / 4;
#pragma unroll 4
    for (int i = rg; i < dqk; i += 16) {
      float4 c = cin[(size_t)i * stride4];
      const float ik = inp * kk[i], qi = qs[i];
      c.x = fmaf(decay, c.x, ik * vj[0]);
      c.y = fmaf(decay, c.y, ik * vj[1]);
      c.z = fmaf(decay, c.z, ik * vj[2]);
      c.w = fmaf(decay, c.w, ik * vj[3]);
      cout[(size_t)i * stride4] = c;
      acc[0] = fmaf(c.x, qi, acc[0]);
      acc[1] = fmaf(c.y, qi, acc[1]);
      acc[2] = fmaf(c.z, qi, acc[2]);
      acc[3] = fmaf(c.w, qi, acc[3]);
    }
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) red[rg * 64 + 4 * cg + e] = acc[e];
  float den = 1.f;
  if (EXPV) {
    // n' = decay n + inp k; den = max(|n' . q'|, exp(-m'))
    float part = 0.f;
    for (int i = tid; i < dqk; i += 256) {
      const float ni = fmaf(decay, nin[(size_t)bh * dqk + i], inp * kk[i]);
      if (blockIdx.x == 0) nout[(size_t)bh * dqk + i] = ni;
      part = fmaf(ni, qs[i], part);
    }
    part = warp_sum(part);
    if ((tid & 31) == 0) nred[tid >> 5] = part;
    if (blockIdx.x == 0 && tid == 0) mout[bh] = m_new;
  }
  __syncthreads();
  if (EXPV) {
    float a = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) a += nred[w];
    den = fmaxf(fabsf(a), expf(-m_new));
  }
  if (tid < 64) {
    float num = 0.f;
#pragma unroll
    for (int r = 0; r < 16; ++r) num += red[r * 64 + tid];
    h[(size_t)bh * dhv + j0 + tid] = from_f32<TIO>(num / den);
  }
}

__global__ void fill_neg_inf_kernel(float* __restrict__ m, int count) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < count) m[i] = kNegInf;
}

// Total log forget gate of a segment, per head: G = sum_t log sigmoid(f~_t).  One CTA
// per head; each thread sums a strided share, then a block reduction.
template <typename TIO>
__global__ void __launch_bounds__(256) log_decay_kernel(const TIO* __restrict__ fg,
                                                        float* __restrict__ G, int T) {
  // summed in fp64, like the in-chunk cumsums of gate_prep, and rounded once
  __shared__ double part[8];
  const size_t base = (size_t)blockIdx.x * T;
  double acc = 0.0;
  for (int t = threadIdx.x; t < T; t += blockDim.x) acc += (double)log_sigmoid(to_f32(fg[base + t]));
  acc = warp_sum(acc);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double g = 0.0;
    for (int w = 0; w < 8; ++w) g += part[w];
    G[blockIdx.x] = (float)g;
  }
}

// The state after segment b when b starts from state a instead of the zero state:
// the true state is exp(G_b) (state a) + (state b), G_b the segment's total log
// forget gate.  mLSTMexp keeps the stabilised form: m = max(G_b + m_a, m_b), the
// max-state recurrence unrolled over the segment, and C~ = exp(G_b + m_a - m) C~_a
// + exp(m_b - m) C~_b (n~ likewise).  One CTA per head.
template <bool EXPV>
__global__ void __launch_bounds__(256) state_chain_kernel(
    const float* __restrict__ Ca, const float* __restrict__ na, const float* __restrict__ ma,
    const float* __restrict__ Cb, const float* __restrict__ nb, const float* __restrict__ mb,
    const float* __restrict__ G, float* __restrict__ Co, float* __restrict__ no,
    float* __restrict__ mo, int dqk, int dhv) {
  const int bh = blockIdx.x;
  const float g = G[bh];
  float fa = expf(g), fb = 1.f;
  if (EXPV) {
    const float x = g + ma[bh], y = mb[bh];
    const float m = fmaxf(x, y);
    // both -inf: two zero states, and the result is the zero state
    fa = m == kNegInf ? 0.f : expf(x - m);
    fb = m == kNegInf ? 0.f : expf(y - m);
    if (threadIdx.x == 0) mo[bh] = m;
  }
  const size_t n4 = (size_t)dqk * dhv / 4, off = (size_t)bh * dqk * dhv / 4;
  const float4* a4 = reinterpret_cast<const float4*>(Ca) + off;
  const float4* b4 = reinterpret_cast<const float4*>(Cb) + off;
  float4* o4 = reinterpret_cast<float4*>(Co) + off;
  for (size_t i = threadIdx.x; i < n4; i += blockDim.x) {
    const float4 a = a4[i], b = b4[i];
    o4[i] = make_float4(fmaf(fa, a.x, fb * b.x), fmaf(fa, a.y, fb * b.y), fmaf(fa, a.z, fb * b.z),
                        fmaf(fa, a.w, fb * b.w));
  }
  if (EXPV)
    for (int i = threadIdx.x; i < dqk; i += blockDim.x)
      no[(size_t)bh * dqk + i] = fmaf(fa, na[(size_t)bh * dqk + i], fb * nb[(size_t)bh * dqk + i]);
}

// Gradient with respect to the state entering segment b: its own share (g_local, from the
// segment's outputs) plus the gradient with respect to the state leaving b carried back
// through the segment.  The state map through b is S_out = exp(G_b + m_in - m_out) S_in +
// (b's own state) in the stabilised form, so the carried share is that factor times the
// leaving state's gradient (C and n; the max states are held constant).
template <bool EXPV>
__global__ void __launch_bounds__(256) dstate_chain_kernel(
    const float* __restrict__ Cl, const float* __restrict__ nl, const float* __restrict__ Cd,
    const float* __restrict__ nd, const float* __restrict__ m_in, const float* __restrict__ m_out,
    const float* __restrict__ G, float* __restrict__ Co, float* __restrict__ no, int dqk,
    int dhv) {
  const int bh = blockIdx.x;
  float f;
  if (EXPV) {
    const float x = G[bh] + m_in[bh], y = m_out[bh];
    f = x == kNegInf ? 0.f : expf(x - y);
  } else {
    f = expf(G[bh]);
  }
  const size_t n4 = (size_t)dqk * dhv / 4, off = (size_t)bh * dqk * dhv / 4;
  const float4* l4 = reinterpret_cast<const float4*>(Cl) + off;
  const float4* d4 = reinterpret_cast<const float4*>(Cd) + off;
  float4* o4 = reinterpret_cast<float4*>(Co) + off;
  for (size_t i = threadIdx.x; i < n4; i += blockDim.x) {
    const float4 a = l4[i], b = d4[i];
    o4[i] = make_float4(fmaf(f, b.x, a.x), fmaf(f, b.y, a.y), fmaf(f, b.z, a.z), fmaf(f, b.w, a.w));
  }
  if (EXPV)
    for (int i = threadIdx.x; i < dqk; i += blockDim.x)
      no[(size_t)bh * dqk + i] = fmaf(f, nd[(size_t)bh * dqk + i], nl[(size_t)bh * dqk + i]);
}

// out[bh] = <C_a, C_b> + <n_a, n_b> over one head's state (n for mLSTMexp only).
template <bool EXPV>
__global__ void __launch_bounds__(256) state_dot_kernel(const float* __restrict__ Ca,
                                                        const float* __restrict__ na,
                                                        const float* __restrict__ Cb,
                                                        const float* __restrict__ nb,
                                                        float* __restrict__ out, int dqk, int dhv) {
  __shared__ float part[8];
  const int bh = blockIdx.x;
  const size_t n4 = (size_t)dqk * dhv / 4, off = (size_t)bh * dqk * dhv / 4;
  const float4* a4 = reinterpret_cast<const float4*>(Ca) + off;
  const float4* b4 = reinterpret_cast<const float4*>(Cb) + off;
  float acc = 0.f;
  for (size_t i = threadIdx.x; i < n4; i += blockDim.x) {
    const float4 a = a4[i], b = b4[i];
    acc = fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, fmaf(a.w, b.w, acc))));
  }
  if (EXPV)
    for (int i = threadIdx.x; i < dqk; i += blockDim.x)
      acc = fmaf(na[(size_t)bh * dqk + i], nb[(size_t)bh * dqk + i], acc);
  acc = warp_sum(acc);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < 8; ++w) t += part[w];
    out[bh] = t;
  }
}

}  // namespace

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

cudaError_t launch_final_state(const Problem& p, const void* k, const void* v, const float* b,
                               const float* li, const float* m, const void* C, const float* n,
                               const InitState& init, float* Cout, float* nout, float* mout,
                               cudaStream_t s) {
  const float* m0 = (init.on() && p.exp_variant()) ? init.m : nullptr;
  const size_t plane = (size_t)p.BH * p.NC * p.dqk * p.dhv;
  dim3 grid((unsigned)((p.dhv + 63) / 64), (unsigned)p.BH), block(256);
#define MLSTM_FS(TIO, TS, E, D)                                                                     \
  final_state_kernel<TIO, TS, E, D><<<grid, block, 0, s>>>((const TIO*)k, (const TIO*)v, b, li, m, \
                                                          (const TS*)C, n, plane, Cout, nout, mout, \
                                                          p.T, p.L, p.NC, p.dhv, init.on(), m0)
#define MLSTM_FS_D(TIO, TS, E)                       \
  if (p.dqk == 64) MLSTM_FS(TIO, TS, E, 64);         \
  else if (p.dqk == 128) MLSTM_FS(TIO, TS, E, 128);  \
  else if (p.dqk == 256) MLSTM_FS(TIO, TS, E, 256);  \
  else return cudaErrorInvalidValue;
  if (p.bf16()) {
    if (p.exp_variant()) { MLSTM_FS_D(bf16, bf16, true) } else { MLSTM_FS_D(bf16, bf16, false) }
  } else {
    if (p.exp_variant()) { MLSTM_FS_D(float, float, true) } else { MLSTM_FS_D(float, float, false) }
  }
#undef MLSTM_FS_D
#undef MLSTM_FS
  return cudaGetLastError();
}

cudaError_t launch_step(const Problem& p, const void* q, const void* k, const void* v,
                        const void* ig, const void* fg, void* h, const float* Cin, const float* nin,
                        const float* min_, float* Cout, float* nout, float* mout, cudaStream_t s) {
  dim3 grid((unsigned)((p.dhv + 63) / 64), (unsigned)p.BH), block(256);
  const size_t smem = (2 * (size_t)p.dqk + 1024 + 8) * sizeof(float);
#define MLSTM_ST(TIO, E)                                                                           \
  step_kernel<TIO, E><<<grid, block, smem, s>>>((const TIO*)q, (const TIO*)k, (const TIO*)v,       \
                                               (const TIO*)ig, (const TIO*)fg, (TIO*)h, Cin, nin,  \
                                               min_, Cout, nout, mout, p.dqk, p.dhv, p.scale)
  if (p.bf16()) {
    if (p.exp_variant()) MLSTM_ST(bf16, true); else MLSTM_ST(bf16, false);
  } else {
    if (p.exp_variant()) MLSTM_ST(float, true); else MLSTM_ST(float, false);
  }
#undef MLSTM_ST
  return cudaGetLastError();
}

cudaError_t launch_state_zero(int BH, int dqk, int dhv, bool exp_variant, float* C, float* n, float* m,
                              cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(C, 0, (size_t)BH * dqk * dhv * sizeof(float), s);
  if (e != cudaSuccess || !exp_variant) return e;
  e = cudaMemsetAsync(n, 0, (size_t)BH * dqk * sizeof(float), s);
  if (e != cudaSuccess) return e;
  fill_neg_inf_kernel<<<(BH + 255) / 256, 256, 0, s>>>(m, BH);
  return cudaGetLastError();
}

cudaError_t launch_log_decay(const Problem& p, const void* fg, float* G, cudaStream_t s) {
  if (p.bf16())
    log_decay_kernel<bf16><<<p.BH, 256, 0, s>>>((const bf16*)fg, G, p.T);
  else
    log_decay_kernel<float><<<p.BH, 256, 0, s>>>((const float*)fg, G, p.T);
  return cudaGetLastError();
}

cudaError_t launch_state_chain(int BH, int dqk, int dhv, bool exp_variant, const float* Ca,
                               const float* na, const float* ma, const float* Cb, const float* nb,
                               const float* mb, const float* G, float* Co, float* no, float* mo,
                               cudaStream_t s) {
  if (exp_variant)
    state_chain_kernel<true><<<BH, 256, 0, s>>>(Ca, na, ma, Cb, nb, mb, G, Co, no, mo, dqk, dhv);
  else
    state_chain_kernel<false><<<BH, 256, 0, s>>>(Ca, na, ma, Cb, nb, mb, G, Co, no, mo, dqk, dhv);
  return cudaGetLastError();
}

cudaError_t launch_state_dot(int BH, int dqk, int dhv, bool exp_variant, const float* Ca,
                             const float* na, const float* Cb, const float* nb, float* out,
                             cudaStream_t s) {
  if (exp_variant)
    state_dot_kernel<true><<<BH, 256, 0, s>>>(Ca, na, Cb, nb, out, dqk, dhv);
  else
    state_dot_kernel<false><<<BH, 256, 0, s>>>(Ca, na, Cb, nb, out, dqk, dhv);
  return cudaGetLastError();
}

cudaError_t launch_dstate_chain(int BH, int dqk, int dhv, bool exp_variant, const float* Cl,
                                const float* nl, const float* Cd, const float* nd,
                                const float* m_in, const float* m_out, const float* G, float* Co,
                                float* no, cudaStream_t s) {
  if (exp_variant)
    dstate_chain_kernel<true><<<BH, 256, 0, s>>>(Cl, nl, Cd, nd, m_in, m_out, G, Co, no, dqk, dhv);
  else
    dstate_chain_kernel<false><<<BH, 256, 0, s>>>(Cl, nl, Cd, nd, m_in, m_out, G, Co, no, dqk, dhv);
  return cudaGetLastError();
}

}  // namespace mlstm
