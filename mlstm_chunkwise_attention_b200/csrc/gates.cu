// Gate kernels of the chunkwise mLSTM: forward gate preprocessing (K-a), the
// per-token backward preparation (K-d0) and the gate gradients (K-d3).
//
// "Tiled Flash Linear Attention: More Efficient Linear RNN and xLSTM Kernels"
// (TFLA summary page, Approach): mLSTMexp has an exponential input gate and a
// max state; mLSTMsig a sigmoid input gate and no max state; both a sigmoid
// forget gate.  These kernels are bandwidth-bound warp scans over [B*NH, T].
#include "common.cuh"
#include "internal.h"

namespace mlstm {

// ---------------------------------------------------------------------------
// K-a: per chunk, b_t = inclusive cumsum of log f_t inside the chunk and
// log i_t; for EXP the max state m_t = b_t + max(m_{c-1}, max_{s<=t in c}(log i_s - b_s)),
// where m_c (the max state at the chunk's last row) obeys the max-plus
// recurrence m_c = max(g_c + m_{c-1}, g_c + max_{s in c}(log i_s - b_s)).
// One CTA of 32 warps per (b, h) (mLSTMsig with few heads: several, each
// with a share of the chunks); a chunk goes to one warp, or to several warps
// in contiguous segments when the CTA has fewer chunks than warps, each lane a
// contiguous run of rows.  The chunk recurrence is an inclusive warp scan of the affine
// max-plus maps x -> max(x + g_c, u_c).  The sums run in fp64 and are rounded
// once to fp32: b reaches tens in magnitude over a long chunk, and fp32
// partial sums would carry an error of many fp32 ulps of it into every decay
// exp(b_t - b_s + ...) and into the normaliser, where it is amplified when the
// normaliser nearly cancels.
// ---------------------------------------------------------------------------
// Per-chunk gate tables of the large-chunk output kernel (layout in
// internal.h).  With R_t + CC_s = log2 D_ts / sqrt(d_qk) for s <= t, the decay
// factor separates as exp2(R_t + MU_j) * KP_s over a block j of 32 keys that
// lies wholly before row t; both factors are at most 1, because the max state
// m_t bounds every b_t - b_s + log i_s with s <= t (SIG: log i <= 0, b falls).
// One warp handles one block of 32 keys, so MU_j is a warp max.  The CTA covers
// chunks blockIdx.y, blockIdx.y + gridDim.y, ... of its head.
template <bool EXPV>
__device__ void write_xl_tables(const float* b, const float* li, const float* m, float* xt,
                                size_t base, int T, int L, int NC, float scale,
                                float log2_scale, bool has_init, const float* m0) {
  constexpr float kLog2e = 1.4426950408889634f;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  const int stride = xl_table_stride(L), bpc = L / 32;
  const int G = (int)gridDim.y, cy = (int)blockIdx.y;
  const int nloc = (NC - cy + G - 1) / G;  // this CTA's chunks
  for (int blk = warp; blk < nloc * bpc; blk += nwarps) {
    const int c = cy + G * (blk / bpc), r = (blk % bpc) * 32 + lane;
    const int t = c * L + r;
    const bool valid = t < T;
    float R = -INFINITY, QF = 0.f, FL = 1.f, CC = -INFINITY;
    if (valid) {
      const float bt = b[base + t];
      const float mt = EXPV ? m[base + t] : 0.f;
      R = (bt - mt) * kLog2e + log2_scale;
      if (c > 0 || has_init)
        QF = expf(bt + (EXPV ? chunk_mprev(m, base + (size_t)c * L, c, m0, blockIdx.x) : 0.f) - mt) * scale;
      if (EXPV) FL = expf(-mt);
      CC = (li[base + t] - bt) * kLog2e;
    }
    const float mu = warp_max(CC);
    float* tb = xt + ((size_t)blockIdx.x * NC + c) * (size_t)stride;
    tb[r] = R;
    tb[L + r] = QF;
    tb[2 * L + r] = FL;
    tb[3 * L + r] = CC;
    tb[4 * L + r] = valid ? exp2f(CC - mu) : 0.f;
    if (lane == 0) tb[5 * L + r / 32] = mu;
  }
}

template <typename TIO, bool EXPV>
__global__ void __launch_bounds__(1024) gate_prep_kernel(
    const TIO* __restrict__ ig, const TIO* __restrict__ fg, float* __restrict__ b_out,
    float* __restrict__ li_out, float* __restrict__ m_out, float* __restrict__ xt, int T, int L,
    int NC, float scale, float log2_scale, bool has_init, const float* __restrict__ m0) {
  extern __shared__ float smem[];
  float* sg = smem;       // g_c  (chunk decay)
  float* su = smem + NC;  // u_c, then m_c
  const size_t base = (size_t)blockIdx.x * T;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  const unsigned full = 0xffffffffu;

  // mLSTMsig has no dependency between chunks, so a head's chunks may be spread over
  // gridDim.y CTAs (chunks blockIdx.y, blockIdx.y + gridDim.y, ...); mLSTMexp's max-state
  // scan needs them all in one CTA (gridDim.y == 1).  The CTA's chunks go to groups of
  // wpc warps (more warps per chunk when the CTA has fewer chunks than warps); warp j of a
  // group takes the j-th contiguous segment of its chunk, each lane a contiguous run of it.
  // Segment totals (and, for mLSTMexp, segment maxima of log i - b) pass through shared
  // memory, so every sum is still accumulated in fp64 and rounded once.
  __shared__ double s_sum[32], s_max[32];
  const int nloc = (NC - (int)blockIdx.y + (int)gridDim.y - 1) / (int)gridDim.y;  // this CTA's chunks
  int wpc = 1;
  while (wpc < nwarps && 2 * wpc * nloc <= nwarps) wpc *= 2;
  const int G = nwarps / wpc, grp = warp / wpc, j = warp % wpc;
  const int iters = (nloc + G - 1) / G;
  for (int it = 0; it < iters; ++it) {
    const int lc = grp + G * it;  // the CTA's local chunk index
    const bool active = lc < nloc;
    const int c = (int)blockIdx.y + (int)gridDim.y * (active ? lc : 0);
    const int c0 = c * L;
    const int len = min(L, T - c0);
    const int seglen = (len + wpc - 1) / wpc;
    const int s0 = min(j * seglen, len), s1 = min(s0 + seglen, len);
    const int per = (s1 - s0 + 31) / 32;
    const int r0 = min(s0 + lane * per, s1), r1 = min(r0 + per, s1);
    // pass 1: this lane's sum, the warp's (segment's) total; for mLSTMexp with several
    // segments also the segment's largest log i - b, b counted from the segment's start
    double seg = 0.0;
    if (active)
      for (int r = r0; r < r1; ++r) seg += (double)log_sigmoid(to_f32(fg[base + c0 + r]));
    const double incl = warp_incl_sum(seg);
    const double lane_excl = incl - seg;
    if (wpc > 1) {
      double lmax = -INFINITY;
      if (EXPV && active) {
        double run = lane_excl;
        for (int r = r0; r < r1; ++r) {
          const size_t idx = base + c0 + r;
          run += (double)log_sigmoid(to_f32(fg[idx]));
          lmax = fmax(lmax, (double)to_f32(ig[idx]) - run);
        }
      }
      if (EXPV) lmax = (double)warp_max((float)lmax);
      const double wtot = __shfl_sync(full, incl, 31);
      if (lane == 0) {
        s_sum[warp] = wtot;
        s_max[warp] = lmax;
      }
      __syncthreads();
    }
    // the segment's prefix within its chunk, and the largest log i - b before it
    double prefix = 0.0, prevmax = -INFINITY;
    for (int k = 0; k < j; ++k) {
      prevmax = fmax(prevmax, s_max[grp * wpc + k] - prefix);
      prefix += s_sum[grp * wpc + k];
    }
    // pass 2: b, log i and the running max of log i - b for this lane's run
    double run = prefix + lane_excl;
    double umax = -INFINITY;
    if (active) {
      for (int r = r0; r < r1; ++r) {
        const size_t idx = base + c0 + r;
        run += (double)log_sigmoid(to_f32(fg[idx]));
        const float x = to_f32(ig[idx]);
        const float li = EXPV ? x : log_sigmoid(x);
        b_out[idx] = (float)run;
        li_out[idx] = li;
        if (EXPV) {
          umax = fmax(umax, (double)li - run);
          m_out[idx] = (float)umax;
        }
      }
    }
    if (EXPV) {
      const float pm = warp_incl_max((float)umax);
      float excl = __shfl_up_sync(full, pm, 1);
      if (lane == 0) excl = -INFINITY;
      excl = fmaxf(excl, (float)prevmax);
      if (active)
        for (int r = r0; r < r1; ++r) {
          const size_t idx = base + c0 + r;
          m_out[idx] = fmaxf(m_out[idx], excl);
        }
      // the chunk's totals, from its last segment's warp
      const double g = prefix + __shfl_sync(full, incl, 31);
      const double tot = fmax(prevmax, (double)__shfl_sync(full, pm, 31));
      if (active && j == wpc - 1 && lane == 0) {
        sg[c] = (float)g;
        su[c] = (float)(g + tot);
      }
    }
    if (wpc > 1) __syncthreads();  // the shared partials are rewritten next iteration
  }
  if (!EXPV) {
    if (xt != nullptr) {
      __syncthreads();
      write_xl_tables<false>(b_out, li_out, m_out, xt, base, T, L, NC, scale, log2_scale, has_init, m0);
    }
    return;
  }
  __syncthreads();
  // the max state before the first chunk: the initial state's, -inf without one
  const float m_init = m0 != nullptr ? m0[blockIdx.x] : -INFINITY;
  if (warp == 0) {
    double carry = m_init;
    for (int cb = 0; cb < NC; cb += 32) {
      const int c = cb + lane;
      double g = c < NC ? (double)sg[c] : 0.0;
      double u = c < NC ? (double)su[c] : -INFINITY;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const double g2 = __shfl_up_sync(full, g, o);
        const double u2 = __shfl_up_sync(full, u, o);
        if (lane >= o) {
          u = fmax(u2 + g, u);
          g = g2 + g;
        }
      }
      const double mc = fmax(carry + g, u);
      if (c < NC) su[c] = (float)mc;
      carry = __shfl_sync(full, mc, 31);
    }
  }
  __syncthreads();
  for (int t = threadIdx.x; t < T; t += blockDim.x) {
    const int c = t / L;
    const float mprev = c > 0 ? su[c - 1] : m_init;
    const size_t idx = base + t;
    m_out[idx] = b_out[idx] + fmaxf(mprev, m_out[idx]);
  }
  if (xt != nullptr) {
    __syncthreads();
    write_xl_tables<true>(b_out, li_out, m_out, xt, base, T, L, NC, scale, log2_scale, has_init, m0);
  }
}

cudaError_t launch_gate_prep(const Problem& p, const FwdArgs& a, cudaStream_t s) {
  const size_t smem = p.exp_variant() ? 2 * sizeof(float) * (size_t)p.NC : 0;
  // mLSTMsig with few heads: several CTAs per head (at least a few chunks each), up to two
  // CTAs per SM
  int per_head = 1;
  if (!p.exp_variant()) {
    const int want = (2 * 148 + p.BH - 1) / p.BH, most = (p.NC + 7) / 8;
    per_head = want < most ? want : most;
    if (per_head < 1) per_head = 1;
  }
  dim3 grid(p.BH, per_head), block(1024);
  if (p.bf16()) {
    if (p.exp_variant())
      gate_prep_kernel<bf16, true><<<grid, block, smem, s>>>((const bf16*)a.ig, (const bf16*)a.fg, a.b, a.li, a.m, a.xt, p.T, p.L, p.NC, p.scale, log2f(p.scale), a.init.on(), a.init.on() && p.exp_variant() ? a.init.m : nullptr);
    else
      gate_prep_kernel<bf16, false><<<grid, block, smem, s>>>((const bf16*)a.ig, (const bf16*)a.fg, a.b, a.li, a.m, a.xt, p.T, p.L, p.NC, p.scale, log2f(p.scale), a.init.on(), a.init.on() && p.exp_variant() ? a.init.m : nullptr);
  } else {
    if (p.exp_variant())
      gate_prep_kernel<float, true><<<grid, block, smem, s>>>((const float*)a.ig, (const float*)a.fg, a.b, a.li, a.m, a.xt, p.T, p.L, p.NC, p.scale, log2f(p.scale), a.init.on(), a.init.on() && p.exp_variant() ? a.init.m : nullptr);
    else
      gate_prep_kernel<float, false><<<grid, block, smem, s>>>((const float*)a.ig, (const float*)a.fg, a.b, a.li, a.m, a.xt, p.T, p.L, p.NC, p.scale, log2f(p.scale), a.init.on(), a.init.on() && p.exp_variant() ? a.init.m : nullptr);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// K-d0: per token, 1/den_t and the gradient of the stabilised normaliser,
// da_t = -(dh_t . h_t) sign(a~_t) / den_t when |a~_t| > exp(-m_t), else 0
// (den_t = max(|a~_t|, exp(-m_t)), h_t = num_t / den_t).  Also zeroes the
// per-token dot-product accumulators.  Groups of LPT lanes own one token and
// read its rows with 16-byte loads, at least two of each row per lane so that
// several are in flight; warps stride over the tokens.
// ---------------------------------------------------------------------------
template <typename TIO, bool EXPV>
__global__ void __launch_bounds__(256) bwd_token_prep_kernel(
    const TIO* __restrict__ h, const TIO* __restrict__ dh, const float* __restrict__ abar,
    const float* __restrict__ m, float* __restrict__ inv_den, float* __restrict__ da,
    float* __restrict__ pq, float* __restrict__ pk, long long ntok, int dhv) {
  constexpr int VEC = 16 / sizeof(TIO);  // elements per 16-byte load
  const int lane = threadIdx.x & 31;
  const int lpt = max(1, min(32, dhv / VEC) / 2);  // lanes per token (a power of two)
  const int tpw = 32 / lpt;              // tokens per warp step
  const int sub = lane / lpt, sl = lane % lpt;
  const long long warp_id = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long base = warp_id * tpw; base < ntok; base += nwarps * tpw) {
    const long long tok = base + sub;
    const bool valid = tok < ntok;
    // the token's normaliser and max state load alongside its rows, not after the dot product
    const float a = (EXPV && valid && sl == 0) ? abar[tok] : 0.f;
    const float mtok = (EXPV && valid && sl == 0) ? m[tok] : 0.f;
    float dot = 0.f;
    if (EXPV && valid) {
      const TIO* hr = h + tok * dhv;
      const TIO* dr = dh + tok * dhv;
#pragma unroll 2
      for (int j = sl * VEC; j < dhv; j += lpt * VEC) {
        const uint4 hv = *reinterpret_cast<const uint4*>(hr + j);
        const uint4 dv = *reinterpret_cast<const uint4*>(dr + j);
        const TIO* he = reinterpret_cast<const TIO*>(&hv);
        const TIO* de = reinterpret_cast<const TIO*>(&dv);
#pragma unroll
        for (int e = 0; e < VEC; ++e) dot = fmaf(to_f32(he[e]), to_f32(de[e]), dot);
      }
    }
    for (int o = lpt >> 1; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    if (valid && sl == 0) {
      pq[tok] = 0.f;
      pk[tok] = 0.f;
      if (EXPV) {
        const float floor_ = expf(-mtok);
        const float den = fmaxf(fabsf(a), floor_);
        inv_den[tok] = 1.f / den;
        da[tok] = fabsf(a) > floor_ ? -dot * copysignf(1.f, a) / den : 0.f;
      } else {
        inv_den[tok] = 1.f;
      }
    }
  }
}

cudaError_t launch_bwd_token_prep(const Problem& p, const BwdArgs& a, cudaStream_t s) {
  const long long ntok = (long long)p.BH * p.T;
  const long long want = (ntok + 15) / 16;  // blocks of 8 warps, ~2 tokens per warp
  dim3 block(256), grid((unsigned)(want < 148LL * 16 ? want : 148LL * 16));
  if (p.bf16()) {
    if (p.exp_variant())
      bwd_token_prep_kernel<bf16, true><<<grid, block, 0, s>>>((const bf16*)a.h, (const bf16*)a.dh, a.abar, a.m, a.inv_den, a.da, a.pq, a.pk, ntok, p.dhv);
    else
      bwd_token_prep_kernel<bf16, false><<<grid, block, 0, s>>>((const bf16*)a.h, (const bf16*)a.dh, a.abar, a.m, a.inv_den, a.da, a.pq, a.pk, ntok, p.dhv);
  } else {
    if (p.exp_variant())
      bwd_token_prep_kernel<float, true><<<grid, block, 0, s>>>((const float*)a.h, (const float*)a.dh, a.abar, a.m, a.inv_den, a.da, a.pq, a.pk, ntok, p.dhv);
    else
      bwd_token_prep_kernel<float, false><<<grid, block, 0, s>>>((const float*)a.h, (const float*)a.dh, a.abar, a.m, a.inv_den, a.da, a.pq, a.pk, ntok, p.dhv);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// K-d3: gate gradients from the per-token dot products of the total
// gradients.  With G_ts = dA_ts A_ts, d log i_s = sum_t G_ts = k_s . dk_s, and
// d log f_r = sum_{t>=r} sum_{s<r} G_ts = sum_{t>=r} (q_t . dq_t - k_t . dk_t),
// a reverse cumulative sum over the whole sequence.  Then the chain rule to
// the preactivations: d/dx logsigmoid(x) = sigmoid(-x); the exponential input
// gate has log i = i~.  One CTA (32 warps) per (b, h) and segment of T (one
// segment, or with few heads gridDim.y of them, whose totals gate_grad_sums
// wrote first); each warp owns one contiguous piece of its CTA's segment.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void grad_segment(int T, int& tb, int& te) {
  const int G = (int)gridDim.y, Tc = (T + G - 1) / G;
  tb = min(T, (int)blockIdx.y * Tc);
  te = min(T, tb + Tc);
}

// q.dq - k.dk of one token: each is the sum of its planes in plane order (the
// large-chunk backward stores one share per 32-column block; otherwise one plane)
__device__ __forceinline__ float pdot_diff(const float* pq, const float* pk, size_t idx, int planes,
                                           size_t stride, float& pkt) {
  float q = pq[idx], k = pk[idx];
  for (int i = 1; i < planes; ++i) {
    q += pq[idx + (size_t)i * stride];
    k += pk[idx + (size_t)i * stride];
  }
  pkt = k;
  return q - k;
}

// The total of q.dq - k.dk over each segment of a head, for the segments after it.
__global__ void __launch_bounds__(256) gate_grad_sums_kernel(const float* __restrict__ pq,
                                                             const float* __restrict__ pk,
                                                             float* __restrict__ gsum, int T,
                                                             int planes, size_t stride) {
  __shared__ float s_w[8];
  const size_t base = (size_t)blockIdx.x * T;
  int tb, te;
  grad_segment(T, tb, te);
  float part = 0.f;
  float pkt;
  for (int t = tb + (int)threadIdx.x; t < te; t += blockDim.x)
    part += pdot_diff(pq, pk, base + t, planes, stride, pkt);
  part = warp_sum(part);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) s_w[warp] = part;
  __syncthreads();
  if (threadIdx.x == 0) {
    float tot = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += s_w[w];
    gsum[(size_t)blockIdx.x * gridDim.y + blockIdx.y] = tot;
  }
}

template <typename TIO, bool EXPV>
__global__ void __launch_bounds__(1024) gate_grad_kernel(
    const TIO* __restrict__ ig, const TIO* __restrict__ fg, const float* __restrict__ pq,
    const float* __restrict__ pk, TIO* __restrict__ dig, TIO* __restrict__ dfg, int T,
    const float* __restrict__ fdot, const float* __restrict__ gsum, int planes, size_t stride) {
  __shared__ float s_tot[32];
  const size_t base = (size_t)blockIdx.x * T;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int tb, te;
  grad_segment(T, tb, te);
  const int seg = (te - tb + 31) / 32;
  const int sb = min(tb + warp * seg, te), se = min(sb + seg, te);
  float part = 0.f;
  float pkt;
  for (int t = sb + lane; t < se; t += 32) part += pdot_diff(pq, pk, base + t, planes, stride, pkt);
  part = warp_sum(part);
  if (lane == 0) s_tot[warp] = part;
  __syncthreads();
  if (warp == 0) {
    const float x = s_tot[lane];
    const float incl = warp_incl_suffix_sum(x);
    s_tot[lane] = incl - x;  // sum of the later segments
  }
  __syncthreads();
  // a loss on the final state adds <dC_T, C_T> + <dn_T, n_T> to every d log f_r: the
  // final state is one more row after the last token, and it reads every key; the later
  // segments of the head add their totals (summed from the last one down)
  float later = 0.f;
  for (int y = (int)gridDim.y - 1; y > (int)blockIdx.y; --y)
    later += gsum[(size_t)blockIdx.x * gridDim.y + y];
  float carry = s_tot[warp] + (fdot != nullptr ? fdot[blockIdx.x] : 0.f) + later;
  for (int e = se; e > sb; e -= 32) {
    const int t = e - 32 + lane;
    const bool valid = t >= sb;
    float x = 0.f;
    pkt = 0.f;
    if (valid) x = pdot_diff(pq, pk, base + t, planes, stride, pkt);
    const float sfx = warp_incl_suffix_sum(x);
    const float dlf = carry + sfx;
    carry += __shfl_sync(0xffffffffu, sfx, 0);
    if (valid) {
      const float f = to_f32(fg[base + t]);
      dfg[base + t] = from_f32<TIO>(dlf * dlog_sigmoid(f));
      const float dli = pkt;
      dig[base + t] = from_f32<TIO>(EXPV ? dli : dli * dlog_sigmoid(to_f32(ig[base + t])));
    }
  }
}

int gate_grad_segments(const Problem& p) {
  // few heads: enough CTAs for the 148 SMs, each at least 4096 tokens, at most 64
  int g = 148 / (p.BH > 0 ? p.BH : 1);
  const int most = p.T / 4096;
  if (g > most) g = most;
  if (g > 64) g = 64;
  return g < 1 ? 1 : g;
}

cudaError_t launch_gate_grad_sums(const Problem& p, const BwdArgs& a, cudaStream_t s) {
  const int G = gate_grad_segments(p);
  if (G < 2 || a.gsum == nullptr) return cudaErrorInvalidValue;  // planned only for a split
  gate_grad_sums_kernel<<<dim3(p.BH, G), 256, 0, s>>>(a.pq, a.pk, a.gsum, p.T, a.pdot_planes,
                                                       a.pdot_stride);
  return cudaGetLastError();
}

cudaError_t launch_gate_grad(const Problem& p, const BwdArgs& a, cudaStream_t s) {
  const int G = gate_grad_segments(p);
  if (G > 1 && a.gsum == nullptr) return cudaErrorInvalidValue;
  dim3 grid(p.BH, G), block(1024);
  if (p.bf16()) {
    if (p.exp_variant())
      gate_grad_kernel<bf16, true><<<grid, block, 0, s>>>((const bf16*)a.ig, (const bf16*)a.fg, a.pq, a.pk, (bf16*)a.dig, (bf16*)a.dfg, p.T, a.fdot, a.gsum, a.pdot_planes, a.pdot_stride);
    else
      gate_grad_kernel<bf16, false><<<grid, block, 0, s>>>((const bf16*)a.ig, (const bf16*)a.fg, a.pq, a.pk, (bf16*)a.dig, (bf16*)a.dfg, p.T, a.fdot, a.gsum, a.pdot_planes, a.pdot_stride);
  } else {
    if (p.exp_variant())
      gate_grad_kernel<float, true><<<grid, block, 0, s>>>((const float*)a.ig, (const float*)a.fg, a.pq, a.pk, (float*)a.dig, (float*)a.dfg, p.T, a.fdot, a.gsum, a.pdot_planes, a.pdot_stride);
    else
      gate_grad_kernel<float, false><<<grid, block, 0, s>>>((const float*)a.ig, (const float*)a.fg, a.pq, a.pk, (float*)a.dig, (float*)a.dfg, p.T, a.fdot, a.gsum, a.pdot_planes, a.pdot_stride);
  }
  return cudaGetLastError();
}

}  // namespace mlstm
