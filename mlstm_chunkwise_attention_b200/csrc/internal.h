// Internal interfaces between the C ABI (mlstm_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace mlstm {

struct Problem {
  int B, NH, T, dqk, dhv, L, variant, dtype;
  int BH, NC;
  float scale;  // 1 / sqrt(d_qk)
  bool exp_variant() const { return variant == 1; }
  bool bf16() const { return dtype == 0; }
};

// The state a sequence starts from, in the recurrent-state layout (fp32):
// C [BH, dqk, dhv], n [BH, dqk] and m [BH] (n and m for mLSTMexp only), the
// stabilised form whose true state is exp(m) (C, n).  C == nullptr: the zero
// state (m = -inf), which every kernel then treats as "no state enters the
// first chunk".
struct InitState {
  const float *C = nullptr, *n = nullptr, *m = nullptr;
  __host__ __device__ bool on() const { return C != nullptr; }
};

// m_{c-1} as chunk c sees it (mLSTMexp): the max state at the previous chunk's
// last row, or the initial state's for the first chunk (-inf without one).
__device__ __forceinline__ float chunk_mprev(const float* m, size_t tok_first, int c, const float* m0,
                                             int bh) {
  return c > 0 ? m[tok_first - 1] : (m0 != nullptr ? m0[bh] : -__int_as_float(0x7f800000));
}

// Device pointers of one forward call.
struct FwdArgs {
  const void *q, *k, *v, *ig, *fg;
  void* h;
  float *b, *li, *m, *abar;  // per token [BH, T]
  void* C;                   // [BH, NC, dqk, dhv] state entering each chunk (planes, see StatePlanes)
  float* n;                  // [BH, NC, dqk]
  bool keep_lo;              // write the low plane of bf16 states (needed by the backward)
  float* xt;                 // per-chunk gate tables of the large-chunk output kernel, or null
  InitState init;            // the state entering the first chunk
};

// Per-chunk gate tables, [BH, NC, xl_table_stride(L)] floats, written by
// gate_prep when FwdArgs::xt is set.  For token t (row) or s (key) of chunk c:
//   R  [0, L)    (b_t - m_t) log2 e + log2(1/sqrt(d_qk))    (m_t = 0 for SIG)
//   QF [L, 2L)   exp(b_t + m_{c-1} - m_t) / sqrt(d_qk)       (0 in the first chunk)
//   FL [2L, 3L)  exp(-m_t) (EXP; 1 for SIG)
//   CC [3L, 4L)  (log i_s - b_s) log2 e
//   KP [4L, 5L)  exp2(CC_s - MU_{s/32})
//   MU [5L, ..)  max of CC over each block of 32 keys
// Past the end of the sequence: R = CC = MU = -inf, QF = KP = 0, FL = 1.
// Every block of a chunk starts 16-byte aligned (L is a multiple of 128).
__host__ __device__ inline int xl_table_stride(int L) { return 5 * L + (L / 32 > 32 ? L / 32 : 32); }

// Per-chunk gate table of the large-chunk backward, [BH, NC, bwd_xl_table_stride(L)]
// floats, written by bwd_xl_table.  For token t (query side) or s (key side) of chunk c:
//   QX [0, L)    (b_t - m_t) log2 e + log2(1/den_t)          (m_t = 0, den_t = 1 for SIG)
//   QE [L, 2L)   da_t den_t                                   (0 for SIG)
//   KX [2L, 3L)  (log i_s - b_s) log2 e
//   KG [3L, 4L)  exp2(KX_s - KM_{s/32})
//   RQ [4L, 5L)  alpha_t / den_t, alpha_t = exp(b_t + m_{c-1} - m_t)  (0 with no entering state)
//   RV [5L, 6L)  alpha_t da_t
//   RK [6L, 7L)  exp(b_last - b_s + log i_s - m_last)  (last: the chunk's last token)
//   KM [7L, ..)  max of KX over each block of 32 keys (0 for a block wholly past the end)
// Past the end of the sequence: QX = KX = -inf, QE = KG = RQ = RV = RK = 0.
__host__ __device__ inline int bwd_xl_table_stride(int L) { return 7 * L + (L / 32 > 32 ? L / 32 : 32); }

// Device pointers of one backward call.
struct BwdArgs {
  const void *q, *k, *v, *ig, *fg, *h, *dh;
  const float *b, *li, *m, *abar;
  const void* C;
  const float* n;
  void *dq, *dk, *dv, *dig, *dfg;
  float* inv_den;  // [BH, T] 1 / den_t
  float* da;       // [BH, T] gradient of the stabilised normaliser (EXP)
  float* pq;       // [pdot_planes, BH, T] q_t . dq_t, the sum of the planes in plane order
  float* pk;       // [pdot_planes, BH, T] k_t . dk_t, likewise
  int pdot_planes;    // 4 on the large-chunk backward (one share per 32 columns), else 1
  size_t pdot_stride; // elements per plane (BH T)
  void* dC;        // [BH, NC, dqk, dhv] gradient of the state leaving each chunk (planes, see StatePlanes)
  float* dn;       // [BH, NC, dqk]
  InitState init;  // the state the forward started from (held constant)
  float* dC0;      // gradient of the initial state: C [BH, dqk, dhv] (null: not wanted)
  float* dn0;      // and n [BH, dqk] (mLSTMexp)
  const float* dCT;  // gradient with respect to the final state: C [BH, dqk, dhv] (null: none)
  const float* dnT;  // and n [BH, dqk] (mLSTMexp)
  float* fdot;       // [BH] <dC_T, C_T> + <dn_T, n_T>, added to every forget-gate gradient
  float* btab;       // per-chunk gate table of the large-chunk backward (null: not used)
  float* gsum;       // [BH, gate_grad_segments] totals of q.dq - k.dk per segment (null: one segment)
};

// gate kernels (gates.cu)
cudaError_t launch_gate_prep(const Problem& p, const FwdArgs& a, cudaStream_t s);
cudaError_t launch_bwd_token_prep(const Problem& p, const BwdArgs& a, cudaStream_t s);
cudaError_t launch_gate_grad(const Problem& p, const BwdArgs& a, cudaStream_t s);
// few heads: gate_grad runs over segments of T whose totals gate_grad_sums writes first
int gate_grad_segments(const Problem& p);
cudaError_t launch_gate_grad_sums(const Problem& p, const BwdArgs& a, cudaStream_t s);

// CUDA-core (fp32 FMA) kernels (simt_fwd.cu, simt_bwd.cu)
cudaError_t launch_state_fwd_simt(const Problem& p, const FwdArgs& a, cudaStream_t s);
cudaError_t launch_output_fwd_simt(const Problem& p, const FwdArgs& a, cudaStream_t s);
cudaError_t launch_state_bwd_simt(const Problem& p, const BwdArgs& a, cudaStream_t s);
cudaError_t launch_dq_simt(const Problem& p, const BwdArgs& a, cudaStream_t s);
cudaError_t launch_dk_simt(const Problem& p, const BwdArgs& a, cudaStream_t s);
cudaError_t launch_dv_simt(const Problem& p, const BwdArgs& a, cudaStream_t s);

// Abort epoch for the next launch of a tensor-core kernel: a process-wide launch
// counter, never 0 (see tc::Abort).  Each kernel family keeps a device flag that
// holds the epoch of its last launch that gave up; fetch_tc_*_error read it
// without clearing it.
unsigned int next_epoch();

// tensor-core kernels (tc_*.cu) and their host helpers (tmap.cu)
bool make_tmap_3d_bf16(void* map, const void* base, uint64_t inner, uint64_t mid, uint64_t outer,
                       uint32_t box_inner, uint32_t box_mid);
bool make_tmap_3d_bf16_rows(void* map, const void* base, uint64_t inner, uint64_t mid,
                            uint64_t outer, uint32_t box_inner, uint32_t box_mid);
bool output_fwd_tc_supported(const Problem& p);
cudaError_t launch_output_fwd_tc(const Problem& p, const FwdArgs& a, cudaStream_t s);
cudaError_t fetch_tc_fwd_error(unsigned int* flag);
cudaError_t launch_selftest_timeout(cudaStream_t s);
bool output_fwd_xl_supported(const Problem& p);
cudaError_t launch_output_fwd_xl(const Problem& p, const FwdArgs& a, cudaStream_t s);
cudaError_t fetch_tc_fwd_xl_error(unsigned int* flag);
bool intra_bwd_tc_supported(const Problem& p);
cudaError_t launch_dq_tc(const Problem& p, const BwdArgs& a, cudaStream_t s);
cudaError_t launch_dk_tc(const Problem& p, const BwdArgs& a, cudaStream_t s);
cudaError_t launch_dv_tc(const Problem& p, const BwdArgs& a, cudaStream_t s);
// large chunks, d_qk = d_hv = 128, bf16 (tc_bwd_xl.cu): the gate table, then dq, dk, dv
bool intra_bwd_xl_supported(const Problem& p);
cudaError_t launch_bwd_xl_table(const Problem& p, const BwdArgs& a, cudaStream_t s);
cudaError_t launch_dq_xl(const Problem& p, const BwdArgs& a, cudaStream_t s);
cudaError_t launch_dk_xl(const Problem& p, const BwdArgs& a, cudaStream_t s);
cudaError_t launch_dv_xl(const Problem& p, const BwdArgs& a, cudaStream_t s);
cudaError_t fetch_tc_bwd_error(unsigned int* flag);
cudaError_t fetch_tc_bwd_xl_error(unsigned int* flag);
bool state_tc_supported(const Problem& p);
cudaError_t launch_state_fwd_tc(const Problem& p, const FwdArgs& a, cudaStream_t s);
cudaError_t launch_state_bwd_tc(const Problem& p, const BwdArgs& a, cudaStream_t s);
// few heads and many chunks: the state walks run in segments, completed by state_*_fix
bool state_split_needed(const Problem& p);
cudaError_t launch_state_fwd_fix(const Problem& p, const FwdArgs& a, cudaStream_t s);
cudaError_t launch_state_bwd_fix(const Problem& p, const BwdArgs& a, cudaStream_t s);
cudaError_t fetch_tc_state_error(unsigned int* flag);
bool bwd_walk_supported(const Problem& p);
cudaError_t launch_bwd_walk(const Problem& p, const BwdArgs& a, cudaStream_t s);
cudaError_t fetch_tc_walk_error(unsigned int* flag);
bool fwd_walk_supported(const Problem& p);
cudaError_t launch_fwd_walk(const Problem& p, const FwdArgs& a, cudaStream_t s);
cudaError_t fetch_tc_fwalk_error(unsigned int* flag);

// recurrent-form kernels (recurrent.cu)
cudaError_t launch_final_state(const Problem& p, const void* k, const void* v, const float* b,
                               const float* li, const float* m, const void* C, const float* n,
                               const InitState& init, float* Cout, float* nout, float* mout,
                               cudaStream_t s);
cudaError_t launch_step(const Problem& p, const void* q, const void* k, const void* v,
                        const void* ig, const void* fg, void* h, const float* Cin, const float* nin,
                        const float* min_, float* Cout, float* nout, float* mout, cudaStream_t s);
cudaError_t launch_state_zero(int BH, int dqk, int dhv, bool exp_variant, float* C, float* n, float* m,
                              cudaStream_t s);
cudaError_t launch_log_decay(const Problem& p, const void* fg, float* G, cudaStream_t s);
cudaError_t launch_dstate_chain(int BH, int dqk, int dhv, bool exp_variant, const float* Cl,
                                const float* nl, const float* Cd, const float* nd,
                                const float* m_in, const float* m_out, const float* G, float* Co,
                                float* no, cudaStream_t s);
cudaError_t launch_state_dot(int BH, int dqk, int dhv, bool exp_variant, const float* Ca,
                             const float* na, const float* Cb, const float* nb, float* out,
                             cudaStream_t s);
cudaError_t launch_state_chain(int BH, int dqk, int dhv, bool exp_variant, const float* Ca,
                               const float* na, const float* ma, const float* Cb, const float* nb,
                               const float* mb, const float* G, float* Co, float* no, float* mo,
                               cudaStream_t s);

}  // namespace mlstm
