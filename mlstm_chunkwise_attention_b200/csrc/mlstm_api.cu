// C ABI of the chunkwise mLSTM library: argument checks, buffer layouts and
// the launch sequence of the forward and backward passes.  Declared in
// include/mlstm.h, which states the operation, layouts, ownership and errors.
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "internal.h"
#include "mlstm.h"

namespace {

using mlstm::Problem;

constexpr int kMaxChunks = 6144;  // gate_prep keeps 2 floats per chunk in shared memory

thread_local char g_last_error[256] = "";

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

int check_sizes(int B, int NH, int T, int d_qk, int d_hv, int chunk, int variant, int dtype) {
  if (B < 0 || NH < 0 || T < 0 || d_qk <= 0 || d_hv <= 0 || chunk <= 0) return MLSTM_ERR_INVALID;
  if (variant != MLSTM_SIG && variant != MLSTM_EXP) return MLSTM_ERR_INVALID;
  if (dtype != MLSTM_BF16 && dtype != MLSTM_FP32) return MLSTM_ERR_INVALID;
  if (!(d_qk == 64 || d_qk == 128 || d_qk == 256)) return MLSTM_ERR_UNSUPPORTED;
  if (!(d_hv == 64 || d_hv == 128 || d_hv == 256 || d_hv == 512)) return MLSTM_ERR_UNSUPPORTED;
  if (!is_pow2(chunk) || chunk < 64 || chunk > 4096) return MLSTM_ERR_UNSUPPORTED;
  const long long tokens = (long long)B * NH * T;
  if (tokens >= (1LL << 31)) return MLSTM_ERR_UNSUPPORTED;
  if ((T + chunk - 1) / chunk > kMaxChunks) return MLSTM_ERR_UNSUPPORTED;
  return MLSTM_OK;
}

Problem make_problem(int B, int NH, int T, int d_qk, int d_hv, int chunk, int variant, int dtype) {
  Problem p;
  p.B = B; p.NH = NH; p.T = T; p.dqk = d_qk; p.dhv = d_hv; p.L = chunk;
  p.variant = variant; p.dtype = dtype;
  p.BH = B * NH;
  p.NC = (T + chunk - 1) / chunk;
  p.scale = 1.0f / sqrtf((float)d_qk);
  return p;
}

void saved_layout(const Problem& p, mlstm_saved_layout_t* L) {
  memset(L, 0, sizeof(*L));
  const size_t tok = (size_t)p.BH * p.T;
  const size_t state_elem = p.bf16() ? 2 : 4;
  L->gate_b_bytes = tok * 4;
  L->gate_li_bytes = tok * 4;
  L->gate_m_bytes = p.exp_variant() ? tok * 4 : 0;
  L->norm_bytes = p.exp_variant() ? tok * 4 : 0;
  // bf16 path: hi and lo bf16 planes; fp32 path: one fp32 plane
  L->state_c_bytes = (size_t)p.BH * p.NC * p.dqk * p.dhv * (p.bf16() ? 2 * state_elem : state_elem);
  L->state_n_bytes = p.exp_variant() ? (size_t)p.BH * p.NC * p.dqk * 4 : 0;
  L->tile_table_bytes = mlstm::output_fwd_xl_supported(p)
                            ? (size_t)p.BH * p.NC * mlstm::xl_table_stride(p.L) * 4
                            : 0;
  size_t off = 0;
  L->gate_b = off;  off = align256(off + L->gate_b_bytes);
  L->gate_li = off; off = align256(off + L->gate_li_bytes);
  L->gate_m = off;  off = align256(off + L->gate_m_bytes);
  L->norm = off;    off = align256(off + L->norm_bytes);
  L->state_c = off; off = align256(off + L->state_c_bytes);
  L->state_n = off; off = align256(off + L->state_n_bytes);
  L->tile_table = off; off = align256(off + L->tile_table_bytes);
  L->total = off;
}

struct StateLayout {
  size_t C, n, m, total;
};

// Recurrent state of one call: C [BH, d_qk, d_hv], then (EXP) n [BH, d_qk] and m [BH],
// fp32, 256-byte aligned regions.
StateLayout state_layout(int BH, int dqk, int dhv, bool exp_variant) {
  StateLayout L;
  L.C = 0;
  size_t off = align256((size_t)BH * dqk * dhv * 4);
  L.n = off;
  if (exp_variant) off = align256(off + (size_t)BH * dqk * 4);
  L.m = off;
  if (exp_variant) off = align256(off + (size_t)BH * 4);
  L.total = off;
  return L;
}

bool overlaps(const void* a, const void* b, size_t bytes) {
  const uintptr_t x = (uintptr_t)a, y = (uintptr_t)b;
  return x < y + bytes && y < x + bytes;
}

// The initial state held in a recurrent-state buffer (null: the zero state).
mlstm::InitState init_from(const void* state, const Problem& p) {
  mlstm::InitState in;
  if (!state) return in;
  const StateLayout S = state_layout(p.BH, p.dqk, p.dhv, p.exp_variant());
  const char* base = (const char*)state;
  in.C = (const float*)(base + S.C);
  if (p.exp_variant()) {
    in.n = (const float*)(base + S.n);
    in.m = (const float*)(base + S.m);
  }
  return in;
}

struct BwdLayout {
  size_t inv_den, da, pq, pk, dC, dn, fstate, fdot, btab, btab_bytes, gsum, gsum_bytes, total;
};

BwdLayout bwd_layout(const Problem& p) {
  BwdLayout L;
  const size_t tok = (size_t)p.BH * p.T;
  size_t off = 0;
  L.inv_den = off; off = align256(off + tok * 4);
  L.da = off;      off = align256(off + tok * 4);
  // q.dq and k.dk: the large-chunk backward writes four column-block shares per token
  const size_t planes = mlstm::intra_bwd_xl_supported(p) ? 4 : 1;
  L.pq = off;      off = align256(off + planes * tok * 4);
  L.pk = off;      off = align256(off + planes * tok * 4);
  L.dC = off;      off = align256(off + (size_t)p.BH * p.NC * p.dqk * p.dhv * 4);
  L.dn = off;      off = align256(off + (p.exp_variant() ? (size_t)p.BH * p.NC * p.dqk * 4 : 0));
  // the final state, rebuilt when the loss has a term on it, and its dot product with that term
  L.fstate = off;  off = align256(off + state_layout(p.BH, p.dqk, p.dhv, p.exp_variant()).total);
  L.fdot = off;    off = align256(off + (size_t)p.BH * 4);
  // the large-chunk backward's per-chunk gate table
  L.btab_bytes = mlstm::intra_bwd_xl_supported(p)
                     ? (size_t)p.BH * p.NC * mlstm::bwd_xl_table_stride(p.L) * 4
                     : 0;
  L.btab = off;    off = align256(off + L.btab_bytes);
  // the gate gradients' segment totals, with few heads
  const int gseg = mlstm::gate_grad_segments(p);
  L.gsum_bytes = gseg > 1 ? (size_t)p.BH * gseg * 4 : 0;
  L.gsum = off;    off = align256(off + L.gsum_bytes);
  L.total = off;
  return L;
}

bool misaligned(const void* ptr) { return ((uintptr_t)ptr & 15) != 0; }


int cuda_status(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return MLSTM_OK;
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s", where, cudaGetErrorString(e));
  return MLSTM_ERR_CUDA;
}

// Optional per-kernel timing events (mlstm_set_timing_events).
thread_local void* const* g_events = nullptr;
thread_local int g_nevents = 0;

typedef cudaError_t (*FwdLauncher)(const Problem&, const mlstm::FwdArgs&, cudaStream_t);
typedef cudaError_t (*BwdLauncher)(const Problem&, const mlstm::BwdArgs&, cudaStream_t);
// side: the step runs on the calling thread's high-priority side stream, forked from the
// caller's stream after the steps before it, while the following steps continue on the
// caller's stream; join: the caller's stream waits for the side work before this step.
struct FwdStep { const char* name; FwdLauncher fn; bool side = false, join = false; };
struct BwdStep { const char* name; BwdLauncher fn; bool side = false, join = false; };
constexpr int kMaxSteps = 10;

// The side stream and fork / join events of the calling thread on the current device,
// created on its first use there (a call that forks must not be the first one made during
// a stream capture) and kept until the process exits.  Per thread: one thread enqueues its
// calls in order, so reusing the events is safe; a capture of the caller's stream takes
// the side stream in through the fork event.
struct SideStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
constexpr int kMaxSideDevices = 64;
thread_local SideStream g_side[kMaxSideDevices];
thread_local bool g_serial = false;  // mlstm_set_serial_launches: every step on the caller's stream

cudaError_t side_stream(SideStream** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxSideDevices) return cudaErrorInvalidDevice;
  SideStream& r = g_side[dev];
  if (r.stream == nullptr) {
    int least = 0, greatest = 0;
    if ((e = cudaDeviceGetStreamPriorityRange(&least, &greatest)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&r.fork, cudaEventDisableTiming)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&r.join, cudaEventDisableTiming)) != cudaSuccess) return e;
    if ((e = cudaStreamCreateWithPriority(&r.stream, cudaStreamNonBlocking, greatest)) != cudaSuccess)
      return e;
  }
  *out = &r;
  return cudaSuccess;
}

// The kernels each pass enqueues, in order.
// want_h false: the state-only pass (the plan without its last step, the output kernel).
int fwd_plan(const Problem& p, FwdStep* st, bool want_h = true) {
  int n = 0;
  st[n++] = {"gate_prep", mlstm::launch_gate_prep};
  if (want_h && mlstm::fwd_walk_supported(p)) {
    // one pass per head over its chunks gives the states and the outputs
    st[n++] = {"fwd_walk_tc", mlstm::launch_fwd_walk};
    return n;
  }
  if (mlstm::state_tc_supported(p)) {
    st[n++] = {"state_fwd_tc", mlstm::launch_state_fwd_tc};
    if (mlstm::state_split_needed(p)) st[n++] = {"state_fwd_fix", mlstm::launch_state_fwd_fix};
  } else
    st[n++] = {"state_fwd_simt", mlstm::launch_state_fwd_simt};
  if (mlstm::output_fwd_xl_supported(p))
    st[n++] = {"output_fwd_xl", mlstm::launch_output_fwd_xl};
  else if (mlstm::output_fwd_tc_supported(p))
    st[n++] = {"output_fwd_tc", mlstm::launch_output_fwd_tc};
  else
    st[n++] = {"output_fwd_simt", mlstm::launch_output_fwd_simt};
  return n;
}

// grads false: the state-gradient-only pass (token prep and the state recurrence).
int bwd_plan(const Problem& p, BwdStep* st, bool grads = true) {
  int n = 0;
  st[n++] = {"bwd_token_prep", mlstm::launch_bwd_token_prep};
  if (grads && mlstm::bwd_walk_supported(p)) {
    // one pass per head over its chunks in reverse gives the state gradients, dk and dv; it
    // runs on the high-priority side stream with dq alongside, whose CTAs take the SMs the
    // walker's last wave (one CTA per SM and head) leaves idle
    st[n++] = {"dkv_walk_tc", mlstm::launch_bwd_walk, true, false};
    st[n++] = {"dq_tc", mlstm::launch_dq_tc};
    if (mlstm::gate_grad_segments(p) > 1) {
      st[n++] = {"gate_grad_sums", mlstm::launch_gate_grad_sums, false, true};
      st[n++] = {"gate_grad", mlstm::launch_gate_grad};
    } else {
      st[n++] = {"gate_grad", mlstm::launch_gate_grad, false, true};
    }
    return n;
  }
  if (mlstm::state_tc_supported(p)) {
    st[n++] = {"state_bwd_tc", mlstm::launch_state_bwd_tc};
    if (mlstm::state_split_needed(p)) st[n++] = {"state_bwd_fix", mlstm::launch_state_bwd_fix};
  } else
    st[n++] = {"state_bwd_simt", mlstm::launch_state_bwd_simt};
  if (!grads) return n;
  if (mlstm::intra_bwd_xl_supported(p)) {
    st[n++] = {"bwd_xl_table", mlstm::launch_bwd_xl_table};
    st[n++] = {"dq_xl", mlstm::launch_dq_xl};
    st[n++] = {"dk_xl", mlstm::launch_dk_xl};
    st[n++] = {"dv_xl", mlstm::launch_dv_xl};
  } else if (mlstm::intra_bwd_tc_supported(p)) {
    st[n++] = {"dq_tc", mlstm::launch_dq_tc};
    st[n++] = {"dk_tc", mlstm::launch_dk_tc};
    st[n++] = {"dv_tc", mlstm::launch_dv_tc};
  } else {
    st[n++] = {"dq_simt", mlstm::launch_dq_simt};
    st[n++] = {"dk_simt", mlstm::launch_dk_simt};
    st[n++] = {"dv_simt", mlstm::launch_dv_simt};
  }
  if (mlstm::gate_grad_segments(p) > 1) st[n++] = {"gate_grad_sums", mlstm::launch_gate_grad_sums};
  st[n++] = {"gate_grad", mlstm::launch_gate_grad};
  return n;
}

template <typename Step, typename Args>
int run_plan(const Step* steps, int n, const Problem& p, const Args& a, cudaStream_t s) {
  SideStream* side = nullptr;
  bool forked = false;
  for (int i = 0; i < n; ++i) {
    cudaStream_t si = s;
    if (steps[i].join && forked) {
      int st = cuda_status(cudaEventRecord(side->join, side->stream), "side join");
      if (st == MLSTM_OK) st = cuda_status(cudaStreamWaitEvent(s, side->join, 0), "side join");
      if (st != MLSTM_OK) return st;
      forked = false;
    }
    if (steps[i].side && !g_serial) {
      int st = cuda_status(side_stream(&side), "side stream");
      if (st == MLSTM_OK) st = cuda_status(cudaEventRecord(side->fork, s), "side fork");
      if (st == MLSTM_OK) st = cuda_status(cudaStreamWaitEvent(side->stream, side->fork, 0), "side fork");
      if (st != MLSTM_OK) return st;
      si = side->stream;
      forked = true;
    }
    if (g_events && 2 * i + 1 < g_nevents) {
      int st = cuda_status(cudaEventRecord((cudaEvent_t)g_events[2 * i], si), "event record");
      if (st != MLSTM_OK) return st;
    }
    int st = cuda_status(steps[i].fn(p, a, si), steps[i].name);
    if (st != MLSTM_OK) return st;
    if (g_events && 2 * i + 1 < g_nevents) {
      st = cuda_status(cudaEventRecord((cudaEvent_t)g_events[2 * i + 1], si), "event record");
      if (st != MLSTM_OK) return st;
    }
  }
  if (forked) {  // a plan whose side work no later step joined: join at its end
    int st = cuda_status(cudaEventRecord(side->join, side->stream), "side join");
    if (st == MLSTM_OK) st = cuda_status(cudaStreamWaitEvent(s, side->join, 0), "side join");
    if (st != MLSTM_OK) return st;
  }
  return MLSTM_OK;
}

}  // namespace

namespace mlstm {

unsigned int next_epoch() {
  static std::atomic<unsigned int> counter{0};
  unsigned int e = counter.fetch_add(1, std::memory_order_relaxed) + 1;
  while (e == 0u) e = counter.fetch_add(1, std::memory_order_relaxed) + 1;  // 0 means "no failure"
  return e;
}

}  // namespace mlstm

extern "C" {

int mlstm_saved_layout(int B, int NH, int T, int d_qk, int d_hv, int chunk, int variant,
                       int dtype, mlstm_saved_layout_t* layout) {
  if (!layout) return MLSTM_ERR_INVALID;
  const int st = check_sizes(B, NH, T, d_qk, d_hv, chunk, variant, dtype);
  if (st != MLSTM_OK) return st;
  saved_layout(make_problem(B, NH, T, d_qk, d_hv, chunk, variant, dtype), layout);
  return MLSTM_OK;
}

size_t mlstm_saved_size(int B, int NH, int T, int d_qk, int d_hv, int chunk, int variant,
                        int dtype) {
  mlstm_saved_layout_t L;
  if (mlstm_saved_layout(B, NH, T, d_qk, d_hv, chunk, variant, dtype, &L) != MLSTM_OK) return 0;
  return L.total;
}

size_t mlstm_fwd_workspace_size(int B, int NH, int T, int d_qk, int d_hv, int chunk, int variant,
                                int dtype) {
  return mlstm_saved_size(B, NH, T, d_qk, d_hv, chunk, variant, dtype);
}

size_t mlstm_bwd_workspace_size(int B, int NH, int T, int d_qk, int d_hv, int chunk, int variant,
                                int dtype) {
  if (check_sizes(B, NH, T, d_qk, d_hv, chunk, variant, dtype) != MLSTM_OK) return 0;
  return bwd_layout(make_problem(B, NH, T, d_qk, d_hv, chunk, variant, dtype)).total;
}

int mlstm_fwd_launch_count(int B, int NH, int T, int d_qk, int d_hv, int chunk, int variant,
                           int dtype) {
  if (check_sizes(B, NH, T, d_qk, d_hv, chunk, variant, dtype) != MLSTM_OK) return 0;
  if ((long long)B * NH * T == 0) return 0;
  FwdStep steps[kMaxSteps];
  return fwd_plan(make_problem(B, NH, T, d_qk, d_hv, chunk, variant, dtype), steps);
}

int mlstm_bwd_launch_count(int B, int NH, int T, int d_qk, int d_hv, int chunk, int variant,
                           int dtype) {
  if (check_sizes(B, NH, T, d_qk, d_hv, chunk, variant, dtype) != MLSTM_OK) return 0;
  if ((long long)B * NH * T == 0) return 0;
  BwdStep steps[kMaxSteps];
  return bwd_plan(make_problem(B, NH, T, d_qk, d_hv, chunk, variant, dtype), steps);
}

const char* mlstm_launch_name(int pass, int index, int B, int NH, int T, int d_qk, int d_hv,
                              int chunk, int variant, int dtype) {
  if (check_sizes(B, NH, T, d_qk, d_hv, chunk, variant, dtype) != MLSTM_OK || index < 0) return "";
  const Problem p = make_problem(B, NH, T, d_qk, d_hv, chunk, variant, dtype);
  if (pass == 0) {
    FwdStep steps[kMaxSteps];
    const int n = fwd_plan(p, steps);
    return index < n ? steps[index].name : "";
  }
  if (pass == 1) {
    BwdStep steps[kMaxSteps];
    const int n = bwd_plan(p, steps);
    return index < n ? steps[index].name : "";
  }
  return "";
}

int mlstm_set_serial_launches(int serial) {
  g_serial = serial != 0;
  return MLSTM_OK;
}

int mlstm_set_timing_events(void* const* events, int count) {
  if (count < 0 || (count > 0 && !events)) return MLSTM_ERR_INVALID;
  g_events = count > 0 ? events : nullptr;
  g_nevents = count;
  return MLSTM_OK;
}

}  // extern "C"

namespace {

int fwd_impl(const void* q, const void* k, const void* v, const void* igate_pre,
             const void* fgate_pre, void* h, void* saved, void* workspace, size_t workspace_bytes,
             const void* state_in, void* state_out, int B, int NH, int T, int d_qk, int d_hv,
             int chunk, int variant, int dtype, void* stream) {
  int st = check_sizes(B, NH, T, d_qk, d_hv, chunk, variant, dtype);
  if (st != MLSTM_OK) return st;
  if (misaligned(state_in) || misaligned(state_out)) return MLSTM_ERR_INVALID;
  if ((long long)B * NH == 0) return MLSTM_OK;
  const StateLayout SL = state_layout(B * NH, d_qk, d_hv, variant == MLSTM_EXP);
  if (state_in && state_out && overlaps(state_in, state_out, SL.total)) return MLSTM_ERR_INVALID;
  if (T == 0) {  // the final state is the initial one
    if (!state_out) return MLSTM_OK;
    if (!state_in) return mlstm_state_zero(state_out, B, NH, d_qk, d_hv, variant, stream);
    return cuda_status(cudaMemcpyAsync(state_out, state_in, SL.total, cudaMemcpyDeviceToDevice,
                                       (cudaStream_t)stream),
                       "state copy");
  }
  // h == NULL with a state_out: the state-only pass (no output kernel)
  if (!q || !k || !v || !igate_pre || !fgate_pre || (!h && !state_out)) return MLSTM_ERR_INVALID;
  if (misaligned(q) || misaligned(k) || misaligned(v) || misaligned(h) ||
      misaligned(igate_pre) || misaligned(fgate_pre) || misaligned(saved) ||
      misaligned(workspace))
    return MLSTM_ERR_INVALID;
  const Problem p = make_problem(B, NH, T, d_qk, d_hv, chunk, variant, dtype);
  mlstm_saved_layout_t L;
  saved_layout(p, &L);
  char* base = (char*)saved;
  if (!base) {
    if (!workspace || workspace_bytes < L.total) return MLSTM_ERR_WORKSPACE;
    base = (char*)workspace;
  }
  mlstm::FwdArgs a;
  a.q = q; a.k = k; a.v = v; a.ig = igate_pre; a.fg = fgate_pre; a.h = h;
  a.b = (float*)(base + L.gate_b);
  a.li = (float*)(base + L.gate_li);
  a.m = p.exp_variant() ? (float*)(base + L.gate_m) : nullptr;
  a.abar = p.exp_variant() ? (float*)(base + L.norm) : nullptr;
  a.C = base + L.state_c;
  a.n = p.exp_variant() ? (float*)(base + L.state_n) : nullptr;
  a.keep_lo = saved != nullptr || state_out != nullptr;  // the final state reads both planes
  a.xt = L.tile_table_bytes ? (float*)(base + L.tile_table) : nullptr;
  a.init = init_from(state_in, p);
  cudaStream_t s = (cudaStream_t)stream;

  st = cuda_status(cudaPeekAtLastError(), "before mlstm_fwd");
  if (st != MLSTM_OK) return st;
  FwdStep steps[kMaxSteps];
  const int n = fwd_plan(p, steps, h != nullptr);
  st = run_plan(steps, h ? n : n - 1, p, a, s);  // the output kernel is the plan's last step
  if (st != MLSTM_OK || !state_out) return st;
  char* out = (char*)state_out;
  return cuda_status(mlstm::launch_final_state(p, k, v, a.b, a.li, a.m, a.C, a.n, a.init,
                                               (float*)(out + SL.C), (float*)(out + SL.n),
                                               (float*)(out + SL.m), s),
                     "final_state");
}

}  // namespace

extern "C" {

int mlstm_fwd(const void* q, const void* k, const void* v, const void* igate_pre,
              const void* fgate_pre, void* h, void* saved, void* workspace,
              size_t workspace_bytes, int B, int NH, int T, int d_qk, int d_hv, int chunk,
              int variant, int dtype, void* stream) {
  return fwd_impl(q, k, v, igate_pre, fgate_pre, h, saved, workspace, workspace_bytes, nullptr,
                  nullptr, B, NH, T, d_qk, d_hv, chunk, variant, dtype, stream);
}

int mlstm_fwd_state(const void* q, const void* k, const void* v, const void* igate_pre,
                    const void* fgate_pre, void* h, void* saved, void* workspace,
                    size_t workspace_bytes, const void* state_in, void* state_out, int B, int NH,
                    int T, int d_qk, int d_hv, int chunk, int variant, int dtype, void* stream) {
  return fwd_impl(q, k, v, igate_pre, fgate_pre, h, saved, workspace, workspace_bytes, state_in,
                  state_out, B, NH, T, d_qk, d_hv, chunk, variant, dtype, stream);
}

}  // extern "C"

namespace {

int bwd_impl(const void* q, const void* k, const void* v, const void* igate_pre,
             const void* fgate_pre, const void* h, const void* dh, const void* saved,
             const void* state_in, void* dstate_in, const void* dstate_out, void* dq, void* dk,
             void* dv, void* digate_pre, void* dfgate_pre, void* workspace,
             size_t workspace_bytes, int B, int NH, int T, int d_qk, int d_hv, int chunk,
             int variant, int dtype, void* stream) {
  int st = check_sizes(B, NH, T, d_qk, d_hv, chunk, variant, dtype);
  if (st != MLSTM_OK) return st;
  if (misaligned(state_in) || misaligned(dstate_in) || misaligned(dstate_out)) return MLSTM_ERR_INVALID;
  const StateLayout SL = state_layout(B * NH, d_qk, d_hv, variant == MLSTM_EXP);
  if (dstate_in && ((state_in && overlaps(state_in, dstate_in, SL.total)) ||
                    (dstate_out && overlaps(dstate_out, dstate_in, SL.total))))
    return MLSTM_ERR_INVALID;
  if ((long long)B * NH == 0) return MLSTM_OK;
  if (T == 0) {  // the final state is the initial one
    if (!dstate_in) return MLSTM_OK;
    if (dstate_out)
      return cuda_status(cudaMemcpyAsync(dstate_in, dstate_out, SL.total, cudaMemcpyDeviceToDevice,
                                         (cudaStream_t)stream),
                         "state copy");
    return cuda_status(cudaMemsetAsync(dstate_in, 0, SL.total, (cudaStream_t)stream), "memset");
  }
  // all five outputs NULL with a dstate_in: the state-gradient-only pass
  const bool grads = dq || dk || dv || digate_pre || dfgate_pre;
  if (!q || !k || !v || !igate_pre || !fgate_pre || !h || !dh || !saved ||
      (grads && (!dq || !dk || !dv || !digate_pre || !dfgate_pre)) || (!grads && !dstate_in))
    return MLSTM_ERR_INVALID;
  const void* ptrs[] = {q, k, v, igate_pre, fgate_pre, h, dh, saved, dq, dk, dv,
                        digate_pre, dfgate_pre, workspace};
  for (const void* ptr : ptrs)
    if (misaligned(ptr)) return MLSTM_ERR_INVALID;
  const Problem p = make_problem(B, NH, T, d_qk, d_hv, chunk, variant, dtype);
  const BwdLayout W = bwd_layout(p);
  if (!workspace || workspace_bytes < W.total) return MLSTM_ERR_WORKSPACE;
  mlstm_saved_layout_t L;
  saved_layout(p, &L);
  const char* sv = (const char*)saved;
  char* ws = (char*)workspace;
  mlstm::BwdArgs a;
  a.q = q; a.k = k; a.v = v; a.ig = igate_pre; a.fg = fgate_pre; a.h = h; a.dh = dh;
  a.b = (const float*)(sv + L.gate_b);
  a.li = (const float*)(sv + L.gate_li);
  a.m = p.exp_variant() ? (const float*)(sv + L.gate_m) : nullptr;
  a.abar = p.exp_variant() ? (const float*)(sv + L.norm) : nullptr;
  a.C = sv + L.state_c;
  a.n = p.exp_variant() ? (const float*)(sv + L.state_n) : nullptr;
  a.dq = dq; a.dk = dk; a.dv = dv; a.dig = digate_pre; a.dfg = dfgate_pre;
  a.inv_den = (float*)(ws + W.inv_den);
  a.da = (float*)(ws + W.da);
  a.pq = (float*)(ws + W.pq);
  a.pk = (float*)(ws + W.pk);
  a.pdot_planes = mlstm::intra_bwd_xl_supported(p) ? 4 : 1;
  a.pdot_stride = (size_t)p.BH * p.T;
  a.dC = ws + W.dC;
  a.dn = p.exp_variant() ? (float*)(ws + W.dn) : nullptr;
  a.init = init_from(state_in, p);
  a.dC0 = dstate_in ? (float*)((char*)dstate_in + SL.C) : nullptr;
  a.dn0 = (dstate_in && p.exp_variant()) ? (float*)((char*)dstate_in + SL.n) : nullptr;
  a.dCT = dstate_out ? (const float*)((const char*)dstate_out + SL.C) : nullptr;
  a.dnT = (dstate_out && p.exp_variant()) ? (const float*)((const char*)dstate_out + SL.n) : nullptr;
  a.fdot = dstate_out ? (float*)(ws + W.fdot) : nullptr;
  a.btab = W.btab_bytes ? (float*)(ws + W.btab) : nullptr;
  a.gsum = W.gsum_bytes ? (float*)(ws + W.gsum) : nullptr;
  cudaStream_t s = (cudaStream_t)stream;

  st = cuda_status(cudaPeekAtLastError(), "before mlstm_bwd");
  if (st != MLSTM_OK) return st;
  if (dstate_out) {
    // the final state (from the saved buffer) and its dot product with its gradient
    float* fs = (float*)(ws + W.fstate);
    const float* fC = fs + SL.C / 4;
    const float* fn = fs + SL.n / 4;
    st = cuda_status(mlstm::launch_final_state(p, k, v, a.b, a.li, a.m, a.C, a.n, a.init,
                                               fs + SL.C / 4, fs + SL.n / 4, fs + SL.m / 4, s),
                     "final_state");
    if (st != MLSTM_OK) return st;
    st = cuda_status(mlstm::launch_state_dot(p.BH, p.dqk, p.dhv, p.exp_variant(), a.dCT, a.dnT, fC,
                                             fn, a.fdot, s),
                     "state_dot");
    if (st != MLSTM_OK) return st;
  }
  BwdStep steps[kMaxSteps];
  const int n = bwd_plan(p, steps, grads);
  return run_plan(steps, n, p, a, s);
}

}  // namespace

extern "C" {

int mlstm_bwd(const void* q, const void* k, const void* v, const void* igate_pre,
              const void* fgate_pre, const void* h, const void* dh, const void* saved, void* dq,
              void* dk, void* dv, void* digate_pre, void* dfgate_pre, void* workspace,
              size_t workspace_bytes, int B, int NH, int T, int d_qk, int d_hv, int chunk,
              int variant, int dtype, void* stream) {
  return bwd_impl(q, k, v, igate_pre, fgate_pre, h, dh, saved, nullptr, nullptr, nullptr, dq, dk,
                  dv, digate_pre, dfgate_pre, workspace, workspace_bytes, B, NH, T, d_qk, d_hv,
                  chunk, variant, dtype, stream);
}

int mlstm_bwd_state(const void* q, const void* k, const void* v, const void* igate_pre,
                    const void* fgate_pre, const void* h, const void* dh, const void* saved,
                    const void* state_in, void* dstate_in, const void* dstate_out, void* dq,
                    void* dk, void* dv, void* digate_pre, void* dfgate_pre, void* workspace,
                    size_t workspace_bytes, int B, int NH, int T, int d_qk, int d_hv, int chunk,
                    int variant, int dtype, void* stream) {
  return bwd_impl(q, k, v, igate_pre, fgate_pre, h, dh, saved, state_in, dstate_in, dstate_out, dq,
                  dk, dv, digate_pre, dfgate_pre, workspace, workspace_bytes, B, NH, T, d_qk, d_hv,
                  chunk, variant, dtype, stream);
}

}  // extern "C"

extern "C" {

size_t mlstm_state_size(int B, int NH, int d_qk, int d_hv, int variant) {
  if (check_sizes(B, NH, 1, d_qk, d_hv, 64, variant, MLSTM_FP32) != MLSTM_OK) return 0;
  return state_layout(B * NH, d_qk, d_hv, variant == MLSTM_EXP).total;
}

int mlstm_state_zero(void* state, int B, int NH, int d_qk, int d_hv, int variant, void* stream) {
  int st = check_sizes(B, NH, 1, d_qk, d_hv, 64, variant, MLSTM_FP32);
  if (st != MLSTM_OK) return st;
  if ((long long)B * NH == 0) return MLSTM_OK;
  if (!state || misaligned(state)) return MLSTM_ERR_INVALID;
  const bool e = variant == MLSTM_EXP;
  const StateLayout L = state_layout(B * NH, d_qk, d_hv, e);
  char* base = (char*)state;
  return cuda_status(mlstm::launch_state_zero(B * NH, d_qk, d_hv, e, (float*)(base + L.C),
                                              (float*)(base + L.n), (float*)(base + L.m),
                                              (cudaStream_t)stream),
                     "state_zero");
}

int mlstm_final_state(const void* k, const void* v, const void* saved, void* state, int B, int NH,
                      int T, int d_qk, int d_hv, int chunk, int variant, int dtype, void* stream) {
  int st = check_sizes(B, NH, T, d_qk, d_hv, chunk, variant, dtype);
  if (st != MLSTM_OK) return st;
  if ((long long)B * NH == 0) return MLSTM_OK;
  if (T == 0) return mlstm_state_zero(state, B, NH, d_qk, d_hv, variant, stream);
  if (!k || !v || !saved || !state) return MLSTM_ERR_INVALID;
  if (misaligned(k) || misaligned(v) || misaligned(saved) || misaligned(state)) return MLSTM_ERR_INVALID;
  const Problem p = make_problem(B, NH, T, d_qk, d_hv, chunk, variant, dtype);
  mlstm_saved_layout_t L;
  saved_layout(p, &L);
  const StateLayout S = state_layout(p.BH, d_qk, d_hv, p.exp_variant());
  const char* sv = (const char*)saved;
  char* out = (char*)state;
  st = cuda_status(cudaPeekAtLastError(), "before mlstm_final_state");
  if (st != MLSTM_OK) return st;
  return cuda_status(
      mlstm::launch_final_state(p, k, v, (const float*)(sv + L.gate_b), (const float*)(sv + L.gate_li),
                                p.exp_variant() ? (const float*)(sv + L.gate_m) : nullptr,
                                sv + L.state_c,
                                p.exp_variant() ? (const float*)(sv + L.state_n) : nullptr,
                                mlstm::InitState{}, (float*)(out + S.C), (float*)(out + S.n),
                                (float*)(out + S.m),
                                (cudaStream_t)stream),
      "final_state");
}

int mlstm_step(const void* q, const void* k, const void* v, const void* igate_pre,
               const void* fgate_pre, void* h, const void* state_in, void* state_out, int B,
               int NH, int d_qk, int d_hv, int variant, int dtype, void* stream) {
  int st = check_sizes(B, NH, 1, d_qk, d_hv, 64, variant, dtype);
  if (st != MLSTM_OK) return st;
  if ((long long)B * NH == 0) return MLSTM_OK;
  if (!q || !k || !v || !igate_pre || !fgate_pre || !h || !state_in || !state_out)
    return MLSTM_ERR_INVALID;
  const void* ptrs[] = {q, k, v, h, state_in, state_out};
  for (const void* ptr : ptrs)
    if (misaligned(ptr)) return MLSTM_ERR_INVALID;
  const Problem p = make_problem(B, NH, 1, d_qk, d_hv, 64, variant, dtype);
  const StateLayout S = state_layout(p.BH, d_qk, d_hv, p.exp_variant());
  if (overlaps(state_in, state_out, S.total)) return MLSTM_ERR_INVALID;
  const char* si = (const char*)state_in;
  char* so = (char*)state_out;
  st = cuda_status(cudaPeekAtLastError(), "before mlstm_step");
  if (st != MLSTM_OK) return st;
  return cuda_status(
      mlstm::launch_step(p, q, k, v, igate_pre, fgate_pre, h, (const float*)(si + S.C),
                         (const float*)(si + S.n), (const float*)(si + S.m), (float*)(so + S.C),
                         (float*)(so + S.n), (float*)(so + S.m), (cudaStream_t)stream),
      "step");
}

int mlstm_log_decay(const void* fgate_pre, float* log_decay, int B, int NH, int T, int dtype,
                    void* stream) {
  int st = check_sizes(B, NH, T, 64, 64, 64, MLSTM_SIG, dtype);
  if (st != MLSTM_OK) return st;
  if ((long long)B * NH == 0) return MLSTM_OK;
  if (!log_decay || misaligned(log_decay) || (T > 0 && (!fgate_pre || misaligned(fgate_pre))))
    return MLSTM_ERR_INVALID;
  if (T == 0)
    return cuda_status(cudaMemsetAsync(log_decay, 0, (size_t)B * NH * sizeof(float),
                                       (cudaStream_t)stream),
                       "memset");
  const Problem p = make_problem(B, NH, T, 64, 64, 64, MLSTM_SIG, dtype);
  st = cuda_status(cudaPeekAtLastError(), "before mlstm_log_decay");
  if (st != MLSTM_OK) return st;
  return cuda_status(mlstm::launch_log_decay(p, fgate_pre, log_decay, (cudaStream_t)stream),
                     "log_decay");
}

int mlstm_state_chain(const void* state_a, const void* state_b, const float* log_decay_b,
                      void* state_out, int B, int NH, int d_qk, int d_hv, int variant,
                      void* stream) {
  int st = check_sizes(B, NH, 1, d_qk, d_hv, 64, variant, MLSTM_FP32);
  if (st != MLSTM_OK) return st;
  if ((long long)B * NH == 0) return MLSTM_OK;
  if (!state_a || !state_b || !log_decay_b || !state_out) return MLSTM_ERR_INVALID;
  const void* ptrs[] = {state_a, state_b, log_decay_b, state_out};
  for (const void* ptr : ptrs)
    if (misaligned(ptr)) return MLSTM_ERR_INVALID;
  const bool e = variant == MLSTM_EXP;
  const StateLayout S = state_layout(B * NH, d_qk, d_hv, e);
  if (overlaps(state_out, state_a, S.total) || overlaps(state_out, state_b, S.total))
    return MLSTM_ERR_INVALID;
  const char* pa = (const char*)state_a;
  const char* pb = (const char*)state_b;
  char* po = (char*)state_out;
  st = cuda_status(cudaPeekAtLastError(), "before mlstm_state_chain");
  if (st != MLSTM_OK) return st;
  return cuda_status(
      mlstm::launch_state_chain(B * NH, d_qk, d_hv, e, (const float*)(pa + S.C),
                                (const float*)(pa + S.n), (const float*)(pa + S.m),
                                (const float*)(pb + S.C), (const float*)(pb + S.n),
                                (const float*)(pb + S.m), log_decay_b, (float*)(po + S.C),
                                (float*)(po + S.n), (float*)(po + S.m), (cudaStream_t)stream),
      "state_chain");
}

int mlstm_dstate_chain(const void* dstate_local, const void* dstate_out, const void* state_in,
                       const void* state_out, const float* log_decay, void* dstate_in, int B,
                       int NH, int d_qk, int d_hv, int variant, void* stream) {
  int st = check_sizes(B, NH, 1, d_qk, d_hv, 64, variant, MLSTM_FP32);
  if (st != MLSTM_OK) return st;
  if ((long long)B * NH == 0) return MLSTM_OK;
  if (!dstate_local || !dstate_out || !state_in || !state_out || !log_decay || !dstate_in)
    return MLSTM_ERR_INVALID;
  const void* ptrs[] = {dstate_local, dstate_out, state_in, state_out, log_decay, dstate_in};
  for (const void* ptr : ptrs)
    if (misaligned(ptr)) return MLSTM_ERR_INVALID;
  const bool e = variant == MLSTM_EXP;
  const StateLayout S = state_layout(B * NH, d_qk, d_hv, e);
  if (overlaps(dstate_in, dstate_local, S.total) || overlaps(dstate_in, dstate_out, S.total))
    return MLSTM_ERR_INVALID;
  const char* pl = (const char*)dstate_local;
  const char* pd = (const char*)dstate_out;
  const char* pi = (const char*)state_in;
  const char* po = (const char*)state_out;
  char* pr = (char*)dstate_in;
  st = cuda_status(cudaPeekAtLastError(), "before mlstm_dstate_chain");
  if (st != MLSTM_OK) return st;
  return cuda_status(
      mlstm::launch_dstate_chain(B * NH, d_qk, d_hv, e, (const float*)(pl + S.C),
                                 (const float*)(pl + S.n), (const float*)(pd + S.C),
                                 (const float*)(pd + S.n), (const float*)(pi + S.m),
                                 (const float*)(po + S.m), log_decay, (float*)(pr + S.C),
                                 (float*)(pr + S.n), (cudaStream_t)stream),
      "dstate_chain");
}

const char* mlstm_status_string(int status) {
  switch (status) {
    case MLSTM_OK: return "ok";
    case MLSTM_ERR_INVALID: return "invalid argument";
    case MLSTM_ERR_UNSUPPORTED: return "unsupported size";
    case MLSTM_ERR_WORKSPACE: return "workspace or saved buffer too small";
    case MLSTM_ERR_CUDA: return "CUDA error";
    case MLSTM_ERR_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
  }
}

const char* mlstm_last_error(void) { return g_last_error; }

}  // extern "C"

namespace {
// Failures already reported, per device and kernel family: the flag values
// mlstm_device_status saw last.  A flag holds the epoch of the last launch of
// its family that gave up, so a value that differs from the last one seen is a
// failure not yet reported.
constexpr int kFlagDevices = 64, kFlagFamilies = 7;
std::mutex g_flag_mu;
unsigned int g_flag_seen[kFlagDevices][kFlagFamilies] = {};
}  // namespace

extern "C" {

int mlstm_device_status(void* stream) {
  int st = cuda_status(cudaStreamSynchronize((cudaStream_t)stream), "stream synchronize");
  if (st != MLSTM_OK) return st;
  int dev = 0;
  st = cuda_status(cudaGetDevice(&dev), "device");
  if (st != MLSTM_OK) return st;
  if (dev < 0 || dev >= kFlagDevices) return MLSTM_ERR_UNSUPPORTED;
  // read every flag before deciding anything; nothing is cleared
  typedef cudaError_t (*Fetch)(unsigned int*);
  const Fetch fetch[kFlagFamilies] = {mlstm::fetch_tc_fwd_error,    mlstm::fetch_tc_bwd_error,
                                      mlstm::fetch_tc_state_error,  mlstm::fetch_tc_fwd_xl_error,
                                      mlstm::fetch_tc_walk_error,   mlstm::fetch_tc_fwalk_error,
                                      mlstm::fetch_tc_bwd_xl_error};
  unsigned int flag[kFlagFamilies] = {};
  for (int i = 0; i < kFlagFamilies; ++i) {
    st = cuda_status(fetch[i](&flag[i]), "device error flag");
    if (st != MLSTM_OK) return st;
  }
  bool fresh = false;
  {
    std::lock_guard<std::mutex> lock(g_flag_mu);
    for (int i = 0; i < kFlagFamilies; ++i) {
      if (flag[i] != g_flag_seen[dev][i]) fresh = true;
      g_flag_seen[dev][i] = flag[i];
    }
  }
  if (fresh) {
    snprintf(g_last_error, sizeof(g_last_error), "a tensor-core kernel timed out waiting");
    return MLSTM_ERR_TIMEOUT;
  }
  return MLSTM_OK;
}

int mlstm_selftest_timeout(void* stream) {
  return cuda_status(mlstm::launch_selftest_timeout((cudaStream_t)stream), "selftest_timeout");
}

}  // extern "C"
