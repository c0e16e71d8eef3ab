// Allocation-free forward entry point.
//
// Some callers cannot call cudaMalloc at the point where they run the
// forward pass: code running under a custom allocator that must not be
// bypassed, plugins whose host framework owns all device allocations, or
// launch paths where an allocation would synchronise the device.  For them
// mlstm_fwd_noalloc runs the ordinary forward with its scratch (the gate
// cumulative sums, max states and chunk states that mlstm_fwd otherwise keeps
// in the caller's workspace) placed in a fixed array compiled into this
// library.  The caller still passes the inputs and the output.
#include <mutex>

#include "internal.h"
#include "mlstm.h"

namespace {

constexpr size_t kScratchBytes = 32ull << 20;  // 32 MiB, held on every GPU that loads the library
constexpr int kMaxDevices = 64;

// Device-side scratch.  In host code this name is only a host-side stand-in;
// its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_fwd_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

}  // namespace

extern "C" int mlstm_fwd_noalloc(const void* q, const void* k, const void* v, const void* igate_pre,
                                 const void* fgate_pre, void* h, int B, int NH, int T, int d_qk,
                                 int d_hv, int chunk, int variant, int dtype, void* stream) {
  mlstm_saved_layout_t layout;
  const int st = mlstm_saved_layout(B, NH, T, d_qk, d_hv, chunk, variant, dtype, &layout);
  if (st != MLSTM_OK) return st;
  if (layout.total > kScratchBytes) return MLSTM_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLSTM_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MLSTM_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  {
    // once per device, with that device current: the device address of the array
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    scratch = g_scratch_addr[dev];
    if (scratch == nullptr) {
      if (cudaGetSymbolAddress(&scratch, g_fwd_scratch) != cudaSuccess || scratch == nullptr)
        return MLSTM_ERR_CUDA;
      g_scratch_addr[dev] = scratch;
    }
  }
  // Nothing in the scratch has to start at zero: every region the forward
  // reads is written earlier in the same call.
  return mlstm_fwd(q, k, v, igate_pre, fgate_pre, h, nullptr, scratch, kScratchBytes, B, NH, T,
                   d_qk, d_hv, chunk, variant, dtype, stream);
}
