// dt_tree_accept_noalloc: the acceptance walk for callers that cannot
// allocate device memory (see the declaration in dtree.h for who and why).
//
// The walk's scratch (status word, per-row partial statistics, the two
// residual buffers) lives in one file-scope device array of fixed size
// instead of a caller-provided workspace.  Host code cannot use the array's
// name as a device address, so the address is looked up once per device with
// cudaGetSymbolAddress and then handed to the same launch path that
// dt_tree_accept uses.  Nothing here allocates or frees memory.
#include <mutex>

#include "dtree.h"
#include "common.cuh"

namespace {

// Largest scratch the walk may need: 2 MiB covers a batch-1 round at a
// 151936-token vocabulary (two fp32 residual rows plus per-row partials).
constexpr size_t kNoAllocScratchBytes = 2u << 20;

// Shared by every call on a device and kept between calls; it holds no
// results, only the walk's temporaries.  Calls that overlap on the GPU race.
static __device__ __align__(256) unsigned char g_accept_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void* g_addr[64] = {nullptr};  // device address of the array, per device

// Resolves the array's device address on the current device (first call on a
// device only).  Returns nullptr if the lookup fails.
void* scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_accept_scratch) != cudaSuccess) return nullptr;
    g_addr[dev] = p;
  }
  return g_addr[dev];
}

}  // namespace

extern "C" dt_status dt_tree_accept_noalloc(const void* d_target_logits, dt_dtype tdt,
                                            const dt_tree* tree, int batch, int Bk, int V,
                                            int Nmax, float temp, uint64_t philox_seed,
                                            uint64_t philox_offset, int32_t* d_acc_nodes,
                                            int32_t* d_n_acc, int32_t* d_bonus,
                                            dt_stream stream) {
  if (batch < 1 || Nmax < 1 || V < 1) return DT_EINVAL;
  const size_t need = dt_tree_accept_workspace_bytes(batch, Nmax, V);
  if (need == 0 || need > kNoAllocScratchBytes) return DT_EUNSUPPORTED;  // beyond the fixed scratch
  void* ws = scratch_address();
  if (!ws) return DT_ECUDA;
  // dt_tree_accept clears the status word and its arrival counters itself;
  // nothing else in the scratch must start at zero
  return dt_tree_accept(d_target_logits, tdt, tree, batch, Bk, V, Nmax, temp, philox_seed,
                        philox_offset, d_acc_nodes, d_n_acc, d_bonus, ws, kNoAllocScratchBytes,
                        stream);
}
