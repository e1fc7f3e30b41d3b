// dt_tree_load_budget: the load-adaptive tree size.  One survival signal
// allocates a round's verification capacity over the requests of a batch.
//
// Sources: TreeSpark article, "core idea" (the load-adaptive serving policy
// sizes the trees with the same calibrated path survival that drives
// expansion and stopping) and "measured gains" (as load rises the trees
// shrink back toward the chain).
//
// A verified node of request b costs w_b = 1 + floor(P_b / prefix_unit)
// units.  The nodes of the batch are ordered by (fp32 key desc, request asc,
// pop index asc) and the batch keeps the longest prefix of that order whose
// cost fits the capacity C.  Every request's keys are non-increasing along
// its pop order, so the prefix holds, per request, a prefix of its tree.
//
// One CTA, one thread per request.  A binary search over the order-preserving
// 32-bit image of the keys finds the key T of the first node that does not
// fit: the largest v with W(>= v) > C, where W(>= v) is the cost of the nodes
// whose key image is >= v (each request counts its own by binary search).
// Every node above T is kept; the nodes equal to T go to the requests in
// order while they fit.
#include "dtree.h"
#include "common.cuh"

namespace dt {
namespace {

constexpr int kBudgetThreads = 1024;

// nodes of a request (keys non-increasing) whose key image is >= v
__device__ __forceinline__ int count_ge(const float* keys, int n, uint32_t v) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (f32_ordered(keys[mid]) >= v)
      lo = mid + 1;
    else
      hi = mid;
  }
  return lo;
}

// sum over the CTA; every thread must call it
__device__ long long block_sum(long long x, long long* red) {
  for (int o = 16; o; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();  // red is free again
  if (lane == 0) red[warp] = x;
  __syncthreads();
  long long s = 0;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) s += red[i];
  return s;
}

__global__ void __launch_bounds__(kBudgetThreads)
    load_budget_kernel(dt_tree t, int batch, int Nmax, const int32_t* __restrict__ plen,
                       long long cap, int unit, int32_t* __restrict__ n_keep,
                       int32_t* status) {
  __shared__ long long red[32];
  __shared__ int s_ties[kBudgetThreads];
  __shared__ long long s_w[kBudgetThreads];
  __shared__ int s_take[kBudgetThreads];
  const int b = threadIdx.x;
  const bool own = b < batch;
  int n = 0;
  long long w = 1;
  const float* keys = t.d_keys + (size_t)b * Nmax;
  if (own) {
    n = t.d_n_nodes[b];
    if (n < 0 || n > Nmax) {
      set_status(status, DT_EDEVICE);
      n = n < 0 ? 0 : Nmax;
    }
    const int p = plen ? plen[b] : 0;
    if (p < 0) set_status(status, DT_EDEVICE);
    w = 1 + ((unit > 0 && p > 0) ? p / unit : 0);
  }
  int keep = n;
  const long long total = block_sum(own ? (long long)n * w : 0, red);
  if (total > cap) {
    // largest v with W(>= v) > cap; W(>= 0) = total > cap
    uint32_t lo = 0;
    uint64_t hi = 1ull << 32;
    while (hi - lo > 1) {
      const uint32_t mid = (uint32_t)((lo + hi) >> 1);
      const long long wv = block_sum(own ? (long long)count_ge(keys, n, mid) * w : 0, red);
      if (wv > cap)
        lo = mid;
      else
        hi = mid;
    }
    const int ge = own ? count_ge(keys, n, lo) : 0;
    const int gt = (own && lo != 0xffffffffu) ? count_ge(keys, n, lo + 1) : 0;
    const long long rem0 = cap - block_sum(own ? (long long)gt * w : 0, red);
    s_ties[b] = ge - gt;
    s_w[b] = w;
    __syncthreads();
    if (b == 0) {
      // nodes with key T, request by request, until one does not fit
      long long rem = rem0;
      for (int i = 0; i < batch; ++i) {
        long long m = 0;
        if (rem >= 0) {
          m = rem / s_w[i];
          if (m >= s_ties[i]) {
            m = s_ties[i];
            rem -= m * s_w[i];
          } else {
            rem = -1;
          }
        }
        s_take[i] = (int)m;
      }
    }
    __syncthreads();
    keep = gt + (own ? s_take[b] : 0);
  }
  if (own) {
    t.d_n_nodes[b] = keep;
    if (n_keep) n_keep[b] = keep;
  }
}

}  // namespace
}  // namespace dt

using namespace dt;

extern "C" {

size_t dt_tree_load_budget_workspace_bytes(void) { return kWsHeader; }

dt_status dt_tree_load_budget(const dt_tree* tree, int batch, int Nmax,
                              const int32_t* d_prefix_len, int64_t capacity, int prefix_unit,
                              int32_t* d_n_keep, void* ws, size_t ws_bytes, dt_stream stream) {
  if (!tree || !tree->d_keys || !tree->d_n_nodes) return DT_EINVAL;
  if (batch < 1 || Nmax < 1 || capacity < 0 || prefix_unit < 0) return DT_EINVAL;
  if (batch > kBudgetThreads || Nmax > 64) return DT_EUNSUPPORTED;
  if (!ws || ws_bytes < kWsHeader) return DT_EWORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  int32_t* status = (int32_t*)ws;
  if (cudaMemsetAsync(status, 0, 4, s) != cudaSuccess) return DT_ECUDA;
  ProfileScope ps(DT_K_OTHER, s);
  load_budget_kernel<<<1, kBudgetThreads, 0, s>>>(*tree, batch, Nmax, d_prefix_len,
                                                  (long long)capacity, prefix_unit, d_n_keep,
                                                  status);
  return cudaGetLastError() == cudaSuccess ? DT_OK : DT_ECUDA;
}

}  // extern "C"
