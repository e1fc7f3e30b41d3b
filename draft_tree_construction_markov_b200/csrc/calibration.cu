// dt_calib_log / dt_calib_fit: calibration of the edge-acceptance estimate
// from logged verification outcomes.
//
// Source: TreeSpark article, "core idea": the parent-conditioned probability
// is calibrated into an estimate of the edge's acceptance; path survival,
// the product of those estimates, drives the tree.  The pages give neither
// the form nor the fit.  The form is the build's,
//   c_d(l) = min(0, alpha_d * l + beta_d),  estimate exp(c_d(l)),
// and the fit is, per child depth d, the grid point with the largest
// Bernoulli log-likelihood of the logged outcomes
//   sum_{y=1} c(l) + sum_{y=0} log(1 - exp(c(l)))
// (ties to the smaller alpha index, then the smaller beta index).
//
// dt_calib_log: one warp per request.  For every child of a node the greedy
// walk reached (the root and each accepted node) it writes (depth, l, y):
// l = key(child) - key(parent) in fp32, the child's log-probability when the
// tree was built with the identity calibration, and y = 1 iff accepted.
//
// dt_calib_fit: one thread per grid point and depth, in CTAs of 256 points
// per depth.  Every CTA compacts the samples of its depth into shared memory
// a chunk at a time (in sample order) and accumulates each point's fp64
// log-likelihood; a CTA arg-max and then a per-depth pick over the blocks
// (in block order) select the point.
#include "dtree.h"
#include "common.cuh"

namespace dt {
namespace {

constexpr int kLogWarps = 8;
constexpr int kFitThreads = 256;  // grid points per CTA
constexpr int kChunk = 2048;      // samples staged per pass
constexpr int kMaxPoints = 1 << 20;

struct FitPartial {
  double ll;
  int32_t idx;   // grid point index i * n_beta + j (INT_MAX: none)
  int32_t seen;  // samples of the depth
};

__global__ void __launch_bounds__(kLogWarps * 32)
    calib_log_kernel(dt_tree t, const int32_t* __restrict__ acc_nodes,
                     const int32_t* __restrict__ n_acc, int batch, int Bk, int Nmax,
                     int32_t* __restrict__ depth_out, float* __restrict__ ell_out,
                     int8_t* __restrict__ y_out, int32_t* status) {
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.x * kLogWarps + (threadIdx.x >> 5);
  if (b >= batch) return;
  int n = t.d_n_nodes[b];
  if (n < 0 || n > Nmax) {
    if (lane == 0) set_status(status, DT_EDEVICE);
    n = n < 0 ? 0 : Nmax;
  }
  int na = n_acc[b];
  if (na < 0 || na > Bk) {
    if (lane == 0) set_status(status, DT_EDEVICE);
    na = na < 0 ? 0 : Bk;
  }
  // nodes on the accepted path
  uint64_t mine = 0;
  for (int j = lane; j < na; j += 32) {
    const int v = acc_nodes[(size_t)b * Bk + j];
    if (v >= 0 && v < n)
      mine |= 1ull << v;
    else
      set_status(status, DT_EDEVICE);
  }
  for (int o = 16; o; o >>= 1) mine |= __shfl_xor_sync(0xffffffffu, mine, o);
  const size_t base = (size_t)b * Nmax;
  for (int i = lane; i < Nmax; i += 32) {
    int dep = -1;
    float l = 0.f;
    int8_t yy = 0;
    if (i < n) {
      const int p = t.d_parents[base + i];
      if (p < -1 || p >= i) {
        set_status(status, DT_EDEVICE);  // parents precede children in pop order
      } else if (p < 0 || ((mine >> p) & 1)) {
        dep = t.d_depths[base + i];
        const float kp = p < 0 ? 0.f : t.d_keys[base + p];
        l = __fsub_rn(t.d_keys[base + i], kp);
        yy = (int8_t)((mine >> i) & 1);
      }
    }
    depth_out[base + i] = dep;
    ell_out[base + i] = l;
    y_out[base + i] = yy;
  }
}

// One thread per grid point, grid (depth, point block): every CTA stages the
// samples of its depth and writes the best point of its block.
__global__ void __launch_bounds__(kFitThreads)
    calib_fit_partial_kernel(const int32_t* __restrict__ depth, const float* __restrict__ ell,
                             const int8_t* __restrict__ y, int n, double a0, double da,
                             int na, double b0, double db, int nb, FitPartial* __restrict__ part) {
  __shared__ double s_l[kChunk];
  __shared__ int8_t s_y[kChunk];
  __shared__ int s_cnt[kFitThreads / 32];
  __shared__ int s_total;
  __shared__ double r_ll[kFitThreads / 32];
  __shared__ int r_idx[kFitThreads / 32];
  const int d = blockIdx.x + 1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int npts = na * nb;
  const int gp = blockIdx.y * kFitThreads + tid;
  const bool live = gp < npts;
  // the grid point (separate roundings, as written)
  const double a = __dadd_rn(a0, __dmul_rn((double)(gp / nb), da));
  const double bb = __dadd_rn(b0, __dmul_rn((double)(gp % nb), db));
  double acc = 0.0;
  int seen = 0;
  constexpr int per = kChunk / kFitThreads;  // consecutive samples per thread
  for (int c0 = 0; c0 < n; c0 += kChunk) {
    // compact this chunk's samples of depth d, keeping their order
    bool take[per];
    int mycnt = 0;
#pragma unroll
    for (int q = 0; q < per; ++q) {
      const int i = c0 + tid * per + q;
      take[q] = i < n && depth[i] == d;
      mycnt += take[q];
    }
    int incl = mycnt;
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) s_cnt[warp] = incl;
    __syncthreads();
    if (tid == 0) {
      int run = 0;
      for (int w = 0; w < kFitThreads / 32; ++w) {
        const int v = s_cnt[w];
        s_cnt[w] = run;
        run += v;
      }
      s_total = run;
    }
    __syncthreads();
    int pos = s_cnt[warp] + incl - mycnt;
#pragma unroll
    for (int q = 0; q < per; ++q) {
      if (take[q]) {
        const int i = c0 + tid * per + q;
        s_l[pos] = (double)ell[i];
        s_y[pos] = y[i] ? 1 : 0;
        ++pos;
      }
    }
    __syncthreads();
    const int m = s_total;
    seen += m;
    if (live) {
      for (int s = 0; s < m; ++s) {
        const double x = fmin(0.0, __dadd_rn(__dmul_rn(a, s_l[s]), bb));
        acc += s_y[s] ? x : log1p(-exp(x));
      }
    }
    __syncthreads();
  }
  // arg-max over the block: larger log-likelihood, then the smaller index
  double best = live ? acc : -INFINITY;
  int bidx = live ? gp : 0x7fffffff;
  for (int o = 16; o; o >>= 1) {
    const double ov = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bidx, o);
    if (ov > best || (ov == best && oi < bidx)) {
      best = ov;
      bidx = oi;
    }
  }
  if (lane == 0) {
    r_ll[warp] = best;
    r_idx[warp] = bidx;
  }
  __syncthreads();
  if (tid == 0) {
    for (int w = 1; w < kFitThreads / 32; ++w)
      if (r_ll[w] > best || (r_ll[w] == best && r_idx[w] < bidx)) {
        best = r_ll[w];
        bidx = r_idx[w];
      }
    FitPartial fp;
    fp.ll = best;
    fp.idx = bidx;
    fp.seen = seen;
    part[(size_t)blockIdx.x * gridDim.y + blockIdx.y] = fp;
  }
}

// One thread per depth: the best of its blocks, in block order.
__global__ void calib_fit_pick_kernel(const FitPartial* __restrict__ part, int nblk, int Bk,
                                      double a0, double da, double b0, double db, int nb,
                                      int min_samples, float* __restrict__ calib,
                                      double* __restrict__ loglik) {
  const int d = blockIdx.x * blockDim.x + threadIdx.x;
  if (d >= Bk) return;
  double best = -INFINITY;
  int bidx = 0x7fffffff, seen = 0;
  for (int j = 0; j < nblk; ++j) {
    const FitPartial p = part[(size_t)d * nblk + j];
    seen = p.seen;
    if (p.idx == 0x7fffffff) continue;
    if (bidx == 0x7fffffff || p.ll > best || (p.ll == best && p.idx < bidx)) {
      best = p.ll;
      bidx = p.idx;
    }
  }
  if (seen < min_samples || bidx == 0x7fffffff) {
    calib[2 * d] = 1.f;  // too few logged edges at this depth: identity
    calib[2 * d + 1] = 0.f;
    if (loglik) loglik[d] = NAN;
  } else {
    calib[2 * d] = (float)__dadd_rn(a0, __dmul_rn((double)(bidx / nb), da));
    calib[2 * d + 1] = (float)__dadd_rn(b0, __dmul_rn((double)(bidx % nb), db));
    if (loglik) loglik[d] = best;
  }
}

}  // namespace
}  // namespace dt

using namespace dt;

extern "C" {

static size_t fit_blocks(int n_alpha, int n_beta) {
  return ((size_t)n_alpha * n_beta + kFitThreads - 1) / kFitThreads;
}

size_t dt_calib_workspace_bytes(int Bk, int n_alpha, int n_beta) {
  if (Bk < 1 || n_alpha < 1 || n_beta < 1) return kWsHeader;
  return kWsHeader + (size_t)Bk * fit_blocks(n_alpha, n_beta) * sizeof(FitPartial);
}

dt_status dt_calib_log(const dt_tree* tree, const int32_t* d_acc_nodes, const int32_t* d_n_acc,
                       int batch, int Bk, int Nmax, int32_t* d_depth, float* d_ell,
                       int8_t* d_y, void* ws, size_t ws_bytes, dt_stream stream) {
  if (!tree || !tree->d_parents || !tree->d_depths || !tree->d_keys || !tree->d_n_nodes ||
      !d_acc_nodes || !d_n_acc || !d_depth || !d_ell || !d_y)
    return DT_EINVAL;
  if (batch < 1 || Bk < 1 || Nmax < 1) return DT_EINVAL;
  if (batch > 1024 || Bk > 16 || Nmax > 64) return DT_EUNSUPPORTED;
  if (!ws || ws_bytes < kWsHeader) return DT_EWORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  int32_t* status = (int32_t*)ws;
  if (cudaMemsetAsync(status, 0, 4, s) != cudaSuccess) return DT_ECUDA;
  ProfileScope ps(DT_K_OTHER, s);
  calib_log_kernel<<<(batch + kLogWarps - 1) / kLogWarps, kLogWarps * 32, 0, s>>>(
      *tree, d_acc_nodes, d_n_acc, batch, Bk, Nmax, d_depth, d_ell, d_y, status);
  return cudaGetLastError() == cudaSuccess ? DT_OK : DT_ECUDA;
}

dt_status dt_calib_fit(const int32_t* d_depth, const float* d_ell, const int8_t* d_y, int n,
                       int Bk, float alpha0, float dalpha, int n_alpha, float beta0,
                       float dbeta, int n_beta, int min_samples, float* d_calib,
                       double* d_loglik, void* ws, size_t ws_bytes, dt_stream stream) {
  if (!d_calib || (n > 0 && (!d_depth || !d_ell || !d_y))) return DT_EINVAL;
  min_samples = min_samples < 1 ? 1 : min_samples;
  if (n < 0 || Bk < 1 || n_alpha < 1 || n_beta < 1) return DT_EINVAL;
  if (!(alpha0 >= 0.f) || !(dalpha >= 0.f) || !(dbeta >= 0.f) || !(beta0 == beta0))
    return DT_EINVAL;
  if (Bk > 16 || (long long)n_alpha * n_beta > kMaxPoints) return DT_EUNSUPPORTED;
  if (!ws || ws_bytes < dt_calib_workspace_bytes(Bk, n_alpha, n_beta)) return DT_EWORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(ws, 0, 4, s) != cudaSuccess) return DT_ECUDA;
  FitPartial* part = (FitPartial*)((uint8_t*)ws + kWsHeader);
  const int nblk = (int)fit_blocks(n_alpha, n_beta);
  {
    ProfileScope ps(DT_K_OTHER, s);
    calib_fit_partial_kernel<<<dim3(Bk, nblk), kFitThreads, 0, s>>>(
        d_depth, d_ell, d_y, n, (double)alpha0, (double)dalpha, n_alpha, (double)beta0,
        (double)dbeta, n_beta, part);
    if (cudaGetLastError() != cudaSuccess) return DT_ECUDA;
  }
  ProfileScope ps(DT_K_OTHER, s);
  calib_fit_pick_kernel<<<1, 32, 0, s>>>(part, nblk, Bk, (double)alpha0, (double)dalpha,
                                         (double)beta0, (double)dbeta, n_beta, min_samples,
                                         d_calib, d_loglik);
  return cudaGetLastError() == cudaSuccess ? DT_OK : DT_ECUDA;
}

}  // extern "C"
