// Lossless acceptance walk over a verified draft tree.
//
// Sources: TreeSpark article, introduction (draft-then-verify with an
// accept/reject rule that preserves the target distribution) and "lossless"
// section (siblings sampled without replacement, residuals matched in
// recursive rejection); PCTree summary, "setup" (greedy verification).
//
// A pre-pass over every target row of every request (row 0 = root, row i+1 =
// node i, rows past n_nodes skipped) computes, per row chunk, the argmax
// (T = 0) or the max and sum of exp(t / T) (T > 0).  At T = 0 that is the
// only launch: the last pre-pass CTA of a request (an arrival counter per
// request) walks the tree with one warp, comparing child tokens with row
// argmaxes.  At T > 0 a second launch walks each request on one thread-block
// cluster, where every rejected sibling costs one vocabulary-wide residual
// pass, r <- max(p - q_j, 0), split over the cluster's CTAs.
#include <cooperative_groups.h>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace dt {

int num_sms();  // SMs of the current device (api_build.cu)

constexpr int kPreThreads = 256;
constexpr int kWalkThreads = 1024;
constexpr float kL2e = 1.4426950408889634f;

__device__ __forceinline__ float ld_logit(const void* base, int bf16, size_t i) {
  return bf16 ? bf16_to_f32(((const uint16_t*)base)[i]) : ((const float*)base)[i];
}

// Four consecutive logits from index i (a multiple of 4; the row is 16-byte
// aligned in fp32 and 8-byte aligned in bf16).
__device__ __forceinline__ void ld_logit4(const void* base, int bf16, size_t i, float (&v)[4]) {
  if (bf16) {
    const uint2 u = __ldg((const uint2*)((const uint16_t*)base + i));
    v[0] = __uint_as_float(u.x << 16);
    v[1] = __uint_as_float(u.x & 0xffff0000u);
    v[2] = __uint_as_float(u.y << 16);
    v[3] = __uint_as_float(u.y & 0xffff0000u);
  } else {
    const float4 f = __ldg((const float4*)((const float*)base + i));
    v[0] = f.x;
    v[1] = f.y;
    v[2] = f.z;
    v[3] = f.w;
  }
}

struct AccParts {
  float* pv;    // [rows_total][splits] argmax value or (T>0) max
  int32_t* pi;  // [rows_total][splits] argmax id
  float* ps;    // [rows_total][splits] sum exp(t/T - max)   (T > 0)
};

// Partial statistics of chunk blockIdx.x of target row row_g (all threads of
// the CTA): argmax (T = 0) or (max, sum exp(t / T - max)) (T > 0).
template <bool STOCH>
__device__ __forceinline__ void prepass_chunk(const void* t, int tbf16, int row_g, int V,
                                              int splits, float temp, AccParts parts) {
  const int chunk = ((V + splits - 1) / splits + 7) & ~7;
  const int x0 = blockIdx.x * chunk, x1 = min(V, x0 + chunk);
  const size_t base = (size_t)row_g * V;
  float best = -INFINITY;
  int32_t bid = 0x7fffffff;
  float mx = -INFINITY, sm = 0.f;
  auto consume = [&](float v, int x) {
    if (!STOCH) {
      if (v > best) {  // x increases within a thread: strict keeps the lower id
        best = v;
        bid = x;
      }
    } else {
      const float s = __fdiv_rn(v, temp);
      const float d = s - mx;
      const float ex = exp2f(-fabsf(d) * kL2e);
      sm = d > 0.f ? fmaf(sm, ex, 1.f) : sm + ex;
      mx = fmaxf(mx, s);
    }
  };
  const bool vec = tbf16 ? (V % 8 == 0) : (V % 4 == 0);
  if (vec && tbf16) {
    const uint4* p4 = (const uint4*)((const uint16_t*)t + base + x0);
    const int n8 = (x1 - x0) >> 3;
#pragma unroll 4
    for (int i = threadIdx.x; i < n8; i += kPreThreads) {
      const uint4 u = p4[i];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
      const int x = x0 + 8 * i;
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        consume(__uint_as_float(w[h] << 16), x + 2 * h);
        consume(__uint_as_float(w[h] & 0xFFFF0000u), x + 2 * h + 1);
      }
    }
    for (int x = x0 + 8 * n8 + threadIdx.x; x < x1; x += kPreThreads)
      consume(ld_logit(t, tbf16, base + x), x);
  } else if (vec) {
    const float4* p4 = (const float4*)((const float*)t + base + x0);
    const int n4 = (x1 - x0) >> 2;
#pragma unroll 4
    for (int i = threadIdx.x; i < n4; i += kPreThreads) {
      const float4 u = p4[i];
      const int x = x0 + 4 * i;
      consume(u.x, x);
      consume(u.y, x + 1);
      consume(u.z, x + 2);
      consume(u.w, x + 3);
    }
    for (int x = x0 + 4 * n4 + threadIdx.x; x < x1; x += kPreThreads)
      consume(ld_logit(t, tbf16, base + x), x);
  } else {
    for (int x = x0 + threadIdx.x; x < x1; x += kPreThreads) consume(ld_logit(t, tbf16, base + x), x);
  }
  __shared__ float sv[kPreThreads / 32];
  __shared__ int32_t si[kPreThreads / 32];
  __shared__ float ss[kPreThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (!STOCH) {
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, best, o);
      const int32_t oi = __shfl_xor_sync(0xffffffffu, bid, o);
      if (ov > best || (ov == best && oi < bid)) {
        best = ov;
        bid = oi;
      }
    }
    if (lane == 0) {
      sv[warp] = best;
      si[warp] = bid;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      for (int w = 1; w < kPreThreads / 32; ++w)
        if (sv[w] > best || (sv[w] == best && si[w] < bid)) {
          best = sv[w];
          bid = si[w];
        }
      parts.pv[(size_t)row_g * splits + blockIdx.x] = best;
      parts.pi[(size_t)row_g * splits + blockIdx.x] = bid;
    }
  } else {
    const float wm = warp_max(mx);
    float ws = (mx == -INFINITY) ? 0.f : sm * exp2f((mx - wm) * kL2e);
    ws = warp_sum(ws);
    if (lane == 0) {
      sv[warp] = wm;
      ss[warp] = ws;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      float m2 = -INFINITY;
      for (int w = 0; w < kPreThreads / 32; ++w) m2 = fmaxf(m2, sv[w]);
      float s2 = 0.f;
      for (int w = 0; w < kPreThreads / 32; ++w)
        if (sv[w] != -INFINITY) s2 += ss[w] * exp2f((sv[w] - m2) * kL2e);
      parts.pv[(size_t)row_g * splits + blockIdx.x] = m2;
      parts.ps[(size_t)row_g * splits + blockIdx.x] = s2;
    }
  }
}

// Pre-pass: grid (splits, batch * (Nmax + 1)).
template <bool STOCH>
__global__ void __launch_bounds__(kPreThreads)
    accept_prepass_kernel(const void* t, int tbf16, const int32_t* n_nodes, int Nmax, int V,
                          int splits, float temp, AccParts parts) {
  const int row_g = blockIdx.y;
  const int b = row_g / (Nmax + 1), row = row_g % (Nmax + 1);
  if (row > min(n_nodes[b], Nmax)) return;
  prepass_chunk<STOCH>(t, tbf16, row_g, V, splits, temp, parts);
}

struct WalkArgs {
  const void* t;
  int tbf16;
  const int32_t* tokens;
  const int32_t* parents;
  const int32_t* ranks;
  const int32_t* n_nodes;
  const float* draft_q;
  int Bk, V, Nmax, splits;
  float temp;
  uint64_t seed;
  uint32_t offset;
  AccParts parts;
  float* rbuf;  // [batch][2][V] residual buffers (T > 0)
  int32_t* acc_nodes;
  int32_t* n_acc;
  int32_t* bonus;
  int32_t* status;
};

// T = 0 in one launch: grid (splits, batch * (Nmax + 1)); each CTA the argmax
// of one chunk of one target row; the last CTA of a request to finish walks
// its tree: one warp per row merges the row's split partials, then one warp
// follows the argmax tokens down the tree in shared memory.  counters [batch]
// start at zero and are left at zero.
__global__ void __launch_bounds__(kPreThreads)
    accept_greedy_kernel(WalkArgs w, int32_t* counters) {
  const int row_g = blockIdx.y;
  const int b = row_g / (w.Nmax + 1), row = row_g % (w.Nmax + 1);
  const int n_raw = w.n_nodes[b];
  const int n = min(max(n_raw, 0), w.Nmax);
  if (row > n) return;  // uniform; rows past the tree are not counted
  prepass_chunk<false>(w.t, w.tbf16, row_g, w.V, w.splits, 0.f, w.parts);
  __shared__ int s_last;
  __shared__ int32_t s_tok[64], s_par[64], s_arg[65];
  if (threadIdx.x == 0) {
    __threadfence();  // this CTA's partial before its arrival
    const int total = w.splits * (n + 1);
    s_last = atomicAdd(&counters[b], 1) == total - 1;
    if (s_last) counters[b] = 0;  // every CTA of the request has arrived
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0 && (n_raw < 0 || n_raw > w.Nmax)) set_status(w.status, DT_EDEVICE);
  for (int r = warp; r <= n; r += kPreThreads / 32) {
    const size_t rg = (size_t)b * (w.Nmax + 1) + r;
    float best = -INFINITY;
    int32_t bi = 0x7fffffff;
    for (int s = lane; s < w.splits; s += 32) {
      const float v = __ldcg(w.parts.pv + rg * w.splits + s);
      const int32_t id = __ldcg(w.parts.pi + rg * w.splits + s);
      if (v > best || (v == best && id < bi)) {
        best = v;
        bi = id;
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, best, o);
      const int32_t oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > best || (ov == best && oi < bi)) {
        best = ov;
        bi = oi;
      }
    }
    if (lane == 0) s_arg[r] = bi;
  }
  for (int i = threadIdx.x; i < n; i += kPreThreads) {
    s_tok[i] = w.tokens[(size_t)b * w.Nmax + i];
    s_par[i] = w.parents[(size_t)b * w.Nmax + i];
  }
  __syncthreads();
  if (warp != 0) return;
  int node = -1, nacc = 0;
  int32_t a = 0;
  while (true) {
    a = s_arg[node + 1];
    // children of `node` carry distinct tokens: at most one matches
    int next = -1;
    for (int i0 = 0; i0 < n; i0 += 32) {
      const int i = i0 + lane;
      const bool m = i < n && s_par[i] == node && s_tok[i] == a;
      const unsigned bal = __ballot_sync(0xffffffffu, m);
      if (bal && next < 0) next = i0 + __ffs(bal) - 1;
    }
    if (next < 0 || nacc >= w.Bk) break;
    if (lane == 0) w.acc_nodes[(size_t)b * w.Bk + nacc] = next;
    ++nacc;
    node = next;
  }
  for (int i = nacc + lane; i < w.Bk; i += 32) w.acc_nodes[(size_t)b * w.Bk + i] = -1;
  if (lane == 0) {
    w.n_acc[b] = nacc;
    w.bonus[b] = a;
  }
}

// Stochastic walk, one thread-block cluster per request.  The C CTAs of the
// cluster own consecutive slices of the vocabulary; a residual pass or the
// bonus race runs over all slices at once, and its sums (or arg-max) are
// combined through distributed shared memory in a fixed order, so every CTA
// of the cluster holds the same totals and takes the same decisions.  A
// child's p(x) and q(x) are read from global memory by every CTA (the
// residual written by the slice's owner is visible after the cluster barrier
// of the reduction that followed it).
struct __align__(8) WalkPart {
  float a, b;
};

// Totals of (a, b) over the cluster, identical in every thread of every CTA:
// warp sums, the CTA's sum over its warps (warp 0), then the CTAs' values
// combined by one fixed shuffle tree.  `slot` alternates between consecutive
// calls, so a slot of red2 or xs is rewritten only after a later barrier has
// ordered every read of it.
__device__ __forceinline__ WalkPart cluster_sum2(cg::cluster_group& cl, float a, float b,
                                                 WalkPart* xs, int slot, WalkPart (*red2)[32],
                                                 WalkPart* bcast) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  a = warp_sum(a);
  b = warp_sum(b);
  if (lane == 0) red2[slot][warp] = WalkPart{a, b};
  __syncthreads();
  if (warp == 0) {
    WalkPart v = lane < kWalkThreads / 32 ? red2[slot][lane] : WalkPart{0.f, 0.f};
    v.a = warp_sum(v.a);
    v.b = warp_sum(v.b);
    if (lane == 0) xs[slot] = v;
  }
  cl.sync();
  if (warp == 0) {
    WalkPart v{0.f, 0.f};
    if (lane < (int)cl.num_blocks()) v = *cl.map_shared_rank(&xs[slot], lane);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      v.a += __shfl_xor_sync(0xffffffffu, v.a, o);
      v.b += __shfl_xor_sync(0xffffffffu, v.b, o);
    }
    if (lane == 0) *bcast = v;
  }
  __syncthreads();
  return *bcast;
}

__global__ void __launch_bounds__(kWalkThreads) stoch_walk_kernel(WalkArgs w) {
  cg::cluster_group cl = cg::this_cluster();
  const int C = (int)cl.num_blocks(), rank = (int)cl.block_rank();
  const int b = blockIdx.x / C;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __shared__ float red[32];
  __shared__ int32_t redi[32];
  __shared__ int32_t s_removed[64];  // tokens of the rejected siblings, in order
  __shared__ int32_t s_tok[64], s_par[64], s_rank[64];
  // per target row r (0 = root, r = node r - 1): log-sum-exp of t_r / T, the
  // node's children in rank order, and the first child if its coin accepts
  __shared__ float s_lse_row[65];
  __shared__ int8_t s_kid[65][64];
  __shared__ int s_nkid[65];
  __shared__ int s_first_acc[65];
  __shared__ WalkPart xs[2], bcast;
  __shared__ WalkPart red2[2][32];
  __shared__ float x_best;
  __shared__ int32_t x_bid;
  int n = w.n_nodes[b];
  if (n < 0 || n > w.Nmax) {
    if (tid == 0 && rank == 0) set_status(w.status, DT_EDEVICE);
    n = n < 0 ? 0 : w.Nmax;
  }
  const int V = w.V;
  for (int i = tid; i < n; i += kWalkThreads) {
    int tok = w.tokens[(size_t)b * w.Nmax + i];
    if (tok < 0 || tok >= V) {  // range check: the walk indexes rows by token
      if (rank == 0) set_status(w.status, DT_EDEVICE);
      tok = 0;
    }
    s_tok[i] = tok;
    s_par[i] = w.parents[(size_t)b * w.Nmax + i];
    s_rank[i] = w.ranks[(size_t)b * w.Nmax + i];
  }
  for (int r0 = tid; r0 <= n; r0 += kWalkThreads) s_nkid[r0] = 0;
  __syncthreads();
  // Everything the walk needs per node that does not depend on the path
  // taken, for all rows at once: the rows' log-sum-exp (one warp per row,
  // from the pre-pass's split partials), the children in rank order (ties
  // to the lower index, as a stable sort gives), and the coin of each
  // node's first child, which meets p and q before any residual.
  for (int r0 = warp; r0 <= n; r0 += kWalkThreads / 32) {
    const size_t rg = (size_t)b * (w.Nmax + 1) + r0;
    float m2 = -INFINITY;
    for (int s = lane; s < w.splits; s += 32) m2 = fmaxf(m2, w.parts.pv[rg * w.splits + s]);
    m2 = warp_max(m2);
    float s2 = 0.f;
    for (int s = lane; s < w.splits; s += 32) {
      const float mv = w.parts.pv[rg * w.splits + s];
      if (mv != -INFINITY) s2 += w.parts.ps[rg * w.splits + s] * exp2f((mv - m2) * kL2e);
    }
    s2 = warp_sum(s2);
    if (lane == 0) s_lse_row[r0] = m2 + logf(s2);
  }
  for (int c = tid; c < n; c += kWalkThreads) {
    const int p = s_par[c];
    if (p < -1 || p >= n) continue;  // a child of no node the walk can visit
    int pos = 0;
    for (int j = 0; j < n; ++j)
      pos += (s_par[j] == p && (s_rank[j] < s_rank[c] || (s_rank[j] == s_rank[c] && j < c))) ? 1
                                                                                            : 0;
    s_kid[p + 1][pos] = (int8_t)c;
    atomicAdd(&s_nkid[p + 1], 1);
  }
  __syncthreads();
  const float temp = w.temp;
  for (int r0 = tid; r0 <= n; r0 += kWalkThreads) {
    int acc = -1;
    if (s_nkid[r0] > 0) {
      const int c = s_kid[r0][0];
      const int x = s_tok[c];
      const size_t rg = (size_t)b * (w.Nmax + 1) + r0;
      const float px = expf(__fdiv_rn(ld_logit(w.t, w.tbf16, rg * V + x), temp) - s_lse_row[r0]);
      const float qx = w.draft_q[rg * V + x] / 1.f;
      const float u = philox_uniform(w.seed, w.offset, 1u, (uint32_t)b, (uint32_t)c, 0u, 0u);
      if (u < px / qx) acc = c;
    }
    s_first_acc[r0] = acc;
  }
  __syncthreads();
  // Vector mode: rows of a multiple of 4 tokens on 16-byte boundaries, read
  // and written four tokens per load; every slice starts on a multiple of 4.
  const bool vec = (V & 3) == 0 && ((uintptr_t)w.t & 15) == 0 && ((uintptr_t)w.draft_q & 15) == 0 &&
                   ((uintptr_t)w.rbuf & 15) == 0;
  const int sh = vec ? 2 : 0;  // log2 of the tokens a thread reads at once
  const int chunk = vec ? ((V + 4 * C - 1) / (4 * C)) * 4 : (V + C - 1) / C;
  const int v0 = min(V, rank * chunk), v1 = min(V, v0 + chunk);  // this CTA's slice
  float* rb[2] = {w.rbuf + (size_t)b * 2 * V, w.rbuf + (size_t)b * 2 * V + V};
  int node = -1, nacc = 0, slot = 0;
  int32_t bonus = 0;
  // Residual buffer holding p (unnormalised) while `resid`.  It carries over
  // from node to node: a node's first pass writes the other buffer, so it
  // never overwrites what a slower CTA may still read for the previous
  // node's last coin (the pass after it follows a cluster barrier).
  int cur = 0;
  while (true) {
    const int row = node + 1;
    const size_t rg = (size_t)b * (w.Nmax + 1) + row;
    const float lse_t = s_lse_row[row];
    const int nk = s_nkid[row];
    const size_t tbase = rg * V;
    const float* q = w.draft_q + rg * V;
    bool resid = false;  // p is softmax(t / T) until the first effective residual
    float zr = 1.f;      // normaliser of the residual
    float qn = 1.f;      // sum of q over the tokens not yet removed
    // The removed set is the sibling being rejected (xr) and the first
    // n_removed entries of s_removed, the siblings rejected before it (fewer
    // than nk, and a node has fewer than Nmax <= 64 children).  A pass looks
    // up the removed tokens that fall in this thread's groups of the slice
    // (group g = (y - v0) >> sh belongs to thread g % kWalkThreads) only when
    // it reaches the previous one, and meets them in ascending order as y
    // advances.
    int n_removed = 0;
    auto next_owned = [&](int after, int xr) {
      auto mine = [&](int t) {
        return t > after && t >= v0 && t < v1 && ((t - v0) >> sh) % kWalkThreads == tid;
      };
      int best = mine(xr) ? xr : 0x7fffffff;
      for (int i = 0; i < n_removed; ++i) {
        const int t = s_removed[i];
        if (mine(t)) best = min(best, t);
      }
      return best;
    };
    int acc = -1;
    for (int ci = 0; ci < nk; ++ci) {
      const int c = s_kid[row][ci];
      const int x = s_tok[c];
      bool take;
      if (ci == 0) {
        take = s_first_acc[row] >= 0;
      } else {
        const float px = resid ? __ldcg(rb[cur] + x) / zr
                               : expf(__fdiv_rn(ld_logit(w.t, w.tbf16, tbase + x), temp) - lse_t);
        const float qx = q[x] / qn;
        const float u = philox_uniform(w.seed, w.offset, 1u, (uint32_t)b, (uint32_t)c, 0u, 0u);
        take = u < px / qx;
      }
      if (take) {
        acc = c;
        break;  // uniform over the cluster: every thread computed the same values
      }
      // residual pass over this CTA's slice: r'(y) = max(p(y) - q_j(y), 0),
      // q_j = q without the tokens removed before x, over the normaliser qn
      float* dst = rb[cur ^ 1];
      float zsum = 0.f, qsum = 0.f;
      int nxt = next_owned(-1, x);
      // one token: p(y), then r'(y) = max(p(y) - q_j(y), 0) with q_j(y) = 0
      // for tokens removed before x, over the normaliser qn
      auto resid_one = [&](int y, float praw, float qv) {
        const float py = resid ? praw / zr : expf(__fdiv_rn(praw, temp) - lse_t);
        const bool rm = (y == nxt);
        if (rm) nxt = next_owned(y, x);
        const float rv = fmaxf(py - (rm && y != x ? 0.f : qv) / qn, 0.f);
        zsum += rv;
        if (!rm) qsum += qv;
        return rv;
      };
      if (vec) {
        constexpr int kU = 2;  // groups of 4 tokens in flight per thread
        const int g1 = v1 >> 2;
        for (int g = (v0 >> 2) + tid; g < g1; g += kU * kWalkThreads) {
          float pr[kU][4], qr[kU][4];
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            const int gg = g + u * kWalkThreads;
            if (gg < g1) {
              if (resid) {
                const float4 f = __ldcg((const float4*)rb[cur] + gg);
                pr[u][0] = f.x, pr[u][1] = f.y, pr[u][2] = f.z, pr[u][3] = f.w;
              } else {
                ld_logit4(w.t, w.tbf16, tbase + 4 * (size_t)gg, pr[u]);
              }
              const float4 f = __ldg((const float4*)q + gg);
              qr[u][0] = f.x, qr[u][1] = f.y, qr[u][2] = f.z, qr[u][3] = f.w;
            }
          }
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            const int gg = g + u * kWalkThreads;
            if (gg < g1) {
              float4 o;
              o.x = resid_one(4 * gg, pr[u][0], qr[u][0]);
              o.y = resid_one(4 * gg + 1, pr[u][1], qr[u][1]);
              o.z = resid_one(4 * gg + 2, pr[u][2], qr[u][2]);
              o.w = resid_one(4 * gg + 3, pr[u][3], qr[u][3]);
              __stcg((float4*)dst + gg, o);
            }
          }
        }
      } else {
        for (int y = v0 + tid; y < v1; y += kWalkThreads)
          dst[y] = resid_one(y, resid ? rb[cur][y] : ld_logit(w.t, w.tbf16, tbase + y), q[y]);
      }
      // x joins the removed set for the next pass: no thread reads this entry
      // before the barriers of the reduction below
      if (tid == 0) s_removed[n_removed] = x;
      ++n_removed;
      const WalkPart tot = cluster_sum2(cl, zsum, qsum, xs, slot, red2, &bcast);
      slot ^= 1;
      if (tot.a > 0.f) {
        cur ^= 1;
        zr = tot.a;
        resid = true;
      }
      qn = tot.b;
    }
    if (acc >= 0 && nacc < w.Bk) {
      if (tid == 0 && rank == 0) w.acc_nodes[(size_t)b * w.Bk + nacc] = acc;
      ++nacc;
      node = acc;
      continue;
    }
    // bonus: exponential race argmax_y p(y) / E_y over every slice
    float best = -INFINITY;
    int32_t bid = 0x7fffffff;
    // one token: its race score p(y) / E_y, E_y = -log U_y
    auto race_one = [&](int y, float praw, float u) {
      const float py = resid ? praw / zr : expf(__fdiv_rn(praw, temp) - lse_t);
      const float sc = py / (-logf(u));
      if (sc > best) {
        best = sc;
        bid = y;
      }
    };
    if (vec) {
      // the four tokens of a group share one Philox block (word y & 3)
      const int g1 = v1 >> 2;
      const uint32_t key0 = (uint32_t)w.seed, key1 = (uint32_t)(w.seed >> 32);
      for (int g = (v0 >> 2) + tid; g < g1; g += kWalkThreads) {
        float pr[4];
        if (resid) {
          const float4 f = __ldcg((const float4*)rb[cur] + g);
          pr[0] = f.x, pr[1] = f.y, pr[2] = f.z, pr[3] = f.w;
        } else {
          ld_logit4(w.t, w.tbf16, tbase + 4 * (size_t)g, pr);
        }
        const U4 o = philox10(U4{(uint32_t)g | ((uint32_t)b << 18) | (2u << 28),
                                 (uint32_t)(node + 1), 0u, w.offset},
                              key0, key1);
        race_one(4 * g, pr[0], u23(o.x));
        race_one(4 * g + 1, pr[1], u23(o.y));
        race_one(4 * g + 2, pr[2], u23(o.z));
        race_one(4 * g + 3, pr[3], u23(o.w));
      }
    } else {
      for (int y = v0 + tid; y < v1; y += kWalkThreads)
        race_one(y, resid ? rb[cur][y] : ld_logit(w.t, w.tbf16, tbase + y),
                 philox_uniform(w.seed, w.offset, 2u, (uint32_t)b, (uint32_t)(node + 1), 0u,
                                (uint32_t)y));
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, best, o);
      const int32_t oi = __shfl_xor_sync(0xffffffffu, bid, o);
      if (ov > best || (ov == best && oi < bid)) {
        best = ov;
        bid = oi;
      }
    }
    if (lane == 0) {
      red[warp] = best;
      redi[warp] = bid;
    }
    __syncthreads();
    if (tid == 0) {
      for (int i = 1; i < kWalkThreads / 32; ++i)
        if (red[i] > best || (red[i] == best && redi[i] < bid)) {
          best = red[i];
          bid = redi[i];
        }
      x_best = best;
      x_bid = bid;
    }
    cl.sync();
    if (tid < 32) {
      float vb = -INFINITY;
      int32_t vi = 0x7fffffff;
      if (lane < C) {
        vb = *cl.map_shared_rank(&x_best, lane);
        vi = *cl.map_shared_rank(&x_bid, lane);
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, vb, o);
        const int32_t oi = __shfl_xor_sync(0xffffffffu, vi, o);
        if (ov > vb || (ov == vb && oi < vi)) {
          vb = ov;
          vi = oi;
        }
      }
      bonus = vi;
    }
    break;
  }
  if (tid == 0 && rank == 0) {
    for (int i = nacc; i < w.Bk; ++i) w.acc_nodes[(size_t)b * w.Bk + i] = -1;
    w.n_acc[b] = nacc;
    w.bonus[b] = bonus;
  }
  // no CTA leaves while a peer may still read its shared memory
  cl.sync();
}

}  // namespace dt

using namespace dt;

namespace {
int accept_splits(int rows_total, int V) {
  const int want = (4 * 148 + rows_total - 1) / rows_total;
  const int most = (V + 2047) / 2048;
  return std::max(1, std::min(want, most));
}
size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
}  // namespace

extern "C" {

size_t dt_tree_accept_workspace_bytes(int batch, int Nmax, int V) {
  if (batch <= 0 || Nmax <= 0 || V <= 0) return 0;
  const int rows = batch * (Nmax + 1);
  const int sp = accept_splits(rows, V);
  size_t b = kWsHeader + align256((size_t)batch * 4);  // status word, T = 0 arrival counters
  b += align256((size_t)rows * sp * 4) * 3;
  b += align256((size_t)batch * 2 * V * 4);
  return b;
}

dt_status dt_tree_accept(const void* d_target_logits, dt_dtype tdt, const dt_tree* tree,
                         int batch, int Bk, int V, int Nmax, float temp, uint64_t philox_seed,
                         uint64_t philox_offset, int32_t* d_acc_nodes, int32_t* d_n_acc,
                         int32_t* d_bonus, void* ws, size_t ws_bytes, dt_stream stream) {
  if (!d_target_logits || !tree || !d_acc_nodes || !d_n_acc || !d_bonus) return DT_EINVAL;
  if (!tree->d_tokens || !tree->d_parents || !tree->d_ranks || !tree->d_n_nodes) return DT_EINVAL;
  if (tdt != DT_F32 && tdt != DT_BF16) return DT_EINVAL;
  if (batch < 1 || Bk < 1 || V < 1 || Nmax < 1 || !(temp >= 0.f)) return DT_EINVAL;
  if (philox_offset >= (1ull << 32)) return DT_EINVAL;
  if (temp > 0.f && !tree->d_draft_q) return DT_EINVAL;
  if (batch > 1024 || Bk > 16 || Nmax > 64 || V >= (1 << 20)) return DT_EUNSUPPORTED;
  const size_t need = dt_tree_accept_workspace_bytes(batch, Nmax, V);
  if (!ws || ws_bytes < need) return DT_EWORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  const int rows = batch * (Nmax + 1);
  const int sp = accept_splits(rows, V);
  uint8_t* p = (uint8_t*)ws;
  int32_t* status = (int32_t*)p;
  p += kWsHeader;
  int32_t* counters = (int32_t*)p;
  p += align256((size_t)batch * 4);
  AccParts parts;
  parts.pv = (float*)p;
  p += align256((size_t)rows * sp * 4);
  parts.pi = (int32_t*)p;
  p += align256((size_t)rows * sp * 4);
  parts.ps = (float*)p;
  p += align256((size_t)rows * sp * 4);
  float* rbuf = (float*)p;
  // the status word and the arrival counters, which sit right after it
  if (cudaMemsetAsync(status, 0, kWsHeader + (size_t)batch * 4, s) != cudaSuccess) return DT_ECUDA;
  dim3 grid(sp, rows);
  const int tb = tdt == DT_BF16;
  if (temp > 0.f) {
    ProfileScope ps(DT_K_ACCEPT_PREPASS, s);
    accept_prepass_kernel<true><<<grid, kPreThreads, 0, s>>>(d_target_logits, tb, tree->d_n_nodes,
                                                             Nmax, V, sp, temp, parts);
    if (cudaGetLastError() != cudaSuccess) return DT_ECUDA;
  }
  WalkArgs w;
  w.t = d_target_logits;
  w.tbf16 = tb;
  w.tokens = tree->d_tokens;
  w.parents = tree->d_parents;
  w.ranks = tree->d_ranks;
  w.n_nodes = tree->d_n_nodes;
  w.draft_q = tree->d_draft_q;
  w.Bk = Bk;
  w.V = V;
  w.Nmax = Nmax;
  w.splits = sp;
  w.temp = temp;
  w.seed = philox_seed;
  w.offset = (uint32_t)philox_offset;
  w.parts = parts;
  w.rbuf = rbuf;
  w.acc_nodes = d_acc_nodes;
  w.n_acc = d_n_acc;
  w.bonus = d_bonus;
  w.status = status;
  ProfileScope ps(DT_K_ACCEPT_WALK, s);
  if (temp > 0.f) {
    // one cluster of C CTAs per request: as many as keep every request's
    // cluster resident at once (one 1024-thread CTA per SM), at most 8
    int C = 8;
    while (C > 1 && (long long)batch * C > num_sms()) C >>= 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(batch * C);
    cfg.blockDim = dim3(kWalkThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, stoch_walk_kernel, w) != cudaSuccess) return DT_ECUDA;
  } else {
    // pre-pass and walk in one launch
    accept_greedy_kernel<<<grid, kPreThreads, 0, s>>>(w, counters);
  }
  if (cudaGetLastError() != cudaSuccess) return DT_ECUDA;
  return DT_OK;
}

}  // extern "C"
