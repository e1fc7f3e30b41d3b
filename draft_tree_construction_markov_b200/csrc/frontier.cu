// Best-first frontier of the draft tree, one CTA per request.
//
// Sources: TreeSpark article, "core idea" (path survival drives best-first
// expansion and per-round stopping); PCTree summary, "k=4, N=32" paragraph
// (budget N, k children per node).
//
// Exact level-synchronous schedule.  Sequential best-first pops nodes in the
// total order (key desc, depth asc, parent index asc, rank asc); a child never
// ranks above its parent.  The wave schedule keeps the top-N of all candidates
// known so far, expands every kept node that is not yet expanded (and has depth
// < Bk), and repeats until no kept node is waiting.  Any unknown node has a
// kept-but-unexpanded ancestor ranking above it, so when nothing waits the
// kept set is the sequential result; and a node outside the top-N of a subset
// of candidates is outside the top-N of any superset, so at most Bk waves run.
#include "build.cuh"

namespace dt {

constexpr int kFrontierThreads = 1024;
constexpr float kLog2eF = 1.4426950408889634f;

__device__ __forceinline__ uint64_t sort_key(const Cand& c, int idx) {
  const uint32_t hi = ~f32_ordered(c.key);
  const uint32_t lo = ((uint32_t)c.depth << 27) | ((uint32_t)(c.parent_pos & 127) << 20) |
                      ((uint32_t)(c.rank & 15) << 16) | (uint32_t)idx;
  return ((uint64_t)hi << 32) | lo;
}

__device__ __forceinline__ void gather_row(uint16_t* dst, const uint16_t* A, int token, int r,
                                           int lane, int nlanes) {
  const uint4* s = (const uint4*)(A + (size_t)token * r);
  uint4* d = (uint4*)dst;
  for (int i = lane; i < r / 8; i += nlanes) d[i] = s[i];
}

// Best remaining entry of a lane's partial lists (val desc, id asc), strictly
// after (pv, pi) in that order.
__device__ __forceinline__ void warp_best(float& v, int32_t& id) {
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, v, o);
    const int32_t oi = __shfl_xor_sync(0xffffffffu, id, o);
    if (ov > v || (ov == v && oi < id)) {
      v = ov;
      id = oi;
    }
  }
}

// Exact fallback: kb rounds, each picks the best entry ranked strictly after
// the previous pick (used only when ties overflow the candidate buffer).
__device__ void merge_topk_slow(const float* lv, const int32_t* li, int ncta, size_t Mcap, int row,
                                int k, int kb, float* out_v, int32_t* out_i) {
  const int lane = threadIdx.x & 31;
  float pv = INFINITY;
  int32_t pi = -1;
  for (int j = 0; j < kb; ++j) {
    float bv = -INFINITY;
    int32_t bi = 0x7fffffff;
    for (int c = lane; c < ncta; c += 32) {
      const size_t base = ((size_t)c * Mcap + row) * k;
      for (int i = 0; i < k; ++i) {
        const float v = lv[base + i];
        const int32_t id = li[base + i];
        const bool after = v < pv || (v == pv && id > pi);
        if (!after) continue;
        if (v > bv || (v == bv && id < bi)) {
          bv = v;
          bi = id;
        }
        break;  // lists are sorted: the first entry after the pick is this list's best
      }
    }
    warp_best(bv, bi);
    pv = bv;
    pi = bi;
    if (lane == 0) {
      out_v[j] = bv;
      out_i[j] = bi;
    }
  }
}

constexpr int kMergeCap = 128;  // candidates per warp that survive the threshold

// Top-kb over the per-CTA sorted top-k lists of one row, by one warp.
// Threshold: the largest kb-th value of any single list; every member of the
// global top-kb is >= it (that list alone holds kb values >= it), and usually
// only a handful of entries pass.  buf: kMergeCap (value, id) pairs of smem.
__device__ void merge_topk(const float* lv, const int32_t* li, int ncta, size_t Mcap, int row,
                           int k, int kb, float* out_v, int32_t* out_i, float* bv_s,
                           int32_t* bi_s, int* bcount) {
  const int lane = threadIdx.x & 31;
  float tau = -INFINITY;
  for (int c = lane; c < ncta; c += 32) tau = fmaxf(tau, lv[((size_t)c * Mcap + row) * k + kb - 1]);
  tau = warp_max(tau);
  if (lane == 0) *bcount = 0;
  __syncwarp();
  for (int c = lane; c < ncta; c += 32) {
    const size_t base = ((size_t)c * Mcap + row) * k;
    for (int i = 0; i < k; ++i) {
      const float v = lv[base + i];
      if (!(v >= tau)) break;  // sorted descending
      const int slot = atomicAdd(bcount, 1);
      if (slot < kMergeCap) {
        bv_s[slot] = v;
        bi_s[slot] = li[base + i];
      }
    }
  }
  __syncwarp();
  const int nb = *bcount;
  if (nb > kMergeCap) {
    merge_topk_slow(lv, li, ncta, Mcap, row, k, kb, out_v, out_i);
    return;
  }
  // kb rounds of a warp argmax over the buffer (at most 4 entries per lane)
  float ev[kMergeCap / 32];
  int32_t ei[kMergeCap / 32];
#pragma unroll
  for (int t = 0; t < kMergeCap / 32; ++t) {
    const int sidx = lane + 32 * t;
    ev[t] = sidx < nb ? bv_s[sidx] : -INFINITY;
    ei[t] = sidx < nb ? bi_s[sidx] : 0x7fffffff;
  }
  for (int j = 0; j < kb; ++j) {
    int bt = 0;
#pragma unroll
    for (int t = 1; t < kMergeCap / 32; ++t)
      if (ev[t] > ev[bt] || (ev[t] == ev[bt] && ei[t] < ei[bt])) bt = t;
    float wv = ev[0];
    int32_t wi = ei[0];
#pragma unroll
    for (int t = 1; t < kMergeCap / 32; ++t)
      if (t == bt) {
        wv = ev[t];
        wi = ei[t];
      }
    const float mv = wv;
    const int32_t mi = wi;
    warp_best(wv, wi);
#pragma unroll
    for (int t = 0; t < kMergeCap / 32; ++t)
      if (t == bt && mv == wv && mi == wi) {
        ev[t] = -INFINITY;
        ei[t] = 0x7fffffff;
      }
    if (lane == 0) {
      out_v[j] = wv;
      out_i[j] = wi;
    }
  }
  __syncwarp();
}

__global__ void __launch_bounds__(kFrontierThreads) frontier_kernel(FrontierArgs f) {
  extern __shared__ __align__(16) uint8_t fsm[];
  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int kWarps = kFrontierThreads / 32;
  __shared__ ReqState st;
  __shared__ int s_n_keep, s_n_next, s_next_base, s_mat_base;
  __shared__ float s_thr;
  __shared__ int s_kb, s_nb;
  __shared__ uint64_t s_anc[64];
  __shared__ int32_t s_par[64];
  __shared__ float s_mv[kFrontierThreads / 32][kMergeCap];
  __shared__ int32_t s_mi[kFrontierThreads / 32][kMergeCap];
  __shared__ int s_mc[kFrontierThreads / 32];
  if (tid == 0) {
    st = f.req[b];
    int kb = f.k_req ? f.k_req[b] : f.k;
    if (kb < 1 || kb > f.k) {
      set_status(f.status, DT_EDEVICE);
      kb = kb < 1 ? 1 : f.k;
    }
    int nb = f.n_budget[b];
    if (nb < 0 || nb > f.Nmax) {
      set_status(f.status, DT_EDEVICE);
      nb = nb < 0 ? 0 : f.Nmax;
    }
    s_kb = kb;
    s_nb = nb;
    const float lam = f.lambda[b];
    s_thr = (lam > 0.f) ? (float)log((double)lam) : -INFINITY;
  }
  __syncthreads();
  if (st.done) return;
  const int kb = s_kb, k = f.k, Nmax = f.Nmax;
  const int rows_n = st.row_count;
  const int n_old = st.n_list;
  const int cap = Nmax + Nmax * k;  // list + children of at most Nmax expanded nodes
  Cand* cands = (Cand*)fsm;                                   // [cap]
  Cand* sorted = cands + cap;                                 // [Nmax]
  uint64_t* keys = (uint64_t*)(sorted + Nmax);                // [cap]
  float* r_lse = (float*)(keys + cap);                        // [Nmax]
  float* r_lq = r_lse + Nmax;                                 // [Nmax][k]
  int32_t* r_tok = (int32_t*)(r_lq + Nmax * k);               // [Nmax][k]
  float* r_sv = (float*)(r_tok + Nmax * k);                   // scratch [Nmax][k]
  int32_t* r_si = (int32_t*)(r_sv + Nmax * k);                // scratch [Nmax][k]

  for (int i = tid; i < n_old; i += kFrontierThreads) cands[i] = f.lists[(size_t)b * Nmax + i];

  // 1. merge the per-CTA partial results of each node expanded in this wave
  for (int e = warp; e < rows_n; e += kWarps) {
    const int row = st.row_base + e;
    float mx = -INFINITY;
    for (int c = lane; c < f.ncta_v; c += 32) mx = fmaxf(mx, f.stats[(size_t)c * f.Mcap + row].x);
    mx = warp_max(mx);
    float sv = 0.f;
    for (int c = lane; c < f.ncta_v; c += 32) {
      const float2 p = f.stats[(size_t)c * f.Mcap + row];
      if (p.x != -INFINITY) sv += p.y * exp2f((p.x - mx) * kLog2eF);
    }
    sv = warp_sum(sv);
    const float lse = mx + logf(sv);
    // order statistics of s (and, at T = 0, the children themselves)
    merge_topk(f.lv, f.li, f.ncta_v, f.Mcap, row, k, kb, r_sv + e * k, r_si + e * k, s_mv[warp],
               s_mi[warp], &s_mc[warp]);
    if (f.temp > 0.f)
      merge_topk(f.gv, f.gi, f.ncta_v, f.Mcap, row, k, kb, r_lq + e * k, r_tok + e * k,
                 s_mv[warp], s_mi[warp], &s_mc[warp]);
    __syncwarp();
    if (lane == 0) {
      r_lse[e] = lse;
      for (int j = 0; j < kb; ++j) {
        if (f.temp <= 0.f) r_tok[e * k + j] = r_si[e * k + j];
        r_lq[e * k + j] = r_sv[e * k + j] - lse;
      }
    }
  }
  __syncthreads();

  // 2. children of the expanded nodes become candidates
  const int n_new = rows_n * kb;
  for (int i = tid; i < n_new; i += kFrontierThreads) {
    const int e = i / kb, j = i % kb;
    const Row rw = f.rows[st.row_base + e];
    float pkey = 0.f;
    int ppos = 0;
    if (rw.aux >= 0) {
      for (int p = 0; p < n_old; ++p)
        if (cands[p].serial == rw.aux) {
          ppos = p + 1;
          pkey = cands[p].key;
          break;
        }
      if (ppos == 0) set_status(f.status, DT_EDEVICE);
    }
    const int d = rw.depth + 1;
    float al = 1.f, be = 0.f;
    if (f.calib) {
      al = f.calib[2 * (d - 1)];
      be = f.calib[2 * (d - 1) + 1];
    }
    const float c = fminf(0.f, fmaf(al, r_lq[e * k + j], be));
    Cand cd;
    cd.key = (pkey + c) + 0.0f;
    cd.token = r_tok[e * k + j];
    cd.serial = st.serial_next + i;
    cd.parent_serial = rw.aux;
    cd.path = (rw.path & ((1ull << 60) - 1)) | ((uint64_t)j << (4 * rw.depth)) |
              ((uint64_t)d << 60);
    cd.depth = (int16_t)d;
    cd.rank = (int8_t)j;
    cd.expanded = 0;
    cd.parent_pos = (int16_t)ppos;
    cd.pad0 = 0;
    cd.lse = 0.f;
    cands[n_old + i] = cd;
  }
  __syncthreads();
  // record the expanded nodes' log-sum-exp (root in the request state)
  if (tid < rows_n) {
    const Row rw = f.rows[st.row_base + tid];
    if (rw.aux < 0) {
      st.root_lse = r_lse[tid];
    } else {
      for (int p = 0; p < n_old; ++p)
        if (cands[p].serial == rw.aux) cands[p].lse = r_lse[tid];
    }
  }
  // 3. rank list + candidates by the total order (keys are unique: the low
  // bits hold the slot); keys below log(lambda) are dropped
  const int n_all = n_old + n_new;
  const float thr = s_thr;
  for (int i = tid; i < n_all; i += kFrontierThreads)
    keys[i] = (cands[i].key >= thr) ? sort_key(cands[i], i) : ~0ull;
  if (tid == 0) s_n_keep = 0;
  __syncthreads();
  for (int i = tid; i < n_all; i += kFrontierThreads) {
    const uint64_t ki = keys[i];
    if (ki == ~0ull) continue;
    int rank = 0;
    for (int j = 0; j < n_all; ++j) rank += keys[j] < ki;
    if (rank < s_nb) {
      sorted[rank] = cands[i];
      atomicAdd(&s_n_keep, 1);
    }
  }
  __syncthreads();
  const int n_keep = s_n_keep;

  // 4. schedule the next wave: kept nodes not yet expanded, depth < Bk
  if (tid == 0) {
    int m = 0;
    for (int i = 0; i < n_keep; ++i)
      if (!sorted[i].expanded && sorted[i].depth < f.Bk) ++m;
    s_n_next = m;
    s_next_base = m ? atomicAdd(f.next_count, m) : 0;
    if (m && s_next_base + m > f.Mcap) {
      set_status(f.status, DT_EDEVICE);
      s_n_next = 0;
    }
    st.serial_next += n_new;
  }
  __syncthreads();
  const int m_next = s_n_next;
  if (m_next > 0) {
    // rank among the waiting nodes -> row; one warp per row
    for (int i = warp; i < n_keep; i += kWarps) {
      const Cand c = sorted[i];
      if (c.expanded || c.depth >= f.Bk) continue;
      int before = 0;
      for (int p = 0; p < i; ++p) before += (!sorted[p].expanded && sorted[p].depth < f.Bk);
      const int row = s_next_base + before;
      if (lane == 0) {
        Row rw;
        rw.b = b;
        rw.depth = c.depth;
        rw.token = c.token;
        rw.aux = c.serial;
        rw.path = c.path;
        rw.lse = 0.f;
        rw.key = c.key;
        f.next_rows[row] = rw;
      }
      gather_row(f.H + (size_t)row * f.r, f.A, c.token, f.r, lane, 32);
    }
    __syncthreads();
    for (int i = tid; i < n_keep; i += kFrontierThreads)
      if (!sorted[i].expanded && sorted[i].depth < f.Bk) sorted[i].expanded = 1;
    __syncthreads();
    if (tid == 0) {
      st.row_base = s_next_base;
      st.row_count = m_next;
    }
  } else {
    // 5. the tree is final: emit it in pop order
    int32_t* tok = f.out.d_tokens + (size_t)b * Nmax;
    for (int i = tid; i < n_keep; i += kFrontierThreads) {
      const Cand c = sorted[i];
      int par = -1;
      if (c.parent_serial >= 0) {
        for (int p = 0; p < i; ++p)
          if (sorted[p].serial == c.parent_serial) par = p;
        if (par < 0) set_status(f.status, DT_EDEVICE);
      }
      s_par[i] = par;
      tok[i] = c.token;
      f.out.d_parents[(size_t)b * Nmax + i] = par;
      f.out.d_depths[(size_t)b * Nmax + i] = c.depth;
      f.out.d_ranks[(size_t)b * Nmax + i] = c.rank;
      f.out.d_keys[(size_t)b * Nmax + i] = c.key;
    }
    __syncthreads();
    if (tid == 0) {
      for (int i = 0; i < n_keep; ++i)
        s_anc[i] = (s_par[i] >= 0 ? s_anc[s_par[i]] : 0ull) | (1ull << i);
      f.out.d_n_nodes[b] = n_keep;
      st.done = 1;
      st.row_count = 0;
      if (f.temp > 0.f) {
        int m2 = 1;
        for (int i = 0; i < n_keep; ++i) m2 += (sorted[i].depth < f.Bk);
        s_mat_base = atomicAdd(f.mat_count, m2);
      }
    }
    __syncthreads();
    for (int i = tid; i < n_keep; i += kFrontierThreads)
      f.out.d_anc[(size_t)b * Nmax + i] = s_anc[i];
    if (f.temp > 0.f) {
      // rows whose draft distribution the accept walk needs: root + inner nodes
      for (int i = warp - 1; i < n_keep; i += kWarps) {
        int row, token, depth, aux;
        float lse;
        if (i < 0) {
          row = s_mat_base;
          token = st.pad[0];
          depth = 0;
          aux = 0;
          lse = st.root_lse;
        } else {
          const Cand c = sorted[i];
          if (c.depth >= f.Bk) continue;
          int before = 1;
          for (int p = 0; p < i; ++p) before += (sorted[p].depth < f.Bk);
          row = s_mat_base + before;
          token = c.token;
          depth = c.depth;
          aux = i + 1;
          lse = c.lse;
        }
        if (lane == 0) {
          Row rw;
          rw.b = b;
          rw.depth = depth;
          rw.token = token;
          rw.aux = aux;
          rw.path = 0;
          rw.lse = lse;
          rw.key = 0.f;
          f.mat_rows[row] = rw;
        }
        gather_row(f.Hm + (size_t)row * f.r, f.A, token, f.r, lane, 32);
      }
    }
  }
  // persist the kept list and the request state
  for (int i = tid; i < n_keep; i += kFrontierThreads) f.lists[(size_t)b * Nmax + i] = sorted[i];
  __syncthreads();
  if (tid == 0) {
    st.n_list = n_keep;
    f.req[b] = st;
  }
}

// Wave 1: every request with a non-empty budget expands its root.
__global__ void build_init_kernel(FrontierArgs f, const int32_t* root_token, Row* rows0,
                                  int32_t* count0) {
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  for (int b = blockIdx.x * wpb + (threadIdx.x >> 5); b < f.batch; b += gridDim.x * wpb) {
    ReqState st;
    st.n_list = 0;
    st.serial_next = 0;
    st.done = 0;
    st.row_base = b;
    st.row_count = 1;
    st.root_lse = 0.f;
    int root = root_token[b];
    if (root < 0 || root >= f.V) {
      if (lane == 0) set_status(f.status, DT_EDEVICE);
      root = 0;
    }
    st.pad[0] = root;
    st.pad[1] = 0;
    int nb = f.n_budget[b];
    Row rw;
    rw.b = b;
    rw.depth = 0;
    rw.token = root;
    rw.aux = -1;
    rw.path = 0;
    rw.lse = 0.f;
    rw.key = 0.f;
    if (nb <= 0) {
      rw.b = -1;
      st.done = 1;
      st.row_count = 0;
      if (lane == 0) f.out.d_n_nodes[b] = 0;
    } else {
      gather_row(f.H + (size_t)b * f.r, f.A, root, f.r, lane, 32);
    }
    if (lane == 0) {
      rows0[b] = rw;
      f.req[b] = st;
    }
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    *count0 = f.batch;
    *f.mat_count = 0;
  }
}

size_t frontier_smem_bytes(int Nmax, int k) {
  const int cap = Nmax + Nmax * k;
  return (size_t)cap * sizeof(Cand) + (size_t)Nmax * sizeof(Cand) + (size_t)cap * 8 +
         (size_t)Nmax * 4 + (size_t)Nmax * k * 4 * 4;
}

cudaError_t launch_frontier(const FrontierArgs& f, cudaStream_t s) {
  const size_t smem = frontier_smem_bytes(f.Nmax, f.k);
  cudaError_t e = ensure_smem(frontier_kernel, smem);
  if (e != cudaSuccess) return e;
  frontier_kernel<<<f.batch, kFrontierThreads, smem, s>>>(f);
  return cudaGetLastError();
}

cudaError_t launch_build_init(const FrontierArgs& f, const int32_t* root_token, Row* rows0,
                              int32_t* count0, cudaStream_t s) {
  build_init_kernel<<<(f.batch + 7) / 8, 256, 0, s>>>(f, root_token, rows0, count0);
  return cudaGetLastError();
}

}  // namespace dt
