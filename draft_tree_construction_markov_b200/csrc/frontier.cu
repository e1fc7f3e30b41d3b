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
#include "merge.cuh"

namespace dt {

constexpr int kFrontierThreads = 256;

__device__ __forceinline__ uint64_t sort_key(const Cand& c, int idx) {
  const uint32_t hi = ~f32_ordered(c.key);
  const uint32_t lo = ((uint32_t)c.depth << 27) | ((uint32_t)(c.parent_pos & 127) << 20) |
                      ((uint32_t)(c.rank & 15) << 16) | (uint32_t)idx;
  return ((uint64_t)hi << 32) | lo;
}

// Row A[token] of the Markov head (zeros for token -1) into H.
__device__ __forceinline__ void gather_row(uint16_t* dst, const uint16_t* A, int token, int r,
                                           int lane, int nlanes) {
  uint4* d = (uint4*)dst;
  if (token < 0) {
    for (int i = lane; i < r / 8; i += nlanes) d[i] = make_uint4(0, 0, 0, 0);
    return;
  }
  const uint4* s = (const uint4*)(A + (size_t)token * r);
  for (int i = lane; i < r / 8; i += nlanes) d[i] = s[i];
}

// Token whose Markov row conditions the children of a node of request b at
// depth d: the node's own token (the method), or the per-depth token of a
// baseline variant (-1 = block logits alone).
__device__ __forceinline__ int markov_token(const FrontierArgs& f, int b, int depth, int token) {
  return f.cond ? f.cond[(size_t)b * f.Bk + depth] : token;
}

template <int KMAX>
__global__ void __launch_bounds__(kFrontierThreads) frontier_kernel(FrontierArgs f) {
  extern __shared__ __align__(16) uint8_t fsm[];
  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int kWarps = kFrontierThreads / 32;
  __shared__ ReqState st;
  __shared__ Row s_rows[64];
  __shared__ int s_cnt[4];        // kept nodes, next-wave base, rows scheduled, q-row base
  __shared__ int16_t s_pos[64];   // position among the scheduled (or q-row) nodes, -1 if none
  __shared__ int32_t s_par[64];
  __shared__ float s_mv[kWarps][32];  // per-warp scratch of the partial merge
  __shared__ int32_t s_mi[kWarps][32];
  if (tid == 0) st = f.req[b];  // written by the previous frontier step (two kernels back)
  __syncthreads();
  if (st.done) {
    pdl_wait();
    pdl_launch_dependents();
    return;
  }
  const int kb = st.kb, k = f.k, Nmax = f.Nmax, Bk = f.Bk;
  const int rows_n = min(st.row_count, Nmax);
  const int n_old = st.n_list;
  const int cap = Nmax + Nmax * k;  // list + children of at most Nmax expanded nodes
  Cand* cands = (Cand*)fsm;                     // [cap]
  Cand* sorted = cands + cap;                   // [Nmax]
  uint64_t* keys = (uint64_t*)(sorted + Nmax);  // [cap]
  float* r_lse = (float*)(keys + cap);          // [Nmax]
  float* r_lq = r_lse + Nmax;                   // [Nmax][k]
  int32_t* r_tok = (int32_t*)(r_lq + Nmax * k); // [Nmax][k]
  for (int i = tid; i < n_old; i += kFrontierThreads) cands[i] = f.lists[(size_t)b * Nmax + i];
  for (int i = tid; i < rows_n; i += kFrontierThreads) s_rows[i] = f.rows[st.row_base + i];
  if (tid < 4) s_cnt[tid] = 0;
  // the per-CTA partials come from the wave GEMM launched just before
  pdl_wait();

  // 1. merge each expanded node's partials: its log-sum-exp and its kb best
  // (T = 0) or sampled (T > 0, Gumbel-top-k) children, one warp per node
  for (int e = warp; e < rows_n; e += kWarps) {
    const size_t prow = (size_t)(st.row_base + e) * f.ncta;
    // values of the k best (order statistics of s); tokens of the best (T = 0)
    // or of the Gumbel sample (T > 0)
    const bool stoch = f.temp > 0.f;
    const float lse = merge_node<KMAX>(f.pstats + prow, f.plv + prow * k, f.pli + prow * k,
                                       stoch ? f.pgv + prow * k : nullptr,
                                       stoch ? f.pgi + prow * k : nullptr, f.ncta, k, kb, lane,
                                       r_lq + e * k, stoch ? nullptr : r_tok + e * k,
                                       stoch ? r_tok + e * k : nullptr, s_mv[warp], s_mi[warp]);
    __syncwarp();
    if (lane == 0) r_lse[e] = lse;
    for (int j = lane; j < kb; j += 32) r_lq[e * k + j] -= lse;
  }
  __syncthreads();
  // Only now let the next wave's GEMM start: its weight stream saturates the
  // memory system, and the partial loads above would queue behind it.
  pdl_launch_dependents();

  // 2. the children become candidates, keyed by calibrated path survival
  const int n_new = rows_n * kb;
  for (int i = tid; i < n_new; i += kFrontierThreads) {
    const int e = i / kb, j = i % kb;
    const Row rw = s_rows[e];
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
  // the expanded nodes' log-sum-exp (the root's lives in the request state),
  // and every candidate's sort key; keys below log(lambda) are dropped
  const int n_all = n_old + n_new;
  if (tid < rows_n) {
    const Row rw = s_rows[tid];
    if (rw.aux < 0) {
      st.root_lse = r_lse[tid];
    } else {
      for (int p = 0; p < n_old; ++p)
        if (cands[p].serial == rw.aux) cands[p].lse = r_lse[tid];
    }
  }
  for (int i = tid; i < n_all; i += kFrontierThreads)
    keys[i] = (cands[i].key >= st.thr) ? sort_key(cands[i], i) : ~0ull;
  __syncthreads();

  // 3. rank by counting (keys are unique: the low bits hold the slot)
  for (int i = tid; i < n_all; i += kFrontierThreads) {
    const uint64_t ki = keys[i];
    if (ki == ~0ull) continue;
    int rank = 0;
    for (int j = 0; j < n_all; ++j) rank += keys[j] < ki;
    if (rank < st.nb) {
      sorted[rank] = cands[i];
      atomicAdd(&s_cnt[0], 1);
    }
  }
  __syncthreads();
  const int n_keep = s_cnt[0];

  // 4. nodes waiting for expansion (kept, not yet expanded, depth < B)
  if (warp == 0) {
    int prefix = 0;
    for (int c0 = 0; c0 < n_keep; c0 += 32) {
      const int i = c0 + lane;
      const bool wt = i < n_keep && !sorted[i].expanded && sorted[i].depth < Bk;
      const unsigned bal = __ballot_sync(0xffffffffu, wt);
      if (i < n_keep) s_pos[i] = wt ? (int16_t)(prefix + __popc(bal & ((1u << lane) - 1))) : -1;
      prefix += __popc(bal);
    }
    if (lane == 0) {
      // one request: its rows start at 0 of the list the GEMM just cleared
      int base = 0;
      if (prefix) {
        if (f.batch == 1)
          *f.next_count = prefix;
        else
          base = atomicAdd(f.next_count, prefix);
      }
      if (prefix && base + prefix > f.Mcap) {
        set_status(f.status, DT_EDEVICE);
        prefix = 0;
      }
      s_cnt[1] = base;
      s_cnt[2] = prefix;
    }
  }
  __syncthreads();
  const int m_next = s_cnt[2];
  if (m_next > 0) {
    const int base = s_cnt[1];
    for (int i = warp; i < n_keep; i += kWarps) {
      if (s_pos[i] < 0) continue;
      const Cand c = sorted[i];
      const int row = base + s_pos[i];
      if (lane == 0) {
        Row rw;
        rw.b = b;
        rw.depth = c.depth;
        rw.token = markov_token(f, b, c.depth, c.token);
        rw.aux = c.serial;
        rw.path = c.path;
        rw.lse = 0.f;
        rw.key = c.key;
        f.next_rows[row] = rw;
      }
      if (f.H) gather_row(f.H + (size_t)row * f.r, f.A, markov_token(f, b, c.depth, c.token), f.r,
                          lane, 32);
      __syncwarp();
      if (lane == 0) sorted[i].expanded = 1;
    }
    if (tid == 0) {
      st.serial_next += n_new;
      st.row_base = base;
      st.row_count = m_next;
    }
  } else {
    // 5. the tree is final: emit it in pop order
    for (int i = tid; i < n_keep; i += kFrontierThreads) {
      const Cand c = sorted[i];
      int par = -1;
      if (c.parent_serial >= 0) {
        for (int p = 0; p < i; ++p)
          if (sorted[p].serial == c.parent_serial) par = p;
        if (par < 0) set_status(f.status, DT_EDEVICE);
      }
      s_par[i] = par;
    }
    __syncthreads();
    const size_t ob = (size_t)b * Nmax;
    for (int i = tid; i < n_keep; i += kFrontierThreads) {
      const Cand c = sorted[i];
      uint64_t anc = 1ull << i;
      for (int p = s_par[i], hops = 0; p >= 0 && hops < 64; p = s_par[p], ++hops) anc |= 1ull << p;
      f.out.d_tokens[ob + i] = c.token;
      f.out.d_parents[ob + i] = s_par[i];
      f.out.d_depths[ob + i] = c.depth;
      f.out.d_ranks[ob + i] = c.rank;
      f.out.d_keys[ob + i] = c.key;
      f.out.d_anc[ob + i] = anc;
    }
    if (tid == 0) {
      f.out.d_n_nodes[b] = n_keep;
      st.done = 1;
      st.row_count = 0;
    }
    if (f.temp > 0.f) {
      // draft rows the accept walk needs: the root and every inner node
      if (warp == 0) {
        int prefix = 1;  // row 0 of the request's block is the root
        for (int c0 = 0; c0 < n_keep; c0 += 32) {
          const int i = c0 + lane;
          const bool in = i < n_keep && sorted[i].depth < Bk;
          const unsigned bal = __ballot_sync(0xffffffffu, in);
          if (i < n_keep) s_pos[i] = in ? (int16_t)(prefix + __popc(bal & ((1u << lane) - 1))) : -1;
          prefix += __popc(bal);
        }
        if (lane == 0) {
          if (f.batch == 1) {
            *f.mat_count = prefix;
            s_cnt[3] = 0;
          } else {
            s_cnt[3] = atomicAdd(f.mat_count, prefix);
          }
        }
      }
      __syncthreads();
      const int mbase = s_cnt[3];
      for (int i = warp - 1; i < n_keep; i += kWarps) {
        int token, depth, aux, pos;
        float lse;
        if (i < 0) {
          pos = 0;
          token = st.root_token;
          depth = 0;
          aux = 0;
          lse = st.root_lse;
        } else {
          if (s_pos[i] < 0) continue;
          const Cand c = sorted[i];
          pos = s_pos[i];
          token = c.token;
          depth = c.depth;
          aux = i + 1;
          lse = c.lse;
        }
        token = markov_token(f, b, depth, token);
        const int row = mbase + pos;
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
        if (f.Hm) gather_row(f.Hm + (size_t)row * f.r, f.A, token, f.r, lane, 32);
      }
    }
  }
  __syncthreads();
  // persist the kept list and the request state
  for (int i = tid; i < n_keep; i += kFrontierThreads) f.lists[(size_t)b * Nmax + i] = sorted[i];
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
    st.root_token = root;
    st.pad[0] = st.pad[1] = 0;
    int kb = f.k_req ? f.k_req[b] : f.k;
    if (kb < 1 || kb > f.k) {
      if (lane == 0) set_status(f.status, DT_EDEVICE);
      kb = kb < 1 ? 1 : f.k;
    }
    st.kb = kb;
    const float lam = f.lambda[b];
    st.thr = (lam > 0.f) ? (float)log((double)lam) : -INFINITY;
    int nb = f.n_budget[b];
    if (nb > f.Nmax) {
      if (lane == 0) set_status(f.status, DT_EDEVICE);
      nb = f.Nmax;
    }
    st.nb = nb < 0 ? 0 : nb;
    Row rw;
    rw.b = b;
    rw.depth = 0;
    rw.token = markov_token(f, b, 0, root);
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
      if (f.H) gather_row(f.H + (size_t)b * f.r, f.A, rw.token, f.r, lane, 32);
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
         (size_t)Nmax * 4 + (size_t)Nmax * k * 4 * 2;
}

int gemm_kmax(int k);

cudaError_t launch_frontier(const FrontierArgs& f, cudaStream_t s) {
  const size_t smem = frontier_smem_bytes(f.Nmax, f.k);
  auto kern = gemm_kmax(f.k) == 4 ? frontier_kernel<4> : frontier_kernel<16>;
  cudaError_t e = ensure_smem(kern, smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kern, dim3(f.batch), dim3(kFrontierThreads), smem, s, f);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_build_init(const FrontierArgs& f, const int32_t* root_token, Row* rows0,
                              int32_t* count0, cudaStream_t s) {
  build_init_kernel<<<(f.batch + 7) / 8, 256, 0, s>>>(f, root_token, rows0, count0);
  return cudaGetLastError();
}

}  // namespace dt
