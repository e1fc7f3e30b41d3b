// TreeFlash round: a SwiGLU AR-approximator over a one-shot drafter block,
// then a draft tree chosen from the approximator's distributions.
//
// Sources (TreeFlash explainer):
//  * method section 1: h'_i = h_i + SwiGLU(rmsnorm(h_i) :: rmsnorm(e_prev)),
//    where e_prev is the input embedding of the previous token; logits are
//    the LM head applied to h'.
//  * method section 2: stage 1 builds a top-M tree from the unmodified drafter
//    distributions, with exactly M unique tokens per depth (S_i = the M best
//    tokens of W_lm h_i); stage 2 evaluates the approximator on that tree's
//    nodes, at most M * gamma evaluations whatever the budget; the final tree
//    is chosen from the modified distributions.
// Readings (the explainer names OPT-Tree without defining it): the final
// tree is the best-first top-`budget` nodes by cumulative log q' under the
// same total order as the Markov tree (key desc, depth asc, parent index asc,
// rank asc); a node's candidates are the top-M tokens of its distribution; a
// node whose token is outside S_depth has no evaluated distribution and is a
// leaf.  RMSNorm uses eps = 1e-6 and its weight vector.  The approximator's
// activations are rounded to bf16 where they feed a GEMM (x, silu(g) * u,
// h'), which is where a bf16 network stores them.
//
// Device pipeline (one round, all requests of the batch at once):
//   1. LM head over the block rows h (node-batched GEMM, EXPAND epilogue
//      without bias) -> per-CTA top-M partials;  tf_merge -> S sets.
//   2. tf_prep: one row per evaluation (depth d, previous token t):
//      x = [rmsnorm(h_d) :: rmsnorm(E[t])] in bf16.
//   3. gate/up GEMM with the fused silu(g) * u epilogue (SWIGLU).
//   4. down GEMM + residual h_d (ZDUMP with the block rows as bias) -> h'.
//   5. LM head over h' (EXPAND) -> partials;  tf_merge -> log-sum-exp and
//      top-M of every evaluated distribution.
//   6. tf_select: best-first selection per request, tree arrays out.
#include <cstring>

#include "build.cuh"
#include "merge.cuh"

namespace dt {

bool make_tmap_bf16_kmajor(CUtensorMap* map, const void* base, uint64_t K, uint64_t rows,
                           uint32_t box_rows);
int gemm_node_tile(int max_cols);
int gemm_kmax(int k);
cudaError_t launch_markov_gemm(int mode, bool stoch, const CUtensorMap& tmW,
                               const CUtensorMap& tmW2, const CUtensorMap& tmH, GemmArgs a,
                               int batch, int nt, cudaStream_t s);
int num_sms();

namespace {

constexpr float kRmsEps = 1e-6f;

__device__ __forceinline__ uint16_t to_bf16(float f) {
  const uint32_t u = __float_as_uint(f);
  return (uint16_t)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

// Stage-1 rows (one per block position) and the row counters of both stages.
__global__ void tf_rows_kernel(Row* rows1, int n1, int gamma, int32_t* counts, int n2) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n1) {
    Row r;
    r.b = i / gamma;
    r.depth = i % gamma;
    r.token = 0;
    r.aux = i;
    r.path = 0;
    r.lse = 0.f;
    r.key = 0.f;
    rows1[i] = r;
  }
  if (i == 0) {
    counts[0] = n1;
    counts[1] = n2;
  }
}

// One warp per row: log-sum-exp and the M best (value, token) of the row's
// partials.  lse may be NULL.
template <int KMAX>
__global__ void tf_merge_kernel(const float2* pstats, const float* plv, const int32_t* pli,
                                int ncta, int n_rows, int M, float* lse, float* top_v,
                                int32_t* top_i) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= n_rows) return;
  const size_t prow = (size_t)row * ncta;
  if (lse) {
    const float l = merge_lse(pstats + prow, ncta, lane);
    if (lane == 0) lse[row] = l;
  }
  merge_lists<KMAX>(plv + prow * M, pli + prow * M, ncta, M, M, lane, top_v + (size_t)row * M,
                    top_i + (size_t)row * M);
}

// 1 / rms of a bf16 row of length D (a multiple of 64), one warp, 16-byte loads.
__device__ __forceinline__ float row_inv_rms(const uint16_t* x, int D, int lane) {
  float ss = 0.f;
  const uint4* v = (const uint4*)x;
  for (int i = lane; i < D / 8; i += 32) {
    const uint4 u = v[i];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float lo = __uint_as_float(w[h] << 16), hi = __uint_as_float(w[h] & 0xFFFF0000u);
      ss = fmaf(lo, lo, ss);
      ss = fmaf(hi, hi, ss);
    }
  }
  ss = warp_sum(ss);
  return rsqrtf(ss / (float)D + kRmsEps);
}

// dst[0..D) = bf16(src * inv * w), 8 elements per 16-byte access.
__device__ __forceinline__ void row_norm_store(const uint16_t* src, const float* w, float inv,
                                               uint16_t* dst, int D, int lane) {
  const uint4* s4 = (const uint4*)src;
  const float4* w4 = (const float4*)w;
  uint4* d4 = (uint4*)dst;
  for (int i = lane; i < D / 8; i += 32) {
    const uint4 u = s4[i];
    const float4 wa = w4[2 * i], wb = w4[2 * i + 1];
    const float ww[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
    const uint32_t in[4] = {u.x, u.y, u.z, u.w};
    uint32_t out[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float lo = __uint_as_float(in[h] << 16) * inv * ww[2 * h];
      const float hi = __uint_as_float(in[h] & 0xFFFF0000u) * inv * ww[2 * h + 1];
      out[h] = (uint32_t)to_bf16(lo) | ((uint32_t)to_bf16(hi) << 16);
    }
    d4[i] = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

// One warp per evaluation row: its Row, and x = [rmsnorm(h_d) :: rmsnorm(E[t])].
__global__ void tf_prep_kernel(const uint16_t* h, const uint16_t* E, const float* w_h,
                               const float* w_e, const int32_t* root, const int32_t* S1, int batch,
                               int gamma, int D, int V, int M, Row* rows2, uint16_t* X,
                               int32_t* status) {
  const int lane = threadIdx.x & 31;
  const int per = 1 + (gamma - 1) * M;
  const int e = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (e >= batch * per) return;
  const int b = e / per, j = e % per;
  int d, prev;
  if (j == 0) {
    d = 1;
    prev = root[b];
  } else {
    d = 2 + (j - 1) / M;
    prev = S1[((size_t)b * gamma + (d - 2)) * M + (j - 1) % M];
  }
  if (prev < 0 || prev >= V) {
    if (lane == 0) set_status(status, DT_EDEVICE);
    prev = 0;
  }
  const uint16_t* hr = h + ((size_t)b * gamma + (d - 1)) * D;
  const uint16_t* er = E + (size_t)prev * D;
  const float ih = row_inv_rms(hr, D, lane);
  const float ie = row_inv_rms(er, D, lane);
  uint16_t* xr = X + (size_t)e * 2 * D;
  row_norm_store(hr, w_h, ih, xr, D, lane);
  row_norm_store(er, w_e, ie, xr + D, D, lane);
  if (lane == 0) {
    Row r;
    r.b = b;
    r.depth = d - 1;  // residual row h_d of the block
    r.token = prev;
    r.aux = e;
    r.path = 0;
    r.lse = 0.f;
    r.key = 0.f;
    rows2[e] = r;
  }
}

// (key desc, depth asc, parent index asc, rank asc) as one 64-bit key, smaller first.
__device__ __forceinline__ uint64_t tf_order(float key, int depth, int parent, int rank) {
  const uint32_t hi = ~f32_ordered(key);
  const uint32_t lo = ((uint32_t)depth << 24) | ((uint32_t)(parent + 1) << 12) | (uint32_t)rank;
  return ((uint64_t)hi << 32) | lo;
}

// One warp per request: sequential best-first over the evaluated
// distributions (pop the best candidate, emit it, push its M children when
// its token was evaluated at its depth).
__global__ void tf_select_kernel(const int32_t* S1, const float* lse2, const float* v2,
                                 const int32_t* i2, int gamma, int M, int budget, int cap,
                                 dt_tree out, int32_t* status) {
  extern __shared__ __align__(16) uint8_t sm[];
  const int b = blockIdx.x, lane = threadIdx.x;
  const int per = 1 + (gamma - 1) * M;
  float* c_key = (float*)sm;              // [cap]
  int32_t* c_tok = (int32_t*)(c_key + cap);
  int32_t* c_par = c_tok + cap;            // emitted index of the parent (-1: root)
  int32_t* c_dep = c_par + cap;
  int32_t* c_rank = c_dep + cap;
  int32_t* c_live = c_rank + cap;
  uint64_t* anc = (uint64_t*)(c_live + cap);  // [budget]; 24 cap bytes keep 8-byte alignment
  int n_c = 0;
  // children of a node (depth d, token t, emitted index p, key k0)
  auto push = [&](int d, int t, int p, float k0) {
    int ev;
    if (d == 0) {
      ev = 0;
    } else {
      if (d >= gamma) return;
      int pos = -1;
      for (int m = 0; m < M; ++m)
        if (S1[((size_t)b * gamma + (d - 1)) * M + m] == t) pos = m;
      if (pos < 0) return;  // not evaluated at this depth: a leaf
      ev = 1 + (d - 1) * M + pos;
    }
    const size_t er = (size_t)b * per + ev;
    const float l = lse2[er];
    for (int j = lane; j < M; j += 32) {
      if (n_c + j >= cap) continue;
      c_key[n_c + j] = k0 + (v2[er * M + j] - l);
      c_tok[n_c + j] = i2[er * M + j];
      c_par[n_c + j] = p;
      c_dep[n_c + j] = d + 1;
      c_rank[n_c + j] = j;
      c_live[n_c + j] = 1;
    }
    if (n_c + M > cap && lane == 0) set_status(status, DT_EDEVICE);
    n_c = min(cap, n_c + M);
    __syncwarp();
  };
  push(0, 0, -1, 0.f);
  const size_t ob = (size_t)b * budget;
  int n = 0;
  for (; n < budget; ++n) {
    uint64_t best = ~0ull;
    int arg = -1;
    for (int c = lane; c < n_c; c += 32) {
      if (!c_live[c]) continue;
      const uint64_t o = tf_order(c_key[c], c_dep[c], c_par[c], c_rank[c]);
      if (o < best) {
        best = o;
        arg = c;
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const uint64_t ob2 = __shfl_xor_sync(0xffffffffu, best, o);
      const int oa = __shfl_xor_sync(0xffffffffu, arg, o);
      if (ob2 < best || (ob2 == best && oa < arg)) {
        best = ob2;
        arg = oa;
      }
    }
    if (arg < 0) break;
    const float key = c_key[arg];
    const int tok = c_tok[arg], par = c_par[arg], dep = c_dep[arg], rk = c_rank[arg];
    __syncwarp();
    if (lane == 0) {
      c_live[arg] = 0;
      const uint64_t a = (par < 0 ? 0ull : anc[par]) | (1ull << n);
      anc[n] = a;
      out.d_tokens[ob + n] = tok;
      out.d_parents[ob + n] = par;
      out.d_depths[ob + n] = dep;
      out.d_ranks[ob + n] = rk;
      out.d_keys[ob + n] = key;
      out.d_anc[ob + n] = a;
    }
    __syncwarp();
    push(dep, tok, n, key);
  }
  if (lane == 0) out.d_n_nodes[b] = n;
}

struct TfLayout {
  int32_t* status;
  int32_t* counts;
  Row* rows1;
  Row* rows2;
  float2* p1s;
  float* p1v;
  int32_t* p1i;
  float2* p2s;
  float* p2v;
  int32_t* p2i;
  float* v1;
  int32_t* S1;
  uint16_t* X;
  uint16_t* act;
  uint16_t* hp;
  float* lse2;
  float* v2;
  int32_t* i2;
  size_t bytes;
  int n1, n2, ncta;
};

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

TfLayout tf_layout(void* ws, int batch, int gamma, int D, int Dff, int V, int M) {
  TfLayout L;
  L.n1 = batch * gamma;
  L.n2 = batch * (1 + (gamma - 1) * M);
  L.ncta = std::min(num_sms(), (V + 127) / 128);
  uint8_t* base = (uint8_t*)ws;
  size_t off = 0;
  auto take = [&](size_t bytes) -> void* {
    off = align256(off);
    void* p = base ? base + off : nullptr;
    off += bytes;
    return p;
  };
  int32_t* hdr = (int32_t*)take(kWsHeader);
  L.status = hdr;
  L.counts = hdr + 4;
  L.rows1 = (Row*)take(sizeof(Row) * L.n1);
  L.rows2 = (Row*)take(sizeof(Row) * L.n2);
  L.p1s = (float2*)take(sizeof(float2) * (size_t)L.n1 * L.ncta);
  L.p1v = (float*)take(4 * (size_t)L.n1 * L.ncta * M);
  L.p1i = (int32_t*)take(4 * (size_t)L.n1 * L.ncta * M);
  L.p2s = (float2*)take(sizeof(float2) * (size_t)L.n2 * L.ncta);
  L.p2v = (float*)take(4 * (size_t)L.n2 * L.ncta * M);
  L.p2i = (int32_t*)take(4 * (size_t)L.n2 * L.ncta * M);
  L.v1 = (float*)take(4 * (size_t)L.n1 * M);
  L.S1 = (int32_t*)take(4 * (size_t)L.n1 * M);
  L.X = (uint16_t*)take(2 * (size_t)L.n2 * 2 * D);
  L.act = (uint16_t*)take(2 * (size_t)L.n2 * Dff);
  L.hp = (uint16_t*)take(2 * (size_t)L.n2 * D);
  L.lse2 = (float*)take(4 * (size_t)L.n2);
  L.v2 = (float*)take(4 * (size_t)L.n2 * M);
  L.i2 = (int32_t*)take(4 * (size_t)L.n2 * M);
  L.bytes = align256(off);
  return L;
}

}  // namespace
}  // namespace dt

using namespace dt;

extern "C" {

size_t dt_treeflash_workspace_bytes(int batch, int gamma, int D, int Dff, int V, int M,
                                    int budget) {
  if (batch < 1 || gamma < 1 || D < 1 || Dff < 1 || V < 1 || M < 1 || budget < 1) return 0;
  return tf_layout(nullptr, batch, gamma, D, Dff, V, M).bytes;
}

dt_status dt_treeflash_build(const uint16_t* d_h, const uint16_t* d_embed, const float* d_w_norm_h,
                             const float* d_w_norm_e, const uint16_t* d_w_gate,
                             const uint16_t* d_w_up, const uint16_t* d_w_down,
                             const uint16_t* d_w_lm, const int32_t* d_root, int batch, int gamma,
                             int D, int Dff, int V, int M, int budget, const dt_tree* out,
                             void* ws, size_t ws_bytes, dt_stream stream) {
  if (!d_h || !d_embed || !d_w_norm_h || !d_w_norm_e || !d_w_gate || !d_w_up || !d_w_down ||
      !d_w_lm || !d_root || !out)
    return DT_EINVAL;
  if (!out->d_tokens || !out->d_parents || !out->d_depths || !out->d_ranks || !out->d_keys ||
      !out->d_anc || !out->d_n_nodes)
    return DT_EINVAL;
  if (batch < 1 || gamma < 1 || D < 1 || Dff < 1 || V < 1 || M < 1 || budget < 1)
    return DT_EINVAL;
  if (M > V) return DT_EINVAL;
  if (D % 64 || Dff % 64 || M > 16 || budget > 64 || gamma > 64 || V >= (1 << 24) ||
      batch > 1024)
    return DT_EUNSUPPORTED;
  TfLayout L = tf_layout(nullptr, batch, gamma, D, Dff, V, M);
  if (!ws || ws_bytes < L.bytes) return DT_EWORKSPACE;
  L = tf_layout(ws, batch, gamma, D, Dff, V, M);
  cudaStream_t s = (cudaStream_t)stream;
  const int nt1 = gemm_node_tile(L.n1), nt2 = gemm_node_tile(L.n2);

  CUtensorMap tmLm, tmH1, tmGate, tmUp, tmX, tmDown, tmAct, tmHp;
  if (!make_tmap_bf16_kmajor(&tmLm, d_w_lm, D, V, 128) ||
      !make_tmap_bf16_kmajor(&tmH1, d_h, D, L.n1, nt1) ||
      !make_tmap_bf16_kmajor(&tmGate, d_w_gate, 2 * D, Dff, 64) ||
      !make_tmap_bf16_kmajor(&tmUp, d_w_up, 2 * D, Dff, 64) ||
      !make_tmap_bf16_kmajor(&tmX, L.X, 2 * D, L.n2, nt2) ||
      !make_tmap_bf16_kmajor(&tmDown, d_w_down, Dff, D, 128) ||
      !make_tmap_bf16_kmajor(&tmAct, L.act, Dff, L.n2, nt2) ||
      !make_tmap_bf16_kmajor(&tmHp, L.hp, D, L.n2, nt2))
    return DT_ECUDA;

  if (cudaMemsetAsync(L.status, 0, 4, s) != cudaSuccess) return DT_ECUDA;
  {
    ProfileScope ps(DT_K_OTHER, s);
    tf_rows_kernel<<<(L.n1 + 255) / 256, 256, 0, s>>>(L.rows1, L.n1, gamma, L.counts, L.n2);
    if (cudaGetLastError() != cudaSuccess) return DT_ECUDA;
  }
  const int kmax = gemm_kmax(M);
  GemmArgs g;
  memset(&g, 0, sizeof(g));
  g.L = nullptr;
  g.Bk = gamma;
  g.V = V;
  g.r = D;
  g.k = M;
  g.n_vtiles = (V + 127) / 128;
  g.ncta_v = L.ncta;
  g.status = L.status;
  // 1. stage 1: the drafter's own distributions, top-M per block position
  {
    GemmArgs a = g;
    a.rows = L.rows1;
    a.n_rows = L.counts + 0;
    a.Mcap = L.n1;
    a.pstats = L.p1s;
    a.plv = L.p1v;
    a.pli = L.p1i;
    ProfileScope ps(DT_K_TF_LMHEAD, s);
    if (launch_markov_gemm(EPI_EXPAND, false, tmLm, tmLm, tmH1, a, batch, nt1, s) != cudaSuccess)
      return DT_ECUDA;
  }
  {
    ProfileScope ps(DT_K_OTHER, s);
    const int wpb = 8;
    if (kmax == 4)
      tf_merge_kernel<4><<<(L.n1 + wpb - 1) / wpb, 32 * wpb, 0, s>>>(
          L.p1s, L.p1v, L.p1i, L.ncta, L.n1, M, nullptr, L.v1, L.S1);
    else
      tf_merge_kernel<16><<<(L.n1 + wpb - 1) / wpb, 32 * wpb, 0, s>>>(
          L.p1s, L.p1v, L.p1i, L.ncta, L.n1, M, nullptr, L.v1, L.S1);
    if (cudaGetLastError() != cudaSuccess) return DT_ECUDA;
  }
  // 2. approximator inputs of every evaluation
  {
    ProfileScope ps(DT_K_OTHER, s);
    const int wpb = 8;
    tf_prep_kernel<<<(L.n2 + wpb - 1) / wpb, 32 * wpb, 0, s>>>(
        d_h, d_embed, d_w_norm_h, d_w_norm_e, d_root, L.S1, batch, gamma, D, V, M, L.rows2, L.X,
        L.status);
    if (cudaGetLastError() != cudaSuccess) return DT_ECUDA;
  }
  // 3. silu(x W_gate^T) * (x W_up^T)
  {
    GemmArgs a = g;
    a.rows = L.rows2;
    a.n_rows = L.counts + 1;
    a.Mcap = L.n2;
    a.V = Dff;
    a.r = 2 * D;
    a.n_vtiles = Dff / 64;
    a.ncta_v = std::min(num_sms(), a.n_vtiles);
    a.out = (float*)L.act;
    a.ldo = Dff;
    ProfileScope ps(DT_K_TF_MLP, s);
    if (launch_markov_gemm(EPI_SWIGLU, false, tmGate, tmUp, tmX, a, batch, nt2, s) != cudaSuccess)
      return DT_ECUDA;
  }
  // 4. h' = h_d + act W_down^T (bf16)
  {
    GemmArgs a = g;
    a.L = d_h;
    a.l_bf16 = 1;
    a.rows = L.rows2;
    a.n_rows = L.counts + 1;
    a.Mcap = L.n2;
    a.V = D;
    a.r = Dff;
    a.n_vtiles = (D + 127) / 128;
    a.ncta_v = std::min(num_sms(), a.n_vtiles);
    a.out = (float*)L.hp;
    a.ldo = D;
    a.out_bf16 = 1;
    ProfileScope ps(DT_K_TF_MLP, s);
    if (launch_markov_gemm(EPI_ZDUMP, false, tmDown, tmDown, tmAct, a, batch, nt2, s) !=
        cudaSuccess)
      return DT_ECUDA;
  }
  // 5. stage 2: the approximator's distributions, log-sum-exp and top-M
  {
    GemmArgs a = g;
    a.rows = L.rows2;
    a.n_rows = L.counts + 1;
    a.Mcap = L.n2;
    a.pstats = L.p2s;
    a.plv = L.p2v;
    a.pli = L.p2i;
    ProfileScope ps(DT_K_TF_LMHEAD, s);
    if (launch_markov_gemm(EPI_EXPAND, false, tmLm, tmLm, tmHp, a, batch, nt2, s) != cudaSuccess)
      return DT_ECUDA;
  }
  {
    ProfileScope ps(DT_K_OTHER, s);
    const int wpb = 8;
    if (kmax == 4)
      tf_merge_kernel<4><<<(L.n2 + wpb - 1) / wpb, 32 * wpb, 0, s>>>(
          L.p2s, L.p2v, L.p2i, L.ncta, L.n2, M, L.lse2, L.v2, L.i2);
    else
      tf_merge_kernel<16><<<(L.n2 + wpb - 1) / wpb, 32 * wpb, 0, s>>>(
          L.p2s, L.p2v, L.p2i, L.ncta, L.n2, M, L.lse2, L.v2, L.i2);
    if (cudaGetLastError() != cudaSuccess) return DT_ECUDA;
  }
  // 6. best-first selection
  {
    ProfileScope ps(DT_K_FRONTIER, s);
    const int cap = M + budget * M;
    const size_t smem = (size_t)cap * 24 + (size_t)budget * 8;
    if (smem > 48 * 1024 &&
        ensure_smem(tf_select_kernel, smem) != cudaSuccess)
      return DT_ECUDA;
    tf_select_kernel<<<batch, 32, smem, s>>>(L.S1, L.lse2, L.v2, L.i2, gamma, M, budget, cap,
                                              *out, L.status);
    if (cudaGetLastError() != cudaSuccess) return DT_ECUDA;
  }
  return DT_OK;
}

}  // extern "C"
