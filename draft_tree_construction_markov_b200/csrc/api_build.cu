// C ABI: dt_tree_build, dt_markov_logits and the shared status helpers.
#include <cstring>
#include <mutex>
#include <vector>

#include "build.cuh"

namespace dt {
bool make_tmap_bf16_kmajor(CUtensorMap* map, const void* base, uint64_t K, uint64_t rows,
                           uint32_t box_rows);
int gemm_node_tile(int max_cols);
bool gemm_can_gather(int r, int nt);
cudaError_t launch_markov_gemm(int mode, bool stoch, const CUtensorMap& tmW,
                               const CUtensorMap& tmW2, const CUtensorMap& tmH, GemmArgs a,
                               int batch, int nt, cudaStream_t s);
cudaError_t launch_frontier(const FrontierArgs& f, cudaStream_t s);
cudaError_t launch_build_init(const FrontierArgs& f, const int32_t* root_token, Row* rows0,
                              int32_t* count0, cudaStream_t s);
int pbuild_cols(int batch, int Nmax, int r);
cudaError_t launch_pbuild(const uint16_t* d_markov_b, PBuildArgs a, int ncta, cudaStream_t s);

// How dt_tree_build runs its waves (dt_set_build_path) and the wait-limit
// test hook (dt_set_build_wait_test); both per host thread.
static thread_local int g_build_path = DT_BUILD_AUTO;
static thread_local int g_stall_cta = -1;
static thread_local uint64_t g_stall_wait_ns = 0;

// ------------------------------------------------------------ profile hook --
static thread_local void** g_prof_events = nullptr;
static thread_local int32_t* g_prof_kinds = nullptr;
static thread_local int g_prof_cap = 0;
static thread_local int32_t* g_prof_count = nullptr;

ProfileScope::ProfileScope(int kind, cudaStream_t stream) : slot(-1), s(stream) {
  if (!g_prof_events || !g_prof_count || *g_prof_count >= g_prof_cap) return;
  slot = (*g_prof_count)++;
  if (g_prof_kinds) g_prof_kinds[slot] = kind;
  cudaEventRecord((cudaEvent_t)g_prof_events[2 * slot], s);
}
ProfileScope::~ProfileScope() {
  if (slot >= 0) cudaEventRecord((cudaEvent_t)g_prof_events[2 * slot + 1], s);
}

cudaError_t ensure_smem_ptr(const void* kernel, size_t bytes) {
  struct Entry {
    const void* k;
    int dev;
    size_t bytes;
  };
  static std::mutex mu;
  static std::vector<Entry> done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> g(mu);
  for (auto& e : done)
    if (e.k == kernel && e.dev == dev && e.bytes >= bytes) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  for (auto& x : done)
    if (x.k == kernel && x.dev == dev) {
      x.bytes = bytes;
      return cudaSuccess;
    }
  done.push_back(Entry{kernel, dev, bytes});
  return cudaSuccess;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Sequential carving of a workspace; every region 256-byte aligned.
struct Carver {
  uint8_t* base;
  size_t off;
  template <class T>
  T* take(size_t count) {
    off = align_up(off, 256);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += count * sizeof(T);
    return p;
  }
};

struct BuildLayout {
  int32_t* status;
  int32_t* counts;  // [0], [1] wave lists, [2] materialised rows
  ReqState* req;
  Cand* lists;
  Row* rows[2];
  Row* mat_rows;
  uint16_t* H;
  uint16_t* Hm;
  float2* pstats;  // [Mcap][ncta_v] per-CTA partials of the wave GEMM
  float* plv;      // [Mcap][k][ncta_v]
  int32_t* pli;
  float* pgv;
  int32_t* pgi;
  // the persistent build alternates two partial buffers by wave parity
  float2* pstats2;
  float* plv2;
  int32_t* pli2;
  float* pgv2;
  int32_t* pgi2;
  float* mrg_lse;      // merged rows of a persistent-build wave
  float* mrg_val;
  int32_t* mrg_tok;
  unsigned* grid_bar;  // header words 8-10: grid-barrier arrivals, abort flag, exits
  int32_t* grid_abort;
  int32_t* cond;       // [batch][Bk] per-depth Markov-row tokens of a baseline variant
  int32_t* chain_nb;   // [batch] Shared-Markov chain: node budget min(Bk, n_budget)
  float* chain_lam;    // [batch] Shared-Markov chain: no survival stop
  size_t bytes;
  int ncta_v, n_vtiles, nt, Mcap, Mcap_pad, Mmat, Mmat_pad;
  int nt_x;  // node tile of the expansion GEMMs
};

// ncta: partials per node (0: one per SM, at most one per vocabulary tile)
static BuildLayout build_layout(void* ws, int batch, int Bk, int V, int r, int k, int Nmax,
                                int ncta = 0) {
  BuildLayout L;
  L.n_vtiles = (V + 127) / 128;
  L.ncta_v = ncta > 0 ? ncta : std::min(num_sms(), L.n_vtiles);
  L.nt = gemm_node_tile(Nmax);
  // With several requests a wave has many columns: 64-column tiles halve the
  // passes over the weights and give the epilogue two warps per quadrant
  // (when the rows still fit the shared-memory gather).
  L.nt_x = (batch > 1 && L.nt == 32 && gemm_can_gather(r, 64)) ? 64 : L.nt;
  L.Mcap = batch * Nmax;
  L.Mcap_pad = (int)align_up(L.Mcap, L.nt);
  L.Mmat = batch * (Nmax + 1);
  L.Mmat_pad = (int)align_up(L.Mmat, L.nt);
  Carver c{(uint8_t*)ws, 0};
  int32_t* hdr = c.take<int32_t>(kWsHeader / 4);
  L.status = hdr;
  L.counts = hdr + 4;
  L.req = c.take<ReqState>(batch);
  L.lists = c.take<Cand>((size_t)batch * Nmax);
  L.rows[0] = c.take<Row>(L.Mcap);
  L.rows[1] = c.take<Row>(L.Mcap);
  L.mat_rows = c.take<Row>(L.Mmat);
  L.H = c.take<uint16_t>((size_t)L.Mcap_pad * r);
  L.Hm = c.take<uint16_t>((size_t)L.Mmat_pad * r);
  const size_t np = (size_t)L.ncta_v * L.Mcap;
  L.pstats = c.take<float2>(np);
  L.plv = c.take<float>(np * k);
  L.pli = c.take<int32_t>(np * k);
  L.pgv = c.take<float>(np * k);
  L.pgi = c.take<int32_t>(np * k);
  L.pstats2 = c.take<float2>(np);
  L.plv2 = c.take<float>(np * k);
  L.pli2 = c.take<int32_t>(np * k);
  L.pgv2 = c.take<float>(np * k);
  L.pgi2 = c.take<int32_t>(np * k);
  L.mrg_lse = c.take<float>(L.Mcap);
  L.mrg_val = c.take<float>((size_t)L.Mcap * k);
  L.mrg_tok = c.take<int32_t>((size_t)L.Mcap * k);
  L.grid_bar = (unsigned*)(hdr + 8);
  L.grid_abort = hdr + 9;
  L.cond = c.take<int32_t>((size_t)batch * Bk);
  L.chain_nb = c.take<int32_t>(batch);
  L.chain_lam = c.take<float>(batch);
  L.bytes = align_up(c.off, 256);
  return L;
}

// Per-request set-up of a baseline variant (one thread per request): no
// Markov row at any depth yet (the marginal-ranked tree keeps this), and the
// budget of the greedy chain that the Shared-Markov tree walks first:
// min(Bk, n_budget) nodes, no survival stop.
__global__ void variant_prep_kernel(const int32_t* n_budget, int batch, int Bk, int Nmax,
                                    int32_t* cond, int32_t* chain_nb, float* chain_lam) {
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < batch; b += gridDim.x * blockDim.x) {
    for (int d = 0; d < Bk; ++d) cond[(size_t)b * Bk + d] = -1;
    int nb = n_budget[b];
    nb = nb < 0 ? 0 : (nb > Nmax ? Nmax : nb);  // the build flags a budget above Nmax
    chain_nb[b] = min(Bk, nb);
    chain_lam[b] = 0.f;
  }
}

// Shared-Markov conditioning from the greedy chain: depth 0 uses the root,
// depth d >= 1 the chain's depth-d token (one thread per request).
__global__ void chain_cond_kernel(dt_tree chain, const int32_t* root, int batch, int Bk, int Nmax,
                                  int V, int32_t* cond) {
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < batch; b += gridDim.x * blockDim.x) {
    const int rt = root[b];
    cond[(size_t)b * Bk] = (rt >= 0 && rt < V) ? rt : -1;  // a bad root is flagged by the build
    int n = chain.d_n_nodes[b];
    n = n < 0 ? 0 : (n > Nmax ? Nmax : n);
    for (int i = 0; i < n; ++i) {
      const int d = chain.d_depths[(size_t)b * Nmax + i];
      const int t = chain.d_tokens[(size_t)b * Nmax + i];
      if (d >= 1 && d < Bk && t >= 0 && t < V) cond[(size_t)b * Bk + d] = t;
    }
  }
}


// Frontier arguments of a build laid out by L.
static FrontierArgs frontier_args(const BuildLayout& L, const uint16_t* d_markov_a,
                                  const float* d_calib, const int32_t* d_n_budget,
                                  const int32_t* d_k_req, const float* d_lambda, int batch,
                                  int Bk, int V, int r, int k, int Nmax, float temp,
                                  const dt_tree* out) {
  FrontierArgs f;
  memset(&f, 0, sizeof(f));
  f.mat_rows = L.mat_rows;
  f.mat_count = L.counts + 2;
  // the GEMM gathers its node rows A[token] itself when they fit in shared
  // memory; otherwise the frontier writes them to H / Hm for TMA
  const bool gather = gemm_can_gather(r, L.nt);
  f.H = gather ? nullptr : L.H;
  f.Hm = gather ? nullptr : L.Hm;
  f.A = d_markov_a;
  f.req = L.req;
  f.lists = L.lists;
  f.pstats = L.pstats;
  f.plv = L.plv;
  f.pli = L.pli;
  f.pgv = L.pgv;
  f.pgi = L.pgi;
  f.ncta = L.ncta_v;
  f.calib = d_calib;
  f.n_budget = d_n_budget;
  f.k_req = d_k_req;
  f.lambda = d_lambda;
  f.Mcap = L.Mcap;
  f.Bk = Bk;
  f.V = V;
  f.r = r;
  f.k = k;
  f.Nmax = Nmax;
  f.batch = batch;
  f.temp = temp;
  f.out = *out;
  f.status = L.status;
  return f;
}

// Expansion-GEMM arguments of a build laid out by L (the whole vocabulary).
static GemmArgs gemm_args(const BuildLayout& L, const void* d_block_logits, dt_dtype ldt,
                          const uint16_t* d_markov_a, int batch, int Bk, int V, int r, int k,
                          int Nmax, float temp, uint64_t philox_seed, uint64_t philox_offset) {
  (void)batch;
  GemmArgs g;
  memset(&g, 0, sizeof(g));
  g.L = d_block_logits;
  g.l_bf16 = ldt == DT_BF16;
  g.gatherA = gemm_can_gather(r, L.nt) ? d_markov_a : nullptr;
  g.Bk = Bk;
  g.V = V;
  g.vfull = V;
  g.r = r;
  g.k = k;
  g.n_vtiles = L.n_vtiles;
  g.ncta_v = L.ncta_v;
  g.Mcap = L.Mcap;
  g.temp = temp;
  g.seed = philox_seed;
  g.offset = (uint32_t)philox_offset;
  g.pstats = L.pstats;
  g.plv = L.plv;
  g.pli = L.pli;
  g.pgv = L.pgv;
  g.pgi = L.pgi;
  g.nmax1 = Nmax + 1;
  g.status = L.status;
  // a wave's column count is only known on the device: one CTA per weight
  // range loops over the node tiles that have columns
  g.n_nslots = 1;
  // every wave of the build streams the same Markov factor: keep it in L2
  g.l2_keep = 1;
  return g;
}

static dt_status run_wave_launches(FrontierArgs f, GemmArgs g, const BuildLayout& L,
                                   const int32_t* d_root_token, const CUtensorMap& tmW,
                                   const CUtensorMap& tmH, int batch, int Bk, cudaStream_t s);

// Arguments of the persistent build, from the wave launches' arguments.
static PBuildArgs pbuild_args(const FrontierArgs& f, const GemmArgs& g, const BuildLayout& L,
                              const int32_t* d_root_token) {
  PBuildArgs a;
  memset(&a, 0, sizeof(a));
  a.L = g.L;
  a.l_bf16 = g.l_bf16;
  a.A = f.A;
  a.Bk = f.Bk;
  a.V = f.V;
  a.r = f.r;
  a.k = f.k;
  a.Nmax = f.Nmax;
  a.batch = f.batch;
  a.n_vtiles = L.n_vtiles;
  a.temp = f.temp;
  a.seed = g.seed;
  a.offset = g.offset;
  a.calib = f.calib;
  a.root_token = d_root_token;
  a.n_budget = f.n_budget;
  a.k_req = f.k_req;
  a.lambda = f.lambda;
  a.cond = f.cond;
  a.pstats[0] = L.pstats;
  a.plv[0] = L.plv;
  a.pli[0] = L.pli;
  a.pgv[0] = L.pgv;
  a.pgi[0] = L.pgi;
  a.pstats[1] = L.pstats2;
  a.plv[1] = L.plv2;
  a.pli[1] = L.pli2;
  a.pgv[1] = L.pgv2;
  a.pgi[1] = L.pgi2;
  a.mrg_lse = L.mrg_lse;
  a.mrg_val = L.mrg_val;
  a.mrg_tok = L.mrg_tok;
  a.grid_bar = L.grid_bar;
  a.grid_abort = L.grid_abort;
  a.mat_rows = L.mat_rows;
  a.mat_count = L.counts + 2;
  a.out = f.out;
  a.status = L.status;
  a.wait_ns = kWaitLimitNs;
  a.stall_cta = -1;
  return a;
}

// init + Bk waves of GEMM and frontier, or one persistent launch for them
// all (+ the draft-q pass at T > 0)
static dt_status run_waves(FrontierArgs f, GemmArgs g, const BuildLayout& L,
                           const int32_t* d_root_token, const uint16_t* d_markov_b,
                           const CUtensorMap& tmW,
                           const CUtensorMap& tmH, const CUtensorMap& tmHm, int batch, int Bk,
                           int Nmax, float* d_draft_q, cudaStream_t s) {
  // At T > 0 the draft-q GEMM after the build reads its node rows through Hm
  // when r is too large to gather them in shared memory; only the per-wave
  // frontier fills Hm, so those builds run as waves.
  const bool fits = pbuild_cols(batch, Nmax, f.r) > 0 && (f.temp == 0.f || f.Hm == nullptr);
  if (g_build_path == DT_BUILD_PERSISTENT && !fits) return DT_EUNSUPPORTED;
  bool waves = g_build_path == DT_BUILD_WAVES || !fits;
  if (!waves) {
    PBuildArgs a = pbuild_args(f, g, L, d_root_token);
    if (g_stall_cta >= 0) {
      a.stall_cta = g_stall_cta;
      a.wait_ns = g_stall_wait_ns;
      g_stall_cta = -1;
    }
    cudaError_t e;
    {
      ProfileScope ps(DT_K_PBUILD, s);
      e = launch_pbuild(d_markov_b, a, L.ncta_v, s);
    }
    if (e == cudaErrorNotSupported || e == cudaErrorCooperativeLaunchTooLarge) {
      (void)cudaGetLastError();
      if (g_build_path == DT_BUILD_PERSISTENT) return DT_EUNSUPPORTED;
      waves = true;  // nothing was enqueued: run the waves instead
    } else if (e != cudaSuccess) {
      return DT_ECUDA;
    }
  }
  if (waves) {
    const dt_status st = run_wave_launches(f, g, L, d_root_token, tmW, tmH, batch, Bk, s);
    if (st != DT_OK) return st;
  }
  const bool stoch = f.temp > 0.f;
  if (stoch) {
    GemmArgs gq = g;
    gq.rows = L.mat_rows;
    gq.n_rows = L.counts + 2;
    gq.reset_count = nullptr;
    gq.Mcap = L.Mmat;
    gq.out = d_draft_q;
    gq.nmax1 = Nmax + 1;
    ProfileScope ps(DT_K_DRAFT_Q, s);
    if (launch_markov_gemm(EPI_QROWS, true, tmW, tmW, tmHm, gq, batch, L.nt, s) != cudaSuccess)
      return DT_ECUDA;
  }
  return DT_OK;
}

// init + Bk waves of GEMM and frontier
static dt_status run_wave_launches(FrontierArgs f, GemmArgs g, const BuildLayout& L,
                                   const int32_t* d_root_token, const CUtensorMap& tmW,
                                   const CUtensorMap& tmH, int batch, int Bk, cudaStream_t s) {
  {
    ProfileScope ps(DT_K_BUILD_INIT, s);
    if (launch_build_init(f, d_root_token, L.rows[0], L.counts + 0, s) != cudaSuccess)
      return DT_ECUDA;
  }
  const bool stoch = f.temp > 0.f;
  for (int w = 0; w < Bk; ++w) {
    const int cur = w & 1, nxt = cur ^ 1;
    g.rows = L.rows[cur];
    g.n_rows = L.counts + cur;
    g.reset_count = L.counts + nxt;
    {
      ProfileScope ps(DT_K_MARKOV_GEMM, s);
      if (launch_markov_gemm(EPI_EXPAND, stoch, tmW, tmW, tmH, g, batch, L.nt_x, s) !=
          cudaSuccess)
        return DT_ECUDA;
    }
    f.rows = L.rows[cur];
    f.next_rows = L.rows[nxt];
    f.next_count = L.counts + nxt;
    {
      ProfileScope ps(DT_K_FRONTIER, s);
      if (launch_frontier(f, s) != cudaSuccess) return DT_ECUDA;
    }
  }
  return DT_OK;
}

static dt_status build_impl(const void* d_block_logits, dt_dtype ldt, const uint16_t* d_markov_a,
                            const uint16_t* d_markov_b, int r, const float* d_calib,
                            const int32_t* d_root_token, const int32_t* d_n_budget,
                            const int32_t* d_k_req, const float* d_lambda, int batch, int Bk,
                            int V, int k, int Nmax, float temp, uint64_t philox_seed,
                            uint64_t philox_offset, int variant, const dt_tree* out, void* ws,
                            size_t ws_bytes, cudaStream_t s);

}  // namespace dt

using namespace dt;

extern "C" {

int dt_num_sms(void) { return num_sms(); }

void dt_set_build_path(int path) {
  g_build_path = (path == DT_BUILD_WAVES || path == DT_BUILD_PERSISTENT) ? path : DT_BUILD_AUTO;
}

void dt_set_build_wait_test(int stall_cta, uint64_t wait_ns) {
  g_stall_cta = stall_cta;
  g_stall_wait_ns = wait_ns;
}

void dt_set_profile_events(void** events, int32_t* kinds, int capacity, int32_t* count) {
  g_prof_events = events;
  g_prof_kinds = kinds;
  g_prof_cap = events ? capacity : 0;
  g_prof_count = count;
}

size_t dt_tree_build_workspace_bytes(int batch, int Bk, int V, int r, int k, int Nmax) {
  if (batch <= 0 || Nmax <= 0 || V <= 0 || r <= 0 || k <= 0) return 0;
  return build_layout(nullptr, batch, Bk, V, r, k, Nmax).bytes;
}

dt_status dt_tree_build(const void* d_block_logits, dt_dtype ldt, const uint16_t* d_markov_a,
                        const uint16_t* d_markov_b, int r, const float* d_calib,
                        const int32_t* d_root_token, const int32_t* d_n_budget,
                        const int32_t* d_k_req, const float* d_lambda, int batch, int Bk, int V,
                        int k, int Nmax, float temp, uint64_t philox_seed,
                        uint64_t philox_offset, const dt_tree* out, void* ws, size_t ws_bytes,
                        dt_stream stream) {
  return build_impl(d_block_logits, ldt, d_markov_a, d_markov_b, r, d_calib, d_root_token,
                    d_n_budget, d_k_req, d_lambda, batch, Bk, V, k, Nmax, temp, philox_seed,
                    philox_offset, DT_TREE_PCTREE, out, ws, ws_bytes, (cudaStream_t)stream);
}

dt_status dt_tree_build_ex(const void* d_block_logits, dt_dtype ldt, const uint16_t* d_markov_a,
                           const uint16_t* d_markov_b, int r, const float* d_calib,
                           const int32_t* d_root_token, const int32_t* d_n_budget,
                           const int32_t* d_k_req, const float* d_lambda, int batch, int Bk,
                           int V, int k, int Nmax, float temp, uint64_t philox_seed,
                           uint64_t philox_offset, dt_tree_variant variant, const dt_tree* out,
                           void* ws, size_t ws_bytes, dt_stream stream) {
  if (variant != DT_TREE_PCTREE && variant != DT_TREE_CHAIN && variant != DT_TREE_MARGINAL &&
      variant != DT_TREE_SHARED_MARKOV)
    return DT_EINVAL;
  return build_impl(d_block_logits, ldt, d_markov_a, d_markov_b, r, d_calib, d_root_token,
                    d_n_budget, d_k_req, d_lambda, batch, Bk, V, k, Nmax, temp, philox_seed,
                    philox_offset, variant, out, ws, ws_bytes, (cudaStream_t)stream);
}

}  // extern "C"

namespace dt {

static dt_status build_impl(const void* d_block_logits, dt_dtype ldt, const uint16_t* d_markov_a,
                            const uint16_t* d_markov_b, int r, const float* d_calib,
                            const int32_t* d_root_token, const int32_t* d_n_budget,
                            const int32_t* d_k_req, const float* d_lambda, int batch, int Bk,
                            int V, int k, int Nmax, float temp, uint64_t philox_seed,
                            uint64_t philox_offset, int variant, const dt_tree* out, void* ws,
                            size_t ws_bytes, cudaStream_t s) {
  if (!d_block_logits || !d_markov_a || !d_markov_b || !d_root_token || !d_n_budget ||
      !d_lambda || !out)
    return DT_EINVAL;
  if (!out->d_tokens || !out->d_parents || !out->d_depths || !out->d_ranks || !out->d_keys ||
      !out->d_anc || !out->d_n_nodes)
    return DT_EINVAL;
  if (ldt != DT_F32 && ldt != DT_BF16) return DT_EINVAL;
  if (batch < 1 || Bk < 1 || V < 1 || k < 1 || Nmax < 1 || r < 1) return DT_EINVAL;
  if (!(temp >= 0.f) || philox_offset >= (1ull << 32)) return DT_EINVAL;
  if (temp > 0.f && !out->d_draft_q) return DT_EINVAL;
  if (batch > 1024 || Bk > 16 || k > 16 || Nmax > 64 || V >= (1 << 20) || r % 16 || r > 1024)
    return DT_EUNSUPPORTED;
  if (k > V) return DT_EINVAL;
  BuildLayout L = build_layout(nullptr, batch, Bk, V, r, k, Nmax);
  if (!ws || ws_bytes < L.bytes) return DT_EWORKSPACE;
  L = build_layout(ws, batch, Bk, V, r, k, Nmax);

  CUtensorMap tmW, tmH, tmHm;
  if (!make_tmap_bf16_kmajor(&tmW, d_markov_b, r, V, 128) ||
      !make_tmap_bf16_kmajor(&tmH, L.H, r, L.Mcap_pad, L.nt) ||
      !make_tmap_bf16_kmajor(&tmHm, L.Hm, r, L.Mmat_pad, L.nt))
    return DT_ECUDA;

  // status, wave counters and the persistent build's grid-barrier words
  if (cudaMemsetAsync(L.status, 0, 64, s) != cudaSuccess) return DT_ECUDA;

  FrontierArgs f = frontier_args(L, d_markov_a, d_calib, d_n_budget, d_k_req, d_lambda, batch,
                                 Bk, V, r, k, Nmax, temp, out);
  GemmArgs g = gemm_args(L, d_block_logits, ldt, d_markov_a, batch, Bk, V, r, k, Nmax, temp,
                         philox_seed, philox_offset);

  if (variant == DT_TREE_CHAIN) {
    // the method with one child per node (k = 1 everywhere)
    f.k = g.k = 1;
    f.k_req = nullptr;
  }
  if (variant == DT_TREE_MARGINAL || variant == DT_TREE_SHARED_MARKOV) {
    ProfileScope ps(DT_K_OTHER, s);
    variant_prep_kernel<<<(batch + 127) / 128, 128, 0, s>>>(d_n_budget, batch, Bk, Nmax, L.cond,
                                                           L.chain_nb, L.chain_lam);
    if (cudaGetLastError() != cudaSuccess) return DT_ECUDA;
  }
  if (variant == DT_TREE_MARGINAL) f.cond = L.cond;
  if (variant == DT_TREE_SHARED_MARKOV) {
    // walk the greedy chain first (into the caller's tree arrays, which the
    // tree build then overwrites), then condition depth d on its token
    FrontierArgs fc = f;
    GemmArgs gc = g;
    fc.n_budget = L.chain_nb;
    fc.k = gc.k = 1;
    fc.k_req = nullptr;
    fc.lambda = L.chain_lam;
    fc.temp = 0.f;
    gc.temp = 0.f;
    const dt_status st = run_waves(fc, gc, L, d_root_token, d_markov_b, tmW, tmH, tmHm, batch, Bk, Nmax,
                                   nullptr, s);
    if (st != DT_OK) return st;
    {
      ProfileScope ps(DT_K_OTHER, s);
      chain_cond_kernel<<<(batch + 127) / 128, 128, 0, s>>>(*out, d_root_token, batch, Bk, Nmax,
                                                           V, L.cond);
      if (cudaGetLastError() != cudaSuccess) return DT_ECUDA;
    }
    f.cond = L.cond;
  }
  return run_waves(f, g, L, d_root_token, d_markov_b, tmW, tmH, tmHm, batch, Bk, Nmax,
                   out->d_draft_q, s);
}

}  // namespace dt

// --------------------------------------------------- vocabulary-sharded build --
namespace dt {

// Tiles [t_lo, t_hi) of rank `rank` among `world` (the tiles split as evenly
// as whole tiles allow, lower ranks first).
static void shard_range(int V, int world, int rank, int* v_base, int* v_len) {
  const int T = (V + 127) / 128;
  const int t_lo = (int)((long long)rank * T / world);
  const int t_hi = (int)((long long)(rank + 1) * T / world);
  *v_base = t_lo * 128;
  *v_len = std::min(V, t_hi * 128) - *v_base;
}

static bool shard_cfg_ok(const dt_shard_cfg* c) {
  return c && c->batch >= 1 && c->batch <= 1024 && c->Bk >= 1 && c->Bk <= 16 && c->k >= 1 &&
         c->k <= 16 && c->k <= c->V && c->Nmax >= 1 && c->Nmax <= 64 && c->V >= 1 &&
         c->V < (1 << 20) && c->r >= 16 && c->r <= 1024 && c->r % 16 == 0 && c->world >= 1 &&
         c->world <= 64 && c->ncta >= 1 && c->ncta * c->world <= 64 * 148 &&
         c->ncta <= ((c->V + 127) / 128) / c->world;
}

// One rank's partials of a wave: statistics [Mcap][ncta], list values and
// tokens [Mcap][k][ncta].
struct ShardBlock {
  float2* pstats;
  float* plv;
  int32_t* pli;
  size_t off_lv, off_li;  // byte offsets of plv and pli within the block
  size_t bytes;
};

static ShardBlock shard_block(void* base, const dt_shard_cfg* c) {
  ShardBlock s;
  Carver cv{(uint8_t*)base, 0};
  const size_t np = (size_t)c->batch * c->Nmax * c->ncta;
  s.pstats = cv.take<float2>(np);
  s.off_lv = align_up(cv.off, 256);
  s.plv = cv.take<float>(np * c->k);
  s.off_li = align_up(cv.off, 256);
  s.pli = cv.take<int32_t>(np * c->k);
  s.bytes = align_up(cv.off, 256);
  return s;
}

// The gathered blocks [world] -> the frontier's [row][k][world * ncta]
// layout, for the rows of this wave.
__global__ void shard_interleave_kernel(const uint8_t* gathered, size_t block_bytes,
                                        size_t off_lv, size_t off_li, int world, int ncta, int k,
                                        const int32_t* n_rows, int Mcap, float2* pstats,
                                        float* plv, int32_t* pli) {
  const int rows = min(max(*n_rows, 0), Mcap);
  const int nt = world * ncta;
  const long long per_row = (long long)nt * (1 + k);
  const long long total = (long long)rows * per_row;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int row = (int)(e / per_row);
    const int rem = (int)(e % per_row);
    const int i = rem / nt - 1;  // -1: statistics, else list entry i
    const int col = rem % nt;
    const int w = col / ncta, c = col % ncta;
    const uint8_t* blk = gathered + (size_t)w * block_bytes;
    if (i < 0) {
      pstats[(size_t)row * nt + col] = ((const float2*)blk)[(size_t)row * ncta + c];
    } else {
      const size_t src = ((size_t)row * k + i) * ncta + c;
      const size_t dst = ((size_t)row * k + i) * nt + col;
      plv[dst] = ((const float*)(blk + off_lv))[src];
      pli[dst] = ((const int32_t*)(blk + off_li))[src];
    }
  }
}

}  // namespace dt

extern "C" {

void dt_shard_range(int V, int world, int rank, int* v_base, int* v_len) {
  if (!v_base || !v_len) return;
  if (V < 1 || world < 1 || rank < 0 || rank >= world) {
    *v_base = *v_len = 0;
    return;
  }
  shard_range(V, world, rank, v_base, v_len);
}

int dt_shard_ncta(int V, int world) {
  if (V < 1 || world < 1) return 0;
  return std::max(0, std::min(num_sms(), ((V + 127) / 128) / world));
}

size_t dt_sharded_workspace_bytes(const dt_shard_cfg* c) {
  if (!shard_cfg_ok(c)) return 0;
  return build_layout(nullptr, c->batch, c->Bk, c->V, c->r, c->k, c->Nmax, c->world * c->ncta)
      .bytes;
}

size_t dt_sharded_partials_bytes(const dt_shard_cfg* c) {
  if (!shard_cfg_ok(c)) return 0;
  return shard_block(nullptr, c).bytes;
}

dt_status dt_sharded_build_begin(const dt_shard_cfg* c, const int32_t* d_root_token,
                                 const int32_t* d_n_budget, const int32_t* d_k_req,
                                 const float* d_lambda, const dt_tree* out, void* ws,
                                 size_t ws_bytes, dt_stream stream) {
  if (!shard_cfg_ok(c)) return c ? DT_EUNSUPPORTED : DT_EINVAL;
  if (!d_root_token || !d_n_budget || !d_lambda || !out || !out->d_tokens || !out->d_parents ||
      !out->d_depths || !out->d_ranks || !out->d_keys || !out->d_anc || !out->d_n_nodes)
    return DT_EINVAL;
  BuildLayout L = build_layout(nullptr, c->batch, c->Bk, c->V, c->r, c->k, c->Nmax,
                               c->world * c->ncta);
  if (!ws || ws_bytes < L.bytes) return DT_EWORKSPACE;
  L = build_layout(ws, c->batch, c->Bk, c->V, c->r, c->k, c->Nmax, c->world * c->ncta);
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(L.status, 0, 4, s) != cudaSuccess) return DT_ECUDA;
  FrontierArgs f = frontier_args(L, nullptr, nullptr, d_n_budget, d_k_req, d_lambda, c->batch,
                                 c->Bk, c->V, c->r, c->k, c->Nmax, 0.f, out);
  f.H = nullptr;  // the sharded GEMM always gathers its node rows
  f.Hm = nullptr;
  ProfileScope ps(DT_K_BUILD_INIT, s);
  return launch_build_init(f, d_root_token, L.rows[0], L.counts + 0, s) == cudaSuccess
             ? DT_OK
             : DT_ECUDA;
}

dt_status dt_sharded_build_gemm(const dt_shard_cfg* c, int wave, int rank,
                                const void* d_block_logits, dt_dtype ldt,
                                const uint16_t* d_markov_a, const uint16_t* d_markov_b_shard,
                                void* ws, size_t ws_bytes, void* d_partials,
                                dt_stream stream) {
  if (!shard_cfg_ok(c)) return c ? DT_EUNSUPPORTED : DT_EINVAL;
  if (!d_block_logits || !d_markov_a || !d_markov_b_shard || !d_partials) return DT_EINVAL;
  if (ldt != DT_F32 && ldt != DT_BF16) return DT_EINVAL;
  if (wave < 0 || wave >= c->Bk || rank < 0 || rank >= c->world) return DT_EINVAL;
  if ((uintptr_t)d_partials % 256) return DT_EINVAL;
  BuildLayout L = build_layout(nullptr, c->batch, c->Bk, c->V, c->r, c->k, c->Nmax,
                               c->world * c->ncta);
  if (!ws || ws_bytes < L.bytes) return DT_EWORKSPACE;
  if (!gemm_can_gather(c->r, L.nt_x)) return DT_EUNSUPPORTED;
  L = build_layout(ws, c->batch, c->Bk, c->V, c->r, c->k, c->Nmax, c->world * c->ncta);
  int v_base = 0, v_len = 0;
  shard_range(c->V, c->world, rank, &v_base, &v_len);
  CUtensorMap tmW;
  if (!make_tmap_bf16_kmajor(&tmW, d_markov_b_shard, c->r, v_len, 128)) return DT_ECUDA;
  const ShardBlock blk = shard_block(d_partials, c);
  GemmArgs g = gemm_args(L, d_block_logits, ldt, d_markov_a, c->batch, c->Bk, c->V, c->r, c->k,
                         c->Nmax, 0.f, 0, 0);
  g.V = v_len;  // this shard's rows of Bm
  g.v_base = v_base;
  g.vfull = c->V;
  g.n_vtiles = (v_len + 127) / 128;
  g.ncta_v = c->ncta;
  g.pstats = blk.pstats;
  g.plv = blk.plv;
  g.pli = blk.pli;
  g.pgv = nullptr;
  g.pgi = nullptr;
  const int cur = wave & 1;
  g.rows = L.rows[cur];
  g.n_rows = L.counts + cur;
  g.reset_count = L.counts + (cur ^ 1);
  ProfileScope ps(DT_K_MARKOV_GEMM, (cudaStream_t)stream);
  return launch_markov_gemm(EPI_EXPAND, false, tmW, tmW, tmW, g, c->batch, L.nt_x,
                            (cudaStream_t)stream) == cudaSuccess
             ? DT_OK
             : DT_ECUDA;
}

dt_status dt_sharded_build_frontier(const dt_shard_cfg* c, int wave, const void* d_gathered,
                                    const float* d_calib, const int32_t* d_n_budget,
                                    const int32_t* d_k_req, const float* d_lambda,
                                    const dt_tree* out, void* ws, size_t ws_bytes,
                                    dt_stream stream) {
  if (!shard_cfg_ok(c)) return c ? DT_EUNSUPPORTED : DT_EINVAL;
  if (!d_gathered || !d_n_budget || !d_lambda || !out) return DT_EINVAL;
  if (wave < 0 || wave >= c->Bk) return DT_EINVAL;
  BuildLayout L = build_layout(nullptr, c->batch, c->Bk, c->V, c->r, c->k, c->Nmax,
                               c->world * c->ncta);
  if (!ws || ws_bytes < L.bytes) return DT_EWORKSPACE;
  L = build_layout(ws, c->batch, c->Bk, c->V, c->r, c->k, c->Nmax, c->world * c->ncta);
  cudaStream_t s = (cudaStream_t)stream;
  const ShardBlock rel = shard_block(nullptr, c);  // layout of one rank's block
  const int cur = wave & 1;
  {
    ProfileScope ps(DT_K_OTHER, s);
    shard_interleave_kernel<<<num_sms(), 256, 0, s>>>(
        (const uint8_t*)d_gathered, rel.bytes, rel.off_lv, rel.off_li, c->world, c->ncta, c->k,
        L.counts + cur, L.Mcap, L.pstats, L.plv, L.pli);
    if (cudaGetLastError() != cudaSuccess) return DT_ECUDA;
  }
  FrontierArgs f = frontier_args(L, nullptr, d_calib, d_n_budget, d_k_req, d_lambda, c->batch,
                                 c->Bk, c->V, c->r, c->k, c->Nmax, 0.f, out);
  f.H = nullptr;
  f.Hm = nullptr;
  f.rows = L.rows[cur];
  f.next_rows = L.rows[cur ^ 1];
  f.next_count = L.counts + (cur ^ 1);
  ProfileScope ps(DT_K_FRONTIER, s);
  return launch_frontier(f, s) == cudaSuccess ? DT_OK : DT_ECUDA;
}

}  // extern "C"

extern "C" {

// ---------------------------------------------------------------- z rows --
namespace {
// One warp per row: the row descriptor and the gathered Markov row A[token]
// (r is a multiple of 16, so rows move in 16-byte pieces).
__global__ void zrows_prep_kernel(const int32_t* req, const int32_t* depth, const int32_t* token,
                                  int n, int V, int r, const uint16_t* __restrict__ A, Row* rows,
                                  uint16_t* __restrict__ H, int32_t* count, int32_t* status) {
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  for (int i = blockIdx.x * wpb + (threadIdx.x >> 5); i < n; i += gridDim.x * wpb) {
    int t = token[i];
    const bool bad = t < 0 || t >= V;
    if (bad) t = 0;
    if (lane == 0) {
      Row rw;
      rw.b = bad ? -1 : req[i];
      rw.depth = depth[i];
      if (bad) set_status(status, DT_EDEVICE);
      rw.token = t;
      rw.aux = i;
      rw.path = 0;
      rw.lse = 0.f;
      rw.key = 0.f;
      rows[i] = rw;
    }
    const uint4* src = (const uint4*)(A + (size_t)t * r);
    uint4* dst = (uint4*)(H + (size_t)i * r);
    for (int j = lane; j < r / 8; j += 32) dst[j] = src[j];
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) *count = n;
}
}  // namespace

size_t dt_markov_logits_workspace_bytes(int n_rows, int V, int r) {
  (void)V;
  if (n_rows <= 0 || r <= 0) return 0;
  Carver c{nullptr, 0};
  c.take<int32_t>(kWsHeader / 4);
  c.take<Row>(n_rows);
  c.take<uint16_t>(align_up(n_rows, 64) * r);
  return align_up(c.off, 256);
}

dt_status dt_markov_logits(const void* d_block_logits, dt_dtype ldt, const uint16_t* d_markov_a,
                           const uint16_t* d_markov_b, int r, int batch, int Bk, int V,
                           const int32_t* d_req, const int32_t* d_depth, const int32_t* d_token,
                           int n_rows, float* d_z, void* ws, size_t ws_bytes, dt_stream stream) {
  if (!d_block_logits || !d_markov_a || !d_markov_b || !d_req || !d_depth || !d_token || !d_z)
    return DT_EINVAL;
  if (ldt != DT_F32 && ldt != DT_BF16) return DT_EINVAL;
  if (n_rows < 1 || batch < 1 || Bk < 1 || V < 1 || r < 1) return DT_EINVAL;
  if (V >= (1 << 20) || r % 16 || r > 1024 || batch > 1024 || Bk > 16) return DT_EUNSUPPORTED;
  const size_t need = dt_markov_logits_workspace_bytes(n_rows, V, r);
  if (!ws || ws_bytes < need) return DT_EWORKSPACE;
  Carver c{(uint8_t*)ws, 0};
  int32_t* hdr = c.take<int32_t>(kWsHeader / 4);
  Row* rows = c.take<Row>(n_rows);
  const int nt = gemm_node_tile(n_rows);
  const int n_pad = (int)align_up(n_rows, nt);
  uint16_t* H = c.take<uint16_t>((size_t)align_up(n_rows, 64) * r);
  cudaStream_t s = (cudaStream_t)stream;
  CUtensorMap tmW, tmH;
  if (!make_tmap_bf16_kmajor(&tmW, d_markov_b, r, V, 128) ||
      !make_tmap_bf16_kmajor(&tmH, H, r, n_pad, nt))
    return DT_ECUDA;
  if (cudaMemsetAsync(hdr, 0, 4, s) != cudaSuccess) return DT_ECUDA;
  zrows_prep_kernel<<<(n_rows + 7) / 8, 256, 0, s>>>(d_req, d_depth, d_token, n_rows, V, r,
                                                          d_markov_a, rows, H, hdr + 4, hdr);
  if (cudaGetLastError() != cudaSuccess) return DT_ECUDA;
  GemmArgs g;
  memset(&g, 0, sizeof(g));
  g.L = d_block_logits;
  g.l_bf16 = ldt == DT_BF16;
  g.Bk = Bk;
  g.V = V;
  g.r = r;
  g.k = 1;
  g.rows = rows;
  g.n_rows = hdr + 4;
  g.n_vtiles = (V + 127) / 128;
  g.ncta_v = std::min(num_sms(), g.n_vtiles);
  g.Mcap = n_rows;
  g.out = d_z;
  g.status = hdr;
  if (launch_markov_gemm(EPI_ZDUMP, false, tmW, tmW, tmH, g, batch, nt, s) != cudaSuccess)
    return DT_ECUDA;
  return DT_OK;
}

dt_status dt_read_status(void* ws, dt_stream stream, int32_t* host_status) {
  if (!ws || !host_status) return DT_EINVAL;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaStreamSynchronize(s) != cudaSuccess) return DT_ECUDA;
  int32_t v = 0;
  if (cudaMemcpy(&v, ws, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return DT_ECUDA;
  if (cudaMemset(ws, 0, 4) != cudaSuccess) return DT_ECUDA;
  *host_status = v;
  return DT_OK;
}

}  // extern "C"
