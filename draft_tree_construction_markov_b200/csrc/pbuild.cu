// Persistent tree build: all waves of a small batch in one cooperative launch.
//
// Sources: PCTree summary, DSpark paragraph (the Markov head biases the
// shared block logits by the previous token) and "k=4, N=32" paragraph
// (budget N, k children per node); TreeSpark article, "core idea" (path
// survival drives best-first expansion and per-round stopping) and
// "lossless" section (siblings sampled without replacement at T > 0).
//
// What one wave computes is the same as the wave GEMM (markov_gemm.cu) plus
// the frontier (frontier.cu): for every node u to expand,
//   z_u[x] = L[b][depth(u)][x] + sum_rho A[tok(u)][rho] * Bm[x][rho],
// its log-sum-exp, its k best (T = 0) or Gumbel-sampled (T > 0) children, and
// then the best-first selection over all known candidates, which yields the
// next wave's nodes or the final tree.
//
// Why one launch.  At batch 1 a wave expands a handful of nodes, so the wave
// is bound by latency, not by the 78 MB of the Markov factor: separate GEMM
// and frontier launches spend most of a wave in launch gaps, kernel
// prologues (TMEM allocation, bias and row loads) and a frontier that merges
// the 148 per-CTA partials of every node on a single CTA.  Here:
//  * one CTA per SM owns a contiguous vocabulary range of Bm for the whole
//    build.  Its block-logit rows (every request and depth) are loaded once.
//  * a producer thread streams the range through a TMA stage ring.  Each
//    wave's pass over the range is released as soon as the previous wave's
//    merged rows are read, so its first tiles are in flight while the
//    selection that decides its nodes still runs.  The loads carry an L2
//    evict-last hint: waves 2.. re-read the same 78 MB.
//  * after its epilogue every CTA writes one partial per node and meets the
//    others at a grid barrier (bounded wait).  The merge of a node row's
//    per-CTA partials is then spread over the grid: row e is merged by CTA
//    e % ncta alone (148 CTAs reading the same lines at once would queue on
//    the same L2 slices), which writes the row's log-sum-exp and k best
//    entries to a merged-row buffer.  After a second grid barrier EVERY CTA
//    reads the merged rows and runs the selection itself: all read the same
//    bytes and take the same decisions in the same order, so the next wave's
//    nodes need no further exchange.  CTA 0 writes the tree.
//  * partial buffers alternate by wave parity: a CTA can only write wave
//    w + 2's partials after every CTA has passed the barriers of wave w + 1,
//    i.e. has finished merging wave w.
#include "build.cuh"
#include "epi_util.cuh"
#include "merge.cuh"

namespace dt {

// Roles of the 10 warps.  The nodes of a wave are the rows of the MMA's A
// operand (M = 128) and the streamed Bm tiles the B operand, 256 vocabulary
// rows per MMA.  tcgen05.ld lets warp w read TMEM lane quadrant w % 4 only,
// and the four quadrants belong to the SM's four sub-partitions.  So that
// the epilogue runs on all four, the NT node rows are replicated R = 128 / NT
// times down the A operand (the MMA computes every replica at no extra
// cost): quadrant q holds node group q % (NT / 32) of replica q / (NT / 32).
// Epilogue warps 0-7 (two per quadrant) split a tile's 256 columns: the
// 2R warps that see the same node group take one part of 256 / (2R) = NT
// columns each.  NT is the kernel's capacity (32 or 64 rows); a wave of the
// 64-row kernel with at most 32 rows uses the 32-row layout (four replicas).
template <int NG>
struct PShape {
  static constexpr int NT = 32 * NG;          // node rows per replica
  static constexpr int R = 4 / NG;            // replicas down the 128 A rows
  static constexpr int kThreads = 320;
  static constexpr int kEpiWarps = 8;         // warps 0-7
  static constexpr int kWarpMma = 8;
  static constexpr int kWarpProd = 9;
  static constexpr int kParts = 2 * R;        // column parts of a tile per node group
  static constexpr int kPartCols = 256 / kParts;  // = NT
  static constexpr int kCompute = kThreads - 32;  // every warp but the producer
  static constexpr int kCWarps = kCompute / 32;
  static constexpr int kMergeWarps = 4;       // warps of a CTA that merge node rows
  static constexpr int kTileN = 256;          // vocabulary rows per MMA tile
  static constexpr int kStageBytes = kTileN * 128;  // 256 rows x 64 bf16 of Bm
  static constexpr int kAccBufs = 2;          // TMEM accumulators of 128 x 256 fp32
  static constexpr uint32_t kTmemCols = kAccBufs * kTileN;  // the whole TMEM
  static_assert(NG == 1 || NG == 2, "32 or 64 node rows");
};

// Column of this wave's tile as the epilogue sees it.
struct PMeta {
  int32_t valid;
  int32_t b;
  int32_t bslot;  // row of the bias cache: b * Bk + depth
  uint32_t c1, c2;
  int32_t pad[3];
};

// Shared-memory layout, computed the same way on the host (size) and the
// device (offsets).  Offsets are from a 1024-byte aligned base.
//
// The A operand: chunk kc (K columns 64 kc .. 64 kc + 63) of A row i at
// a + (kc * 128 + i) * 128, 128-byte swizzled; A row i holds node i % nte,
// nte = 32 or 64 the node rows per replica of the wave.
struct PLayout {
  size_t a, bias, lists, cands, sorted, keys, rlse, rlq, rtok, spos, spar, msv, msi, misc, req,
      rows0, rows1, meta, exch, bars, flags, stage, total;
};

__host__ __device__ inline size_t p_align(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Elements per row of the bias cache: the CTA's vocabulary range (span) plus
// 16 bytes, so that the rows of different depths start in different banks.
__host__ __device__ inline int p_bias_stride(int span, int esz) { return span + 16 / esz; }

template <int NG>
__host__ __device__ inline PLayout p_layout(int stages, int r, int k, int Nmax, int batch, int Bk,
                                            int span, int esz, int kmax, bool stoch) {
  using S = PShape<NG>;
  const int KC = (r + 63) / 64;
  PLayout l;
  size_t o = 0;
  l.a = o;
  o += (size_t)KC * 128 * 128;
  l.bias = o;
  o += (size_t)batch * Bk * p_bias_stride(span, esz) * esz;
  o = p_align(o, 16);
  l.lists = o;
  o += (size_t)batch * Nmax * sizeof(Cand);
  l.cands = o;
  o += (size_t)(Nmax + Nmax * k) * sizeof(Cand);
  l.sorted = o;
  o += (size_t)Nmax * sizeof(Cand);
  l.keys = o;
  o += (size_t)(Nmax + Nmax * k) * 8;
  // the epilogue's exchange of every column part's per-node partial shares
  // these bytes with the selection scratch: within a wave the epilogue is
  // done with it before the selection starts, and vice versa
  l.exch = l.cands;
  {
    const size_t ex = (size_t)S::kParts * S::NT * (8 + (size_t)kmax * 8 * (stoch ? 2 : 1));
    if (o < l.cands + ex) o = l.cands + ex;
  }
  l.rlse = o;
  o += (size_t)S::NT * 4;
  l.rlq = o;
  o += (size_t)S::NT * k * 4;
  l.rtok = o;
  o += (size_t)S::NT * k * 4;
  l.spos = o;
  o += (size_t)Nmax * 4;
  l.spar = o;
  o += (size_t)Nmax * 4;
  l.msv = o;
  o += (size_t)S::kMergeWarps * 32 * 4;
  l.msi = o;
  o += (size_t)S::kMergeWarps * 32 * 4;
  l.misc = o;
  o += 16 * 4;
  o = p_align(o, 16);
  l.req = o;
  o += (size_t)batch * sizeof(ReqState);
  o = p_align(o, 32);
  l.rows0 = o;
  o += (size_t)S::NT * sizeof(Row);
  l.rows1 = o;
  o += (size_t)S::NT * sizeof(Row);
  l.meta = o;
  o += (size_t)S::NT * sizeof(PMeta);
  o = p_align(o, 8);
  l.bars = o;
  o += (size_t)(2 * stages + 2 * S::kAccBufs + 2) * 8;  // + MMA drain, prefetch gate
  l.flags = o;
  o += 16;
  o = p_align(o, 1024);
  l.stage = o;
  o += (size_t)stages * S::kStageBytes;
  l.total = o;
  return l;
}

// Bounded wait on an mbarrier phase with the launch's limit; gives up early
// once the CTA (or another CTA) has given up.
__device__ __forceinline__ bool p_wait(uint64_t* bar, uint32_t parity, const PBuildArgs& a,
                                       volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > a.wait_ns) {
      *abort_flag = 1;
      set_status(a.status, DT_ETIMEOUT);
      atomicExch(a.grid_abort, 1);
      return false;
    }
  }
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ int ld_relaxed_s32(const int32_t* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// One thread of the CTA: arrive at grid barrier `epoch` (0, 1, ...) and wait
// for every CTA, bounded.  The caller brackets it with CTA barriers.
__device__ __forceinline__ bool grid_sync(const PBuildArgs& a, unsigned epoch, bool arrive,
                                          volatile int* abort_flag) {
  if (arrive) {
    __threadfence();
    atomicAdd(a.grid_bar, 1u);
  }
  const unsigned target = (epoch + 1) * gridDim.x;
  const uint64_t t0 = globaltimer_ns();
  while (ld_acquire_u32(a.grid_bar) < target) {
    if (ld_relaxed_s32(a.grid_abort)) {
      *abort_flag = 1;
      return false;
    }
    if (globaltimer_ns() - t0 > a.wait_ns) {
      *abort_flag = 1;
      set_status(a.status, DT_ETIMEOUT);
      atomicExch(a.grid_abort, 1);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ uint64_t p_sort_key(const Cand& c, int idx) {
  const uint32_t hi = ~f32_ordered(c.key);
  const uint32_t lo = ((uint32_t)c.depth << 27) | ((uint32_t)(c.parent_pos & 127) << 20) |
                      ((uint32_t)(c.rank & 15) << 16) | (uint32_t)idx;
  return ((uint64_t)hi << 32) | lo;
}

__device__ __forceinline__ int p_markov_token(const PBuildArgs& a, int b, int depth, int token) {
  return a.cond ? a.cond[(size_t)b * a.Bk + depth] : token;
}

}  // namespace dt

namespace dt {

// Best-first selection of request b after this wave's merge (every compute
// thread of the CTA; identical in every CTA).  The children of the request's
// expanded rows become candidates keyed by calibrated path survival; the
// top-N of all known candidates (total order: key desc, depth asc, parent
// position asc, rank asc; keys below log(lambda) dropped) is kept; kept nodes
// not yet expanded (depth < Bk) become the request's rows of the next wave,
// appended in request order.  When none waits, the tree is final: CTA 0
// writes it in pop order (and, at T > 0, the draft rows the accept walk needs).
template <int NCT>
__device__ void p_select(const PBuildArgs& a, int b, ReqState* reqs, Cand* lists, Cand* cands,
                         Cand* sorted, uint64_t* keys, const float* r_lse, const float* r_lq,
                         const int32_t* r_tok, const Row* cur, Row* nxt, int nt, int* s_pos,
                         int* s_par, int* misc, int ct, bool writer) {
  ReqState& st = reqs[b];
  if (st.done) return;  // uniform: written only between barriers
  const int kb = st.kb, k = a.k, Nmax = a.Nmax, Bk = a.Bk;
  const int rows_n = st.row_count, rb = st.row_base, n_old = st.n_list;
  Cand* lb = lists + (size_t)b * Nmax;
  for (int i = ct; i < n_old; i += NCT) cands[i] = lb[i];
  if (ct == 0) misc[0] = 0;
  named_bar(1, NCT);
  const int n_new = rows_n * kb;
  for (int i = ct; i < n_new; i += NCT) {
    const int e = i / kb, j = i % kb;
    const Row rw = cur[rb + e];
    float pkey = 0.f;
    int ppos = 0;
    if (rw.aux >= 0) {
      for (int p = 0; p < n_old; ++p)
        if (cands[p].serial == rw.aux) {
          ppos = p + 1;
          pkey = cands[p].key;
          break;
        }
      if (ppos == 0) set_status(a.status, DT_EDEVICE);
    }
    const int d = rw.depth + 1;
    float al = 1.f, be = 0.f;
    if (a.calib) {
      al = a.calib[2 * (d - 1)];
      be = a.calib[2 * (d - 1) + 1];
    }
    const float c = fminf(0.f, fmaf(al, r_lq[(rb + e) * k + j], be));
    Cand cd;
    cd.key = (pkey + c) + 0.0f;
    cd.token = r_tok[(rb + e) * k + j];
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
    cd.pad1[0] = cd.pad1[1] = cd.pad1[2] = 0;
    cands[n_old + i] = cd;
  }
  named_bar(1, NCT);
  const int n_all = n_old + n_new;
  if (ct < rows_n) {
    const Row rw = cur[rb + ct];
    if (rw.aux < 0) {
      st.root_lse = r_lse[rb + ct];
    } else {
      for (int p = 0; p < n_old; ++p)
        if (cands[p].serial == rw.aux) cands[p].lse = r_lse[rb + ct];
    }
  }
  for (int i = ct; i < n_all; i += NCT)
    keys[i] = (cands[i].key >= st.thr) ? p_sort_key(cands[i], i) : ~0ull;
  named_bar(1, NCT);
  // rank by counting (keys are unique: the low bits hold the slot)
  for (int i = ct; i < n_all; i += NCT) {
    const uint64_t ki = keys[i];
    if (ki == ~0ull) continue;
    int rank = 0;
    for (int j = 0; j < n_all; ++j) rank += keys[j] < ki;
    if (rank < st.nb) {
      sorted[rank] = cands[i];
      atomicAdd(&misc[0], 1);
    }
  }
  named_bar(1, NCT);
  const int n_keep = misc[0];
  // kept nodes waiting for expansion (not expanded yet, depth < Bk)
  if (ct < 32) {
    const int lane = ct;
    int prefix = 0;
    for (int c0 = 0; c0 < n_keep; c0 += 32) {
      const int i = c0 + lane;
      const bool wt = i < n_keep && !sorted[i].expanded && sorted[i].depth < Bk;
      const unsigned bal = __ballot_sync(0xffffffffu, wt);
      if (i < n_keep) s_pos[i] = wt ? prefix + __popc(bal & ((1u << lane) - 1)) : -1;
      prefix += __popc(bal);
    }
    if (lane == 0) {
      const int base = misc[1];
      if (prefix && base + prefix > nt) {
        set_status(a.status, DT_EDEVICE);
        prefix = 0;
      }
      misc[1] = base + prefix;
      misc[3] = prefix;
      misc[4] = base;
    }
  }
  named_bar(1, NCT);
  const int m_next = misc[3];
  if (m_next > 0) {
    const int base = misc[4];
    for (int i = ct; i < n_keep; i += NCT) {
      if (s_pos[i] < 0) continue;
      const Cand c = sorted[i];
      Row rw;
      rw.b = b;
      rw.depth = c.depth;
      rw.token = p_markov_token(a, b, c.depth, c.token);
      rw.aux = c.serial;
      rw.path = c.path;
      rw.lse = 0.f;
      rw.key = c.key;
      nxt[base + s_pos[i]] = rw;
      sorted[i].expanded = 1;
    }
  } else {
    // the tree is final: parents by serial, ancestor masks, pop order
    for (int i = ct; i < n_keep; i += NCT) {
      const Cand c = sorted[i];
      int par = -1;
      if (c.parent_serial >= 0) {
        for (int p = 0; p < i; ++p)
          if (sorted[p].serial == c.parent_serial) par = p;
        if (par < 0) set_status(a.status, DT_EDEVICE);
      }
      s_par[i] = par;
    }
    named_bar(1, NCT);
    if (writer) {
      const size_t ob = (size_t)b * Nmax;
      for (int i = ct; i < n_keep; i += NCT) {
        const Cand c = sorted[i];
        uint64_t anc = 1ull << i;
        for (int p = s_par[i], hops = 0; p >= 0 && hops < 64; p = s_par[p], ++hops)
          anc |= 1ull << p;
        a.out.d_tokens[ob + i] = c.token;
        a.out.d_parents[ob + i] = s_par[i];
        a.out.d_depths[ob + i] = c.depth;
        a.out.d_ranks[ob + i] = c.rank;
        a.out.d_keys[ob + i] = c.key;
        a.out.d_anc[ob + i] = anc;
      }
    }
    if (a.temp > 0.f) {
      // draft rows of the accept walk: the root (row 0) and every inner node
      if (ct < 32) {
        const int lane = ct;
        int prefix = 1;
        for (int c0 = 0; c0 < n_keep; c0 += 32) {
          const int i = c0 + lane;
          const bool in = i < n_keep && sorted[i].depth < Bk;
          const unsigned bal = __ballot_sync(0xffffffffu, in);
          if (i < n_keep) s_pos[i] = in ? prefix + __popc(bal & ((1u << lane) - 1)) : -1;
          prefix += __popc(bal);
        }
        if (lane == 0) {
          misc[4] = misc[2];
          misc[2] += prefix;
        }
      }
      named_bar(1, NCT);
      const int mbase = misc[4];
      if (writer) {
        for (int i = ct - 1; i < n_keep; i += NCT) {
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
          Row rw;
          rw.b = b;
          rw.depth = depth;
          rw.token = p_markov_token(a, b, depth, token);
          rw.aux = aux;
          rw.path = 0;
          rw.lse = lse;
          rw.key = 0.f;
          a.mat_rows[mbase + pos] = rw;
        }
      }
    }
  }
  named_bar(1, NCT);
  for (int i = ct; i < n_keep; i += NCT) lb[i] = sorted[i];
  if (ct == 0) {
    st.n_list = n_keep;
    if (m_next > 0) {
      st.serial_next += n_new;
      st.row_base = misc[4];
      st.row_count = m_next;
    } else {
      st.done = 1;
      st.row_count = 0;
      if (writer) a.out.d_n_nodes[b] = n_keep;
    }
  }
  named_bar(1, NCT);
}

}  // namespace dt

namespace dt {

template <int NG, bool STOCH, int KMAX>
__global__ void __launch_bounds__(PShape<NG>::kThreads, 1)
    pbuild_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmW128,
                  const PBuildArgs a) {
  using S = PShape<NG>;
  constexpr int NT = S::NT, NCT = S::kCompute;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int esz = a.l_bf16 ? 2 : 4;
  const PLayout lay =
      p_layout<NG>(a.stages, a.r, a.k, a.Nmax, a.batch, a.Bk, a.span, esz, KMAX, STOCH);
  const int bstride = p_bias_stride(a.span, esz);
  uint8_t* aop = smem + lay.a;  // node rows A[token]: [KC][NT][128 B], 128-byte swizzle
  uint8_t* stage_mem = smem + lay.stage;
  uint64_t* full = (uint64_t*)(smem + lay.bars);
  uint64_t* empty = full + a.stages;
  uint64_t* tfull = empty + a.stages;
  uint64_t* tempty = tfull + S::kAccBufs;
  uint64_t* drain = tempty + S::kAccBufs;
  uint32_t* tmem_slot = (uint32_t*)(smem + lay.flags);
  volatile int* abort_flag = (volatile int*)(smem + lay.flags + 4);
  volatile int* done_flag = (volatile int*)(smem + lay.flags + 8);
  // pass w >= 1 of the producer (the weights of wave w) starts once phase
  // w - 1 of this barrier is complete: the compute warps complete one phase
  // per wave, after reading that wave's merged rows
  uint64_t* gate = drain + 1;
  Row* rows_buf[2] = {(Row*)(smem + lay.rows0), (Row*)(smem + lay.rows1)};
  PMeta* meta = (PMeta*)(smem + lay.meta);
  uint8_t* bias_cache = smem + lay.bias;  // [batch * Bk][bstride], the element type of L
  Cand* lists = (Cand*)(smem + lay.lists);
  Cand* cands = (Cand*)(smem + lay.cands);
  Cand* sorted = (Cand*)(smem + lay.sorted);
  uint64_t* keys = (uint64_t*)(smem + lay.keys);
  float* r_lse = (float*)(smem + lay.rlse);
  float* r_lq = (float*)(smem + lay.rlq);
  int32_t* r_tok = (int32_t*)(smem + lay.rtok);
  int* s_pos = (int*)(smem + lay.spos);
  int* s_par = (int*)(smem + lay.spar);
  float* msv = (float*)(smem + lay.msv);
  int32_t* msi = (int32_t*)(smem + lay.msi);
  float* exch = (float*)(smem + lay.exch);
  // misc: [0] kept count, [1] next-wave rows, [2] draft rows, [3] waiting rows of
  // a request, [4] its base, [5] rows of this wave, [6] abort snapshot
  int* misc = (int*)(smem + lay.misc);
  ReqState* reqs = (ReqState*)(smem + lay.req);

  const int cx = blockIdx.x, ncta = gridDim.x;
  const bool writer = cx == 0;
  // this CTA's range: 128-row tiles [t0, t0 + n128), as MMA tiles of 256 rows
  // (and one of 128 rows when n128 is odd)
  const int base_t = a.n_vtiles / ncta, extra = a.n_vtiles % ncta;
  const int t0 = cx * base_t + min(cx, extra);
  const int n128 = base_t + (cx < extra ? 1 : 0);
  const int n_mt = (n128 + 1) >> 1;
  const bool odd = (n128 & 1) != 0;
  const int KC = (a.r + 63) >> 6;
  const int ks_last = (((a.r - 1) & 63) >> 4) + 1;
  const int per_wave = n_mt * KC;  // stages of one pass over this CTA's range
  const int x0 = t0 * kTileV;
  const int x1 = min((t0 + n128) * kTileV, a.V);
  const int k = a.k;

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < S::kAccBufs; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], S::kEpiWarps);
    }
    mbar_init(drain, 1);
    mbar_init(gate, 1);
    *abort_flag = 0;
    *done_flag = 0;
    fence_barrier_init();
  }
  if (warp == S::kWarpProd && lane == 0) {
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmW128);
  }
  if (warp == S::kWarpMma) {
    tmem_alloc(tmem_slot, S::kTmemCols);
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == S::kWarpProd) {
    // ---------------------------------------------------------------- producer
    // Streams this CTA's range of Bm over and over, one pass per wave, as
    // far ahead as the ring allows; stops when the build is over.
    if (lane == 0) {
      const uint64_t pol = l2_evict_last_policy();
      uint32_t issued = 0, last_par = 0;
      for (uint32_t g = 0;; ++g) {
        const int stage = (int)(g % (uint32_t)a.stages);
        const uint32_t ph = (g / (uint32_t)a.stages) & 1u;
        bool got = mbar_try_wait(&empty[stage], ph ^ 1);
        if (!got) {
          const uint64_t tw = globaltimer_ns();
          while (!(got = mbar_try_wait_sleep(&empty[stage], ph ^ 1))) {
            if (*done_flag || *abort_flag) break;
            if (globaltimer_ns() - tw > a.wait_ns) {
              *abort_flag = 1;
              set_status(a.status, DT_ETIMEOUT);
              atomicExch(a.grid_abort, 1);
              break;
            }
          }
        }
        if (!got || *done_flag || *abort_flag) break;
        const int i = (int)(g % (uint32_t)per_wave);
        if (i == 0 && g > 0) {
          // a pass starts only when the compute warps open it: the merge's
          // global loads of the previous wave must not queue behind it
          const uint32_t pass = g / (uint32_t)per_wave;
          const uint64_t tw = globaltimer_ns();
          bool open = false;
          while (!(open = mbar_try_wait_sleep(gate, (pass - 1) & 1u))) {
            if (*done_flag || *abort_flag) break;
            if (globaltimer_ns() - tw > a.wait_ns) {
              *abort_flag = 1;
              set_status(a.status, DT_ETIMEOUT);
              atomicExch(a.grid_abort, 1);
              break;
            }
          }
          if (!open || *done_flag || *abort_flag) break;
        }
        const int j = i / KC, kc = i % KC;
        const bool half = odd && j == n_mt - 1;  // the 128-row tile
        const int y = (t0 + 2 * j) * kTileV;
        uint8_t* sa = stage_mem + (size_t)stage * S::kStageBytes;
        mbar_arrive_expect_tx(&full[stage], half ? S::kStageBytes / 2 : S::kStageBytes);
        tma_load_2d_hint(sa, half ? &tmW128 : &tmW, &full[stage], kc * 64, y, pol);
        issued |= 1u << stage;
        last_par = (last_par & ~(1u << stage)) | (ph << stage);
      }
      // let the copies in flight land before the CTA exits (bounded)
      const uint64_t tw = globaltimer_ns();
      for (int st = 0; st < a.stages; ++st) {
        if (!((issued >> st) & 1u)) continue;
        while (!mbar_try_wait(&full[st], (last_par >> st) & 1u) &&
               globaltimer_ns() - tw < 50000000ull) {
        }
      }
    }
  } else {
    // every warp but the producer; ct numbers their threads
    const int ct = threadIdx.x < 32 * S::kWarpProd ? threadIdx.x : threadIdx.x - 32;
    // ---------------------------------------------------------------- set-up
    // block-logit rows of every (request, depth) over [x0, x1), once
    {
      const int nrow = a.batch * a.Bk;
      const int nx = x1 - x0;
      const bool vec = ((uintptr_t)a.L % 16 == 0) && (((size_t)a.V * esz) % 16 == 0);
      if (vec) {
        const int np = nx * esz / 16;  // whole: x0 and V are multiples of 16 bytes here
        for (int idx = ct; idx < nrow * np; idx += NCT) {
          const int u = idx / np, i = idx % np;
          cp_async16_g2s(bias_cache + ((size_t)u * bstride * esz + (size_t)i * 16),
                         (const uint8_t*)a.L + ((size_t)u * a.V + x0) * esz + (size_t)i * 16);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
      } else {
        for (int idx = ct; idx < nrow * nx; idx += NCT) {
          const int u = idx / nx, i = idx % nx;
          if (esz == 2)
            ((uint16_t*)bias_cache)[(size_t)u * bstride + i] =
                ((const uint16_t*)a.L)[(size_t)u * a.V + x0 + i];
          else
            ((float*)bias_cache)[(size_t)u * bstride + i] =
                ((const float*)a.L)[(size_t)u * a.V + x0 + i];
        }
      }
    }
    // request state (the same in every CTA)
    for (int b = ct; b < a.batch; b += NCT) {
      ReqState st;
      st.n_list = 0;
      st.serial_next = 0;
      st.done = 0;
      st.row_base = 0;
      st.row_count = 0;
      st.root_lse = 0.f;
      int root = a.root_token[b];
      if (root < 0 || root >= a.V) {
        set_status(a.status, DT_EDEVICE);
        root = 0;
      }
      st.root_token = root;
      st.pad[0] = st.pad[1] = 0;
      int kb = a.k_req ? a.k_req[b] : a.k;
      if (kb < 1 || kb > a.k) {
        set_status(a.status, DT_EDEVICE);
        kb = kb < 1 ? 1 : a.k;
      }
      st.kb = kb;
      const float lam = a.lambda[b];
      st.thr = (lam > 0.f) ? (float)log((double)lam) : -INFINITY;
      int nb = a.n_budget[b];
      if (nb > a.Nmax) {
        set_status(a.status, DT_EDEVICE);
        nb = a.Nmax;
      }
      st.nb = nb < 0 ? 0 : nb;
      if (st.nb == 0) {
        st.done = 1;
        if (writer) a.out.d_n_nodes[b] = 0;
      }
      reqs[b] = st;
    }
    if (ct == 0) {
      misc[1] = misc[2] = 0;
      misc[6] = 0;
    }
    named_bar(1, NCT);
    if (ct == 0) {
      // wave 1: the roots of the requests with a budget, in request order
      int n = 0;
      for (int b = 0; b < a.batch; ++b) {
        if (reqs[b].done) continue;
        Row rw;
        rw.b = b;
        rw.depth = 0;
        rw.token = p_markov_token(a, b, 0, reqs[b].root_token);
        rw.aux = -1;
        rw.path = 0;
        rw.lse = 0.f;
        rw.key = 0.f;
        rows_buf[0][n] = rw;
        reqs[b].row_base = n;
        reqs[b].row_count = 1;
        ++n;
      }
      misc[5] = n;
    }

    // pipeline positions carried across waves by the threads that own them
    int m_stage = 0;
    uint32_t m_phase = 0, m_tile = 0, e_tile = 0;  // tile n uses accumulator n % kAccBufs
    const int cw = warp < S::kWarpProd ? warp : warp - 1;  // compute-warp index
    int cur = 0;
    for (int wave = 0;; ++wave) {
      named_bar(1, NCT);
      const int n_rows = misc[5];
      if (n_rows == 0 || misc[6]) break;  // uniform (shared memory after a barrier)
      Row* rows = rows_buf[cur];
      // A wave of at most 32 node rows runs in the one-group layout even in
      // the 64-row kernel: its rows replicated four times, so that all eight
      // epilogue warps share 32 nodes instead of half of them idling on an
      // empty second node group.
      const int ge = (NG == 2 && n_rows > 32) ? 2 : 1;  // node groups of this wave
      const int nte = 32 * ge;                          // node rows per replica
      const int re = 4 / ge;                            // replicas down the 128 A rows
      const int parts = 2 * re;                         // column parts per node group
      const int pcols = S::kTileN / parts;              // columns per part (= nte)
      // ---- this wave's node rows, and their Markov rows A[token] as the A operand
      for (int c = ct; c < NT; c += NCT) {
        PMeta m;
        m.valid = 0;
        m.b = 0;
        m.bslot = 0;
        m.c1 = m.c2 = 0;
        m.pad[0] = m.pad[1] = m.pad[2] = 0;
        if (c < n_rows) {
          const Row rw = rows[c];
          m.valid = 1;
          m.b = rw.b;
          m.bslot = rw.b * a.Bk + rw.depth;
          m.c1 = (uint32_t)rw.path;
          m.c2 = (uint32_t)(rw.path >> 32);
          // token -1: no Markov term (zero row); anything else must index A
          if (rw.token < -1 || rw.token >= a.V) {
            set_status(a.status, DT_EDEVICE);
            m.valid = 0;
          }
        }
        meta[c] = m;
      }
      named_bar(1, NCT);
      {
        // rows 0 .. nte-1 of every chunk from global memory
        const int npieces = KC * nte * 8;
        for (int idx = ct; idx < npieces; idx += NCT) {
          const int ch = idx & 7, c = (idx >> 3) % nte, kc = (idx >> 3) / nte;
          const int col_k = kc * 64 + ch * 8;
          const int tok = c < n_rows ? rows[c].token : -1;
          const bool ok = meta[c].valid && tok >= 0 && col_k < a.r;
          const uint16_t* src = ok ? a.A + (size_t)tok * a.r + col_k : a.A;
          uint8_t* dst = aop + ((size_t)kc * 128 + c) * 128 + ((ch ^ (c & 7)) << 4);
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)),
                       "l"(src), "r"(ok ? 16 : 0)
                       : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        asm volatile("cp.async.wait_all;" ::: "memory");
      }
      named_bar(1, NCT);
      {
        // A row i (of 128) is node i % nte: the replicas are byte copies of
        // rows 0 .. nte-1 (nte is a multiple of the 8-row swizzle period)
        const int per = nte * 128 / 16;  // 16-byte pieces of one replica of a chunk
        const int n = KC * (re - 1) * per;
        for (int idx = ct; idx < n; idx += NCT) {
          const int kc = idx / ((re - 1) * per);
          const int rr = 1 + (idx / per) % (re - 1);
          const int pc = idx % per;
          const uint4* src = (const uint4*)(aop + (size_t)kc * 128 * 128) + pc;
          uint4* dst = (uint4*)(aop + (size_t)kc * 128 * 128 + (size_t)rr * nte * 128) + pc;
          *dst = *src;
        }
        // the tensor cores read these bytes through the async proxy
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
      named_bar(1, NCT);
      if (warp == S::kWarpMma) {
        // ---------------------------------------------------------- MMA issuer
        // D[i][x] (+)= A[i][k] . Bm[x][k] over the K chunks of a tile:
        // M = 128 rows (R replicas of the NT node rows), N = 256 vocabulary rows.
        if (lane == 0) {
          constexpr uint32_t idesc_full = idesc_bf16_f32(kTileV, S::kTileN);
          constexpr uint32_t idesc_half = idesc_bf16_f32(kTileV, S::kTileN / 2);
          bool ok = true;
          for (int j = 0; j < n_mt && ok; ++j) {
            const int ab = (int)(m_tile % S::kAccBufs);
            if (!p_wait(&tempty[ab], ((m_tile / S::kAccBufs) & 1u) ^ 1u, a, abort_flag)) break;
            tc_fence_after();
            const uint32_t idesc = (odd && j == n_mt - 1) ? idesc_half : idesc_full;
            const uint32_t d_tmem = tmem_base + (uint32_t)(ab * S::kTileN);
            for (int kc = 0; kc < KC; ++kc) {
              if (!p_wait(&full[m_stage], m_phase, a, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint64_t da = smem_desc_k_sw128(smem_u32(aop + (size_t)kc * 128 * 128));
              const uint64_t db =
                  smem_desc_k_sw128(smem_u32(stage_mem + (size_t)m_stage * S::kStageBytes));
              const int ks = (kc == KC - 1) ? ks_last : 4;
              for (int s = 0; s < ks; ++s)
                tc_mma_bf16(d_tmem, da + 2 * s, db + 2 * s, idesc, (kc | s) != 0 ? 1u : 0u);
              tc_commit(&empty[m_stage]);
              if (++m_stage == a.stages) {
                m_stage = 0;
                m_phase ^= 1;
              }
            }
            if (!ok) break;
            tc_commit(&tfull[ab]);
            ++m_tile;
          }
        }
        __syncwarp();
      } else if (warp < S::kEpiWarps) {
        // ------------------------------------------------ epilogue (node rows)
        // Lane = node 32 g + lane of node group g, in quadrant q (replica
        // q / NG); this warp reduces column part p of every tile (NT columns,
        // in blocks of 32 read straight from TMEM).  Per node: bias from the
        // cache, 1/T, an online max / sum-exp, the top-k of s (ties to the
        // lower token) and, at T > 0, the Gumbel-top-k of s + G.
        const int q = warp & 3;
        const int c = 32 * (q % ge) + lane;
        const int part = (q / ge) * 2 + (warp >> 2);
        const float temp = a.temp;
        const PMeta mc = meta[c];
        const bool any = __any_sync(0xffffffffu, mc.valid) != 0;
        float m = -INFINITY, ssum = 0.f, thr = -INFINITY, gthr = -INFINITY;
        float L1[KMAX], L2[KMAX];
        int32_t I1[KMAX], I2[KMAX];
#pragma unroll
        for (int i = 0; i < KMAX; ++i) {
          L1[i] = L2[i] = -INFINITY;
          I1[i] = I2[i] = 0x7fffffff;
        }
        for (int j = 0; j < n_mt; ++j) {
          // one lane waits; the warp follows it as one (tcgen05.ld is warp-wide)
          __syncwarp();
          const int ab = (int)(e_tile % S::kAccBufs);
          int ok = 1;
          if (lane == 0) ok = p_wait(&tfull[ab], (e_tile / S::kAccBufs) & 1u, a, abort_flag) ? 1 : 0;
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          tc_fence_after();
          // the 128-row tile at the end of an odd range has columns 0-127 only
          const bool has_part = !(odd && j == n_mt - 1) || part * pcols < kTileV;
          if (any && has_part) {
#pragma unroll 1
            for (int c4 = 0; c4 < pcols / 32; ++c4) {
              __syncwarp();
              const int col = part * pcols + 32 * c4;  // within the tile
              const int xq = (t0 + 2 * j) * kTileV + col;    // first token of the block
              const int nv = min(32, a.V - xq);
              float acc[32];
              tmem_ld32(tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(ab * S::kTileN + col),
                        acc);
              if (!mc.valid || nv <= 0) continue;
              float bias[32];
              const size_t ci = (size_t)mc.bslot * bstride + (size_t)(xq - x0);
              if (nv == 32) {
                uint4 cr[8];
                const uint4* src = (const uint4*)(bias_cache + ci * esz);
#pragma unroll
                for (int cc = 0; cc < 8; ++cc)
                  if (cc < 4 || !a.l_bf16) cr[cc] = src[cc];
                decode_bias(cr, a.l_bf16, bias);
              } else {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                  bias[i] = i < nv ? (a.l_bf16 ? bf16_to_f32(((const uint16_t*)bias_cache)[ci + i])
                                               : ((const float*)bias_cache)[ci + i])
                                   : 0.f;
              }
              float sv[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const float z = acc[i] + bias[i];
                sv[i] = i < nv ? (STOCH ? __fdiv_rn(z, temp) : z) : -INFINITY;
              }
              float mx[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) mx[i] = fmaxf(sv[i], sv[i + 16]);
#pragma unroll
              for (int w = 8; w; w >>= 1)
#pragma unroll
                for (int i = 0; i < w; ++i) mx[i] = fmaxf(mx[i], mx[i + w]);
              const float mt = mx[0];
              float ex[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) ex[i] = ex2_approx((sv[i] - mt) * kLog2e);
#pragma unroll
              for (int w = 16; w; w >>= 1)
#pragma unroll
                for (int i = 0; i < w; ++i) ex[i] += ex[i + w];
              const float st = ex[0];
              if (mt > m) {
                ssum = ssum * ex2_approx((m - mt) * kLog2e) + st;
                m = mt;
              } else {
                ssum += st * ex2_approx((mt - m) * kLog2e);
              }
              if constexpr (STOCH) {
                // Gumbel keys; four consecutive tokens share one Philox counter.
                // The block's eight draws are independent and issued together;
                // the exact key is computed only where it may beat the bar.
                if (mt + kGumbelMax > gthr) {
                  uint32_t wds[32];
#pragma unroll
                  for (int gi = 0; gi < 8; ++gi) {
                    const uint32_t x4 = (uint32_t)(xq + 4 * gi);
                    const U4 o =
                        philox10(U4{(x4 >> 2) | ((uint32_t)mc.b << 18), mc.c1, mc.c2, a.offset},
                                 (uint32_t)a.seed, (uint32_t)(a.seed >> 32));
                    wds[4 * gi] = o.x;
                    wds[4 * gi + 1] = o.y;
                    wds[4 * gi + 2] = o.z;
                    wds[4 * gi + 3] = o.w;
                  }
#pragma unroll
                  for (int i = 0; i < 32; ++i) {
                    if (i < nv && gumbel_may_beat(sv[i], gthr, wds[i])) {
                      const float gk = sv[i] + (-logf(-logf(u23(wds[i]))));
                      if (gk > gthr) {
                        topk_insert<KMAX>(L2, I2, gk, xq + i);
                        gthr = kth<KMAX>(L2, k);
                      }
                    }
                  }
                }
              }
              // top-k of s: while the block's best left beats the k-th best so
              // far (at most k rounds), insert it (lowest token among equal
              // values first) and take it out of the block
              if (mt > thr) {
                float bm = mt;
#pragma unroll 1
                for (int rd = 0; rd < k && bm > thr; ++rd) {
                  uint32_t eq = 0;
#pragma unroll
                  for (int i = 0; i < 32; ++i) eq |= (sv[i] == bm ? 1u : 0u) << i;
                  const int ix = __ffs(eq) - 1;
                  topk_insert<KMAX>(L1, I1, bm, xq + ix);
                  thr = kth<KMAX>(L1, k);
#pragma unroll
                  for (int i = 0; i < 32; ++i) sv[i] = (i == ix) ? -INFINITY : sv[i];
#pragma unroll
                  for (int i = 0; i < 16; ++i) mx[i] = fmaxf(sv[i], sv[i + 16]);
#pragma unroll
                  for (int w = 8; w; w >>= 1)
#pragma unroll
                    for (int i = 0; i < w; ++i) mx[i] = fmaxf(mx[i], mx[i + w]);
                  bm = mx[0];
                }
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[ab]);
          ++e_tile;
        }
        // every part's partial of every node into the exchange, then one
        // thread per node merges them into the CTA's partial of the node
        constexpr int kEx = 2 + 2 * KMAX * (STOCH ? 2 : 1);  // words per (part, node)
        {
          float* mine = exch + ((size_t)part * nte + c) * kEx;
          mine[0] = m;
          mine[1] = ssum;
#pragma unroll
          for (int i = 0; i < KMAX; ++i) {
            mine[2 + i] = L1[i];
            mine[2 + KMAX + i] = __int_as_float(I1[i]);
            if (STOCH) {
              mine[2 + 2 * KMAX + i] = L2[i];
              mine[2 + 3 * KMAX + i] = __int_as_float(I2[i]);
            }
          }
        }
        named_bar(2, S::kEpiWarps * 32);
        const int cn = threadIdx.x;  // node merged by this thread
        if (cn < nte && meta[cn].valid) {
          const int par = wave & 1;
          float mx = -INFINITY;
          for (int pp = 0; pp < parts; ++pp)
            mx = fmaxf(mx, exch[((size_t)pp * nte + cn) * kEx]);
          float sv = 0.f;
          if (mx != -INFINITY)
            for (int pp = 0; pp < parts; ++pp) {
              const float* e = exch + ((size_t)pp * nte + cn) * kEx;
              if (e[0] != -INFINITY) sv += e[1] * exp2f((e[0] - mx) * kLog2e);
            }
          a.pstats[par][(size_t)cn * ncta + cx] = make_float2(mx, sv);
          for (int lst = 0; lst < (STOCH ? 2 : 1); ++lst) {
            float* OV = (lst ? a.pgv[par] : a.plv[par]) + (size_t)cn * k * ncta + cx;
            int32_t* OI = (lst ? a.pgi[par] : a.pli[par]) + (size_t)cn * k * ncta + cx;
            const int off = 2 + (lst ? 2 * KMAX : 0);
            constexpr int kPartsMax = 8;  // parts of the one-group layout
            int hd[kPartsMax];            // heads of the parts' sorted lists
#pragma unroll
            for (int pp = 0; pp < kPartsMax; ++pp) hd[pp] = 0;
            for (int i = 0; i < k; ++i) {
              int bw = 0;
              float bv = -INFINITY;
              int32_t bi = 0x7fffffff;
              bool have = false;
#pragma unroll
              for (int pp = 0; pp < kPartsMax; ++pp) {
                if (pp >= parts || hd[pp] >= k) continue;
                const float* e = exch + ((size_t)pp * nte + cn) * kEx + off;
                const float v = e[hd[pp]];
                const int32_t id = __float_as_int(e[KMAX + hd[pp]]);
                if (!have || ranks_first(v, id, bv, bi)) {
                  have = true;
                  bw = pp;
                  bv = v;
                  bi = id;
                }
              }
#pragma unroll
              for (int pp = 0; pp < kPartsMax; ++pp) hd[pp] += (pp == bw) ? 1 : 0;
              OV[(size_t)i * ncta] = bv;
              OI[(size_t)i * ncta] = bi;
            }
          }
        }
      }
      named_bar(1, NCT);
      // ---- every CTA's partials of this wave are written: meet, bounded
      if (ct == 0) {
        const bool arrive = !(wave == 0 && cx == a.stall_cta);
        if (!*abort_flag) grid_sync(a, 2u * wave, arrive, abort_flag);
        if (*abort_flag) atomicExch(a.grid_abort, 1);
        misc[6] = *abort_flag;
        misc[1] = 0;
      }
      named_bar(1, NCT);
      if (misc[6]) break;
      // ---- merge: node row e is merged by one warp of CTA e % ncta, which
      // alone reads the row's ncta partials (148 CTAs reading the same lines
      // at once would queue on the same L2 slices).  Per row: its log-sum-exp
      // and the kb best values of s with their tokens (T = 0) or the tokens
      // of its Gumbel sample (T > 0), into the merged-row buffer.
      {
        const int par = wave & 1;
        for (int e = cx + cw * ncta; cw < S::kMergeWarps && e < n_rows;
             e += ncta * S::kMergeWarps) {
          const Row rw = rows[e];
          const int kb = reqs[rw.b].kb;
          const size_t prow = (size_t)e * ncta;
          const float lse = merge_node<KMAX>(
              a.pstats[par] + prow, a.plv[par] + prow * k, a.pli[par] + prow * k,
              STOCH ? a.pgv[par] + prow * k : nullptr, STOCH ? a.pgi[par] + prow * k : nullptr,
              ncta, k, kb, lane, a.mrg_val + (size_t)e * k,
              STOCH ? nullptr : a.mrg_tok + (size_t)e * k, STOCH ? a.mrg_tok + (size_t)e * k : nullptr,
              msv + cw * 32, msi + cw * 32);
          if (lane == 0) a.mrg_lse[e] = lse;
          __syncwarp();
        }
      }
      named_bar(1, NCT);
      if (ct == 0) {
        if (!*abort_flag) grid_sync(a, 2u * wave + 1, true, abort_flag);
        if (*abort_flag) atomicExch(a.grid_abort, 1);
        misc[6] = *abort_flag;
      }
      named_bar(1, NCT);
      if (misc[6]) break;
      // ---- every CTA reads the merged rows: log q of the kb best, tokens
      for (int idx = ct; idx < n_rows * k; idx += NCT) {
        const int e = idx / k, j = idx % k;
        const float lse = __ldcg(a.mrg_lse + e);
        r_lq[idx] = __ldcg(a.mrg_val + idx) - lse;
        r_tok[idx] = __ldcg(a.mrg_tok + idx);
        if (j == 0) r_lse[e] = lse;
      }
      named_bar(1, NCT);
      // the weights of the next wave may stream while the selection runs
      if (ct == 0) mbar_arrive(gate);
      // ---- best-first selection, request by request (the same in every CTA)
      for (int b = 0; b < a.batch; ++b)
        p_select<NCT>(a, b, reqs, lists, cands, sorted, keys, r_lse, r_lq, r_tok, rows,
                      rows_buf[cur ^ 1], min(NT, a.batch * a.Nmax), s_pos, s_par, misc, ct,
                      writer);
      if (ct == 0) misc[5] = misc[1];
      cur ^= 1;
    }  // waves
    // the build is over (or was abandoned): the producer stops
    if (ct == 0) {
      *done_flag = 1;
      // the producer may be suspended on the gate or on a ring slot that no
      // MMA will free any more: complete those phases so that it wakes, sees
      // the flag and stops (every MMA of the build has completed by now)
      mbar_arrive(gate);
      for (int st = 0; st < a.stages; ++st) mbar_arrive(&empty[st]);
      if (writer && STOCH && !misc[6]) *a.mat_count = misc[2];
      // The last CTA out resets the barrier words for the next launch on this
      // workspace: every CTA has left its last barrier wait by then.
      unsigned* exits = a.grid_bar + 2;
      __threadfence();
      if (atomicAdd(exits, 1u) == (unsigned)ncta - 1) {
        atomicExch(a.grid_bar, 0u);
        atomicExch(a.grid_abort, 0);
        atomicExch(exits, 0u);
      }
    }
    if (warp == S::kWarpMma && lane == 0) {
      // every MMA this thread issued has completed before TMEM is released
      tc_commit(drain);
      const uint64_t tw = globaltimer_ns();
      while (!mbar_try_wait(drain, 0) && globaltimer_ns() - tw < 50000000ull) {
      }
    }
  }
  __syncthreads();
  if (warp == S::kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem_base, S::kTmemCols);
  }
}

}  // namespace dt

namespace dt {

// ---------------------------------------------------------------- host side --
int gemm_kmax(int k);
bool make_tmap_bf16_kmajor(CUtensorMap* map, const void* base, uint64_t K, uint64_t rows,
                           uint32_t box_rows);

// Node rows of a persistent build of this shape (every wave fits one MMA
// tile of them), or 0 when the build runs as one launch pair per wave.
int pbuild_cols(int batch, int Nmax, int r) {
  const long long m = (long long)batch * Nmax;
  const int nt = m <= 32 ? 32 : m <= 64 ? 64 : 0;
  return (nt && r <= 512) ? nt : 0;
}

template <int NG, bool STOCH, int KMAX>
static cudaError_t pbuild_cfg(const CUtensorMap& tmW, const CUtensorMap& tmW128, PBuildArgs a,
                              int ncta, cudaStream_t s) {
  using S = PShape<NG>;
  auto kern = pbuild_kernel<NG, STOCH, KMAX>;
  const int esz = a.l_bf16 ? 2 : 4;
  int dev = 0, optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return cudaErrorInvalidDevice;
  // the deepest stage ring (32 KB stages) that fits next to everything else
  int stages = 8;
  size_t bytes = 0;
  for (; stages >= 2; --stages) {
    bytes = p_layout<NG>(stages, a.r, a.k, a.Nmax, a.batch, a.Bk, a.span, esz, KMAX, STOCH).total +
            1024;
    if (bytes <= (size_t)optin) break;
  }
  if (stages < 2) return cudaErrorNotSupported;
  a.stages = stages;
  cudaError_t e = ensure_smem(kern, bytes);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, S::kThreads, bytes);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorNotSupported;
  // every CTA waits for every other at the grid barriers: co-residency is
  // what a cooperative launch guarantees (or it fails to launch)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ncta);
  cfg.blockDim = dim3(S::kThreads);
  cfg.dynamicSmemBytes = bytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tmW, tmW128, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// One cooperative launch for the whole build (see the top of this file).
// Returns cudaErrorNotSupported, with nothing enqueued, when the shape does
// not fit it.  Bm [V][r] bf16 is streamed in tiles of 256 (and 128) rows.
cudaError_t launch_pbuild(const uint16_t* d_markov_b, PBuildArgs a, int ncta, cudaStream_t s) {
  const int nt = pbuild_cols(a.batch, a.Nmax, a.r);
  if (!nt || ncta < 1) return cudaErrorNotSupported;
  CUtensorMap tmW, tmW128;
  if (!make_tmap_bf16_kmajor(&tmW, d_markov_b, a.r, a.V, 256) ||
      !make_tmap_bf16_kmajor(&tmW128, d_markov_b, a.r, a.V, 128))
    return cudaErrorInvalidValue;
  a.span = ((a.n_vtiles + ncta - 1) / ncta) * kTileV;
  a.cap = a.Nmax + a.Nmax * a.k;
  const bool st = a.temp > 0.f;
  const int km = gemm_kmax(a.k);
#define DT_PB_CASE(NG, ST, KM)                  \
  if (nt == 32 * NG && st == ST && km == KM) \
    return pbuild_cfg<NG, ST, KM>(tmW, tmW128, a, ncta, s);
  DT_PB_CASE(1, false, 4)
  DT_PB_CASE(1, false, 16)
  DT_PB_CASE(1, true, 4)
  DT_PB_CASE(1, true, 16)
  DT_PB_CASE(2, false, 4)
  DT_PB_CASE(2, false, 16)
  DT_PB_CASE(2, true, 4)
  DT_PB_CASE(2, true, 16)
#undef DT_PB_CASE
  return cudaErrorNotSupported;
}

}  // namespace dt
