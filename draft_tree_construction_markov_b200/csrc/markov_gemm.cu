// Node-batched GEMMs on the 5th-generation tensor cores, with fused epilogues.
//
// Markov head (PCTree summary, DSpark paragraph: the Markov head biases the
// shared block logits by the previous token; here the previous token is the
// node's own token, i.e. the children are parent-conditioned).  For every
// GEMM column n (a tree node u with depth d and token t) and every vocabulary
// row x:
//   z[x][n] = L[b][d][x] + sum_rho Bm[x][rho] * A[t][rho]
// The same kernel serves the TreeFlash AR-approximator (TreeFlash explainer,
// method section 1): the SwiGLU gate/up projections, the down projection
// with the residual, and the LM head, whose columns are approximator rows.
//
// Swap-AB tcgen05 GEMM: the weight rows (vocabulary, or features) are the MMA
// M axis (128 rows per tile, streamed by TMA), node rows are the N axis (32,
// 64 or 256 per tile, also by TMA), K is the inner dimension.  The fp32
// accumulator lives in TMEM, two or four tiles deep, so the tensor pipe runs
// ahead of the epilogue.  Each CTA owns a contiguous range of weight tiles and
// one node tile; CTAs of the same range are adjacent in the grid, so the
// weight tiles that several node tiles share are re-read from L2.
//
// Epilogues:
//  * EXPAND (the hot path of both trees): four warps per 32 node columns read
//    the accumulator back with tcgen05.ld (each warp its 32-lane quadrant = 32
//    vocabulary rows) and transpose each 32 x 32 block through shared memory,
//    so every thread owns one node column and scans consecutive vocabulary
//    entries of it per tile (several lanes share a column when the block has
//    few live columns).  Per column it fuses the block-logit bias (prefetched
//    one tile ahead), the temperature, an online max / sum-exp, a private
//    top-k of s (ties to the lower token id) and, at T > 0, the
//    Gumbel-top-k of s + G (TreeSpark article, "lossless" section;
//    Gumbel-top-k: Kool, van Hoof and Welling 2019), one Philox call per four
//    consecutive tokens.  The CTA writes one partial result per node; a later
//    kernel merges the partials.
//  * ZDUMP: z (+ optional bias rows), fp32 or bf16, lane = weight row so that
//    stores coalesce.  Also the down projection + residual of TreeFlash.
//  * QROWS: q = exp(s - lse) rows of the final tree (T > 0).
//  * SWIGLU: a tile holds 64 gate rows (TMEM lanes 0-63) and the 64 up rows of
//    the same features (lanes 64-127); the up quadrants hand their values to
//    the gate quadrants through shared memory, which store silu(g) * u (bf16).
#include "build.cuh"
#include "epi_util.cuh"
#include "merge.cuh"

namespace dt {


// NG groups of 32 node columns per tile.  The epilogue serves EG groups at a
// time with four warps each (one per TMEM lane quadrant); each epilogue thread
// handles CPT groups of its quadrant in turn.
template <int NG>
struct GemmShape {
  static constexpr int NT = 32 * NG;  // MMA N: node columns per tile
  static constexpr int EG = NG < 2 ? NG : 2;
  static constexpr int CPT = NG / EG;
  static constexpr int kEpiWarps = 4 * EG;
  static constexpr int kThreads = 32 * (2 + kEpiWarps);
  static constexpr int kAccBufs = NG <= 2 ? 4 : 2;  // accumulator tiles in TMEM
  static constexpr int kABytes = kTileV * 128;      // 128 weight rows x 64 bf16
  static constexpr int kBBytes = NT * 128;          // NT node rows x 64 bf16
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr uint32_t kTmemCols = kAccBufs * NT;
  static_assert(NG == 1 || NG == 2 || NG == 8, "node tile of 32, 64 or 256 columns");
  static_assert(kTmemCols == 128 || kTmemCols == 256 || kTmemCols == 512,
                "TMEM allocation is a power of two");
};

struct ColMeta {
  int64_t bias_off;  // element offset of the column's bias row (block logits / residual)
  uint32_t c1, c2;   // Philox counter words 1-2 (path id)
  int32_t b;
  int32_t valid;
  float lse;
  int32_t out_row;
  int32_t bslot;     // row of the shared-memory bias cache (-1: not cached)
  int32_t token;     // the column's token (row of A gathered as the B operand)
};

// Most distinct bias rows a CTA keeps in shared memory for its vocabulary range.
constexpr int kBiasRowsMax = 32;

template <int NG>
__host__ __device__ inline size_t gemm_epi_bytes(int mode, int kmax, bool stoch) {
  using S = GemmShape<NG>;
  const size_t tbuf = (size_t)S::kEpiWarps * 32 * kTLD * 4;
  if (mode == EPI_SWIGLU) return tbuf;
  if (mode != EPI_EXPAND) return 0;
  // after the tile loop the transpose buffers hold the per-quadrant partials
  const size_t lists = (size_t)4 * S::NT * kmax * 8 * (stoch ? 2 : 1) + (size_t)4 * S::NT * 8;
  return tbuf > lists ? tbuf : lists;
}

template <int NG>
static size_t gemm_smem_bytes(int stages, int mode, int kmax, bool stoch, size_t bias_bytes,
                              size_t gather_bytes) {
  using S = GemmShape<NG>;
  size_t off = 1024;  // alignment slack
  off += gather_bytes ? (size_t)stages * S::kABytes + gather_bytes
                      : (size_t)stages * S::kStageBytes;
  off += (size_t)(2 * stages + 2 * S::kAccBufs + 5) * 8;  // barriers
  off += 16;                                             // tmem slot + abort flag
  off = (off + 15) & ~(size_t)15;
  off += (size_t)S::NT * sizeof(ColMeta) + 16 + kBiasRowsMax * 8;
  off += gemm_epi_bytes<NG>(mode, kmax, stoch);
  off = (off + 15) & ~(size_t)15;
  off += bias_bytes;
  return off;
}

template <int NG, int MODE, bool STOCH, int KMAX>
__global__ void __launch_bounds__(GemmShape<NG>::kThreads, 1)
    markov_gemm_kernel(const __grid_constant__ CUtensorMap tmW,
                       const __grid_constant__ CUtensorMap tmW2,
                       const __grid_constant__ CUtensorMap tmH, GemmArgs a, int batch) {
  using S = GemmShape<NG>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Node-tile slots fastest: the CTAs that share a weight range run side by
  // side.  The CTA of slot s handles node tiles s, s + n_nslots, ... up to the
  // column count of this launch, so a launch whose count is only known on
  // the device (a wave of the tree build) needs no CTA per possible tile.
  const int cx = blockIdx.x / a.n_nslots, slot = blockIdx.x % a.n_nslots;
  // Slot 0 has work whenever any node does: its CTAs set up and start
  // streaming weights before the previous kernel finishes.  CTAs of later
  // slots first check that they have columns at all.
  const bool early = slot == 0;
  int M = 0;
  if (!early) {
    pdl_wait();
    M = min(*a.n_rows, a.Mcap);
    if (slot * S::NT >= M) {
      pdl_launch_dependents();
      return;  // uniform over the CTA
    }
  }
  const int base = a.n_vtiles / a.ncta_v, extra = a.n_vtiles % a.ncta_v;
  const int t0 = cx * base + min(cx, extra);
  const int t1 = t0 + base + (cx < extra ? 1 : 0);
  const int KC = (a.r + 63) >> 6;
  const int ks_last = (((a.r - 1) & 63) >> 4) + 1;
  const int stages = a.stages;
  const int k = a.k;

  // Markov columns: the B operand rows A[token] are gathered once into shared
  // memory (resident for every stage) instead of streamed with each stage.
  const bool gather = a.gatherA != nullptr;
  const int sbytes = gather ? S::kABytes : S::kStageBytes;  // bytes per stage

  // ---- carve shared memory
  uint8_t* p = smem;
  uint8_t* stage_mem = p;
  p += (size_t)stages * sbytes;
  uint8_t* bres = p;  // gathered B rows: [KC][NT][128 B], 128-byte swizzle
  if (gather) p += (size_t)KC * S::NT * 128;
  uint64_t* full = (uint64_t*)p;
  uint64_t* empty = full + stages;
  uint64_t* tfull = empty + stages;
  uint64_t* tempty = tfull + S::kAccBufs;
  uint64_t* drain = tempty + S::kAccBufs;
  uint64_t* xfull = drain + 1;   // [2] SwiGLU: up values staged for column group eg
  uint64_t* xempty = xfull + 2;  // [2] SwiGLU: staged values consumed
  p = (uint8_t*)(xempty + 2);
  uint32_t* tmem_slot = (uint32_t*)p;
  volatile int* abort_flag = (volatile int*)(p + 4);
  p += 16;
  p = (uint8_t*)(((uintptr_t)p + 15) & ~(uintptr_t)15);
  ColMeta* meta = (ColMeta*)p;
  p += S::NT * sizeof(ColMeta);
  int* n_bias = (int*)p;  // distinct cached bias rows (-1: cache not used)
  p += 16;
  int64_t* brow = (int64_t*)p;  // [kBiasRowsMax] element offsets of the cached rows
  p += kBiasRowsMax * 8;
  float* tbuf = (float*)p;  // [kEpiWarps][32][kTLD]; EXPAND: then the quadrant partials
  p += gemm_epi_bytes<NG>(MODE, KMAX, STOCH);
  p = (uint8_t*)(((uintptr_t)p + 15) & ~(uintptr_t)15);
  // [kBiasRows][bias_span] values of the distinct bias rows over this CTA's
  // vocabulary range (same element type as L)
  uint8_t* bias_cache = p;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < S::kAccBufs; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], S::kEpiWarps);
    }
    mbar_init(drain, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&xfull[i], 64);
      mbar_init(&xempty[i], 64);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmW);
    if (MODE == EPI_SWIGLU) prefetch_tmap(&tmW2);
    prefetch_tmap(&tmH);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, S::kTmemCols);
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // The weight tiles do not depend on the previous kernel: the first stages
  // start streaming while it finishes (each stage's barrier also waits for
  // its node-row box, issued below once those rows exist).
  const int total = (t1 - t0) * KC;
  const int npre = early ? min(stages, total) : 0;
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < npre; ++i) {
      const int t = t0 + i / KC, kc = i % KC;
      uint8_t* sa = stage_mem + (size_t)i * sbytes;
      mbar_expect_tx(&full[i], S::kABytes);
      if (MODE == EPI_SWIGLU) {
        // 64 gate rows, then the 64 up rows of the same features
        tma_load_2d(sa, &tmW, &full[i], kc * 64, t * 64);
        tma_load_2d(sa + S::kABytes / 2, &tmW2, &full[i], kc * 64, t * 64);
      } else if (a.l2_keep) {
        tma_load_2d_hint(sa, &tmW, &full[i], kc * 64, t * kTileV, l2_evict_last_policy());
      } else {
        tma_load_2d(sa, &tmW, &full[i], kc * 64, t * kTileV);
      }
    }
  }

  // the node rows, their count and the gathered rows come from the previous kernel
  if (early) {
    pdl_wait();
    M = min(*a.n_rows, a.Mcap);
  }
  if (blockIdx.x == 0 && threadIdx.x == 0 && a.reset_count) *a.reset_count = 0;
  pdl_launch_dependents();

  // pipeline positions, carried from one node tile to the next by the
  // thread that owns them (weight loads issued, MMA stage and accumulator,
  // epilogue accumulator, SwiGLU exchanges)
  uint32_t p_next = 0, p_issued = 0, p_last_parity = 0;
  bool p_ok = true, any_active = false;
  int c_stage = 0, c_ab = 0;
  uint32_t c_phase = 0, c_aphase = 0, c_xn = 0;
  for (int ny = slot, it = 0;; ny += a.n_nslots, ++it) {
    const bool active = ny * S::NT < M;  // uniform over the CTA
    // the first tile also completes the weight copies issued before the wait;
    // a CTA without node columns does only that
    if (it > 0 && !active) break;
    any_active |= active;
    const int t_end = active ? t1 : t0;
    for (int c = threadIdx.x; c < S::NT; c += blockDim.x) {
      const int row = ny * S::NT + c;
      ColMeta cm;
      cm.valid = 0;
      cm.bias_off = 0;
      cm.c1 = cm.c2 = 0;
      cm.b = 0;
      cm.lse = 0.f;
      cm.out_row = 0;
      cm.bslot = -1;
      cm.token = 0;
      if (row < M) {
        const Row r = a.rows[row];
        if (r.b >= 0) {
          if (r.b >= batch || r.depth < 0 || r.depth >= a.Bk) {
            set_status(a.status, DT_EDEVICE);
          } else {
            cm.valid = 1;
            cm.b = r.b;
            // block-logit row over the full vocabulary, from this shard's first token
            cm.bias_off = ((int64_t)r.b * a.Bk + r.depth) * a.vfull + a.v_base;
            cm.c1 = (uint32_t)r.path;
            cm.c2 = (uint32_t)(r.path >> 32);
            cm.lse = r.lse;
            cm.out_row = r.aux;
            cm.token = r.token;
            // token -1: no Markov term (zero row); anything else must index A
            if (gather && (r.token < -1 || r.token >= a.vfull)) {
              set_status(a.status, DT_EDEVICE);
              cm.valid = 0;
            }
          }
        }
      }
      meta[c] = cm;
    }
    __syncthreads();
    if (gather && active) {
      // 16-byte pieces of A[token] into the swizzled K-major layout the MMA
      // descriptors expect; columns without a node, token -1 (no Markov term)
      // and K beyond r read as zero
      const int npieces = KC * S::NT * 8;
      for (int idx = threadIdx.x; idx < npieces; idx += blockDim.x) {
        const int ch = idx & 7, c = (idx >> 3) % S::NT, kc = (idx >> 3) / S::NT;
        const int col_k = kc * 64 + ch * 8;
        const bool ok = meta[c].valid && meta[c].token >= 0 && col_k < a.r;
        const uint16_t* src = ok ? a.gatherA + (size_t)meta[c].token * a.r + col_k : a.gatherA;
        uint8_t* dst = bres + ((size_t)kc * S::NT + c) * 128 + ((ch ^ (c & 7)) << 4);
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)),
                     "l"(src), "r"(ok ? 16 : 0)
                     : "memory");
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
      asm volatile("cp.async.wait_all;" ::: "memory");
      // the tensor cores read these bytes through the async proxy
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    __syncthreads();
    // The epilogues read their bias rows from shared memory: global loads
    // issued during the weight stream wait behind it for microseconds.
    if (MODE != EPI_SWIGLU) {
      if (threadIdx.x == 0) {
        int nb = 0;
        bool ok = a.bias_span > 0 && a.bias_rows > 0 && a.L != nullptr && active;
        for (int c = 0; c < S::NT && ok; ++c) {
          if (!meta[c].valid) continue;
          int u = -1;
          for (int i = 0; i < nb; ++i)
            if (brow[i] == meta[c].bias_off) u = i;
          if (u < 0) {
            if (nb == a.bias_rows) {
              ok = false;
              break;
            }
            brow[nb] = meta[c].bias_off;
            u = nb++;
          }
          meta[c].bslot = u;
        }
        *n_bias = ok ? nb : -1;
      }
      __syncthreads();
      const int nb = *n_bias;
      if (warp >= 2 && nb > 0) {
        // every 16-byte piece of [t0 * 128, min(t1 * 128, V)) of each distinct row
        const int esz = a.l_bf16 ? 2 : 4;
        const int x0 = t0 * kTileV;
        const int nx = min(t1 * kTileV, a.V) - x0;
        const int npieces = (nx * esz + 15) / 16;
        for (int u = 0; u < nb; ++u) {
          const uint8_t* src = (const uint8_t*)a.L + (brow[u] + x0) * esz;
          uint8_t* dst = bias_cache + (size_t)u * a.bias_span * esz;
          for (int i = threadIdx.x - 64; i < npieces; i += S::kEpiWarps * 32)
            cp_async16_g2s(dst + (size_t)i * 16, src + (size_t)i * 16);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
      }
    }

    if (warp == 0) {
      // ------------------------------------------------------------ producer
      if (lane == 0 && p_ok) {
        const uint64_t pol_keep = l2_evict_last_policy();
        // p_issued / p_last_parity, per stage: issued at least once, parity of the last issue
        const int pre = it == 0 ? npre : 0;
        for (int i = 0; i < pre; ++i) {
          uint8_t* sa = stage_mem + (size_t)i * sbytes;
          if (gather) {
            mbar_arrive(&full[i]);
          } else {
            mbar_arrive_expect_tx(&full[i], S::kBBytes);
            tma_load_2d(sa + S::kABytes, &tmH, &full[i], (i % KC) * 64, ny * S::NT);
          }
          p_issued |= 1u << i;
        }
        const int n_all = active ? total : pre;
        for (int i = pre; i < n_all; ++i) {
          const uint32_t g = p_next + (uint32_t)i;  // weight loads issued by this CTA before
          const int stage = (int)(g % (uint32_t)stages);
          const uint32_t phase = (g / (uint32_t)stages) & 1u;
          const int t = t0 + i / KC, kc = i % KC;
          if (!mbar_wait(&empty[stage], phase ^ 1, a.status, abort_flag)) {
            p_ok = false;
            break;
          }
          uint8_t* sa = stage_mem + (size_t)stage * sbytes;
          mbar_arrive_expect_tx(&full[stage], sbytes);
          if (MODE == EPI_SWIGLU) {
            tma_load_2d(sa, &tmW, &full[stage], kc * 64, t * 64);
            tma_load_2d(sa + S::kABytes / 2, &tmW2, &full[stage], kc * 64, t * 64);
          } else if (a.l2_keep) {
            tma_load_2d_hint(sa, &tmW, &full[stage], kc * 64, t * kTileV, pol_keep);
          } else {
            tma_load_2d(sa, &tmW, &full[stage], kc * 64, t * kTileV);
          }
          if (!gather) tma_load_2d(sa + S::kABytes, &tmH, &full[stage], kc * 64, ny * S::NT);
          p_issued |= 1u << stage;
          p_last_parity = (p_last_parity & ~(1u << stage)) | (phase << stage);
        }
        p_next += (uint32_t)n_all;
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------- MMA issuer
      if (lane == 0) {
        constexpr uint32_t idesc = idesc_bf16_f32(kTileV, S::NT);
        int& stage = c_stage;
        uint32_t& phase = c_phase;
        int& ab = c_ab;
        uint32_t& aphase = c_aphase;
        bool ok = true;
        for (int t = t0; t < t_end && ok; ++t) {
          if (!mbar_wait(&tempty[ab], aphase ^ 1, a.status, abort_flag)) break;
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + (uint32_t)(ab * S::NT);
          for (int kc = 0; kc < KC; ++kc) {
            if (!mbar_wait(&full[stage], phase, a.status, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = smem_u32(stage_mem + (size_t)stage * sbytes);
            const uint64_t da = smem_desc_k_sw128(sa);
            const uint64_t db = smem_desc_k_sw128(
                gather ? smem_u32(bres + (size_t)kc * S::NT * 128) : sa + S::kABytes);
            const int ks = (kc == KC - 1) ? ks_last : 4;
            for (int s = 0; s < ks; ++s)
              tc_mma_bf16(d_tmem, da + 2 * s, db + 2 * s, idesc, (kc | s) != 0 ? 1u : 0u);
            tc_commit(&empty[stage]);
            if (++stage == stages) {
              stage = 0;
              phase ^= 1;
            }
          }
          if (!ok) break;
          tc_commit(&tfull[ab]);
          if (++ab == S::kAccBufs) {
            ab = 0;
            aphase ^= 1;
          }
        }
        // every MMA issued by this thread has completed once `drain` flips
        // (once per node tile), so the next tile may rewrite the gathered rows
        tc_commit(drain);
        const uint64_t t_start = globaltimer_ns();
        while (!mbar_try_wait(drain, (uint32_t)it & 1u) &&
               globaltimer_ns() - t_start < kWaitLimitNs) {
        }
      }
    } else if (MODE == EPI_ZDUMP || MODE == EPI_QROWS) {
      // ------------------------------------- z / draft-q epilogue (lane = row)
      const int e = warp - 2;
      const int q = warp & 3;  // TMEM lane quadrant accessible to this warp
      const int eg = e >> 2;   // column group served by this warp
      int& ab = c_ab;
      uint32_t& aphase = c_aphase;
      const bool cached = *n_bias > 0;
      if (cached) {
        asm volatile("cp.async.wait_all;" ::: "memory");
        named_bar(1, S::kEpiWarps * 32);
      }
      for (int t = t0; t < t_end; ++t) {
        const int x = t * kTileV + 32 * q + lane;
        if (!mbar_wait(&tfull[ab], aphase, a.status, abort_flag)) break;
        tc_fence_after();
  #pragma unroll 1
        for (int j = 0; j < S::CPT; ++j) {
          const int grp = eg + j * S::EG;
          float acc[32];
          tmem_ld32(tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(ab * S::NT + grp * 32), acc);
          if (j == S::CPT - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[ab]);
          }
          if (x >= a.V) continue;
  #pragma unroll
          for (int i = 0; i < 32; ++i) {
            const ColMeta& cm = meta[grp * 32 + i];
            if (!cm.valid) continue;  // warp-uniform
            float bias = 0.f;
            if (cached) {
              const size_t ci = (size_t)cm.bslot * a.bias_span + (x - t0 * kTileV);
              bias = a.l_bf16 ? bf16_to_f32(((const uint16_t*)bias_cache)[ci])
                              : ((const float*)bias_cache)[ci];
            } else if (a.L) {
              bias = load_bias1(a.L, a.l_bf16, cm.bias_off + x);
            }
            const float z = acc[i] + bias;
            if (MODE == EPI_ZDUMP) {
              if (a.out_bf16)
                ((uint16_t*)a.out)[(size_t)cm.out_row * a.ldo + x] = f32_to_bf16_rne(z);
              else
                a.out[(size_t)cm.out_row * a.ldo + x] = z;
            } else {
              a.out[((size_t)cm.b * a.nmax1 + cm.out_row) * a.ldo + x] =
                  expf(__fdiv_rn(z, a.temp) - cm.lse);
            }
          }
        }
        if (++ab == S::kAccBufs) {
          ab = 0;
          aphase ^= 1;
        }
      }
    } else if (MODE == EPI_SWIGLU) {
      // -------------------------- SwiGLU epilogue: silu(gate) * up, bf16 rows
      // The two up warps of column group eg stage their values in their own
      // transpose buffers (xfull), the two gate warps consume them (xempty);
      // every wait is bounded, so a timed-out warp cannot strand the others.
      const int e = warp - 2;
      const int q = warp & 3;
      const int eg = e >> 2;
      const bool up = q >= 2;  // TMEM lanes 64-127 hold the up projection
      // warp e = 4 eg + ((q - 2) & 3); the up warp of quadrant q + 2 is 4 eg + q
      float* tb_own = tbuf + (size_t)e * 32 * kTLD;
      float* tb_up = tbuf + (size_t)(4 * eg + (q & 1)) * 32 * kTLD;
      int& ab = c_ab;
      uint32_t& aphase = c_aphase;
      uint32_t& xn = c_xn;  // exchanges so far (phase parity)
      bool ok = true;
      for (int t = t0; t < t_end && ok; ++t) {
        const int f = t * 64 + 32 * (q & 1) + lane;  // feature of this lane
        if (!mbar_wait(&tfull[ab], aphase, a.status, abort_flag)) break;
        tc_fence_after();
  #pragma unroll 1
        for (int j = 0; j < S::CPT; ++j, ++xn) {
          const int grp = eg + j * S::EG;
          float acc[32];
          tmem_ld32(tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(ab * S::NT + grp * 32), acc);
          if (j == S::CPT - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[ab]);
          }
          if (up) {
            if (!mbar_wait(&xempty[eg], (xn & 1) ^ 1, a.status, abort_flag)) {
              ok = false;
              break;
            }
  #pragma unroll
            for (int i = 0; i < 32; ++i) tb_own[lane * kTLD + i] = acc[i];
            mbar_arrive(&xfull[eg]);
          } else {
            if (!mbar_wait(&xfull[eg], xn & 1, a.status, abort_flag)) {
              ok = false;
              break;
            }
            if (f < a.V) {
  #pragma unroll
              for (int i = 0; i < 32; ++i) {
                const ColMeta& cm = meta[grp * 32 + i];
                if (!cm.valid) continue;  // warp-uniform
                const float g = acc[i];
                const float u = tb_up[lane * kTLD + i];
                const float act = __fdiv_rn(g, 1.f + expf(-g)) * u;
                ((uint16_t*)a.out)[(size_t)cm.out_row * a.ldo + f] = f32_to_bf16_rne(act);
              }
            }
            mbar_arrive(&xempty[eg]);
          }
        }
        if (++ab == S::kAccBufs) {
          ab = 0;
          aphase ^= 1;
        }
      }
    } else {
      // --------------------------------------------- expansion epilogue (columns)
      // Each 32 x 32 accumulator block (32 vocabulary rows of quadrant q, 32
      // node columns) is transposed through the warp's buffer so that lane c
      // owns column c and holds its 32 consecutive rows.  The arithmetic per
      // block is branch-free (tree max and sum, independent 2^x); the top-k
      // lists are only touched when the block's maximum beats the entry bar.
      const int e = warp - 2;
      const int q = warp & 3;  // TMEM lane quadrant accessible to this warp
      const int eg = e >> 2;   // first column group of this warp
      const float temp = a.temp;
      float* tb = tbuf + (size_t)e * 32 * kTLD;
      ColMeta mc[S::CPT];
  #pragma unroll
      for (int j = 0; j < S::CPT; ++j) mc[j] = meta[(eg + j * S::EG) * 32 + lane];
      float m[S::CPT], ssum[S::CPT], thr[S::CPT], gthr[S::CPT];
      float L1[S::CPT][KMAX];
      int32_t I1[S::CPT][KMAX];
      float L2[S::CPT][KMAX];
      int32_t I2[S::CPT][KMAX];
  #pragma unroll
      for (int j = 0; j < S::CPT; ++j) {
        m[j] = -INFINITY;
        ssum[j] = 0.f;
        thr[j] = -INFINITY;
        gthr[j] = -INFINITY;
  #pragma unroll
        for (int i = 0; i < KMAX; ++i) {
          L1[j][i] = -INFINITY;
          I1[j][i] = 0x7fffffff;
          L2[j][i] = -INFINITY;
          I2[j][i] = 0x7fffffff;
        }
      }
      // bias rows: from the shared-memory cache when it holds them all, else
      // (one column group per thread only) global loads one tile ahead
      const int nbc = *n_bias;
      const bool cached = nbc > 0;
      if (cached) {
        asm volatile("cp.async.wait_all;" ::: "memory");
        named_bar(1, S::kEpiWarps * 32);
      }
      const bool ldg_bias = S::CPT == 1 && a.L != nullptr && !cached;
      const bool vec = (a.l_bf16 ? (a.vfull % 8 == 0) : (a.vfull % 4 == 0)) &&
                       ((uintptr_t)a.L % 16 == 0);
      uint4 raw[8];
      bool raw_ok = false;
      if (ldg_bias) {
        const int xq = t0 * kTileV + 32 * q;
        raw_ok = mc[0].valid && vec && xq + 32 <= a.V && t0 < t_end;
        if (raw_ok) load_bias_raw(a.L, a.l_bf16, mc[0].bias_off + xq, raw);
      }
      int& ab = c_ab;
      uint32_t& aphase = c_aphase;
      for (int t = t0; t < t_end; ++t) {
        if (!mbar_wait(&tfull[ab], aphase, a.status, abort_flag)) break;
        tc_fence_after();
        const int xq = t * kTileV + 32 * q;  // first vocabulary row of this quadrant
        const int nv = min(32, a.V - xq);
  #pragma unroll
        for (int j = 0; j < S::CPT; ++j) {
          const int grp = eg + j * S::EG;
          float acc[32];
          tmem_ld32(tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(ab * S::NT + grp * 32), acc);
          if (j == S::CPT - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[ab]);
          }
          float bias[32];
          bool had_raw = false;
          if (ldg_bias) {
            if (raw_ok) decode_bias(raw, a.l_bf16, bias);
            had_raw = raw_ok;
            const int xn = xq + kTileV;
            raw_ok = mc[0].valid && vec && t + 1 < t_end && xn + 32 <= a.V;
            if (raw_ok) load_bias_raw(a.L, a.l_bf16, mc[0].bias_off + xn, raw);
          }
          // transpose 32 rows x 32 columns: lane takes column grp*32+lane
  #pragma unroll
          for (int i = 0; i < 32; ++i) tb[lane * kTLD + i] = acc[i];
          __syncwarp();
  #pragma unroll
          for (int i = 0; i < 32; ++i) acc[i] = tb[i * kTLD + lane];
          __syncwarp();
          if (!mc[j].valid || nv <= 0) continue;
          if (cached) {
            // 32 consecutive values of this column's bias row (16-byte reads)
            const int xo = xq - t0 * kTileV;
            if (nv == 32) {
              uint4 cr[8];
              const uint4* src = (const uint4*)(bias_cache + ((size_t)mc[j].bslot * a.bias_span + xo) *
                                                                 (a.l_bf16 ? 2 : 4));
  #pragma unroll
              for (int c = 0; c < 8; ++c)
                if (c < 4 || !a.l_bf16) cr[c] = src[c];
              decode_bias(cr, a.l_bf16, bias);
            } else {
  #pragma unroll
              for (int i = 0; i < 32; ++i)
                bias[i] = i < nv ? (a.l_bf16 ? bf16_to_f32(((const uint16_t*)bias_cache)[
                                                   (size_t)mc[j].bslot * a.bias_span + xo + i])
                                             : ((const float*)bias_cache)[
                                                   (size_t)mc[j].bslot * a.bias_span + xo + i])
                                 : 0.f;
            }
          } else if (ldg_bias) {
            if (!had_raw) {
  #pragma unroll
              for (int i = 0; i < 32; ++i)
                bias[i] = i < nv ? load_bias1(a.L, a.l_bf16, mc[j].bias_off + xq + i) : 0.f;
            }
          } else {
  #pragma unroll
            for (int i = 0; i < 32; ++i) bias[i] = 0.f;
          }
          float s[32];
  #pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float z = acc[i] + bias[i];
            s[i] = i < nv ? (STOCH ? __fdiv_rn(z, temp) : z) : -INFINITY;
          }
          // log-sum-exp of the block: tree max, independent 2^x, tree sum
          float mx[16];
  #pragma unroll
          for (int i = 0; i < 16; ++i) mx[i] = fmaxf(s[i], s[i + 16]);
  #pragma unroll
          for (int w = 8; w; w >>= 1)
  #pragma unroll
            for (int i = 0; i < w; ++i) mx[i] = fmaxf(mx[i], mx[i + w]);
          const float mt = mx[0];
          float ex[32];
  #pragma unroll
          for (int i = 0; i < 32; ++i) ex[i] = ex2_approx((s[i] - mt) * kLog2e);
  #pragma unroll
          for (int w = 16; w; w >>= 1)
  #pragma unroll
            for (int i = 0; i < w; ++i) ex[i] += ex[i + w];
          const float st = ex[0];
          if (mt > m[j]) {
            ssum[j] = ssum[j] * ex2_approx((m[j] - mt) * kLog2e) + st;
            m[j] = mt;
          } else {
            ssum[j] += st * ex2_approx((mt - m[j]) * kLog2e);
          }
          // top-k of s (values arrive in increasing token order)
          if (mt > thr[j]) {
  #pragma unroll
            for (int i = 0; i < 32; ++i) {
              if (s[i] > thr[j]) {
                topk_insert<KMAX>(L1[j], I1[j], s[i], a.v_base + xq + i);
                thr[j] = kth<KMAX>(L1[j], k);
              }
            }
          }
          if constexpr (STOCH) {
            // Gumbel keys; four consecutive tokens share one Philox counter.
            // The block's eight draws are independent and issued together;
            // the exact key is computed only where it may beat the bar.
            if (mt + kGumbelMax > gthr[j]) {
              uint32_t wds[32];
  #pragma unroll
              for (int gi = 0; gi < 8; ++gi) {
                const uint32_t x4 = (uint32_t)(a.v_base + xq + 4 * gi);
                const U4 o = philox10(
                    U4{(x4 >> 2) | ((uint32_t)mc[j].b << 18), mc[j].c1, mc[j].c2, a.offset},
                    (uint32_t)a.seed, (uint32_t)(a.seed >> 32));
                wds[4 * gi] = o.x;
                wds[4 * gi + 1] = o.y;
                wds[4 * gi + 2] = o.z;
                wds[4 * gi + 3] = o.w;
              }
  #pragma unroll
              for (int i = 0; i < 32; ++i) {
                if (i < nv && gumbel_may_beat(s[i], gthr[j], wds[i])) {
                  const float gk = s[i] + (-logf(-logf(u23(wds[i]))));
                  if (gk > gthr[j]) {
                    topk_insert<KMAX>(L2[j], I2[j], gk, a.v_base + xq + i);
                    gthr[j] = kth<KMAX>(L2[j], k);
                  }
                }
              }
            }
          }
        }
        if (++ab == S::kAccBufs) {
          ab = 0;
          aphase ^= 1;
        }
      }
      // publish this quadrant's partials of the owned columns (the transpose
      // buffers are free once every epilogue warp has left the tile loop)
      named_bar(1, S::kEpiWarps * 32);
      float* ql1v = tbuf;  // [4][NT][KMAX] per-quadrant top-k of s
      int32_t* ql1i = (int32_t*)(ql1v + 4 * S::NT * KMAX);
      float* ql2v = (float*)(ql1i + 4 * S::NT * KMAX);  // Gumbel lists (T > 0)
      int32_t* ql2i = (int32_t*)(ql2v + (STOCH ? 4 * S::NT * KMAX : 0));
      float2* qst = (float2*)(ql2i + (STOCH ? 4 * S::NT * KMAX : 0));  // [4][NT]
  #pragma unroll
      for (int j = 0; j < S::CPT; ++j) {
        const int col = (eg + j * S::EG) * 32 + lane;
        qst[q * S::NT + col] = make_float2(m[j], ssum[j]);
  #pragma unroll
        for (int i = 0; i < KMAX; ++i) {
          ql1v[(q * S::NT + col) * KMAX + i] = L1[j][i];
          ql1i[(q * S::NT + col) * KMAX + i] = I1[j][i];
          if (STOCH) {
            ql2v[(q * S::NT + col) * KMAX + i] = L2[j][i];
            ql2i[(q * S::NT + col) * KMAX + i] = I2[j][i];
          }
        }
      }
      named_bar(1, S::kEpiWarps * 32);
      // one thread per column merges the four quadrants into the CTA's partial
      const int et = threadIdx.x - 64;
      for (int c = et; c < S::NT; c += S::kEpiWarps * 32) {
        if (!meta[c].valid) continue;
        const int row = ny * S::NT + c;
        float mx = -INFINITY;
        for (int qq = 0; qq < 4; ++qq) mx = fmaxf(mx, qst[qq * S::NT + c].x);
        float sv = 0.f;
        if (mx != -INFINITY)
          for (int qq = 0; qq < 4; ++qq) {
            const float2 rv = qst[qq * S::NT + c];
            if (rv.x != -INFINITY) sv += rv.y * exp2f((rv.x - mx) * kLog2e);
          }
        const size_t pidx = (size_t)row * a.ncta_v + cx;
        a.pstats[pidx] = make_float2(mx, sv);
        for (int lst = 0; lst < (STOCH ? 2 : 1); ++lst) {
          const float* LV = lst ? ql2v : ql1v;
          const int32_t* LI = lst ? ql2i : ql1i;
          // list entry i of this CTA at [row][i][cta]: a merging warp reads one
          // entry of 32 consecutive CTAs per load
          float* OV = (lst ? a.pgv : a.plv) + (size_t)row * k * a.ncta_v + cx;
          int32_t* OI = (lst ? a.pgi : a.pli) + (size_t)row * k * a.ncta_v + cx;
          int h0 = 0, h1 = 0, h2 = 0, h3 = 0;  // heads of the four quadrant lists
          for (int i = 0; i < k; ++i) {
            int bw = -1;
            float bv = -INFINITY;
            int32_t bi = 0x7fffffff;
  #pragma unroll
            for (int w = 0; w < 4; ++w) {
              const int hw = w == 0 ? h0 : w == 1 ? h1 : w == 2 ? h2 : h3;
              if (hw >= k) continue;
              const float v = LV[(w * S::NT + c) * KMAX + hw];
              const int32_t id = LI[(w * S::NT + c) * KMAX + hw];
              if (bw < 0 || ranks_first(v, id, bv, bi)) {
                bw = w;
                bv = v;
                bi = id;
              }
            }
            h0 += bw == 0;
            h1 += bw == 1;
            h2 += bw == 2;
            h3 += bw == 3;
            OV[(size_t)i * a.ncta_v] = bv;
            OI[(size_t)i * a.ncta_v] = bi;
          }
        }
      }
    }
    // the node tile is done: its rows, bias rows and transpose buffers may be
    // reused; after a timed-out wait every role stops
    __syncthreads();
    if (*abort_flag) break;
  }  // node tiles
  if (warp == 0 && lane == 0 && (!p_ok || !any_active || *abort_flag)) {
    // let the copies in flight land (bounded) before the CTA exits
    const uint64_t t_start = globaltimer_ns();
    for (int st = 0; st < stages; ++st) {
      if (!((p_issued >> st) & 1)) continue;
      while (!mbar_try_wait(&full[st], (p_last_parity >> st) & 1) &&
             globaltimer_ns() - t_start < 50000000ull) {
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, S::kTmemCols);
  }
}

// ---------------------------------------------------------------- host side --
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) !=
            cudaSuccess ||
        qres != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = (EncodeTiledFn)ptr;
  }
  return fn;
}

// 2-D bf16 tensor [rows][K] (K contiguous), boxes of 64 x box_rows, 128B swizzle.
bool make_tmap_bf16_kmajor(CUtensorMap* map, const void* base, uint64_t K, uint64_t rows,
                           uint32_t box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {K, rows};
  cuuint64_t strides[1] = {K * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NG, int MODE, bool STOCH, int KMAX>
static cudaError_t launch_cfg(const CUtensorMap& tmW, const CUtensorMap& tmW2,
                              const CUtensorMap& tmH, GemmArgs a, int batch, cudaStream_t s) {
  using SH = GemmShape<NG>;
  auto kern = markov_gemm_kernel<NG, MODE, STOCH, KMAX>;
  // bias cache: the longest vocabulary range of a CTA, padded to 16 bytes;
  // only when 16-byte copies of the rows are aligned
  size_t bias_bytes = 0;
  a.bias_span = 0;
  a.bias_rows = 0;
  if (MODE != EPI_SWIGLU && a.L) {
    const int esz = a.l_bf16 ? 2 : 4;
    const bool aligned = ((uintptr_t)a.L % 16 == 0) && ((size_t)a.vfull * esz) % 16 == 0;
    const int span = ((a.n_vtiles + a.ncta_v - 1) / a.ncta_v) * 128;
    // distinct rows a node tile can need: one per (request, depth), at most NT
    const int rows = std::min(std::min(SH::NT, kBiasRowsMax), batch * a.Bk);
    const size_t bytes = (size_t)rows * span * esz;
    if (aligned && bytes <= 80 * 1024) {
      a.bias_span = span;
      a.bias_rows = rows;
      bias_bytes = bytes;
    }
  }
  // gathered B rows: KC x NT x 128 B, only while that stays small
  const size_t gather_bytes = ((a.r + 63) / 64) * (size_t)SH::NT * 128;
  if (a.gatherA && (MODE == EPI_SWIGLU || gather_bytes > 32 * 1024)) return cudaErrorInvalidValue;
  const size_t gb = a.gatherA ? gather_bytes : 0;
  // the deepest pipeline that fits in 200 KB of shared memory, which leaves room
  // on each SM for a small kernel of the wave loop running alongside
  int stages = 12;
  while (stages > 2 && gemm_smem_bytes<NG>(stages, MODE, KMAX, STOCH, bias_bytes, gb) > 200 * 1024)
    --stages;
  a.stages = stages;
  const size_t smem = gemm_smem_bytes<NG>(stages, MODE, KMAX, STOCH, bias_bytes, gb);
  cudaError_t e = ensure_smem(kern, smem);
  if (e != cudaSuccess) return e;
  const dim3 grid(a.ncta_v * a.n_nslots);
  e = launch_pdl(kern, grid, dim3(SH::kThreads), smem, s, tmW, tmW2, tmH, a, batch);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Node columns per tile the launcher uses for a given column capacity.
int gemm_node_tile(int max_cols) { return max_cols <= 32 ? 32 : max_cols <= 64 ? 64 : 256; }

// Largest top-k list a launch keeps per column for k children per node.
int gemm_kmax(int k) { return k <= 4 ? 4 : 16; }

// Launches one GEMM.  tmW: weight rows (box 128 rows; SwiGLU: the gate rows,
// box 64, with tmW2 the up rows); tmH: node rows (box nt rows), unused when
// a.gatherA is set (the rows A[token] are then gathered by the kernel).
// Whether a launch can gather its rows.
bool gemm_can_gather(int r, int nt) { return ((r + 63) / 64) * (size_t)nt * 128 <= 32 * 1024; }

cudaError_t launch_markov_gemm(int mode, bool stoch, const CUtensorMap& tmW,
                               const CUtensorMap& tmW2, const CUtensorMap& tmH, GemmArgs a,
                               int batch, int nt, cudaStream_t s) {
  const int ng = nt / 32;
  a.n_ntiles = (a.Mcap + nt - 1) / nt;
  if (a.vfull == 0) a.vfull = a.V;
  // a vocabulary shard starts on a tile and only expands nodes
  if (a.v_base != 0 && (mode != EPI_EXPAND || a.v_base % kTileV)) return cudaErrorInvalidValue;
  // node-tile slots per weight range: every tile gets its own CTA unless the
  // caller asks for fewer (then each CTA loops over tiles)
  a.n_nslots = (a.n_nslots > 0 && a.n_nslots < a.n_ntiles) ? a.n_nslots : a.n_ntiles;
  if (a.ldo == 0) a.ldo = a.V;
  if (ng == 8 && mode == EPI_EXPAND && a.L) return cudaErrorInvalidValue;  // no bias path
  const int kmax = gemm_kmax(a.k);
#define DT_GEMM_CASE(NG, MODE, ST, KM)                                                  \
  if (ng == NG && mode == MODE && stoch == ST && (MODE != EPI_EXPAND || kmax == KM)) \
    return launch_cfg<NG, MODE, ST, KM>(tmW, tmW2, tmH, a, batch, s);
  DT_GEMM_CASE(1, EPI_EXPAND, false, 4)
  DT_GEMM_CASE(1, EPI_EXPAND, false, 16)
  DT_GEMM_CASE(2, EPI_EXPAND, false, 4)
  DT_GEMM_CASE(2, EPI_EXPAND, false, 16)
  DT_GEMM_CASE(8, EPI_EXPAND, false, 4)
  DT_GEMM_CASE(8, EPI_EXPAND, false, 16)
  DT_GEMM_CASE(1, EPI_EXPAND, true, 4)
  DT_GEMM_CASE(1, EPI_EXPAND, true, 16)
  DT_GEMM_CASE(2, EPI_EXPAND, true, 4)
  DT_GEMM_CASE(2, EPI_EXPAND, true, 16)
  DT_GEMM_CASE(1, EPI_ZDUMP, false, 4)
  DT_GEMM_CASE(2, EPI_ZDUMP, false, 4)
  DT_GEMM_CASE(8, EPI_ZDUMP, false, 4)
  DT_GEMM_CASE(1, EPI_QROWS, true, 4)
  DT_GEMM_CASE(2, EPI_QROWS, true, 4)
  DT_GEMM_CASE(1, EPI_SWIGLU, false, 4)
  DT_GEMM_CASE(2, EPI_SWIGLU, false, 4)
  DT_GEMM_CASE(8, EPI_SWIGLU, false, 4)
#undef DT_GEMM_CASE
  return cudaErrorInvalidValue;
}

}  // namespace dt
