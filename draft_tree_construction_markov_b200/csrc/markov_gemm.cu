// Parent-conditioned logits on the 5th-generation tensor cores.
//
// For every GEMM column n (a tree node u with depth d and token t) and every
// vocabulary row x:
//   z[x][n] = L[b][d][x] + sum_rho Bm[x][rho] * A[t][rho]
// (PCTree summary, DSpark paragraph: the Markov head biases the shared block
// logits by the previous token; here the previous token is the node's own
// token, i.e. the children are parent-conditioned.)
//
// Swap-AB tcgen05 GEMM: the vocabulary is the MMA M axis (128 rows per tile,
// the Markov factor Bm streamed by TMA), nodes are the N axis (the gathered
// rows A[t], also by TMA), K = r.  The fp32 accumulator lives in TMEM (double
// buffered); epilogue warps read it back with tcgen05.ld, one 32-lane quadrant
// each (lane = vocabulary row), add the block-logit bias and store one fp32
// row per node: s = z / T for the top-k pass (EXPAND), z itself (ZDUMP) or
// q = exp(s - lse) (QROWS).  Columns without a node are skipped.  Each CTA
// owns a contiguous range of vocabulary tiles.
#include "build.cuh"

namespace dt {

constexpr int kTileV = 128;

// NG groups of 32 node columns per tile; every epilogue warp reads CW columns
// of one 32-lane TMEM quadrant, so each quadrant is served by NT / CW warps.
template <int NG, int CW>
struct GemmShape {
  static constexpr int NT = 32 * NG;  // MMA N: node columns per tile
  static constexpr int EPQ = NT / CW;  // epilogue warps per quadrant
  static constexpr int kEpiWarps = 4 * EPQ;
  static constexpr int kThreads = 32 * (2 + kEpiWarps);
  static constexpr int kABytes = kTileV * 128;  // 128 vocab rows x 64 bf16
  static constexpr int kBBytes = NT * 128;      // NT node rows x 64 bf16
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr uint32_t kTmemCols = (2 * NT <= 64) ? 64 : (2 * NT <= 128) ? 128 : 256;
  static_assert(NT % 16 == 0 && NT <= 256, "MMA N must be a multiple of 16, at most 256");
};

struct ColMeta {
  int64_t bias_off;  // element offset of the node's block-logit row
  uint32_t c1, c2;   // Philox counter words 1-2 (path id)
  int32_t b;
  int32_t valid;
  float lse;
  int32_t out_row;
};

template <int NG, int CW>
static size_t gemm_smem_bytes(int stages) {
  using S = GemmShape<NG, CW>;
  size_t off = 1024;  // alignment slack
  off += (size_t)stages * S::kStageBytes;
  off += (size_t)(2 * stages + 5) * 8;  // barriers
  off += 16;                             // tmem slot + abort flag
  off = (off + 15) & ~(size_t)15;
  off += (size_t)S::NT * sizeof(ColMeta);
  return off;
}

template <int NG, int CW, int MODE, bool STOCH>
__global__ void __launch_bounds__(GemmShape<NG, CW>::kThreads, 1)
    markov_gemm_kernel(const __grid_constant__ CUtensorMap tmW,
                       const __grid_constant__ CUtensorMap tmH, GemmArgs a, int batch) {
  using S = GemmShape<NG, CW>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cx = blockIdx.x, ny = blockIdx.y;
  // the node rows, their count and the gathered Markov rows come from the
  // previous kernel
  pdl_wait();
  const int M = min(*a.n_rows, a.Mcap);
  if (cx == 0 && ny == 0 && threadIdx.x == 0 && a.reset_count) *a.reset_count = 0;
  pdl_launch_dependents();
  if (ny * S::NT >= M) return;  // uniform over the CTA

  const int base = a.n_vtiles / a.ncta_v, extra = a.n_vtiles % a.ncta_v;
  const int t0 = cx * base + min(cx, extra);
  const int t1 = t0 + base + (cx < extra ? 1 : 0);
  const int KC = (a.r + 63) >> 6;
  const int ks_last = (((a.r - 1) & 63) >> 4) + 1;
  const int stages = a.stages;

  // ---- carve shared memory
  uint8_t* p = smem;
  uint8_t* stage_mem = p;
  p += (size_t)stages * S::kStageBytes;
  uint64_t* full = (uint64_t*)p;
  uint64_t* empty = full + stages;
  uint64_t* tfull = empty + stages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  p = (uint8_t*)(drain + 1);
  uint32_t* tmem_slot = (uint32_t*)p;
  volatile int* abort_flag = (volatile int*)(p + 4);
  p += 16;
  p = (uint8_t*)(((uintptr_t)p + 15) & ~(uintptr_t)15);
  ColMeta* meta = (ColMeta*)p;
  p += S::NT * sizeof(ColMeta);
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], S::kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmH);
  }
  for (int c = threadIdx.x; c < S::NT; c += blockDim.x) {
    const int row = ny * S::NT + c;
    ColMeta cm;
    cm.valid = 0;
    cm.bias_off = 0;
    cm.c1 = cm.c2 = 0;
    cm.b = 0;
    cm.lse = 0.f;
    cm.out_row = 0;
    if (row < M) {
      const Row r = a.rows[row];
      if (r.b >= 0) {
        if (r.b >= batch || r.depth < 0 || r.depth >= a.Bk) {
          set_status(a.status, DT_EDEVICE);
        } else {
          cm.valid = 1;
          cm.b = r.b;
          cm.bias_off = ((int64_t)r.b * a.Bk + r.depth) * a.V;
          cm.c1 = (uint32_t)r.path;
          cm.c2 = (uint32_t)(r.path >> 32);
          cm.lse = r.lse;
          cm.out_row = r.aux;
        }
      }
    }
    meta[c] = cm;
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, S::kTmemCols);
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      uint32_t issued = 0, last_parity = 0;  // per stage: issued at least once, parity of last issue
      for (int t = t0; t < t1 && ok; ++t) {
        for (int kc = 0; kc < KC; ++kc) {
          if (!mbar_wait(&empty[stage], phase ^ 1, a.status, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* sa = stage_mem + (size_t)stage * S::kStageBytes;
          mbar_arrive_expect_tx(&full[stage], S::kStageBytes);
          tma_load_2d(sa, &tmW, &full[stage], kc * 64, t * kTileV);
          tma_load_2d(sa + S::kABytes, &tmH, &full[stage], kc * 64, ny * S::NT);
          issued |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == stages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        // let the copies already in flight land (bounded) before the CTA exits
        const uint64_t t_start = globaltimer_ns();
        for (int st = 0; st < stages; ++st) {
          if (!((issued >> st) & 1)) continue;
          while (!mbar_try_wait(&full[st], (last_parity >> st) & 1) &&
                 globaltimer_ns() - t_start < 50000000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kTileV, S::NT);
      int stage = 0;
      uint32_t phase = 0;
      int ab = 0;
      uint32_t aphase = 0;
      bool ok = true;
      for (int t = t0; t < t1 && ok; ++t) {
        if (!mbar_wait(&tempty[ab], aphase ^ 1, a.status, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(ab * S::NT);
        for (int kc = 0; kc < KC; ++kc) {
          if (!mbar_wait(&full[stage], phase, a.status, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(stage_mem + (size_t)stage * S::kStageBytes);
          const uint64_t da = smem_desc_k_sw128(sa);
          const uint64_t db = smem_desc_k_sw128(sa + S::kABytes);
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
        ab ^= 1;
        if (ab == 0) aphase ^= 1;
      }
      // every MMA issued by this thread has completed once `drain` flips
      tc_commit(drain);
      const uint64_t t_start = globaltimer_ns();
      while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t_start < kWaitLimitNs) {
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Warp e reads TMEM quadrant q (vocabulary rows 32q..32q+31 of each tile;
    // lane = row) for the CW node columns of group cg; stores coalesce.
    const int e = warp - 2;
    const int q = warp & 3;
    const int cg = e >> 2;
    const float temp = a.temp;
    int ab = 0;
    uint32_t aphase = 0;
    for (int t = t0; t < t1; ++t) {
      const int x0 = t * kTileV + 32 * q;
      const int x = x0 + lane;
      const bool xin = x < a.V;
      // block-logit bias of every node column of this tile, loaded before
      // waiting for the accumulator so the latency overlaps the MMA
      float bias[CW];
#pragma unroll
      for (int j = 0; j < CW; ++j) {
        const ColMeta& cm = meta[cg * CW + j];
        bias[j] = 0.f;
        if (cm.valid && xin)
          bias[j] = a.l_bf16 ? bf16_to_f32(__ldg((const uint16_t*)a.L + cm.bias_off + x))
                             : __ldg((const float*)a.L + cm.bias_off + x);
      }
      if (!mbar_wait(&tfull[ab], aphase, a.status, abort_flag)) break;
      tc_fence_after();
      float acc[CW];
      const uint32_t taddr =
          tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(ab * S::NT + cg * CW);
#pragma unroll
      for (int c = 0; c < CW / 16; ++c) {
        float v[16];
        tmem_ld16(taddr + 16 * c, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[16 * c + i] = v[i];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[ab]);
      ab ^= 1;
      if (ab == 0) aphase ^= 1;
      if (!xin) continue;
#pragma unroll
      for (int j = 0; j < CW; ++j) {
        const int c = cg * CW + j;
        const ColMeta& cm = meta[c];
        if (!cm.valid) continue;  // warp-uniform
        const float z = acc[j] + bias[j];
        if (MODE == EPI_ZDUMP) {
          a.out[(size_t)cm.out_row * a.V + x] = z;
        } else {
          const float s = STOCH ? __fdiv_rn(z, temp) : z;
          if (MODE == EPI_QROWS)
            a.out[((size_t)cm.b * a.nmax1 + cm.out_row) * a.V + x] = expf(s - cm.lse);
          else  // EPI_EXPAND: the scaled logits, one fp32 row per GEMM column
            a.out[(size_t)(ny * S::NT + c) * a.V + x] = s;
        }
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

template <int NG, int CW, int MODE, bool STOCH>
static cudaError_t launch_cfg(const CUtensorMap& tmW, const CUtensorMap& tmH, GemmArgs a,
                              int batch, int n_node_tiles, cudaStream_t s) {
  using SH = GemmShape<NG, CW>;
  auto kern = markov_gemm_kernel<NG, CW, MODE, STOCH>;
  // the deepest pipeline that fits in 220 KB of shared memory
  int stages = 8;
  while (stages > 2 && gemm_smem_bytes<NG, CW>(stages) > 220 * 1024) --stages;
  a.stages = stages;
  const size_t smem = gemm_smem_bytes<NG, CW>(stages);
  cudaError_t e = ensure_smem(kern, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.ncta_v, n_node_tiles);
  e = launch_pdl(kern, grid, dim3(SH::kThreads), smem, s, tmW, tmH, a, batch);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Node columns per tile the launcher uses for a given column capacity.
int gemm_node_tile(int max_cols) { return max_cols <= 32 ? 32 : 64; }

cudaError_t launch_markov_gemm(int mode, bool stoch, const CUtensorMap& tmW,
                               const CUtensorMap& tmH, const GemmArgs& a, int batch, int nt,
                               cudaStream_t s) {
  const int ntiles = (a.Mcap + nt - 1) / nt;
  const int ng = nt / 32;
#define DT_GEMM_CASE(NG, MODE, ST) \
  if (ng == NG && mode == MODE && stoch == ST) \
    return launch_cfg<NG, 16, MODE, ST>(tmW, tmH, a, batch, ntiles, s);
  DT_GEMM_CASE(1, EPI_EXPAND, false)
  DT_GEMM_CASE(2, EPI_EXPAND, false)
  DT_GEMM_CASE(1, EPI_EXPAND, true)
  DT_GEMM_CASE(2, EPI_EXPAND, true)
  DT_GEMM_CASE(1, EPI_ZDUMP, false)
  DT_GEMM_CASE(2, EPI_ZDUMP, false)
  DT_GEMM_CASE(1, EPI_QROWS, true)
  DT_GEMM_CASE(2, EPI_QROWS, true)
#undef DT_GEMM_CASE
  return cudaErrorInvalidValue;
}

}  // namespace dt
