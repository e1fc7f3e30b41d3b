// Parent-conditioned node distributions on the 5th-generation tensor cores.
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
// buffered).  Four epilogue warps per 32 node columns read it back with
// tcgen05.ld (each warp its 32-lane quadrant = 32 vocabulary rows) and
// transpose each 32 x 32 block through shared memory, so that every thread
// owns ONE node column and scans 32 consecutive vocabulary entries of it per
// tile.  Per column it fuses the block-logit bias, the temperature, a batched
// max / sum-exp (log-sum-exp), a private top-k of s (ties to the lower token
// id) and, at T > 0, the Gumbel-top-k of s + G; one Philox call serves four
// consecutive tokens.  Each CTA owns a contiguous range of vocabulary tiles
// and writes one partial result per node; the frontier kernel merges them.
#include "build.cuh"

namespace dt {

constexpr int kTileV = 128;
constexpr float kLog2e = 1.4426950408889634f;
// U <= 1 - 2^-24 gives G = -log(-log U) <= 16.64; tokens with s + 16.75 below
// the current k-th Gumbel key cannot enter the sample and skip the Philox draw.
constexpr float kGumbelMax = 16.75f;
constexpr int kTLD = 33;  // transpose buffer row stride (floats)

template <int NG>
struct GemmShape {
  static constexpr int NT = 32 * NG;  // MMA N: node columns per tile
  static constexpr int kEpiWarps = 4 * NG;
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

template <int NG>
static size_t gemm_smem_bytes(int stages, int kmax, bool stoch) {
  using S = GemmShape<NG>;
  size_t off = 1024;  // alignment slack
  off += (size_t)stages * S::kStageBytes;
  off += (size_t)(2 * stages + 5) * 8;  // barriers
  off += 16;                             // tmem slot + abort flag
  off = (off + 15) & ~(size_t)15;
  off += (size_t)S::NT * sizeof(ColMeta);
  off += (size_t)S::kEpiWarps * 32 * kTLD * 4;             // transpose buffers
  off += (size_t)4 * S::NT * kmax * 8 * (stoch ? 2 : 1);   // per-quadrant lists
  off += (size_t)4 * S::NT * sizeof(float2);               // per-quadrant stats
  return off;
}

// Insert (v, id) into a register list sorted by value (descending); equal
// values keep their earlier (lower-id) entries first.  Entries past k are
// scratch.  Caller guarantees v > list[k-1].
template <int KMAX>
__device__ __forceinline__ void topk_insert(float (&L)[KMAX], int32_t (&I)[KMAX], float v,
                                            int32_t id) {
  float nl[KMAX];
  int32_t ni[KMAX];
#pragma unroll
  for (int i = 0; i < KMAX; ++i) {
    const bool ge = L[i] >= v;
    const bool gep = (i == 0) ? false : (L[i - 1] >= v);
    nl[i] = ge ? L[i] : ((i == 0 || gep) ? v : L[i - 1]);
    ni[i] = ge ? I[i] : ((i == 0 || gep) ? id : I[i - 1]);
  }
#pragma unroll
  for (int i = 0; i < KMAX; ++i) {
    L[i] = nl[i];
    I[i] = ni[i];
  }
}

template <int KMAX>
__device__ __forceinline__ float kth(const float (&L)[KMAX], int k) {
  float t = L[0];
#pragma unroll
  for (int i = 1; i < KMAX; ++i)
    if (i == k - 1) t = L[i];
  return t;
}

// (v1, i1) ranks before (v2, i2): larger value first, then lower id.
__device__ __forceinline__ bool ranks_before(float v1, int32_t i1, float v2, int32_t i2) {
  return v1 > v2 || (v1 == v2 && i1 < i2);
}

__device__ __forceinline__ void named_bar(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// 32 consecutive block-logit values of one row (vectorised when aligned).
__device__ __forceinline__ void load_bias32(const void* L, int bf16, int64_t off, int n,
                                            bool vec, float (&bias)[32]) {
  if (vec && n == 32) {
    if (bf16) {
      const uint4* p = (const uint4*)((const uint16_t*)L + off);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 u = p[c];
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          bias[8 * c + 2 * h] = __uint_as_float(w[h] << 16);
          bias[8 * c + 2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
        }
      }
    } else {
      const float4* p = (const float4*)((const float*)L + off);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float4 u = p[c];
        bias[4 * c] = u.x;
        bias[4 * c + 1] = u.y;
        bias[4 * c + 2] = u.z;
        bias[4 * c + 3] = u.w;
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      bias[i] = i < n ? (bf16 ? bf16_to_f32(((const uint16_t*)L)[off + i]) : ((const float*)L)[off + i])
                      : 0.f;
  }
}

template <int NG, int MODE, bool STOCH, int KMAX>
__global__ void __launch_bounds__(GemmShape<NG>::kThreads, 1)
    markov_gemm_kernel(const __grid_constant__ CUtensorMap tmW,
                       const __grid_constant__ CUtensorMap tmH, GemmArgs a, int batch) {
  using S = GemmShape<NG>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cx = blockIdx.x, ny = blockIdx.y;
  const int M = min(*a.n_rows, a.Mcap);
  if (cx == 0 && ny == 0 && threadIdx.x == 0 && a.reset_count) *a.reset_count = 0;
  if (ny * S::NT >= M) return;  // uniform over the CTA

  const int base = a.n_vtiles / a.ncta_v, extra = a.n_vtiles % a.ncta_v;
  const int t0 = cx * base + min(cx, extra);
  const int t1 = t0 + base + (cx < extra ? 1 : 0);
  const int KC = (a.r + 63) >> 6;
  const int ks_last = (((a.r - 1) & 63) >> 4) + 1;
  const int stages = a.stages;
  const int k = a.k;

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
  float* tbuf = (float*)p;  // [kEpiWarps][32][kTLD]
  p += (size_t)S::kEpiWarps * 32 * kTLD * 4;
  float* ql1v = (float*)p;  // [4][NT][KMAX] per-quadrant top-k of s
  p += (size_t)4 * S::NT * KMAX * 4;
  int32_t* ql1i = (int32_t*)p;
  p += (size_t)4 * S::NT * KMAX * 4;
  float* ql2v = ql1v;  // [4][NT][KMAX] per-quadrant Gumbel top-k
  int32_t* ql2i = ql1i;
  if (STOCH) {
    ql2v = (float*)p;
    p += (size_t)4 * S::NT * KMAX * 4;
    ql2i = (int32_t*)p;
    p += (size_t)4 * S::NT * KMAX * 4;
  }
  float2* qst = (float2*)p;  // [4][NT]

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
    const int e = warp - 2;
    const int q = warp & 3;         // TMEM lane quadrant accessible to this warp
    const int g = e >> 2;           // column group
    const int col = g * 32 + lane;  // EXPAND: the node column this thread owns
    const ColMeta mc = meta[col];
    const float temp = a.temp;
    const bool vec = a.l_bf16 ? (a.V % 8 == 0) : (a.V % 4 == 0);
    float* tb = tbuf + (size_t)e * 32 * kTLD;
    float m = -INFINITY, ssum = 0.f;
    float L1[KMAX];
    int32_t I1[KMAX];
    float L2[KMAX];
    int32_t I2[KMAX];
#pragma unroll
    for (int i = 0; i < KMAX; ++i) {
      L1[i] = -INFINITY;
      I1[i] = 0x7fffffff;
    }
#pragma unroll
    for (int i = 0; i < KMAX; ++i) {
      L2[i] = -INFINITY;
      I2[i] = 0x7fffffff;
    }
    float thr = -INFINITY, gthr = -INFINITY;
    int ab = 0;
    uint32_t aphase = 0;
    for (int t = t0; t < t1; ++t) {
      if (!mbar_wait(&tfull[ab], aphase, a.status, abort_flag)) break;
      tc_fence_after();
      float acc[32];
      const uint32_t taddr =
          tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(ab * S::NT + g * 32);
      {
        float v[16];
        tmem_ld16(taddr, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] = v[i];
        tmem_ld16(taddr + 16, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[16 + i] = v[i];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[ab]);
      ab ^= 1;
      if (ab == 0) aphase ^= 1;
      const int xq = t * kTileV + 32 * q;  // first vocabulary row of this quadrant

      if (MODE != EPI_EXPAND) {
        // lanes = consecutive rows: stores coalesce across the warp
        const int x = xq + lane;
        if (x < a.V) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const ColMeta& cm = meta[g * 32 + j];
            if (!cm.valid) continue;
            const float bias = a.l_bf16 ? bf16_to_f32(((const uint16_t*)a.L)[cm.bias_off + x])
                                        : ((const float*)a.L)[cm.bias_off + x];
            const float z = acc[j] + bias;
            if (MODE == EPI_ZDUMP)
              a.out[(size_t)cm.out_row * a.V + x] = z;
            else
              a.out[((size_t)cm.b * a.nmax1 + cm.out_row) * a.V + x] =
                  expf(__fdiv_rn(z, temp) - cm.lse);
          }
        }
        continue;
      }
      // transpose 32 rows x 32 columns: thread `lane` takes column g*32+lane
#pragma unroll
      for (int j = 0; j < 32; ++j) tb[lane * kTLD + j] = acc[j];
      __syncwarp();
#pragma unroll
      for (int i = 0; i < 32; ++i) acc[i] = tb[i * kTLD + lane];
      __syncwarp();
      if (!mc.valid) continue;
      const int nv = min(32, a.V - xq);
      if (nv <= 0) continue;
      float bias[32];
      load_bias32(a.L, a.l_bf16, mc.bias_off + xq, nv, vec, bias);
      float s[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float z = acc[i] + bias[i];
        s[i] = i < nv ? (STOCH ? __fdiv_rn(z, temp) : z) : -INFINITY;
      }
      // log-sum-exp, batched over the 32 values
      float mt = s[0];
#pragma unroll
      for (int i = 1; i < 32; ++i) mt = fmaxf(mt, s[i]);
      float st = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) st += exp2f((s[i] - mt) * kLog2e);
      if (mt > m) {
        ssum = ssum * exp2f((m - mt) * kLog2e) + st;
        m = mt;
      } else {
        ssum += st * exp2f((mt - m) * kLog2e);
      }
      // top-k of s (values arrive in increasing token order)
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        if (s[i] > thr) {
          topk_insert<KMAX>(L1, I1, s[i], xq + i);
          thr = kth<KMAX>(L1, k);
        }
      }
      if constexpr (STOCH) {
        // Gumbel keys; four consecutive tokens share one Philox counter
#pragma unroll
        for (int gi = 0; gi < 8; ++gi) {
          const float smax =
              fmaxf(fmaxf(s[4 * gi], s[4 * gi + 1]), fmaxf(s[4 * gi + 2], s[4 * gi + 3]));
          if (!(smax + kGumbelMax > gthr)) continue;
          const uint32_t x4 = (uint32_t)(xq + 4 * gi);
          const U4 o = philox10(U4{(x4 >> 2) | ((uint32_t)mc.b << 18), mc.c1, mc.c2, a.offset},
                                (uint32_t)a.seed, (uint32_t)(a.seed >> 32));
          const uint32_t wds[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int i = 4 * gi + j;
            if (i >= nv) continue;
            const float gk = s[i] + (-logf(-logf(u23(wds[j]))));
            if (gk > gthr) {
              topk_insert<KMAX>(L2, I2, gk, xq + i);
              gthr = kth<KMAX>(L2, k);
            }
          }
        }
      }
    }
    if (MODE == EPI_EXPAND) {
      // publish this quadrant's partial of the owned column
      qst[q * S::NT + col] = make_float2(m, ssum);
#pragma unroll
      for (int i = 0; i < KMAX; ++i) {
        ql1v[(q * S::NT + col) * KMAX + i] = L1[i];
        ql1i[(q * S::NT + col) * KMAX + i] = I1[i];
        if (STOCH) {
          ql2v[(q * S::NT + col) * KMAX + i] = L2[i];
          ql2i[(q * S::NT + col) * KMAX + i] = I2[i];
        }
      }
      named_bar(1, S::kEpiWarps * 32);
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
        const size_t pidx = (size_t)cx * a.Mcap + row;
        a.stats[pidx] = make_float2(mx, sv);
        // 4-way merge of the quadrants' sorted lists of this column
        for (int lst = 0; lst < (STOCH ? 2 : 1); ++lst) {
          const float* LV = lst ? ql2v : ql1v;
          const int32_t* LI = lst ? ql2i : ql1i;
          float* OV = (lst ? a.gv : a.lv) + pidx * k;
          int32_t* OI = (lst ? a.gi : a.li) + pidx * k;
          int hpos[4] = {0, 0, 0, 0};
          for (int i = 0; i < k; ++i) {
            int bw = -1;
            float bv = -INFINITY;
            int32_t bi = 0x7fffffff;
            for (int w = 0; w < 4; ++w) {
              if (hpos[w] >= k) continue;
              const float v = LV[(w * S::NT + c) * KMAX + hpos[w]];
              const int32_t id = LI[(w * S::NT + c) * KMAX + hpos[w]];
              if (bw < 0 || ranks_before(v, id, bv, bi)) {
                bw = w;
                bv = v;
                bi = id;
              }
            }
            if (bw >= 0) hpos[bw]++;
            OV[i] = bv;
            OI[i] = bi;
          }
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

template <int NG, int MODE, bool STOCH, int KMAX>
static cudaError_t launch_cfg(const CUtensorMap& tmW, const CUtensorMap& tmH, GemmArgs a,
                              int batch, int n_node_tiles, cudaStream_t s) {
  using SH = GemmShape<NG>;
  auto kern = markov_gemm_kernel<NG, MODE, STOCH, KMAX>;
  // the deepest pipeline that fits in 220 KB of shared memory
  int stages = 8;
  while (stages > 2 && gemm_smem_bytes<NG>(stages, KMAX, STOCH) > 220 * 1024) --stages;
  a.stages = stages;
  const size_t smem = gemm_smem_bytes<NG>(stages, KMAX, STOCH);
  cudaError_t e = ensure_smem(kern, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.ncta_v, n_node_tiles);
  kern<<<grid, SH::kThreads, smem, s>>>(tmW, tmH, a, batch);
  return cudaGetLastError();
}

// Node columns per tile the launcher uses for a given column capacity.
int gemm_node_tile(int max_cols) { return max_cols <= 32 ? 32 : 64; }

cudaError_t launch_markov_gemm(int mode, bool stoch, const CUtensorMap& tmW,
                               const CUtensorMap& tmH, const GemmArgs& a, int batch, int nt,
                               cudaStream_t s) {
  const int ntiles = (a.Mcap + nt - 1) / nt;
  const int ng = nt / 32;
  const int kmax = a.k <= 4 ? 4 : 16;
#define DT_GEMM_CASE(NG, MODE, ST, KM)                                          \
  if (ng == NG && mode == MODE && stoch == ST && (MODE != EPI_EXPAND || kmax == KM)) \
    return launch_cfg<NG, MODE, ST, KM>(tmW, tmH, a, batch, ntiles, s);
  DT_GEMM_CASE(1, EPI_EXPAND, false, 4)
  DT_GEMM_CASE(1, EPI_EXPAND, false, 16)
  DT_GEMM_CASE(2, EPI_EXPAND, false, 4)
  DT_GEMM_CASE(2, EPI_EXPAND, false, 16)
  DT_GEMM_CASE(1, EPI_EXPAND, true, 4)
  DT_GEMM_CASE(1, EPI_EXPAND, true, 16)
  DT_GEMM_CASE(2, EPI_EXPAND, true, 4)
  DT_GEMM_CASE(2, EPI_EXPAND, true, 16)
  DT_GEMM_CASE(1, EPI_ZDUMP, false, 4)
  DT_GEMM_CASE(2, EPI_ZDUMP, false, 4)
  DT_GEMM_CASE(1, EPI_QROWS, true, 4)
  DT_GEMM_CASE(2, EPI_QROWS, true, 4)
#undef DT_GEMM_CASE
  return cudaErrorInvalidValue;
}

}  // namespace dt
