// Tree-masked grouped-query attention: verify every draft node in one pass.
//
// Source: TreeSpark article, introduction (the target model checks all tree
// nodes in one forward); PCTree summary, "setup" (SDPA attention).  Row i of
// request b (0 = root, i = node i-1) attends to the request's KV prefix, the
// root's tree row, and tree row j+1 iff node j is node i-1 or one of its
// ancestors (bit j of anc[b][i-1]).
//
// bf16 path: split-KV ("flash-decoding") over 64-column chunks.  A CTA owns one
// (request, KV head, column split, row block); its query rows are the G = Hq/Hkv
// heads sharing the KV head times the tree rows, so every K/V chunk read from
// HBM serves all of them.  Q.K^T and P.V run on warp-level bf16 MMAs with fp32
// accumulation and an online softmax; the ancestor bitmask is applied only to
// the tree columns.  A combine kernel merges the splits.  fp32 inputs use a
// plain per-(row, head) kernel.
#include <algorithm>

#include "attn_tc.cuh"

namespace dt {

constexpr int kChunk = 64;
constexpr float kAttnL2e = 1.4426950408889634f;

struct AttnArgs {
  const void* q;
  const void* kp;
  const void* vp;
  const int64_t* pstart;
  const int32_t* plen;
  const void* kt;
  const void* vt;
  const uint64_t* anc;
  const int32_t* n_nodes;
  int batch, Nmax, Hq, Hkv, d, G, max_prefix;
  float scale;
  int splits, cols_per_split, rows_per_cta, n_rblocks, rpad;
  float* part_o;   // [splits][batch][Hkv][n_rblocks*rpad][d]
  float2* part_ml; // [splits][batch][Hkv][n_rblocks*rpad]
  void* out;
  int out_bf16;
  int32_t* status;
};

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// 16-byte global -> shared copy that does not block the thread; zero-fills
// the destination when `pred` is false.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool pred) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(pred ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Is tree column j (0 = root, j' + 1 = node j') visible from tree row i?
__device__ __forceinline__ bool tree_visible(int i, int j, uint64_t anc_row) {
  return j == 0 || (i >= 1 && ((anc_row >> (j - 1)) & 1ull));
}

template <int D>
__global__ void __launch_bounds__(512) attn_bf16_kernel(AttnArgs a) {
  constexpr int LD = D + 8;  // padded row (bf16 elements) against bank conflicts
  extern __shared__ __align__(16) uint8_t asmem[];
  uint16_t* sQ = (uint16_t*)asmem;                 // [rows_per_cta][LD]
  uint16_t* sKV = sQ + (size_t)a.rows_per_cta * LD; // 2 x ([kChunk][LD] K, [kChunk][LD] V)
  const int split = blockIdx.x, kvh = blockIdx.y;
  const int b = blockIdx.z / a.n_rblocks, rb = blockIdx.z % a.n_rblocks;
  const int n = min(max(a.n_nodes[b], 0), a.Nmax);
  const int P = min(max(a.plen[b], 0), a.max_prefix);
  if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0 && rb == 0 &&
      (a.n_nodes[b] != n || a.plen[b] != P))
    set_status(a.status, DT_EDEVICE);
  const int R = a.G * (n + 1);
  const int row0 = rb * a.rows_per_cta;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nthreads = blockDim.x;
  const int C = P + n + 1;
  const int c0 = split * a.cols_per_split, c1 = min(C, c0 + a.cols_per_split);
  const size_t pbase = (((size_t)split * a.batch + b) * a.Hkv + kvh) * (size_t)(a.n_rblocks * a.rpad) +
                       row0;
  if (row0 >= R) return;
  // ---- Q rows of this block: rho = i * G + hh  ->  q[b][i][kvh*G + hh]
  const uint16_t* q = (const uint16_t*)a.q;
  for (int idx = tid; idx < a.rows_per_cta * (D / 8); idx += nthreads) {
    const int rr = idx / (D / 8), cc = idx % (D / 8);
    const int rho = row0 + rr;
    const bool ok = rho < R;
    const int i = ok ? rho / a.G : 0, hh = ok ? rho % a.G : 0;
    cp_async16(sQ + (size_t)rr * LD + cc * 8,
               q + (((size_t)b * (a.Nmax + 1) + i) * a.Hq + kvh * a.G + hh) * D + cc * 8, ok);
  }
  // per-lane rows (g and g + 8 of the warp's 16-row tile)
  const int g = lane >> 2, t4 = lane & 3;
  const int rloc0 = warp * 16 + g, rloc1 = rloc0 + 8;
  const int rho0 = row0 + rloc0, rho1 = row0 + rloc1;
  const int i0 = rho0 / a.G, i1 = rho1 / a.G;
  const uint64_t anc0 = (rho0 < R && i0 >= 1) ? a.anc[(size_t)b * a.Nmax + i0 - 1] : 0ull;
  const uint64_t anc1 = (rho1 < R && i1 >= 1) ? a.anc[(size_t)b * a.Nmax + i1 - 1] : 0ull;
  const bool warp_active = warp * 16 < a.rows_per_cta;

  float o[D / 8][4];
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const float sl2 = a.scale * kAttnL2e;
  const uint16_t* kp = (const uint16_t*)a.kp;
  const uint16_t* vp = (const uint16_t*)a.vp;
  const uint16_t* ktr = (const uint16_t*)a.kt;
  const uint16_t* vtr = (const uint16_t*)a.vt;
  const int64_t ps = a.pstart[b];

  // K/V chunk loader: buffer `buf` <- columns [cb, cb + kChunk)
  auto load_chunk = [&](int cb, int buf) {
    uint16_t* dK = sKV + (size_t)buf * 2 * kChunk * LD;
    uint16_t* dV = dK + kChunk * LD;
    for (int idx = tid; idx < kChunk * (D / 8); idx += nthreads) {
      const int rr = idx / (D / 8), cc = idx % (D / 8);
      const int c = cb + rr;
      const bool ok = c < c1;
      size_t off;
      const uint16_t *ks, *vs;
      if (!ok) {  // zero-filled; the source is any valid address
        off = 0;
        ks = ktr;
        vs = vtr;
      } else if (c < P) {
        off = ((size_t)(ps + c) * a.Hkv + kvh) * D + cc * 8;
        ks = kp;
        vs = vp;
      } else {
        off = (((size_t)b * (a.Nmax + 1) + (c - P)) * a.Hkv + kvh) * D + cc * 8;
        ks = ktr;
        vs = vtr;
      }
      cp_async16(dK + (size_t)rr * LD + cc * 8, ks + off, ok);
      cp_async16(dV + (size_t)rr * LD + cc * 8, vs + off, ok);
    }
  };
  if (c0 < c1) load_chunk(c0, 0);
  cp_async_commit();  // group: Q + first chunk
  int buf = 0;
  for (int cb = c0; cb < c1; cb += kChunk, buf ^= 1) {
    if (cb + kChunk < c1) load_chunk(cb + kChunk, buf ^ 1);
    cp_async_commit();
    cp_async_wait<1>();  // everything but the chunk just issued has landed
    __syncthreads();
    const uint16_t* sK = sKV + (size_t)buf * 2 * kChunk * LD;
    const uint16_t* sV = sK + kChunk * LD;
    if (warp_active) {
    // S = Q K^T for 16 rows x 64 columns
    float s[kChunk / 8][4];
#pragma unroll
    for (int nt = 0; nt < kChunk / 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t af[4];
      ldsm_x4(af, smem_u32(sQ + (size_t)(warp * 16 + (lane & 15)) * LD + kk * 16 + (lane >> 4) * 8));
#pragma unroll
      for (int nt = 0; nt < kChunk / 8; nt += 2) {
        uint32_t bf[4];
        const int mi = lane >> 3, rr = lane & 7;
        ldsm_x4(bf, smem_u32(sK + (size_t)(8 * (nt + (mi >> 1)) + rr) * LD + kk * 16 + (mi & 1) * 8));
        mma_bf16_16816(s[nt], af, bf[0], bf[1]);
        mma_bf16_16816(s[nt + 1], af, bf[2], bf[3]);
      }
    }
    // mask + online softmax (rows rho0, rho1)
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < kChunk / 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = cb + nt * 8 + 2 * t4 + (e & 1);
        const bool r1 = e >= 2;
        const int rho = r1 ? rho1 : rho0;
        bool ok = c < c1 && rho < R;
        if (ok && c >= P) ok = tree_visible(r1 ? i1 : i0, c - P, r1 ? anc1 : anc0);
        const float v = ok ? s[nt][e] * sl2 : -INFINITY;
        s[nt][e] = v;
        if (r1)
          mx1 = fmaxf(mx1, v);
        else
          mx0 = fmaxf(mx0, v);
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float al0 = (mn0 == -INFINITY) ? 1.f : exp2f(m0 - mn0);
    const float al1 = (mn1 == -INFINITY) ? 1.f : exp2f(m1 - mn1);
    float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < kChunk / 8; ++nt) {
      s[nt][0] = (mn0 == -INFINITY) ? 0.f : exp2f(s[nt][0] - mn0);
      s[nt][1] = (mn0 == -INFINITY) ? 0.f : exp2f(s[nt][1] - mn0);
      s[nt][2] = (mn1 == -INFINITY) ? 0.f : exp2f(s[nt][2] - mn1);
      s[nt][3] = (mn1 == -INFINITY) ? 0.f : exp2f(s[nt][3] - mn1);
      rs0 += s[nt][0] + s[nt][1];
      rs1 += s[nt][2] + s[nt][3];
    }
    l0 = l0 * al0 + rs0;  // per-lane partial row sums; reduced over the quad at the end
    l1 = l1 * al1 + rs1;
    m0 = mn0;
    m1 = mn1;
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
      o[nt][0] *= al0;
      o[nt][1] *= al0;
      o[nt][2] *= al1;
      o[nt][3] *= al1;
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < kChunk / 16; ++kk) {
      uint32_t af[4];
      af[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      af[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      af[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      af[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int nt = 0; nt < D / 8; nt += 2) {
        uint32_t bf[4];
        const int mi = lane >> 3, rr = lane & 7;
        ldsm_x4_t(bf, smem_u32(sV + (size_t)(kk * 16 + (mi & 1) * 8 + rr) * LD + 8 * (nt + (mi >> 1))));
        mma_bf16_16816(o[nt], af, bf[0], bf[1]);
        mma_bf16_16816(o[nt + 1], af, bf[2], bf[3]);
      }
    }
    }  // warp_active
    __syncthreads();  // buffer `buf` is refilled by the next iteration's loads
  }
  cp_async_wait<0>();
  if (!warp_active) return;
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  if (rloc0 < a.rows_per_cta && rho0 < R) {
    float* po = a.part_o + (pbase + rloc0) * D;
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt)
      *(float2*)(po + nt * 8 + 2 * t4) = make_float2(o[nt][0], o[nt][1]);
    if (t4 == 0) a.part_ml[pbase + rloc0] = make_float2(m0, l0);
  }
  if (rloc1 < a.rows_per_cta && rho1 < R) {
    float* po = a.part_o + (pbase + rloc1) * D;
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt)
      *(float2*)(po + nt * 8 + 2 * t4) = make_float2(o[nt][2], o[nt][3]);
    if (t4 == 0) a.part_ml[pbase + rloc1] = make_float2(m1, l1);
  }
}

constexpr int kMaxSplits = 512;
constexpr int kCombineWarps = 4;

// Merge the column splits: one warp per (request, row, head); lanes cover
// head_dim in 4-float vectors.  grid (ceil(batch*(Nmax+1)*Hq / 4)), 128 threads.
__global__ void attn_combine_kernel(AttnArgs a) {
  pdl_wait();  // the attention kernel's partials (no-op without a programmatic launch)
  const int lane = threadIdx.x & 31;
  const int item = blockIdx.x * kCombineWarps + (threadIdx.x >> 5);
  const int per_b = (a.Nmax + 1) * a.Hq;
  if (item >= a.batch * per_b) return;
  const int b = item / per_b, i = (item % per_b) / a.Hq, h = item % a.Hq;
  if (i > min(a.n_nodes[b], a.Nmax)) return;
  const int kvh = h / a.G, hh = h % a.G;
  const int rho = i * a.G + hh;
  const int rb = rho / a.rows_per_cta, rl = rho % a.rows_per_cta;
  const int P = min(max(a.plen[b], 0), a.max_prefix);
  const int C = P + min(max(a.n_nodes[b], 0), a.Nmax) + 1;
  const int used = min((C + a.cols_per_split - 1) / a.cols_per_split, kMaxSplits);
  const size_t split_stride = (size_t)a.batch * a.Hkv * a.n_rblocks * a.rpad;
  const size_t pb0 = ((size_t)b * a.Hkv + kvh) * (size_t)(a.n_rblocks * a.rpad) +
                     rb * a.rows_per_cta + rl;
  float mx = -INFINITY;
  for (int s = lane; s < used; s += 32) mx = fmaxf(mx, a.part_ml[pb0 + s * split_stride].x);
  mx = warp_max(mx);
  float l = 0.f;
  for (int s = lane; s < used; s += 32) {
    const float2 ml = a.part_ml[pb0 + s * split_stride];
    if (ml.x != -INFINITY) l += exp2f(ml.x - mx) * ml.y;
  }
  l = warp_sum(l);
  const float inv_l = 1.f / l;
  const int nvec = a.d / 4;  // 16 or 32 float4 per row
  if (lane < nvec) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    // kBatch splits per pass: all their loads are issued before the first
    // use, so a pass costs one memory round trip; the sum keeps split order
    constexpr int kBatch = 16;
    for (int s0 = 0; s0 < used; s0 += kBatch) {
      float2 ml[kBatch];
      float4 o[kBatch];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int s = s0 + j;
        if (s < used) {
          ml[j] = a.part_ml[pb0 + s * split_stride];
          o[j] = ((const float4*)(a.part_o + (pb0 + s * split_stride) * a.d))[lane];
        } else {
          ml[j] = make_float2(-INFINITY, 0.f);
          o[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        if (s0 + j >= used) break;
        const float w = ml[j].x == -INFINITY ? 0.f : exp2f(ml[j].x - mx);
        acc.x += w * o[j].x;
        acc.y += w * o[j].y;
        acc.z += w * o[j].z;
        acc.w += w * o[j].w;
      }
    }
    const size_t oi = (((size_t)b * (a.Nmax + 1) + i) * a.Hq + h) * a.d + 4 * lane;
    if (a.out_bf16) {
      uint2 pk;
      pk.x = pack_bf16(acc.x * inv_l, acc.y * inv_l);
      pk.y = pack_bf16(acc.z * inv_l, acc.w * inv_l);
      *(uint2*)((uint16_t*)a.out + oi) = pk;
    } else {
      *(float4*)((float*)a.out + oi) =
          make_float4(acc.x * inv_l, acc.y * inv_l, acc.z * inv_l, acc.w * inv_l);
    }
  }
}

// fp32 inputs: one CTA per (request, row, head); scores staged in shared memory.
__global__ void attn_f32_kernel(AttnArgs a, int max_cols) {
  extern __shared__ float sc[];
  const int b = blockIdx.x / (a.Nmax + 1), i = blockIdx.x % (a.Nmax + 1);
  const int h = blockIdx.y;
  const int n = min(max(a.n_nodes[b], 0), a.Nmax);
  if (i > n) return;
  const int kvh = h / a.G;
  const int P = min(max(a.plen[b], 0), a.max_prefix);
  const int C = P + n + 1;
  if (C > max_cols) {
    set_status(a.status, DT_EDEVICE);
    return;
  }
  const float* q = (const float*)a.q + (((size_t)b * (a.Nmax + 1) + i) * a.Hq + h) * a.d;
  const uint64_t anc = i >= 1 ? a.anc[(size_t)b * a.Nmax + i - 1] : 0ull;
  const int64_t ps = a.pstart[b];
  __shared__ float red[32];
  float mx = -INFINITY;
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    const float* kr;
    bool ok = true;
    if (c < P)
      kr = (const float*)a.kp + ((size_t)(ps + c) * a.Hkv + kvh) * a.d;
    else {
      kr = (const float*)a.kt + (((size_t)b * (a.Nmax + 1) + (c - P)) * a.Hkv + kvh) * a.d;
      ok = tree_visible(i, c - P, anc);
    }
    float dot = 0.f;
    for (int e = 0; e < a.d; ++e) dot = fmaf(q[e], kr[e], dot);
    const float v = ok ? dot * a.scale : -INFINITY;
    sc[c] = v;
    mx = fmaxf(mx, v);
  }
  mx = warp_max(mx);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < blockDim.x / 32 ? red[threadIdx.x] : -INFINITY;
    v = warp_max(v);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  mx = red[0];
  __syncthreads();
  float sum = 0.f;
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    const float e = expf(sc[c] - mx);
    sc[c] = e;
    sum += e;
  }
  sum = warp_sum(sum);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = sum;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < blockDim.x / 32 ? red[threadIdx.x] : 0.f;
    v = warp_sum(v);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float tot = red[0];
  for (int e = threadIdx.x; e < a.d; e += blockDim.x) {
    float acc = 0.f;
    for (int c = 0; c < C; ++c) {
      const float* vr = c < P ? (const float*)a.vp + ((size_t)(ps + c) * a.Hkv + kvh) * a.d
                              : (const float*)a.vt +
                                    (((size_t)b * (a.Nmax + 1) + (c - P)) * a.Hkv + kvh) * a.d;
      acc = fmaf(sc[c], vr[e], acc);
    }
    ((float*)a.out)[(((size_t)b * (a.Nmax + 1) + i) * a.Hq + h) * a.d + e] = acc / tot;
  }
}

struct AttnPlan {
  int splits, cols_per_split, rows_per_cta, n_rblocks, rpad, warps;
  size_t part_o_bytes, part_ml_bytes;
};

// The tensor-core kernel (attn_tc.cu): 128-column splits, one partial row per
// (tree row, query head) of each KV head.
static AttnPlan attn_tc_plan(int batch, int Nmax, int Hq, int Hkv, int d, int max_prefix) {
  AttnPlan p;
  const int G = Hq / Hkv;
  p.n_rblocks = 1;
  p.rows_per_cta = p.rpad = G * (Nmax + 1);
  p.warps = 4;
  p.cols_per_split = 128;
  p.splits = (max_prefix + Nmax + 1 + 127) / 128;
  const size_t rows = (size_t)p.splits * batch * Hkv * p.rpad;
  p.part_o_bytes = rows * d * 4;
  p.part_ml_bytes = rows * 8;
  return p;
}

static AttnPlan attn_plan(int batch, int Nmax, int Hq, int Hkv, int d, int max_prefix) {
  AttnPlan p;
  const int G = Hq / Hkv;
  const int Rmax = G * (Nmax + 1);
  p.n_rblocks = (Rmax + 255) / 256;
  const int per = (Rmax + p.n_rblocks - 1) / p.n_rblocks;
  p.warps = (per + 15) / 16;
  p.rows_per_cta = p.warps * 16;
  p.rpad = p.rows_per_cta;
  const int Cmax = max_prefix + Nmax + 1;
  const int chunks = (Cmax + kChunk - 1) / kChunk;
  const int base_ctas = batch * Hkv * p.n_rblocks;
  int want = (148 + base_ctas - 1) / base_ctas;
  want = std::max(1, std::min(want, chunks));
  const int chunks_per = (chunks + want - 1) / want;
  p.cols_per_split = chunks_per * kChunk;
  p.splits = (chunks + chunks_per - 1) / chunks_per;  // at most 2 * 148 <= kMaxSplits
  const size_t rows = (size_t)p.splits * batch * Hkv * p.n_rblocks * p.rpad;
  p.part_o_bytes = rows * d * 4;
  p.part_ml_bytes = rows * 8;
  return p;
}

}  // namespace dt

using namespace dt;

extern "C" {

size_t dt_tree_verify_attn_workspace_bytes(int batch, int Nmax, int Hq, int Hkv, int d,
                                           int max_prefix) {
  if (batch <= 0 || Nmax <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || d <= 0 || max_prefix < 0)
    return 0;
  AttnPlan p = attn_plan(batch, Nmax, Hq, Hkv, d, max_prefix);
  AttnPlan t = attn_tc_plan(batch, Nmax, Hq, Hkv, d, max_prefix);
  const size_t ml = std::max(p.part_ml_bytes, t.part_ml_bytes);
  const size_t o = std::max(p.part_o_bytes, t.part_o_bytes);
  return kWsHeader + ((ml + 255) & ~(size_t)255) + o + 256;
}

dt_status dt_tree_verify_attn(const void* d_q, const void* d_k_prefix, const void* d_v_prefix,
                              const int64_t* d_prefix_start, const int32_t* d_prefix_len,
                              int max_prefix, const void* d_k_tree, const void* d_v_tree,
                              const uint64_t* d_anc, const int32_t* d_n_nodes, int batch,
                              int Nmax, int Hq, int Hkv, int d, float scale, dt_dtype dt,
                              void* d_out, void* ws, size_t ws_bytes, dt_stream stream) {
  if (!d_q || !d_k_prefix || !d_v_prefix || !d_prefix_start || !d_prefix_len || !d_k_tree ||
      !d_v_tree || !d_anc || !d_n_nodes || !d_out)
    return DT_EINVAL;
  if (dt != DT_F32 && dt != DT_BF16) return DT_EINVAL;
  if (batch < 1 || Nmax < 1 || Hq < 1 || Hkv < 1 || max_prefix < 0 || !(scale > 0.f))
    return DT_EINVAL;
  if (Hq % Hkv) return DT_EINVAL;
  if (Nmax > 64 || (d != 64 && d != 128) || batch > 65535) return DT_EUNSUPPORTED;
  const size_t need = dt_tree_verify_attn_workspace_bytes(batch, Nmax, Hq, Hkv, d, max_prefix);
  if (!ws || ws_bytes < need) return DT_EWORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  // bf16: the tensor-core kernel; fp32 inputs: the plain per-(row, head) kernel
  const bool tc = dt == DT_BF16;
  AttnPlan p = tc ? attn_tc_plan(batch, Nmax, Hq, Hkv, d, max_prefix)
                  : attn_plan(batch, Nmax, Hq, Hkv, d, max_prefix);
  AttnArgs a;
  a.q = d_q;
  a.kp = d_k_prefix;
  a.vp = d_v_prefix;
  a.pstart = d_prefix_start;
  a.plen = d_prefix_len;
  a.kt = d_k_tree;
  a.vt = d_v_tree;
  a.anc = d_anc;
  a.n_nodes = d_n_nodes;
  a.batch = batch;
  a.Nmax = Nmax;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.d = d;
  a.G = Hq / Hkv;
  a.max_prefix = max_prefix;
  a.scale = scale;
  a.splits = p.splits;
  a.cols_per_split = p.cols_per_split;
  a.rows_per_cta = p.rows_per_cta;
  a.n_rblocks = p.n_rblocks;
  a.rpad = p.rpad;
  uint8_t* w = (uint8_t*)ws;
  a.status = (int32_t*)w;
  {
    AttnPlan p0 = attn_plan(batch, Nmax, Hq, Hkv, d, max_prefix);
    const size_t ml = std::max(p0.part_ml_bytes, p.part_ml_bytes);
    a.part_ml = (float2*)(w + kWsHeader);
    a.part_o = (float*)(w + kWsHeader + ((ml + 255) & ~(size_t)255));
  }
  a.out = d_out;
  a.out_bf16 = dt == DT_BF16;
  if (cudaMemsetAsync(a.status, 0, 4, s) != cudaSuccess) return DT_ECUDA;
  if (dt == DT_F32) {
    const int max_cols = max_prefix + Nmax + 1;
    const size_t smem = (size_t)max_cols * 4;
    if (smem > 200 * 1024) return DT_EUNSUPPORTED;
    if (ensure_smem(attn_f32_kernel, smem) != cudaSuccess)
      return DT_ECUDA;
    ProfileScope ps(DT_K_ATTN, s);
    attn_f32_kernel<<<dim3(batch * (Nmax + 1), Hq), 128, smem, s>>>(a, max_cols);
    return cudaGetLastError() == cudaSuccess ? DT_OK : DT_ECUDA;
  }
  {
    AttnTcArgs t;
    t.q = (const uint16_t*)d_q;
    t.kp = (const uint16_t*)d_k_prefix;
    t.vp = (const uint16_t*)d_v_prefix;
    t.pstart = d_prefix_start;
    t.plen = d_prefix_len;
    t.kt = (const uint16_t*)d_k_tree;
    t.vt = (const uint16_t*)d_v_tree;
    t.anc = d_anc;
    t.n_nodes = d_n_nodes;
    t.batch = batch;
    t.Nmax = Nmax;
    t.Hq = Hq;
    t.Hkv = Hkv;
    t.d = d;
    t.G = Hq / Hkv;
    t.max_prefix = max_prefix;
    t.heads_per_cta = attn_tc_heads_per_cta(t.G, Nmax);
    t.n_groups = t.G / t.heads_per_cta;
    t.scale_log2 = scale * kAttnL2e;
    t.part_o = a.part_o;
    t.part_ml = a.part_ml;
    t.splits = p.splits;
    t.rpad = p.rpad;
    t.status = a.status;
    ProfileScope ps(DT_K_ATTN, s);
    if (launch_attn_tc(t, s) != cudaSuccess) return DT_ECUDA;
  }
  ProfileScope ps(DT_K_ATTN_COMBINE, s);
  const int items = batch * (Nmax + 1) * Hq;
  const dim3 cgrid((items + kCombineWarps - 1) / kCombineWarps);
  if (tc) {
    // launched while the attention kernel runs; it waits for its partials
    if (launch_pdl(attn_combine_kernel, cgrid, dim3(32 * kCombineWarps), 0, s, a) != cudaSuccess)
      return DT_ECUDA;
  } else {
    attn_combine_kernel<<<cgrid, 32 * kCombineWarps, 0, s>>>(a);
  }
  return cudaGetLastError() == cudaSuccess ? DT_OK : DT_ECUDA;
}

}  // extern "C"
