// Tree-masked grouped-query attention on the 5th-generation tensor cores.
//
// Source: TreeSpark article, introduction (the target model checks every
// tree node in one forward pass); PCTree summary, "setup" paragraph (SDPA
// attention) and limitations paragraph (verification cost grows with N).
// Row i of request b (0 = root, i = node i-1) attends to the request's KV
// prefix, the root's tree row, and tree row j+1 iff node j is node i-1 or one
// of its ancestors (bit j of anc[b][i-1]).
//
// Split-KV ("flash-decoding"): a CTA owns one split of 128 key columns of one
// request's column space (the prefix, then the tree rows), one KV head and a
// group of the query heads that share it: its M = 128 MMA rows are
// (query head of the group) x (tree row), as many heads as fit.  Per CTA:
//   S = Q K^T      tcgen05.mma, M = 128 rows, N = 128 keys, K = d; fp32 in TMEM
//   softmax        one thread per row reads its S row from TMEM, applies the
//                  scale and the ancestor mask (tree columns only), and writes
//                  P = exp2(s - m) in bf16 to shared memory
//   O = P V        tcgen05.mma, M = 128 rows, N = d, K = 128 keys; V is stored
//                  transposed (V^T [d][key], keys contiguous) so that both
//                  MMAs read K-major 128-byte-swizzled operands
// and writes its unnormalised O rows with (m, l); the split-combine kernel of
// verify_attn.cu merges the splits.  Q, K, V and P tiles sit in shared memory
// in the 128-byte-swizzled layouts the MMA descriptors describe; Q and K are
// loaded with 16-byte cp.async copies, since a split's keys may come partly
// from the packed prefix and partly from the tree rows, and V with 16-byte
// loads that are scattered transposed.
#include <algorithm>

#include "attn_tc.cuh"

namespace dt {

constexpr int kTcRows = 128;   // MMA M: query rows per CTA
constexpr int kTcKeys = 128;   // MMA N of Q K^T: key columns per split
constexpr int kTcThreads = 128;


// 16-byte chunk c of row r of a 128-byte-swizzled tile (8-row, 1024-byte atoms)
__device__ __forceinline__ uint32_t sw128(int r, int c) {
  return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ void cp16(uint32_t dst, const void* src, bool ok) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(ok ? 16 : 0)
               : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1) attn_tc_kernel(AttnTcArgs a) {
  constexpr int KC = D / 64;                   // 64-element chunks of d
  constexpr int kTile = kTcRows * 128;         // bytes of one 128-row x 64 chunk
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sq = smem;                          // Q:  [KC][128 rows][128 B]  K-major
  uint8_t* sk = sq + (KC > 2 ? KC : 2) * kTile; // K:  [KC][128 keys][128 B]  K-major
  uint8_t* sv = sk + KC * kTile;               // V^T: [2 key halves][D rows][128 B] K-major
  uint8_t* sp = sq;                            // P:  [2][128 rows][128 B]   K-major, over Q
                                               //     (Q is dead once S is in TMEM)
  uint64_t* bar = (uint64_t*)(sv + 2 * D * 128);
  uint32_t* tslot = (uint32_t*)(bar + 2);
  volatile int* abort_flag = (volatile int*)(tslot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, kvh = blockIdx.y;
  const int b = blockIdx.z / a.n_groups, grp = blockIdx.z % a.n_groups;
  const int N1 = a.Nmax + 1;
  const int n = min(max(a.n_nodes[b], 0), a.Nmax);
  const int P = min(max(a.plen[b], 0), a.max_prefix);
  const int C = P + n + 1;                     // key columns of this request
  const int c0 = split * kTcKeys;
  pdl_launch_dependents();  // the split combine may be scheduled (it waits for us)
  if (c0 >= C) return;                         // uniform: nothing to attend to here
  const int64_t ps = a.pstart[b];
  const int hpc = a.heads_per_cta;

  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tslot, 256);  // S: columns 0-127, O: columns 128-255
    tc_fence_before();
  }

  // ---- tiles into shared memory (zero where there is no row / key)
  // Q: row m = hh * N1 + i  (query head kvh * G + grp * hpc + hh, tree row i)
  for (int idx = tid; idx < kTcRows * KC * 8; idx += kTcThreads) {
    const int c = idx & 7, m = (idx >> 3) % kTcRows, kc = (idx >> 3) / kTcRows;
    const int hh = m / N1, i = m % N1;
    const bool ok = hh < hpc && i <= n;
    const int head = kvh * a.G + grp * hpc + (ok ? hh : 0);
    const uint16_t* src = a.q + (((size_t)b * N1 + (ok ? i : 0)) * a.Hq + head) * D + kc * 64 + c * 8;
    cp16(smem_u32(sq + kc * kTile + sw128(m, c)), src, ok);
  }
  // K and V: key j of the split is column c0 + j: prefix row, or tree row
  for (int idx = tid; idx < kTcKeys * KC * 8; idx += kTcThreads) {
    const int c = idx & 7, j = (idx >> 3) % kTcKeys, kc = (idx >> 3) / kTcKeys;
    const int col = c0 + j;
    const bool ok = col < C;
    size_t off;
    const uint16_t* kb;
    if (col < P) {
      off = ((size_t)(ps + col) * a.Hkv + kvh) * D;
      kb = a.kp;
    } else {
      off = (((size_t)b * N1 + (ok ? col - P : 0)) * a.Hkv + kvh) * D;
      kb = a.kt;
    }
    off += kc * 64 + c * 8;
    cp16(smem_u32(sk + kc * kTile + sw128(j, c)), kb + (ok ? off : 0), ok);
  }
  // V^T: a thread takes keys 2 u, 2 u + 1 and 8 consecutive d, and stores the
  // 8 key pairs (4 bytes each) into 8 rows of V^T; lanes take consecutive
  // pairs, so a warp's stores fill 128 contiguous bytes of each row
  // (all of a thread's loads are issued before its first store)
  constexpr int kVItems = (kTcKeys / 2) * KC * 8 / kTcThreads;
  uint32_t vw[kVItems][2][4];
#pragma unroll
  for (int it = 0; it < kVItems; ++it) {
    const int idx = tid + it * kTcThreads;
    const int u = idx % (kTcKeys / 2), c = (idx / (kTcKeys / 2)) & 7,
              kc = idx / (kTcKeys / 2 * 8);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int col = c0 + 2 * u + h;
      const bool ok = col < C;
      size_t off;
      const uint16_t* vb;
      if (col < P) {
        off = ((size_t)(ps + col) * a.Hkv + kvh) * D;
        vb = a.vp;
      } else {
        off = (((size_t)b * N1 + (ok ? col - P : 0)) * a.Hkv + kvh) * D;
        vb = a.vt;
      }
      off += kc * 64 + c * 8;
      const uint4 v = ok ? *(const uint4*)(vb + off) : make_uint4(0, 0, 0, 0);
      vw[it][h][0] = v.x;
      vw[it][h][1] = v.y;
      vw[it][h][2] = v.z;
      vw[it][h][3] = v.w;
    }
  }
#pragma unroll
  for (int it = 0; it < kVItems; ++it) {
    const int idx = tid + it * kTcThreads;
    const int u = idx % (kTcKeys / 2), c = (idx / (kTcKeys / 2)) & 7,
              kc = idx / (kTcKeys / 2 * 8);
    // V[j][d] for d = 64 kc + 8 c + e  ->  V^T row d, keys j = 2 u, 2 u + 1
    const int j = 2 * u;
    uint8_t* vt = sv + (j >> 6) * (D * 128);
    const int jc = (j & 63) >> 3, jb = (j & 7) * 2;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int d = kc * 64 + c * 8 + e;
      const uint32_t lo = (vw[it][0][e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
      const uint32_t hi = (vw[it][1][e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
      *(uint32_t*)(vt + sw128(d, jc) + jb) = lo | (hi << 16);
    }
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  asm volatile("cp.async.wait_all;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  // ---- S = Q K^T (M = 128 rows, N = 128 keys, K = D)
  if (tid == 0) {
    constexpr uint32_t idesc = idesc_bf16_f32(kTcRows, kTcKeys);
    for (int kc = 0; kc < KC; ++kc) {
      const uint64_t da = smem_desc_k_sw128(smem_u32(sq + kc * kTile));
      const uint64_t db = smem_desc_k_sw128(smem_u32(sk + kc * kTile));
      for (int s = 0; s < 4; ++s)
        tc_mma_bf16(tmem, da + 2 * s, db + 2 * s, idesc, (kc | s) != 0 ? 1u : 0u);
    }
    tc_commit(&bar[0]);
  }
  // one lane per warp waits; the warp follows it as one (tcgen05.ld is warp-wide)
  __syncwarp();
  int okw = 1;
  if (lane == 0) okw = mbar_wait(&bar[0], 0, a.status, abort_flag) ? 1 : 0;
  bool ok = __shfl_sync(0xffffffffu, okw, 0) != 0;
  tc_fence_after();

  // ---- softmax of row m = tid (TMEM lane quadrant = warp)
  const int m = tid;
  const int hh = m / N1, i = m % N1;
  const bool row_ok = hh < hpc && i <= n;
  const uint64_t am = (row_ok && i >= 1) ? a.anc[(size_t)b * a.Nmax + (i - 1)] : 0ull;
  float s[kTcKeys];
  if (ok) {
    uint32_t r[kTcKeys / 16][16];
#pragma unroll
    for (int c4 = 0; c4 < kTcKeys / 16; ++c4)
      tmem_ld16_nowait(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)(16 * c4), r[c4]);
    tmem_wait_ld();
#pragma unroll
    for (int c4 = 0; c4 < kTcKeys / 16; ++c4)
#pragma unroll
      for (int e = 0; e < 16; ++e) s[16 * c4 + e] = __uint_as_float(r[c4][e]);
  }
  // allowed columns of this row among the split's 128, as 4 words of bits:
  // the prefix, the root's tree row, and the rows of the row's ancestors
  // (tree row t = node t - 1: bit t of 1 | anc << 1)
  uint32_t allow[kTcKeys / 32];
  {
    const uint64_t tlo = 1ull | (am << 1), thi = am >> 63;  // tree-row bits 0..64
#pragma unroll
    for (int wd = 0; wd < kTcKeys / 32; ++wd) {
      const int base = c0 + 32 * wd;  // column of bit 0
      const int npre = min(max(P - base, 0), 32);
      uint32_t word = npre == 32 ? 0xffffffffu : ((1u << npre) - 1u);
      // tree columns: bit k is column base + k = P + t with t = base - P + k
      const int t0 = base - P;
      uint32_t tb = 0;
      if (t0 > -32 && t0 <= 64) {
        // 32 bits of the tree mask from bit t0 (bits below 0 are prefix columns)
        uint64_t lo, hi;
        if (t0 >= 0) {
          lo = t0 < 64 ? (tlo >> t0) | (t0 ? (thi << (64 - t0)) : 0ull) : thi >> (t0 - 64);
          hi = 0;
          tb = (uint32_t)lo;
        } else {
          tb = (uint32_t)(tlo << (-t0));
        }
        (void)hi;
      }
      // columns at or past C (and past the tree) are not keys
      const int nval = min(max(C - base, 0), 32);
      const uint32_t inb = nval == 32 ? 0xffffffffu : ((1u << nval) - 1u);
      word = (word | (tb & ~word)) & inb;
      allow[wd] = row_ok ? word : 0u;
    }
  }
  float mx = -INFINITY;
#pragma unroll
  for (int j = 0; j < kTcKeys; ++j) {
    s[j] = ((allow[j >> 5] >> (j & 31)) & 1u) ? s[j] * a.scale_log2 : -INFINITY;
    mx = fmaxf(mx, s[j]);
  }
  float l = 0.f;
#pragma unroll
  for (int c8 = 0; c8 < kTcKeys / 8; ++c8) {
    float p[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float x = s[8 * c8 + e];
      float y;
      asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x - mx));  // 2^-inf = 0
      p[e] = (x == -INFINITY) ? 0.f : y;
      l += p[e];
    }
    uint4 pk;
    pk.x = pack_bf16x2(p[0], p[1]);
    pk.y = pack_bf16x2(p[2], p[3]);
    pk.z = pack_bf16x2(p[4], p[5]);
    pk.w = pack_bf16x2(p[6], p[7]);
    // key 8 c8 .. 8 c8 + 7 of row m: chunk (c8 & 7) of the 64-key half c8 >> 3
    *(uint4*)(sp + (c8 >> 3) * kTile + sw128(m, c8 & 7)) = pk;
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // ---- O = P V (M = 128 rows, N = D, K = 128 keys): A = P [row][key],
  // B = V^T [d][key], both K-major, one 64-key half per chunk
  if (tid == 0 && ok) {
    constexpr uint32_t idesc = idesc_bf16_f32(kTcRows, D);
    for (int kc = 0; kc < 2; ++kc) {
      const uint64_t da = smem_desc_k_sw128(smem_u32(sp + kc * kTile));
      const uint64_t db = smem_desc_k_sw128(smem_u32(sv + kc * (D * 128)));
      for (int s4 = 0; s4 < 4; ++s4)
        tc_mma_bf16(tmem + 128, da + 2 * s4, db + 2 * s4, idesc, (kc | s4) != 0 ? 1u : 0u);
    }
    tc_commit(&bar[1]);
  }
  __syncwarp();
  okw = 1;
  if (lane == 0) okw = (ok && mbar_wait(&bar[1], 0, a.status, abort_flag)) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, okw, 0) != 0;
  tc_fence_after();

  // ---- partial row: unnormalised O, (max, sum) in log2 units.  The TMEM
  // loads are warp-collective: every lane takes part, only real rows store.
  if (ok) {
    const int rho = i * a.G + grp * hpc + hh;
    const size_t prow = (((size_t)split * a.batch + b) * a.Hkv + kvh) * a.rpad + rho;
    if (row_ok) a.part_ml[prow] = make_float2(mx, l);
    float4* dst = (float4*)(a.part_o + prow * D);
    uint32_t r[D / 16][16];
#pragma unroll
    for (int c4 = 0; c4 < D / 16; ++c4)
      tmem_ld16_nowait(tmem + ((uint32_t)(32 * warp) << 16) + 128u + (uint32_t)(16 * c4), r[c4]);
    tmem_wait_ld();
    if (row_ok) {
#pragma unroll
      for (int c4 = 0; c4 < D / 16; ++c4)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          dst[4 * c4 + e] =
              make_float4(__uint_as_float(r[c4][4 * e]), __uint_as_float(r[c4][4 * e + 1]),
                          __uint_as_float(r[c4][4 * e + 2]), __uint_as_float(r[c4][4 * e + 3]));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// Q (or P over it: at least two chunks), K, V^T, barriers; two CTAs fit an
// SM at d = 128
size_t attn_tc_smem_bytes(int d) {
  const int kc = d / 64;
  return (size_t)((kc > 2 ? kc : 2) + kc) * kTcRows * 128 + (size_t)2 * d * 128 + 64 + 1024;
}

// Query heads per CTA: as many of the G heads of a KV head as fit in 128 rows
// (a divisor of G, so that every CTA of the KV head has the same group size).
int attn_tc_heads_per_cta(int G, int Nmax) {
  int h = std::max(1, std::min(G, kTcRows / (Nmax + 1)));
  while (G % h) --h;
  return h;
}

cudaError_t launch_attn_tc(const AttnTcArgs& a, cudaStream_t s) {
  if ((a.d != 64 && a.d != 128) || a.Nmax + 1 > kTcRows) return cudaErrorInvalidValue;
  const size_t smem = attn_tc_smem_bytes(a.d);
  auto kern = a.d == 128 ? attn_tc_kernel<128> : attn_tc_kernel<64>;
  cudaError_t e = ensure_smem(kern, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.splits, a.Hkv, a.batch * a.n_groups);
  kern<<<grid, kTcThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace dt
