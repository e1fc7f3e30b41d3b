// Tree-masked grouped-query attention: verify every draft node in one pass.
//
// Source: TreeSpark article, introduction (the target model checks all tree
// nodes in one forward); PCTree summary, "setup" (SDPA attention).  Row i of
// request b (0 = root, i = node i-1) attends to the request's KV prefix, the
// root's tree row, and tree row j+1 iff node j is node i-1 or one of its
// ancestors (bit j of anc[b][i-1]).
//
// bf16 inputs: the tensor-core kernel of attn_tc.cu computes split-KV
// partials (128 key columns per split; a CTA's rows are the query heads that
// share one KV head times the tree rows, so every K/V tile read serves all of
// them), and the combine kernel below merges the splits.  fp32 inputs use a
// plain per-(row, head) kernel.
#include "attn_tc.cuh"

namespace dt {

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

// Is tree column j (0 = root, j' + 1 = node j') visible from tree row i?
__device__ __forceinline__ bool tree_visible(int i, int j, uint64_t anc_row) {
  return j == 0 || (i >= 1 && ((anc_row >> (j - 1)) & 1ull));
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
  int splits, cols_per_split, rows_per_cta, n_rblocks, rpad;
  size_t part_o_bytes, part_ml_bytes;
};

// The tensor-core kernel (attn_tc.cu): 128-column splits, one partial row per
// (tree row, query head) of each KV head.
static AttnPlan attn_tc_plan(int batch, int Nmax, int Hq, int Hkv, int d, int max_prefix) {
  AttnPlan p;
  const int G = Hq / Hkv;
  p.n_rblocks = 1;
  p.rows_per_cta = p.rpad = G * (Nmax + 1);
  p.cols_per_split = 128;
  p.splits = (max_prefix + Nmax + 1 + 127) / 128;
  const size_t rows = (size_t)p.splits * batch * Hkv * p.rpad;
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
  const AttnPlan t = attn_tc_plan(batch, Nmax, Hq, Hkv, d, max_prefix);
  return kWsHeader + ((t.part_ml_bytes + 255) & ~(size_t)255) + t.part_o_bytes + 256;
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
  const AttnPlan p = attn_tc_plan(batch, Nmax, Hq, Hkv, d, max_prefix);
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
  a.part_ml = (float2*)(w + kWsHeader);
  a.part_o = (float*)(w + kWsHeader + ((p.part_ml_bytes + 255) & ~(size_t)255));
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
  // launched while the attention kernel runs; it waits for its partials
  if (launch_pdl(attn_combine_kernel, cgrid, dim3(32 * kCombineWarps), 0, s, a) != cudaSuccess)
    return DT_ECUDA;
  return cudaGetLastError() == cudaSuccess ? DT_OK : DT_ECUDA;
}

}  // extern "C"
