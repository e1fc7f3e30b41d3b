// Per-node distribution statistics and candidate children from the scaled
// logit rows the Markov GEMM wrote: log-sum-exp, top-k of s (ties to the lower
// token id) and, at T > 0, the Gumbel-top-k of s + G, i.e. k siblings sampled
// without replacement (TreeSpark article, "lossless" section; Gumbel-top-k:
// Kool, van Hoof and Welling 2019).
//
// grid (nchunk, rows): a CTA scans one chunk of one node row.  Each warp
// streams 32 consecutive tokens per step and keeps a sorted top-k list spread
// over lanes 0..k-1; a step touches the list only when some lane beats the
// entry threshold, which the CTA's warps share through shared memory.  With
// thousands of tokens per warp the threshold converges after a few dozen
// tokens, so almost every step is one compare and one ballot.
#include "build.cuh"

namespace dt {

constexpr int kTopkThreads = 256;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr float kL2eT = 1.4426950408889634f;
// U <= 1 - 2^-24 gives G = -log(-log U) <= 16.64; tokens with s + 16.75 at or
// below the entry threshold cannot enter the sample and skip the Philox draw.
constexpr float kGumbelMaxT = 16.75f;

__device__ __forceinline__ bool before_t(float v1, int32_t i1, float v2, int32_t i2) {
  return v1 > v2 || (v1 == v2 && i1 < i2);
}

__device__ __forceinline__ float from_ordered(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}

// 2^x with the hardware approximation (relative error below 2^-22).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// The next float below a finite x (entry thresholds sit one step under a k-th
// value so that an equal value with a lower token id still enters).
__device__ __forceinline__ float below(float x) {
  if (x == 0.f) return -1.17549435e-38f;
  const uint32_t b = __float_as_uint(x);
  return __uint_as_float(x > 0.f ? b - 1u : b + 1u);
}

// Merge candidate lanes (bits of `bal`, each offering (v, x)) into the warp's
// sorted list held by lanes 0..k-1 in (lv, li).  Returns the new k-th value.
__device__ __forceinline__ float warp_list_merge(float& lv, int32_t& li, int k, unsigned bal,
                                                 float v, int32_t x, int lane) {
  if (__popc(bal) <= 4) {
    while (bal) {
      const int src = __ffs(bal) - 1;
      bal &= bal - 1;
      const float cv = __shfl_sync(0xffffffffu, v, src);
      const int32_t ci = __shfl_sync(0xffffffffu, x, src);
      const bool bef = lane < k && before_t(lv, li, cv, ci);
      const int pos = __popc(__ballot_sync(0xffffffffu, bef));
      const float uv = __shfl_up_sync(0xffffffffu, lv, 1);
      const int32_t ui = __shfl_up_sync(0xffffffffu, li, 1);
      if (pos < k) {
        if (lane == pos) {
          lv = cv;
          li = ci;
        } else if (lane > pos && lane < k) {
          lv = uv;
          li = ui;
        }
      }
    }
  } else {
    // k rounds of a warp-wide argmax over {own list entry, own candidate}
    const bool cand = (bal >> lane) & 1;
    float a_v = cand ? v : -INFINITY;
    int32_t a_i = cand ? x : 0x7fffffff;
    float b_v = lv;
    int32_t b_i = li;
    float o_v = -INFINITY;
    int32_t o_i = 0x7fffffff;
    for (int r = 0; r < k; ++r) {
      const bool use_b = before_t(b_v, b_i, a_v, a_i);
      const float bv = use_b ? b_v : a_v;
      const int32_t bi = use_b ? b_i : a_i;
      float wv = bv;
      int32_t wi = bi;
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, wv, o);
        const int32_t oi = __shfl_xor_sync(0xffffffffu, wi, o);
        if (before_t(ov, oi, wv, wi)) {
          wv = ov;
          wi = oi;
        }
      }
      if (bv == wv && bi == wi) {
        if (use_b) {
          b_v = -INFINITY;
          b_i = 0x7fffffff;
        } else {
          a_v = -INFINITY;
          a_i = 0x7fffffff;
        }
      }
      if (lane == r) {
        o_v = wv;
        o_i = wi;
      }
    }
    lv = o_v;
    li = o_i;
  }
  return __shfl_sync(0xffffffffu, lv, k - 1);
}

template <bool STOCH>
__global__ void __launch_bounds__(kTopkThreads) topk_rows_kernel(TopkArgs a) {
  __shared__ uint32_t s_thr, s_gthr;   // best known k-th value of the CTA (ordered bits)
  __shared__ float2 s_st[kTopkWarps];
  __shared__ float s_lv[kTopkWarps][16], s_gv[kTopkWarps][16];
  __shared__ int32_t s_li[kTopkWarps][16], s_gi[kTopkWarps][16];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int row = blockIdx.y;
  pdl_wait();  // the rows come from the GEMM launched just before
  pdl_launch_dependents();
  const int M = min(*a.n_rows, a.Mcap);
  if (row >= M) return;
  const Row rw = a.rows[row];
  if (rw.b < 0) return;
  const int k = a.k;
  if (threadIdx.x == 0) {
    s_thr = f32_ordered(-INFINITY);
    s_gthr = f32_ordered(-INFINITY);
  }
  __syncthreads();
  const int x0 = blockIdx.x * a.chunk;
  const int x1 = min(a.V, x0 + a.chunk);
  const float* src = a.S + (size_t)row * a.V;
  float m = -INFINITY, ssum = 0.f;
  float lv = -INFINITY, gv = -INFINITY;
  int32_t li = 0x7fffffff, gi = 0x7fffffff;
  float thr = -INFINITY, gthr = -INFINITY;
  const uint32_t c1 = (uint32_t)rw.path, c2 = (uint32_t)(rw.path >> 32);
  constexpr int U = 8;  // steps whose loads are issued together
  for (int base = x0 + warp * 32; base < x1; base += kTopkThreads * U) {
    float vals[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int x = base + u * kTopkThreads + lane;
      vals[u] = x < x1 ? __ldg(src + x) : -INFINITY;
    }
    // entry thresholds: own k-th value, or just below the CTA's best k-th
    float te = thr, gte = gthr;
    {
      const float sh = from_ordered(s_thr);
      if (sh > te) te = below(sh);
      if (STOCH) {
        const float gsh = from_ordered(s_gthr);
        if (gsh > gte) gte = below(gsh);
      }
    }
    // softmax statistics of the group: one rescale, one 2^x per value
    {
      float gm = vals[0];
#pragma unroll
      for (int u = 1; u < U; ++u) gm = fmaxf(gm, vals[u]);
      const float mn = fmaxf(m, gm);
      if (mn != -INFINITY) {
        float acc = ssum * ex2((m - mn) * kL2eT);
#pragma unroll
        for (int u = 0; u < U; ++u) acc += ex2((vals[u] - mn) * kL2eT);
        ssum = acc;
        m = mn;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int x = base + u * kTopkThreads + lane;
      const bool in = x < x1;
      const float s = vals[u];
      const unsigned bal = __ballot_sync(0xffffffffu, in && s > te);
      if (bal) {
        thr = warp_list_merge(lv, li, k, bal, s, x, lane);
        te = fmaxf(te, thr);
        if (lane == 0 && thr != -INFINITY) atomicMax(&s_thr, f32_ordered(thr));
      }
      if constexpr (STOCH) {
        float gk = -INFINITY;
        if (in && s + kGumbelMaxT > gte) {
          const float uu = philox_uniform(a.seed, a.offset, 0u, (uint32_t)rw.b, c1, c2, (uint32_t)x);
          gk = s + (-logf(-logf(uu)));
        }
        const unsigned gbal = __ballot_sync(0xffffffffu, gk > gte);
        if (gbal) {
          gthr = warp_list_merge(gv, gi, k, gbal, gk, x, lane);
          gte = fmaxf(gte, gthr);
          if (lane == 0 && gthr != -INFINITY) atomicMax(&s_gthr, f32_ordered(gthr));
        }
      }
    }
  }
  // CTA reduction: statistics and an 8-way merge of the warps' sorted lists
  const float wm = warp_max(m);
  float ws = (m == -INFINITY) ? 0.f : ssum * exp2f((m - wm) * kL2eT);
  ws = warp_sum(ws);
  if (lane == 0) s_st[warp] = make_float2(wm, ws);
  if (lane < k) {
    s_lv[warp][lane] = lv;
    s_li[warp][lane] = li;
    s_gv[warp][lane] = gv;
    s_gi[warp][lane] = gi;
  }
  __syncthreads();
  const size_t pidx = (size_t)row * a.nchunk + blockIdx.x;
  if (threadIdx.x == 0) {
    float mx = -INFINITY;
    for (int w = 0; w < kTopkWarps; ++w) mx = fmaxf(mx, s_st[w].x);
    float sv = 0.f;
    if (mx != -INFINITY)
      for (int w = 0; w < kTopkWarps; ++w)
        if (s_st[w].x != -INFINITY) sv += s_st[w].y * exp2f((s_st[w].x - mx) * kL2eT);
    a.stats[pidx] = make_float2(mx, sv);
  }
  if (threadIdx.x < (STOCH ? 64 : 32)) {
    const bool g = threadIdx.x >= 32;
    if (lane == 0) {
      int hp[kTopkWarps];
      for (int w = 0; w < kTopkWarps; ++w) hp[w] = 0;
      float* OV = (g ? a.gv : a.lv) + pidx * k;
      int32_t* OI = (g ? a.gi : a.li) + pidx * k;
      for (int i = 0; i < k; ++i) {
        int bw = -1;
        float bv = -INFINITY;
        int32_t bi = 0x7fffffff;
        for (int w = 0; w < kTopkWarps; ++w) {
          if (hp[w] >= k) continue;
          const float v = g ? s_gv[w][hp[w]] : s_lv[w][hp[w]];
          const int32_t id = g ? s_gi[w][hp[w]] : s_li[w][hp[w]];
          if (bw < 0 || before_t(v, id, bv, bi)) {
            bw = w;
            bv = v;
            bi = id;
          }
        }
        if (bw >= 0) hp[bw]++;
        OV[i] = bv;
        OI[i] = bi;
      }
    }
  }
  // the last CTA of this row merges all chunks (partials are visible after
  // the fence + counter), writes the node's final result and resets the counter
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int prev = atomicAdd(&a.row_done[row], 1);
    s_last = prev == a.nchunk - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int nc = a.nchunk;
  if (warp == 0) {
    float mx = -INFINITY;
    for (int c = lane; c < nc; c += 32) mx = fmaxf(mx, __ldcg(&a.stats[(size_t)row * nc + c].x));
    mx = warp_max(mx);
    float sv = 0.f;
    for (int c = lane; c < nc; c += 32) {
      const float2 p = __ldcg(&a.stats[(size_t)row * nc + c]);
      if (p.x != -INFINITY) sv += p.y * exp2f((p.x - mx) * kL2eT);
    }
    sv = warp_sum(sv);
    if (lane == 0) {
      a.fin_lse[row] = mx + logf(sv);
      a.row_done[row] = 0;
    }
  }
  if (warp == 1 || (STOCH && warp == 2)) {
    // k rounds of a warp argmax over the chunk lists' heads (one list per lane)
    const bool g = warp == 2;
    const float* LV = g ? a.gv : a.lv;
    const int32_t* LI = g ? a.gi : a.li;
    int head = 0;
    for (int i = 0; i < k; ++i) {
      float bv = -INFINITY;
      int32_t bi = 0x7fffffff;
      int owner = -1;
      if (lane < nc && head < k) {
        const size_t base = ((size_t)row * nc + lane) * k;
        bv = __ldcg(LV + base + head);
        bi = __ldcg(LI + base + head);
        owner = lane;
      }
      float wv = bv;
      int32_t wi = bi;
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, wv, o);
        const int32_t oi = __shfl_xor_sync(0xffffffffu, wi, o);
        if (before_t(ov, oi, wv, wi)) {
          wv = ov;
          wi = oi;
        }
      }
      if (owner >= 0 && bv == wv && bi == wi) ++head;
      if (lane == 0) {
        if (g) {
          a.fin_g[(size_t)row * k + i] = wi;
        } else {
          a.fin_v[(size_t)row * k + i] = wv;
          a.fin_i[(size_t)row * k + i] = wi;
        }
      }
    }
  }
}

int topk_chunks(int Mcap, int V) {
  int nc = (2 * 148 + Mcap - 1) / Mcap;
  const int most = (V + 2047) / 2048;
  return std::max(1, std::min(nc, std::min(most, 32)));  // one list per lane in the final merge
}

cudaError_t launch_topk_rows(const TopkArgs& a, bool stoch, cudaStream_t s) {
  const dim3 grid(a.nchunk, a.Mcap);
  if (stoch) return launch_pdl(topk_rows_kernel<true>, grid, dim3(kTopkThreads), 0, s, a);
  return launch_pdl(topk_rows_kernel<false>, grid, dim3(kTopkThreads), 0, s, a);
}

}  // namespace dt
