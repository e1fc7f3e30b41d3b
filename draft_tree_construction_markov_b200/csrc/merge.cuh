// Warp-level merges of the per-CTA partial results that the node-batched GEMM
// writes for every node row: (max, sum exp) pairs into a log-sum-exp, and
// sorted top-k lists into the row's best entries (ties to the lower token).
#pragma once
#include "build.cuh"

namespace dt {

// (v1, i1) ranks before (v2, i2): larger value first, then lower token.
__device__ __forceinline__ bool ranks_first(float v1, int32_t i1, float v2, int32_t i2) {
  return v1 > v2 || (v1 == v2 && i1 < i2);
}

// Insert (v, id) into a register list sorted by ranks_first; the caller
// guarantees that it ranks before the k-th entry.  Entries past k are scratch.
template <int KMAX>
__device__ __forceinline__ void list_insert(float (&L)[KMAX], int32_t (&I)[KMAX], float v,
                                            int32_t id) {
  float nl[KMAX];
  int32_t ni[KMAX];
#pragma unroll
  for (int i = 0; i < KMAX; ++i) {
    const bool keep = ranks_first(L[i], I[i], v, id);
    const bool keep_prev = i > 0 && ranks_first(L[i - 1], I[i - 1], v, id);
    nl[i] = keep ? L[i] : ((i == 0 || keep_prev) ? v : L[i - 1]);
    ni[i] = keep ? I[i] : ((i == 0 || keep_prev) ? id : I[i - 1]);
  }
#pragma unroll
  for (int i = 0; i < KMAX; ++i) {
    L[i] = nl[i];
    I[i] = ni[i];
  }
}

template <int KMAX>
__device__ __forceinline__ void list_entry(const float (&L)[KMAX], const int32_t (&I)[KMAX], int j,
                                           float& v, int32_t& id) {
  v = L[0];
  id = I[0];
#pragma unroll
  for (int i = 1; i < KMAX; ++i)
    if (i == j) {
      v = L[i];
      id = I[i];
    }
}

// One warp merges one of the lists of a node's ncta partials (each sorted,
// k long) into its first kb entries: every lane folds its partials into a
// private list, then kb rounds of a warp-wide arg-best pick the winners.
// A lane issues the loads of up to JP partials before it looks at any of
// them, so their latencies overlap.  out_v / out_i may be NULL when the
// values / tokens are not needed.
template <int KMAX>
__device__ __forceinline__ void merge_lists(const float* PV, const int32_t* PI, int ncta, int k,
                                            int kb, int lane, float* out_v, int32_t* out_i) {
  constexpr int JP = KMAX <= 4 ? 5 : 1;
  float L[KMAX];
  int32_t I[KMAX];
#pragma unroll
  for (int i = 0; i < KMAX; ++i) {
    L[i] = -INFINITY;
    I[i] = 0x7fffffff;
  }
  for (int c0 = 0; c0 < ncta; c0 += 32 * JP) {
    float pv[JP][KMAX];
    int32_t pi[JP][KMAX];
#pragma unroll
    for (int j = 0; j < JP; ++j) {
      const int c = c0 + 32 * j + lane;
#pragma unroll
      for (int i = 0; i < KMAX; ++i) {
        const bool in = c < ncta && i < k;
        pv[j][i] = in ? __ldcg(PV + (size_t)c * k + i) : -INFINITY;
        pi[j][i] = in ? __ldcg(PI + (size_t)c * k + i) : 0x7fffffff;
      }
    }
    // entry bar: the best kb-th entry of any partial.  Its partial alone holds
    // kb entries at or above it, so nothing below it can be among the kb best.
    float bv = -INFINITY;
    int32_t bi = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < JP; ++j) {
      float v;
      int32_t id;
      list_entry<KMAX>(pv[j], pi[j], kb - 1, v, id);
      if (ranks_first(v, id, bv, bi)) {
        bv = v;
        bi = id;
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int32_t oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ranks_first(ov, oi, bv, bi)) {
        bv = ov;
        bi = oi;
      }
    }
#pragma unroll
    for (int j = 0; j < JP; ++j) {
#pragma unroll
      for (int i = 0; i < KMAX; ++i) {
        if (ranks_first(bv, bi, pv[j][i], pi[j][i])) break;  // lists are sorted
        float kv;
        int32_t ki;
        list_entry<KMAX>(L, I, kb - 1, kv, ki);
        if (ranks_first(pv[j][i], pi[j][i], kv, ki)) list_insert<KMAX>(L, I, pv[j][i], pi[j][i]);
      }
    }
  }
  for (int j = 0; j < kb; ++j) {
    float wv = L[0];
    int32_t wi = I[0];
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, wv, o);
      const int32_t oi = __shfl_xor_sync(0xffffffffu, wi, o);
      if (ranks_first(ov, oi, wv, wi)) {
        wv = ov;
        wi = oi;
      }
    }
    if (L[0] == wv && I[0] == wi) {  // (value, token) pairs are unique: one owner
#pragma unroll
      for (int i = 0; i + 1 < KMAX; ++i) {
        L[i] = L[i + 1];
        I[i] = I[i + 1];
      }
      L[KMAX - 1] = -INFINITY;
      I[KMAX - 1] = 0x7fffffff;
    }
    if (lane == 0) {
      if (out_v) out_v[j] = wv;
      if (out_i) out_i[j] = wi;
    }
  }
}

// One warp merges the (max, sum exp) partials of a node into its log-sum-exp.
__device__ __forceinline__ float merge_lse(const float2* P, int ncta, int lane) {
  constexpr float kL2e = 1.4426950408889634f;
  float m = -INFINITY, sv = 0.f;
  for (int c0 = 0; c0 < ncta; c0 += 32 * 5) {
    float2 ps[5];
#pragma unroll
    for (int j = 0; j < 5; ++j) {
      const int c = c0 + 32 * j + lane;
      ps[j] = c < ncta ? __ldcg(P + c) : make_float2(-INFINITY, 0.f);
    }
#pragma unroll
    for (int j = 0; j < 5; ++j) {
      if (ps[j].x == -INFINITY) continue;
      if (ps[j].x > m) {
        sv = sv * exp2f((m - ps[j].x) * kL2e) + ps[j].y;
        m = ps[j].x;
      } else {
        sv += ps[j].y * exp2f((ps[j].x - m) * kL2e);
      }
    }
  }
  const float wm = warp_max(m);
  float ws = (m == -INFINITY) ? 0.f : sv * exp2f((m - wm) * kL2e);
  ws = warp_sum(ws);
  return wm + logf(ws);
}

}  // namespace dt
