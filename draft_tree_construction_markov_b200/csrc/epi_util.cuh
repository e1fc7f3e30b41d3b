// Device helpers of the tensor-core epilogues (markov_gemm.cu, pbuild.cu):
// register top-k lists, bias-row decoding, 2^x, TMEM reads of 32 columns.
#pragma once
#include "build.cuh"

namespace dt {

constexpr int kTileV = 128;
constexpr float kLog2e = 1.4426950408889634f;
// U <= 1 - 2^-24 gives G = -log(-log U) <= 16.64; tokens with s + 16.75 below
// the current k-th Gumbel key cannot enter the sample and skip the Philox draw.
constexpr float kGumbelMax = 16.75f;
constexpr int kTLD = 33;  // transpose buffer row stride (floats)

__device__ __forceinline__ void named_bar(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// 16-byte global -> shared copy that does not block the thread.
__device__ __forceinline__ void cp_async16_g2s(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}

// Insert (v, id) into a register list sorted by value (descending) when ids
// arrive in increasing order: equal values keep their earlier entries first.
// Entries past k are scratch.  Caller guarantees v > list[k-1].
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

// Raw 128 bytes of a bias row (32 fp32 or the first 64 bytes = 32 bf16).
__device__ __forceinline__ void load_bias_raw(const void* L, int bf16, int64_t off,
                                              uint4 (&raw)[8]) {
  const uint4* p =
      bf16 ? (const uint4*)((const uint16_t*)L + off) : (const uint4*)((const float*)L + off);
#pragma unroll
  for (int c = 0; c < 8; ++c)
    if (c < 4 || !bf16) raw[c] = __ldg(p + c);
}

__device__ __forceinline__ void decode_bias(const uint4 (&raw)[8], int bf16, float (&bias)[32]) {
  if (bf16) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint32_t w[4] = {raw[c].x, raw[c].y, raw[c].z, raw[c].w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        bias[8 * c + 2 * h] = __uint_as_float(w[h] << 16);
        bias[8 * c + 2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
      }
    }
  } else {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      bias[4 * c] = __uint_as_float(raw[c].x);
      bias[4 * c + 1] = __uint_as_float(raw[c].y);
      bias[4 * c + 2] = __uint_as_float(raw[c].z);
      bias[4 * c + 3] = __uint_as_float(raw[c].w);
    }
  }
}

// 2^x with the hardware approximation (relative error below 2^-22).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Whether the Gumbel key s + G, G = -log(-log U), U = ((word >> 9) + 0.5) 2^-23,
// can exceed thr, decided without the two accurate logarithms of the key:
// s + G > thr  <=>  w = -log U < exp(s - thr).
//  * w is bounded below by v = 1 - U (exact in fp32) when v < 2^-7, since
//    -log(1 - v) >= v, and otherwise by 0.999 (-__logf(U)): __logf's error
//    (below 2^-21 absolute near 1, 2^-21 relative elsewhere) is far below
//    0.1 % of w >= 2^-7.
//  * exp(s - thr) is bounded above by 2^((s - thr) log2(e) + log2(1.001))
//    with ex2.approx (relative error near 2^-22).
// The two factors leave about 1e-3 of room on G, far more than the fp32
// rounding of the key, so every token whose computed key beats thr passes,
// and the caller computes the exact key for those only.  thr = -inf passes
// every finite s; s = -inf never passes.
__device__ __forceinline__ bool gumbel_may_beat(float s, float thr, uint32_t word) {
  const uint32_t m = word >> 9;
  const float v = ((float)(0x7fffffu - m) + 0.5f) * 1.1920928955078125e-07f;  // 1 - U
  const float wlo =
      v < 0.0078125f ? v : -0.999f * __logf(((float)m + 0.5f) * 1.1920928955078125e-07f);
  return wlo < ex2_approx((s - thr) * kLog2e + 0.0014419741f);
}

__device__ __forceinline__ float load_bias1(const void* L, int bf16, int64_t off) {
  return bf16 ? bf16_to_f32(__ldg((const uint16_t*)L + off)) : __ldg((const float*)L + off);
}

// fp32 -> bf16, round to nearest even (finite inputs).
__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
  const uint32_t u = __float_as_uint(f);
  return (uint16_t)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

// 32 lanes x 32 columns of 32-bit TMEM cells -> 32 registers per thread.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&acc)[32]) {
  float v[16];
  tmem_ld16(taddr, v);
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = v[i];
  tmem_ld16(taddr + 16, v);
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[16 + i] = v[i];
}

}  // namespace dt
