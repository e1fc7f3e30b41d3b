// Arguments of the tensor-core tree attention (attn_tc.cu), shared with the
// C entry point in verify_attn.cu.
#pragma once
#include "common.cuh"

namespace dt {

struct AttnTcArgs {
  const uint16_t* q;      // [batch][Nmax+1][Hq][d]
  const uint16_t* kp;     // [sum prefix][Hkv][d]
  const uint16_t* vp;
  const int64_t* pstart;  // [batch] first prefix row of each request
  const int32_t* plen;    // [batch]
  const uint16_t* kt;     // [batch][Nmax+1][Hkv][d]
  const uint16_t* vt;
  const uint64_t* anc;    // [batch][Nmax]
  const int32_t* n_nodes; // [batch]
  int batch, Nmax, Hq, Hkv, d, G, max_prefix;
  int heads_per_cta, n_groups;  // query heads of a CTA, groups per KV head
  float scale_log2;             // scale * log2(e)
  // partials in the split-combine layout: row rho = i * G + hh of (b, kv head)
  float* part_o;   // [splits][batch][Hkv][rpad][d]
  float2* part_ml; // [splits][batch][Hkv][rpad]: (max in log2 units, sum)
  int splits, rpad;
  int32_t* status;
};

cudaError_t launch_attn_tc(const AttnTcArgs& a, cudaStream_t s);
int attn_tc_heads_per_cta(int G, int Nmax);

}  // namespace dt
