// Data structures shared by the tree-build kernels and their host launcher.
#pragma once
#include "common.cuh"

namespace dt {

// One GEMM column: a node to expand in this wave, or a row to materialise.
struct __align__(32) Row {
  int32_t b;      // request (-1 = padding column)
  int32_t depth;  // depth of the node; its children use block-logit row `depth`
  int32_t token;  // token of the node (selects the Markov-head row A[token])
  int32_t aux;    // expand: node serial (-1 = root); q/z rows: output row
  uint64_t path;  // path id (Philox counter words 1-2)
  float lse;      // q rows: log-sum-exp of the node's scaled logits
  float key;      // expand: the node's key
};

// One candidate node of a request's tree (kept list + new children).
struct __align__(16) Cand {
  float key;
  int32_t token;
  int32_t serial;         // unique id within the request
  int32_t parent_serial;  // -1 = child of the root
  uint64_t path;
  int16_t depth;
  int8_t rank;
  int8_t expanded;        // 1 once scheduled for expansion
  int16_t parent_pos;     // parent's position in the list when created (+1; 0 = root)
  int16_t pad0;
  float lse;              // log-sum-exp of the node's own distribution (if expanded)
  int32_t pad1[3];
};
static_assert(sizeof(Cand) == 48, "Cand layout");

struct ReqState {
  int32_t n_list;
  int32_t serial_next;
  int32_t done;
  int32_t row_base;   // rows of this request in the current wave list
  int32_t row_count;
  float root_lse;
  int32_t root_token;
  float thr;          // fp32(log(lambda)), -inf for lambda = 0
  int32_t kb;         // children per node of this request
  int32_t nb;         // node budget of this request
  int32_t pad[2];
};

enum EpiMode { EPI_EXPAND = 0, EPI_ZDUMP = 1, EPI_QROWS = 2 };

struct GemmArgs {
  const void* L;         // block logits [batch][Bk][V]
  int l_bf16;
  int Bk, V, r, k;
  const Row* rows;       // GEMM columns
  const int32_t* n_rows; // device count of valid columns
  int32_t* reset_count;  // set to 0 by CTA (0,0) (next wave's counter), may be NULL
  int n_vtiles;          // vocab tiles of 128 rows
  int ncta_v;            // CTAs along the vocabulary
  int Mcap;              // capacity of rows
  float temp;
  uint64_t seed;
  uint32_t offset;
  // output rows: expand: s = z / T, [row][V]; zdump: z, [aux][V];
  // qrows: q = exp(s - lse), [b][Nmax+1][V] with row aux
  float* out;
  int nmax1;             // Nmax + 1
  int32_t* status;
  int stages;
};

struct TopkArgs {
  const float* S;        // [Mcap][V] scaled logits of this wave's nodes
  const Row* rows;
  const int32_t* n_rows;
  int Mcap, V, k, nchunk, chunk;
  float temp;
  uint64_t seed;
  uint32_t offset;
  float2* stats;         // [Mcap][nchunk] (max, sum exp(s - max))
  float* lv;             // [Mcap][nchunk][k] top-k of s
  int32_t* li;
  float* gv;             // [Mcap][nchunk][k] Gumbel top-k (T > 0)
  int32_t* gi;
  int32_t* row_done;     // [Mcap] chunks finished per row (the last one merges and resets)
  float* fin_lse;        // [Mcap] merged results per node
  float* fin_v;          // [Mcap][k] top-k values of s (order statistics)
  int32_t* fin_i;        // [Mcap][k] their tokens
  int32_t* fin_g;        // [Mcap][k] Gumbel-top-k tokens (T > 0)
  int32_t* status;
};

struct FrontierArgs {
  const GemmArgs* g;     // unused on device
  const Row* rows;       // this wave's rows
  Row* next_rows;        // next wave's rows
  int32_t* next_count;
  Row* mat_rows;         // rows whose draft distribution is materialised (T > 0)
  int32_t* mat_count;
  uint16_t* H;           // gathered Markov rows of the next wave [Mcap][r]
  uint16_t* Hm;          // gathered Markov rows of mat_rows
  const uint16_t* A;     // [V][r]
  ReqState* req;
  Cand* lists;           // [batch][Nmax]
  const float* fin_lse;  // [Mcap] per expanded node: log-sum-exp of s
  const float* fin_v;    // [Mcap][k] top-k values of s
  const int32_t* fin_i;  // [Mcap][k] their tokens
  const int32_t* fin_g;  // [Mcap][k] Gumbel-top-k tokens (T > 0)
  const float* calib;    // [Bk][2] or NULL
  const int32_t* n_budget;
  const int32_t* k_req;
  const float* lambda;
  int Mcap, Bk, V, r, k, Nmax, batch;
  float temp;
  dt_tree out;
  int32_t* status;
};

}  // namespace dt
