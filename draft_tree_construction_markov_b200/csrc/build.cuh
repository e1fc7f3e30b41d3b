// Data structures shared by the tree-build kernels and their host launcher.
#pragma once
#include "common.cuh"

namespace dt {

// One GEMM column: a node to expand in this wave, or a row to materialise.
struct __align__(32) Row {
  int32_t b;      // request (-1 = padding column)
  int32_t depth;  // depth of the node; its children use block-logit row `depth`
  int32_t token;  // Markov-head row A[token] of the node's children (-1: no Markov term)
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

enum EpiMode { EPI_EXPAND = 0, EPI_ZDUMP = 1, EPI_QROWS = 2, EPI_SWIGLU = 3 };

struct GemmArgs {
  const void* L;         // bias rows [batch][Bk][V] (block logits, residual) or NULL
  int l_bf16;
  int Bk, V, r, k;       // V: weight rows (vocabulary / features), r: inner dimension
  int vfull;             // vocabulary of the block logits and of A (0: V); V < vfull for a shard
  int v_base;            // first token of this launch's vocabulary shard (EXPAND only)
  const Row* rows;       // GEMM columns
  const int32_t* n_rows; // device count of valid columns
  int32_t* reset_count;  // set to 0 by CTA (0,0) (next wave's counter), may be NULL
  int n_vtiles;          // weight tiles (128 rows; SwiGLU: 64 features)
  int ncta_v;            // weight ranges (= partials per node)
  int n_ntiles;          // node tiles for Mcap columns (set by the launcher)
  int n_nslots;          // node-tile slots per weight range (0: one per tile); a CTA
                         // loops over tiles slot, slot + n_nslots, ...
  int bias_span;         // bias cache row length (set by the launcher; 0 = no cache)
  int bias_rows;         // bias cache capacity in rows (set by the launcher)
  const uint16_t* gatherA;  // [V][r]: gather B rows A[token] in the kernel (NULL: TMA from H)
  int Mcap;              // capacity of rows
  float temp;
  uint64_t seed;
  uint32_t offset;
  // expand: one partial per (node row, CTA): statistics at row * ncta_v + cta,
  // list entry i at (row * k + i) * ncta_v + cta
  float2* pstats;        // (max, sum exp(s - max)) of the CTA's vocabulary range
  float* plv;            // top-k values of s, best first (ties: lower token)
  int32_t* pli;          // their tokens
  float* pgv;            // Gumbel-top-k keys (T > 0)
  int32_t* pgi;          // their tokens
  // zdump: z, [aux][ldo] (fp32, or bf16 if out_bf16); qrows: q = exp(s - lse),
  // [b][Nmax+1][ldo] with row aux; swiglu: silu(gate) * up, bf16 [aux][ldo]
  float* out;
  int ldo;               // output row stride in elements (0: V)
  int out_bf16;
  int nmax1;             // Nmax + 1
  int32_t* status;
  int stages;
  int l2_keep;           // weight loads carry an L2 evict-last hint (re-read by later waves)
};

struct FrontierArgs {
  const GemmArgs* g;     // unused on device
  const Row* rows;       // this wave's rows
  Row* next_rows;        // next wave's rows
  int32_t* next_count;
  Row* mat_rows;         // rows whose draft distribution is materialised (T > 0)
  int32_t* mat_count;
  uint16_t* H;           // gathered Markov rows of the next wave [Mcap][r] (NULL: the GEMM gathers)
  uint16_t* Hm;          // gathered Markov rows of mat_rows (NULL: the GEMM gathers)
  const uint16_t* A;     // [V][r]
  const int32_t* cond;   // [batch][Bk] Markov-row token per depth (-1: none); NULL: own token
  ReqState* req;
  Cand* lists;           // [batch][Nmax]
  const float2* pstats;  // per-CTA partials of the wave GEMM (see GemmArgs)
  const float* plv;
  const int32_t* pli;
  const float* pgv;
  const int32_t* pgi;
  int ncta;              // partials per node
  const float* calib;    // [Bk][2] or NULL
  const int32_t* n_budget;
  const int32_t* k_req;
  const float* lambda;
  int Mcap, Bk, V, r, k, Nmax, batch;
  float temp;
  dt_tree out;
  int32_t* status;
};

// One persistent launch for every wave of a small build (pbuild.cu).
struct PBuildArgs {
  const void* L;          // block logits [batch][Bk][V]
  int l_bf16;
  const uint16_t* A;      // Markov rows [V][r] (the MMA's B operand, gathered)
  int Bk, V, r, k, Nmax, batch;
  int n_vtiles;           // 128-row tiles of Bm
  float temp;
  uint64_t seed;
  uint32_t offset;
  const float* calib;     // [Bk][2] or NULL
  const int32_t* root_token;
  const int32_t* n_budget;
  const int32_t* k_req;   // or NULL: k for every request
  const float* lambda;
  const int32_t* cond;    // [batch][Bk] Markov-row token per depth of a baseline variant, or NULL
  // per-CTA partials, two buffers (wave parity); same layout as the wave GEMM's
  float2* pstats[2];
  float* plv[2];
  int32_t* pli[2];
  float* pgv[2];
  int32_t* pgi[2];
  float* mrg_lse;         // merged rows of a wave: log-sum-exp [rows]
  float* mrg_val;         //   the k best values of s [rows][k]
  int32_t* mrg_tok;       //   their tokens (T = 0) or the sampled tokens (T > 0) [rows][k]
  unsigned* grid_bar;     // arrivals so far (zeroed before the launch)
  int32_t* grid_abort;    // set by a CTA that gave up (zeroed before the launch)
  Row* mat_rows;          // T > 0: draft rows of the final trees
  int32_t* mat_count;
  dt_tree out;
  int32_t* status;
  int stages;
  int span;               // bias cache row length (elements; a multiple of 128)
  int cap;                // candidate capacity of one request: Nmax + Nmax * k
  uint64_t wait_ns;       // bound of every device-side wait
  int stall_cta;          // test hook: this CTA never arrives at the first grid barrier (-1: none)
};

}  // namespace dt
