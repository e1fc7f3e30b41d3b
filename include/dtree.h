/*
 * dtree.h -- C ABI of the B200 (sm_100a) draft-tree round library (libdtree.so).
 *
 * One decode round of parent-conditioned draft-tree speculative decoding:
 *   dt_tree_build       expand a budget-N draft tree best-first from one block
 *                       of drafter logits and a low-rank Markov head
 *   dt_tree_build_ex    the same, or one of the baseline trees it is compared
 *                       with (chain, marginal-ranked, Shared-Markov)
 *   dt_tree_load_budget cut a batch of trees to a round's verification
 *                       capacity by survival (load-adaptive tree size)
 *   dt_calib_log/_fit   log verified rounds and fit the calibration
 *   dt_sharded_build_*  the build with the Markov factor split by vocabulary
 *                       over several GPUs (partials all-gathered per wave)
 *   dt_tree_verify_attn tree-masked grouped-query attention over prefix + tree
 *   dt_tree_accept      lossless acceptance walk (greedy or recursive residual)
 *
 * Conventions shared by every entry point
 *   - Pointers named d_* are DEVICE pointers; the caller owns every buffer.
 *     The library allocates nothing; scratch space is passed as `ws`.
 *   - All work is enqueued asynchronously on `stream` (a cudaStream_t; NULL =
 *     legacy default stream).  Arguments are validated on the host before
 *     anything is enqueued: a call that returns DT_EINVAL / DT_EUNSUPPORTED /
 *     DT_EWORKSPACE has enqueued nothing.
 *   - DT_ECUDA reports a failed launch (cudaGetLastError after enqueueing).
 *   - Device-side waits are bounded.  A wait that runs out, or an index that a
 *     device-side check finds out of range, writes a non-zero code into the
 *     status word inside `ws`; dt_read_status() returns it.  No kernel traps.
 *   - Calls are stateless and re-entrant; two calls that share a `ws` must not
 *     overlap on the device.
 *   - bf16 tensors are passed as uint16_t bit patterns (IEEE bfloat16).
 *
 * Random numbers: Philox4x32-10 (Salmon et al., SC'11), key = (seed lo32,
 * seed hi32), counter word 3 = philox_offset (must be < 2^32), counter word 0
 * = (x >> 2) | (request << 18) | (purpose << 28), output word x & 3,
 * uniform U = ((w >> 9) + 0.5) * 2^-23 (exact in fp32).  Purposes: 0 = sibling sampling at an
 * expanded node (words 1,2 = 64-bit path id: 4 bits per sibling rank per
 * level, depth in bits 60..63), 1 = acceptance coin of candidate node i
 * (word 1 = i, x = 0), 2 = bonus race at stop node s (word 1 = s + 1, root 0).
 */
#ifndef DTREE_H
#define DTREE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DT_OK = 0,
  DT_EINVAL = 1,        /* bad pointer / shape / value                       */
  DT_EUNSUPPORTED = 2,  /* outside the supported limits listed below          */
  DT_ECUDA = 3,         /* a CUDA call or launch failed                       */
  DT_ETIMEOUT = 4,      /* a bounded device-side wait ran out                 */
  DT_EWORKSPACE = 5,    /* ws is NULL or smaller than the query says          */
  DT_EDEVICE = 6        /* a device-side range check failed                   */
} dt_status;

typedef enum { DT_F32 = 0, DT_BF16 = 1 } dt_dtype;

typedef void* dt_stream; /* cudaStream_t */

/* Limits: Nmax <= 64 (ancestor bitmask), 1 <= k <= 16, 1 <= Bk <= 16,
 * batch <= 1024, V < 2^20, r a multiple of 16 in [16, 1024],
 * head_dim in {64, 128}, Hq a multiple of Hkv. */

/* Draft tree of a batch of requests; every array is caller-owned device memory.
 * Node i of request b is element [b * Nmax + i]; nodes are in best-first pop
 * order, which is topological (a parent precedes its children). */
typedef struct {
  int32_t* d_tokens;   /* [batch][Nmax] token of node i                      */
  int32_t* d_parents;  /* [batch][Nmax] parent node index, -1 = the root     */
  int32_t* d_depths;   /* [batch][Nmax] 1..Bk (the root has depth 0)         */
  int32_t* d_ranks;    /* [batch][Nmax] 0-based sibling rank (sampling order)*/
  float* d_keys;       /* [batch][Nmax] cumulative calibrated log-survival   */
  uint64_t* d_anc;     /* [batch][Nmax] bit j set iff node j is node i or one
                          of its ancestors                                   */
  int32_t* d_n_nodes;  /* [batch] number of nodes of each request's tree     */
  float* d_draft_q;    /* [batch][Nmax+1][V] fp32 draft distribution, row 0 =
                          root, row i+1 = node i; written only when temp > 0
                          and only for the root and nodes of depth < Bk of
                          non-empty trees; may be NULL when temp == 0        */
} dt_tree;

/* ---------------------------------------------------------------- build --
 * Expands each request's tree best-first by calibrated path survival
 * (PCTree summary, "k=4, N=32" paragraph: shared block logits, budget N,
 * k children per node, k = 1 gives the greedy chain; TreeSpark article,
 * "core idea": parent-conditioned distribution from the Markov head,
 * calibrated into an edge-acceptance estimate, path survival drives
 * best-first expansion and per-round stopping; "lossless" section: siblings
 * sampled without replacement).
 *
 * Node u of depth d < Bk with token t has children drawn from
 *   z_u[x] = L[b][d][x] + sum_rho A[t][rho] * Bm[x][rho]      (fp32 accumulate)
 *   s = z / T (T > 0) or z (T == 0),  lse = log sum_x exp(s_x)
 * T == 0: children = top-k of z, ties to the lower token id.
 * T >  0: children = Gumbel-top-k of s + G (G = -log(-log U), Philox purpose 0),
 *         i.e. k tokens sampled without replacement, rank = sampling order.
 * Child of rank j gets key = key(u) + min(0, alpha_{d+1} (s_(j) - lse) + beta_{d+1})
 * with s_(j) the j-th largest s (order statistic); key(root) = 0.
 * Nodes are taken in the order (key desc, depth asc, parent index asc, rank
 * asc) while count < n_budget[b] and key >= fp32(log(lambda[b])).
 *
 *   d_block_logits [batch][Bk][V]  fp32 or bf16 (ldt)
 *   d_markov_a     [V][r] bf16     row t = A[t]
 *   d_markov_b     [V][r] bf16     row x = column x of B (i.e. B transposed)
 *   d_calib        [Bk][2] fp32 (alpha, beta) for child depth 1..Bk; NULL =
 *                  identity (1, 0); every alpha must be >= 0
 *   d_root_token, d_n_budget (each <= Nmax, >= 0), d_k_req (each in [1, k];
 *                  NULL = k for all), d_lambda (>= 0): [batch]
 * Returns DT_OK after enqueueing.  Device-side range failures set DT_EDEVICE
 * in the status word. */
size_t dt_tree_build_workspace_bytes(int batch, int Bk, int V, int r, int k,
                                     int Nmax);

dt_status dt_tree_build(const void* d_block_logits, dt_dtype ldt,
                        const uint16_t* d_markov_a, const uint16_t* d_markov_b,
                        int r, const float* d_calib,
                        const int32_t* d_root_token, const int32_t* d_n_budget,
                        const int32_t* d_k_req, const float* d_lambda,
                        int batch, int Bk, int V, int k, int Nmax, float temp,
                        uint64_t philox_seed, uint64_t philox_offset,
                        const dt_tree* out, void* ws, size_t ws_bytes,
                        dt_stream stream);

/* ----------------------------------------------------- baseline variants --
 * The trees that the PCTree summary's mechanism isolation compares with the
 * parent-conditioned tree (Shared-Markov paragraph; mechanism-isolation
 * paragraph and results table: acceptance length chain < Shared-Markov <
 * PCTree on the same drafter weights).  Every variant runs the same kernels
 * as dt_tree_build and differs only in which token's Markov row conditions
 * the children of a depth-d node:
 *   DT_TREE_PCTREE         the node's own token (exactly dt_tree_build)
 *   DT_TREE_CHAIN          the node's own token with k = 1 for every request
 *                          (d_k_req ignored): the drafter's chain
 *   DT_TREE_MARGINAL       none: z_u = L[b][d] (block logits alone)
 *   DT_TREE_SHARED_MARKOV  c_d: the greedy (T = 0, k = 1, lambda = 0) chain of
 *                          min(Bk, n_budget[b]) nodes is built first, c_0 =
 *                          the root and c_d its depth-d token; every node of
 *                          depth d then draws its children from
 *                          L[b][d] + A[c_d] . Bm, at the call's temperature.
 * The chain walk of DT_TREE_SHARED_MARKOV writes the caller's tree arrays
 * before the tree overwrites them.  Arguments, limits, workspace size
 * (dt_tree_build_workspace_bytes) and errors are those of dt_tree_build;
 * an unknown variant returns DT_EINVAL. */
typedef enum {
  DT_TREE_PCTREE = 0,
  DT_TREE_CHAIN = 1,
  DT_TREE_MARGINAL = 2,
  DT_TREE_SHARED_MARKOV = 3
} dt_tree_variant;

dt_status dt_tree_build_ex(const void* d_block_logits, dt_dtype ldt,
                           const uint16_t* d_markov_a, const uint16_t* d_markov_b,
                           int r, const float* d_calib,
                           const int32_t* d_root_token, const int32_t* d_n_budget,
                           const int32_t* d_k_req, const float* d_lambda,
                           int batch, int Bk, int V, int k, int Nmax, float temp,
                           uint64_t philox_seed, uint64_t philox_offset,
                           dt_tree_variant variant, const dt_tree* out, void* ws,
                           size_t ws_bytes, dt_stream stream);

/* Diagnostic: z rows for given (request, depth, token) triples, fp32
 * [n_rows][V] (d_z), through the same tensor-core GEMM the build uses. */
dt_status dt_markov_logits(const void* d_block_logits, dt_dtype ldt,
                           const uint16_t* d_markov_a,
                           const uint16_t* d_markov_b, int r, int batch,
                           int Bk, int V, const int32_t* d_req,
                           const int32_t* d_depth, const int32_t* d_token,
                           int n_rows, float* d_z, void* ws, size_t ws_bytes,
                           dt_stream stream);
size_t dt_markov_logits_workspace_bytes(int n_rows, int V, int r);

/* ------------------------------------------------------------- TreeFlash --
 * One TreeFlash draft-tree build (TreeFlash explainer, method sections 1-2)
 * for `batch` requests, greedy (T = 0):
 *   stage 1: S_i = the M best tokens of W_lm h_i, i = 1..gamma (ties to the
 *            lower id): M unique tokens per depth;
 *   stage 2: for depth 1 with the root as previous token, and for depth
 *            i >= 2 with every t in S_{i-1}: 1 + (gamma-1) M evaluations of
 *            h' = h_i + W_down(silu(W_gate x) * (W_up x)),
 *            x = [rmsnorm(h_i) w_h :: rmsnorm(E[t]) w_e] (eps 1e-6),
 *            q' = softmax(W_lm h');
 *   select:  the best-first top-`budget` nodes by cumulative log q' (the
 *            explainer names OPT-Tree; this reading takes the nodes of
 *            highest path probability) under the order key desc, depth asc,
 *            parent index asc, rank asc.  A node's candidates are the M best
 *            tokens of its distribution; a node whose token is outside
 *            S_depth was not evaluated and is a leaf.
 * x, silu(g) * u and h' are rounded to bf16 where they feed the next GEMM.
 * Inputs (device, bf16 unless noted): d_h [batch][gamma][D] drafter hidden
 * states of the block; d_embed [V][D]; d_w_norm_h, d_w_norm_e [D] fp32;
 * d_w_gate, d_w_up [Dff][2D]; d_w_down [D][Dff]; d_w_lm [V][D];
 * d_root [batch] int32 (last committed token).  Base pointers 16-byte
 * aligned.  Outputs: the dt_tree arrays with Nmax = budget (d_draft_q
 * unused).  Limits: D and Dff multiples of 64, M <= 16, budget <= 64,
 * gamma <= 64, batch <= 1024, V < 2^24. */
size_t dt_treeflash_workspace_bytes(int batch, int gamma, int D, int Dff, int V, int M,
                                    int budget);
dt_status dt_treeflash_build(const uint16_t* d_h, const uint16_t* d_embed,
                             const float* d_w_norm_h, const float* d_w_norm_e,
                             const uint16_t* d_w_gate, const uint16_t* d_w_up,
                             const uint16_t* d_w_down, const uint16_t* d_w_lm,
                             const int32_t* d_root, int batch, int gamma, int D, int Dff,
                             int V, int M, int budget, const dt_tree* out, void* ws,
                             size_t ws_bytes, dt_stream stream);

/* ---------------------------------------------------------- verify attn --
 * out[b][i][h] = sum_j softmax_j(scale * q[b][i][h] . k_j + mask) v_j over
 * the columns request b's row i may see (TreeSpark article, introduction:
 * every tree node verified in one target forward): the prefix rows
 * [0, prefix_len[b]) of request b, the root's tree row 0, and tree row j+1 iff
 * bit j of anc[b][i-1] is set (rows i >= 1).  Row 0 is the root; rows
 * > n_nodes[b] are left untouched.  GQA: head h uses KV head h / (Hq/Hkv).
 *   d_q, d_out     [batch][Nmax+1][Hq][d]
 *   d_k_prefix, d_v_prefix  [total_prefix_rows][Hkv][d], request b's rows
 *                  start at row d_prefix_start[b] (int64)
 *   d_k_tree, d_v_tree      [batch][Nmax+1][Hkv][d]
 *   d_anc [batch][Nmax] (from dt_tree), d_n_nodes [batch]
 * dt selects fp32 or bf16 for q/k/v/out alike; accumulation is fp32. */
size_t dt_tree_verify_attn_workspace_bytes(int batch, int Nmax, int Hq, int Hkv,
                                           int d, int max_prefix);

dt_status dt_tree_verify_attn(const void* d_q, const void* d_k_prefix,
                              const void* d_v_prefix,
                              const int64_t* d_prefix_start,
                              const int32_t* d_prefix_len, int max_prefix,
                              const void* d_k_tree, const void* d_v_tree,
                              const uint64_t* d_anc, const int32_t* d_n_nodes,
                              int batch, int Nmax, int Hq, int Hkv, int d,
                              float scale, dt_dtype dt, void* d_out, void* ws,
                              size_t ws_bytes, dt_stream stream);

/* --------------------------------------------------------------- accept --
 * Lossless acceptance walk from the root (TreeSpark article, introduction and
 * "lossless" section; PCTree summary, "setup": greedy verification).
 * T == 0: move to the child whose token is argmax of the target row (ties to
 *   the lower id); the bonus token is that argmax where the walk stops.
 * T >  0: at node u, p = softmax(t_u / T), q = draft row of u; children in rank
 *   order: accept x iff U < p(x)/q(x) (Philox purpose 1); on rejection
 *   p <- max(p - q, 0) normalised (unchanged if it sums to 0) and q <- q with x
 *   removed, renormalised.  With no child accepted, or at a leaf, the bonus is
 *   argmax_x p(x) / E_x, E_x = -log U'_x (Philox purpose 2).
 *   d_target_logits [batch][Nmax+1][V] fp32 or bf16, row 0 = root, row i+1 =
 *   node i; tree = the dt_tree of dt_tree_build, or any tree in its layout
 *   (d_draft_q needed iff T > 0).  A node may have any number of children
 *   (up to Nmax - 1), taken in rank order with equal ranks in node order.
 *   At T > 0 a token outside [0, V) records DT_EDEVICE in the status word and
 *   reads as token 0; a node whose parent is outside [-1, n) is never
 *   reached.
 * Outputs (device): d_acc_nodes [batch][Bk] accepted node indices by depth
 * (-1 padded), d_n_acc [batch], d_bonus [batch].
 * At T > 0 each request's walk runs on one thread-block cluster of up to 8
 * CTAs of 1024 threads (fewer when the batch would not fit the SMs at once);
 * a launch that cannot place its clusters returns DT_ECUDA. */
size_t dt_tree_accept_workspace_bytes(int batch, int Nmax, int V);

dt_status dt_tree_accept(const void* d_target_logits, dt_dtype tdt,
                         const dt_tree* tree, int batch, int Bk, int V,
                         int Nmax, float temp, uint64_t philox_seed,
                         uint64_t philox_offset, int32_t* d_acc_nodes,
                         int32_t* d_n_acc, int32_t* d_bonus, void* ws,
                         size_t ws_bytes, dt_stream stream);

/* dt_tree_accept for callers that cannot allocate device memory.  The pages
 * have no counterpart of this entry point; it is a deployment convenience.
 * Some callers cannot hand the library a workspace: a plugin running inside a
 * host framework whose caching allocator owns the device's memory and offers
 * it no allocation hook, or a latency-critical serving loop that must never
 * call cudaMalloc (it may synchronise the device and its latency is
 * unbounded).  This variant takes the same arguments as dt_tree_accept
 * without `ws`/`ws_bytes`; its scratch is a fixed 2 MiB array in the library's
 * device memory, which every GPU that loads the library holds until the
 * process exits.  It allocates nothing and frees nothing.
 *   - Supported sizes: dt_tree_accept_workspace_bytes(batch, Nmax, V) <= 2 MiB
 *     (e.g. batch 1 at V = 151936); larger sizes return DT_EUNSUPPORTED with
 *     nothing enqueued.
 *   - The first call on a device looks up the array's device address (once
 *     per device, with that device current); make that first call before any
 *     stream capture.
 *   - All calls on a device share the array and it keeps the last call's
 *     temporaries; calls that overlap on the GPU race, so serialise them
 *     (e.g. one stream).  Outputs are written to the caller's buffers only.
 *   - Device-side range failures of this variant are not reported through a
 *     readable status word.
 *   - The looked-up address is cached for the life of the process.  After
 *     cudaDeviceReset (or anything else that destroys and recreates the
 *     device's primary context) the library's device memory is loaded anew
 *     and the cached address is stale: do not call this entry point on a
 *     device after resetting it. */
dt_status dt_tree_accept_noalloc(const void* d_target_logits, dt_dtype tdt,
                                 const dt_tree* tree, int batch, int Bk, int V,
                                 int Nmax, float temp, uint64_t philox_seed,
                                 uint64_t philox_offset, int32_t* d_acc_nodes,
                                 int32_t* d_n_acc, int32_t* d_bonus,
                                 dt_stream stream);

/* ---------------------------------------------- vocabulary-sharded build --
 * dt_tree_build (T = 0) with the Markov factor Bm split by vocabulary over
 * `world` ranks (one process per GPU), for a Bm too large for one GPU or to
 * spread one request's weight stream over several GPUs.  Rank w holds the
 * rows [v_base, v_base + v_len) of Bm given by dt_shard_range (whole
 * 128-token tiles, split as evenly as tiles allow); every rank holds the
 * block logits, A and the request arrays, and builds the same tree.  Per
 * wave w = 0 .. Bk-1 the caller runs, on every rank:
 *   dt_sharded_build_gemm      this rank's expansion GEMM over its shard:
 *                              per node row, `ncta` partial (max, sum exp)
 *                              statistics and top-k lists, into d_partials
 *                              (dt_sharded_partials_bytes, 256-byte aligned);
 *   an all-gather of the partial blocks in rank order (e.g. NCCL), giving
 *                              [world][block] at d_gathered;
 *   dt_sharded_build_frontier  merges the world * ncta partials per node
 *                              (log-sum-exp and the k best, exactly as the
 *                              one-GPU build merges its per-CTA partials)
 *                              and runs the best-first frontier.
 * after dt_sharded_build_begin, which clears the status word and seeds wave 0
 * with the roots.  Every rank takes the same decisions from the same merged
 * values, so the trees are identical; each equals dt_tree_build's on the
 * same inputs up to the fp32 order of the log-sum-exp (keys within 1e-5).
 *   cfg.ncta   partials per rank: dt_shard_ncta(V, world) (one per SM, at
 *              most the smallest shard's tile count), the same on all ranks
 *   limits     those of dt_tree_build with r <= 512 (Nmax <= 32) or r <= 256
 *              (Nmax <= 64), so that the GEMM gathers its node rows in shared
 *              memory; world <= 64
 *   ws         >= dt_sharded_workspace_bytes(&cfg), one per rank
 * Device-side checks report through the status word of ws. */
typedef struct {
  int batch, Bk, V, r, k, Nmax; /* as dt_tree_build (V: the whole vocabulary) */
  int world;                    /* ranks sharing the vocabulary */
  int ncta;                     /* partials per rank per node row */
} dt_shard_cfg;

void dt_shard_range(int V, int world, int rank, int* v_base, int* v_len);
int dt_shard_ncta(int V, int world);
size_t dt_sharded_workspace_bytes(const dt_shard_cfg* cfg);
size_t dt_sharded_partials_bytes(const dt_shard_cfg* cfg);

dt_status dt_sharded_build_begin(const dt_shard_cfg* cfg, const int32_t* d_root_token,
                                 const int32_t* d_n_budget, const int32_t* d_k_req,
                                 const float* d_lambda, const dt_tree* out, void* ws,
                                 size_t ws_bytes, dt_stream stream);

dt_status dt_sharded_build_gemm(const dt_shard_cfg* cfg, int wave, int rank,
                                const void* d_block_logits, dt_dtype ldt,
                                const uint16_t* d_markov_a,
                                const uint16_t* d_markov_b_shard, void* ws,
                                size_t ws_bytes, void* d_partials, dt_stream stream);

dt_status dt_sharded_build_frontier(const dt_shard_cfg* cfg, int wave, const void* d_gathered,
                                    const float* d_calib, const int32_t* d_n_budget,
                                    const int32_t* d_k_req, const float* d_lambda,
                                    const dt_tree* out, void* ws, size_t ws_bytes,
                                    dt_stream stream);

/* ---------------------------------------------------------- load policy --
 * Load-adaptive tree size (TreeSpark article, "core idea": the load-adaptive
 * serving policy sizes the trees with the same calibrated path survival that
 * drives expansion and stopping; "measured gains": under rising load the
 * trees shrink back toward the chain).  Applied to built trees before
 * verification, it cuts them so that the batch fits a round's verification
 * capacity:
 *   - a verified node of request b costs w_b = 1 + floor(P_b / prefix_unit)
 *     units, P_b = d_prefix_len[b] (NULL or prefix_unit == 0: w_b = 1);
 *   - the batch's nodes are ordered by (fp32 key desc, request asc, pop index
 *     asc) and the longest prefix of that order whose total cost is
 *     <= capacity is kept.
 * Keys are non-increasing along a tree's pop order, so request b keeps its
 * first n'_b nodes, an ancestor-closed subtree: d_n_nodes[b] is overwritten
 * with n'_b (also written to d_n_keep[b] unless NULL); every other tree array
 * stays valid as it is.  With all nodes fitting nothing changes; capacity 0
 * leaves every tree empty (the round emits the bonus token only).
 *   tree      the dt_tree of dt_tree_build (d_keys and d_n_nodes are used)
 *   limits    1 <= batch <= 1024, 1 <= Nmax <= 64, capacity >= 0,
 *             prefix_unit >= 0
 *   ws        >= dt_tree_load_budget_workspace_bytes() bytes (status word)
 * A node count outside [0, Nmax] or a negative prefix length sets DT_EDEVICE
 * in the status word. */
size_t dt_tree_load_budget_workspace_bytes(void);

dt_status dt_tree_load_budget(const dt_tree* tree, int batch, int Nmax,
                              const int32_t* d_prefix_len, int64_t capacity,
                              int prefix_unit, int32_t* d_n_keep, void* ws,
                              size_t ws_bytes, dt_stream stream);

/* ---------------------------------------------------------- calibration --
 * Fitting the calibration c_d(l) = min(0, alpha_d l + beta_d) that
 * dt_tree_build takes as d_calib (TreeSpark article, "core idea": the
 * drafter's parent-conditioned probability is calibrated into an estimate of
 * the edge's acceptance; the pages give no fitting method).
 *
 * dt_calib_log logs one greedily verified round: for node i of request b
 * whose parent the walk reached (the root, or a node of the accepted path
 * d_acc_nodes[b][0 .. d_n_acc[b]) of dt_tree_accept), it writes
 *   d_depth[b][i] = depth of i,  d_ell[b][i] = key(i) - key(parent) in fp32
 *   (key(root) = 0), d_y[b][i] = 1 iff i is on the accepted path;
 * every other slot of [batch][Nmax] gets depth -1.  With a tree built with
 * the identity calibration, l is the child's drafter log-probability (the
 * order statistic of its rank).  Limits: batch <= 1024, Bk <= 16,
 * Nmax <= 64; ws >= dt_calib_workspace_bytes(1, 1, 1).  Out-of-range counts,
 * path nodes or parents set DT_EDEVICE.
 *
 * dt_calib_fit fits every child depth d = 1..Bk on the n logged samples
 * (entries with depth outside 1..Bk are ignored): it scans the grid
 *   alpha_i = alpha0 + i * dalpha (i < n_alpha),
 *   beta_j = beta0 + j * dbeta (j < n_beta)   (fp64; alpha0, dalpha, dbeta >= 0)
 * and keeps the point with the largest Bernoulli log-likelihood
 *   sum_{y=1} c(l) + sum_{y=0} log(1 - exp(c(l))),  c(l) = min(0, alpha l + beta)
 * computed in fp64 (ties to the smaller i, then the smaller j).  Output:
 * d_calib [Bk][2] fp32 (alpha, beta), directly usable by dt_tree_build; a
 * depth with fewer than max(1, min_samples) samples keeps the identity
 * (1, 0).  d_loglik [Bk] (fp64, NaN where the identity is kept) may be NULL.  Limits: Bk <= 16, n_alpha * n_beta
 * <= 2^20; ws >= dt_calib_workspace_bytes(Bk, n_alpha, n_beta). */
size_t dt_calib_workspace_bytes(int Bk, int n_alpha, int n_beta);

dt_status dt_calib_log(const dt_tree* tree, const int32_t* d_acc_nodes,
                       const int32_t* d_n_acc, int batch, int Bk, int Nmax,
                       int32_t* d_depth, float* d_ell, int8_t* d_y, void* ws,
                       size_t ws_bytes, dt_stream stream);

dt_status dt_calib_fit(const int32_t* d_depth, const float* d_ell, const int8_t* d_y,
                       int n, int Bk, float alpha0, float dalpha, int n_alpha,
                       float beta0, float dbeta, int n_beta, int min_samples,
                       float* d_calib, double* d_loglik, void* ws, size_t ws_bytes,
                       dt_stream stream);

/* Synchronises `stream` and returns the status word that device code of the
 * last call using `ws` wrote (DT_OK, DT_ETIMEOUT or DT_EDEVICE), then clears
 * it.  `ws` is the workspace passed to that call. */
dt_status dt_read_status(void* ws, dt_stream stream, int32_t* host_status);

/* Number of streaming multiprocessors the library sizes its grids for. */
int dt_num_sms(void);

/* Kernel kinds reported by the profiling hook. */
typedef enum {
  DT_K_BUILD_INIT = 0,
  DT_K_MARKOV_GEMM = 1,   /* one wave of the Markov-head GEMM + fused epilogue */
  DT_K_FRONTIER = 2,      /* one wave of the best-first frontier              */
  DT_K_DRAFT_Q = 3,       /* draft distributions of the final tree (T > 0)    */
  DT_K_ACCEPT_PREPASS = 4,
  DT_K_ACCEPT_WALK = 5,
  DT_K_ATTN = 6,
  DT_K_ATTN_COMBINE = 7,
  DT_K_OTHER = 8,
  DT_K_TF_LMHEAD = 9,     /* TreeFlash LM head + top-M epilogue               */
  DT_K_TF_MLP = 10,       /* TreeFlash SwiGLU / down projection               */
  DT_K_PBUILD = 11        /* every wave of a small build in one launch        */
} dt_kernel_kind;

/* How dt_tree_build and dt_tree_build_ex run the waves of the best-first
 * expansion (TreeSpark article, "core idea"; the exact wave schedule is
 * described with dt_tree_build).  The result is the same either way; this is
 * a tuning and diagnostic switch, set per host thread.
 *   DT_BUILD_AUTO        one persistent launch when batch * Nmax <= 64,
 *                        r <= 512 (at temp > 0 also r <= 256 when Nmax > 32)
 *                        and the device can hold one such CTA per SM,
 *                        otherwise one GEMM and one frontier launch per wave
 *                        (the default);
 *   DT_BUILD_WAVES       always one launch pair per wave;
 *   DT_BUILD_PERSISTENT  always the persistent launch: calls that do not fit
 *                        it return DT_EUNSUPPORTED with nothing enqueued.
 * The persistent launch is cooperative (all its CTAs are resident at once):
 * its CTAs meet at a grid barrier after every wave, each wait bounded by two
 * seconds, after which the call records DT_ETIMEOUT (dt_read_status). */
typedef enum { DT_BUILD_AUTO = 0, DT_BUILD_WAVES = 1, DT_BUILD_PERSISTENT = 2 } dt_build_path;
void dt_set_build_path(int path);

/* Test hook for the bounded waits of the persistent build (no counterpart in
 * the pages).  The next persistent build started from the calling host thread
 * runs with every device-side wait bounded by wait_ns instead of two seconds,
 * and its CTA number stall_cta never arrives at the first grid barrier, so
 * every CTA gives up at that barrier: the call's status becomes DT_ETIMEOUT,
 * every CTA lets its copies in flight land, frees its tensor memory and
 * returns, and the tree outputs are left unspecified.  The hook then clears
 * itself.  stall_cta < 0 clears it without a build. */
void dt_set_build_wait_test(int stall_cta, uint64_t wait_ns);

/* Profiling hook (measurement only; off by default).  While set, every kernel
 * the library launches from the calling host thread is bracketed by
 * cudaEventRecord(events[2*i]) and cudaEventRecord(events[2*i+1]) on its
 * stream, with kinds[i] = its dt_kernel_kind and i = (*count)++, as long as
 * i < capacity.  events are cudaEvent_t handles created by the caller; all
 * arrays are host memory owned by the caller.  Pass events = NULL to turn the
 * hook off. */
void dt_set_profile_events(void** events, int32_t* kinds, int capacity, int32_t* count);

#ifdef __cplusplus
}
#endif
#endif /* DTREE_H */
